"""Pins for the oracle's fp8 / bf16 / fp16 codecs (CPU only).

What fixes the codecs, independently of the oracle's own code:
* the format definitions (torch.finfo: e4m3fn max 448, e5m2 max 57344, code
  counts, subnormal spacing) -- exhaustive checks over all 256 codes;
* torch's own .to(float8_*) / .to(bfloat16) casts and numpy's float16 cast,
  which are exactly the casts the pages call -- compared over every fp32 bit
  pattern in each format's rounding band and a structured sample elsewhere;
* hand-derived boundary values (tests/golden/fp8_boundaries.txt).
"""
import threading

import numpy as np
import pytest
import torch

from helpers import (assert_codes_equal, assert_h16_equal, fp8_is_nan, hex_list,
                     load_golden)

E4M3FN, E5M2 = 0, 1
TORCH_FP8 = {E4M3FN: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}
ALL_CODES = np.arange(256, dtype=np.uint8)


def torch_encode(v: np.ndarray, fmt: int) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(TORCH_FP8[fmt]).view(torch.uint8).numpy()


def torch_decode(c: np.ndarray, fmt: int) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(c, np.uint8)).view(TORCH_FP8[fmt]).float().numpy()


# ---------------------------------------------------------------------------
# the 256-code tables
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_decode_matches_torch_on_all_codes(orc, fmt):
    got = orc.fp8_decode(ALL_CODES, fmt)
    want = torch_decode(ALL_CODES, fmt)
    gn, wn = np.isnan(got), np.isnan(want)
    assert (gn == wn).all()
    assert (got.view(np.uint32)[~gn] == want.view(np.uint32)[~gn]).all()


@pytest.mark.parametrize("fmt,finite,fmax", [(E4M3FN, 254, 448.0), (E5M2, 248, 57344.0)])
def test_code_table_structure(orc, fmt, finite, fmax):
    v = orc.fp8_decode(ALL_CODES, fmt)
    fin = np.isfinite(v)
    # finite code count; NaN set
    nan = np.isnan(v)
    assert fin.sum() == finite  # e5m2: 256 - 6 NaN - 2 Inf
    assert (nan == fp8_is_nan(ALL_CODES, fmt)).all()
    if fmt == E4M3FN:
        assert not np.isinf(v).any()
        assert nan.sum() == 2
    else:
        assert np.isposinf(v[0x7C]) and np.isneginf(v[0xFC]) and nan.sum() == 6
    # monotone over the positive codes, sign bit mirrors
    pos = v[:0x80][np.isfinite(v[:0x80])]
    assert (np.diff(pos) > 0).all()
    assert (v[0x80:][fin[:0x80]] == -v[:0x80][fin[:0x80]]).all()
    assert np.signbit(v[0x80]) and v[0x80] == 0.0 and v[0] == 0.0 and not np.signbit(v[0])
    assert pos.max() == fmax == orc.fp8_max(fmt)
    if fmt == E4M3FN:
        assert v[0x7E] == 448.0 and v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    else:
        assert v[0x7B] == 57344.0 and v[0x04] == 2.0 ** -14 and v[0x01] == 2.0 ** -16 and v[0x03] == 3 * 2.0 ** -16
    # subnormal spacing is uniform and equals the first normal step
    sub = v[0 : (0x08 if fmt == E4M3FN else 0x04) + 2]
    assert np.allclose(np.diff(sub), sub[1]) and np.all(np.diff(sub) == sub[1])


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_encode_decode_round_trip_all_codes(orc, fmt):
    v = orc.fp8_decode(ALL_CODES, fmt)
    back = orc.fp8_encode(v, fmt)
    nonnan = ~np.isnan(v)
    assert (back[nonnan] == ALL_CODES[nonnan]).all()
    assert fp8_is_nan(back[~nonnan], fmt).all()


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_midpoints_round_to_even(orc, fmt):
    """The midpoint of adjacent codes rounds to the even code; one fp32 ulp
    either side rounds to the nearer code."""
    v = orc.fp8_decode(ALL_CODES, fmt).astype(np.float64)
    top = 0x7E if fmt == E4M3FN else 0x7B
    lo_c = np.arange(0, top)
    mids = ((v[lo_c] + v[lo_c + 1]) / 2).astype(np.float32)
    assert (mids.astype(np.float64) == (v[lo_c] + v[lo_c + 1]) / 2).all()  # exact in fp32
    even = np.where(lo_c % 2 == 0, lo_c, lo_c + 1).astype(np.uint8)
    assert (orc.fp8_encode(mids, fmt) == even).all()
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(-np.inf))
    assert (orc.fp8_encode(up, fmt) == (lo_c + 1)).all()
    assert (orc.fp8_encode(dn, fmt) == lo_c).all()
    # negative mirror
    assert (orc.fp8_encode(-mids, fmt) == (even | 0x80)).all()


def test_boundary_values(orc):
    g = load_golden("fp8_boundaries.txt")
    for fmt, key in [(E4M3FN, "e4m3fn"), (E5M2, "e5m2")]:
        x = hex_list(g[key + "_in"], np.uint32).view(np.float32)
        want = hex_list(g[key + "_out"], np.uint8)
        assert_codes_equal(orc.fp8_encode(x, fmt), want, fmt)
        assert_codes_equal(torch_encode(x, fmt), want, fmt)   # the fixture itself agrees with torch


# ---------------------------------------------------------------------------
# library cross-checks over fp32 bit patterns
# ---------------------------------------------------------------------------
def _parallel_chunks(fn, starts, nthreads=8):
    errs = []
    lock = threading.Lock()
    it = iter(starts)

    def work():
        while True:
            with lock:
                s = next(it, None)
            if s is None:
                return
            try:
                fn(s)
            except AssertionError as e:
                errs.append(e)
                return

    ts = [threading.Thread(target=work) for _ in range(nthreads)]
    [t.start() for t in ts]
    [t.join() for t in ts]
    if errs:
        raise errs[0]


BANDS = {
    # biased fp32 exponent fields whose values round to something other than 0 /
    # overflow: from half the smallest subnormal down one binade, to just past
    # the overflow threshold
    E4M3FN: (127 - 11, 127 + 9),
    E5M2: (127 - 18, 127 + 16),
}


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_encode_matches_torch_exhaustive_in_band(orc, fmt):
    """Every fp32 bit pattern (both signs) whose exponent lies in the rounding band."""
    e_lo, e_hi = BANDS[fmt]
    chunk = 1 << 23  # one binade

    def check(e):
        for sign in (0, 1):
            u = (np.arange(chunk, dtype=np.uint32) | np.uint32((sign << 31) | (e << 23)))
            v = u.view(np.float32)
            got = orc.fp8_encode(v, fmt)
            want = torch_encode(v, fmt)
            assert_codes_equal(got, want, fmt, name=f"fmt {fmt} exponent field {e} sign {sign}")

    _parallel_chunks(check, list(range(e_lo, e_hi + 1)))


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_encode_matches_torch_outside_band(orc, fmt):
    """Exponents outside the band: every exponent field x sign x a mantissa sample
    (0, 1, the tie bits, all-ones, random) -- including subnormal fp32, Inf and NaN."""
    g = np.random.default_rng(7)
    mants = np.concatenate([np.array([0, 1, 0x3FFFFF, 0x400000, 0x400001, 0x7FFFFF], np.uint32),
                            g.integers(0, 1 << 23, 4096, dtype=np.uint32)])
    e = np.arange(256, dtype=np.uint32)
    s = np.array([0, 1], np.uint32)
    u = (s[:, None, None] << 31) | (e[None, :, None] << 23) | mants[None, None, :]
    v = u.reshape(-1).view(np.float32)
    assert_codes_equal(orc.fp8_encode(v, fmt), torch_encode(v, fmt), fmt)


def _structured_16bit_sample(low_bits: int):
    """Every upper (32 - low_bits)-bit prefix x low-bit patterns that decide rounding."""
    g = np.random.default_rng(11)
    half = 1 << (low_bits - 1)
    lows = np.concatenate([np.array([0, 1, half - 1, half, half + 1, (1 << low_bits) - 1], np.uint32),
                           g.integers(0, 1 << low_bits, 2, dtype=np.uint32)])
    hi = np.arange(1 << (32 - low_bits), dtype=np.uint32) << np.uint32(low_bits)
    return (hi[:, None] | lows[None, :]).reshape(-1).view(np.float32)


def test_bf16_encode_matches_torch(orc):
    v = _structured_16bit_sample(16)
    got = orc.bf16_encode(v)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert_h16_equal(got, want, "bf16")


def test_f16_encode_matches_numpy(orc):
    v = _structured_16bit_sample(13)
    got = orc.f16_encode(v)
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).view(np.uint16)
    assert_h16_equal(got, want, "f16")


def test_f16_encode_matches_numpy_subnormal_band(orc):
    """fp16 subnormal outputs: the tie moves into the kept bits, so check every
    fp32 pattern whose value lands in or just below the fp16 subnormal range."""
    def check(e):
        u = np.arange(1 << 23, dtype=np.uint32) | np.uint32(e << 23)
        v = u.view(np.float32)
        assert_h16_equal(orc.f16_encode(v), v.astype(np.float16).view(np.uint16), "f16", f"exp {e}")
        assert_h16_equal(orc.f16_encode(-v), (-v).astype(np.float16).view(np.uint16), "f16", f"exp {e}-")

    _parallel_chunks(check, list(range(127 - 26, 127 - 13)))


def test_16bit_decoders_are_exact(orc):
    import ctypes
    L = orc.lib()
    L.orc_bf16_decode.restype = ctypes.c_float
    L.orc_bf16_decode.argtypes = [ctypes.c_uint16]
    L.orc_f16_decode.restype = ctypes.c_float
    L.orc_f16_decode.argtypes = [ctypes.c_uint16]
    allh = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got_bf = np.array([L.orc_bf16_decode(int(h)) for h in allh[::97]], np.float32)
    want_bf = torch.from_numpy(allh[::97].view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    got_h = np.array([L.orc_f16_decode(int(h)) for h in allh[::97]], np.float32)
    want_h = allh[::97].view(np.float16).astype(np.float32)
    for got, want in ((got_bf, want_bf), (got_h, want_h)):
        n = np.isnan(want)
        assert (np.isnan(got) == n).all()
        assert (got.view(np.uint32)[~n] == want.view(np.uint32)[~n]).all()
