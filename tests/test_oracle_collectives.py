"""Pins for the oracle's fp8-compressed collectives (CPU only).

ColossalAI colossalai/quantization/fp8.py: all_gather_fp8 /
all_gather_fp8_lagacy (each rank sends [scale | fp8 payload], every rank
dequantises every chunk with its sender's scale), all_to_all_fp8 (a scale
per sent tensor) and all_to_all_single_fp8 (one scale for the sender's whole
tensor, chunks to the ranks, scales all-gathered).

Pinned by: a hand-worked record (tests/golden/record_small.txt); closed-form
round trips on tensors whose scaled values are fp8 codes exactly (the scale
is then a power of two, so a dropped scale, a wrong sign, a transposed rank
index or a wrong chunk shows up as a changed value); the whole-tensor scale
of all_to_all_single_fp8 shown by a chunk that underflows; and the format's
rounding bound on random data.
"""
import numpy as np
import pytest

from helpers import assert_codes_equal, hex_list, load_golden

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
FMAX = {E4M3FN: 448.0, E5M2: 57344.0}
FMAX_CODE = {E4M3FN: 0x7E, E5M2: 0x7B}


def test_record_golden(orc):
    g = load_golden("record_small.txt")
    x = hex_list(g["x_f32_bits"], np.uint32).view(np.float32)
    for fmt, key in ((E4M3FN, "record_e4m3"), (E5M2, "record_e5m2")):
        want = hex_list(g[key], np.uint8)
        got = orc.record(x, F32, fmt)
        assert orc.record_size(3) == 32 == want.size
        np.testing.assert_array_equal(got, want)
        y = orc.record_decode(got, 3, fmt, F32)
        np.testing.assert_array_equal(y.view(np.uint32), hex_list(g["y_f32_bits"], np.uint32))


def test_record_size():
    from oracle import record_size
    assert [record_size(n) for n in (0, 1, 15, 16, 17, 4096)] == [16, 32, 32, 32, 48, 4112]
    assert [record_size(n, 4) for n in (0, 1, 15, 16, 17, 4096)] == [4, 5, 19, 20, 21, 4100]


def test_record_golden_packed4(orc):
    """The page's own record layout (all_gather_fp8_lagacy, SCALE_BYTES = 4): the fp32 scale
    then the codes, no padding; the same hand-worked values as the 16-byte layout."""
    g = load_golden("record_small.txt")
    x = hex_list(g["x_f32_bits"], np.uint32).view(np.float32)
    for fmt, key in ((E4M3FN, "record_e4m3_packed4"), (E5M2, "record_e5m2_packed4")):
        want = hex_list(g[key], np.uint8)
        got = orc.record(x, F32, fmt, header=4)
        assert got.size == 7 == orc.record_size(3, 4)
        np.testing.assert_array_equal(got, want)
        y = orc.record_decode(got, 3, fmt, F32, header=4)
        np.testing.assert_array_equal(y.view(np.uint32), hex_list(g["y_f32_bits"], np.uint32))
        # the two layouts carry the same scale and codes
        r16 = orc.record(x, F32, fmt)
        np.testing.assert_array_equal(r16[:4], got[:4])
        np.testing.assert_array_equal(r16[16:19], got[4:7])


def _exact_tensor(g, n, fmt, k):
    """A fp32 tensor whose elements are fp8 values times 2^k, with |max| =
    FMAX * 2^k: the per-tensor scale is 2^-k exactly and the codes come back."""
    from oracle import fp8_decode
    codes = g.integers(0, 256, n).astype(np.uint8)
    v = fp8_decode(codes, fmt)
    fin = np.isfinite(v)
    codes[~fin] = 0
    codes[g.integers(0, n)] = FMAX_CODE[fmt] | (0x80 if g.integers(0, 2) else 0)
    v = fp8_decode(codes, fmt).astype(np.float32)
    return (v * np.float32(2.0 ** k)).astype(np.float32)


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
@pytest.mark.parametrize("rule", [0, 1])
def test_all_gather_exact_round_trip(orc, fmt, rule):
    g = np.random.default_rng(40 + fmt + 2 * rule)
    xs = [_exact_tensor(g, n, fmt, k) for n, k in ((1000, -7), (33, 5), (4097, 0), (1, 19))]
    out = orc.all_gather_fp8(xs, F32, fmt, rule)
    assert len(out) == len(xs)
    for x, y in zip(xs, out):
        np.testing.assert_array_equal(y.view(np.uint32), x.view(np.uint32))


def test_all_gather_each_output_depends_on_its_rank_only(orc):
    g = np.random.default_rng(3)
    xs = [(g.standard_normal(500) * 10.0 ** e).astype(np.float32) for e in (-3, 0, 2)]
    out = orc.all_gather_fp8(xs, F32, E4M3FN)
    ys = [orc.all_gather_fp8([x], F32, E4M3FN)[0] for x in xs]
    for a, b in zip(out, ys):
        np.testing.assert_array_equal(a, b)
    # permuting the ranks permutes the outputs
    perm = orc.all_gather_fp8(xs[::-1], F32, E4M3FN)
    for a, b in zip(perm, out[::-1]):
        np.testing.assert_array_equal(a, b)
    # every rank's own scale: rank 0's tiny values survive next to rank 2's large ones
    assert np.abs(out[0] - xs[0]).max() <= np.abs(xs[0]).max() / 8


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_all_to_all_transposes(orc, fmt):
    g = np.random.default_rng(70 + fmt)
    W = 3
    inputs = [[_exact_tensor(g, 64, fmt, 3 * j - 2 * i) for i in range(W)] for j in range(W)]
    outputs = orc.all_to_all_fp8(inputs, F32, fmt)
    for i in range(W):
        for j in range(W):
            np.testing.assert_array_equal(outputs[i][j], inputs[j][i])


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_all_to_all_single_chunks_and_shared_scale(orc, fmt):
    g = np.random.default_rng(80 + fmt)
    W, c = 4, 50
    inputs = [_exact_tensor(g, W * c, fmt, j - 1) for j in range(W)]
    outputs = orc.all_to_all_single_fp8(inputs, F32, fmt)
    for i in range(W):
        want = np.concatenate([inputs[j][i * c:(i + 1) * c] for j in range(W)])
        np.testing.assert_array_equal(outputs[i], want)
    # one scale for the sender's whole tensor: chunk 0 holds values that
    # underflow at the scale chunk 1 sets, so rank 0 receives zeros
    tiny = 2.0 ** -12 if fmt == E4M3FN else 2.0 ** -19
    x = np.concatenate([np.full(c, tiny, np.float32), np.full(c, FMAX[fmt], np.float32)])
    out = orc.all_to_all_single_fp8([x, x], F32, fmt)
    np.testing.assert_array_equal(out[0], np.zeros(2 * c, np.float32))
    np.testing.assert_array_equal(out[1], np.full(2 * c, FMAX[fmt], np.float32))


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_round_trip_error_bound(orc, fmt):
    """|y - x| <= half an fp8 ulp at the scaled magnitude, times scale_inv:
    2^-4 |x| for e4m3fn (3 mantissa bits), 2^-3 |x| for e5m2, plus half the
    smallest subnormal (2^-10, 2^-17) times scale_inv, plus fp32 rounding."""
    g = np.random.default_rng(90 + fmt)
    x = (g.standard_normal(20000) * 10.0 ** g.uniform(-6, 6)).astype(np.float32)
    y = orc.all_gather_fp8([x], F32, fmt)[0]
    sinv = float(np.abs(x).max()) / FMAX[fmt]
    rel, sub = (2.0 ** -4, 2.0 ** -10) if fmt == E4M3FN else (2.0 ** -3, 2.0 ** -17)
    bound = rel * np.abs(x.astype(np.float64)) + sub * sinv + 2.0 ** -22 * np.abs(x.astype(np.float64))
    assert (np.abs(y.astype(np.float64) - x) <= bound).all()


def test_record_bf16_payload_matches_per_tensor_cast(orc):
    """The payload of a record is the per-tensor cast's codes; the padding is zero."""
    import workloads
    g = np.random.default_rng(5)
    x = workloads.to_bf16_bits((g.standard_normal(37) * 3).astype(np.float32))
    r = orc.record(x, BF16, E5M2)
    q, s = orc.cast_per_tensor(x, BF16, E5M2)
    assert_codes_equal(r[16:16 + 37], q, E5M2)
    assert r[:4].tobytes() == s.astype("<f4").tobytes()
    assert not r[4:16].any() and not r[16 + 37:].any() and r.size == 64
