"""Pins for the oracle's method functions (CPU only).

Each operation is pinned by something other than itself:
* hand-worked tensors (tests/golden/*.txt, each citing its page);
* closed-form constants (the clamp bound, zero-amax scales);
* invariants that hold for any input (the amax element lands on +-FMAX, the
  round-trip error bound, unit-scale dequant is exact);
* brute force against a second, naive formulation (tests/naive.py) on small
  random inputs with every dtype, format, granularity and ragged edge.
"""
import numpy as np
import pytest

import naive
import workloads
from helpers import (assert_codes_equal, assert_f32_equal, assert_out_equal,
                     bf16_to_f32, hex_list, load_golden)

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
FMT = {"e4m3fn": E4M3FN, "e5m2": E5M2}


# ---------------------------------------------------------------------------
# hand-worked fixtures
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["per_token_one_group.txt", "per_token_two_groups.txt",
                                  "per_token_nonfinite.txt"])
def test_per_token_golden(orc, name):
    g = load_golden(name)
    m, n, group, fmt = int(g["m"]), int(g["n"]), int(g["group"]), FMT[g["fmt"]]
    x = hex_list(g["x_bf16"], np.uint16).reshape(m, n)
    q, s = orc.per_token_group_quant(x, BF16, group, fmt)
    assert_codes_equal(q.reshape(-1), hex_list(g["q"], np.uint8), fmt)
    assert_f32_equal(s.reshape(-1), hex_list(g["scale_inv_bits"], np.uint32).view(np.float32))


def test_per_tensor_golden(orc):
    g = load_golden("per_tensor_zero.txt")
    x = hex_list(g["x_bits"], np.uint16)
    q, s = orc.cast_per_tensor(x, F16, FMT[g["fmt"]])
    assert_codes_equal(q, hex_list(g["q"], np.uint8), E4M3FN)
    assert_f32_equal(s, hex_list(g["scale_inv_bits"], np.uint32).view(np.float32))
    g = load_golden("per_tensor_single.txt")
    x = hex_list(g["x_f32"], np.uint32).view(np.float32)
    for key, fmt in FMT.items():
        q, s = orc.cast_per_tensor(x, F32, fmt)
        assert_codes_equal(q, hex_list(g["q_" + key], np.uint8), fmt)
        assert_f32_equal(s, hex_list(g[f"scale_inv_{key}_bits"], np.uint32).view(np.float32))


@pytest.mark.parametrize("name,xt", [("per_channel_small.txt", BF16), ("per_channel_e5m2_overflow.txt", F32)])
def test_per_channel_golden(orc, name, xt):
    g = load_golden(name)
    R, C, fmt = int(g["rows"]), int(g["cols"]), FMT[g["fmt"]]
    if xt == BF16:
        x = hex_list(g["x_bf16"], np.uint16).reshape(R, C)
    else:
        x = hex_list(g["x_f32"], np.uint32).view(np.float32).reshape(R, C)
    q, s = orc.cast_per_channel(x, xt, fmt)
    assert_codes_equal(q.reshape(-1), hex_list(g["q"], np.uint8), fmt)
    assert_f32_equal(s, hex_list(g["scale_inv_bits"], np.uint32).view(np.float32))


@pytest.mark.parametrize("name", ["block_dequant_small.txt", "block_dequant_rounding.txt"])
def test_block_dequant_golden(orc, name):
    g = load_golden(name)
    M, N, B, fmt = int(g["M"]), int(g["N"]), int(g["block"]), FMT[g["fmt"]]
    w = hex_list(g["w"], np.uint8).reshape(M, N)
    sh = workloads.scale_shape(M, N, B)
    s = hex_list(g["s_f32"], np.uint32).view(np.float32).reshape(sh)
    y = orc.block_dequant(w, s, fmt, B, BF16)
    assert_out_equal(y.reshape(-1), hex_list(g["y_bf16"], np.uint16), BF16)


def test_cast_from_fp8_golden(orc):
    g = load_golden("cast_from_fp8_small.txt")
    R, C, fmt = int(g["rows"]), int(g["cols"]), FMT[g["fmt"]]
    q = hex_list(g["q"], np.uint8).reshape(R, C)
    s = hex_list(g["scale_inv_f32"], np.uint32).view(np.float32)
    for yt, key, dt in [(F32, "y_f32", np.uint32), (BF16, "y_bf16", np.uint16), (F16, "y_f16", np.uint16)]:
        y = orc.cast_from_fp8(q, s, orc.GRAN_ROW, fmt, 0, yt)
        want = hex_list(g[key], dt)
        assert_out_equal(y.reshape(-1), want.view(np.float32) if yt == F32 else want, yt)


# ---------------------------------------------------------------------------
# closed-form constants
# ---------------------------------------------------------------------------
def test_constants(orc):
    assert np.float32(1e-4).view(np.uint32) == 0x38D1B717
    assert orc.fp8_max(E4M3FN) == 448.0 and orc.fp8_max(E5M2) == 57344.0
    # all-zero per-token group: scale_inv = fl(fl32(1e-4) / 448)
    x = np.zeros((1, 128), np.uint16)
    _, s = orc.per_token_group_quant(x, BF16)
    assert s.view(np.uint32)[0, 0] == 0x346FACAD
    # ... and the scale it implies, 4480000, maps the clamp bound onto 448:
    one = np.zeros((1, 128), np.float32)
    one[0, 0] = np.float32(1e-4)
    q, s = orc.per_token_group_quant(one, F32)
    assert q[0, 0] == 0x7E and s.view(np.uint32)[0, 0] == 0x346FACAD
    # all-zero per-tensor: scale_inv = fl(1/448)
    _, s = orc.cast_per_tensor(np.zeros(5, np.float32), F32, E4M3FN)
    assert s.view(np.uint32)[0] == 0x3B124925


def test_empty_tensors(orc):
    q, s = orc.cast_per_tensor(np.zeros(0, np.float32), F32, E4M3FN)
    assert q.size == 0 and s[0] == 1.0
    q, s = orc.cast_per_channel(np.zeros((0, 4), np.float32), F32, E4M3FN)
    assert q.size == 0 and s[0] == 1.0
    q, s = orc.cast_per_channel(np.zeros((3, 0), np.uint16), BF16, E4M3FN)
    assert (s == 1.0).all()
    q, s = orc.per_token_group_quant(np.zeros((0, 256), np.uint16), BF16)
    assert q.size == 0 and s.size == 0


def test_rejects_bad_arguments(orc):
    with pytest.raises(ValueError):
        orc.per_token_group_quant(np.zeros((2, 130), np.uint16), BF16, 128)
    with pytest.raises(ValueError):
        orc.per_token_group_quant(np.zeros((2, 128), np.uint16), BF16, 128, fmt=7)
    with pytest.raises(ValueError):
        orc.cast_from_fp8(np.zeros((2, 130), np.uint8), np.ones(4, np.float32), orc.GRAN_GROUP, gb=128)


# ---------------------------------------------------------------------------
# invariants on the small per-token workload (bf16 x[128, 1024])
# ---------------------------------------------------------------------------
@pytest.fixture(scope="module")
def c1(orc):
    x = workloads.c1_x()
    q, s = orc.per_token_group_quant(x, BF16, 128, E4M3FN)
    return x, q, s


def test_c1_zero_row(c1):
    x, q, s = c1
    assert (q[3] == 0).all()
    assert (s[3].view(np.uint32) == 0x346FACAD).all()


def test_c1_outlier_row(c1):
    x, q, s = c1
    g = 517 // 128
    xf = bf16_to_f32(x[7])
    sign = 0x80 if xf[517] < 0 else 0
    assert q[7, 517] == (0x7E | sign)
    assert s[7, g] == np.float32(np.abs(xf[517])) / np.float32(448.0)


def test_amax_element_lands_on_fmax(c1):
    """In every group whose amax exceeds the clamp bound, the element(s) with
    |x| == amax encode to +-448 (0x7E / 0xFE), and no code of a finite input
    lies above 448 (no NaN code appears)."""
    x, q, s = c1
    xf = np.abs(bf16_to_f32(x)).reshape(128, 8, 128)
    qq = q.reshape(128, 8, 128)
    amax = xf.max(axis=2)
    live = amax >= np.float32(1e-4)
    is_max = (xf == amax[:, :, None]) & live[:, :, None]
    top = (qq & 0x7F) == 0x7E
    assert top[is_max].all()
    assert live.sum() == 127 * 8
    assert ((qq & 0x7F) <= 0x7E).all()


def test_round_trip_error_bound(orc, c1):
    """|dequant(q) - x| <= scale_inv * (2^-4 |x * scale| + 2^-10) per element
    (half an e4m3 ulp relative, or half the subnormal spacing), plus the bf16
    rounding of the output; checked through the oracle's own dequant."""
    x, q, s = c1
    y = orc.cast_from_fp8(q, s, orc.GRAN_GROUP, E4M3FN, 128, F32)
    xf = bf16_to_f32(x).astype(np.float64)
    sinv = np.repeat(s.astype(np.float64), 128, axis=1)
    err = np.abs(y.astype(np.float64) - xf)
    bound = sinv * (2.0 ** -4 * np.abs(xf / sinv) + 2.0 ** -10) * (1 + 2.0 ** -20)
    assert (err <= bound).all()


def test_unit_scale_block_dequant_is_exact(orc):
    """With every scale 1.0 the dequant is the exact code value: bf16 holds
    every e4m3fn / e5m2 value, so the result must equal torch's fp8 -> bf16."""
    import torch
    for fmt, codes in ((E4M3FN, workloads.finite_e4m3fn_codes()), (E5M2, workloads.finite_e5m2_codes())):
        w = np.resize(codes, (3, 256)).astype(np.uint8)
        s = np.ones(workloads.scale_shape(3, 256), np.float32)
        y = orc.block_dequant(w, s, fmt, 128, BF16)
        tdt = torch.float8_e4m3fn if fmt == E4M3FN else torch.float8_e5m2
        want = torch.from_numpy(w).view(tdt).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert_out_equal(y, want, BF16)


def test_per_tensor_single_nonzero_hits_fmax(orc):
    g = np.random.default_rng(3)
    for fmt in (E4M3FN, E5M2):
        for _ in range(20):
            x = np.zeros(97, np.float32)
            k = int(g.integers(0, 97))
            x[k] = np.float32(g.normal() * 10.0 ** g.uniform(-30, 30))
            q, _ = orc.cast_per_tensor(x, F32, fmt)
            top = 0x7E if fmt == E4M3FN else 0x7B
            assert q[k] == (top | (0x80 if x[k] < 0 else 0))
            assert (np.delete(q, k) == 0).all()


# ---------------------------------------------------------------------------
# brute force against the naive formulation
# ---------------------------------------------------------------------------
def _rand_values(g, shape, kind):
    if kind == "normal":
        v = g.standard_normal(shape)
    elif kind == "wide":      # magnitudes over many binades, incl. fp32-subnormal-scale values
        v = g.standard_normal(shape) * 10.0 ** g.uniform(-40, 38, shape)
    elif kind == "ties":      # values on fp8-grid midpoints after scaling by a power of two
        v = (g.integers(-60, 60, shape) + 0.5) * 2.0 ** g.integers(-12, 4, shape)
    else:                     # sparse with exact zeros and signed zeros
        v = np.where(g.random(shape) < 0.7, 0.0, g.standard_normal(shape))
        v = np.where(g.random(shape) < 0.3, -v, v)
    with np.errstate(over="ignore"):
        return v.astype(np.float32)


def _store(v32, xt):
    if xt == F32:
        return v32
    if xt == BF16:
        return naive.narrow(v32, BF16)
    with np.errstate(over="ignore"):
        return v32.astype(np.float16).view(np.uint16)


KINDS = ["normal", "wide", "ties", "sparse"]


@pytest.mark.parametrize("xt", [BF16, F32, F16])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
@pytest.mark.parametrize("shape,group", [((1, 128), 128), ((2, 256), 128), ((5, 384), 128),
                                         ((3, 64), 32), ((4, 96), 16)])
def test_per_token_vs_naive(orc, xt, fmt, shape, group):
    g = np.random.default_rng(hash((xt, fmt, shape, group)) & 0xFFFF)
    for kind in KINDS:
        x = _store(_rand_values(g, shape, kind), xt)
        q, s = orc.per_token_group_quant(x, xt, group, fmt)
        qn, sn = naive.per_token_group_quant(x, xt, group, fmt)
        assert_codes_equal(q, qn, fmt, name=kind)
        assert_f32_equal(s, sn, name=kind)


@pytest.mark.parametrize("xt", [BF16, F32, F16])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
@pytest.mark.parametrize("shape", [(1, 1), (1, 7), (3, 130), (8, 33)])
def test_per_channel_vs_naive(orc, xt, fmt, shape):
    g = np.random.default_rng(hash((xt, fmt, shape, 1)) & 0xFFFF)
    for kind in KINDS:
        x = _store(_rand_values(g, shape, kind), xt)
        q, s = orc.cast_per_channel(x, xt, fmt)
        qn, sn = naive.cast_per_channel(x, xt, fmt)
        assert_codes_equal(q, qn, fmt, name=kind)
        assert_f32_equal(s[: shape[0]], sn, name=kind)


@pytest.mark.parametrize("xt", [BF16, F32, F16])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
@pytest.mark.parametrize("numel", [1, 2, 127, 1000])
def test_per_tensor_vs_naive(orc, xt, fmt, numel):
    g = np.random.default_rng(hash((xt, fmt, numel, 2)) & 0xFFFF)
    for kind in KINDS:
        x = _store(_rand_values(g, (numel,), kind), xt)
        q, s = orc.cast_per_tensor(x, xt, fmt)
        qn, sn = naive.cast_per_tensor(x, xt, fmt)
        assert_codes_equal(q, qn, fmt, name=kind)
        assert_f32_equal(s, sn, name=kind)


@pytest.mark.parametrize("yt", [BF16, F16, F32])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
@pytest.mark.parametrize("shape,block", [((129, 130), 128), ((256, 384), 128), ((7, 9), 4), ((1, 1), 128)])
def test_block_dequant_vs_naive(orc, yt, fmt, shape, block):
    g = np.random.default_rng(hash((yt, fmt, shape, block)) & 0xFFFF)
    w = g.integers(0, 256, shape).astype(np.uint8)              # all codes, NaN included
    sh = workloads.scale_shape(*shape, block)
    for sk in ("lognormal", "wide"):
        if sk == "lognormal":
            s = workloads.lognormal_scales(g, sh)
        else:
            with np.errstate(over="ignore"):
                s = (g.standard_normal(sh) * 10.0 ** g.uniform(-45, 38, sh)).astype(np.float32)
        y = orc.block_dequant(w, s, fmt, block, yt)
        with np.errstate(over="ignore"):
            yn = naive.block_dequant(w, s, fmt, block, yt)
        assert_out_equal(y, yn, yt, name=sk)


@pytest.mark.parametrize("gran,gb", [(0, 0), (1, 0), (2, 128), (2, 32), (3, 128), (3, 16)])
@pytest.mark.parametrize("yt", [BF16, F16, F32])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_cast_from_fp8_vs_naive(orc, gran, gb, yt, fmt):
    g = np.random.default_rng(hash((gran, gb, yt, fmt)) & 0xFFFF)
    R, C = (37, 256) if gran != 3 else (130, 257)
    q = g.integers(0, 256, (R, C)).astype(np.uint8)
    ns = {0: 1, 1: R, 2: R * (C // max(gb, 1)), 3: int(np.prod(workloads.scale_shape(R, C, max(gb, 1))))}[gran]
    s = workloads.lognormal_scales(g, (ns,), 0.0, 3.0)
    y = orc.cast_from_fp8(q, s, gran, fmt, gb, yt)
    with np.errstate(over="ignore"):
        yn = naive.cast_from_fp8(q, s, gran, fmt, gb, yt)
    assert_out_equal(y, yn, yt)


def test_round_trip_through_group_dequant_matches_naive(orc, c1):
    x, q, s = c1
    y = orc.cast_from_fp8(q, s, orc.GRAN_GROUP, E4M3FN, 128, BF16)
    yn = naive.cast_from_fp8(q, s, 2, E4M3FN, 128, BF16)
    assert_out_equal(y, yn, BF16)


def test_row_ranges_compose(orc):
    """Computing rows in pieces (as the threaded and sampled callers do)
    gives the same bytes as one call."""
    x = workloads.c1_x()
    q1, s1 = orc.per_token_group_quant(x, BF16)
    q2, s2 = orc.per_token_group_quant(x, BF16, threads=5)
    assert (q1 == q2).all() and (s1.view(np.uint32) == s2.view(np.uint32)).all()
