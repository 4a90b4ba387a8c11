"""Pins for the oracle's pipeline cast (ColossalAI cast_to_fp8_pipeline /
cast_from_fp8_pipeline): hand-worked tensors for both formats and the edge
rules, torch's own CPU operators for the codes, brute force against the
naive formulation, and the round-trip bound."""
import numpy as np
import pytest
import torch

import naive
from helpers import assert_codes_equal, assert_f32_equal, assert_out_equal, hex_list, load_golden
from test_oracle_method import KINDS, _rand_values, _store

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
TORCH_FP8 = {E4M3FN: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


@pytest.mark.parametrize("case", ["a", "b", "c", "d"])
def test_pipeline_golden(orc, case):
    g = load_golden("pipeline_cast.txt")
    x = hex_list(g[case + "_x_f32"], np.uint32).view(np.float32)
    q, s, fmt = orc.cast_pipeline(x, F32)
    assert fmt == int(g[case + "_fmt"])
    assert_codes_equal(q, hex_list(g[case + "_q"], np.uint8), fmt)
    assert_f32_equal(s, hex_list(g[case + "_scale_inv_bits"], np.uint32).view(np.float32))
    if case == "b":
        y = orc.cast_from_pipeline(q, fmt, s, F32)
        assert_f32_equal(y, hex_list(g["b_y_f32"], np.uint32).view(np.float32))


def test_pipeline_format_boundary_and_nonfinite(orc):
    above = np.nextafter(np.float32(448.0), np.float32(1e9))
    assert orc.cast_pipeline(np.array([448.0, 1.0], np.float32), F32)[2] == E4M3FN
    assert orc.cast_pipeline(np.array([above, 1.0], np.float32), F32)[2] == E5M2
    # NaN: amax NaN fails `> 448` (e4m3fn) and `== 0`, so the scale and every code are NaN
    q, s, fmt = orc.cast_pipeline(np.array([np.nan, 1.0, -2.0], np.float32), F32)
    assert fmt == E4M3FN and np.isnan(s[0]) and ((q & 0x7F) == 0x7F).all()
    # Inf: amax Inf > 448 -> e5m2, scale 57344 / Inf = 0, scale_inv = Inf
    q, s, fmt = orc.cast_pipeline(np.array([np.inf, 1.0, -2.0], np.float32), F32)
    assert fmt == E5M2 and np.isposinf(s[0])
    assert q[1] == 0x00 and q[2] == 0x80 and (q[0] & 0x7F) > 0x7C


@pytest.mark.parametrize("rule", [0, 1])
@pytest.mark.parametrize("xt", [BF16, F32, F16])
def test_pipeline_vs_naive(orc, rule, xt):
    g = np.random.default_rng(hash((rule, xt, 21)) & 0xFFFF)
    for kind in KINDS + ["big"]:
        if kind == "big":
            v = (g.standard_normal(999) * 5000).astype(np.float32)
        else:
            v = _rand_values(g, (999,), kind)
        x = _store(v, xt)
        q, s, fmt = orc.cast_pipeline(x, xt, rule)
        qn, sn, fn = naive.cast_pipeline(x, xt, rule)
        assert fmt == fn, kind
        assert_codes_equal(q, qn, fmt, name=kind)
        assert_f32_equal(s, sn, name=kind)
        for yt in (F32, BF16, F16):
            assert_out_equal(orc.cast_from_pipeline(q, fmt, s, yt), naive.cast_from_pipeline(q, fmt, s, yt), yt)


@pytest.mark.parametrize("mag", [1e-3, 30.0, 5000.0])
def test_pipeline_codes_match_torch_cpu_operators(orc, mag):
    """Under the torch rule the codes equal torch computing FMAX / amax with its
    number-by-tensor division, the product and the fp8 cast in the format the
    amax selects; scale_inv equals torch's reciprocal of that scale."""
    g = np.random.default_rng(int(mag))
    v = (g.standard_normal(4096) * mag).astype(np.float32)
    t = torch.from_numpy(v)
    amax = t.abs().max()
    fmt = E5M2 if amax.item() > 448.0 else E4M3FN
    scale = float(torch.finfo(TORCH_FP8[fmt]).max) / amax
    q_ref = (t * scale).to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
    q, s, f = orc.cast_pipeline(v, F32, orc.RULE_TORCH)
    assert f == fmt
    assert_codes_equal(q, q_ref, fmt)
    assert_f32_equal(s, np.array([scale.reciprocal().item()], np.float32))


def test_pipeline_round_trip_bound(orc):
    g = np.random.default_rng(3)
    for mag in (0.01, 100.0, 3000.0):
        v = (g.standard_normal(10000) * mag).astype(np.float32)
        q, s, fmt = orc.cast_pipeline(v, F32)
        y = orc.cast_from_pipeline(q, fmt, s, F32).astype(np.float64)
        rel = 2.0 ** -4 if fmt == E4M3FN else 2.0 ** -3       # half an ulp of 3 / 2 mantissa bits
        sub = 2.0 ** -10 if fmt == E4M3FN else 2.0 ** -17      # half the subnormal spacing
        bound = rel * np.abs(v) + float(s[0]) * sub * 1.0001 + 1e-30
        assert (np.abs(y - v) <= bound * 1.0001).all()
