"""Pins for the oracle's two scale rules (CPU only).

rule 0 (IEEE): scale = fl(FMAX / amax), scale_inv = fl(amax / FMAX).
rule 1 (torch): the order torch evaluates the pages' `FMAX / amax` (a Python
number divided by a tensor: reciprocal, then multiply) and, on a GPU,
`amax / FMAX` (a multiply by fl(1 / FMAX)).

Pinned by: a hand-worked group where the two rules give different codes and
scales (tests/golden/per_token_scale_rules.txt); torch's own CPU operators,
whose number-by-tensor division is the reciprocal-then-multiply of rule 1
and whose tensor-by-number division is the true division of rule 0; and
brute force against the naive formulation.
"""
import numpy as np
import pytest
import torch

import naive
import workloads
from helpers import assert_codes_equal, assert_f32_equal, bf16_to_f32, hex_list, load_golden
from test_oracle_method import KINDS, _rand_values, _store

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
FMAXES = {E4M3FN: 448.0, E5M2: 57344.0}
TORCH_FP8 = {E4M3FN: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def test_rule_golden(orc):
    g = load_golden("per_token_scale_rules.txt")
    x = hex_list(g["x_bf16"], np.uint16).reshape(1, 128)
    for rule, key in ((orc.RULE_IEEE, "ieee"), (orc.RULE_TORCH, "torch")):
        q, s = orc.per_token_group_quant(x, BF16, 128, E4M3FN, rule=rule)
        assert_codes_equal(q.reshape(-1), hex_list(g["q_" + key], np.uint8), E4M3FN)
        assert_f32_equal(s.reshape(-1), hex_list(g[f"scale_inv_{key}_bits"], np.uint32).view(np.float32))


def _group_amax(xf, group):
    m, n = xf.shape
    a = np.abs(xf.reshape(m, n // group, group)).max(axis=2)
    return np.maximum(a, np.float32(1e-4)).astype(np.float32)


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_torch_rule_codes_match_torch_cpu_operators(orc, fmt):
    """Codes: torch computes FMAX / amax (its number-by-tensor division), the
    fp32 product and the fp8 cast; they must equal the oracle's rule-1 codes.
    Scales: torch's CPU tensor-by-number division is a true division, so
    amax / FMAX must equal the oracle's rule-0 scale_inv."""
    g = np.random.default_rng(91 + fmt)
    m, n = 64, 1024
    v = (g.standard_normal((m, n)) * 10.0 ** g.uniform(-4, 2, (m, 1))).astype(np.float32)
    x = workloads.to_bf16_bits(v)
    xf = bf16_to_f32(x)
    amax = torch.from_numpy(_group_amax(xf, 128))
    F = FMAXES[fmt]
    scale = F / amax                                        # torch: amax.reciprocal() * F
    q_torch = (torch.from_numpy(xf).view(m, n // 128, 128) * scale[..., None]).to(TORCH_FP8[fmt])
    q_torch = q_torch.view(torch.uint8).numpy().reshape(m, n)
    q1, s1 = orc.per_token_group_quant(x, BF16, 128, fmt, rule=orc.RULE_TORCH)
    assert_codes_equal(q1, q_torch, fmt)
    _, s0 = orc.per_token_group_quant(x, BF16, 128, fmt, rule=orc.RULE_IEEE)
    assert_f32_equal(s0, (amax / F).numpy())
    # the two rules really differ on this data
    assert (s0.view(np.uint32) != s1.view(np.uint32)).mean() > 0.2


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_torch_rule_scaled_casts_match_torch_cpu_operators(orc, fmt):
    g = np.random.default_rng(17 + fmt)
    R, C = 48, 300
    v = (g.standard_normal((R, C)) * 10.0 ** g.uniform(-5, 5, (R, 1))).astype(np.float32)
    F = FMAXES[fmt]
    t = torch.from_numpy(v)
    # per-channel: scale per row from torch's number-by-tensor division
    amax = t.abs().amax(dim=1)
    scale = F / torch.where(amax > 0, amax, torch.ones_like(amax))
    q_torch = (t * scale[:, None]).to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
    q1, _ = orc.cast_per_channel(v, F32, fmt, rule=orc.RULE_TORCH)
    assert_codes_equal(q1, q_torch, fmt)
    # per-tensor: also scale_inv = 1 / scale, a number-by-tensor division as well
    amax = t.abs().max()
    scale = F / torch.where(amax > 0, amax, torch.ones_like(amax))
    q_torch = (t.reshape(-1) * scale).to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
    q1, s1 = orc.cast_per_tensor(v, F32, fmt, rule=orc.RULE_TORCH)
    assert_codes_equal(q1, q_torch, fmt)
    assert_f32_equal(s1, np.array([(1.0 / scale).item()], np.float32))


@pytest.mark.parametrize("xt", [BF16, F32, F16])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_torch_rule_vs_naive(orc, xt, fmt):
    g = np.random.default_rng(hash((xt, fmt, 5)) & 0xFFFF)
    for kind in KINDS:
        x = _store(_rand_values(g, (7, 384), kind), xt)
        q, s = orc.per_token_group_quant(x, xt, 128, fmt, rule=orc.RULE_TORCH)
        qn, sn = naive.per_token_group_quant(x, xt, 128, fmt, rule=1)
        assert_codes_equal(q, qn, fmt, name=kind)
        assert_f32_equal(s, sn, name=kind)
        q, s = orc.cast_per_channel(x, xt, fmt, rule=orc.RULE_TORCH)
        qn, sn = naive.cast_per_channel(x, xt, fmt, rule=1)
        assert_codes_equal(q, qn, fmt, name=kind)
        assert_f32_equal(s[:7], sn, name=kind)
        q, s = orc.cast_per_tensor(x, xt, fmt, rule=orc.RULE_TORCH)
        qn, sn = naive.cast_per_tensor(x, xt, fmt, rule=1)
        assert_codes_equal(q, qn, fmt, name=kind)
        assert_f32_equal(s, sn, name=kind)


def test_bad_rule_rejected(orc):
    with pytest.raises(ValueError):
        orc.per_token_group_quant(np.zeros((1, 128), np.uint16), BF16, rule=2)
