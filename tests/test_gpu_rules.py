"""GPU parity for the torch scale rule (FP8Q_SCALE_TORCH).

1. Kernels against the CPU oracle under rule 1, bit for bit.
2. Kernels against torch itself on the GPU evaluating the pages' scale
   expressions: a number divided by a CUDA tensor (reciprocal, then
   multiply), a CUDA tensor divided by a number (multiply by the number's
   reciprocal), the fp32 product and torch's fp8 cast.  Codes and scale_inv
   must match byte for byte: this is the parity with real torch outputs that
   the IEEE default does not claim."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import dev, host
from helpers import assert_codes_equal, assert_f32_equal
from test_gpu_per_token import make_input, TORCH_DT

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
FMAXES = {E4M3FN: 448.0, E5M2: 57344.0}
TORCH_FP8 = {E4M3FN: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def to_dev(x, xt):
    return dev(x, TORCH_DT[xt]) if xt != F32 else dev(x)


@pytest.mark.parametrize("xt", [BF16, F32, F16])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
@pytest.mark.parametrize("group", [128, 64])
def test_per_token_torch_rule_vs_oracle(fp8q, orc, xt, fmt, group):
    g = np.random.default_rng(hash((xt, fmt, group, 8)) & 0xFFFF)
    m, n = 37, group * 9
    for kind in ("normal", "wide", "nonfinite"):
        x = make_input(g, (m, n), xt, kind)
        q = torch.empty((m, n), dtype=torch.uint8, device="cuda")
        s = torch.empty((m, n // group), dtype=torch.float32, device="cuda")
        fp8q.fp8q_per_token_group_quant_ex(to_dev(x, xt), q, s, group, fmt, "torch")
        qo, so = orc.per_token_group_quant(x, xt, group, fmt, rule=orc.RULE_TORCH)
        assert_codes_equal(host(q), qo, fmt, name=kind)
        assert_f32_equal(host(s), so, name=kind)


@pytest.mark.parametrize("xt", [BF16, F32])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_scaled_casts_torch_rule_vs_oracle(fp8q, orc, xt, fmt):
    g = np.random.default_rng(hash((xt, fmt, 9)) & 0xFFFF)
    for kind in ("normal", "wide", "nonfinite"):
        x = make_input(g, (21, 2048), xt, kind)
        q = torch.empty((21, 2048), dtype=torch.uint8, device="cuda")
        s = torch.empty((21,), dtype=torch.float32, device="cuda")
        fp8q.fp8q_cast_per_channel_ex(to_dev(x, xt), q, s, fmt, "torch")
        qo, so = orc.cast_per_channel(x, xt, fmt, rule=orc.RULE_TORCH)
        assert_codes_equal(host(q), qo, fmt, name=kind)
        assert_f32_equal(host(s), so, name=kind)
        xf = x.reshape(-1)
        q = torch.empty(xf.size, dtype=torch.uint8, device="cuda")
        s = torch.empty(1, dtype=torch.float32, device="cuda")
        ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
        fp8q.fp8q_cast_per_tensor_ex(to_dev(xf, xt), q, s, ws, fmt, "torch")
        qo, so = orc.cast_per_tensor(xf, xt, fmt, rule=orc.RULE_TORCH)
        assert_codes_equal(host(q), qo, fmt, name=kind)
        assert_f32_equal(host(s), so, name=kind)


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_per_token_torch_rule_matches_torch_cuda(fp8q, fmt):
    """Per-token activations: torch on the GPU computes the amax, FMAX / amax,
    the product, the fp8 cast and amax / FMAX; the library must agree."""
    x = dev(workloads.c2_x(), torch.bfloat16)
    m, n = x.shape
    F = FMAXES[fmt]
    xf = x.float().view(m, n // 128, 128)
    amax = xf.abs().amax(dim=-1).clamp(min=1e-4)
    q_ref = (xf * (F / amax)[..., None]).to(TORCH_FP8[fmt]).view(m, n)
    s_ref = amax / F
    q, s = fp8q.per_token_cast_to_fp8(x, 128, fmt, rule="torch")
    assert_codes_equal(host(q), host(q_ref), fmt)
    assert_f32_equal(host(s), host(s_ref))
    # and the IEEE default differs from torch on this workload
    _, s_ieee = fp8q.per_token_cast_to_fp8(x, 128, fmt)
    assert (host(s_ieee).view(np.uint32) != host(s).view(np.uint32)).mean() > 0.2


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_scaled_casts_torch_rule_match_torch_cuda(fp8q, fmt):
    """ColossalAI casts on the GPU: per-channel (bf16 [8192, 8192] with row
    magnitudes over 1e-3..1e3 and a zero row) and per-tensor (fp32 [64 Mi])."""
    F = FMAXES[fmt]
    x = dev(workloads.c4a_x(), torch.bfloat16)
    xf = x.float()
    amax = xf.abs().amax(dim=-1)
    amax = torch.where(amax > 0, amax, torch.ones_like(amax))
    q_ref = (xf * (F / amax)[:, None]).to(TORCH_FP8[fmt])
    s_ref = amax / F
    q, s = fp8q.cast_to_fp8(x, "e4m3" if fmt == E4M3FN else "e5m2", per_channel_scale=True, rule="torch")
    assert_codes_equal(host(q), host(q_ref), fmt)
    assert_f32_equal(host(s), host(s_ref))
    v = dev(workloads.c4b_v())
    amax = v.abs().max()
    amax = torch.where(amax > 0, amax, torch.ones_like(amax))
    scale = F / amax
    q_ref = (v * scale).to(TORCH_FP8[fmt])
    s_ref = (1.0 / scale).reshape(1)
    q, s = fp8q.cast_to_fp8(v, "e4m3" if fmt == E4M3FN else "e5m2", rule="torch")
    assert_codes_equal(host(q), host(q_ref), fmt)
    assert_f32_equal(host(s), host(s_ref))
