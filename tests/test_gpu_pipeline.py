"""GPU parity: the pipeline cast (ColossalAI cast_to_fp8_pipeline /
cast_from_fp8_pipeline) through the C ABI, against the CPU oracle under both
scale rules and against torch on CUDA under the torch rule."""
import numpy as np
import pytest
import torch

from gpu_util import Guarded, dev, host, offset_input
from helpers import assert_codes_equal, assert_f32_equal, assert_out_equal, hex_list, load_golden
from test_gpu_per_token import make_input, TORCH_DT

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
YDT = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}
TORCH_FP8 = {E4M3FN: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def to_dev(x, xt, off=0):
    if off:
        return offset_input(x, off, TORCH_DT[xt])
    return dev(x, TORCH_DT[xt]) if xt != F32 else dev(x)


def gpu_pipeline(fp8q, xd, numel, rule, q_off=0):
    q = Guarded(numel, torch.uint8, offset=q_off)
    s = Guarded(1, torch.float32)
    tag = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    fp8q.fp8q_cast_pipeline(xd, q.t, s.t, tag, ws, rule)
    q.check()
    s.check()
    return host(q.t), host(s.t), int(tag.item()), (q.t, s.t, tag)


def make(g, numel, xt, kind):
    if kind == "big":          # amax above 448: the e5m2 branch
        v = (g.standard_normal(numel) * 3000).astype(np.float32)
        if xt == BF16:
            from workloads import to_bf16_bits
            return to_bf16_bits(v)
        if xt == F16:
            return np.clip(v, -60000, 60000).astype(np.float16).view(np.uint16)
        return v
    if kind == "zero":
        return np.zeros(numel, np.float32 if xt == F32 else np.uint16)
    return make_input(g, (numel,), xt, kind)


@pytest.mark.parametrize("rule", [0, 1])
@pytest.mark.parametrize("xt", [BF16, F32, F16])
@pytest.mark.parametrize("numel", [1, 77, 4096, 1_000_003])
def test_pipeline_vs_oracle(fp8q, orc, rule, xt, numel):
    g = np.random.default_rng(hash((rule, xt, numel)) & 0xFFFF)
    for kind in ("normal", "big", "wide", "nonfinite", "zero"):
        x = make(g, numel, xt, kind)
        qg, sg, fg, (qd, sd, tag) = gpu_pipeline(fp8q, to_dev(x, xt), numel, rule)
        qo, so, fo = orc.cast_pipeline(x, xt, rule)
        assert fg == fo, kind
        assert_codes_equal(qg, qo, fo, name=kind)
        assert_f32_equal(sg, so, name=kind)
        for yt in (BF16, F32, F16):
            y = Guarded(numel, YDT[yt])
            fp8q.fp8q_cast_from_pipeline(qd, sd, tag, y.t)
            y.check()
            assert_out_equal(host(y.t), orc.cast_from_pipeline(qo, fo, so, yt), yt, name=f"{kind} decode")


@pytest.mark.parametrize("x_off,q_off", [(2, 0), (0, 1), (4, 3)])
def test_pipeline_unaligned(fp8q, orc, x_off, q_off):
    g = np.random.default_rng(x_off + 7 * q_off)
    x = make(g, 30011, BF16, "big")
    qg, sg, fg, _ = gpu_pipeline(fp8q, to_dev(x, BF16, x_off), x.size, 0, q_off)
    qo, so, fo = orc.cast_pipeline(x, BF16)
    assert fg == fo == E5M2
    assert_codes_equal(qg, qo, fo)
    assert_f32_equal(sg, so)


@pytest.mark.parametrize("case", ["a", "b", "c", "d"])
def test_pipeline_goldens_on_gpu(fp8q, case):
    gd = load_golden("pipeline_cast.txt")
    x = hex_list(gd[case + "_x_f32"], np.uint32).view(np.float32)
    qg, sg, fg, (qd, sd, tag) = gpu_pipeline(fp8q, dev(x), x.size, 0)
    assert fg == int(gd[case + "_fmt"])
    assert_codes_equal(qg, hex_list(gd[case + "_q"], np.uint8), fg)
    assert_f32_equal(sg, hex_list(gd[case + "_scale_inv_bits"], np.uint32).view(np.float32))
    if case == "b":
        y = torch.empty(x.size, dtype=torch.float32, device="cuda")
        fp8q.fp8q_cast_from_pipeline(qd, sd, tag, y)
        assert_f32_equal(host(y), hex_list(gd["b_y_f32"], np.uint32).view(np.float32))


@pytest.mark.parametrize("mag", [0.05, 20.0, 4000.0])
def test_pipeline_torch_rule_matches_torch_cuda(fp8q, mag):
    """torch on the GPU: the amax, the format test, FMAX / amax (number by
    tensor), the product, the fp8 cast and the reciprocal of the scale."""
    g = np.random.default_rng(int(mag * 10))
    v = dev((g.standard_normal(1 << 22) * mag).astype(np.float32))
    amax = v.abs().max()
    fmt = E5M2 if amax.item() > 448.0 else E4M3FN
    scale = float(torch.finfo(TORCH_FP8[fmt]).max) / amax
    q_ref = (v * scale).to(TORCH_FP8[fmt])
    s_ref = scale.reciprocal().reshape(1)
    q, s, tag = fp8q.cast_to_fp8_pipeline(v, rule="torch")
    assert int(tag.item()) == fmt
    assert_codes_equal(host(q), host(q_ref), fmt)
    assert_f32_equal(host(s), host(s_ref))
    y = fp8q.cast_from_fp8_pipeline(q, s, tag, torch.float32)
    assert (torch.abs(y - v) <= torch.abs(v) * 0.13 + s.item() * 2.0 ** -9).all()


def test_pipeline_empty(fp8q):
    x = torch.empty(0, dtype=torch.float32, device="cuda")
    q, s, tag = fp8q.cast_to_fp8_pipeline(x)
    assert s.item() == 1.0 and tag.item() == 0
