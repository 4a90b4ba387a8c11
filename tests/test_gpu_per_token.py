"""GPU parity: per-token group quantisation (DeepEP per_token_cast_to_fp8)
through the C ABI, element by element against the CPU oracle.  Bit-exact on
fp8 codes and fp32 scales (NaN compares as a class)."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import Guarded, dev, host, offset_input
from helpers import assert_codes_equal, assert_f32_equal, hex_list, load_golden

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
TORCH_DT = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}


def make_input(g, shape, xt, kind):
    if kind == "normal":
        v = g.standard_normal(shape)
    elif kind == "wide":
        v = g.standard_normal(shape) * 10.0 ** g.uniform(-42, 38, shape)
    elif kind == "ties":
        v = (g.integers(-60, 60, shape) + 0.5) * 2.0 ** g.integers(-12, 4, shape)
    elif kind == "sparse":
        v = np.where(g.random(shape) < 0.7, 0.0, g.standard_normal(shape))
        v = np.where(g.random(shape) < 0.3, -v, v)
    elif kind == "nonfinite":
        v = g.standard_normal(shape)
        flat = v.reshape(-1)
        k = max(1, flat.size // 500)
        flat[g.choice(flat.size, k, replace=False)] = np.inf
        flat[g.choice(flat.size, k, replace=False)] = -np.inf
        flat[g.choice(flat.size, k, replace=False)] = np.nan
    else:
        raise ValueError(kind)
    with np.errstate(over="ignore", invalid="ignore"):
        v32 = v.astype(np.float32)
        if xt == F32:
            return v32
        if xt == BF16:
            return workloads.to_bf16_bits(v32)
        return v32.astype(np.float16).view(np.uint16)


def to_dev(x, xt):
    return dev(x, TORCH_DT[xt]) if xt != F32 else dev(x)


def run_gpu(fp8q, xd, m, n, group, fmt, q_off=0):
    q = Guarded(m * n, torch.uint8, offset=q_off)
    s = Guarded(m * (n // group), torch.float32)
    fp8q.fp8q_per_token_group_quant(xd, q.t, s.t, group, fmt)
    q.check()
    s.check()
    return host(q.t).reshape(m, n), host(s.t).reshape(m, n // group)


def check(fp8q, orc, x, xt, m, n, group, fmt, x_off=0, q_off=0):
    xd = offset_input(x, x_off, TORCH_DT[xt]) if x_off else to_dev(x, xt)
    qg, sg = run_gpu(fp8q, xd, m, n, group, fmt, q_off)
    qo, so = orc.per_token_group_quant(x, xt, group, fmt)
    assert_codes_equal(qg, qo, fmt)
    assert_f32_equal(sg, so)


KINDS = ["normal", "wide", "ties", "sparse", "nonfinite"]


@pytest.mark.parametrize("xt", [BF16, F32, F16])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
@pytest.mark.parametrize("kind", KINDS)
def test_group128_ragged_tiles(fp8q, orc, xt, fmt, kind):
    # 37 rows x 5 groups = 185 groups: several CTAs (64 groups each for bf16) and a ragged tail
    g = np.random.default_rng(1000 + 10 * xt + fmt)
    m, n = 37, 640
    check(fp8q, orc, make_input(g, (m, n), xt, kind), xt, m, n, 128, fmt)


@pytest.mark.parametrize("group", [16, 32, 64, 256, 512, 1024])
@pytest.mark.parametrize("xt", [BF16, F32, F16])
def test_other_power_of_two_groups(fp8q, orc, group, xt):
    g = np.random.default_rng(group + xt)
    m, n = 19, group * 7
    for kind in ("normal", "wide", "nonfinite"):
        check(fp8q, orc, make_input(g, (m, n), xt, kind), xt, m, n, group, E4M3FN)


@pytest.mark.parametrize("group", [1, 3, 96, 100, 2048])
def test_generic_groups(fp8q, orc, group):
    g = np.random.default_rng(group)
    m, n = 11, group * 3
    for xt in (BF16, F32):
        for fmt in (E4M3FN, E5M2):
            check(fp8q, orc, make_input(g, (m, n), xt, "normal"), xt, m, n, group, fmt)


@pytest.mark.parametrize("x_off,q_off", [(2, 0), (0, 1), (6, 3), (8, 4)])
def test_unaligned_pointers(fp8q, orc, x_off, q_off):
    g = np.random.default_rng(77)
    m, n = 9, 384
    check(fp8q, orc, make_input(g, (m, n), BF16, "normal"), BF16, m, n, 128, E4M3FN, x_off, q_off)


@pytest.mark.parametrize("m,n", [(1, 128), (2, 256), (129, 128), (1, 7168), (65, 1024)])
def test_shapes(fp8q, orc, m, n):
    g = np.random.default_rng(m * 7 + n)
    check(fp8q, orc, make_input(g, (m, n), BF16, "normal"), BF16, m, n, 128, E4M3FN)


def test_tiny_and_clamped_groups(fp8q, orc):
    """Groups below the 1e-4 clamp, all-zero groups, signed zeros and subnormal bf16."""
    g = np.random.default_rng(5)
    m, n = 8, 512
    v = g.standard_normal((m, n)).astype(np.float32) * np.float32(1e-6)
    v[1] = 0.0
    v[2] = -0.0
    v[3] = np.float32(1e-40) * g.standard_normal(n).astype(np.float32)   # bf16 subnormals
    v[4, ::2] = np.float32(1e-4)
    x = workloads.to_bf16_bits(v)
    check(fp8q, orc, x, BF16, m, n, 128, E4M3FN)
    check(fp8q, orc, x, BF16, m, n, 128, E5M2)


@pytest.mark.parametrize("name", ["per_token_one_group.txt", "per_token_two_groups.txt",
                                  "per_token_nonfinite.txt"])
def test_goldens_on_gpu(fp8q, name):
    gd = load_golden(name)
    m, n, group = int(gd["m"]), int(gd["n"]), int(gd["group"])
    x = hex_list(gd["x_bf16"], np.uint16).reshape(m, n)
    qg, sg = run_gpu(fp8q, dev(x), m, n, group, E4M3FN)
    assert_codes_equal(qg.reshape(-1), hex_list(gd["q"], np.uint8), E4M3FN)
    assert_f32_equal(sg.reshape(-1), hex_list(gd["scale_inv_bits"], np.uint32).view(np.float32))


def test_empty_and_errors(fp8q):
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((0, 256), dtype=torch.uint8, device="cuda")
    s = torch.empty((0, 2), dtype=torch.float32, device="cuda")
    fp8q.fp8q_per_token_group_quant(x, q, s, 128)            # nothing to do, no error
    x = torch.zeros((2, 130), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp8q.Fp8qError) as e:
        fp8q.fp8q_per_token_group_quant(x, torch.empty((2, 130), dtype=torch.uint8, device="cuda"),
                                        torch.empty((2, 2), dtype=torch.float32, device="cuda"), 128)
    assert e.value.status == 4
    with pytest.raises(TypeError):
        fp8q.per_token_cast_to_fp8(torch.zeros((2, 128), dtype=torch.int32, device="cuda"))


def test_allocating_helper_matches_entry_point(fp8q, orc):
    x = workloads.c1_x()
    q, s = fp8q.per_token_cast_to_fp8(dev(x))
    assert q.dtype == torch.float8_e4m3fn and s.shape == (128, 8)
    qo, so = orc.per_token_group_quant(x, BF16)
    assert_codes_equal(host(q), qo, E4M3FN)
    assert_f32_equal(host(s), so)


def test_runs_on_a_side_stream(fp8q, orc):
    x = workloads.c1_x()
    xd = dev(x)
    st = torch.cuda.Stream()
    q = torch.empty((128, 1024), dtype=torch.uint8, device="cuda")
    s = torch.empty((128, 8), dtype=torch.float32, device="cuda")
    with torch.cuda.stream(st):
        fp8q.fp8q_per_token_group_quant(xd, q, s, 128)
    st.synchronize()
    qo, so = orc.per_token_group_quant(x, BF16)
    assert_codes_equal(host(q), qo, E4M3FN)
