"""GPU parity: block dequant (DeepSeek-V3 weight_dequant), its grouped form and
cast_from_fp8 at every granularity, through the C ABI against the CPU oracle.
Bit-exact on every output element (NaN compares as a class)."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import Guarded, dev, host, offset_input
from helpers import assert_out_equal, hex_list, load_golden

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
YDT = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}


def scales(g, shape, kind):
    if kind == "lognormal":
        return workloads.lognormal_scales(g, shape)
    with np.errstate(over="ignore"):
        return (g.standard_normal(shape) * 10.0 ** g.uniform(-45, 38, shape)).astype(np.float32)


def gpu_block(fp8q, w, s, block, fmt, yt, w_off=0, y_off=0):
    M, N = w.shape
    wd = offset_input(w, w_off) if w_off else dev(w)
    y = Guarded(M * N, YDT[yt], offset=y_off)
    fp8q.fp8q_block_dequant(wd, dev(s), y.t.view(M, N) if M * N else y.t, block, fmt)
    y.check()
    return host(y.t).reshape(M, N)


@pytest.mark.parametrize("yt", [BF16, F16, F32])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
@pytest.mark.parametrize("shape,block", [((129, 130), 128), ((300, 1000), 128), ((257, 999), 128),
                                         ((64, 7168), 128), ((1, 16), 128), ((33, 48), 16),
                                         ((40, 40), 3), ((130, 130), 1000), ((70, 520), 8)])
def test_block_dequant(fp8q, orc, yt, fmt, shape, block):
    g = np.random.default_rng(hash((yt, fmt, shape, block)) & 0xFFFF)
    w = g.integers(0, 256, shape).astype(np.uint8)        # every code, NaN codes included
    for kind in ("lognormal", "wide"):
        s = scales(g, workloads.scale_shape(*shape, block), kind)
        y = gpu_block(fp8q, w, s, block, fmt, yt)
        assert_out_equal(y, orc.block_dequant(w, s, fmt, block, yt), yt, name=kind)


@pytest.mark.parametrize("w_off,y_off", [(1, 0), (8, 2), (0, 2), (4, 8)])
def test_block_dequant_unaligned(fp8q, orc, w_off, y_off):
    g = np.random.default_rng(w_off * 16 + y_off)
    w = g.integers(0, 256, (130, 256)).astype(np.uint8)
    s = scales(g, workloads.scale_shape(130, 256), "lognormal")
    y = gpu_block(fp8q, w, s, 128, E4M3FN, BF16, w_off, y_off)
    assert_out_equal(y, orc.block_dequant(w, s, E4M3FN, 128, BF16), BF16)


@pytest.mark.parametrize("name", ["block_dequant_small.txt", "block_dequant_rounding.txt"])
def test_goldens_on_gpu(fp8q, name):
    gd = load_golden(name)
    M, N, B = int(gd["M"]), int(gd["N"]), int(gd["block"])
    w = hex_list(gd["w"], np.uint8).reshape(M, N)
    s = hex_list(gd["s_f32"], np.uint32).view(np.float32).reshape(workloads.scale_shape(M, N, B))
    y = gpu_block(fp8q, w, s, B, E4M3FN, BF16)
    assert_out_equal(y.reshape(-1), hex_list(gd["y_bf16"], np.uint16), BF16)


def test_unit_scales_all_codes_exact(fp8q):
    """Scale 1.0: the output is each code's exact value (torch's fp8 -> bf16)."""
    for fmt, tdt in ((E4M3FN, torch.float8_e4m3fn), (E5M2, torch.float8_e5m2)):
        w = np.tile(np.arange(256, dtype=np.uint8), (4, 2))
        s = np.ones(workloads.scale_shape(4, 512), np.float32)
        y = gpu_block(fp8q, w, s, 128, fmt, BF16)
        want = torch.from_numpy(w).view(tdt).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert_out_equal(y, want, BF16)


def test_grouped_equals_single_calls(fp8q, orc):
    g = np.random.default_rng(9)
    shapes = [(256, 512), (7, 1000), (129, 130), (0, 64), (300, 48), (1, 1), (128, 7168)]
    ws, ss, ys_grp, ys_one = [], [], [], []
    for M, N in shapes:
        w = g.integers(0, 256, (M, N)).astype(np.uint8)
        s = workloads.lognormal_scales(g, workloads.scale_shape(M, N))
        ws.append(dev(w))
        ss.append(dev(s))
        ys_grp.append(torch.empty((M, N), dtype=torch.bfloat16, device="cuda"))
        ys_one.append(torch.empty((M, N), dtype=torch.bfloat16, device="cuda"))
    fp8q.fp8q_block_dequant_grouped(ws, ss, ys_grp, 128)
    for w, s, y in zip(ws, ss, ys_one):
        fp8q.fp8q_block_dequant(w, s, y, 128)
    for (M, N), w, s, a, b in zip(shapes, ws, ss, ys_grp, ys_one):
        ha, hb = host(a), host(b)
        assert (ha == hb).all()
        if M * N:
            assert_out_equal(ha, orc.block_dequant(host(w), host(s), E4M3FN, 128, BF16), BF16)


def test_grouped_many_problems_split_across_launches(fp8q, orc):
    g = np.random.default_rng(10)
    n = 250
    shapes = [(int(g.integers(1, 70)), int(g.integers(1, 300))) for _ in range(n)]
    ws = [g.integers(0, 256, sh).astype(np.uint8) for sh in shapes]
    ss = [workloads.lognormal_scales(g, workloads.scale_shape(*sh, 32)) for sh in shapes]
    ys = [torch.empty(sh, dtype=torch.float16, device="cuda") for sh in shapes]
    fp8q.fp8q_block_dequant_grouped([dev(w) for w in ws], [dev(s) for s in ss], ys, 32, E5M2)
    for w, s, y in zip(ws, ss, ys):
        assert_out_equal(host(y), orc.block_dequant(w, s, E5M2, 32, F16), F16)


@pytest.mark.parametrize("gran,gb", [(0, 0), (1, 0), (2, 128), (2, 32), (2, 24), (3, 128), (3, 16), (3, 5)])
@pytest.mark.parametrize("yt", [BF16, F16, F32])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_cast_from_fp8(fp8q, orc, gran, gb, yt, fmt):
    g = np.random.default_rng(hash((gran, gb, yt, fmt)) & 0xFFFF)
    R, C = (45, 768) if gran != 3 else (130, 257)
    q = g.integers(0, 256, (R, C)).astype(np.uint8)
    ns = {0: 1, 1: R, 2: R * (C // max(gb, 1)), 3: int(np.prod(workloads.scale_shape(R, C, max(gb, 1))))}[gran]
    s = workloads.lognormal_scales(g, (ns,), 0.0, 3.0)
    y = Guarded(R * C, YDT[yt])
    fp8q.fp8q_cast_from_fp8(dev(q), dev(s), y.t, gran, gb, fmt)
    y.check()
    assert_out_equal(host(y.t).reshape(R, C), orc.cast_from_fp8(q, s, gran, fmt, gb, yt), yt)


def test_cast_from_fp8_golden_on_gpu(fp8q):
    gd = load_golden("cast_from_fp8_small.txt")
    q = hex_list(gd["q"], np.uint8).reshape(2, 2)
    s = hex_list(gd["scale_inv_f32"], np.uint32).view(np.float32)
    for yt, key, dt in [(F32, "y_f32", np.uint32), (BF16, "y_bf16", np.uint16), (F16, "y_f16", np.uint16)]:
        y = torch.empty((2, 2), dtype=YDT[yt], device="cuda")
        fp8q.fp8q_cast_from_fp8(dev(q), dev(s), y, fp8q.GRAN_ROW, 0, E5M2)
        want = hex_list(gd[key], dt)
        assert_out_equal(host(y).reshape(-1), want.view(np.float32) if yt == F32 else want, yt)


def test_dequant_errors(fp8q):
    w = torch.zeros((4, 4), dtype=torch.uint8, device="cuda")
    s = torch.ones((1, 1), dtype=torch.float32, device="cuda")
    y = torch.empty((4, 4), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp8q.Fp8qError) as e:
        fp8q.fp8q_block_dequant(w, s, y, 0)
    assert e.value.status == 4
    with pytest.raises(fp8q.Fp8qError) as e:
        fp8q.fp8q_cast_from_fp8(w, s, y, 7, 0)
    assert e.value.status == 8
    with pytest.raises(fp8q.Fp8qError) as e:
        fp8q.fp8q_cast_from_fp8(w, torch.ones(8, device="cuda"), y, fp8q.GRAN_GROUP, 3)
    assert e.value.status == 4
    with pytest.raises(ValueError):
        fp8q.fp8q_block_dequant(w.cpu(), s, y, 128)          # host tensor refused before the C call
