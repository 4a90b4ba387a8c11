"""GPU parity: ColossalAI-style cast_to_fp8, per-channel and per-tensor, through
the C ABI against the CPU oracle (bit-exact codes and scales)."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import Guarded, dev, host, offset_input
from helpers import assert_codes_equal, assert_f32_equal, hex_list, load_golden
from test_gpu_per_token import make_input, TORCH_DT

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2


def to_dev(x, xt, off=0):
    if off:
        return offset_input(x, off, TORCH_DT[xt])
    return dev(x, TORCH_DT[xt]) if xt != F32 else dev(x)


def gpu_channel(fp8q, xd, rows, cols, fmt, q_off=0):
    q = Guarded(rows * cols, torch.uint8, offset=q_off)
    s = Guarded(max(rows, 1), torch.float32)
    fp8q.fp8q_cast_per_channel(xd, q.t, s.t, fmt)
    q.check()
    s.check()
    return host(q.t).reshape(rows, cols), host(s.t)


def gpu_tensor(fp8q, xd, numel, fmt, q_off=0):
    q = Guarded(numel, torch.uint8, offset=q_off)
    s = Guarded(1, torch.float32)
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    fp8q.fp8q_cast_per_tensor(xd, q.t, s.t, ws, fmt)
    q.check()
    s.check()
    return host(q.t), host(s.t)


# ---------------------------------------------------------------------------
# per-channel
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("cols", [8, 128, 2048, 4096, 8192, 16384, 20000, 1001, 3])
@pytest.mark.parametrize("xt", [BF16, F32, F16])
def test_per_channel_row_lengths(fp8q, orc, cols, xt):
    g = np.random.default_rng(cols * 3 + xt)
    rows = 6
    for kind in ("normal", "wide", "nonfinite"):
        x = make_input(g, (rows, cols), xt, kind)
        qg, sg = gpu_channel(fp8q, to_dev(x, xt), rows, cols, E4M3FN)
        qo, so = orc.cast_per_channel(x, xt, E4M3FN)
        assert_codes_equal(qg, qo, E4M3FN, name=kind)
        assert_f32_equal(sg, so, name=kind)


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
@pytest.mark.parametrize("kind", ["normal", "wide", "ties", "sparse", "nonfinite"])
def test_per_channel_kinds(fp8q, orc, fmt, kind):
    g = np.random.default_rng(hash((fmt, kind)) & 0xFFFF)
    rows, cols = 33, 1024
    x = make_input(g, (rows, cols), BF16, kind)
    x[5] = 0
    qg, sg = gpu_channel(fp8q, to_dev(x, BF16), rows, cols, fmt)
    qo, so = orc.cast_per_channel(x, BF16, fmt)
    assert_codes_equal(qg, qo, fmt)
    assert_f32_equal(sg, so)


def test_per_channel_nan_and_tiny_rows(fp8q, orc):
    """A NaN row amax is replaced by 1 (so finite elements may overflow to NaN
    or Inf), and a tiny amax makes the scale overflow to Inf."""
    for fmt in (E4M3FN, E5M2):
        x = np.array([[np.nan, 2.0, -3.0, 0.5] * 64,
                      [2.0 ** -130, 0.0, -(2.0 ** -131), 0.0] * 64,
                      [np.inf, 1.0, -1.0, 0.0] * 64], np.float32)
        qg, sg = gpu_channel(fp8q, dev(x), 3, 256, fmt)
        qo, so = orc.cast_per_channel(x, F32, fmt)
        assert_codes_equal(qg, qo, fmt)
        assert_f32_equal(sg, so)


@pytest.mark.parametrize("name,xt", [("per_channel_small.txt", BF16), ("per_channel_e5m2_overflow.txt", F32)])
def test_per_channel_goldens_on_gpu(fp8q, name, xt):
    gd = load_golden(name)
    R, C, fmt = int(gd["rows"]), int(gd["cols"]), {"e4m3fn": 0, "e5m2": 1}[gd["fmt"]]
    if xt == BF16:
        x = hex_list(gd["x_bf16"], np.uint16).reshape(R, C)
    else:
        x = hex_list(gd["x_f32"], np.uint32).view(np.float32).reshape(R, C)
    qg, sg = gpu_channel(fp8q, to_dev(x, xt), R, C, fmt)
    assert_codes_equal(qg.reshape(-1), hex_list(gd["q"], np.uint8), fmt)
    assert_f32_equal(sg, hex_list(gd["scale_inv_bits"], np.uint32).view(np.float32))


@pytest.mark.parametrize("x_off,q_off", [(2, 0), (0, 3), (4, 8)])
def test_per_channel_unaligned(fp8q, orc, x_off, q_off):
    g = np.random.default_rng(x_off + q_off)
    x = make_input(g, (7, 512), BF16, "normal")
    qg, sg = gpu_channel(fp8q, to_dev(x, BF16, x_off), 7, 512, E4M3FN, q_off)
    qo, so = orc.cast_per_channel(x, BF16, E4M3FN)
    assert_codes_equal(qg, qo, E4M3FN)
    assert_f32_equal(sg, so)


def test_per_channel_empty(fp8q):
    for shape in ((0, 16), (3, 0)):
        x = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        q = torch.empty(shape, dtype=torch.uint8, device="cuda")
        s = torch.zeros((max(shape[0], 1),), dtype=torch.float32, device="cuda")
        fp8q.fp8q_cast_per_channel(x, q, s)
        assert (s.cpu() == 1.0).all()


# ---------------------------------------------------------------------------
# per-tensor
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("numel", [1, 7, 8, 1000, 12345, (1 << 20) + 3, 4 << 20])
@pytest.mark.parametrize("xt", [F32, BF16, F16])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_per_tensor_sizes(fp8q, orc, numel, xt, fmt):
    g = np.random.default_rng(numel + 10 * xt + fmt)
    for kind in (("normal", "wide") if numel < (1 << 20) else ("normal",)):
        x = make_input(g, (numel,), xt, kind)
        qg, sg = gpu_tensor(fp8q, to_dev(x, xt), numel, fmt)
        qo, so = orc.cast_per_tensor(x, xt, fmt)
        assert_codes_equal(qg, qo, fmt, name=kind)
        assert_f32_equal(sg, so, name=kind)


@pytest.mark.parametrize("kind", ["ties", "sparse", "nonfinite"])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_per_tensor_kinds(fp8q, orc, kind, fmt):
    g = np.random.default_rng(hash((kind, fmt)) & 0xFFFF)
    x = make_input(g, (50001,), F32, kind)
    qg, sg = gpu_tensor(fp8q, dev(x), x.size, fmt)
    qo, so = orc.cast_per_tensor(x, F32, fmt)
    assert_codes_equal(qg, qo, fmt)
    assert_f32_equal(sg, so)


def test_per_tensor_nan_amax_and_tiny(fp8q, orc):
    for fmt in (E4M3FN, E5M2):
        x = np.array([np.nan, 2.0, -3.0, 0.5, np.inf, 1e30] * 40, np.float32)
        qg, sg = gpu_tensor(fp8q, dev(x), x.size, fmt)
        qo, so = orc.cast_per_tensor(x, F32, fmt)
        assert_codes_equal(qg, qo, fmt)
        assert_f32_equal(sg, so)
        x = np.array([2.0 ** -130, 0.0, -(2.0 ** -131)] * 50, np.float32)
        qg, sg = gpu_tensor(fp8q, dev(x), x.size, fmt)
        qo, so = orc.cast_per_tensor(x, F32, fmt)
        assert_codes_equal(qg, qo, fmt)
        assert_f32_equal(sg, so)


def test_per_tensor_goldens_on_gpu(fp8q):
    gd = load_golden("per_tensor_zero.txt")
    x = hex_list(gd["x_bits"], np.uint16)
    qg, sg = gpu_tensor(fp8q, dev(x, torch.float16), x.size, E4M3FN)
    assert_codes_equal(qg, hex_list(gd["q"], np.uint8), E4M3FN)
    assert_f32_equal(sg, hex_list(gd["scale_inv_bits"], np.uint32).view(np.float32))
    gd = load_golden("per_tensor_single.txt")
    x = hex_list(gd["x_f32"], np.uint32).view(np.float32)
    for key, fmt in (("e4m3fn", E4M3FN), ("e5m2", E5M2)):
        qg, sg = gpu_tensor(fp8q, dev(x), x.size, fmt)
        assert_codes_equal(qg, hex_list(gd["q_" + key], np.uint8), fmt)
        assert_f32_equal(sg, hex_list(gd[f"scale_inv_{key}_bits"], np.uint32).view(np.float32))


@pytest.mark.parametrize("x_off,q_off", [(4, 0), (0, 1), (2, 2), (12, 4)])
def test_per_tensor_unaligned(fp8q, orc, x_off, q_off):
    g = np.random.default_rng(x_off * 5 + q_off)
    xt = F32 if x_off % 4 == 0 else BF16
    x = make_input(g, (30011,), xt, "normal")
    qg, sg = gpu_tensor(fp8q, to_dev(x, xt, x_off), x.size, E4M3FN, q_off)
    qo, so = orc.cast_per_tensor(x, xt, E4M3FN)
    assert_codes_equal(qg, qo, E4M3FN)
    assert_f32_equal(sg, so)


def test_per_tensor_empty_and_workspace_errors(fp8q):
    s = torch.zeros(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    fp8q.fp8q_cast_per_tensor(torch.empty(0, device="cuda"), torch.empty(0, dtype=torch.uint8, device="cuda"),
                              s, ws)
    assert s.item() == 1.0
    x = torch.ones(10, device="cuda")
    q = torch.empty(10, dtype=torch.uint8, device="cuda")
    with pytest.raises(fp8q.Fp8qError) as e:
        fp8q.fp8q_cast_per_tensor(x, q, s, ws[:16])
    assert e.value.status == 6


def test_workspace_reuse_is_stateless(fp8q, orc):
    """Consecutive calls sharing one workspace give each tensor its own scale."""
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    g = np.random.default_rng(1)
    big = (g.standard_normal(1 << 20) * 100).astype(np.float32)
    small = (g.standard_normal(999) * 0.01).astype(np.float32)
    for x in (big, small, big):
        q = torch.empty(x.size, dtype=torch.uint8, device="cuda")
        s = torch.empty(1, dtype=torch.float32, device="cuda")
        fp8q.fp8q_cast_per_tensor(dev(x), q, s, ws, E5M2)
        qo, so = orc.cast_per_tensor(x, F32, E5M2)
        assert_codes_equal(host(q), qo, E5M2)
        assert_f32_equal(host(s), so)


def test_cast_to_from_helpers_round_trip(fp8q, orc):
    x = workloads.c1_x()
    xd = dev(x)
    q, s = fp8q.cast_to_fp8(xd, "e4m3", per_channel_scale=True)
    y = fp8q.cast_from_fp8(q, s, torch.bfloat16, per_channel_scale=True)
    qo, so = orc.cast_per_channel(x, BF16, E4M3FN)
    assert_codes_equal(host(q), qo, E4M3FN)
    yo = orc.cast_from_fp8(qo, so, orc.GRAN_ROW, E4M3FN, 0, BF16)
    assert (host(y) == yo).all()
    q, s = fp8q.cast_to_fp8(xd, "e5m2")
    assert q.shape == xd.shape and s.shape == (1,)
    qo, so = orc.cast_per_tensor(x, BF16, E5M2)
    assert_codes_equal(host(q).reshape(-1), qo, E5M2)
    y = fp8q.cast_from_fp8(q, s, torch.float32)
    want = orc.cast_from_fp8(qo.reshape(x.shape), so, orc.GRAN_TENSOR, E5M2, 0, F32)
    assert (host(y).view(np.uint32) == want.view(np.uint32)).all()
