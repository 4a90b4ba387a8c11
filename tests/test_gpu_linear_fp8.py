"""GPU parity of ColossalAI's _LinearFp8 (colossalai/quantization/fp8.py):
forward and backward through libfp8q, against the composition of the
oracle's per-tensor cast, operand transpose, fp8 product and column sum.

The operand transpose moves bytes and is compared bit for bit.  The column
sum is exact on small integers (bit for bit) and otherwise within its fp32
accumulation bound: at most rows additions of one rounding each, so within
rows * 2^-24 * sum |x| of the exact sum, plus one ulp of the output type.
The products follow the bound of the fp8 product tests."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import THREADS, Guarded, dev, host, offset_input

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
TORCH_T = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}


def tdec(codes, fmt):
    dt = torch.float8_e4m3fn if fmt == E4M3FN else torch.float8_e5m2
    return torch.from_numpy(np.ascontiguousarray(codes)).view(dt).to(torch.float64).numpy()


def ulp(v, yt):
    mant, emin = {F32: (23, -126), F16: (10, -14), BF16: (7, -126)}[yt]
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** emin)))
    return 2.0 ** (e - mant)


def to_f64(bits, yt):
    if yt == F32:
        return bits.astype(np.float64)
    return torch.from_numpy(bits.view(np.int16)).view(TORCH_T[yt]).to(torch.float64).numpy()


def bits_of(v32, yt):
    """fp32 values -> the bit patterns of type yt (torch's RNE cast)."""
    t = torch.from_numpy(np.ascontiguousarray(v32, dtype=np.float32)).to(TORCH_T[yt])
    return t.numpy() if yt == F32 else t.view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------------------
# transpose
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("rows,cols,ld", [(1, 1, 16), (64, 64, 64), (130, 333, 144), (300, 1024, 304),
                                          (7, 5000, 7), (1000, 3, 1008)])
def test_transpose_bit_exact(fp8q, orc, rows, cols, ld):
    g = np.random.default_rng(rows * 7 + cols)
    src = g.integers(0, 256, (rows, cols), dtype=np.uint8)
    out = Guarded(cols * ld, torch.uint8)
    fp8q.fp8q_transpose_fp8(dev(src), out.t.view(cols, ld), ld)
    out.check()
    np.testing.assert_array_equal(host(out.t).reshape(cols, ld), orc.transpose_u8(src, ld))


def test_transpose_unaligned_pointers(fp8q, orc):
    g = np.random.default_rng(5)
    src = g.integers(0, 256, (200, 260), dtype=np.uint8)
    s = offset_input(src, 3)
    out = Guarded(260 * 208, torch.uint8, offset=1)
    fp8q.fp8q_transpose_fp8(s, out.t.view(260, 208), 208)
    out.check()
    np.testing.assert_array_equal(host(out.t).reshape(260, 208), orc.transpose_u8(src, 208))


def test_transpose_full_size_activation(fp8q, orc):
    """The 4096 x 7168 activation codes, as the weight-gradient product reads them."""
    g = np.random.default_rng(6)
    src = g.integers(0, 256, (4096, 7168), dtype=np.uint8)
    dst = torch.empty((7168, 4096), dtype=torch.uint8, device="cuda")
    fp8q.fp8q_transpose_fp8(dev(src), dst, 4096)
    np.testing.assert_array_equal(host(dst), src.T)


# ---------------------------------------------------------------------------
# column sums (bias gradient)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("yt", [F32, F16, BF16])
@pytest.mark.parametrize("rows,cols", [(1, 1), (300, 50), (4096, 7168), (17, 130),
                                       (700, 72),      # 16-byte rows: a full and a partial column block
                                       (65, 8)])       # one row past the 64 subsets
def test_sum_rows_exact_on_integers(fp8q, orc, yt, rows, cols):
    g = np.random.default_rng(rows + cols + yt)
    x = bits_of(g.integers(-64, 65, (rows, cols)).astype(np.float32), yt)
    out = Guarded(cols, TORCH_T[yt])
    fp8q.fp8q_sum_rows(dev(x, TORCH_T[yt]) if yt != F32 else dev(x), out.t)
    out.check()
    want = orc.sum_rows(x, yt)
    np.testing.assert_array_equal(to_f64(host(out.t), yt), to_f64(bits_of(want.astype(np.float32), yt), yt))


@pytest.mark.parametrize("yt", [F32, BF16])
def test_sum_rows_general_within_the_bound(fp8q, orc, yt):
    g = np.random.default_rng(9 + yt)
    rows, cols = 4096, 1000
    x = bits_of((g.standard_normal((rows, cols)) * np.exp(g.normal(0, 2, (1, cols)))).astype(np.float32), yt)
    out = torch.empty((cols,), dtype=TORCH_T[yt], device="cuda")
    xt = dev(x, TORCH_T[yt]) if yt != F32 else dev(x)
    fp8q.fp8q_sum_rows(xt, out)
    first = host(out).copy()
    fp8q.fp8q_sum_rows(xt, out)
    np.testing.assert_array_equal(host(out), first)              # a fixed summation order
    exact = orc.sum_rows(x, yt)
    mag = np.abs(to_f64(x, yt)).sum(0)
    err = np.abs(to_f64(first, yt) - exact)
    assert np.all(err <= rows * 2.0 ** -24 * mag + ulp(exact, yt))


@pytest.mark.parametrize("yt", [F32, BF16])
def test_sum_rows_unaligned_base_takes_the_element_path(fp8q, orc, yt):
    # the same rows one element into a buffer: 16-byte loads are not allowed,
    # the element kernel keeps the same summation order
    g = np.random.default_rng(31 + yt)
    rows, cols = 513, 96
    x = bits_of((g.standard_normal((rows, cols)) * 3).astype(np.float32), yt)
    flat = np.concatenate([np.zeros(1, x.dtype), x.reshape(-1)])
    buf = dev(flat, TORCH_T[yt]) if yt != F32 else dev(flat)
    xa = (dev(x, TORCH_T[yt]) if yt != F32 else dev(x))
    xu = buf[1:].view(rows, cols)
    assert xu.data_ptr() % 16 != 0 and xa.data_ptr() % 16 == 0
    a = torch.empty((cols,), dtype=TORCH_T[yt], device="cuda")
    u = torch.empty((cols,), dtype=TORCH_T[yt], device="cuda")
    fp8q.fp8q_sum_rows(xa, a)
    fp8q.fp8q_sum_rows(xu, u)
    np.testing.assert_array_equal(host(u), host(a))
    exact = orc.sum_rows(x, yt)
    mag = np.abs(to_f64(x, yt)).sum(0)
    assert np.all(np.abs(to_f64(host(a), yt) - exact) <= rows * 2.0 ** -24 * mag + ulp(exact, yt))


def test_sum_rows_zero_rows_writes_zeros(fp8q):
    out = torch.full((5,), 7.0, dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_sum_rows(torch.empty((0, 5), dtype=torch.bfloat16, device="cuda"), out)
    assert (out.float().cpu() == 0).all()


# ---------------------------------------------------------------------------
# _LinearFp8 forward and backward
# ---------------------------------------------------------------------------
def check_bound(got, exact, mag, K, yt):
    rel = (-(-K // 32) + 1) * 2.0 ** -23
    err = np.abs(got - exact)
    bad = ~(err <= rel * mag + ulp(exact, yt))
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outside the bound"


@pytest.mark.parametrize("T,K,N,bias", [(300, 1024, 384, True), (256, 512, 128, False), (37, 256, 64, True)])
def test_linear_fp8_forward_and_backward(fp8q, orc, T, K, N, bias):
    g = np.random.default_rng(T + K + N)
    x = workloads.to_bf16_bits(g.standard_normal((T, K), dtype=np.float32))
    w = workloads.to_bf16_bits((g.standard_normal((N, K)) * 0.05).astype(np.float32))
    go = workloads.to_bf16_bits((g.standard_normal((T, N)) * 1e-3).astype(np.float32))
    b = workloads.to_bf16_bits(g.standard_normal(N).astype(np.float32)) if bias else None

    xt = dev(x, torch.bfloat16).requires_grad_(True)
    wt = dev(w, torch.bfloat16).requires_grad_(True)
    bt = dev(b, torch.bfloat16).requires_grad_(True) if bias else None
    y = fp8q.linear_fp8(xt, wt, bt)
    y.backward(dev(go, torch.bfloat16))

    # the oracle's composition of the page's steps
    qx, sx = orc.cast_per_tensor(x, orc.BF16, E4M3FN)
    qw, sw = orc.cast_per_tensor(w, orc.BF16, E4M3FN)
    qg, sg = orc.cast_per_tensor(go, orc.BF16, E5M2)
    qx, qw, qg = qx.reshape(T, K), qw.reshape(N, K), qg.reshape(T, N)
    sx, sw, sg = float(sx[0]), float(sw[0]), float(sg[0])
    bias64 = to_f64(b, BF16) if bias else None
    fwd = orc.scaled_mm(qx, E4M3FN, qw, E4M3FN, sx, sw, bias=bias64)
    mag = (np.abs(tdec(qx, E4M3FN)) @ np.abs(tdec(qw, E4M3FN)).T) * float(np.float32(sx) * np.float32(sw))
    check_bound(to_f64(host(y.detach()), BF16), fwd, mag + (np.abs(bias64) if bias else 0), K, BF16)

    wT = orc.transpose_u8(qw)                                    # [K, N]
    dx = orc.scaled_mm(qg, E5M2, wT, E4M3FN, sg, sw)
    mag = (np.abs(tdec(qg, E5M2)) @ np.abs(tdec(wT, E4M3FN)).T) * float(np.float32(sg) * np.float32(sw))
    check_bound(to_f64(host(xt.grad), BF16), dx, mag, N, BF16)

    Tp = -(-T // 16) * 16
    gT, xT = orc.transpose_u8(qg, Tp), orc.transpose_u8(qx, Tp)  # [N, Tp], [K, Tp]
    dw = orc.scaled_mm(gT, E5M2, xT, E4M3FN, sg, sx)
    mag = (np.abs(tdec(gT, E5M2)) @ np.abs(tdec(xT, E4M3FN)).T) * float(np.float32(sg) * np.float32(sx))
    check_bound(to_f64(host(wt.grad), BF16), dw, mag, Tp, BF16)

    if bias:
        db = orc.sum_rows(go, orc.BF16)
        mag = np.abs(to_f64(go, BF16)).sum(0)
        err = np.abs(to_f64(host(bt.grad), BF16) - db)
        assert np.all(err <= T * 2.0 ** -24 * mag + ulp(db, BF16))
