"""GPU parity of the two fp8 matrix products (tcgen05 tensor cores) with the
CPU oracle.

ColossalAI _LinearFp8.forward (torch._scaled_mm with per-tensor scales) and
the fine-grained product of DeepEP per-token activations (1 x 128 group
scales) with a DeepSeek-V3 block-scaled weight (128 x 128 block scales).

Two kinds of comparison:

* Exact-grid operands (every value a multiple of 1/8, magnitude <= 4): every
  partial sum of the fp8 products is an fp32 number, so the tensor cores'
  sum is exact whatever its internal order, and the output must equal the
  oracle's single-precision rounding of the product bit for bit.  This pins
  every index, operand, scale, bias and conversion of the data path.
* General operands (all finite codes): the tensor cores round their fp32
  sum.  Model: each 32-deep MMA step adds its products to the fp32
  accumulator with one rounding of at most one fp32 ulp (2^-23 relative),
  and the products inside a step are summed with at most one more.  Over
  ceil(K/32) steps that bounds the sum's error by
  (ceil(K/32) + 1) * 2^-23 * sum |a * b|; the fine-grained product adds one
  rounding of 2^-24 per k-block for its fused multiply-adds.  The output may
  then round to either neighbour in T: one ulp of T on top.
"""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import THREADS, Guarded, dev, host

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
TORCH_T = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}


def tdec(codes, fmt):
    dt = torch.float8_e4m3fn if fmt == E4M3FN else torch.float8_e5m2
    return torch.from_numpy(np.ascontiguousarray(codes)).view(dt).to(torch.float64).numpy()


def grid_codes(g, shape, fmt):
    codes = workloads.finite_e4m3fn_codes() if fmt == E4M3FN else workloads.finite_e5m2_codes()
    v = tdec(codes, fmt)
    keep = codes[(np.abs(v) <= 4) & (v * 8 == np.round(v * 8))]
    return keep[g.integers(0, keep.size, size=shape)].astype(np.uint8)


def finite_codes(g, shape, fmt):
    codes = workloads.finite_e4m3fn_codes() if fmt == E4M3FN else workloads.finite_e5m2_codes()
    c = workloads.uniform_codes(g, shape, codes)
    if fmt == E5M2:
        c[(c & 0x7F) == 0x7C] = 0
    return c


def t_bias(g, N, yt):
    """A bias in the output type (as the page requires) and its fp32 values."""
    b = torch.from_numpy((g.integers(-512, 512, N) / 64.0).astype(np.float32)).to(TORCH_T[yt])
    return b, b.to(torch.float32).numpy()


def run(fp8q, fine, a, fa, b, fb, sa, sb, bias_t, yt, guarded=True):
    M, K = a.shape
    N = b.shape[0]
    out = Guarded(M * N, TORCH_T[yt]) if guarded else None
    o = out.t.view(M, N) if guarded else torch.empty((M, N), dtype=TORCH_T[yt], device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    A, B = dev(a), dev(b)
    bt = None if bias_t is None else bias_t.cuda()
    if fine:
        fp8q.fp8q_scaled_mm_blockwise(A, dev(sa), B, dev(sb), o, bt, fa=fa, fb=fb, status=st)
    else:
        fp8q.fp8q_scaled_mm(A, B, dev(np.array([sa], np.float32)), dev(np.array([sb], np.float32)), o, bt,
                            fa=fa, fb=fb, status=st)
    if guarded:
        out.check()
    assert int(st.item()) == 0, "a bounded wait ran out"
    return o


def scales(g, M, N, K):
    kb = -(-K // 128)
    sa = np.exp(g.normal(-2, 0.5, (M, kb))).astype(np.float32)
    sb = np.exp(g.normal(-2, 0.5, (-(-N // 128), kb))).astype(np.float32)
    return sa, sb


def oracle_rounded(orc, fine, a, fa, b, fb, sa, sb, bias, yt, rows=None):
    if fine:
        return orc.scaled_mm_blockwise_rounded(a, fa, sa, b, fb, sb, bias=bias, yt=yt, rows=rows, threads=THREADS)
    return orc.scaled_mm_rounded(a, fa, b, fb, sa, sb, bias=bias, yt=yt, rows=rows, threads=THREADS)


def bits_equal(got, want, yt):
    if yt == F32:
        return got.view(np.uint32) == want.view(np.uint32)
    return got == want


# ---------------------------------------------------------------------------
# exact-grid operands: bit for bit
# ---------------------------------------------------------------------------
SMALL = [(128, 256, 128),     # one tile, one k-block
         (1, 16, 16),         # the smallest legal product
         (200, 300, 272),     # partial row / column tiles, a partial last k-block, no vector stores
         (130, 512, 384)]     # two row tiles, vector stores
FORMATS = [(E4M3FN, E4M3FN), (E5M2, E4M3FN), (E4M3FN, E5M2), (E5M2, E5M2)]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("fa,fb", FORMATS)
@pytest.mark.parametrize("fine", [False, True], ids=["tensor", "blockwise"])
@pytest.mark.parametrize("yt", [F32, F16, BF16])
def test_exact_grid_bit_exact(fp8q, orc, shape, fa, fb, fine, yt):
    M, N, K = shape
    g = np.random.default_rng(hash((M, N, K, fa, fb, fine, yt)) % 2**32)
    a, b = grid_codes(g, (M, K), fa), grid_codes(g, (N, K), fb)
    sa, sb = scales(g, M, N, K) if fine else (0.0123, 3.5)
    bias_t, bias = t_bias(g, N, yt) if (M + yt) % 2 == 0 else (None, None)
    out = run(fp8q, fine, a, fa, b, fb, sa, sb, bias_t, yt)
    want = oracle_rounded(orc, fine, a, fa, b, fb, sa, sb, bias, yt)
    bad = ~bits_equal(host(out), want, yt)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs differ, first at {np.argwhere(bad)[:4].tolist()}"


@pytest.mark.parametrize("fine", [False, True], ids=["tensor", "blockwise"])
def test_exact_grid_many_tiles(fp8q, orc, fine):
    """192 tiles on at most 148 persistent CTAs (two tiles for some CTAs, both
    TMEM accumulators in use); rows of the first, a middle and the last row tile."""
    M, N, K = 2048, 3000, 512
    g = np.random.default_rng(77 + fine)
    a, b = grid_codes(g, (M, K), E4M3FN), grid_codes(g, (N, K), E4M3FN)
    sa, sb = scales(g, M, N, K) if fine else (0.5, 0.25)
    bias_t, bias = t_bias(g, N, BF16)
    got = host(run(fp8q, fine, a, E4M3FN, b, E4M3FN, sa, sb, bias_t, BF16))
    for r0, r1 in [(0, 40), (1000, 1040), (M - 40, M)]:
        want = oracle_rounded(orc, fine, a, E4M3FN, b, E4M3FN, sa, sb, bias, BF16, rows=(r0, r1))
        np.testing.assert_array_equal(got[r0:r1], want[r0:r1])


# ---------------------------------------------------------------------------
# general operands: error bound
# ---------------------------------------------------------------------------
def ulp(v, yt):
    """The spacing of T at |v| (its normal-range ulp, or the subnormal spacing)."""
    mant, emin = {F32: (23, -126), F16: (10, -14), BF16: (7, -126)}[yt]
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** emin)))
    return 2.0 ** (e - mant)


def check_bound(got, exact, mag, K, yt, fine):
    steps = -(-K // 32) + 1
    rel = steps * 2.0 ** -23 + ((-(-K // 128)) * 2.0 ** -24 if fine else 0.0)
    tol = rel * mag + ulp(exact, yt)
    err = np.abs(got.astype(np.float64) - exact)
    bad = ~(err <= tol)
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} outside the bound; worst err/mag "
                           f"{float((err / np.maximum(mag, 1e-300)).max()):.3g}")


def to_f64(bits, yt):
    if yt == F32:
        return bits.astype(np.float64)
    t = torch.from_numpy(bits.view(np.int16)).view(TORCH_T[yt])
    return t.to(torch.float64).numpy()


@pytest.mark.parametrize("fine", [False, True], ids=["tensor", "blockwise"])
@pytest.mark.parametrize("yt", [F32, BF16])
def test_general_operands_within_the_bound(fp8q, orc, fine, yt):
    M, N, K = 256, 640, 7168
    g = np.random.default_rng(5 + 2 * fine + yt)
    a, b = finite_codes(g, (M, K), E4M3FN), finite_codes(g, (N, K), E4M3FN)
    kb = K // 128
    if fine:
        sa = np.exp(g.normal(-4, 2, (M, kb))).astype(np.float32)
        sb = np.exp(g.normal(-8, 1, (-(-N // 128), kb))).astype(np.float32)
    else:
        sa, sb = 0.0123, 3.5
    got = host(run(fp8q, fine, a, E4M3FN, b, E4M3FN, sa, sb, None, yt))
    rows = (0, 48)
    A, W = np.abs(tdec(a[:48], E4M3FN)), np.abs(tdec(b, E4M3FN))
    if fine:
        exact = orc.scaled_mm_blockwise(a, E4M3FN, sa, b, E4M3FN, sb, rows=rows, threads=THREADS)[:48]
        mag = (A * np.repeat(sa[:48], 128, 1)) @ (W * np.repeat(np.repeat(sb, 128, 0), 128, 1)[:N]).T
    else:
        exact = orc.scaled_mm(a, E4M3FN, b, E4M3FN, sa, sb, rows=rows, threads=THREADS)[:48]
        mag = (A @ W.T) * float(np.float32(sa) * np.float32(sb))
    check_bound(to_f64(got[:48], yt), exact, mag, K, yt, fine)


def test_full_size_sampled_rows(fp8q, orc):
    """The product bench.py times: c2's activations quantised per token
    (4096 x 7168, by the oracle) times the 18432 x 7168 e4m3fn weight with
    128 x 128 block scales, bf16 out, both scale modes; sampled rows."""
    x = workloads.c2_x()
    q, sa = orc.per_token_group_quant(x, orc.BF16, 128, E4M3FN, threads=THREADS)
    w, sb = workloads.mm_w_s()
    M, K = q.shape
    N = w.shape[0]
    A, B = dev(q), dev(w)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rows = [0, 1, 3, 7, 2047, 4095]
    # the bound's magnitudes, in fp32 (they only scale the tolerance)
    Aabs = np.abs(tdec(q[rows], E4M3FN)).astype(np.float32)
    Wabs = np.abs(torch.from_numpy(w).view(torch.float8_e4m3fn).to(torch.float32).numpy())
    # fine-grained
    fp8q.fp8q_scaled_mm_blockwise(A, dev(sa), B, dev(sb), out, status=st)
    got = host(out)
    mag = ((Aabs * np.repeat(sa[rows], 128, 1)) @ (Wabs * np.repeat(np.repeat(sb, 128, 0), 128, 1)).T
           ).astype(np.float64)
    for i, r in enumerate(rows):
        exact = orc.scaled_mm_blockwise(q, E4M3FN, sa, w, E4M3FN, sb, rows=(r, r + 1), threads=THREADS)[r]
        check_bound(to_f64(got[r], BF16), exact, mag[i], K, BF16, True)
    # per-tensor, same codes, the scales of row 0's first group and the weight's first block
    s1, s2 = float(sa[0, 0]), float(sb[0, 0])
    fp8q.fp8q_scaled_mm(A, B, dev(np.array([s1], np.float32)), dev(np.array([s2], np.float32)), out, status=st)
    got = host(out)
    mag = (Aabs @ Wabs.T).astype(np.float64) * float(np.float32(s1) * np.float32(s2))
    for i, r in enumerate(rows):
        exact = orc.scaled_mm(q, E4M3FN, w, E4M3FN, s1, s2, rows=(r, r + 1), threads=THREADS)[r]
        check_bound(to_f64(got[r], BF16), exact, mag[i], K, BF16, False)
    assert int(st.item()) == 0


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------
def test_k_zero_writes_the_bias(fp8q):
    g = np.random.default_rng(2)
    for fine in (False, True):
        bias_t, bias = t_bias(g, 5, BF16)
        out = run(fp8q, fine, np.zeros((3, 0), np.uint8), E4M3FN, np.zeros((5, 0), np.uint8), E4M3FN,
                  np.zeros((3, 0), np.float32) if fine else 1.0, np.zeros((1, 0), np.float32) if fine else 1.0,
                  bias_t, BF16)
        np.testing.assert_array_equal(out.float().cpu().numpy(), np.tile(bias, (3, 1)))
        out = run(fp8q, fine, np.zeros((3, 0), np.uint8), E4M3FN, np.zeros((5, 0), np.uint8), E4M3FN,
                  np.zeros((3, 0), np.float32) if fine else 1.0, np.zeros((1, 0), np.float32) if fine else 1.0,
                  None, F32)
        assert (host(out) == 0).all()


def test_empty_rows_or_columns_write_nothing(fp8q):
    a = dev(np.zeros((0, 32), np.uint8))
    b = dev(np.zeros((8, 32), np.uint8))
    s = dev(np.ones(1, np.float32))
    out = torch.empty((0, 8), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_scaled_mm(a, b, s, s, out)
    g = Guarded(0, torch.bfloat16)
    fp8q.fp8q_scaled_mm(dev(np.zeros((4, 32), np.uint8)), dev(np.zeros((0, 32), np.uint8)), s, s,
                        g.t.view(4, 0))
    g.check()


def test_nan_operand_poisons_its_row_only(fp8q):
    g = np.random.default_rng(3)
    a, b = grid_codes(g, (128, 256), E4M3FN), grid_codes(g, (256, 256), E4M3FN)
    a[5, 7] = 0x7F                       # e4m3fn NaN
    for fine in (False, True):
        sa, sb = scales(g, 128, 256, 256) if fine else (1.0, 1.0)
        o = host(run(fp8q, fine, a, E4M3FN, b, E4M3FN, sa, sb, None, F32))
        assert np.isnan(o[5]).all()
        assert not np.isnan(np.delete(o, 5, 0)).any()


def test_repeat_calls_are_deterministic(fp8q):
    g = np.random.default_rng(4)
    M, N, K = 300, 520, 1024
    a, b = finite_codes(g, (M, K), E4M3FN), finite_codes(g, (N, K), E4M3FN)
    sa, sb = scales(g, M, N, K)
    first = host(run(fp8q, True, a, E4M3FN, b, E4M3FN, sa, sb, None, F32))
    second = host(run(fp8q, True, a, E4M3FN, b, E4M3FN, sa, sb, None, F32))
    np.testing.assert_array_equal(first.view(np.uint32), second.view(np.uint32))


# ---------------------------------------------------------------------------
# the allocating helpers named after the pages' functions
# ---------------------------------------------------------------------------
def test_linear_fp8_matches_the_oracle_composition(fp8q, orc):
    """ColossalAI linear_fp8 forward: per-tensor e4m3 casts of x and w, then
    the scaled product in x's dtype, with a bias."""
    g = np.random.default_rng(6)
    T, Kd, Nd = 300, 1024, 384
    x = workloads.to_bf16_bits(g.standard_normal((T, Kd), dtype=np.float32))
    w = workloads.to_bf16_bits((g.standard_normal((Nd, Kd)) * 0.05).astype(np.float32))
    bias_t, bias = t_bias(g, Nd, BF16)
    y = fp8q.linear_fp8(dev(x, torch.bfloat16).view(3, 100, Kd), dev(w, torch.bfloat16), bias_t.cuda())
    assert y.shape == (3, 100, Nd) and y.dtype == torch.bfloat16
    qx, sx = orc.cast_per_tensor(x, orc.BF16, E4M3FN)
    qw, sw = orc.cast_per_tensor(w, orc.BF16, E4M3FN)
    qx, qw = qx.reshape(T, Kd), qw.reshape(Nd, Kd)
    exact = orc.scaled_mm(qx, E4M3FN, qw, E4M3FN, float(sx[0]), float(sw[0]), bias=bias.astype(np.float64))
    mag = (np.abs(tdec(qx, E4M3FN)) @ np.abs(tdec(qw, E4M3FN)).T) * float(sx[0] * sw[0])
    check_bound(to_f64(host(y).reshape(T, Nd), BF16), exact, mag, Kd, BF16, False)


def test_linear_fp8_blockwise_matches_the_oracle_composition(fp8q, orc):
    g = np.random.default_rng(8)
    T, Kd, Nd = 200, 512, 300
    x = workloads.to_bf16_bits(g.standard_normal((T, Kd), dtype=np.float32))
    w = finite_codes(g, (Nd, Kd), E4M3FN)
    sw = workloads.lognormal_scales(g, workloads.scale_shape(Nd, Kd))
    y = fp8q.linear_fp8_blockwise(dev(x, torch.bfloat16), dev(w).view(torch.float8_e4m3fn), dev(sw))
    qx, sx = orc.per_token_group_quant(x, orc.BF16, 128, E4M3FN)
    exact = orc.scaled_mm_blockwise(qx, E4M3FN, sx, w, E4M3FN, sw)
    mag = (np.abs(tdec(qx, E4M3FN)) * np.repeat(sx, 128, 1)) @ \
        (np.abs(tdec(w, E4M3FN)) * np.repeat(np.repeat(sw, 128, 0), 128, 1)[:Nd]).T
    check_bound(to_f64(host(y), BF16), exact, mag, Kd, BF16, True)


@pytest.mark.parametrize("fine", [False, True], ids=["tensor", "blockwise"])
@pytest.mark.parametrize("M,N,K", [(64, 3000, 512),       # decode-sized rows: 24 tiles 128 columns wide
                                   (1, 18432, 256),       # one token against a full weight row count
                                   (33, 3000, 2560),      # a 48-row A box; 20 k-blocks wrap the 6-stage ring
                                   (64, 1000, 1408),      # a 64-row A box, 11 k-blocks
                                   (100, 40000, 128)])    # enough columns to keep 256-wide tiles
def test_exact_grid_small_m(fp8q, orc, fine, M, N, K):
    g = np.random.default_rng(M + N + K + fine)
    a, b = grid_codes(g, (M, K), E4M3FN), grid_codes(g, (N, K), E5M2)
    sa, sb = scales(g, M, N, K) if fine else (0.25, 0.75)
    bias_t, bias = t_bias(g, N, BF16)
    got = host(run(fp8q, fine, a, E4M3FN, b, E5M2, sa, sb, bias_t, BF16))
    want = oracle_rounded(orc, fine, a, E4M3FN, b, E5M2, sa, sb, bias, BF16)
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------------------
# decode-sized products (at most 128 rows): 128 x 128 tiles, A boxes of M rows
# rounded up to 16, one tile of 128 weight rows per CTA
# ---------------------------------------------------------------------------
DECODE = [(1, 3000, 1024),     # one row, 24 tiles, 8 k-blocks: the 6-stage ring wraps
          (2, 1000, 144),      # a partial second k-block, a partial last tile
          (16, 384, 272),      # a 16-row A box; a partial last k-block
          (17, 2000, 400),     # a 32-row A box
          (32, 640, 16),       # one 16-deep k-block
          (33, 1280, 2000),    # a 48-row A box, 16 k-blocks
          (64, 3000, 1168),
          (65, 1000, 384),     # an 80-row A box: rows in three TMEM lane quarters
          (128, 2048, 640),    # a whole 128-row tile
          (5, 30000, 384)]     # 235 tiles: two for some CTAs


@pytest.mark.parametrize("M,N,K", DECODE, ids=lambda v: str(v))
@pytest.mark.parametrize("fine", [False, True], ids=["tensor", "blockwise"])
def test_exact_grid_decode_sized(fp8q, orc, M, N, K, fine):
    i = DECODE.index((M, N, K))
    fa, fb = FORMATS[i % 4]
    yt = (F32, F16, BF16)[i % 3]
    g = np.random.default_rng(9000 + 7 * i + fine)
    a, b = grid_codes(g, (M, K), fa), grid_codes(g, (N, K), fb)
    sa, sb = scales(g, M, N, K) if fine else (0.375, 1.25)
    bias_t, bias = t_bias(g, N, yt) if i % 2 == 0 else (None, None)
    got = host(run(fp8q, fine, a, fa, b, fb, sa, sb, bias_t, yt))
    want = oracle_rounded(orc, fine, a, fa, b, fb, sa, sb, bias, yt)
    bad = ~bits_equal(got, want, yt)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs differ, first at {np.argwhere(bad)[:4].tolist()}"


@pytest.mark.parametrize("M", [1, 64])
@pytest.mark.parametrize("fine", [False, True], ids=["tensor", "blockwise"])
def test_general_operands_decode_sized(fp8q, orc, M, fine):
    """All finite codes, K = 7168: within the same bound as the large products."""
    N, K = 640, 7168
    g = np.random.default_rng(31 + M + fine)
    a, b = finite_codes(g, (M, K), E4M3FN), finite_codes(g, (N, K), E4M3FN)
    kb = K // 128
    if fine:
        sa = np.exp(g.normal(-4, 2, (M, kb))).astype(np.float32)
        sb = np.exp(g.normal(-8, 1, (-(-N // 128), kb))).astype(np.float32)
    else:
        sa, sb = 0.0123, 3.5
    got = host(run(fp8q, fine, a, E4M3FN, b, E4M3FN, sa, sb, None, BF16))
    A, W = np.abs(tdec(a, E4M3FN)), np.abs(tdec(b, E4M3FN))
    if fine:
        exact = orc.scaled_mm_blockwise(a, E4M3FN, sa, b, E4M3FN, sb, threads=THREADS)
        mag = (A * np.repeat(sa, 128, 1)) @ (W * np.repeat(np.repeat(sb, 128, 0), 128, 1)[:N]).T
    else:
        exact = orc.scaled_mm(a, E4M3FN, b, E4M3FN, sa, sb, threads=THREADS)
        mag = (A @ W.T) * float(np.float32(sa) * np.float32(sb))
    check_bound(to_f64(got, BF16), exact, mag, K, BF16, fine)


# ---------------------------------------------------------------------------
# operand layouts (fp8q_scaled_mm_ex): K-major or MN-major, bit for bit
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("a_mn,b_mn,M,N,K", [
    (0, 1, 128, 256, 128), (0, 1, 200, 304, 272), (0, 1, 64, 3008, 512),
    (1, 0, 208, 300, 272), (1, 0, 128, 256, 384),
    (1, 1, 128, 256, 128), (1, 1, 256, 512, 300), (1, 1, 144, 3008, 37), (1, 1, 32, 16, 1),
    (0, 0, 200, 300, 272),
    (1, 1, 512, 17008, 100), (1, 0, 512, 17008, 64), (0, 1, 512, 17008, 64),    # enough tiles for 256-row tiles
    (0, 0, 256, 17008, 256), (1, 1, 256, 17408, 128)])   # one row of 256 x 256 tiles, one CTA pair per tile
@pytest.mark.parametrize("yt", [F32, BF16])
def test_exact_grid_layouts(fp8q, orc, a_mn, b_mn, M, N, K, yt):
    g = np.random.default_rng(1000 * a_mn + 100 * b_mn + M + N + K + yt)
    a, b = grid_codes(g, (M, K), E4M3FN), grid_codes(g, (N, K), E5M2)   # logical [M, K], [N, K]
    A = dev(np.ascontiguousarray(a.T) if a_mn else a)
    B = dev(np.ascontiguousarray(b.T) if b_mn else b)
    bias_t, bias = t_bias(g, N, yt)
    out = Guarded(M * N, TORCH_T[yt])
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8q.fp8q_scaled_mm_ex(A, B, dev(np.array([0.0123], np.float32)), dev(np.array([3.5], np.float32)),
                           out.t.view(M, N), bias_t.cuda(), a_layout=a_mn, b_layout=b_mn, fa=E4M3FN, fb=E5M2,
                           status=st)
    out.check()
    assert int(st.item()) == 0
    want = orc.scaled_mm_rounded(a, E4M3FN, b, E5M2, 0.0123, 3.5, bias=bias, yt=yt)
    bad = ~bits_equal(host(out.t).reshape(M, N), want, yt)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs differ, first at {np.argwhere(bad)[:4].tolist()}"


def test_scaled_mm_helper_takes_either_layout(fp8q, orc):
    """torch._scaled_mm-style calls: b given as w.t() (ColossalAI) or as a row-major [K, N]
    matrix, a row-major or transposed; the same bits either way."""
    g = np.random.default_rng(21)
    M, N, K = 144, 272, 256
    a, w = grid_codes(g, (M, K), E4M3FN), grid_codes(g, (N, K), E4M3FN)
    sa, sb = dev(np.array([0.5], np.float32)), dev(np.array([0.25], np.float32))
    want = orc.scaled_mm_rounded(a, E4M3FN, w, E4M3FN, 0.5, 0.25, yt=BF16)
    A = dev(a).view(torch.float8_e4m3fn)
    W = dev(w).view(torch.float8_e4m3fn)
    At = dev(np.ascontiguousarray(a.T)).view(torch.float8_e4m3fn).t()      # a, stored transposed
    Wt = dev(np.ascontiguousarray(w.T)).view(torch.float8_e4m3fn)          # b = w^T, row-major [K, N]
    for lhs in (A, At):
        for rhs in (W.t(), Wt):
            np.testing.assert_array_equal(host(fp8q.scaled_mm(lhs, rhs, sa, sb)), want)


@pytest.mark.parametrize("M,N,K", [(257, 300, 272), (300, 512, 128), (520, 768, 384)])
@pytest.mark.parametrize("yt", [F32, BF16])
def test_exact_grid_tall_tiles(fp8q, orc, M, N, K, yt):
    """Per-tensor products of at least 256 rows run 256 x 256 tiles (two MMAs per k step
    sharing the B tile); ragged last row tiles, partial second halves, bias."""
    g = np.random.default_rng(M * 3 + N + K + yt)
    a, b = grid_codes(g, (M, K), E5M2), grid_codes(g, (N, K), E4M3FN)
    bias_t, bias = t_bias(g, N, yt)
    out = run(fp8q, False, a, E5M2, b, E4M3FN, 0.0123, 3.5, bias_t, yt)
    want = oracle_rounded(orc, False, a, E5M2, b, E4M3FN, 0.0123, 3.5, bias, yt)
    bad = ~bits_equal(host(out), want, yt)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs differ, first at {np.argwhere(bad)[:4].tolist()}"


@pytest.mark.parametrize("M,N,K,fa,fb,yt,with_bias", [
    (2000, 4100, 1008, E4M3FN, E4M3FN, BF16, True),     # 8 x 17 tiles: ragged rows in the second CTA, 4 ragged columns, a partial k-block
    (4096, 2304, 256, E4M3FN, E5M2, F32, False),        # 16 x 9 tiles
    (2304, 4352, 384, E5M2, E4M3FN, F16, True)])        # 9 x 17 tiles: an odd row-tile count
def test_exact_grid_cta_pairs(fp8q, orc, M, N, K, fa, fb, yt, with_bias):
    """Per-tensor products with enough 256 x 256 tiles to fill the GPU and both operands K-major
    run on CTA pairs (tcgen05.mma.cta_group::2: each CTA loads 128 rows of A and 128 rows of B
    and holds its 128 rows of the tile in TMEM).  Every output is compared bit for bit."""
    g = np.random.default_rng(M + N + K + yt)
    a, b = grid_codes(g, (M, K), fa), grid_codes(g, (N, K), fb)
    bias_t, bias = t_bias(g, N, yt) if with_bias else (None, None)
    out = run(fp8q, False, a, fa, b, fb, 0.375, 1.75, bias_t, yt)
    want = oracle_rounded(orc, False, a, fa, b, fb, 0.375, 1.75, bias, yt)
    bad = ~bits_equal(host(out), want, yt)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs differ, first at {np.argwhere(bad)[:4].tolist()}"


@pytest.mark.parametrize("M,N,K,yt", [(2000, 4100, 1008, BF16), (2304, 4352, 384, F32)])
def test_exact_grid_fine_wide_products(fp8q, orc, M, N, K, yt):
    """Fine-grained products with enough 256 x 256 tiles to fill the GPU (on CTA pairs where the
    build takes them for these scales): ragged rows and columns, a partial last k-block, per-token
    and block scales, bias; every output bit for bit against the oracle's rounding."""
    g = np.random.default_rng(M * 7 + N + K)
    a, b = grid_codes(g, (M, K), E4M3FN), grid_codes(g, (N, K), E4M3FN)
    sa, sb = scales(g, M, N, K)
    bias_t, bias = t_bias(g, N, yt)
    out = run(fp8q, True, a, E4M3FN, b, E4M3FN, sa, sb, bias_t, yt)
    want = oracle_rounded(orc, True, a, E4M3FN, b, E4M3FN, sa, sb, bias, yt)
    bad = ~bits_equal(host(out), want, yt)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs differ, first at {np.argwhere(bad)[:4].tolist()}"


# ---------------------------------------------------------------------------
# bounded waits: a wait that runs out is reported, and the context stays usable
# ---------------------------------------------------------------------------
def test_bounded_waits_run_out_report_and_return(fp8q, orc):
    """The copies of k-block 2 of each CTA's first tile are left out, so the barrier they would
    complete never does: with a 20 ms limit every wait that depends on it runs out, the kernel sets
    its WAIT_* bits, writes nothing outside d, frees its tensor memory and returns.  The same
    product then runs normally on the same stream, under the same short limit and without it, and
    both equal the oracle bit for bit."""
    import time
    M, N, K = 256, 512, 1024                     # two 128 x 256 tiles, 8 k-blocks (the ring wraps)
    g = np.random.default_rng(404)
    a, b = grid_codes(g, (M, K), E4M3FN), grid_codes(g, (N, K), E4M3FN)
    A, B = dev(a), dev(b)
    sa, sb = dev(np.array([0.5], np.float32)), dev(np.array([0.25], np.float32))
    want = oracle_rounded(orc, False, a, E4M3FN, b, E4M3FN, 0.5, 0.25, None, BF16)

    out = Guarded(M * N, torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    fp8q.fp8q_scaled_mm_wait_test(A, B, sa, sb, out.t.view(M, N), st, 20_000_000, 2)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    out.check()
    bits = int(st.item())
    assert bits & fp8q.WAIT_MMA and bits & fp8q.WAIT_DRAIN, f"status {bits:#x}"
    assert bits & ~0xF == 0, f"status {bits:#x}"
    assert dt < 2.0, f"the stalled kernel took {dt:.2f} s"

    for limit in (20_000_000, 4_000_000_000):
        out2 = Guarded(M * N, torch.bfloat16)
        st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
        fp8q.fp8q_scaled_mm_wait_test(A, B, sa, sb, out2.t.view(M, N), st2, limit, -1)
        out2.check()
        assert int(st2.item()) == 0
        np.testing.assert_array_equal(host(out2.t.view(M, N)), want)
    out3 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_scaled_mm(A, B, sa, sb, out3)
    np.testing.assert_array_equal(host(out3), want)




@pytest.mark.parametrize("M,N,K", [(256, 512, 1024),     # two 128 x 256 tiles, 8 k-blocks
                                   (1, 3000, 1024)],     # decode-sized 128 x 128 tiles
                         ids=["tiles", "decode"])
def test_bounded_waits_run_out_fine_grained(fp8q, orc, M, N, K):
    """The fine-grained product (one accumulator per k-block, folded by the epilogue warps) with
    k-block 2 of each CTA's first tile left out: the MMA's wait runs out, the fold's and the drains'
    waits end, the status bits are reported, and the same product then runs normally."""
    import time
    g = np.random.default_rng(407 + M)
    a, b = grid_codes(g, (M, K), E4M3FN), grid_codes(g, (N, K), E4M3FN)
    sa, sb = scales(g, M, N, K)
    A, B, SA, SB = dev(a), dev(b), dev(sa), dev(sb)
    want = oracle_rounded(orc, True, a, E4M3FN, b, E4M3FN, sa, sb, None, BF16)
    out = Guarded(M * N, torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    fp8q.fp8q_scaled_mm_blockwise_wait_test(A, SA, B, SB, out.t.view(M, N), st, 20_000_000, 2)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    out.check()
    bits = int(st.item())
    assert bits & fp8q.WAIT_MMA and bits & fp8q.WAIT_DRAIN, f"status {bits:#x}"
    assert bits & ~0xF == 0, f"status {bits:#x}"
    assert dt < 2.0, f"the stalled kernel took {dt:.2f} s"
    out2 = Guarded(M * N, torch.bfloat16)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8q.fp8q_scaled_mm_blockwise_wait_test(A, SA, B, SB, out2.t.view(M, N), st2, 20_000_000, -1)
    out2.check()
    assert int(st2.item()) == 0
    np.testing.assert_array_equal(host(out2.t.view(M, N)), want)

def test_bounded_waits_run_out_cta_pairs(fp8q, orc):
    """The same for a product on CTA pairs (256 x 256 tiles, tcgen05.mma.cta_group::2): the
    leader CTA leaves out its half of k-block 2 of its pair's tile, so that stage never completes;
    the leader's MMA wait runs out, the follower's epilogue and both CTAs' drains run out on their
    own limits, both CTAs meet at the final cluster barrier, free TMEM and return."""
    import time
    M, N, K = 512, 8704, 512                     # 68 tiles of 256 x 256: CTA pairs; 4 k-blocks
    g = np.random.default_rng(406)
    a, b = grid_codes(g, (M, K), E4M3FN), grid_codes(g, (N, K), E4M3FN)
    A, B = dev(a), dev(b)
    sa, sb = dev(np.array([0.5], np.float32)), dev(np.array([0.125], np.float32))
    want = oracle_rounded(orc, False, a, E4M3FN, b, E4M3FN, 0.5, 0.125, None, BF16)
    out = Guarded(M * N, torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    fp8q.fp8q_scaled_mm_wait_test(A, B, sa, sb, out.t.view(M, N), st, 20_000_000, 2)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    out.check()
    bits = int(st.item())
    assert bits & fp8q.WAIT_MMA and bits & fp8q.WAIT_DRAIN, f"status {bits:#x}"
    assert bits & ~0xF == 0, f"status {bits:#x}"
    assert dt < 2.0, f"the stalled kernel took {dt:.2f} s"
    out2 = Guarded(M * N, torch.bfloat16)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8q.fp8q_scaled_mm_wait_test(A, B, sa, sb, out2.t.view(M, N), st2, 20_000_000, -1)
    out2.check()
    assert int(st2.item()) == 0
    np.testing.assert_array_equal(host(out2.t.view(M, N)), want)

def test_bounded_waits_run_out_decode_sized(fp8q, orc):
    """The same for a one-row product (128 x 128 tiles, a 16-row A box): k-block 2 of each CTA's
    tile never arrives, every wait that depends on it runs out and is reported, and the same
    product then runs normally on the same stream."""
    import time
    M, N, K = 1, 3000, 1024                      # 24 tiles of 128 weight rows, 8 k-blocks
    g = np.random.default_rng(405)
    a, b = grid_codes(g, (M, K), E4M3FN), grid_codes(g, (N, K), E4M3FN)
    A, B = dev(a), dev(b)
    sa, sb = dev(np.array([0.5], np.float32)), dev(np.array([0.25], np.float32))
    want = oracle_rounded(orc, False, a, E4M3FN, b, E4M3FN, 0.5, 0.25, None, BF16)
    out = Guarded(M * N, torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    fp8q.fp8q_scaled_mm_wait_test(A, B, sa, sb, out.t.view(M, N), st, 20_000_000, 2)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    out.check()
    bits = int(st.item())
    assert bits & fp8q.WAIT_MMA and bits & fp8q.WAIT_DRAIN, f"status {bits:#x}"
    assert bits & ~0xF == 0, f"status {bits:#x}"
    assert dt < 2.0, f"the stalled kernel took {dt:.2f} s"
    out2 = Guarded(M * N, torch.bfloat16)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8q.fp8q_scaled_mm_wait_test(A, B, sa, sb, out2.t.view(M, N), st2, 20_000_000, -1)
    out2.check()
    assert int(st2.item()) == 0
    np.testing.assert_array_equal(host(out2.t.view(M, N)), want)
