"""Pins for the oracle's scaled fp8 matrix product (CPU only).

ColossalAI colossalai/quantization/fp8.py, _LinearFp8.forward:
torch._scaled_mm(x_fp8, w_fp8.t(), scale_a, scale_b, bias) with the
per-tensor scale_inv of each operand, i.e.
    out[m][n] = (sum_k dec(a[m][k]) * dec(b[n][k])) * sa * sb + bias[n].

Pinned by: closed forms (constant operands), an identity operand that
returns the other operand transposed (a transposed or swapped operand fails),
exact integer arithmetic (every e4m3fn value is a multiple of 2^-9, so the
exact sum is an integer count of 2^-18 units), numpy's float64 product of the
decoded operands, and the row range.
"""
import numpy as np
import pytest

E4M3FN, E5M2 = 0, 1
ONE = {E4M3FN: 0x38, E5M2: 0x3C}          # the code of 1.0


def _finite_codes(g, shape, fmt):
    import workloads
    codes = workloads.finite_e4m3fn_codes() if fmt == E4M3FN else workloads.finite_e5m2_codes()
    c = workloads.uniform_codes(g, shape, codes)
    if fmt == E5M2:
        c[(c & 0x7F) == 0x7C] = 0                # no infinities in the random operands
    return c


def test_closed_form_constants(orc):
    for fa, fb in ((E4M3FN, E4M3FN), (E5M2, E4M3FN), (E4M3FN, E5M2)):
        M, N, K = 3, 5, 96
        a = np.full((M, K), ONE[fa], np.uint8)                 # 1.0
        b = np.full((N, K), ONE[fb] + (4 if fb == E4M3FN else 2), np.uint8)   # 1.5
        bias = np.arange(N, dtype=np.float64) - 2.0
        out = orc.scaled_mm(a, fa, b, fb, 0.5, 0.25, bias=bias)
        np.testing.assert_array_equal(out, np.tile(K * 1.5 * 0.125 + bias, (M, 1)))
        # negative codes flip the sign; no bias
        out = orc.scaled_mm(a | 0x80, fa, b, fb, 2.0, 1.0)
        np.testing.assert_array_equal(out, np.full((M, N), -K * 1.5 * 2.0))


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_identity_operand_gives_the_other_transposed(orc, fmt):
    g = np.random.default_rng(11 + fmt)
    K, N = 48, 7
    a = np.zeros((K, K), np.uint8)
    a[np.arange(K), np.arange(K)] = ONE[fmt]
    b = _finite_codes(g, (N, K), fmt)
    out = orc.scaled_mm(a, fmt, b, fmt, 1.0, 1.0)
    np.testing.assert_array_equal(out, orc.fp8_decode(b, fmt).astype(np.float64).T)
    # and as the right operand: out = dec(a_rand) (b = identity, stored [N][K])
    out = orc.scaled_mm(b, fmt, a, fmt, 1.0, 1.0)
    np.testing.assert_array_equal(out, orc.fp8_decode(b, fmt).astype(np.float64))


def test_e4m3_sum_is_exact(orc):
    """Every e4m3fn value is an integer multiple of 2^-9: the exact sum,
    counted in 2^-18 units with Python integers, equals the oracle's."""
    g = np.random.default_rng(5)
    M, N, K = 4, 6, 1000
    a = _finite_codes(g, (M, K), E4M3FN)
    b = _finite_codes(g, (N, K), E4M3FN)
    out = orc.scaled_mm(a, E4M3FN, b, E4M3FN, 1.0, 1.0)
    ia = (orc.fp8_decode(a, E4M3FN).astype(np.float64) * 512).astype(np.int64)
    ib = (orc.fp8_decode(b, E4M3FN).astype(np.float64) * 512).astype(np.int64)
    for m in range(M):
        for n in range(N):
            exact = sum(int(x) * int(y) for x, y in zip(ia[m], ib[n]))
            assert out[m, n] == exact / float(1 << 18)


@pytest.mark.parametrize("fa,fb", [(E4M3FN, E4M3FN), (E5M2, E5M2), (E5M2, E4M3FN)])
def test_matches_numpy_float64_product(orc, fa, fb):
    g = np.random.default_rng(7 + fa + 2 * fb)
    M, N, K = 33, 17, 256
    a = _finite_codes(g, (M, K), fa)
    b = _finite_codes(g, (N, K), fb)
    sa, sb = np.float32(0.0123), np.float32(3.5)
    bias = g.standard_normal(N)
    out = orc.scaled_mm(a, fa, b, fb, float(sa), float(sb), bias=bias)
    ref = (orc.fp8_decode(a, fa).astype(np.float64) @ orc.fp8_decode(b, fb).astype(np.float64).T)
    ref = ref * float(sa) * float(sb) + bias
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_row_range_and_empty(orc):
    g = np.random.default_rng(3)
    a = _finite_codes(g, (10, 32), E4M3FN)
    b = _finite_codes(g, (4, 32), E4M3FN)
    full = orc.scaled_mm(a, E4M3FN, b, E4M3FN, 1.0, 1.0)
    part = orc.scaled_mm(a, E4M3FN, b, E4M3FN, 1.0, 1.0, rows=(3, 7))
    np.testing.assert_array_equal(part[3:7], full[3:7])
    assert not part[:3].any() and not part[7:].any()
    # K = 0: the sum is empty, so out is the bias alone
    out = orc.scaled_mm(np.zeros((2, 0), np.uint8), E4M3FN, np.zeros((3, 0), np.uint8), E4M3FN, 1.0, 1.0,
                        bias=np.array([1.0, -2.0, 0.5]))
    np.testing.assert_array_equal(out, np.array([[1.0, -2.0, 0.5]] * 2))


# ---------------------------------------------------------------------------
# fine-grained scales: DeepEP per-token activations (sa[M][K/G]) times a
# DeepSeek-V3 block-scaled weight (sb[ceil(N/B)][ceil(K/B)])
# ---------------------------------------------------------------------------
def _torch_decode(codes, fmt):
    """Exact fp8 values from torch's own fp8 -> float64 conversion."""
    import torch
    dt = torch.float8_e4m3fn if fmt == E4M3FN else torch.float8_e5m2
    return torch.from_numpy(np.ascontiguousarray(codes)).view(dt).to(torch.float64).numpy()


def _golden(name):
    import os
    p = os.path.join(os.path.dirname(__file__), "golden", name)
    d = {}
    for line in open(p):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = (s.strip() for s in line.split("=", 1))
            d[k] = v
    return d


def test_blockwise_hand_worked(orc):
    d = _golden("scaled_mm_blockwise_small.txt")
    M, N, K, G, B = (int(d[k]) for k in ("M", "N", "K", "group", "block"))
    a = np.array([int(t, 16) for t in d["a"].split()], np.uint8).reshape(M, K)
    b = np.array([int(t, 16) for t in d["b"].split()], np.uint8).reshape(N, K)
    sa = np.array(d["sa"].split(), np.float32).reshape(M, -(-K // G))
    sb = np.array(d["sb"].split(), np.float32).reshape(-(-N // B), -(-K // B))
    bias = np.array(d["bias"].split(), np.float64)
    want = np.array(d["out"].split(), np.float64).reshape(M, N)
    out = orc.scaled_mm_blockwise(a, E4M3FN, sa, b, E4M3FN, sb, group=G, block=B, bias=bias)
    np.testing.assert_array_equal(out, want)


@pytest.mark.parametrize("fa,fb,M,N,K", [(E4M3FN, E4M3FN, 37, 300, 384), (E5M2, E4M3FN, 5, 129, 256),
                                         (E4M3FN, E5M2, 130, 17, 200)])
def test_blockwise_matches_dequantise_then_matmul(orc, fa, fb, M, N, K):
    """The definition with library routines: decode with torch, scale every
    element by its group / block scale, numpy float64 matmul.  Non-square
    scale grids, a partial last weight block-row (N % 128) and a partial last
    K group make a transposed or shifted scale index fail."""
    g = np.random.default_rng(100 + M)
    G = B = 128
    a = _finite_codes(g, (M, K), fa)
    b = _finite_codes(g, (N, K), fb)
    sa = np.exp(g.normal(-4, 2, (M, -(-K // G)))).astype(np.float32)
    sb = np.exp(g.normal(-8, 1, (-(-N // B), -(-K // B)))).astype(np.float32)
    bias = g.standard_normal(N)
    out = orc.scaled_mm_blockwise(a, fa, sa, b, fb, sb, bias=bias)
    A = _torch_decode(a, fa) * np.repeat(sa.astype(np.float64), G, axis=1)[:, :K]
    W = _torch_decode(b, fb) * np.repeat(np.repeat(sb.astype(np.float64), B, axis=0), B, axis=1)[:N, :K]
    ref = A @ W.T + bias
    mag = np.abs(A) @ np.abs(W).T + np.abs(bias)
    assert np.all(np.abs(out - ref) <= 1e-13 * mag)


def test_blockwise_power_of_two_scales_are_exact(orc):
    """With power-of-two scales every dequantised product is a multiple of a
    fixed power of two: the exact sum, in Python integers, equals the
    oracle's value exactly."""
    from fractions import Fraction
    g = np.random.default_rng(9)
    M, N, K = 3, 130, 256
    a = _finite_codes(g, (M, K), E4M3FN)
    b = _finite_codes(g, (N, K), E4M3FN)
    ea = g.integers(-6, 7, (M, 2))
    eb = g.integers(-6, 7, (2, 2))
    sa = np.ldexp(1.0, ea).astype(np.float32)
    sb = np.ldexp(1.0, eb).astype(np.float32)
    out = orc.scaled_mm_blockwise(a, E4M3FN, sa, b, E4M3FN, sb)
    va = (_torch_decode(a, E4M3FN) * 512).astype(np.int64)     # integer multiples of 2^-9
    vb = (_torch_decode(b, E4M3FN) * 512).astype(np.int64)
    for m in range(M):
        for n in (0, 1, 127, 128, 129):
            exact = Fraction(0)
            for k in range(K):
                exact += Fraction(int(va[m, k]) * int(vb[n, k]), 1 << 18) * \
                    Fraction(2) ** int(ea[m, k // 128]) * Fraction(2) ** int(eb[n // 128, k // 128])
            assert Fraction(out[m, n]) == exact, (m, n)


def test_blockwise_uniform_scales_reduce_to_per_tensor(orc):
    g = np.random.default_rng(4)
    M, N, K = 9, 140, 256
    a = _finite_codes(g, (M, K), E4M3FN)
    b = _finite_codes(g, (N, K), E4M3FN)
    sa = np.full((M, 2), 0.375, np.float32)
    sb = np.full((2, 2), 2.0 ** -7, np.float32)
    out = orc.scaled_mm_blockwise(a, E4M3FN, sa, b, E4M3FN, sb)
    np.testing.assert_array_equal(out, orc.scaled_mm(a, E4M3FN, b, E4M3FN, 0.375, 2.0 ** -7))


def test_blockwise_rows_and_empty(orc):
    g = np.random.default_rng(8)
    a = _finite_codes(g, (10, 128), E4M3FN)
    b = _finite_codes(g, (4, 128), E4M3FN)
    sa = np.ones((10, 1), np.float32)
    sb = np.ones((1, 1), np.float32)
    full = orc.scaled_mm_blockwise(a, E4M3FN, sa, b, E4M3FN, sb)
    part = orc.scaled_mm_blockwise(a, E4M3FN, sa, b, E4M3FN, sb, rows=(2, 5))
    np.testing.assert_array_equal(part[2:5], full[2:5])
    assert not part[:2].any() and not part[5:].any()
    out = orc.scaled_mm_blockwise(np.zeros((2, 0), np.uint8), E4M3FN, np.zeros((2, 0), np.float32),
                                  np.zeros((3, 0), np.uint8), E4M3FN, np.zeros((1, 0), np.float32),
                                  bias=np.array([1.0, -2.0, 0.5]))
    np.testing.assert_array_equal(out, np.array([[1.0, -2.0, 0.5]] * 2))


# ---------------------------------------------------------------------------
# the library's single-precision rounding of the two products
# ---------------------------------------------------------------------------
def _exact_grid_codes(g, shape, fmt):
    """Codes whose values are multiples of 1/8 of magnitude <= 4: products are
    multiples of 2^-6 below 16, so every partial sum of up to 2^12 of them is
    an fp32 number and any fp32 summation order is exact."""
    import workloads
    codes = workloads.finite_e4m3fn_codes() if fmt == E4M3FN else workloads.finite_e5m2_codes()
    v = _torch_decode(codes, fmt)
    keep = codes[(np.abs(v) <= 4) & (v * 8 == np.round(v * 8))]
    return keep[g.integers(0, keep.size, size=shape)].astype(np.uint8)


def _torch_round(v64, yt):
    import torch
    dt = {0: torch.float32, 1: torch.float16, 2: torch.bfloat16}[yt]
    t = torch.from_numpy(np.ascontiguousarray(v64)).to(dt)
    return t.numpy() if yt == 0 else t.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("yt", [0, 1, 2])
def test_rounded_forms_closed_form(orc, yt):
    """Exact-grid operands, power-of-two scales and a bias on the same grid:
    every fp32 step is exact, so the output is the exact value rounded once to
    T, which torch's own float64 -> T conversion gives."""
    g = np.random.default_rng(30 + yt)
    M, N, K = 7, 300, 1024
    fa, fb = E4M3FN, E5M2
    a = _exact_grid_codes(g, (M, K), fa)
    b = _exact_grid_codes(g, (N, K), fb)
    bias = (g.integers(-512, 512, N) / 64.0).astype(np.float32)
    A, W = _torch_decode(a, fa), _torch_decode(b, fb)
    exact = (A @ W.T) * 0.25 * 0.5 + bias
    got = orc.scaled_mm_rounded(a, fa, b, fb, 0.25, 0.5, bias=bias, yt=yt)
    np.testing.assert_array_equal(got, _torch_round(exact, yt))
    # fine-grained: power-of-two scales 1/2 .. 2 per group / block keep every
    # product a multiple of 2^-8 and every sum below 2^16 (24 bits)
    kb = K // 128
    sa = np.ldexp(1.0, g.integers(-1, 2, (M, kb))).astype(np.float32)
    sb = np.ldexp(1.0, g.integers(-1, 2, (-(-N // 128), kb))).astype(np.float32)
    Af = A * np.repeat(sa.astype(np.float64), 128, axis=1)
    Wf = W * np.repeat(np.repeat(sb.astype(np.float64), 128, axis=0), 128, axis=1)[:N]
    exact = Af @ Wf.T + bias
    got = orc.scaled_mm_blockwise_rounded(a, fa, sa, b, fb, sb, bias=bias, yt=yt)
    np.testing.assert_array_equal(got, _torch_round(exact, yt))


def test_rounded_epilogue_order_hand_worked(orc):
    d = _golden("scaled_mm_epilogue_order.txt")
    K = int(d["K"])
    a = np.array([int(t, 16) for t in d["a"].split()], np.uint8).reshape(1, K)
    b = np.array([int(t, 16) for t in d["b"].split()], np.uint8).reshape(1, K)
    s = float(np.array(int(d["scale_f32"], 16), np.uint32).view(np.float32))
    got = orc.scaled_mm_rounded(a, E4M3FN, b, E4M3FN, s, s, yt=0)
    assert got.view(np.uint32)[0, 0] == int(d["out_f32"], 16)
    got = orc.scaled_mm_rounded(a, E4M3FN, b, E4M3FN, s, s, bias=np.array([float(d["bias"])]), yt=0)
    assert got.view(np.uint32)[0, 0] == int(d["out_f32_bias"], 16)
    got = orc.scaled_mm_rounded(a, E4M3FN, b, E4M3FN, s, s, yt=2)
    assert got[0, 0] == int(d["out_bf16"], 16)


def test_rounded_forms_stay_within_half_an_ulp_of_the_exact_product(orc):
    """General operands: each fp32 step rounds once, so the fp32 result lies
    within a few fp32 ulps of the binary64 definition (a dropped k-block, a
    swapped scale or a wrong bias would be far outside)."""
    g = np.random.default_rng(44)
    M, N, K = 6, 140, 512
    a = _finite_codes(g, (M, K), E4M3FN)
    b = _finite_codes(g, (N, K), E4M3FN)
    sa = np.exp(g.normal(-4, 2, (M, 4))).astype(np.float32)
    sb = np.exp(g.normal(-8, 1, (2, 4))).astype(np.float32)
    bias = g.standard_normal(N).astype(np.float32)
    exact = orc.scaled_mm_blockwise(a, E4M3FN, sa, b, E4M3FN, sb, bias=bias.astype(np.float64))
    A, W = _torch_decode(a, E4M3FN), _torch_decode(b, E4M3FN)
    mag = (np.abs(A) * np.repeat(sa, 128, axis=1)) @ (np.abs(W) * np.repeat(np.repeat(sb, 128, 0), 128, 1)[:N]).T
    got = orc.scaled_mm_blockwise_rounded(a, E4M3FN, sa, b, E4M3FN, sb, bias=bias, yt=0)
    assert np.all(np.abs(got - exact) <= 2.0 ** -21 * (mag + np.abs(bias)))
    got = orc.scaled_mm_rounded(a, E4M3FN, b, E4M3FN, 0.01, 3.0, bias=bias, yt=0)
    exact = orc.scaled_mm(a, E4M3FN, b, E4M3FN, 0.01, 3.0, bias=bias.astype(np.float64))
    mag = (np.abs(A) @ np.abs(W).T) * 0.03
    assert np.all(np.abs(got - exact) <= 2.0 ** -21 * (mag + np.abs(bias)))


# ---------------------------------------------------------------------------
# _LinearFp8.backward's transpose and bias gradient
# ---------------------------------------------------------------------------
def test_transpose_by_index(orc):
    """Brute force on a small case: every destination byte by its index rule."""
    g = np.random.default_rng(12)
    rows, cols, ld = 5, 7, 16
    src = g.integers(0, 256, (rows, cols), dtype=np.uint8)
    dst = orc.transpose_u8(src, ld)
    for c in range(cols):
        for r in range(ld):
            assert dst[c, r] == (src[r, c] if r < rows else 0)
    big = g.integers(0, 256, (130, 333), dtype=np.uint8)
    np.testing.assert_array_equal(orc.transpose_u8(big), big.T)


def test_sum_rows_exact_integers(orc):
    """Small integers are exact in bf16 and in the sum: the oracle's column
    sums equal Python's integer sums."""
    import torch
    g = np.random.default_rng(13)
    v = g.integers(-100, 101, (300, 50)).astype(np.float32)
    bits = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    out = orc.sum_rows(bits, orc.BF16)
    for c in range(50):
        assert out[c] == sum(int(t) for t in v[:, c])
    f = g.standard_normal((64, 9)).astype(np.float32)
    np.testing.assert_allclose(orc.sum_rows(f, orc.F32), f.astype(np.float64).sum(0), rtol=1e-14, atol=1e-14)
    assert (orc.sum_rows(np.zeros((0, 4), np.float32), orc.F32) == 0).all()
