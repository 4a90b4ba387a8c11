"""GPU pins of the NaN bit patterns the library writes, one test per cast kind.

IEEE 754 leaves the sign (and payload) of a NaN produced by arithmetic
unspecified, so the oracle-versus-kernel comparisons elsewhere treat any NaN of
a format as equal.  This file pins which NaN the library actually writes:

- fp8 codes: 0x7F, the positive NaN code of e4m3fn and of e5m2;
- fp32 values: 0x7FFFFFFF; bf16 and fp16 values: 0x7FFF;

whatever the sign of the NaN (or of the +/-Inf times zero) that produced it.
A finite or infinite value that overflows e4m3fn also becomes a NaN code, but
its sign is defined and kept (0xFF for a negative value), as torch's cast does.
These are the canonical NaNs of GPU arithmetic and conversion, so they are also
what the pages' own torch expressions give when they run on a CUDA device.
Each test therefore checks two things at every position where either side
holds a NaN: the library's bits are the canonical pattern, and torch on the
GPU, evaluating the page's expression for the same operation, holds the same
bits there.  Finite results are compared with the oracle as everywhere else.
"""
import numpy as np
import pytest
import torch

from gpu_util import dev, host
from helpers import assert_codes_equal, assert_f32_equal, assert_out_equal, fp8_is_nan, f32_is_nan, h16_is_nan

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
FP8_DT = {E4M3FN: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}
FMAX = {E4M3FN: 448.0, E5M2: 57344.0}
OUT_DT = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}


def _nan_input(rows, cols, seed):
    """fp32 [rows, cols] ~ N(0, 1) with NaNs of both signs and +/-Inf in chosen groups: row 0 a
    +NaN, row 1 a -NaN, row 2 one of each, row 3 +Inf and -Inf (no NaN), row 4 a -NaN and a -Inf."""
    g = np.random.default_rng(seed)
    x = g.standard_normal((rows, cols)).astype(np.float32)
    neg_nan = np.array([0xFFC00001], np.uint32).view(np.float32)[0]
    pos_nan = np.array([0x7FC00002], np.uint32).view(np.float32)[0]
    x[0, 5] = pos_nan
    x[1, 130] = neg_nan
    x[2, 7], x[2, cols - 1] = pos_nan, neg_nan
    x[3, 3], x[3, 300 % cols] = np.inf, -np.inf
    x[4, 9], x[4, 200 % cols] = neg_nan, -np.inf
    return x


def _bits_u8(t):
    return host(t.contiguous().view(torch.uint8))


def _check_codes(ours, torch_codes, fmt, nan_product):
    """Wherever the scaled product is a NaN the library writes 0x7F; every other NaN code comes
    from a finite or infinite value that overflows e4m3fn, whose sign is defined and kept.  At
    every position where either side holds a NaN, the bytes equal torch's on the GPU."""
    ours = np.asarray(ours, np.uint8)
    theirs = np.asarray(torch_codes, np.uint8)
    nan_product = np.asarray(nan_product, bool)
    on, tn = fp8_is_nan(ours, fmt), fp8_is_nan(theirs, fmt)
    assert nan_product.any(), "the input was meant to produce NaN products"
    assert on[nan_product].all()
    assert (ours[nan_product] == 0x7F).all(), sorted({hex(v) for v in ours[nan_product]})
    assert (on == tn).all(), "NaN positions differ from torch on the GPU"
    assert (ours[on] == theirs[on]).all(), "NaN codes differ from torch on the GPU"


def _check_f32(ours, theirs):
    u = np.ascontiguousarray(ours, np.float32).view(np.uint32)
    t = np.ascontiguousarray(theirs, np.float32).view(np.uint32)
    un, tn = f32_is_nan(u), f32_is_nan(t)
    assert (un == tn).all(), "NaN positions differ from torch on the GPU"
    assert (u[un] == 0x7FFFFFFF).all(), sorted({hex(v) for v in u[un]})
    assert (u[un] == t[un]).all()
    return int(un.sum())


def _check_h16(ours, theirs, kind):
    u = np.ascontiguousarray(ours).view(np.uint16)
    t = np.ascontiguousarray(theirs).view(np.uint16)
    un, tn = h16_is_nan(u, kind), h16_is_nan(t, kind)
    assert (un == tn).all(), "NaN positions differ from torch on the GPU"
    assert (u[un] == 0x7FFF).all(), sorted({hex(v) for v in u[un]})
    assert (u[un] == t[un]).all()
    return int(un.sum())


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
@pytest.mark.parametrize("xt", [BF16, F32])
def test_per_token_nan_bits(fp8q, orc, fmt, xt):
    """DeepEP per_token_cast_to_fp8 on a CUDA tensor: amax over each 1 x 128 group (NaN
    propagates), clamp(1e-4), x * (FMAX / amax) cast to fp8, scale_inv = amax / FMAX."""
    m, n = 6, 512
    x32 = _nan_input(m, n, 11 + fmt + 2 * xt)
    xd = torch.from_numpy(x32).cuda()
    if xt == BF16:
        xd = xd.to(torch.bfloat16)
    q = torch.empty((m, n), dtype=torch.uint8, device="cuda")
    s = torch.empty((m, n // 128), dtype=torch.float32, device="cuda")
    fp8q.fp8q_per_token_group_quant(xd, q, s, 128, fmt)
    xv = xd.view(m, -1, 128)
    amax = xv.abs().float().amax(dim=2).view(m, -1).clamp(1e-4)
    prod = (xv * (FMAX[fmt] / amax.unsqueeze(2))).view(m, n)
    tq = prod.to(FP8_DT[fmt])
    ts = (amax / FMAX[fmt]).view(m, -1)
    torch.cuda.synchronize()
    _check_codes(host(q), _bits_u8(tq), fmt, prod.isnan().cpu().numpy())
    assert _check_f32(host(s), host(ts)) > 0
    xo = host(xd.view(torch.int16) if xt == BF16 else xd)
    qo, so = orc.per_token_group_quant(xo, xt, 128, fmt)
    assert_codes_equal(host(q), qo, fmt)
    assert_f32_equal(host(s), so)


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_per_channel_nan_bits(fp8q, orc, fmt):
    """ColossalAI cast_to_fp8, per_channel_scale=True: a NaN row amax is replaced by 1, so a NaN
    element times FMAX is the NaN, and +/-Inf overflows (e4m3fn: NaN with the Inf's sign)."""
    rows, cols = 6, 384
    x32 = _nan_input(rows, cols, 21 + fmt)
    xd = torch.from_numpy(x32).cuda().to(torch.bfloat16)
    q = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    fp8q.fp8q_cast_per_channel(xd, q, s, fmt)
    pmax = xd.abs().max(dim=-1).values.float()
    pmax = torch.where(pmax > 0, pmax, 1.0)
    prod = FMAX[fmt] / pmax[:, None] * xd.float()
    tq = prod.to(FP8_DT[fmt])
    torch.cuda.synchronize()
    _check_codes(host(q), _bits_u8(tq), fmt, prod.isnan().cpu().numpy())
    qo, so = orc.cast_per_channel(host(xd.view(torch.int16)), BF16, fmt)
    assert_codes_equal(host(q), qo, fmt)
    assert_f32_equal(host(s), so)
    qh = host(q)
    # row 3: amax = Inf, scale = 0, so both infinities give Inf * 0, a NaN product
    assert qh[3, 3] == 0x7F and qh[3, 300] == 0x7F
    if fmt == E4M3FN:   # row 4: its NaN amax becomes 1, so -Inf * FMAX overflows and keeps its sign
        assert qh[4, 200] == 0xFF


@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_per_tensor_nan_bits(fp8q, orc, fmt):
    """ColossalAI cast_to_fp8 per-tensor: a NaN amax is replaced by 1 (scale = FMAX)."""
    x32 = _nan_input(6, 256, 31 + fmt).reshape(-1)
    xd = torch.from_numpy(x32).cuda().to(torch.float16)
    q = torch.empty(x32.size, dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    fp8q.fp8q_cast_per_tensor(xd, q, s, ws, fmt)
    amax = xd.abs().max().float()
    amax = torch.where(amax > 0, amax, 1.0)
    prod = (FMAX[fmt] / amax) * xd.float()
    tq = prod.to(FP8_DT[fmt])
    torch.cuda.synchronize()
    _check_codes(host(q), _bits_u8(tq), fmt, prod.isnan().cpu().numpy())
    qo, so = orc.cast_per_tensor(host(xd.view(torch.int16)), F16, fmt)
    assert_codes_equal(host(q), qo, fmt)
    assert_f32_equal(host(s), so)


NAN_CODES = {E4M3FN: [0x7F, 0xFF], E5M2: [0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF]}
INF_CODES = {E4M3FN: [], E5M2: [0x7C, 0xFC]}


@pytest.mark.parametrize("yt", [BF16, F16, F32])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_dequant_nan_bits(fp8q, orc, fmt, yt):
    """ColossalAI cast_from_fp8 (per-tensor and per-row) and the DeepSeek-V3 block dequant on
    NaN codes of both signs, and e5m2 +/-Inf codes times a zero scale: the result type's
    canonical NaN, as torch's q.float() * scale_inv, then .to(T), gives on the GPU."""
    rows, cols = 130, 256
    g = np.random.default_rng(41 + fmt + 3 * yt)
    codes = g.integers(0, 256, (rows, cols)).astype(np.uint8)
    codes[fp8_is_nan(codes, fmt)] = 0x10
    specials = NAN_CODES[fmt] + INF_CODES[fmt]
    for i, c in enumerate(specials):
        codes[i, 3 * i] = c
        codes[129, 5 + 7 * i] = c           # the partial block row
    srow = np.exp(g.standard_normal(rows)).astype(np.float32)
    srow[:len(specials)] = 0.0              # Inf codes in these rows meet a zero scale
    sblk = np.exp(g.standard_normal((2, 2))).astype(np.float32)
    sblk[0, 0] = 0.0
    qd = dev(codes)
    q8 = qd.view(FP8_DT[fmt])
    kind = "bf16" if yt == BF16 else "f16"
    total_nan = 0
    for gran, s, expand in ((0, np.array([0.5], np.float32), lambda t: t[0]),
                            (1, srow, lambda t: t[:, None]),
                            (3, sblk, lambda t: t.repeat_interleave(128, 0)[:rows].repeat_interleave(128, 1)[:, :cols])):
        sd = dev(s)
        y = torch.empty((rows, cols), dtype=OUT_DT[yt], device="cuda")
        fp8q.fp8q_cast_from_fp8(qd, sd, y, gran, 128 if gran == 3 else 0, fmt=fmt)
        ty = (q8.float() * expand(sd)).to(OUT_DT[yt])
        torch.cuda.synchronize()
        yo = orc.cast_from_fp8(codes, s, gran, fmt, 128 if gran == 3 else 0, yt)
        assert_out_equal(host(y), yo, yt)
        total_nan += _check_f32(host(y), host(ty)) if yt == F32 else _check_h16(host(y), host(ty), kind)
    assert total_nan > 0
