"""A second, deliberately naive formulation of the method (test-only).

It shares nothing with the oracle in oracle/:

* fp8 code values come from torch's own fp8 -> fp32 cast of all 256 codes
  (a library routine), not from a bit-level decoder;
* encoding searches the sorted code values for the nearest one (ties to the
  code with an even mantissa bit) instead of shifting bits;
* every IEEE binary32 operation fl(a op b) is computed exactly in float64 and
  rounded once to float32.  For +, -, *, / of binary32 operands this double
  rounding is innocuous (53 >= 2 * 24 + 2), so the result is the correctly
  rounded binary32 value;
* bf16 / fp16 narrowing uses torch's and numpy's casts.

It is vectorised numpy and slow only in the sense of being simple; it is used
for brute-force comparison on small inputs.
"""
from __future__ import annotations

import numpy as np
import torch

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2

_TORCH_FP8 = {E4M3FN: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def code_values(fmt: int) -> np.ndarray:
    t = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(_TORCH_FP8[fmt])
    return t.to(torch.float32).numpy().astype(np.float64)


def fmax(fmt: int) -> float:
    return float(torch.finfo(_TORCH_FP8[fmt]).max)


def fl(x) -> np.ndarray:
    """Round float64 to the nearest binary32 (overflow gives +-Inf)."""
    with np.errstate(all="ignore"):
        return np.asarray(x, dtype=np.float64).astype(np.float32)


def _positive_table(fmt: int):
    vals = code_values(fmt)
    top = 0x7E if fmt == E4M3FN else 0x7B
    codes = np.arange(top + 1)
    v = vals[: top + 1]
    assert np.all(np.diff(v) > 0)
    # the value one step past the largest finite code: rounding onto it means overflow
    step = v[top] - v[top - 1]
    virt = v[top] + step
    virt_code = 0x7F if fmt == E4M3FN else 0x7C
    return np.append(v, virt), np.append(codes, virt_code)


def encode(v, fmt: int) -> np.ndarray:
    """fp32 -> fp8 code by nearest-value search (ties to even code), non-saturating."""
    v = np.asarray(v, dtype=np.float32)
    bits = v.view(np.uint32)
    sign = ((bits >> 24) & 0x80).astype(np.uint8)
    a = np.abs(v.astype(np.float64))
    table, codes = _positive_table(fmt)
    hi = np.clip(np.searchsorted(table, a, side="left"), 0, table.size - 1)
    lo = np.clip(hi - 1, 0, table.size - 1)
    dlo = np.abs(a - table[lo])
    dhi = np.abs(table[hi] - a)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (codes[hi] % 2 == 0) & (hi != lo))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(a > table[-1], table.size - 1, idx)
    out = codes[idx].astype(np.uint8)
    overflow_code = 0x7F if fmt == E4M3FN else 0x7C
    out = np.where(np.isinf(a), overflow_code, out)
    out = np.where(np.isnan(a), 0x7F, out).astype(np.uint8)
    return out | sign


def decode(c, fmt: int) -> np.ndarray:
    return code_values(fmt)[np.asarray(c, dtype=np.uint8)]


def widen(bits_or_f32, xt: int) -> np.ndarray:
    if xt == F32:
        return np.asarray(bits_or_f32, dtype=np.float32)
    if xt == BF16:
        return torch.from_numpy(np.asarray(bits_or_f32, dtype=np.uint16).view(np.int16)).view(
            torch.bfloat16).float().numpy()
    return np.asarray(bits_or_f32, dtype=np.uint16).view(np.float16).astype(np.float32)


def narrow(v32: np.ndarray, yt: int) -> np.ndarray:
    v32 = np.asarray(v32, dtype=np.float32)
    if yt == F32:
        return v32
    if yt == BF16:
        return torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    with np.errstate(all="ignore"):
        return v32.astype(np.float16).view(np.uint16)


def _amax_nan(a: np.ndarray, axis) -> np.ndarray:
    """max |a| along axis, NaN if any element is NaN."""
    m = np.max(np.where(np.isnan(a), 0.0, np.abs(a)), axis=axis)
    return np.where(np.isnan(a).any(axis=axis), np.nan, m)


def _scale(F, amax, rule):
    """fl(F / amax), or torch's fl(fl(1 / amax) * F)."""
    if rule == 1:
        return fl(fl(1.0 / amax).astype(np.float64) * F).astype(np.float64)
    return fl(F / amax).astype(np.float64)


def _scale_inv(F, amax, rule):
    """fl(amax / F), or torch's GPU form fl(amax * fl(1 / F))."""
    if rule == 1:
        return fl(amax * float(fl(1.0 / F)))
    return fl(amax / F)


@np.errstate(all="ignore")
def per_token_group_quant(x, xt, group, fmt, rule=0):
    xf = widen(x, xt).astype(np.float64)
    m, n = xf.shape
    g = xf.reshape(m, n // group, group)
    amax = _amax_nan(g, 2)
    lo = float(np.float32(1e-4))
    amax = np.where(amax < lo, lo, amax)           # clamp; NaN stays NaN
    amax = fl(amax).astype(np.float64)
    F = fmax(fmt)
    scale = _scale(F, amax, rule)
    sinv = _scale_inv(F, amax, rule)
    q = encode(fl(g * scale[:, :, None]), fmt).reshape(m, n)
    return q, sinv


@np.errstate(all="ignore")
def cast_per_channel(x, xt, fmt, rule=0):
    xf = widen(x, xt).astype(np.float64)
    amax = _amax_nan(xf, 1)
    amax = np.where(amax > 0, amax, 1.0)           # NaN fails > 0
    F = fmax(fmt)
    scale = _scale(F, amax, rule)
    sinv = _scale_inv(F, amax, rule)
    return encode(fl(xf * scale[:, None]), fmt), sinv


def cast_per_tensor(x, xt, fmt, rule=0):
    xf = widen(x, xt).astype(np.float64).reshape(-1)
    if xf.size == 0:
        return np.zeros(0, np.uint8), np.array([1.0], np.float32)
    amax = np.float64(_amax_nan(xf, 0))
    amax = amax if amax > 0 else np.float64(1.0)
    F = np.float64(fmax(fmt))
    with np.errstate(all="ignore"):
        scale = np.float64(_scale(F, amax, rule))
        sinv = fl(np.float64(1.0) / scale).reshape(1)
        return encode(fl(xf * scale), fmt), sinv


@np.errstate(all="ignore")
def block_dequant(w, s, fmt, block, yt):
    w = np.asarray(w, dtype=np.uint8)
    M, N = w.shape
    i = np.arange(M)[:, None] // block
    j = np.arange(N)[None, :] // block
    sc = np.asarray(s, dtype=np.float32).astype(np.float64)[i, j]
    return narrow(fl(decode(w, fmt) * sc), yt)


@np.errstate(all="ignore")
def cast_from_fp8(q, scale_inv, gran, fmt, gb, yt):
    q = np.asarray(q, dtype=np.uint8)
    R, C = q.shape
    s = np.asarray(scale_inv, dtype=np.float32).astype(np.float64).reshape(-1)
    r = np.arange(R)[:, None]
    c = np.arange(C)[None, :]
    if gran == 0:
        sc = np.broadcast_to(s[0], (R, C))
    elif gran == 1:
        sc = np.broadcast_to(s[r], (R, C))
    elif gran == 2:
        sc = s[r * (C // gb) + c // gb]
    else:
        sc = s[(r // gb) * ((C + gb - 1) // gb) + c // gb]
    return narrow(fl(decode(q, fmt) * sc), yt)


@np.errstate(all="ignore")
def cast_pipeline(x, xt, rule=0):
    """Format by amax (e5m2 above 448), scale 1 for an all-zero tensor."""
    xf = widen(x, xt).astype(np.float64).reshape(-1)
    amax = np.float64(_amax_nan(xf, 0)) if xf.size else np.float64(0.0)
    fmt = E5M2 if amax > 448.0 else E4M3FN
    scale = np.float64(1.0) if amax == 0 else np.float64(_scale(fmax(fmt), amax, rule))
    sinv = fl(np.float64(1.0) / scale).reshape(1)
    return encode(fl(xf * scale), fmt), sinv, fmt


@np.errstate(all="ignore")
def cast_from_pipeline(q, fmt, scale_inv, yt):
    return narrow(fl(decode(q, fmt) * np.float64(np.float32(scale_inv[0]))), yt)
