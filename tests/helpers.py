"""Comparison helpers shared by the tests (test-only; no method arithmetic).

Bit-exact comparison is the bar.  The one place where several results are
equally correct is the sign and payload of a NaN: IEEE 754 leaves the sign of
a NaN produced by arithmetic (Inf * 0, x * NaN) unspecified, and x86 and the
GPU choose differently.  So a NaN compares equal to any NaN of the same
format, and everything else must match bit for bit.
"""
from __future__ import annotations

import numpy as np


def fp8_is_nan(c: np.ndarray, fmt: int) -> np.ndarray:
    c = np.asarray(c, dtype=np.uint8)
    if fmt == 0:  # e4m3fn: S.1111.111
        return (c & 0x7F) == 0x7F
    return ((c & 0x7C) == 0x7C) & ((c & 0x03) != 0)  # e5m2: exponent 31, mantissa != 0


def f32_is_nan(u: np.ndarray) -> np.ndarray:
    u = np.asarray(u).view(np.uint32)
    return (u & 0x7FFFFFFF) > 0x7F800000


def h16_is_nan(u: np.ndarray, kind: str) -> np.ndarray:
    u = np.asarray(u).view(np.uint16)
    if kind == "bf16":
        return (u & 0x7FFF) > 0x7F80
    return (u & 0x7FFF) > 0x7C00


def _report(name, a, b, bad):
    idx = np.argwhere(bad)
    first = idx[:8].tolist()
    av = a[tuple(idx[:8].T)] if idx.size else []
    bv = b[tuple(idx[:8].T)] if idx.size else []
    return (f"{name}: {int(bad.sum())} of {bad.size} differ; first at {first}: "
            f"got {[hex(int(v)) for v in av]} want {[hex(int(v)) for v in bv]}")


def assert_codes_equal(got, want, fmt: int, name: str = "fp8 codes"):
    got = np.asarray(got, dtype=np.uint8)
    want = np.asarray(want, dtype=np.uint8)
    assert got.shape == want.shape, (got.shape, want.shape)
    gn, wn = fp8_is_nan(got, fmt), fp8_is_nan(want, fmt)
    bad = (gn != wn) | (~gn & (got != want))
    assert not bad.any(), _report(name, got, want, bad)


def assert_f32_equal(got, want, name: str = "fp32"):
    got = np.ascontiguousarray(got, dtype=np.float32).view(np.uint32)
    want = np.ascontiguousarray(want, dtype=np.float32).view(np.uint32)
    assert got.shape == want.shape, (got.shape, want.shape)
    gn, wn = f32_is_nan(got), f32_is_nan(want)
    bad = (gn != wn) | (~gn & (got != want))
    assert not bad.any(), _report(name, got, want, bad)


def assert_h16_equal(got, want, kind: str = "bf16", name: str = "16-bit"):
    got = np.ascontiguousarray(got).view(np.uint16)
    want = np.ascontiguousarray(want).view(np.uint16)
    assert got.shape == want.shape, (got.shape, want.shape)
    gn, wn = h16_is_nan(got, kind), h16_is_nan(want, kind)
    bad = (gn != wn) | (~gn & (got != want))
    assert not bad.any(), _report(name, got, want, bad)


def assert_out_equal(got, want, yt: int, name: str = "y"):
    """Compare dequantised outputs in output type yt (0 f32, 1 f16, 2 bf16)."""
    if yt == 0:
        assert_f32_equal(got, want, name)
    else:
        assert_h16_equal(got, want, "f16" if yt == 1 else "bf16", name)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def load_golden(name: str) -> dict:
    """Parse a tests/golden/*.txt fixture: '# ...' comments, 'key = value' lines."""
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)
    out = {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = line.split("=", 1)
            out[k.strip()] = v.strip()
    return out


def hex_list(s: str, dtype) -> np.ndarray:
    """'3f80 3f00 0000*3' -> array; 'v*k' repeats v k times."""
    vals = []
    for tok in s.split():
        if "*" in tok:
            v, k = tok.split("*")
            vals.extend([int(v, 16)] * int(k))
        else:
            vals.append(int(tok, 16))
    return np.array(vals, dtype=dtype)
