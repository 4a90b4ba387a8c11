"""CPU oracle for scaled FP8 casting -- TEST INFRASTRUCTURE ONLY.

Thin ctypes wrapper over ``libfp8q_oracle.so`` (plain C, ``fp8q_oracle.c``).
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package; the CUDA library and its Python
binding never touch it, and the two share no code.

Functions take and return numpy arrays.  Row-structured operations accept a
``rows=(r0, r1)`` range so that callers can sample rows or split work across
threads (ctypes releases the GIL during each C call).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8q_oracle.c")
_LIB = os.path.join(_HERE, "libfp8q_oracle.so")

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
GRAN_TENSOR, GRAN_ROW, GRAN_GROUP, GRAN_BLOCK = 0, 1, 2, 3
RULE_IEEE, RULE_TORCH = 0, 1

CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
          "-fno-finite-math-only", "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (SSE binary32, no FMA contraction)."""
    hdr = os.path.join(_HERE, "fp8q_oracle.h")
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= max(os.path.getmtime(_SRC), os.path.getmtime(hdr))):
        return _LIB
    tmp = _LIB + ".tmp.%d" % os.getpid()
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            c_void, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            L.orc_fp8_max.restype = ctypes.c_float
            L.orc_fp8_max.argtypes = [i32]
            L.orc_fp8_encode.restype = ctypes.c_uint8
            L.orc_fp8_encode.argtypes = [ctypes.c_float, i32]
            L.orc_fp8_decode.restype = ctypes.c_float
            L.orc_fp8_decode.argtypes = [ctypes.c_uint8, i32]
            for name in ("orc_fp8_encode_n", "orc_fp8_decode_n"):
                getattr(L, name).restype = None
                getattr(L, name).argtypes = [c_void, i64, i32, c_void]
            for name in ("orc_bf16_encode_n", "orc_f16_encode_n"):
                getattr(L, name).restype = None
                getattr(L, name).argtypes = [c_void, i64, c_void]
            L.orc_per_token_group_quant.restype = i32
            L.orc_per_token_group_quant.argtypes = [c_void, i32, i64, i64, i32, i32, c_void, c_void, i64, i64]
            L.orc_cast_per_channel.restype = i32
            L.orc_cast_per_channel.argtypes = [c_void, i32, i64, i64, i32, c_void, c_void, i64, i64]
            L.orc_cast_per_tensor.restype = i32
            L.orc_cast_per_tensor.argtypes = [c_void, i32, i64, i32, c_void, c_void, i64, i64]
            L.orc_per_token_group_quant_rule.restype = i32
            L.orc_per_token_group_quant_rule.argtypes = [c_void, i32, i64, i64, i32, i32, c_void, c_void, i64, i64, i32]
            L.orc_cast_per_channel_rule.restype = i32
            L.orc_cast_per_channel_rule.argtypes = [c_void, i32, i64, i64, i32, c_void, c_void, i64, i64, i32]
            L.orc_cast_per_tensor_rule.restype = i32
            L.orc_cast_per_tensor_rule.argtypes = [c_void, i32, i64, i32, c_void, c_void, i64, i64, i32]
            L.orc_cast_pipeline.restype = i32
            L.orc_cast_pipeline.argtypes = [c_void, i32, i64, c_void, c_void, c_void, i32, i64, i64]
            L.orc_cast_from_pipeline.restype = i32
            L.orc_cast_from_pipeline.argtypes = [c_void, i32, i64, c_void, i32, c_void, i64, i64]
            L.orc_block_dequant.restype = i32
            L.orc_block_dequant.argtypes = [c_void, i32, i64, i64, c_void, i32, i32, c_void, i64, i64]
            L.orc_cast_from_fp8.restype = i32
            L.orc_cast_from_fp8.argtypes = [c_void, i32, i64, i64, c_void, i32, i32, i32, c_void, i64, i64]
            L.orc_scaled_mm.restype = i32
            L.orc_scaled_mm.argtypes = [c_void, i32, c_void, i32, i64, i64, i64, ctypes.c_float, ctypes.c_float,
                                        c_void, c_void, i64, i64]
            L.orc_scaled_mm_rounded.restype = i32
            L.orc_scaled_mm_rounded.argtypes = [c_void, i32, c_void, i32, i64, i64, i64, ctypes.c_float,
                                                ctypes.c_float, c_void, i32, c_void, i64, i64]
            L.orc_scaled_mm_blockwise_rounded.restype = i32
            L.orc_scaled_mm_blockwise_rounded.argtypes = [c_void, i32, c_void, c_void, i32, c_void, i64, i64, i64,
                                                          i64, c_void, i32, c_void, i64, i64]
            L.orc_transpose_u8.restype = i32
            L.orc_transpose_u8.argtypes = [c_void, i64, i64, c_void, i64]
            L.orc_sum_rows.restype = i32
            L.orc_sum_rows.argtypes = [c_void, i32, i64, i64, c_void]
            L.orc_scaled_mm_blockwise.restype = i32
            L.orc_scaled_mm_blockwise.argtypes = [c_void, i32, c_void, i64, c_void, i32, c_void, i64,
                                                  i64, i64, i64, c_void, c_void, i64, i64]
            _lib = L
    return _lib


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
_NP_OF = {F32: np.float32, F16: np.uint16, BF16: np.uint16}


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what}: rejected arguments")


def _split(r0: int, r1: int, threads: int):
    threads = max(1, min(threads, r1 - r0))
    step = (r1 - r0 + threads - 1) // threads if r1 > r0 else 0
    return [(a, min(a + step, r1)) for a in range(r0, r1, step)] if step else [(r0, r1)]


def _run(fn, r0: int, r1: int, threads: int) -> None:
    parts = _split(r0, r1, threads)
    if len(parts) == 1:
        fn(*parts[0])
        return
    errs = []

    def work(a, b):
        try:
            fn(a, b)
        except Exception as e:  # pragma: no cover - surfaced below
            errs.append(e)

    ts = [threading.Thread(target=work, args=p) for p in parts]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    if errs:
        raise errs[0]


# ---------------------------------------------------------------------------
# scalar / bulk codecs
# ---------------------------------------------------------------------------
def fp8_max(fmt: int) -> float:
    return float(lib().orc_fp8_max(fmt))


def fp8_encode(v: np.ndarray, fmt: int) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_fp8_encode_n(_ptr(v), v.size, fmt, _ptr(out))
    return out


def fp8_decode(c: np.ndarray, fmt: int) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().orc_fp8_decode_n(_ptr(c), c.size, fmt, _ptr(out))
    return out


def bf16_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint16)
    lib().orc_bf16_encode_n(_ptr(v), v.size, _ptr(out))
    return out


def f16_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint16)
    lib().orc_f16_encode_n(_ptr(v), v.size, _ptr(out))
    return out


# ---------------------------------------------------------------------------
# the method
# ---------------------------------------------------------------------------
def per_token_group_quant(x: np.ndarray, xt: int, group: int = 128, fmt: int = E4M3FN,
                          rows=None, out=None, threads: int = 1, rule: int = RULE_IEEE):
    """DeepEP per_token_cast_to_fp8 over x[m, n]; returns (q uint8[m,n], scale_inv f32[m,n/group])."""
    x = np.ascontiguousarray(x)
    m, n = x.shape
    if out is None:
        q = np.zeros((m, n), np.uint8)
        s = np.zeros((m, n // group if group > 0 else 0), np.float32)
    else:
        q, s = out
    r0, r1 = rows if rows is not None else (0, m)
    L = lib()
    _run(lambda a, b: _check(L.orc_per_token_group_quant_rule(_ptr(x), xt, m, n, group, fmt,
                                                             _ptr(q), _ptr(s), a, b, rule),
                             "per_token_group_quant"), r0, r1, threads)
    return q, s


def cast_per_channel(x: np.ndarray, xt: int, fmt: int = E4M3FN, rows=None, out=None, threads: int = 1,
                     rule: int = RULE_IEEE):
    """ColossalAI cast_to_fp8(per_channel_scale=True) over x[rows, cols]; returns (q, scale_inv[rows])."""
    x = np.ascontiguousarray(x)
    R, C = x.shape
    if out is None:
        q = np.zeros((R, C), np.uint8)
        s = np.zeros((max(R, 1),), np.float32)
    else:
        q, s = out
    r0, r1 = rows if rows is not None else (0, R)
    L = lib()
    _run(lambda a, b: _check(L.orc_cast_per_channel_rule(_ptr(x), xt, R, C, fmt, _ptr(q), _ptr(s), a, b, rule),
                             "cast_per_channel"), r0, r1, threads)
    return q, s


def cast_per_tensor(x: np.ndarray, xt: int, fmt: int = E4M3FN, elems=None, out=None, threads: int = 1,
                    rule: int = RULE_IEEE):
    """ColossalAI cast_to_fp8(per_channel_scale=False) over flat x; returns (q, scale_inv[1])."""
    x = np.ascontiguousarray(x).reshape(-1)
    n = x.size
    if out is None:
        q = np.zeros((n,), np.uint8)
        s = np.zeros((1,), np.float32)
    else:
        q, s = out
    e0, e1 = elems if elems is not None else (0, n)
    L = lib()
    _run(lambda a, b: _check(L.orc_cast_per_tensor_rule(_ptr(x), xt, n, fmt, _ptr(q), _ptr(s), a, b, rule),
                             "cast_per_tensor"), e0, e1, threads)
    return q, s


def cast_pipeline(x: np.ndarray, xt: int, rule: int = RULE_IEEE, elems=None, threads: int = 1):
    """ColossalAI cast_to_fp8_pipeline over flat x; returns (q, scale_inv[1], fmt)."""
    x = np.ascontiguousarray(x).reshape(-1)
    n = x.size
    q = np.zeros((n,), np.uint8)
    s = np.zeros((1,), np.float32)
    f = np.zeros((1,), np.int32)
    e0, e1 = elems if elems is not None else (0, n)
    L = lib()
    _run(lambda a, b: _check(L.orc_cast_pipeline(_ptr(x), xt, n, _ptr(q), _ptr(s), _ptr(f), rule, a, b),
                             "cast_pipeline"), e0, e1, threads)
    return q, s, int(f[0])


def cast_from_pipeline(q: np.ndarray, fmt: int, scale_inv: np.ndarray, yt: int = BF16):
    """ColossalAI cast_from_fp8_pipeline; returns y with q's size in output type yt."""
    q = np.ascontiguousarray(q, dtype=np.uint8).reshape(-1)
    s = np.ascontiguousarray(scale_inv, dtype=np.float32)
    y = np.zeros((q.size,), _NP_OF[yt])
    _check(lib().orc_cast_from_pipeline(_ptr(q), fmt, q.size, _ptr(s), yt, _ptr(y), 0, q.size),
           "cast_from_pipeline")
    return y


def block_dequant(w: np.ndarray, s: np.ndarray, fmt: int = E4M3FN, block: int = 128, yt: int = BF16,
                  rows=None, out=None, threads: int = 1):
    """DeepSeek-V3 weight_dequant of w[M, N] with s[ceil(M/B), ceil(N/B)]; returns y[M, N]."""
    w = np.ascontiguousarray(w, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    M, N = w.shape
    y = np.zeros((M, N), _NP_OF[yt]) if out is None else out
    r0, r1 = rows if rows is not None else (0, M)
    L = lib()
    _run(lambda a, b: _check(L.orc_block_dequant(_ptr(w), fmt, M, N, _ptr(s), block, yt, _ptr(y), a, b),
                             "block_dequant"), r0, r1, threads)
    return y


def cast_from_fp8(q: np.ndarray, scale_inv: np.ndarray, gran: int, fmt: int = E4M3FN, gb: int = 0,
                  yt: int = BF16, rows=None, out=None, threads: int = 1):
    """ColossalAI cast_from_fp8 (any granularity) of q[rows, cols]; returns y[rows, cols]."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(scale_inv, dtype=np.float32)
    R, C = q.shape
    y = np.zeros((R, C), _NP_OF[yt]) if out is None else out
    r0, r1 = rows if rows is not None else (0, R)
    L = lib()
    _run(lambda a, b: _check(L.orc_cast_from_fp8(_ptr(q), fmt, R, C, _ptr(s), gran, gb, yt, _ptr(y), a, b),
                             "cast_from_fp8"), r0, r1, threads)
    return y


# ---------------------------------------------------------------------------
# fp8-compressed collectives (ColossalAI colossalai/quantization/fp8.py:
# all_gather_fp8, all_gather_fp8_lagacy, all_to_all_fp8, all_to_all_single_fp8).
# Each is the per-tensor cast of what a rank sends, the bytes moved as they
# are, and cast_from_fp8 with the sender's scale_inv on receipt; the ranks
# are plain Python lists here.  The record is the sender's
# [fp32 scale_inv | fp8 codes] buffer of all_gather_fp8_lagacy, with a
# 16-byte header (scale_inv in bytes 0..3, zeros after) and the payload
# zero-padded to a multiple of 16 bytes, or (header 4) exactly the page's
# 4-byte scale followed by the codes.
# ---------------------------------------------------------------------------
RECORD_HEADER = 16


def record_size(numel: int, header: int = RECORD_HEADER) -> int:
    """Bytes of one record.  header 16: 16-byte header, payload padded to a
    multiple of 16.  header 4: the page's own layout (all_gather_fp8_lagacy,
    SCALE_BYTES = 4), the scale then the codes, no padding."""
    if header == 4:
        return 4 + numel
    return RECORD_HEADER + ((numel + 15) // 16) * 16


def record(x: np.ndarray, xt: int, fmt: int, rule: int = RULE_IEEE, header: int = RECORD_HEADER) -> np.ndarray:
    """The sender's record for tensor x: its per-tensor cast, header first."""
    q, s = cast_per_tensor(x, xt, fmt, rule=rule)
    r = np.zeros((record_size(q.size, header),), np.uint8)
    r[0:4] = np.frombuffer(s.astype("<f4").tobytes(), np.uint8)
    r[header:header + q.size] = q
    return r


def record_decode(r: np.ndarray, numel: int, fmt: int, yt: int, header: int = RECORD_HEADER) -> np.ndarray:
    """The receiver's step: cast_from_fp8 of the payload with the header's scale_inv."""
    s = np.frombuffer(r[0:4].tobytes(), "<f4").astype(np.float32)
    q = r[header:header + numel].reshape(1, numel)
    return cast_from_fp8(q, s, GRAN_TENSOR, fmt, yt=yt).reshape(-1)


def all_gather_fp8(xs, xt: int, fmt: int, rule: int = RULE_IEEE, header: int = RECORD_HEADER):
    """xs[r] = rank r's tensor; returns out[r], which every rank receives:
    rank r's tensor cast with rank r's own scale and cast back to xt."""
    return [record_decode(record(x, xt, fmt, rule, header), np.asarray(x).size, fmt, xt, header) for x in xs]


def all_to_all_fp8(inputs, xt: int, fmt: int, rule: int = RULE_IEEE):
    """inputs[j][i] = what rank j sends to rank i (each with its own scale);
    returns outputs[i][j] = what rank i receives from rank j."""
    W = len(inputs)
    return [[record_decode(record(inputs[j][i], xt, fmt, rule), np.asarray(inputs[j][i]).size, fmt, xt)
             for j in range(W)] for i in range(W)]


def all_to_all_single_fp8(inputs, xt: int, fmt: int, rule: int = RULE_IEEE):
    """inputs[j] = rank j's whole tensor (flat, numel divisible by the rank
    count), cast with ONE scale; rank i receives chunk i of every sender's
    codes and decodes each with that sender's scale_inv.  Returns
    outputs[i], the concatenation over senders j."""
    W = len(inputs)
    casts = [cast_per_tensor(x, xt, fmt, rule=rule) for x in inputs]
    out = []
    for i in range(W):
        parts = []
        for j in range(W):
            q, s = casts[j]
            c = q.size // W
            parts.append(cast_from_fp8(q[i * c:(i + 1) * c].reshape(1, c), s, GRAN_TENSOR, fmt, yt=xt).reshape(-1))
        out.append(np.concatenate(parts))
    return out


def scaled_mm(a: np.ndarray, fa: int, b: np.ndarray, fb: int, sa: float, sb: float, bias=None, rows=None,
              threads: int = 1) -> np.ndarray:
    """ColossalAI linear_fp8 forward (torch._scaled_mm with per-tensor scales):
    a[M, K] and b[N, K] fp8 codes; returns out[M, N] in float64 (rows outside
    `rows` are zero)."""
    a = np.ascontiguousarray(a, dtype=np.uint8)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    M, K = a.shape
    N, K2 = b.shape
    if K != K2:
        raise ValueError("a and b need the same K")
    out = np.zeros((M, N), np.float64)
    bp = None
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float64)
        bp = ctypes.c_void_p(bias.ctypes.data)
    r0, r1 = rows if rows is not None else (0, M)
    L = lib()
    _run(lambda x, y: _check(L.orc_scaled_mm(_ptr(a), fa, _ptr(b), fb, M, N, K, ctypes.c_float(sa),
                                             ctypes.c_float(sb), bp, _ptr(out), x, y), "scaled_mm"),
         r0, r1, threads)
    return out


def scaled_mm_blockwise(a: np.ndarray, fa: int, sa: np.ndarray, b: np.ndarray, fb: int, sb: np.ndarray,
                        group: int = 128, block: int = 128, bias=None, rows=None, threads: int = 1) -> np.ndarray:
    """DeepEP per-token activations times a DeepSeek-V3 block-scaled weight:
    a[M, K] codes with sa[M, ceil(K/group)], b[N, K] codes with
    sb[ceil(N/block), ceil(K/block)]; returns out[M, N] in float64, the
    product of the exactly dequantised operands (rows outside `rows` zero)."""
    a = np.ascontiguousarray(a, dtype=np.uint8)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    M, K = a.shape
    N, K2 = b.shape
    if K != K2:
        raise ValueError("a and b need the same K")
    if sa.shape != (M, -(-K // group)) or sb.shape != (-(-N // block), -(-K // block)):
        raise ValueError("scale shapes do not match the operands")
    out = np.zeros((M, N), np.float64)
    bp = None
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float64)
        bp = ctypes.c_void_p(bias.ctypes.data)
    r0, r1 = rows if rows is not None else (0, M)
    L = lib()
    _run(lambda x, y: _check(L.orc_scaled_mm_blockwise(_ptr(a), fa, _ptr(sa), group, _ptr(b), fb, _ptr(sb), block,
                                                       M, N, K, bp, _ptr(out), x, y), "scaled_mm_blockwise"),
         r0, r1, threads)
    return out


def _out_array(M: int, N: int, yt: int) -> np.ndarray:
    return np.zeros((M, N), np.float32 if yt == F32 else np.uint16)


def scaled_mm_rounded(a: np.ndarray, fa: int, b: np.ndarray, fb: int, sa: float, sb: float, bias=None,
                      yt: int = BF16, rows=None, threads: int = 1) -> np.ndarray:
    """The per-tensor product with the library's fp32 epilogue, d = T(fl(fl(acc * fl(sa * sb)) + bias)),
    acc the exact sum rounded once to fp32.  bias: fp32 values or None.  Returns float32 (yt = F32) or
    the uint16 bit patterns of bf16 / fp16."""
    a = np.ascontiguousarray(a, dtype=np.uint8)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b need the same K")
    out = _out_array(M, N, yt)
    bp = None
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float32)
        bp = ctypes.c_void_p(bias.ctypes.data)
    r0, r1 = rows if rows is not None else (0, M)
    L = lib()
    _run(lambda x, y: _check(L.orc_scaled_mm_rounded(_ptr(a), fa, _ptr(b), fb, M, N, K, ctypes.c_float(sa),
                                                     ctypes.c_float(sb), bp, yt, _ptr(out), x, y),
                             "scaled_mm_rounded"), r0, r1, threads)
    return out


def scaled_mm_blockwise_rounded(a: np.ndarray, fa: int, sa: np.ndarray, b: np.ndarray, fb: int, sb: np.ndarray,
                                block: int = 128, bias=None, yt: int = BF16, rows=None,
                                threads: int = 1) -> np.ndarray:
    """The fine-grained product with the library's fp32 rounding: acc = fma(acc_kb, fl(sa * sb), acc)
    over 128-deep k-blocks in order, d = T(fl(acc + bias)); activation groups and weight blocks are
    both `block` wide."""
    a = np.ascontiguousarray(a, dtype=np.uint8)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    M, K = a.shape
    N = b.shape[0]
    kb = -(-K // block)
    if b.shape[1] != K or sa.shape != (M, kb) or sb.shape != (-(-N // block), kb):
        raise ValueError("operand or scale shapes do not match")
    out = _out_array(M, N, yt)
    bp = None
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float32)
        bp = ctypes.c_void_p(bias.ctypes.data)
    r0, r1 = rows if rows is not None else (0, M)
    L = lib()
    _run(lambda x, y: _check(L.orc_scaled_mm_blockwise_rounded(_ptr(a), fa, _ptr(sa), _ptr(b), fb, _ptr(sb),
                                                               block, M, N, K, bp, yt, _ptr(out), x, y),
                             "scaled_mm_blockwise_rounded"), r0, r1, threads)
    return out


def transpose_u8(src: np.ndarray, ld: int = None) -> np.ndarray:
    """ColossalAI _LinearFp8.backward's .t().contiguous() of fp8 codes: src[rows, cols]
    -> dst[cols, ld] with dst[c, r] = src[r, c] and zeros for rows <= r < ld."""
    src = np.ascontiguousarray(src, dtype=np.uint8)
    rows, cols = src.shape
    ld = rows if ld is None else ld
    dst = np.full((cols, ld), 0xA5, np.uint8)
    _check(lib().orc_transpose_u8(_ptr(src), rows, cols, _ptr(dst), ld), "transpose_u8")
    return dst


def sum_rows(x: np.ndarray, xt: int) -> np.ndarray:
    """out_grad.sum(0) of x[rows, cols] (bit patterns of type xt), in float64."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = np.zeros((cols,), np.float64)
    _check(lib().orc_sum_rows(_ptr(x), xt, rows, cols, _ptr(out)), "sum_rows")
    return out
