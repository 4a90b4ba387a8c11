"""The C-ABI library loads on a machine without a GPU, exports every entry
point that include/fp8q.h declares, and rejects bad arguments on the host
before any CUDA call (no compute is attempted here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8q_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from dequantisation_fp8q_token_b200 import build
    build.build()
    import dequantisation_fp8q_token_b200 as fp8q
    return fp8q.lib()


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), f"{n} declared in fp8q.h but not exported"


def test_binding_names_match_the_c_names():
    import dequantisation_fp8q_token_b200 as fp8q
    for n in declared_functions():
        assert hasattr(fp8q, n), f"binding lacks {n}"


def test_enum_values_match_the_binding():
    import dequantisation_fp8q_token_b200 as fp8q
    src = open(HEADER).read()
    for name, val in [("FP8Q_SCALE_IEEE", fp8q.SCALE_IEEE), ("FP8Q_SCALE_TORCH", fp8q.SCALE_TORCH),
                      ("FP8Q_E4M3FN", fp8q.E4M3FN), ("FP8Q_E5M2", fp8q.E5M2), ("FP8Q_F32", fp8q.F32),
                      ("FP8Q_F16", fp8q.F16), ("FP8Q_BF16", fp8q.BF16), ("FP8Q_GRAN_TENSOR", fp8q.GRAN_TENSOR),
                      ("FP8Q_GRAN_ROW", fp8q.GRAN_ROW), ("FP8Q_GRAN_GROUP", fp8q.GRAN_GROUP),
                      ("FP8Q_GRAN_BLOCK", fp8q.GRAN_BLOCK), ("FP8Q_RECORD_PACKED4", fp8q.RECORD_PACKED4),
                      ("FP8Q_RECORD_ALIGNED16", fp8q.RECORD_ALIGNED16)]:
        assert re.search(rf"\b{name}\s*=\s*{val}\b", src), name


def test_status_strings(L):
    import dequantisation_fp8q_token_b200 as fp8q
    for code in range(11):
        s = fp8q.fp8q_status_string(code)
        assert s.startswith("FP8Q_")
    assert "UNKNOWN" in fp8q.fp8q_status_string(99)
    assert fp8q.fp8q_version() == 10100
    assert fp8q.fp8q_cast_per_tensor_workspace_bytes() == 8192


# host-side validation: each of these returns before the library touches CUDA
P = 0x1000   # a fake, never-dereferenced pointer value


def test_per_token_validation(L):
    f = L.fp8q_per_token_group_quant
    assert f(P, 7, 4, 128, 128, 0, P, P, None) == 2             # dtype
    assert f(P, 2, 4, 128, 128, 9, P, P, None) == 3             # format
    assert f(P, 2, 4, 130, 128, 0, P, P, None) == 4             # n % group
    assert f(P, 2, -1, 128, 128, 0, P, P, None) == 4            # negative size
    assert f(P, 2, 4, 128, 0, 0, P, P, None) == 4               # group < 1
    assert f(None, 2, 4, 128, 128, 0, P, P, None) == 1          # null x
    assert f(P, 2, 4, 128, 128, 0, P, None, None) == 1          # null scale_inv
    assert f(P + 1, 2, 4, 128, 128, 0, P, P, None) == 5         # bf16 pointer on an odd address
    assert f(None, 2, 0, 128, 128, 0, None, None, None) == 0    # empty: nothing to do


def test_per_channel_and_tensor_validation(L):
    assert L.fp8q_cast_per_channel(P, 3, 4, 4, 0, P, P, None) == 2
    assert L.fp8q_cast_per_channel(P, 0, 4, 4, 2, P, P, None) == 3
    assert L.fp8q_cast_per_channel(P, 0, -4, 4, 0, P, P, None) == 4
    assert L.fp8q_cast_per_channel(P, 0, 4, 4, 0, P, None, None) == 1
    assert L.fp8q_cast_per_channel(P + 2, 0, 4, 4, 0, P, P, None) == 5
    assert L.fp8q_cast_per_tensor(P, 0, 16, 0, P, P, None, 8192, None) == 6
    assert L.fp8q_cast_per_tensor(P, 0, 16, 0, P, P, P, 100, None) == 6
    assert L.fp8q_cast_per_tensor(P, 0, 16, 0, P, P, P + 4, 8192, None) == 6
    assert L.fp8q_cast_per_tensor(P, 0, -1, 0, P, P, P, 8192, None) == 4
    assert L.fp8q_cast_per_tensor(None, 0, 16, 0, P, P, P, 8192, None) == 1
    f = L.fp8q_cast_per_tensor_noalloc
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    assert f(P, 5, 16, 0, P, P, None) == 2
    assert f(P, 0, 16, 4, P, P, None) == 3
    assert f(None, 0, 16, 0, P, P, None) == 1
    assert f(P + 1, 0, 16, 0, P, P, None) == 5


def test_scale_rule_validation(L):
    f = L.fp8q_per_token_group_quant_ex
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    assert f(P, 2, 4, 128, 128, 0, P, P, 2, None) == 10
    assert f(P, 2, 4, 128, 128, 0, P, P, -1, None) == 10
    assert f(P, 2, 4, 130, 128, 0, P, P, 1, None) == 4
    g = L.fp8q_cast_per_channel_ex
    g.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    assert g(P, 0, 4, 4, 0, P, P, 7, None) == 10
    h = L.fp8q_cast_per_tensor_ex
    h.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]
    assert h(P, 0, 16, 0, P, P, P, 8192, 3, None) == 10


def test_dequant_validation(L):
    assert L.fp8q_block_dequant(P, 2, 4, 4, P, 128, 0, P, None) == 3
    assert L.fp8q_block_dequant(P, 0, 4, 4, P, 128, 5, P, None) == 2
    assert L.fp8q_block_dequant(P, 0, 4, 4, P, 0, 0, P, None) == 4
    assert L.fp8q_block_dequant(P, 0, -4, 4, P, 128, 0, P, None) == 4
    assert L.fp8q_block_dequant(None, 0, 4, 4, P, 128, 0, P, None) == 1
    assert L.fp8q_block_dequant(P, 0, 4, 4, P + 2, 128, 0, P, None) == 5
    assert L.fp8q_block_dequant_grouped(None, -1, 0, 128, 2, None) == 9
    assert L.fp8q_block_dequant_grouped(None, 0, 0, 128, 2, None) == 0
    assert L.fp8q_block_dequant_grouped(None, 3, 0, 128, 2, None) == 1
    assert L.fp8q_cast_from_fp8(P, 0, 4, 4, P, 4, 0, 2, P, None) == 8
    assert L.fp8q_cast_from_fp8(P, 0, 4, 6, P, 2, 4, 2, P, None) == 4
    assert L.fp8q_cast_from_fp8(P, 0, 4, 8, P, 3, 0, 2, P, None) == 4
    assert L.fp8q_cast_from_fp8(P, 0, 4, 8, None, 1, 0, 2, P, None) == 1


def test_scaled_mm_validation(L):
    f = L.fp8q_scaled_mm
    L.fp8q_scaled_mm.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                 ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                 ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    A = 0x10000   # 16-byte aligned fake pointer
    assert f(A, 0, A, 0, 8, 8, 32, P, P, None, 7, A, None, None) == 2       # output dtype
    assert f(A, 5, A, 0, 8, 8, 32, P, P, None, 2, A, None, None) == 3       # format of a
    assert f(A, 0, A, 4, 8, 8, 32, P, P, None, 2, A, None, None) == 3       # format of b
    assert f(A, 0, A, 0, 8, 8, 24, P, P, None, 2, A, None, None) == 4       # K % 16
    assert f(A, 0, A, 0, -1, 8, 32, P, P, None, 2, A, None, None) == 4      # negative M
    assert f(A, 0, A, 0, 8, 1 << 31, 32, P, P, None, 2, A, None, None) == 4  # N above the limit
    assert f(None, 0, A, 0, 8, 8, 32, P, P, None, 2, A, None, None) == 1    # null a
    assert f(A, 0, A, 0, 8, 8, 32, None, P, None, 2, A, None, None) == 1    # null scale_a
    assert f(A, 0, A, 0, 8, 8, 32, P, P, None, 2, None, None, None) == 1    # null out
    assert f(A + 8, 0, A, 0, 8, 8, 32, P, P, None, 2, A, None, None) == 5   # a not 16-byte aligned
    assert f(A, 0, A, 0, 8, 8, 32, P, P, A + 1, 2, A, None, None) == 5      # bf16 bias on an odd address
    assert f(A, 0, A, 0, 8, 8, 32, P, P, None, 2, A, A + 2, None) == 5      # status word misaligned
    assert f(None, 0, None, 0, 0, 8, 32, None, None, None, 2, None, None, None) == 0   # M == 0: nothing


def test_scaled_mm_blockwise_validation(L):
    f = L.fp8q_scaled_mm_blockwise
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    A = 0x10000
    assert f(A, 0, P, A, 0, P, 8, 8, 128, None, 9, A, None, None) == 2      # output dtype
    assert f(A, 2, P, A, 0, P, 8, 8, 128, None, 2, A, None, None) == 3      # format
    assert f(A, 0, P, A, 0, P, 8, 8, 136 + 1, None, 2, A, None, None) == 4  # K % 16
    assert f(A, 0, None, A, 0, P, 8, 8, 128, None, 2, A, None, None) == 1   # null scale_a
    assert f(A, 0, P, A, 0, None, 8, 8, 128, None, 2, A, None, None) == 1   # null scale_b
    assert f(A, 0, P + 2, A, 0, P, 8, 8, 128, None, 2, A, None, None) == 5  # scale_a misaligned
    assert f(A, 0, P, A, 0, P, 8, 0, 128, None, 2, None, None, None) == 0   # N == 0: nothing


def test_scaled_mm_wait_test_validation(L):
    f = L.fp8q_scaled_mm_wait_test
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]
    A = 0x10000
    assert f(A, A, 8, 8, 24, P, P, A, A, 1000, 0, None) == 4                # K % 16
    assert f(A, A, 8, 8, 0, P, P, A, A, 1000, -1, None) == 4                # K == 0
    assert f(A, A, 8, 8, 128, P, P, A, A, 0, 0, None) == 4                  # no wait limit
    assert f(A, A, 8, 8, 128, P, P, A, A, 5_000_000_000, 0, None) == 4      # limit above 4 s
    assert f(A, A, 8, 8, 128, P, P, A, A, 1000, 1, None) == 4               # stall past the last k-block
    assert f(A, A, 8, 8, 128, P, P, A, A, 1000, -2, None) == 4
    assert f(A, A, 8, 8, 128, P, P, A, None, 1000, 0, None) == 1            # the status word is required
    assert f(A, A, 8, 8, 128, None, P, A, A, 1000, 0, None) == 1            # null scale_a
    assert f(A, A, 8, 8, 128, P, P, A, A + 2, 1000, 0, None) == 5           # status word misaligned

    g = L.fp8q_scaled_mm_blockwise_wait_test
    g.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                  ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]
    assert g(A, P, A, P, 8, 8, 24, A, A, 1000, 0, None) == 4                # K % 16
    assert g(A, P, A, P, 8, 8, 0, A, A, 1000, -1, None) == 4                # K == 0
    assert g(A, P, A, P, 8, 8, 128, A, A, 0, 0, None) == 4                  # no wait limit
    assert g(A, P, A, P, 8, 8, 256, A, A, 1000, 2, None) == 4               # stall past the last k-block
    assert g(A, P, A, P, 8, 8, 128, A, None, 1000, 0, None) == 1            # the status word is required
    assert g(A, None, A, P, 8, 8, 128, A, A, 1000, 0, None) == 1            # null scale_a
    assert g(A, P, A, P + 2, 8, 8, 128, A, A, 1000, 0, None) == 5           # scale_b misaligned

def test_transpose_and_sum_rows_validation(L):
    f = L.fp8q_transpose_fp8
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
    assert f(P, 8, 4, P, 7, None) == 4          # ld < rows
    assert f(P, -1, 4, P, 8, None) == 4         # negative size
    assert f(None, 8, 4, P, 8, None) == 1       # null src
    assert f(P, 8, 4, None, 8, None) == 1       # null dst
    assert f(None, 0, 0, None, 0, None) == 0    # nothing to do
    s = L.fp8q_sum_rows
    s.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    assert s(P, 5, 4, 4, P, None) == 2          # dtype
    assert s(P, 2, -1, 4, P, None) == 4         # negative rows
    assert s(P, 2, 4, 4, None, None) == 1       # null out
    assert s(P + 1, 2, 4, 4, P, None) == 5      # bf16 input on an odd address
    assert s(None, 2, 4, 0, None, None) == 0    # no columns


def test_scaled_mm_ex_validation(L):
    f = L.fp8q_scaled_mm_ex
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    A = 0x10000
    assert f(A, 0, 2, A, 0, 0, 32, 32, 32, P, P, None, 2, A, None, None) == 4     # unknown layout
    assert f(A, 0, 1, A, 0, 0, 24, 32, 32, P, P, None, 2, A, None, None) == 4     # MN-major A needs M % 16
    assert f(A, 0, 0, A, 0, 1, 32, 24, 32, P, P, None, 2, A, None, None) == 4     # MN-major B needs N % 16
    assert f(A, 0, 0, A, 0, 1, 32, 32, 24, P, P, None, 2, A, None, None) == 4     # a K-major operand needs K % 16
    assert f(A, 0, 1, A, 0, 1, 32, 32, 24, None, P, None, 2, A, None, None) == 1  # both MN-major: any K; null scale


def test_binding_fails_loudly_without_the_library(tmp_path):
    """With no libfp8q.so every entry point raises: there is no CPU fallback.  Run in a fresh
    interpreter, pointed at a path where no library exists."""
    import subprocess
    import sys
    code = (
        "import sys, torch\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "import dequantisation_fp8q_token_b200 as f\n"
        f"f._LIB_PATH = {str(tmp_path / 'libfp8q.so')!r}\n"
        "for call in (lambda: f.lib(),\n"
        "             lambda: f.fp8q_version(),\n"
        "             lambda: f.per_token_cast_to_fp8(torch.zeros(4, 128, dtype=torch.bfloat16))):\n"
        "    try:\n"
        "        call()\n"
        "        print('returned')\n"
        "    except Exception as e:\n"
        "        print('raised', type(e).__name__)\n")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = r.stdout.strip().splitlines()
    assert lines[0] == "raised ImportError"
    assert all(line.startswith("raised") for line in lines), r.stdout


def test_sharded_pipeline_and_record_validation(L):
    """Host-side checks of the sharded per-tensor cast, the pipeline cast and the all-gather
    records: every case below stops at a check, before any CUDA call."""
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    A = 0x10000
    WS = L.fp8q_cast_per_tensor_workspace_bytes
    WS.restype, WS.argtypes = sz, []
    ws = WS()
    assert ws >= 4 and ws % 4 == 0

    f = L.fp8q_tensor_amax
    f.argtypes = [vp, i32, i64, vp, vp, sz, vp]
    assert f(A, 9, 8, A, A, ws, None) == 2                  # dtype
    assert f(A, 0, -1, A, A, ws, None) == 4                 # negative numel
    assert f(A, 0, 8, None, A, ws, None) == 1               # null amax word
    assert f(A, 0, 8, A + 2, A, ws, None) == 5              # misaligned amax word
    assert f(None, 0, 8, A, A, ws, None) == 1               # null x
    assert f(A + 2, 0, 8, A, A, ws, None) == 5              # fp32 x on a 2-byte boundary
    assert f(A, 0, 8, A, None, ws, None) == 6               # no workspace
    assert f(A, 0, 8, A, A, ws - 4, None) == 6              # workspace too small
    assert f(A, 0, 8, A, A + 4, ws, None) == 6              # workspace not 16-byte aligned

    f = L.fp8q_cast_per_tensor_with_amax
    f.argtypes = [vp, i32, i64, i32, vp, vp, vp, i32, vp]
    assert f(A, 9, 8, 0, A, A, A, 0, None) == 2             # dtype
    assert f(A, 0, 8, 0, A, A, A, 7, None) == 10            # scale rule
    assert f(A, 0, 8, 5, A, A, A, 0, None) == 3             # format
    assert f(A, 0, -8, 0, A, A, A, 0, None) == 4            # negative numel
    assert f(A, 0, 8, 0, None, A, A, 0, None) == 1          # null amax word
    assert f(A, 0, 8, 0, A, A, None, 0, None) == 1          # null scale_inv
    assert f(A, 0, 8, 0, A + 1, A, A, 0, None) == 5         # misaligned amax word
    assert f(None, 0, 8, 0, A, A, A, 0, None) == 1          # null x of a non-empty shard
    assert f(A, 0, 8, 0, A, None, A, 0, None) == 1          # null q of a non-empty shard

    f = L.fp8q_cast_pipeline
    f.argtypes = [vp, i32, i64, vp, vp, vp, vp, sz, i32, vp]
    assert f(A, 9, 8, A, A, A, A, ws, 0, None) == 2         # dtype
    assert f(A, 0, 8, A, A, A, A, ws, 3, None) == 10        # scale rule
    assert f(A, 0, -1, A, A, A, A, ws, 0, None) == 4        # negative numel
    assert f(A, 0, 8, A, None, A, A, ws, 0, None) == 1      # null scale_inv
    assert f(A, 0, 8, A, A, None, A, ws, 0, None) == 1      # null format tag
    assert f(A, 0, 8, A, A, A + 2, A, ws, 0, None) == 5     # misaligned format tag
    assert f(A, 0, 8, None, A, A, A, ws, 0, None) == 1      # null q
    assert f(A, 0, 8, A, A, A, None, ws, 0, None) == 6      # no workspace

    f = L.fp8q_cast_from_pipeline
    f.argtypes = [vp, i64, vp, vp, i32, vp, vp]
    assert f(A, 8, A, A, 9, A, None) == 2                   # dtype
    assert f(A, -8, A, A, 2, A, None) == 4                  # negative numel
    assert f(None, 0, None, None, 2, None, None) == 0       # empty: nothing to do
    assert f(A, 8, A, None, 2, A, None) == 1                # null format tag
    assert f(A, 8, A, A, 2, A + 1, None) == 5               # bf16 output on an odd address

    rb = L.fp8q_record_bytes
    rb.restype, rb.argtypes = sz, [i64]
    assert [rb(n) for n in (0, 1, 16, 17, 4096)] == [16, 32, 32, 48, 4112]
    assert rb(-1) == 0

    f = L.fp8q_pack_record
    f.argtypes = [vp, i32, i64, i32, vp, vp, sz, i32, vp]
    assert f(A, 9, 8, 0, A, A, ws, 0, None) == 2            # dtype
    assert f(A, 0, 8, 0, A, A, ws, 5, None) == 10           # scale rule
    assert f(A, 0, 8, 4, A, A, ws, 0, None) == 3            # format
    assert f(A, 0, -8, 0, A, A, ws, 0, None) == 4           # negative numel
    assert f(A, 0, 8, 0, None, A, ws, 0, None) == 1         # null record
    assert f(A, 0, 8, 0, A + 8, A, ws, 0, None) == 5        # record not 16-byte aligned
    # the cast's own checks come before the header is zeroed, so none of these enqueues anything
    assert f(None, 0, 8, 0, A, A, ws, 0, None) == 1         # null x
    assert f(A + 2, 0, 8, 0, A, A, ws, 0, None) == 5        # fp32 x on a 2-byte boundary
    assert f(A, 0, 8, 0, A, None, ws, 0, None) == 6         # no workspace

    f = L.fp8q_unpack_records
    f.argtypes = [vp, i32, i64, i32, i32, vp, vp]
    assert f(A, 2, 8, 7, 2, A, None) == 3                   # format
    assert f(A, 2, 8, 0, 9, A, None) == 2                   # dtype
    assert f(A, -1, 8, 0, 2, A, None) == 9                  # negative count
    assert f(A, 2, -8, 0, 2, A, None) == 4                  # negative numel
    assert f(None, 0, 8, 0, 2, None, None) == 0             # no records: nothing to do
    assert f(None, 2, 8, 0, 2, A, None) == 1                # null records
    assert f(A + 8, 2, 8, 0, 2, A, None) == 5               # records not 16-byte aligned

    # the two record layouts (4: the page's packed [scale | codes]; 16: aligned)
    rb = L.fp8q_record_bytes_ex
    rb.restype, rb.argtypes = sz, [i64, i32]
    assert [rb(n, 4) for n in (0, 1, 16, 17)] == [4, 5, 20, 21]
    assert [rb(n, 16) for n in (0, 1, 16, 17)] == [16, 32, 32, 48]
    assert rb(8, 8) == 0 and rb(-1, 4) == 0                 # unknown layout, negative numel

    f = L.fp8q_pack_record_ex
    f.argtypes = [vp, i32, i64, i32, vp, vp, sz, i32, i32, vp]
    assert f(A, 0, 8, 0, A, A, ws, 0, 8, None) == 4         # unknown layout
    assert f(A, 0, 8, 0, A + 2, A, ws, 0, 4, None) == 5     # packed record: its scale must be 4-byte aligned
    assert f(A, 0, 8, 0, A + 4, A, ws, 0, 16, None) == 5    # aligned record: 16-byte aligned
    assert f(None, 0, 8, 0, A + 4, A, ws, 0, 4, None) == 1  # packed, 4-byte aligned: on to the cast's checks

    f = L.fp8q_unpack_records_ex
    f.argtypes = [vp, i32, i64, i32, i32, vp, i32, vp]
    assert f(A, 2, 8, 0, 2, A, 8, None) == 4                # unknown layout
    assert f(A + 2, 2, 8, 0, 2, A, 4, None) == 5            # packed records not 4-byte aligned
    assert f(A, 2, 6, 0, 2, A, 4, None) == 5                # record 1's scale at 4 + 6 bytes
    assert f(None, 2, 8, 0, 2, A, 4, None) == 1             # null records


def test_status_strings_and_version(L):
    L.fp8q_status_string.restype = ctypes.c_char_p
    L.fp8q_status_string.argtypes = [ctypes.c_int]
    names = [L.fp8q_status_string(i).decode() for i in range(11)]
    assert names[0] == "FP8Q_OK"
    assert all(n.startswith("FP8Q_ERR_") for n in names[1:])
    assert len(set(names)) == 11
    assert L.fp8q_status_string(99).decode() == "FP8Q_ERR_UNKNOWN"
    L.fp8q_version.restype = ctypes.c_int
    v = L.fp8q_version()
    assert v >= 10000 and v % 100 < 100


def test_every_python_entry_point_refuses_host_tensors(L):
    """No CPU fallback anywhere in the binding: given host tensors, every public helper raises
    because its tensors are not CUDA tensors, before the C library is called."""
    import torch
    import dequantisation_fp8q_token_b200 as f
    bf, u8, f32, i32 = torch.bfloat16, torch.uint8, torch.float32, torch.int32
    x = torch.zeros(4, 256, dtype=bf)
    q = torch.zeros(4, 256, dtype=u8)
    s2 = torch.ones(4, 2, dtype=f32)
    s1 = torch.ones(1, dtype=f32)
    sr = torch.ones(4, dtype=f32)
    ws = torch.zeros(f.fp8q_cast_per_tensor_workspace_bytes(), dtype=u8)
    y = torch.zeros(4, 256, dtype=bf)
    w = torch.zeros(256, 256, dtype=u8)
    sw = torch.ones(2, 2, dtype=f32)
    yw = torch.zeros(256, 256, dtype=bf)
    a8 = torch.zeros(16, 256, dtype=torch.float8_e4m3fn)
    b8 = torch.zeros(32, 256, dtype=torch.float8_e4m3fn)
    out = torch.zeros(16, 32, dtype=bf)
    tag = torch.zeros(1, dtype=i32)
    rec = torch.zeros(f.record_bytes(x.numel()), dtype=u8)
    calls = {
        "fp8q_per_token_group_quant": lambda: f.fp8q_per_token_group_quant(x, q, s2, 128),
        "per_token_cast_to_fp8": lambda: f.per_token_cast_to_fp8(x),
        "per_token_cast_back": lambda: f.per_token_cast_back(q.view(torch.float8_e4m3fn), s2),
        "fp8q_cast_per_channel": lambda: f.fp8q_cast_per_channel(x, q, sr),
        "fp8q_cast_per_tensor": lambda: f.fp8q_cast_per_tensor(x, q, s1, ws),
        "fp8q_cast_per_tensor_noalloc": lambda: f.fp8q_cast_per_tensor_noalloc(x, q, s1),
        "fp8q_tensor_amax": lambda: f.fp8q_tensor_amax(x, tag, ws),
        "fp8q_cast_per_tensor_with_amax": lambda: f.fp8q_cast_per_tensor_with_amax(x, tag, q, s1),
        "cast_to_fp8": lambda: f.cast_to_fp8(x),
        "cast_from_fp8": lambda: f.cast_from_fp8(q.view(torch.float8_e4m3fn), s1, bf),
        "fp8q_cast_pipeline": lambda: f.fp8q_cast_pipeline(x, q, s1, tag, ws),
        "fp8q_cast_from_pipeline": lambda: f.fp8q_cast_from_pipeline(q, s1, tag, y),
        "fp8q_block_dequant": lambda: f.fp8q_block_dequant(w, sw, yw, 128),
        "fp8q_block_dequant_grouped": lambda: f.fp8q_block_dequant_grouped([w], [sw], [yw], 128),
        "weight_dequant": lambda: f.weight_dequant(w.view(torch.float8_e4m3fn), sw),
        "fp8q_cast_from_fp8": lambda: f.fp8q_cast_from_fp8(q, s2, y, f.GRAN_GROUP, 128),
        "fp8q_pack_record": lambda: f.fp8q_pack_record(x, rec, ws),
        "fp8q_unpack_records": lambda: f.fp8q_unpack_records(rec, 1, x.numel(), y),
        "fp8q_pack_record_ex": lambda: f.fp8q_pack_record_ex(x, rec, ws, layout=f.RECORD_PACKED4),
        "fp8q_unpack_records_ex": lambda: f.fp8q_unpack_records_ex(rec, 1, x.numel(), y, layout=f.RECORD_PACKED4),
        "fp8q_scaled_mm": lambda: f.fp8q_scaled_mm(a8, b8, s1, s1, out),
        "fp8q_scaled_mm_ex": lambda: f.fp8q_scaled_mm_ex(a8, b8, s1, s1, out),
        "fp8q_scaled_mm_blockwise": lambda: f.fp8q_scaled_mm_blockwise(
            a8, torch.ones(16, 2, dtype=f32), b8, torch.ones(1, 2, dtype=f32), out),
        "scaled_mm": lambda: f.scaled_mm(a8, b8.t(), s1, s1),
        "fp8q_transpose_fp8": lambda: f.fp8q_transpose_fp8(w, torch.zeros(256, 256, dtype=u8)),
        "transpose_fp8": lambda: f.transpose_fp8(w),
        "fp8q_sum_rows": lambda: f.fp8q_sum_rows(y, torch.zeros(256, dtype=bf)),
        "linear_fp8": lambda: f.linear_fp8(torch.zeros(16, 256, dtype=bf), torch.zeros(32, 256, dtype=bf)),
    }
    did_not_refuse = {}
    for name, call in calls.items():
        try:
            call()
            did_not_refuse[name] = "returned"
        except Exception as e:   # the refusal is a ValueError naming the CUDA requirement
            if "CUDA" not in str(e):
                did_not_refuse[name] = f"{type(e).__name__}: {e}"
    assert not did_not_refuse, did_not_refuse


def test_binding_refuses_a_device_other_than_the_current_one(monkeypatch):
    """The library sizes launches (and picks the allocation-free cast's static scratch) from the
    current device, so the binding refuses tensors on any other device before calling it.  Every
    call into the library takes its stream from the one helper that checks this."""
    import inspect
    import torch
    import dequantisation_fp8q_token_b200 as f
    monkeypatch.setattr(f, "_current_device", lambda: 0)      # the helper the binding reads it with
    with pytest.raises(ValueError, match="current device"):
        f._stream(None, torch.device("cuda", 1))
    src = inspect.getsource(f)
    no_stream = {"fp8q_status_string", "fp8q_version", "fp8q_cast_per_tensor_workspace_bytes",
                 "fp8q_record_bytes", "fp8q_record_bytes_ex"}
    checked = 0
    for m in re.finditer(r"lib\(\)\.(fp8q_\w+)\(", src):
        name = m.group(1)
        depth, i = 1, m.end()
        while depth:                       # the call's argument list, to its matching parenthesis
            depth += {"(": 1, ")": -1}.get(src[i], 0)
            i += 1
        args = src[m.end():i]
        if name not in no_stream:
            assert "_stream(stream, dev)" in args, name
            checked += 1
    assert checked >= 15
