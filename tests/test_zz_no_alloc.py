"""The allocation-free per-tensor cast (fp8q_cast_per_tensor_noalloc).

Some callers cannot allocate device memory -- an allocator owns all of the
GPU, or cudaMalloc is off limits because it can synchronise the device -- so
this entry point keeps its scratch in a static array inside the library
instead of taking a workspace.  These tests call it through the C ABI and
require the same bytes as the workspace entry point, bit for bit, on two
calls in a row (the second must not see anything the first left in the
shared array).  The file sorts last so that a run stopping at the first
failure has already run every other test; it also passes on its own."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, BF16 = 0, 2


def _c_noalloc(lib):
    f = lib.fp8q_cast_per_tensor_noalloc
    p = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, p, p, p]
    return f


def _reference(fp8q, x, fmt):
    q = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    s = torch.empty(1, dtype=torch.float32, device=x.device)
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device=x.device)
    fp8q.fp8q_cast_per_tensor(x, q, s, ws, fmt)
    return q, s


def _noalloc(lib, x, xt, fmt):
    f = _c_noalloc(lib)
    q = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    s = torch.empty(1, dtype=torch.float32, device=x.device)
    st = f(x.data_ptr(), xt, x.numel(), fmt, q.data_ptr(), s.data_ptr(),
           torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.fp8q_status_string(st)
    return q, s


def _same(a, b):
    torch.cuda.synchronize()
    return bool(torch.equal(a[0], b[0])) and bool(torch.equal(a[1].view(torch.int32), b[1].view(torch.int32)))


def test_noalloc_matches_workspace_entry_point_twice(fp8q):
    lib = fp8q.lib()
    g = np.random.default_rng(2026)
    # first call: a large fp32 tensor with a large amax; second: a small bf16
    # tensor with a tiny amax, so stale partials from the first would show
    big = torch.from_numpy((g.standard_normal(64 << 20) * 100).astype(np.float32)).cuda()
    small = torch.from_numpy((g.standard_normal(300_001) * 1e-3).astype(np.float32)).to(torch.bfloat16).cuda()
    for x, xt, fmt in ((big, F32, E5M2), (small, BF16, E4M3FN)):
        assert _same(_noalloc(lib, x, xt, fmt), _reference(fp8q, x, fmt))


def test_noalloc_allocates_no_device_memory(fp8q):
    """The point of the entry point: repeated calls leave the device's free memory unchanged.
    Every tensor is allocated and one warm-up call made (it loads the kernels and looks up the
    scratch address) before the free bytes are read."""
    lib = fp8q.lib()
    f = _c_noalloc(lib)
    x = torch.randn(3_000_000, device="cuda")
    q = torch.empty(x.numel(), dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream

    def call():
        st = f(x.data_ptr(), F32, x.numel(), E4M3FN, q.data_ptr(), s.data_ptr(), stream)
        assert st == 0, lib.fp8q_status_string(st)

    call()
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(8):
        call()
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before


def test_noalloc_binding_and_errors(fp8q):
    x = torch.ones(1000, dtype=torch.float16, device="cuda")
    x[17] = -7.0
    q = torch.empty(1000, dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    fp8q.fp8q_cast_per_tensor_noalloc(x, q, s, E4M3FN)
    assert _same((q, s), _reference(fp8q, x, E4M3FN))
    f = _c_noalloc(fp8q.lib())
    assert f(x.data_ptr(), 9, 1000, E4M3FN, q.data_ptr(), s.data_ptr(), None) == 2       # bad dtype
    assert f(x.data_ptr(), 1, 1000, 5, q.data_ptr(), s.data_ptr(), None) == 3            # bad format
    assert f(None, 1, 1000, E4M3FN, q.data_ptr(), s.data_ptr(), None) == 1               # null input
    e = torch.zeros(1, dtype=torch.float32, device="cuda")
    assert f(None, 1, 0, E4M3FN, None, e.data_ptr(), None) == 0                         # empty tensor
    torch.cuda.synchronize()
    assert e.item() == 1.0
