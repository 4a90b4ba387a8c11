"""Device-side test helpers: move numpy bit patterns to and from CUDA tensors,
and allocate outputs inside guard regions so that any write outside a
tensor's bytes is caught (compute-sanitizer is not available)."""
from __future__ import annotations

import os

import numpy as np
import torch

GUARD = 4096            # bytes of canary before and after every guarded output
CANARY = 0xA5

THREADS = max(1, min(32, os.cpu_count() or 1))


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    """numpy array -> CUDA tensor with the same bytes.  uint16 arrays become bf16
    (or `dtype`, e.g. torch.float16); uint8 stays uint8; float32 stays float32."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(dtype or torch.bfloat16)
    else:
        t = torch.from_numpy(a)
        if dtype is not None:
            t = t.view(dtype)
    return t.cuda()


def host(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> numpy array of its bits (uint8 / uint16 / float32)."""
    t = t.detach().contiguous().cpu()
    if t.element_size() == 1:
        return t.view(torch.uint8).numpy()
    if t.element_size() == 2:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.view(torch.float32).numpy()


class Guarded:
    """A CUDA tensor of `numel` elements of `dtype` placed between canary bytes,
    optionally at a byte offset (to test unaligned pointers)."""

    def __init__(self, numel: int, dtype: torch.dtype, offset: int = 0, device="cuda"):
        esz = torch.empty((), dtype=dtype).element_size()
        self.nbytes = numel * esz
        self.offset = offset
        self.raw = torch.full((GUARD + offset + self.nbytes + GUARD,), CANARY, dtype=torch.uint8, device=device)
        body = self.raw[GUARD + offset: GUARD + offset + self.nbytes]
        self.t = body.view(dtype) if numel > 0 else torch.empty((0,), dtype=dtype, device=device)

    def check(self):
        torch.cuda.synchronize()
        r = self.raw.cpu().numpy()
        head = r[: GUARD + self.offset]
        tail = r[GUARD + self.offset + self.nbytes:]
        assert (head == CANARY).all(), "write before the start of an output tensor"
        assert (tail == CANARY).all(), "write past the end of an output tensor"


def offset_input(a: np.ndarray, offset_bytes: int, dtype=None) -> torch.Tensor:
    """A CUDA tensor holding `a` that starts `offset_bytes` past a 256-byte boundary."""
    a = np.ascontiguousarray(a)
    raw = torch.zeros(a.nbytes + offset_bytes + 256, dtype=torch.uint8, device="cuda")
    body = raw[offset_bytes: offset_bytes + a.nbytes]
    body.copy_(torch.from_numpy(a.view(np.uint8).reshape(-1)).cuda())
    if a.dtype == np.uint16:
        return body.view(dtype or torch.bfloat16).view(a.shape)
    if a.dtype == np.float32:
        return body.view(torch.float32).view(a.shape)
    return body.view(a.shape)
