"""Seeded synthetic inputs for scaled FP8 casting.

This module is shared by the tests (which feed the same bytes to the CUDA
library and to the CPU oracle) and by the benchmark.  It holds none of the
method's arithmetic: it only draws random numbers, places them into the
shapes and value distributions of the workloads, and narrows fp32 draws to
bf16/fp16 storage with torch's CPU cast (input plumbing, not the method).

Workloads (shapes and value mixes of the pages' use cases):

* ``c1`` per-token small: bf16 x[128, 1024] ~ N(0, 1); row 3 all +0; row 7
  has element (7, 517) multiplied by 1000.  Seed 20261201.
* ``c2`` per-token activations: bf16 x[4096, 7168]; row r = N(0, 1) * m_r
  with m_r = exp(N(0, 2^2)) (lognormal, sigma 2); 0.1 % of the entries, at
  uniformly drawn distinct positions, replaced by +-50 * m_r with a random
  sign.  Seed 20261202.
* ``c3`` block dequant: W[7168, 18432] fp8 e4m3fn codes drawn uniformly over
  the 254 finite codes (both zeros included); s[56, 144] = exp(N(-8, 1)).
  Seed 20261203.
* ``c4a`` per-channel: bf16 X[8192, 8192] = N(0, 1) * 10^u_r, u_r evenly
  spaced over [-3, 3] across rows then row order shuffled; row 4096 all +0.
  Seed 20261241.
* ``c4b`` per-tensor: fp32 v[64 Mi] ~ N(0, sigma = 1e-2).  Seed 20261242.
* ``c4c`` per-tensor zero: fp16 [1 Mi] all +0.  Seed 20261243 (unused).
* ``device_normal`` / ``device_codes``: inputs above 2^32 elements (the
  64-bit indexing cases), drawn on the device by torch's seeded CUDA
  generator in chunks, because the host cannot draw them in seconds.  The
  tests copy sampled rows back for the oracle.
* ``mm`` fp8 products: the weight W[18432, 7168] (the DeepSeek-V3 MLP gate /
  up projection shape, [out features][in features], the transpose of c3's
  shape) with codes uniform over the finite e4m3fn codes and 128 x 128 block
  scales s[144, 56] = exp(N(-8, 1)); the activations are c2's x quantised
  per token (1 x 128 groups).  Seed 20261206.
* ``c5`` ragged MoE dequant: 64 weights [2048, 7168] then 8 weights
  [7000, 1000]; codes uniform over the finite e4m3fn codes; ceil-sized
  scales exp(N(-8, 1)).  Weight i draws from seed (20261205, i) so any
  weight can be regenerated alone.
"""
from __future__ import annotations

import numpy as np
import torch

SEED_BASE = 20261200

C1_SHAPE = (128, 1024)
C2_SHAPE = (4096, 7168)
C3_SHAPE = (7168, 18432)
C4A_SHAPE = (8192, 8192)
C4B_NUMEL = 64 * 1024 * 1024
C4C_NUMEL = 1024 * 1024
C5_SHAPES = [(2048, 7168)] * 64 + [(7000, 1000)] * 8
MM_W_SHAPE = (18432, 7168)
BLOCK = 128
GROUP = 128


def rng(seed) -> np.random.Generator:
    return np.random.default_rng(seed)


def to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Store fp32 draws as bf16 (torch CPU cast); returns the uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def to_f16_bits(v: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(v, dtype=np.float32).astype(np.float16).view(np.uint16)


def finite_e4m3fn_codes() -> np.ndarray:
    """All 254 fp8 e4m3fn codes that are not NaN (S.1111.111 is NaN)."""
    return np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def finite_e5m2_codes() -> np.ndarray:
    """All 248 fp8 e5m2 codes that are not NaN (exponent field 31 with a nonzero mantissa)."""
    return np.array([c for c in range(256) if (c & 0x7C) != 0x7C or (c & 0x03) == 0], dtype=np.uint8)


def uniform_codes(g: np.random.Generator, shape, codes: np.ndarray) -> np.ndarray:
    idx = g.integers(0, codes.size, size=shape, dtype=np.int64 if codes.size > 255 else np.uint8)
    return codes[idx]


def lognormal_scales(g: np.random.Generator, shape, mu: float = -8.0, sigma: float = 1.0) -> np.ndarray:
    return np.exp(g.normal(mu, sigma, size=shape)).astype(np.float32)


def scale_shape(M: int, N: int, block: int = BLOCK):
    return ((M + block - 1) // block, (N + block - 1) // block)


# ---------------------------------------------------------------------------
# workload generators (return uint16 bf16/fp16 bits, fp32 arrays or uint8 codes)
# ---------------------------------------------------------------------------
def c1_x() -> np.ndarray:
    g = rng(SEED_BASE + 1)
    v = g.standard_normal(C1_SHAPE, dtype=np.float32)
    v[3, :] = 0.0
    v[7, 517] *= np.float32(1000.0)
    return to_bf16_bits(v)


def c2_x() -> np.ndarray:
    g = rng(SEED_BASE + 2)
    m, n = C2_SHAPE
    mag = np.exp(g.normal(0.0, 2.0, size=m)).astype(np.float32)
    v = g.standard_normal((m, n), dtype=np.float32)
    v *= mag[:, None]
    k = int(round(0.001 * m * n))
    pos = g.choice(m * n, size=k, replace=False)
    sign = np.where(g.integers(0, 2, size=k) == 1, np.float32(1.0), np.float32(-1.0))
    v.reshape(-1)[pos] = sign * np.float32(50.0) * mag[pos // n]
    return to_bf16_bits(v)


def c3_w_s():
    g = rng(SEED_BASE + 3)
    M, N = C3_SHAPE
    w = uniform_codes(g, (M, N), finite_e4m3fn_codes())
    s = lognormal_scales(g, scale_shape(M, N))
    return w, s


def mm_w_s():
    g = rng(SEED_BASE + 6)
    N, K = MM_W_SHAPE
    w = uniform_codes(g, (N, K), finite_e4m3fn_codes())
    s = lognormal_scales(g, scale_shape(N, K))
    return w, s


def c4a_x() -> np.ndarray:
    g = rng(SEED_BASE + 41)
    R, C = C4A_SHAPE
    u = np.linspace(-3.0, 3.0, R)
    g.shuffle(u)
    rowmag = np.power(10.0, u).astype(np.float32)
    v = g.standard_normal((R, C), dtype=np.float32)
    v *= rowmag[:, None]
    v[4096, :] = 0.0
    return to_bf16_bits(v)


def c4b_v() -> np.ndarray:
    g = rng(SEED_BASE + 42)
    return (g.standard_normal(C4B_NUMEL, dtype=np.float32) * np.float32(1e-2)).astype(np.float32)


def c4c_v() -> np.ndarray:
    return np.zeros(C4C_NUMEL, dtype=np.uint16)  # fp16 +0 bit pattern


def c5_weight(i: int):
    M, N = C5_SHAPES[i]
    g = rng([SEED_BASE + 5, i])
    w = uniform_codes(g, (M, N), finite_e4m3fn_codes())
    s = lognormal_scales(g, scale_shape(M, N))
    return w, s


# ---------------------------------------------------------------------------
# device-side draws for the largest sizes
# ---------------------------------------------------------------------------
_CHUNK = 1 << 27


def device_normal(shape, seed: int, dtype=torch.bfloat16, device="cuda", row_scale: bool = True,
                  std: float = 1.0) -> torch.Tensor:
    """N(0, std) draws of `shape` stored as `dtype`, made on the device by a
    torch.Generator seeded with `seed`, 128 Mi elements at a time.  With
    row_scale (2-D shapes), row r is multiplied by 2^((r mod 17) - 8), so
    that rows far apart differ in magnitude and an index that wraps lands
    on visibly different data."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    cols = shape[-1] if len(shape) == 2 else n
    for a in range(0, n, _CHUNK):
        b = min(n, a + _CHUNK)
        v = torch.randn(b - a, generator=g, device=device, dtype=torch.float32) * std
        if row_scale and len(shape) == 2:
            r = torch.arange(a, b, device=device, dtype=torch.int64) // cols
            v *= torch.exp2((r % 17 - 8).to(torch.float32))
        flat[a:b] = v.to(dtype)
    return out


def device_codes(shape, seed: int, device="cuda") -> torch.Tensor:
    """fp8 e4m3fn codes uniform over the 254 finite codes, drawn on the
    device by a torch.Generator seeded with `seed`."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = torch.empty(shape, dtype=torch.uint8, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for a in range(0, n, _CHUNK):
        b = min(n, a + _CHUNK)
        k = torch.randint(0, 254, (b - a,), generator=g, device=device, dtype=torch.int32)
        k = k + (k >= 0x7F).to(torch.int32)               # skip 0x7F; 0xFF is never reached
        flat[a:b] = k.to(torch.uint8)
    return out
