// quant_scaled.cu -- ColossalAI-style cast_to_fp8 (colossalai/quantization/fp8.py):
//   per-channel: one scale per row, amax := amax > 0 ? amax : 1,
//                scale = FMAX / amax, scale_inv = amax / FMAX;
//   per-tensor:  one scale for all elements, scale_inv = 1 / scale.
//
// Per-channel: one CTA per row.  A row of up to kChThreads * 8 16-byte
// vectors (32 KiB; 8192 bf16 needs 4 per thread) is loaded once into
// registers, reduced (integer max on magnitude bits, warp shuffles, then a
// shared-memory step across warps), and cast from the same registers, so x
// is read exactly once.  Longer rows re-read the row (from L2) for the cast.
//
// Per-tensor: two kernels, no grid barrier and no atomics.  Pass 1 writes one
// magnitude-bits maximum per CTA into the caller's workspace; pass 2 has
// every CTA reduce those partials (a few KiB from L2), derive the scale and
// cast.  Pass 2 walks the tensor from the end, so its first reads hit the
// part of x that pass 1 left in L2.
#include "fp8q_device.cuh"
#include "fp8q_internal.h"

namespace fp8q {
namespace {

constexpr int kChThreads = 256;
constexpr int kPtThreads = 256;
constexpr int kPtUnroll = 4;

__device__ __forceinline__ uint32_t block_max_u32(uint32_t m, uint32_t* sh) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) sh[warp] = m;
    __syncthreads();
    m = 0u;
    const int nw = blockDim.x >> 5;
    for (int w = 0; w < nw; ++w) m = max(m, sh[w]);
    return m;
}

template <int XT, int FMT, bool FIX>
__device__ __forceinline__ void encode_store(uint4 v, float scale, uint8_t* dst) {
    if (XT == kF32) {
        const float f0 = __fmul_rn(__uint_as_float(v.x), scale);
        const float f1 = __fmul_rn(__uint_as_float(v.y), scale);
        const float f2 = __fmul_rn(__uint_as_float(v.z), scale);
        const float f3 = __fmul_rn(__uint_as_float(v.w), scale);
        st_u32(dst, enc2_sem<FMT, FIX>(f0, f1) | (enc2_sem<FMT, FIX>(f2, f3) << 16));
    } else {
        float a0, a1, b0, b1, c0, c1, d0, d1;
        widen2<XT>(v.x, a0, a1);
        widen2<XT>(v.y, b0, b1);
        widen2<XT>(v.z, c0, c1);
        widen2<XT>(v.w, d0, d1);
        const uint32_t w0 = enc2_sem<FMT, FIX>(__fmul_rn(a0, scale), __fmul_rn(a1, scale)) |
                            (enc2_sem<FMT, FIX>(__fmul_rn(b0, scale), __fmul_rn(b1, scale)) << 16);
        const uint32_t w1 = enc2_sem<FMT, FIX>(__fmul_rn(c0, scale), __fmul_rn(c1, scale)) |
                            (enc2_sem<FMT, FIX>(__fmul_rn(d0, scale), __fmul_rn(d1, scale)) << 16);
        st_v2(dst, make_uint2(w0, w1));
    }
}

template <int FMT, bool FIX>
__device__ __forceinline__ uint8_t encode_one(float f) {
    return (uint8_t)(enc2_sem<FMT, FIX>(f, 0.0f) & 0xFFu);
}

// ColossalAI scale rule from an fp32 magnitude-bits amax.  `fix` is set when
// the hardware's saturating encode could differ from the non-saturating
// reference: a NaN amax (replaced by 1, so NaN/Inf elements and overflow can
// occur) or a scale that overflowed to Inf (amax < FMAX / FLT_MAX).
template <int FMT>
__device__ __forceinline__ float colossal_scale(uint32_t amax_bits, float& amax_out, bool& fix) {
    const float a = __uint_as_float(amax_bits);
    const float amax = a > 0.0f ? a : 1.0f;
    const float scale = __fdiv_rn(fp8_max<FMT>(), amax);
    fix = (amax_bits > 0x7F800000u) || isinf(scale);
    amax_out = amax;
    return scale;
}

// ---------------------------------------------------------------------------
// per-channel
// ---------------------------------------------------------------------------
template <int XT, int FMT, int K>
__global__ void __launch_bounds__(kChThreads)
per_channel_vec_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ q,
                       float* __restrict__ sinv, int64_t cols) {
    constexpr int ES = ElemBytes<XT>::value;
    constexpr int EPV = 16 / ES;
    __shared__ uint32_t sh[kChThreads / 32];
    const int64_t row = blockIdx.x;
    const int64_t nvec = cols / EPV;
    const uint8_t* xr = x + row * cols * ES;
    uint8_t* qr = q + row * cols;

    uint4 v[K];
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const int64_t i = threadIdx.x + (int64_t)k * kChThreads;
        v[k] = i < nvec ? ld_stream_v4(xr + i * 16) : make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t m;
    if (XT == kF32) {
        m = 0u;
#pragma unroll
        for (int k = 0; k < K; ++k) m = max(m, vec_absmax_bits<kF32>(v[k]));
    } else {
        uint32_t p = 0u;
#pragma unroll
        for (int k = 0; k < K; ++k) p = max_u16x2(p, vec_absmax_packed16(v[k]));
        m = packed16_to_f32bits<XT>(p);
    }
    m = block_max_u32(m, sh);
    float amax;
    bool fix;
    const float scale = colossal_scale<FMT>(m, amax, fix);
    if (threadIdx.x == 0) sinv[row] = __fdiv_rn(amax, fp8_max<FMT>());
    if (!fix) {
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int64_t i = threadIdx.x + (int64_t)k * kChThreads;
            if (i < nvec) encode_store<XT, FMT, false>(v[k], scale, qr + i * EPV);
        }
    } else {
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int64_t i = threadIdx.x + (int64_t)k * kChThreads;
            if (i < nvec) encode_store<XT, FMT, true>(v[k], scale, qr + i * EPV);
        }
    }
}

// rows too long for registers, or layouts the vector path cannot take:
// reduce over the row, then re-read it for the cast.  VEC selects 16-byte
// accesses (row stride and base 16-byte aligned) or scalar accesses.
template <int XT, int FMT, bool VEC>
__global__ void __launch_bounds__(kChThreads)
per_channel_loop_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ q,
                        float* __restrict__ sinv, int64_t cols) {
    constexpr int ES = ElemBytes<XT>::value;
    constexpr int EPV = 16 / ES;
    __shared__ uint32_t sh[kChThreads / 32];
    const int64_t row = blockIdx.x;
    const uint8_t* xr = x + row * cols * ES;
    uint8_t* qr = q + row * cols;
    uint32_t m = 0u;
    if (VEC) {
        const int64_t nvec = cols / EPV;
        for (int64_t i = threadIdx.x; i < nvec; i += kChThreads)
            m = max(m, vec_absmax_bits<XT>(ld_stream_v4(xr + i * 16)));
    } else {
        for (int64_t c = threadIdx.x; c < cols; c += kChThreads) m = max(m, elem_abs_bits<XT>(xr + c * ES));
    }
    m = block_max_u32(m, sh);
    float amax;
    bool fix;
    const float scale = colossal_scale<FMT>(m, amax, fix);
    if (threadIdx.x == 0) sinv[row] = __fdiv_rn(amax, fp8_max<FMT>());
    if (VEC) {
        const int64_t nvec = cols / EPV;
        for (int64_t i = threadIdx.x; i < nvec; i += kChThreads) {
            const uint4 v = *reinterpret_cast<const uint4*>(xr + i * 16);
            if (fix) encode_store<XT, FMT, true>(v, scale, qr + i * EPV);
            else encode_store<XT, FMT, false>(v, scale, qr + i * EPV);
        }
    } else {
        for (int64_t c = threadIdx.x; c < cols; c += kChThreads) {
            const float f = __fmul_rn(elem_load<XT>(xr + c * ES), scale);
            qr[c] = fix ? encode_one<FMT, true>(f) : encode_one<FMT, false>(f);
        }
    }
}

// ---------------------------------------------------------------------------
// per-tensor
// ---------------------------------------------------------------------------
// pass 1: per-CTA magnitude-bits maximum over 16-byte vectors (plus the
// scalar tail of numel % EPV elements, taken by the first threads of CTA 0)
template <int XT, bool VEC>
__global__ void __launch_bounds__(kPtThreads)
tensor_amax_kernel(const uint8_t* __restrict__ x, int64_t numel, uint32_t* __restrict__ partials) {
    constexpr int ES = ElemBytes<XT>::value;
    constexpr int EPV = VEC ? 16 / ES : 1;
    __shared__ uint32_t sh[kPtThreads / 32];
    const int64_t nvec = numel / EPV;
    const int64_t stride = (int64_t)gridDim.x * kPtThreads;
    int64_t i = (int64_t)blockIdx.x * kPtThreads + threadIdx.x;
    uint32_t m = 0u;
    if (VEC) {
        if (XT == kF32) {
            for (; i + 3 * stride < nvec; i += 4 * stride) {
                const uint4 a = ld_stream_v4(x + i * 16), b = ld_stream_v4(x + (i + stride) * 16);
                const uint4 c = ld_stream_v4(x + (i + 2 * stride) * 16), d = ld_stream_v4(x + (i + 3 * stride) * 16);
                m = max(m, max(max(vec_absmax_bits<kF32>(a), vec_absmax_bits<kF32>(b)),
                               max(vec_absmax_bits<kF32>(c), vec_absmax_bits<kF32>(d))));
            }
            for (; i < nvec; i += stride) m = max(m, vec_absmax_bits<kF32>(ld_stream_v4(x + i * 16)));
        } else {
            uint32_t p = 0u;
            for (; i + 3 * stride < nvec; i += 4 * stride) {
                const uint4 a = ld_stream_v4(x + i * 16), b = ld_stream_v4(x + (i + stride) * 16);
                const uint4 c = ld_stream_v4(x + (i + 2 * stride) * 16), d = ld_stream_v4(x + (i + 3 * stride) * 16);
                p = max_u16x2(p, max_u16x2(max_u16x2(vec_absmax_packed16(a), vec_absmax_packed16(b)),
                                           max_u16x2(vec_absmax_packed16(c), vec_absmax_packed16(d))));
            }
            for (; i < nvec; i += stride) p = max_u16x2(p, vec_absmax_packed16(ld_stream_v4(x + i * 16)));
            m = packed16_to_f32bits<XT>(p);
        }
        if (blockIdx.x == 0 && threadIdx.x < numel - nvec * EPV)
            m = max(m, elem_abs_bits<XT>(x + (nvec * EPV + threadIdx.x) * ES));
    } else {
        for (; i < numel; i += stride) m = max(m, elem_abs_bits<XT>(x + i * ES));
    }
    m = block_max_u32(m, sh);
    if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

// pass 2: reduce the partials, derive the scale, cast (walking from the end)
template <int XT, int FMT, bool VEC>
__global__ void __launch_bounds__(kPtThreads)
tensor_cast_kernel(const uint8_t* __restrict__ x, int64_t numel, uint8_t* __restrict__ q,
                   float* __restrict__ sinv, const uint32_t* __restrict__ partials, int nparts) {
    constexpr int ES = ElemBytes<XT>::value;
    constexpr int EPV = VEC ? 16 / ES : 1;
    __shared__ uint32_t sh;
    if (threadIdx.x < 32) {
        uint32_t m = 0u;
        for (int p = threadIdx.x; p < nparts; p += 32) m = max(m, __ldcg(partials + p));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        if (threadIdx.x == 0) sh = m;
    }
    __syncthreads();
    float amax;
    bool fix;
    const float scale = colossal_scale<FMT>(sh, amax, fix);
    if (blockIdx.x == 0 && threadIdx.x == 0) sinv[0] = __fdiv_rn(1.0f, scale);
    const int64_t nvec = numel / EPV;
    const int64_t stride = (int64_t)gridDim.x * kPtThreads;
    const int64_t t0 = (int64_t)blockIdx.x * kPtThreads + threadIdx.x;
    if (VEC) {
        // vector j = nvec - 1 - t, t = t0, t0 + stride, ...; four in flight
        int64_t t = t0;
        if (!fix) {
            for (; t + 3 * stride < nvec; t += 4 * stride) {
                uint4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) v[u] = ld_stream_v4(x + (nvec - 1 - (t + u * stride)) * 16);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    encode_store<XT, FMT, false>(v[u], scale, q + (nvec - 1 - (t + u * stride)) * EPV);
            }
            for (; t < nvec; t += stride)
                encode_store<XT, FMT, false>(ld_stream_v4(x + (nvec - 1 - t) * 16), scale, q + (nvec - 1 - t) * EPV);
        } else {
            for (; t < nvec; t += stride)
                encode_store<XT, FMT, true>(ld_stream_v4(x + (nvec - 1 - t) * 16), scale, q + (nvec - 1 - t) * EPV);
        }
        if (blockIdx.x == 0 && threadIdx.x < numel - nvec * EPV) {
            const int64_t e = nvec * EPV + threadIdx.x;
            const float f = __fmul_rn(elem_load<XT>(x + e * ES), scale);
            q[e] = fix ? encode_one<FMT, true>(f) : encode_one<FMT, false>(f);
        }
    } else {
        for (int64_t e = t0; e < numel; e += stride) {
            const float f = __fmul_rn(elem_load<XT>(x + e * ES), scale);
            q[e] = fix ? encode_one<FMT, true>(f) : encode_one<FMT, false>(f);
        }
    }
}

__global__ void fill_kernel(float* __restrict__ dst, int64_t count, float value) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
         i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = value;
}

template <int XT, int FMT>
fp8q_status run_per_channel(const uint8_t* x, uint8_t* q, float* sinv, int64_t rows, int64_t cols,
                            cudaStream_t s) {
    constexpr int ES = ElemBytes<XT>::value;
    constexpr int EPV = 16 / ES;
    if (rows > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
    const bool vec = ((uintptr_t)x % 16 == 0) && ((cols * ES) % 16 == 0) && ((uintptr_t)q % EPV == 0);
    const unsigned grid = (unsigned)rows;
    if (vec) {
        const int64_t nvec = cols / EPV;
        if (nvec <= 1 * kChThreads) per_channel_vec_kernel<XT, FMT, 1><<<grid, kChThreads, 0, s>>>(x, q, sinv, cols);
        else if (nvec <= 2 * kChThreads) per_channel_vec_kernel<XT, FMT, 2><<<grid, kChThreads, 0, s>>>(x, q, sinv, cols);
        else if (nvec <= 4 * kChThreads) per_channel_vec_kernel<XT, FMT, 4><<<grid, kChThreads, 0, s>>>(x, q, sinv, cols);
        else if (nvec <= 8 * kChThreads) per_channel_vec_kernel<XT, FMT, 8><<<grid, kChThreads, 0, s>>>(x, q, sinv, cols);
        else per_channel_loop_kernel<XT, FMT, true><<<grid, kChThreads, 0, s>>>(x, q, sinv, cols);
    } else {
        per_channel_loop_kernel<XT, FMT, false><<<grid, kChThreads, 0, s>>>(x, q, sinv, cols);
    }
    return cuda_status(cudaGetLastError());
}

template <int XT, int FMT>
fp8q_status run_per_tensor(const uint8_t* x, int64_t numel, uint8_t* q, float* sinv, uint32_t* partials,
                           cudaStream_t s) {
    constexpr int ES = ElemBytes<XT>::value;
    constexpr int EPV = 16 / ES;
    const bool vec = ((uintptr_t)x % 16 == 0) && ((uintptr_t)q % EPV == 0);
    const int64_t units = vec ? numel / EPV : numel;
    int64_t want = (units + kPtThreads * kPtUnroll - 1) / (kPtThreads * kPtUnroll);
    const int64_t cap = (int64_t)sm_count() * 8 < kMaxPartials ? (int64_t)sm_count() * 8 : kMaxPartials;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    const int grid = (int)want;
    if (vec) {
        tensor_amax_kernel<XT, true><<<grid, kPtThreads, 0, s>>>(x, numel, partials);
        fp8q_status st = cuda_status(cudaGetLastError());
        if (st != FP8Q_OK) return st;
        tensor_cast_kernel<XT, FMT, true><<<grid, kPtThreads, 0, s>>>(x, numel, q, sinv, partials, grid);
    } else {
        tensor_amax_kernel<XT, false><<<grid, kPtThreads, 0, s>>>(x, numel, partials);
        fp8q_status st = cuda_status(cudaGetLastError());
        if (st != FP8Q_OK) return st;
        tensor_cast_kernel<XT, FMT, false><<<grid, kPtThreads, 0, s>>>(x, numel, q, sinv, partials, grid);
    }
    return cuda_status(cudaGetLastError());
}

template <int XT>
fp8q_status per_channel_fmt(const uint8_t* x, int fmt, uint8_t* q, float* sinv, int64_t rows, int64_t cols,
                            cudaStream_t s) {
    return fmt == kE4M3 ? run_per_channel<XT, kE4M3>(x, q, sinv, rows, cols, s)
                        : run_per_channel<XT, kE5M2>(x, q, sinv, rows, cols, s);
}

template <int XT>
fp8q_status per_tensor_fmt(const uint8_t* x, int fmt, int64_t numel, uint8_t* q, float* sinv,
                           uint32_t* partials, cudaStream_t s) {
    return fmt == kE4M3 ? run_per_tensor<XT, kE4M3>(x, numel, q, sinv, partials, s)
                        : run_per_tensor<XT, kE5M2>(x, numel, q, sinv, partials, s);
}

}  // namespace

fp8q_status launch_fill(float* dst, int64_t count, float value, cudaStream_t s) {
    if (count <= 0) return FP8Q_OK;
    const int64_t want = (count + 255) / 256;
    const int grid = (int)(want < 1024 ? want : 1024);
    fill_kernel<<<grid, 256, 0, s>>>(dst, count, value);
    return cuda_status(cudaGetLastError());
}

fp8q_status launch_per_channel(const void* x, int xt, int64_t rows, int64_t cols, int fmt,
                               uint8_t* q, float* sinv, cudaStream_t s) {
    const uint8_t* xb = static_cast<const uint8_t*>(x);
    switch (xt) {
    case kF32: return per_channel_fmt<kF32>(xb, fmt, q, sinv, rows, cols, s);
    case kF16: return per_channel_fmt<kF16>(xb, fmt, q, sinv, rows, cols, s);
    default: return per_channel_fmt<kBF16>(xb, fmt, q, sinv, rows, cols, s);
    }
}

fp8q_status launch_per_tensor(const void* x, int xt, int64_t numel, int fmt, uint8_t* q,
                              float* sinv, uint32_t* partials, cudaStream_t s) {
    const uint8_t* xb = static_cast<const uint8_t*>(x);
    switch (xt) {
    case kF32: return per_tensor_fmt<kF32>(xb, fmt, numel, q, sinv, partials, s);
    case kF16: return per_tensor_fmt<kF16>(xb, fmt, numel, q, sinv, partials, s);
    default: return per_tensor_fmt<kBF16>(xb, fmt, numel, q, sinv, partials, s);
    }
}

}  // namespace fp8q
