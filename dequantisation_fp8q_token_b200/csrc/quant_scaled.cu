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
// cast.  Pass 1 reads the last kL2KeepBytes of x with an L2 evict_last policy
// (the rest evict_first), and pass 2 walks the tensor from the end, so the
// second read of that tail comes from L2 instead of HBM.
#include "fp8q_device.cuh"
#include "fp8q_internal.h"

namespace fp8q {
namespace {

#ifndef FP8Q_SCALED_V32
#define FP8Q_SCALED_V32 1  // 32-byte vectors (256-bit loads) where the pointers allow
#endif
constexpr int kChThreads = 256;
constexpr int kPtThreads = 256;
constexpr int kPtUnroll = 4;
#ifndef FP8Q_PT_L2_KEEP_MB
#define FP8Q_PT_L2_KEEP_MB 80
#endif
constexpr int64_t kL2KeepBytes = (int64_t)FP8Q_PT_L2_KEEP_MB << 20;  // well inside the 126 MB L2

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

template <int FMT, bool FIX>
__device__ __forceinline__ uint8_t encode_one(float f) {
    return (uint8_t)(enc2_sem<FMT, FIX>(f, 0.0f) & 0xFFu);
}

// ColossalAI scale rule from an fp32 magnitude-bits amax.  `fix` is set when
// the hardware's saturating encode could differ from the non-saturating
// reference: a NaN amax (replaced by 1, so NaN/Inf elements and overflow can
// occur) or a scale that overflowed to Inf (amax < FMAX / FLT_MAX).
template <int FMT>
__device__ __forceinline__ float colossal_scale(uint32_t amax_bits, float& amax_out, bool& fix, int rule) {
    const float a = __uint_as_float(amax_bits);
    const float amax = a > 0.0f ? a : 1.0f;
    const float scale = scale_from_amax<FMT>(amax, rule);
    fix = (amax_bits > 0x7F800000u) || isinf(scale);
    amax_out = amax;
    return scale;
}

// ---------------------------------------------------------------------------
// per-channel
// ---------------------------------------------------------------------------
template <int XT, int FMT, int K, int VB>
__global__ void __launch_bounds__(kChThreads)
per_channel_vec_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ q,
                       float* __restrict__ sinv, int64_t cols, int rule) {
    constexpr int ES = ElemBytes<XT>::value;
    constexpr int EPV = VB / ES;
    pdl_trigger();
    // the row (cols * ES bytes, a multiple of VB, from a VB-aligned base) into L2
    if (threadIdx.x == 0 && cols > 0) prefetch_l2_bulk(x + (int64_t)blockIdx.x * cols * ES, (uint32_t)(cols * ES));
    pdl_wait();
    __shared__ uint32_t sh[kChThreads / 32];
    const int64_t row = blockIdx.x;
    const int64_t nvec = cols / EPV;
    const uint8_t* xr = x + row * cols * ES;
    uint8_t* qr = q + row * cols;

    Vec<VB> v[K];
    uint32_t m = 0u;
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const int64_t i = threadIdx.x + (int64_t)k * kChThreads;
        if (i < nvec) v[k] = load_vec<VB>(xr + i * VB);
    }
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const int64_t i = threadIdx.x + (int64_t)k * kChThreads;
        if (i < nvec) m = absmax2<XT>(m, vec_absmax<XT, VB>(v[k]));
    }
    const uint32_t bits = block_max_u32(absmax_bits<XT>(m), sh);
    float amax;
    bool fix;
    const float scale = colossal_scale<FMT>(bits, amax, fix, rule);
    if (threadIdx.x == 0) sinv[row] = scale_inv_from_amax<FMT>(amax, rule);
    if (!fix) {
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int64_t i = threadIdx.x + (int64_t)k * kChThreads;
            if (i < nvec) encode_store_vec<XT, FMT, VB, false>(v[k], scale, qr + i * EPV);
        }
    } else {
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int64_t i = threadIdx.x + (int64_t)k * kChThreads;
            if (i < nvec) encode_store_vec<XT, FMT, VB, true>(v[k], scale, qr + i * EPV);
        }
    }
}

// rows too long for registers, or layouts the vector path cannot take:
// reduce over the row, then re-read it for the cast.  VB = 16 / 32 selects
// vector accesses (row stride and base VB-aligned), VB = 0 scalar accesses.
template <int XT, int FMT, int VB>
__global__ void __launch_bounds__(kChThreads)
per_channel_loop_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ q,
                        float* __restrict__ sinv, int64_t cols, int rule) {
    pdl_begin();
    constexpr int ES = ElemBytes<XT>::value;
    constexpr int EPV = VB > 0 ? VB / ES : 1;
    __shared__ uint32_t sh[kChThreads / 32];
    const int64_t row = blockIdx.x;
    const uint8_t* xr = x + row * cols * ES;
    uint8_t* qr = q + row * cols;
    uint32_t bits;
    if constexpr (VB > 0) {
        uint32_t m = 0u;
        const int64_t nvec = cols / EPV;
        for (int64_t i = threadIdx.x; i < nvec; i += kChThreads)
            m = absmax2<XT>(m, vec_absmax<XT, VB>(load_vec<VB>(xr + i * VB)));
        bits = absmax_bits<XT>(m);
    } else {
        bits = 0u;
        for (int64_t c = threadIdx.x; c < cols; c += kChThreads) bits = max(bits, elem_abs_bits<XT>(xr + c * ES));
    }
    bits = block_max_u32(bits, sh);
    float amax;
    bool fix;
    const float scale = colossal_scale<FMT>(bits, amax, fix, rule);
    if (threadIdx.x == 0) sinv[row] = scale_inv_from_amax<FMT>(amax, rule);
    if constexpr (VB > 0) {
        const int64_t nvec = cols / EPV;
        for (int64_t i = threadIdx.x; i < nvec; i += kChThreads) {
            Vec<VB> v;
#pragma unroll
            for (int w = 0; w < VB / 4; ++w) v.w[w] = reinterpret_cast<const uint32_t*>(xr + i * VB)[w];
            if (fix) encode_store_vec<XT, FMT, VB, true>(v, scale, qr + i * EPV);
            else encode_store_vec<XT, FMT, VB, false>(v, scale, qr + i * EPV);
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
// pass 1: per-CTA magnitude-bits maximum over VB-byte vectors (plus the scalar
// tail of numel % EPV elements, taken by the first threads of CTA 0); VB = 0
// is the scalar path for unaligned tensors
template <int XT, int VB>
__global__ void __launch_bounds__(kPtThreads)
tensor_amax_kernel(const uint8_t* __restrict__ x, int64_t numel, uint32_t* __restrict__ partials) {
    constexpr int ES = ElemBytes<XT>::value;
    constexpr int EPV = VB > 0 ? VB / ES : 1;
    __shared__ uint32_t sh[kPtThreads / 32];
    const int64_t nvec = numel / EPV;
    const int64_t stride = (int64_t)gridDim.x * kPtThreads;
    int64_t i = (int64_t)blockIdx.x * kPtThreads + threadIdx.x;
    pdl_trigger();
    if constexpr (VB > 0) {
        // the vectors of this thread's first unrolled step into L2
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (i + u * stride < nvec) prefetch_l2(x + (i + u * stride) * VB);
    }
    pdl_wait();
    uint32_t bits;
    if constexpr (VB > 0) {
        // vectors from keep_from on stay in L2 for pass 2
        const int64_t keep_from = nvec - kL2KeepBytes / VB;
        const uint64_t keep = l2_evict_last_policy(), drop = l2_evict_first_policy();
        auto ld = [&](int64_t j) { return load_vec_policy<VB>(x + j * VB, j >= keep_from ? keep : drop); };
        uint32_t m = 0u;
        for (; i + 3 * stride < nvec; i += 4 * stride) {
            const Vec<VB> a = ld(i), b = ld(i + stride), c = ld(i + 2 * stride), d = ld(i + 3 * stride);
            m = absmax2<XT>(m, absmax2<XT>(absmax2<XT>(vec_absmax<XT, VB>(a), vec_absmax<XT, VB>(b)),
                                           absmax2<XT>(vec_absmax<XT, VB>(c), vec_absmax<XT, VB>(d))));
        }
        for (; i < nvec; i += stride) m = absmax2<XT>(m, vec_absmax<XT, VB>(ld(i)));
        bits = absmax_bits<XT>(m);
        if (blockIdx.x == 0 && threadIdx.x < numel - nvec * EPV)
            bits = max(bits, elem_abs_bits<XT>(x + (nvec * EPV + threadIdx.x) * ES));
    } else {
        bits = 0u;
        for (; i < numel; i += stride) bits = max(bits, elem_abs_bits<XT>(x + i * ES));
    }
    bits = block_max_u32(bits, sh);
    if (threadIdx.x == 0) partials[blockIdx.x] = bits;
}

// magnitude-bits maximum of the amax pass's partials (every thread gets it)
__device__ __forceinline__ uint32_t reduce_partials(const uint32_t* __restrict__ partials, int nparts,
                                                    uint32_t* sh) {
    if (threadIdx.x < 32) {
        uint32_t m = 0u;
        for (int p = threadIdx.x; p < nparts; p += 32) m = max(m, __ldcg(partials + p));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        if (threadIdx.x == 0) *sh = m;
    }
    __syncthreads();
    return *sh;
}

// the cast pass over the whole tensor with a known scale, walking from the
// end so the part of x the amax pass kept in L2 is read first
template <int XT, int FMT, int VB>
__device__ __forceinline__ void cast_tensor_body(const uint8_t* __restrict__ x, int64_t numel,
                                                 uint8_t* __restrict__ q, float scale, bool fix) {
    constexpr int ES = ElemBytes<XT>::value;
    constexpr int EPV = VB > 0 ? VB / ES : 1;
    const int64_t nvec = numel / EPV;
    const int64_t stride = (int64_t)gridDim.x * kPtThreads;
    const int64_t t0 = (int64_t)blockIdx.x * kPtThreads + threadIdx.x;
    if constexpr (VB > 0) {
        // vector j = nvec - 1 - t, t = t0, t0 + stride, ...; four in flight;
        // x is not needed again, so its lines go first
        const uint64_t drop = l2_evict_first_policy();
        int64_t t = t0;
        if (!fix) {
            for (; t + 3 * stride < nvec; t += 4 * stride) {
                Vec<VB> v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) v[u] = load_vec_policy<VB>(x + (nvec - 1 - (t + u * stride)) * VB, drop);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    encode_store_vec<XT, FMT, VB, false>(v[u], scale, q + (nvec - 1 - (t + u * stride)) * EPV);
            }
            for (; t < nvec; t += stride)
                encode_store_vec<XT, FMT, VB, false>(load_vec_policy<VB>(x + (nvec - 1 - t) * VB, drop), scale,
                                                     q + (nvec - 1 - t) * EPV);
        } else {
            for (; t < nvec; t += stride)
                encode_store_vec<XT, FMT, VB, true>(load_vec_policy<VB>(x + (nvec - 1 - t) * VB, drop), scale,
                                                    q + (nvec - 1 - t) * EPV);
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

// pass 2: reduce the partials, derive the scale, cast
template <int XT, int FMT, int VB>
__global__ void __launch_bounds__(kPtThreads)
tensor_cast_kernel(const uint8_t* __restrict__ x, int64_t numel, uint8_t* __restrict__ q,
                   float* __restrict__ sinv, const uint32_t* __restrict__ partials, int nparts, int rule) {
    pdl_begin();
    __shared__ uint32_t sh;
    const uint32_t bits = reduce_partials(partials, nparts, &sh);
    float amax;
    bool fix;
    const float scale = colossal_scale<FMT>(bits, amax, fix, rule);
    if (blockIdx.x == 0 && threadIdx.x == 0) sinv[0] = __fdiv_rn(1.0f, scale);
    cast_tensor_body<XT, FMT, VB>(x, numel, q, scale, fix);
}

// ColossalAI cast_to_fp8_pipeline, pass 2: the format follows the amax
// (e5m2 above the e4m3fn maximum of 448, else e4m3fn; a NaN amax fails the
// test), the scale is 1 for an all-zero tensor; writes the format tag and
// scale_inv = 1 / scale
template <int XT, int VB>
__global__ void __launch_bounds__(kPtThreads)
pipeline_cast_kernel(const uint8_t* __restrict__ x, int64_t numel, uint8_t* __restrict__ q,
                     float* __restrict__ sinv, int32_t* __restrict__ fmt_out,
                     const uint32_t* __restrict__ partials, int nparts, int rule) {
    pdl_begin();
    __shared__ uint32_t sh;
    const float amax = __uint_as_float(reduce_partials(partials, nparts, &sh));
    const bool e5 = amax > 448.0f;
    const float scale = amax == 0.0f ? 1.0f
                        : (e5 ? scale_from_amax<kE5M2>(amax, rule) : scale_from_amax<kE4M3>(amax, rule));
    // finite amax > 0 with a finite scale cannot overflow, and a NaN amax
    // makes every product NaN; only an overflowed scale needs the fix-up
    const bool fix = isinf(scale);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        sinv[0] = __fdiv_rn(1.0f, scale);
        fmt_out[0] = e5 ? kE5M2 : kE4M3;
    }
    if (e5) cast_tensor_body<XT, kE5M2, VB>(x, numel, q, scale, fix);
    else cast_tensor_body<XT, kE4M3, VB>(x, numel, q, scale, fix);
}

// ColossalAI cast_from_fp8_pipeline: y = T(fl(float(q) * scale_inv[0])) in
// the format the tag names (1 = e5m2, anything else e4m3fn); 16 codes per
// thread when q and y allow 16-byte accesses (VEC), else one
template <int FMT, int YT>
__device__ __forceinline__ void decode16(uint4 c, float sc, void* y, int64_t e) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    if (YT == kF32) {
        float* yf = static_cast<float*>(y) + e;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 a = dec2<FMT>(w[i] & 0xFFFFu), b = dec2<FMT>(w[i] >> 16);
            st_v4(yf + 4 * i, make_uint4(__float_as_uint(__fmul_rn(a.x, sc)), __float_as_uint(__fmul_rn(a.y, sc)),
                                         __float_as_uint(__fmul_rn(b.x, sc)), __float_as_uint(__fmul_rn(b.y, sc))));
        }
    } else {
        uint16_t* yh = static_cast<uint16_t*>(y) + e;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float2 a = dec2<FMT>(w[2 * h + i] & 0xFFFFu), b = dec2<FMT>(w[2 * h + i] >> 16);
                o[2 * i] = pack2<YT>(__fmul_rn(a.x, sc), __fmul_rn(a.y, sc));
                o[2 * i + 1] = pack2<YT>(__fmul_rn(b.x, sc), __fmul_rn(b.y, sc));
            }
            st_v4(yh + 8 * h, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
}

template <int FMT, int YT>
__device__ __forceinline__ void decode_one(uint8_t c, float sc, void* y, int64_t e) {
    const float v = __fmul_rn(dec2<FMT>(c).x, sc);
    if (YT == kF32) static_cast<float*>(y)[e] = v;
    else static_cast<uint16_t*>(y)[e] = (uint16_t)(pack2<YT>(v, 0.0f) & 0xFFFFu);
}

template <int FMT, int YT, bool VEC>
__device__ __forceinline__ void decode_body(const uint8_t* __restrict__ q, int64_t numel, float sc, void* y) {
    const int64_t stride = (int64_t)gridDim.x * kPtThreads;
    const int64_t t0 = (int64_t)blockIdx.x * kPtThreads + threadIdx.x;
    if (VEC) {
        const int64_t nch = numel / 16;
        for (int64_t t = t0; t < nch; t += stride) decode16<FMT, YT>(ld_stream_v4(q + t * 16), sc, y, t * 16);
        if (blockIdx.x == 0 && threadIdx.x < numel - nch * 16) {
            const int64_t e = nch * 16 + threadIdx.x;
            decode_one<FMT, YT>(q[e], sc, y, e);
        }
    } else {
        for (int64_t e = t0; e < numel; e += stride) decode_one<FMT, YT>(q[e], sc, y, e);
    }
}

template <int YT, bool VEC>
__global__ void __launch_bounds__(kPtThreads)
pipeline_decode_kernel(const uint8_t* __restrict__ q, int64_t numel, const float* __restrict__ sinv,
                       const int32_t* __restrict__ fmt_in, void* __restrict__ y) {
    pdl_begin();
    const float sc = __ldg(sinv);
    if (__ldg(fmt_in) == kE5M2) decode_body<kE5M2, YT, VEC>(q, numel, sc, y);
    else decode_body<kE4M3, YT, VEC>(q, numel, sc, y);
}

// the amax of a tensor as fp32 magnitude bits, from the amax pass's partials
// (one CTA); ranks holding shards of one tensor combine these words with an
// integer MAX, which orders magnitudes and propagates NaN like the kernels
__global__ void __launch_bounds__(kPtThreads)
amax_finish_kernel(const uint32_t* __restrict__ partials, int nparts, uint32_t* __restrict__ amax_bits) {
    pdl_begin();
    __shared__ uint32_t sh;
    const uint32_t bits = reduce_partials(partials, nparts, &sh);
    if (threadIdx.x == 0) amax_bits[0] = bits;
}

__global__ void fill_kernel(float* __restrict__ dst, int64_t count, float value) {
    pdl_begin();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
         i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = value;
}

// widest vector (32 or 16 bytes) that a base pointer, a row stride in bytes
// and the matching code pointer allow; 0 when neither does
int vector_bytes(const void* x, int64_t stride_bytes, const void* q, int es) {
#if FP8Q_SCALED_V32
    if ((uintptr_t)x % 32 == 0 && stride_bytes % 32 == 0 && (uintptr_t)q % (32 / es) == 0) return 32;
#endif
    if ((uintptr_t)x % 16 == 0 && stride_bytes % 16 == 0 && (uintptr_t)q % (16 / es) == 0) return 16;
    return 0;
}

template <int XT, int FMT, int VB>
cudaError_t per_channel_launch(const uint8_t* x, uint8_t* q, float* sinv, int64_t rows, int64_t cols, int rule,
                               cudaStream_t s) {
    constexpr int ES = ElemBytes<XT>::value;
    const unsigned grid = (unsigned)rows;
    cudaError_t err;
    const int64_t nvec = cols * ES / VB;
    if (nvec <= 1 * kChThreads) err = launch_kernel(per_channel_vec_kernel<XT, FMT, 1, VB>, dim3(grid), dim3(kChThreads), s, x, q, sinv, cols, rule);
    else if (nvec <= 2 * kChThreads) err = launch_kernel(per_channel_vec_kernel<XT, FMT, 2, VB>, dim3(grid), dim3(kChThreads), s, x, q, sinv, cols, rule);
    else if (nvec <= 4 * kChThreads) err = launch_kernel(per_channel_vec_kernel<XT, FMT, 4, VB>, dim3(grid), dim3(kChThreads), s, x, q, sinv, cols, rule);
    else if constexpr (VB == 16) {
        if (nvec <= 8 * kChThreads) err = launch_kernel(per_channel_vec_kernel<XT, FMT, 8, VB>, dim3(grid), dim3(kChThreads), s, x, q, sinv, cols, rule);
        else err = launch_kernel(per_channel_loop_kernel<XT, FMT, VB>, dim3(grid), dim3(kChThreads), s, x, q, sinv, cols, rule);
    } else {
        err = launch_kernel(per_channel_loop_kernel<XT, FMT, VB>, dim3(grid), dim3(kChThreads), s, x, q, sinv, cols, rule);
    }
    return err;
}

template <int XT, int FMT>
fp8q_status run_per_channel(const uint8_t* x, uint8_t* q, float* sinv, int64_t rows, int64_t cols, int rule,
                            cudaStream_t s) {
    constexpr int ES = ElemBytes<XT>::value;
    if (rows > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
    const int vb = vector_bytes(x, cols * ES, q, ES);
    cudaError_t err;
    if (vb == 32) err = per_channel_launch<XT, FMT, 32>(x, q, sinv, rows, cols, rule, s);
    else if (vb == 16) err = per_channel_launch<XT, FMT, 16>(x, q, sinv, rows, cols, rule, s);
    else err = launch_kernel(per_channel_loop_kernel<XT, FMT, 0>, dim3((unsigned)rows), dim3(kChThreads), s, x, q, sinv, cols, rule);
    return cuda_status(err);
}

template <int XT, int FMT, int VB>
fp8q_status per_tensor_launch(const uint8_t* x, int64_t numel, uint8_t* q, float* sinv, uint32_t* partials,
                              int rule, cudaStream_t s) {
    constexpr int ES = ElemBytes<XT>::value;
    const int64_t units = VB > 0 ? numel * ES / VB : numel;
    int64_t want = (units + kPtThreads * kPtUnroll - 1) / (kPtThreads * kPtUnroll);
    // one wave: both passes grid-stride over the tensor with every CTA resident
    static const int per_sm = min(resident_blocks_per_sm(tensor_amax_kernel<XT, VB>, kPtThreads),
                                  resident_blocks_per_sm(tensor_cast_kernel<XT, FMT, VB>, kPtThreads));
    int64_t cap = (int64_t)sm_count() * min(per_sm, 8);
    if (cap > kMaxPartials) cap = kMaxPartials;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    const int grid = (int)want;
    cudaError_t err = launch_kernel(tensor_amax_kernel<XT, VB>, dim3(grid), dim3(kPtThreads), s, x, numel, partials);
    if (err != cudaSuccess) return FP8Q_ERR_CUDA;
    err = launch_kernel(tensor_cast_kernel<XT, FMT, VB>, dim3(grid), dim3(kPtThreads), s, x, numel, q, sinv, partials, grid, rule);
    return cuda_status(err);
}

template <int XT, int FMT>
fp8q_status run_per_tensor(const uint8_t* x, int64_t numel, uint8_t* q, float* sinv, uint32_t* partials,
                           int rule, cudaStream_t s) {
    constexpr int ES = ElemBytes<XT>::value;
    const int vb = vector_bytes(x, 0, q, ES);
    if (vb == 32) return per_tensor_launch<XT, FMT, 32>(x, numel, q, sinv, partials, rule, s);
    if (vb == 16) return per_tensor_launch<XT, FMT, 16>(x, numel, q, sinv, partials, rule, s);
    return per_tensor_launch<XT, FMT, 0>(x, numel, q, sinv, partials, rule, s);
}

template <int XT>
fp8q_status per_channel_fmt(const uint8_t* x, int fmt, uint8_t* q, float* sinv, int64_t rows, int64_t cols,
                            int rule, cudaStream_t s) {
    return fmt == kE4M3 ? run_per_channel<XT, kE4M3>(x, q, sinv, rows, cols, rule, s)
                        : run_per_channel<XT, kE5M2>(x, q, sinv, rows, cols, rule, s);
}

template <int XT>
fp8q_status per_tensor_fmt(const uint8_t* x, int fmt, int64_t numel, uint8_t* q, float* sinv,
                           uint32_t* partials, int rule, cudaStream_t s) {
    return fmt == kE4M3 ? run_per_tensor<XT, kE4M3>(x, numel, q, sinv, partials, rule, s)
                        : run_per_tensor<XT, kE5M2>(x, numel, q, sinv, partials, rule, s);
}

}  // namespace

fp8q_status launch_fill(float* dst, int64_t count, float value, cudaStream_t s) {
    if (count <= 0) return FP8Q_OK;
    const int64_t want = (count + 255) / 256;
    const int grid = (int)(want < 1024 ? want : 1024);
    const cudaError_t err = launch_kernel(fill_kernel, dim3(grid), dim3(256), s, dst, count, value);
    return cuda_status(err);
}

// the pipeline cast: the amax pass, then the format-selecting cast pass
template <int XT, int VB>
fp8q_status pipeline_launch(const uint8_t* x, int64_t numel, uint8_t* q, float* sinv, int32_t* fmt_out,
                            uint32_t* partials, int rule, cudaStream_t s) {
    constexpr int ES = ElemBytes<XT>::value;
    const int64_t units = VB > 0 ? numel * ES / VB : numel;
    int64_t want = (units + kPtThreads * kPtUnroll - 1) / (kPtThreads * kPtUnroll);
    static const int per_sm = min(resident_blocks_per_sm(tensor_amax_kernel<XT, VB>, kPtThreads),
                                  resident_blocks_per_sm(pipeline_cast_kernel<XT, VB>, kPtThreads));
    int64_t cap = (int64_t)sm_count() * min(per_sm, 8);
    if (cap > kMaxPartials) cap = kMaxPartials;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    const int grid = (int)want;
    cudaError_t err = launch_kernel(tensor_amax_kernel<XT, VB>, dim3(grid), dim3(kPtThreads), s, x, numel, partials);
    if (err != cudaSuccess) return FP8Q_ERR_CUDA;
    err = launch_kernel(pipeline_cast_kernel<XT, VB>, dim3(grid), dim3(kPtThreads), s, x, numel, q, sinv, fmt_out,
                        partials, grid, rule);
    return cuda_status(err);
}

template <int XT>
fp8q_status run_pipeline(const uint8_t* x, int64_t numel, uint8_t* q, float* sinv, int32_t* fmt_out,
                         uint32_t* partials, int rule, cudaStream_t s) {
    constexpr int ES = ElemBytes<XT>::value;
    const int vb = vector_bytes(x, 0, q, ES);
    if (vb == 32) return pipeline_launch<XT, 32>(x, numel, q, sinv, fmt_out, partials, rule, s);
    if (vb == 16) return pipeline_launch<XT, 16>(x, numel, q, sinv, fmt_out, partials, rule, s);
    return pipeline_launch<XT, 0>(x, numel, q, sinv, fmt_out, partials, rule, s);
}

template <int YT>
fp8q_status run_pipeline_decode(const uint8_t* q, int64_t numel, const float* sinv, const int32_t* fmt_in,
                                void* y, cudaStream_t s) {
    const int ys = YT == kF32 ? 4 : 2;
    const bool vec = (uintptr_t)q % 16 == 0 && (uintptr_t)y % 16 == 0;
    const int64_t units = vec ? numel / 16 : numel;
    int64_t want = (units + kPtThreads * 4 - 1) / (kPtThreads * 4);
    const int64_t cap = (int64_t)sm_count() * 8;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    (void)ys;
    const cudaError_t err = vec
        ? launch_kernel(pipeline_decode_kernel<YT, true>, dim3((unsigned)want), dim3(kPtThreads), s, q, numel, sinv, fmt_in, y)
        : launch_kernel(pipeline_decode_kernel<YT, false>, dim3((unsigned)want), dim3(kPtThreads), s, q, numel, sinv, fmt_in, y);
    return cuda_status(err);
}

fp8q_status launch_per_channel(const void* x, int xt, int64_t rows, int64_t cols, int fmt,
                               uint8_t* q, float* sinv, int rule, cudaStream_t s) {
    const uint8_t* xb = static_cast<const uint8_t*>(x);
    switch (xt) {
    case kF32: return per_channel_fmt<kF32>(xb, fmt, q, sinv, rows, cols, rule, s);
    case kF16: return per_channel_fmt<kF16>(xb, fmt, q, sinv, rows, cols, rule, s);
    default: return per_channel_fmt<kBF16>(xb, fmt, q, sinv, rows, cols, rule, s);
    }
}

fp8q_status launch_per_tensor(const void* x, int xt, int64_t numel, int fmt, uint8_t* q,
                              float* sinv, uint32_t* partials, int rule, cudaStream_t s) {
    const uint8_t* xb = static_cast<const uint8_t*>(x);
    switch (xt) {
    case kF32: return per_tensor_fmt<kF32>(xb, fmt, numel, q, sinv, partials, rule, s);
    case kF16: return per_tensor_fmt<kF16>(xb, fmt, numel, q, sinv, partials, rule, s);
    default: return per_tensor_fmt<kBF16>(xb, fmt, numel, q, sinv, partials, rule, s);
    }
}

// amax pass + finish: amax_bits[0] = magnitude bits of max |x|
template <int XT, int VB>
fp8q_status tensor_amax_launch(const uint8_t* x, int64_t numel, uint32_t* partials, uint32_t* amax_bits,
                               cudaStream_t s) {
    constexpr int ES = ElemBytes<XT>::value;
    const int64_t units = VB > 0 ? numel * ES / VB : numel;
    int64_t want = (units + kPtThreads * kPtUnroll - 1) / (kPtThreads * kPtUnroll);
    static const int per_sm = resident_blocks_per_sm(tensor_amax_kernel<XT, VB>, kPtThreads);
    int64_t cap = (int64_t)sm_count() * min(per_sm, 8);
    if (cap > kMaxPartials) cap = kMaxPartials;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    const int grid = (int)want;
    cudaError_t err = launch_kernel(tensor_amax_kernel<XT, VB>, dim3(grid), dim3(kPtThreads), s, x, numel, partials);
    if (err != cudaSuccess) return FP8Q_ERR_CUDA;
    err = launch_kernel(amax_finish_kernel, dim3(1), dim3(kPtThreads), s, (const uint32_t*)partials, grid, amax_bits);
    return cuda_status(err);
}

// the cast pass with an amax given on the device (one "partial")
template <int XT, int FMT, int VB>
fp8q_status cast_with_amax_launch(const uint8_t* x, int64_t numel, uint8_t* q, float* sinv,
                                  const uint32_t* amax_bits, int rule, cudaStream_t s) {
    constexpr int ES = ElemBytes<XT>::value;
    const int64_t units = VB > 0 ? numel * ES / VB : numel;
    int64_t want = (units + kPtThreads * kPtUnroll - 1) / (kPtThreads * kPtUnroll);  // >= 1 CTA even when empty
    static const int per_sm = resident_blocks_per_sm(tensor_cast_kernel<XT, FMT, VB>, kPtThreads);
    const int64_t cap = (int64_t)sm_count() * min(per_sm, 8);
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    const cudaError_t err = launch_kernel(tensor_cast_kernel<XT, FMT, VB>, dim3((unsigned)want), dim3(kPtThreads), s,
                                          x, numel, q, sinv, amax_bits, 1, rule);
    return cuda_status(err);
}

template <int XT>
fp8q_status run_tensor_amax(const uint8_t* x, int64_t numel, uint32_t* partials, uint32_t* amax_bits,
                            cudaStream_t s) {
    // the amax pass only reads x: its own alignment picks the vector width
    const int vb = vector_bytes(x, 0, x, 1);
    if (vb == 32) return tensor_amax_launch<XT, 32>(x, numel, partials, amax_bits, s);
    if (vb == 16) return tensor_amax_launch<XT, 16>(x, numel, partials, amax_bits, s);
    return tensor_amax_launch<XT, 0>(x, numel, partials, amax_bits, s);
}

template <int XT, int FMT>
fp8q_status run_cast_with_amax(const uint8_t* x, int64_t numel, uint8_t* q, float* sinv, const uint32_t* amax_bits,
                               int rule, cudaStream_t s) {
    constexpr int ES = ElemBytes<XT>::value;
    const int vb = vector_bytes(x, 0, q, ES);
    if (vb == 32) return cast_with_amax_launch<XT, FMT, 32>(x, numel, q, sinv, amax_bits, rule, s);
    if (vb == 16) return cast_with_amax_launch<XT, FMT, 16>(x, numel, q, sinv, amax_bits, rule, s);
    return cast_with_amax_launch<XT, FMT, 0>(x, numel, q, sinv, amax_bits, rule, s);
}

fp8q_status launch_cast_pipeline(const void* x, int xt, int64_t numel, uint8_t* q, float* sinv,
                                 int32_t* fmt_out, uint32_t* partials, int rule, cudaStream_t s) {
    const uint8_t* xb = static_cast<const uint8_t*>(x);
    switch (xt) {
    case kF32: return run_pipeline<kF32>(xb, numel, q, sinv, fmt_out, partials, rule, s);
    case kF16: return run_pipeline<kF16>(xb, numel, q, sinv, fmt_out, partials, rule, s);
    default: return run_pipeline<kBF16>(xb, numel, q, sinv, fmt_out, partials, rule, s);
    }
}

fp8q_status launch_cast_from_pipeline(const uint8_t* q, int64_t numel, const float* sinv, const int32_t* fmt_in,
                                      int yt, void* y, cudaStream_t s) {
    switch (yt) {
    case kF32: return run_pipeline_decode<kF32>(q, numel, sinv, fmt_in, y, s);
    case kF16: return run_pipeline_decode<kF16>(q, numel, sinv, fmt_in, y, s);
    default: return run_pipeline_decode<kBF16>(q, numel, sinv, fmt_in, y, s);
    }
}

fp8q_status launch_tensor_amax(const void* x, int xt, int64_t numel, uint32_t* partials, uint32_t* amax_bits,
                               cudaStream_t s) {
    const uint8_t* xb = static_cast<const uint8_t*>(x);
    switch (xt) {
    case kF32: return run_tensor_amax<kF32>(xb, numel, partials, amax_bits, s);
    case kF16: return run_tensor_amax<kF16>(xb, numel, partials, amax_bits, s);
    default: return run_tensor_amax<kBF16>(xb, numel, partials, amax_bits, s);
    }
}

fp8q_status launch_cast_with_amax(const void* x, int xt, int64_t numel, int fmt, const uint32_t* amax_bits,
                                  uint8_t* q, float* sinv, int rule, cudaStream_t s) {
    const uint8_t* xb = static_cast<const uint8_t*>(x);
    if (fmt == kE4M3) {
        switch (xt) {
        case kF32: return run_cast_with_amax<kF32, kE4M3>(xb, numel, q, sinv, amax_bits, rule, s);
        case kF16: return run_cast_with_amax<kF16, kE4M3>(xb, numel, q, sinv, amax_bits, rule, s);
        default: return run_cast_with_amax<kBF16, kE4M3>(xb, numel, q, sinv, amax_bits, rule, s);
        }
    }
    switch (xt) {
    case kF32: return run_cast_with_amax<kF32, kE5M2>(xb, numel, q, sinv, amax_bits, rule, s);
    case kF16: return run_cast_with_amax<kF16, kE5M2>(xb, numel, q, sinv, amax_bits, rule, s);
    default: return run_cast_with_amax<kBF16, kE5M2>(xb, numel, q, sinv, amax_bits, rule, s);
    }
}

}  // namespace fp8q
