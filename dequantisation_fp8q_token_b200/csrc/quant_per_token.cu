// quant_per_token.cu -- per-token group quantisation (DeepEP "5 Utils",
// per_token_cast_to_fp8): 1 x G groups along each row, one fp32 scale per
// group, amax clamped at 1e-4, scale = FMAX / amax, scale_inv = amax / FMAX.
//
// Layout: because n % G == 0, group g of the flattened [m][n/G] grid covers
// elements [g*G, (g+1)*G) of x and q and owns scale_inv[g]; the kernel walks
// groups as one flat sequence.
//
// Vector kernel: a group is held by LANES = min(32, G / EPV) consecutive
// lanes, each with VPL 16-byte vectors (EPV elements per vector).  For the
// pages' bf16 G = 128 that is a half warp with one 16-byte load per lane:
// every warp-wide load covers 512 contiguous bytes.  Each thread keeps
// kTokUnroll groups' loads in flight before reducing, the amax is an
// integer max on magnitude bits (NaN-propagating) finished with xor
// shuffles inside the lane segment, and each lane stores its EPV codes in
// one store.
#include "fp8q_device.cuh"
#include "fp8q_internal.h"

namespace fp8q {
namespace {

constexpr int kTokThreads = 256;
constexpr int kTokUnroll = 4;

template <int XT, int G>
struct TokCfg {
    static constexpr int ES = ElemBytes<XT>::value;
    static constexpr int EPV = 16 / ES;
    static constexpr int LANES = (G / EPV) < 32 ? (G / EPV) : 32;
    static constexpr int VPL = G / (EPV * LANES);
    static constexpr int SEGS = 32 / LANES;
    static constexpr int GPI = (kTokThreads / 32) * SEGS;  // groups per CTA iteration
    static constexpr int GPC = GPI * kTokUnroll;            // groups per CTA
};

// encode one 16-byte input vector (already widened on the fly) and store its codes
template <int XT, int FMT, bool FIX>
__device__ __forceinline__ void encode_store_vec(uint4 v, float scale, uint8_t* dst) {
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

template <int XT, int FMT, int G>
__global__ void __launch_bounds__(kTokThreads)
per_token_vec_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ q,
                     float* __restrict__ sinv, int64_t ngroups) {
    using C = TokCfg<XT, G>;
    constexpr int U = kTokUnroll;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int seg = lane / C::LANES;
    const int sl = lane % C::LANES;
    const int64_t g0 = (int64_t)blockIdx.x * C::GPC + warp * C::SEGS + seg;

    uint4 v[U][C::VPL];
#pragma unroll
    for (int k = 0; k < U; ++k) {
        const int64_t g = g0 + (int64_t)k * C::GPI;
#pragma unroll
        for (int j = 0; j < C::VPL; ++j) {
            const int64_t e = g * G + (int64_t)(j * C::LANES + sl) * C::EPV;
            v[k][j] = g < ngroups ? ld_stream_v4(x + e * C::ES) : make_uint4(0u, 0u, 0u, 0u);
        }
    }

#pragma unroll
    for (int k = 0; k < U; ++k) {
        const int64_t g = g0 + (int64_t)k * C::GPI;
        uint32_t m;
        if (XT == kF32) {
            m = 0u;
#pragma unroll
            for (int j = 0; j < C::VPL; ++j) m = max(m, vec_absmax_bits<kF32>(v[k][j]));
        } else {
            uint32_t p = 0u;
#pragma unroll
            for (int j = 0; j < C::VPL; ++j) p = max_u16x2(p, vec_absmax_packed16(v[k][j]));
            m = packed16_to_f32bits<XT>(p);
        }
#pragma unroll
        for (int off = C::LANES / 2; off > 0; off >>= 1)
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));

        float amax = __uint_as_float(m);
        if (amax < 1e-4f) amax = 1e-4f;  // clamp(1e-4); a NaN amax stays NaN
        const float scale = __fdiv_rn(fp8_max<FMT>(), amax);
        if (g < ngroups) {
            if (sl == 0) sinv[g] = __fdiv_rn(amax, fp8_max<FMT>());
            // finite x with a finite scale never overflows, and NaN/Inf inputs
            // give NaN or zero products: the hardware codes are already final
#pragma unroll
            for (int j = 0; j < C::VPL; ++j) {
                const int64_t e = g * G + (int64_t)(j * C::LANES + sl) * C::EPV;
                encode_store_vec<XT, FMT, false>(v[k][j], scale, q + e);
            }
        }
    }
}

// any group size dividing n, any element-aligned pointers: one warp per group
template <int XT, int FMT>
__global__ void __launch_bounds__(256)
per_token_generic_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ q,
                         float* __restrict__ sinv, int64_t ngroups, int G) {
    constexpr int ES = ElemBytes<XT>::value;
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); g < ngroups;
         g += stride) {
        const int64_t base = g * G;
        uint32_t m = 0u;
        for (int k = lane; k < G; k += 32) m = max(m, elem_abs_bits<XT>(x + (base + k) * ES));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        float amax = __uint_as_float(m);
        if (amax < 1e-4f) amax = 1e-4f;
        const float scale = __fdiv_rn(fp8_max<FMT>(), amax);
        if (lane == 0) sinv[g] = __fdiv_rn(amax, fp8_max<FMT>());
        for (int k = lane; k < G; k += 32) {
            const float f = __fmul_rn(elem_load<XT>(x + (base + k) * ES), scale);
            q[base + k] = (uint8_t)(enc2<FMT>(f, 0.0f) & 0xFFu);
        }
    }
}

template <int XT, int FMT, int G>
fp8q_status run_vec(const void* x, uint8_t* q, float* sinv, int64_t ngroups, cudaStream_t s) {
    using C = TokCfg<XT, G>;
    const int64_t blocks = (ngroups + C::GPC - 1) / C::GPC;
    if (blocks > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
    per_token_vec_kernel<XT, FMT, G><<<(unsigned)blocks, kTokThreads, 0, s>>>(
        static_cast<const uint8_t*>(x), q, sinv, ngroups);
    return cuda_status(cudaGetLastError());
}

template <int XT, int FMT>
fp8q_status run_generic(const void* x, uint8_t* q, float* sinv, int64_t ngroups, int group,
                        cudaStream_t s) {
    const int64_t want = (ngroups + 7) / 8;
    const int blocks = (int)(want < (int64_t)sm_count() * 16 ? want : (int64_t)sm_count() * 16);
    per_token_generic_kernel<XT, FMT><<<blocks, 256, 0, s>>>(static_cast<const uint8_t*>(x), q, sinv,
                                                            ngroups, group);
    return cuda_status(cudaGetLastError());
}

template <int XT, int FMT>
fp8q_status dispatch_group(const void* x, uint8_t* q, float* sinv, int64_t ngroups, int group,
                           cudaStream_t s) {
    switch (group) {
    case 16: return run_vec<XT, FMT, 16>(x, q, sinv, ngroups, s);
    case 32: return run_vec<XT, FMT, 32>(x, q, sinv, ngroups, s);
    case 64: return run_vec<XT, FMT, 64>(x, q, sinv, ngroups, s);
    case 128: return run_vec<XT, FMT, 128>(x, q, sinv, ngroups, s);
    case 256: return run_vec<XT, FMT, 256>(x, q, sinv, ngroups, s);
    case 512: return run_vec<XT, FMT, 512>(x, q, sinv, ngroups, s);
    case 1024: return run_vec<XT, FMT, 1024>(x, q, sinv, ngroups, s);
    default: return run_generic<XT, FMT>(x, q, sinv, ngroups, group, s);
    }
}

template <int XT>
fp8q_status dispatch_fmt(const void* x, int fmt, uint8_t* q, float* sinv, int64_t ngroups,
                         int group, bool vec, cudaStream_t s) {
    if (fmt == kE4M3)
        return vec ? dispatch_group<XT, kE4M3>(x, q, sinv, ngroups, group, s)
                   : run_generic<XT, kE4M3>(x, q, sinv, ngroups, group, s);
    return vec ? dispatch_group<XT, kE5M2>(x, q, sinv, ngroups, group, s)
               : run_generic<XT, kE5M2>(x, q, sinv, ngroups, group, s);
}

}  // namespace

fp8q_status launch_per_token(const void* x, int xt, int64_t m, int64_t n, int group, int fmt,
                             uint8_t* q, float* sinv, cudaStream_t s) {
    const int64_t ngroups = m * (n / group);
    if (ngroups == 0) return FP8Q_OK;
    const int es = xt == kF32 ? 4 : 2;
    const int epv = 16 / es;
    const bool pow2 = group >= 16 && group <= 1024 && (group & (group - 1)) == 0;
    // vector path: 16-byte aligned input, codes stored epv bytes at a time
    const bool vec = pow2 && ((uintptr_t)x % 16 == 0) && ((uintptr_t)q % epv == 0);
    switch (xt) {
    case kF32: return dispatch_fmt<kF32>(x, fmt, q, sinv, ngroups, group, vec, s);
    case kF16: return dispatch_fmt<kF16>(x, fmt, q, sinv, ngroups, group, vec, s);
    default: return dispatch_fmt<kBF16>(x, fmt, q, sinv, ngroups, group, vec, s);
    }
}

}  // namespace fp8q
