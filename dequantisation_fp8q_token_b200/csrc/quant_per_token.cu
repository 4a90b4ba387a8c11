// quant_per_token.cu -- per-token group quantisation (DeepEP "5 Utils",
// per_token_cast_to_fp8): 1 x G groups along each row, one fp32 scale per
// group, amax clamped at 1e-4, scale = FMAX / amax, scale_inv = amax / FMAX.
//
// Layout: because n % G == 0, group g of the flattened [m][n/G] grid covers
// elements [g*G, (g+1)*G) of x and q and owns scale_inv[g]; the kernel walks
// groups as one flat sequence.
//
// Vector kernel: a group is held by LANES consecutive lanes, each with VPL
// vectors of VB bytes (EPV elements each); vector j of lane l covers
// elements (j * LANES + l) * EPV .. + EPV of its group, so every warp-wide
// load is LANES * VB contiguous bytes per group and uses whole sectors.  For
// the pages' bf16 G = 128 with 256-bit loads (VB = 32) that is 8 lanes x one
// vector: a warp holds 4 groups, each warp-wide load 4 x 256 contiguous bytes.
//   - amax: NaN-propagating magnitude max (packed for 16-bit types), then
//     xor shuffles inside the lane segment;
//   - scales: the warp's SEGS amaxes are gathered into lanes 0..SEGS-1, so
//     the two IEEE divisions run once per warp for all its groups; each lane
//     then fetches its group's scale, and lanes 0..SEGS-1 store SEGS
//     consecutive scale_inv values in one coalesced store;
//   - encode: four fp32 products -> one 32-bit word of codes, one store per
//     vector.
// Each CTA loads kTokUnroll batches of GPB groups before converting any.
#include "fp8q_device.cuh"
#include "fp8q_internal.h"

namespace fp8q {
namespace {

constexpr int kTokThreads = 256;
#ifndef FP8Q_TOK_UNROLL
#define FP8Q_TOK_UNROLL 2
#endif
#ifndef FP8Q_TOK_VPL
#define FP8Q_TOK_VPL 1
#endif
#ifndef FP8Q_TOK_V32
#define FP8Q_TOK_V32 1  // 32-byte vectors (256-bit loads) where the pointers allow
#endif
constexpr int kTokUnroll = FP8Q_TOK_UNROLL;  // batches per CTA
constexpr int kTokVpl = FP8Q_TOK_VPL;        // target vectors per lane per group

template <int XT, int G, int VB>
struct TokCfg {
    static constexpr int ES = ElemBytes<XT>::value;
    static constexpr int EPV = VB / ES;                    // elements per vector (VB bytes)
    static constexpr int NV = G / EPV;                     // vectors per group
    static constexpr int LANES = NV / kTokVpl < 1 ? 1 : (NV / kTokVpl > 32 ? 32 : NV / kTokVpl);
    static constexpr int VPL = NV / LANES;                 // vectors per lane
    static constexpr int SEGS = 32 / LANES;                // groups per warp
    static constexpr int GPB = (kTokThreads / 32) * SEGS;  // groups per CTA batch
    static constexpr int WPV = VB / 4;                     // 32-bit words per vector
};

template <int XT, int G, int VB>
__device__ __forceinline__ void load_batch(const uint8_t* __restrict__ x, int64_t ngroups, int64_t bt,
                                           int gw, int sl, Vec<VB> (&v)[TokCfg<XT, G, VB>::VPL]) {
    using C = TokCfg<XT, G, VB>;
    const int64_t g = bt * C::GPB + gw;
#pragma unroll
    for (int j = 0; j < C::VPL; ++j) {
        const int64_t e = g * G + (int64_t)(j * C::LANES + sl) * C::EPV;
        if (g < ngroups) v[j] = load_vec<VB>(x + e * C::ES);
        else
#pragma unroll
            for (int i = 0; i < C::WPV; ++i) v[j].w[i] = 0u;
    }
}

template <int XT, int FMT, int G, int VB>
__device__ __forceinline__ void process_batch(const Vec<VB> (&v)[TokCfg<XT, G, VB>::VPL], uint8_t* __restrict__ q,
                                              float* __restrict__ sinv, int64_t ngroups, int64_t bt,
                                              int seg, int sl, int lane, int warp, int rule) {
    using C = TokCfg<XT, G, VB>;
    // magnitude maximum of this lane's elements
    uint32_t m = vec_absmax<XT, VB>(v[0]);
#pragma unroll
    for (int j = 1; j < C::VPL; ++j) m = absmax2<XT>(m, vec_absmax<XT, VB>(v[j]));
#pragma unroll
    for (int off = C::LANES / 2; off > 0; off >>= 1) m = absmax2<XT>(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    const uint32_t bits = absmax_bits<XT>(m);
    // the warp's SEGS scales, one group per lane, computed once
    float amax = __uint_as_float(__shfl_sync(0xFFFFFFFFu, bits, (lane % C::SEGS) * C::LANES));
    if (amax < 1e-4f) amax = 1e-4f;  // clamp(1e-4); a NaN amax stays NaN
    const float scale_l = scale_from_amax<FMT>(amax, rule);
    const float sinv_l = scale_inv_from_amax<FMT>(amax, rule);
    const float scale = __shfl_sync(0xFFFFFFFFu, scale_l, seg);
    const int64_t gbase = bt * C::GPB + (int64_t)warp * C::SEGS;
    if (lane < C::SEGS && gbase + lane < ngroups) sinv[gbase + lane] = sinv_l;
    // finite x with a finite scale never overflows, and NaN/Inf inputs give
    // NaN or zero products: the hardware codes are already final
    const int64_t g = gbase + seg;
    if (g < ngroups) {
#pragma unroll
        for (int j = 0; j < C::VPL; ++j) {
            const int64_t e = g * G + (int64_t)(j * C::LANES + sl) * C::EPV;
            encode_store_vec<XT, FMT, VB, false>(v[j], scale, q + e);
        }
    }
}

// one CTA per kTokUnroll consecutive batches: all their loads are issued
// before any batch is converted
template <int XT, int FMT, int G, int VB>
__global__ void __launch_bounds__(kTokThreads)
per_token_vec_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ q,
                     float* __restrict__ sinv, int64_t ngroups, int64_t nbatch, int rule) {
    using C = TokCfg<XT, G, VB>;
    pdl_trigger();
    const int64_t b0 = (int64_t)blockIdx.x * kTokUnroll;
    if (threadIdx.x == 0) {
        // this CTA's groups are one contiguous range of x (G * ES bytes each,
        // a multiple of 16, from a VB-aligned base)
        const int64_t g0 = b0 * C::GPB;
        const int64_t g1 = (b0 + kTokUnroll) * C::GPB < ngroups ? (b0 + kTokUnroll) * C::GPB : ngroups;
        if (g1 > g0) prefetch_l2_bulk(x + g0 * G * C::ES, (uint32_t)((g1 - g0) * G * C::ES));
    }
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int seg = lane / C::LANES;
    const int sl = lane % C::LANES;
    const int gw = warp * C::SEGS + seg;
    Vec<VB> v[kTokUnroll][C::VPL];
#pragma unroll
    for (int u = 0; u < kTokUnroll; ++u) load_batch<XT, G, VB>(x, ngroups, b0 + u, gw, sl, v[u]);
#pragma unroll
    for (int u = 0; u < kTokUnroll; ++u)
        if (b0 + u < nbatch) process_batch<XT, FMT, G, VB>(v[u], q, sinv, ngroups, b0 + u, seg, sl, lane, warp, rule);
}

// any group size dividing n, any element-aligned pointers: one warp per group
template <int XT, int FMT>
__global__ void __launch_bounds__(256)
per_token_generic_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ q,
                         float* __restrict__ sinv, int64_t ngroups, int G, int rule) {
    pdl_begin();
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
        const float scale = scale_from_amax<FMT>(amax, rule);
        if (lane == 0) sinv[g] = scale_inv_from_amax<FMT>(amax, rule);
        for (int k = lane; k < G; k += 32) {
            const float f = __fmul_rn(elem_load<XT>(x + (base + k) * ES), scale);
            q[base + k] = (uint8_t)(enc2<FMT>(f, 0.0f) & 0xFFu);
        }
    }
}

template <int XT, int FMT, int G, int VB>
fp8q_status run_vec(const void* x, uint8_t* q, float* sinv, int64_t ngroups, int rule, cudaStream_t s) {
    using C = TokCfg<XT, G, VB>;
    const int64_t nbatch = (ngroups + C::GPB - 1) / C::GPB;
    const int64_t grid = (nbatch + kTokUnroll - 1) / kTokUnroll;
    if (grid > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
    const cudaError_t err = launch_kernel(per_token_vec_kernel<XT, FMT, G, VB>, dim3((unsigned)grid), dim3(kTokThreads), s,
                                          static_cast<const uint8_t*>(x), q, sinv, ngroups, nbatch, rule);
    return cuda_status(err);
}

template <int XT, int FMT>
fp8q_status run_generic(const void* x, uint8_t* q, float* sinv, int64_t ngroups, int group, int rule,
                        cudaStream_t s) {
    const int64_t want = (ngroups + 7) / 8;
    const int blocks = (int)(want < (int64_t)sm_count() * 16 ? want : (int64_t)sm_count() * 16);
    const cudaError_t err = launch_kernel(per_token_generic_kernel<XT, FMT>, dim3(blocks), dim3(256), s,
                                          static_cast<const uint8_t*>(x), q, sinv, ngroups, group, rule);
    return cuda_status(err);
}

template <int XT, int FMT, int VB>
fp8q_status dispatch_group(const void* x, uint8_t* q, float* sinv, int64_t ngroups, int group, int rule,
                           cudaStream_t s) {
    switch (group) {
    case 16: return run_vec<XT, FMT, 16, VB>(x, q, sinv, ngroups, rule, s);
    case 32: return run_vec<XT, FMT, 32, VB>(x, q, sinv, ngroups, rule, s);
    case 64: return run_vec<XT, FMT, 64, VB>(x, q, sinv, ngroups, rule, s);
    case 128: return run_vec<XT, FMT, 128, VB>(x, q, sinv, ngroups, rule, s);
    case 256: return run_vec<XT, FMT, 256, VB>(x, q, sinv, ngroups, rule, s);
    case 512: return run_vec<XT, FMT, 512, VB>(x, q, sinv, ngroups, rule, s);
    case 1024: return run_vec<XT, FMT, 1024, VB>(x, q, sinv, ngroups, rule, s);
    default: return run_generic<XT, FMT>(x, q, sinv, ngroups, group, rule, s);
    }
}

// vb: 32 or 16 (vector bytes the pointers allow), 0 for the generic kernel
template <int XT, int FMT>
fp8q_status dispatch_vb(const void* x, uint8_t* q, float* sinv, int64_t ngroups, int group, int vb, int rule,
                        cudaStream_t s) {
#if FP8Q_TOK_V32
    if (vb == 32) return dispatch_group<XT, FMT, 32>(x, q, sinv, ngroups, group, rule, s);
#endif
    if (vb >= 16) return dispatch_group<XT, FMT, 16>(x, q, sinv, ngroups, group, rule, s);
    return run_generic<XT, FMT>(x, q, sinv, ngroups, group, rule, s);
}

template <int XT>
fp8q_status dispatch_fmt(const void* x, int fmt, uint8_t* q, float* sinv, int64_t ngroups,
                         int group, int vb, int rule, cudaStream_t s) {
    if (fmt == kE4M3) return dispatch_vb<XT, kE4M3>(x, q, sinv, ngroups, group, vb, rule, s);
    return dispatch_vb<XT, kE5M2>(x, q, sinv, ngroups, group, vb, rule, s);
}

}  // namespace

fp8q_status launch_per_token(const void* x, int xt, int64_t m, int64_t n, int group, int fmt,
                             uint8_t* q, float* sinv, int rule, cudaStream_t s) {
    const int64_t ngroups = m * (n / group);
    if (ngroups == 0) return FP8Q_OK;
    const int es = xt == kF32 ? 4 : 2;
    const bool pow2 = group >= 16 && group <= 1024 && (group & (group - 1)) == 0;
    // vector paths: VB-byte aligned input, codes stored VB / es bytes at a time
    int vb = 0;
    if (pow2 && (uintptr_t)x % 32 == 0 && (uintptr_t)q % (32 / es) == 0) vb = 32;
    else if (pow2 && (uintptr_t)x % 16 == 0 && (uintptr_t)q % (16 / es) == 0) vb = 16;
    switch (xt) {
    case kF32: return dispatch_fmt<kF32>(x, fmt, q, sinv, ngroups, group, vb, rule, s);
    case kF16: return dispatch_fmt<kF16>(x, fmt, q, sinv, ngroups, group, vb, rule, s);
    default: return dispatch_fmt<kBF16>(x, fmt, q, sinv, ngroups, group, vb, rule, s);
    }
}

}  // namespace fp8q
