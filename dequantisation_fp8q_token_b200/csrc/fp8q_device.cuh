// fp8q_device.cuh -- device-side building blocks shared by the libfp8q kernels.
//
// Conversions use the packed sm_89+/sm_100a cvt instructions:
//   cvt.rn.satfinite.{e4m3x2,e5m2x2}.f32  fp32 pair -> two fp8 codes, RNE
//   cvt.rn.f16x2.{e4m3x2,e5m2x2}          two fp8 codes -> f16x2, exact
// The encode saturates in hardware; torch's .to(float8_*) does not, so the
// few cases where a saturating result would differ are fixed up explicitly
// (fix_code).  Those cases only arise when an amax is NaN (replaced by 1 in
// the ColossalAI casts) or when the scale overflowed to Inf; for finite data
// with a finite scale |x * scale| <= FMAX * (1 + 2^-23), which no rounding
// pushes past the overflow threshold.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#ifndef FP8Q_PDL
#define FP8Q_PDL 1
#endif

namespace fp8q {

enum : int { kE4M3 = 0, kE5M2 = 1 };
enum : int { kF32 = 0, kF16 = 1, kBF16 = 2 };
enum : int { kGranTensor = 0, kGranRow = 1, kGranGroup = 2, kGranBlock = 3 };

template <int XT> struct ElemBytes { static constexpr int value = XT == kF32 ? 4 : 2; };

template <int FMT> __device__ __forceinline__ float fp8_max() {
    return FMT == kE4M3 ? 448.0f : 57344.0f;
}

// ---------------------------------------------------------------------------
// programmatic dependent launch.  Every kernel calls pdl_begin() before it
// touches global memory: it lets the next kernel on the stream be scheduled
// once all of this grid's CTAs have started (so the next grid only fills SMs
// that this one's tail leaves idle), then waits until the previous grid on
// the stream has completed and its writes are visible.  Without a
// programmatic predecessor the wait returns at once.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_begin() {
#if FP8Q_PDL
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
}
// The same in two halves, for kernels that warm L2 with their first input
// lines in between (prefetch_l2 / prefetch_l2_bulk): a prefetch brings a
// line into L2 only, and L2 is where every write lands, so the loads issued
// after pdl_wait still see all writes of the kernel before.
__device__ __forceinline__ void pdl_trigger() {
#if FP8Q_PDL
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
}
__device__ __forceinline__ void pdl_wait() {
#if FP8Q_PDL
    asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
}
// the line holding p, into L2 (p inside a live allocation)
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" :: "l"(p));
}
// [p, p + bytes) into L2: p 16-byte aligned, bytes a positive multiple of 16,
// the whole range inside one live allocation
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(p), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------------------
// scale rules: rule 0 divides once (fl(FMAX / amax), fl(amax / FMAX)); rule 1
// reproduces torch's evaluation of the same expressions on a CUDA tensor
// (fl(fl(1 / amax) * FMAX) and fl(amax * fl(1 / FMAX))).
// ---------------------------------------------------------------------------
template <int FMT> __device__ __forceinline__ float scale_from_amax(float amax, int rule) {
    if (rule) return __fmul_rn(__fdiv_rn(1.0f, amax), FMT == 0 ? 448.0f : 57344.0f);
    return __fdiv_rn(FMT == 0 ? 448.0f : 57344.0f, amax);
}
template <int FMT> __device__ __forceinline__ float scale_inv_from_amax(float amax, int rule) {
    if (rule) return __fmul_rn(amax, __fdiv_rn(1.0f, FMT == 0 ? 448.0f : 57344.0f));
    return __fdiv_rn(amax, FMT == 0 ? 448.0f : 57344.0f);
}

// ---------------------------------------------------------------------------
// global memory access
// ---------------------------------------------------------------------------
// Streaming 16-byte load through the non-coherent path, not kept in L1.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
    uint2 r;
    asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
    uint32_t r;
    asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}
// L2 eviction-priority policies (createpolicy) and a streaming load that
// carries one: evict_last keeps a line in L2 ahead of normal traffic,
// evict_first lets it go first.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint4 ld_stream_v4_policy(const void* p, uint64_t policy) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p), "l"(policy));
    return r;
}
// 256-bit accesses (sm_100): 32 contiguous bytes per thread, 32-byte aligned
struct U8x32 { uint32_t w[8]; };
__device__ __forceinline__ U8x32 ld_stream_v8(const void* p) {
    U8x32 r;
    asm("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]),
          "=r"(r.w[4]), "=r"(r.w[5]), "=r"(r.w[6]), "=r"(r.w[7]) : "l"(p));
    return r;
}
__device__ __forceinline__ void st_v8(void* p, const uint32_t (&w)[8]) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 :: "l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]),
                    "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]) : "memory");
}
__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ void st_v2(void* p, uint2 v) {
    asm volatile("st.global.v2.u32 [%0], {%1,%2};" :: "l"(p), "r"(v.x), "r"(v.y) : "memory");
}
__device__ __forceinline__ void st_u32(void* p, uint32_t v) {
    asm volatile("st.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------
// |x| maxima as integer maxima on magnitude bits.  For non-negative IEEE
// values the bit patterns order like the values, and every NaN pattern lies
// above +Inf, so an integer max propagates NaN (fmaxf would drop it).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// magnitude-bits maximum of one 16-byte vector, returned as fp32 magnitude bits
template <int XT> __device__ __forceinline__ uint32_t vec_absmax_bits(uint4 v);

template <> __device__ __forceinline__ uint32_t vec_absmax_bits<kF32>(uint4 v) {
    uint32_t a = max(v.x & 0x7FFFFFFFu, v.y & 0x7FFFFFFFu);
    uint32_t b = max(v.z & 0x7FFFFFFFu, v.w & 0x7FFFFFFFu);
    return max(a, b);
}
// 16-bit types: packed max over the 8 halves, result still packed
__device__ __forceinline__ uint32_t vec_absmax_packed16(uint4 v) {
    uint32_t a = max_u16x2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
    uint32_t b = max_u16x2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
    return max_u16x2(a, b);
}
// packed 16-bit magnitude maximum -> fp32 magnitude bits (exact, monotone)
template <int XT> __device__ __forceinline__ uint32_t packed16_to_f32bits(uint32_t p) {
    uint32_t h = max(p & 0xFFFFu, p >> 16);
    if (XT == kBF16) return h << 16;
    return __float_as_uint(__half2float(__ushort_as_half((unsigned short)h)));
}
template <> __device__ __forceinline__ uint32_t vec_absmax_bits<kBF16>(uint4 v) {
    return packed16_to_f32bits<kBF16>(vec_absmax_packed16(v));
}
template <> __device__ __forceinline__ uint32_t vec_absmax_bits<kF16>(uint4 v) {
    return packed16_to_f32bits<kF16>(vec_absmax_packed16(v));
}

// magnitude bits of one scalar element
template <int XT> __device__ __forceinline__ uint32_t elem_abs_bits(const uint8_t* p) {
    if (XT == kF32) return *reinterpret_cast<const uint32_t*>(p) & 0x7FFFFFFFu;
    uint32_t h = *reinterpret_cast<const uint16_t*>(p) & 0x7FFFu;
    if (XT == kBF16) return h << 16;
    return __float_as_uint(__half2float(__ushort_as_half((unsigned short)h)));
}
template <int XT> __device__ __forceinline__ float elem_load(const uint8_t* p) {
    if (XT == kF32) return *reinterpret_cast<const float*>(p);
    uint32_t h = *reinterpret_cast<const uint16_t*>(p);
    if (XT == kBF16) return __uint_as_float(h << 16);
    return __half2float(__ushort_as_half((unsigned short)h));
}

// ---------------------------------------------------------------------------
// widening a 32-bit word of two 16-bit elements to fp32 (exact)
// ---------------------------------------------------------------------------
template <int XT> __device__ __forceinline__ void widen2(uint32_t w, float& lo, float& hi) {
    if (XT == kBF16) {
        lo = __uint_as_float(w << 16);
        hi = __uint_as_float(w & 0xFFFF0000u);
    } else {
        __half2 h = *reinterpret_cast<__half2*>(&w);
        float2 f = __half22float2(h);
        lo = f.x;
        hi = f.y;
    }
}

// ---------------------------------------------------------------------------
// fp8 encode / decode
// ---------------------------------------------------------------------------
// two fp32 -> two fp8 codes, lo in bits 0..7, hi in bits 8..15 (RNE, saturating)
template <int FMT> __device__ __forceinline__ uint32_t enc2(float lo, float hi) {
    unsigned short r;
    if (FMT == kE4M3)
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    else
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// four fp32 -> four fp8 codes in one word, a in bits 0..7 ... d in bits 24..31
template <int FMT> __device__ __forceinline__ uint32_t enc4(float a, float b, float c, float d) {
    uint32_t r;
    if (FMT == kE4M3)
        asm("{\n.reg .b16 lo, hi;\n"
            "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n"
            "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n"
            "mov.b32 %0, {lo, hi};\n}"
            : "=r"(r) : "f"(a), "f"(b), "f"(c), "f"(d));
    else
        asm("{\n.reg .b16 lo, hi;\n"
            "cvt.rn.satfinite.e5m2x2.f32 lo, %2, %1;\n"
            "cvt.rn.satfinite.e5m2x2.f32 hi, %4, %3;\n"
            "mov.b32 %0, {lo, hi};\n}"
            : "=r"(r) : "f"(a), "f"(b), "f"(c), "f"(d));
    return r;
}

// Magnitude maxima that propagate NaN, on packed 16-bit pairs or fp32:
// max.NaN.xorsign.abs returns max(|a|, |b|) (NaN if either is NaN) with a
// sign bit we discard, so callers mask the result with 0x7FFF7FFF / 0x7FFFFFFF.
template <int XT> __device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b) {
    uint32_t d;
    if (XT == kBF16)
        asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    else if (XT == kF16)
        asm("max.NaN.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    else
        asm("max.NaN.xorsign.abs.f32 %0, %1, %2;" : "=f"(*reinterpret_cast<float*>(&d))
            : "f"(__uint_as_float(a)), "f"(__uint_as_float(b)));
    return d;
}

// non-saturating semantics for one value given the hardware code c:
//   NaN -> 0x7F, the positive NaN code of either format; e4m3fn: |v| > 464
//   (incl. Inf) -> NaN with v's sign; e5m2: |v| >= 61440 (incl. Inf) -> Inf
//   with v's sign.
// IEEE 754 leaves the sign of a NaN produced by arithmetic unspecified.  GPU
// arithmetic returns the canonical positive NaN, so on a CUDA device the
// pages' torch expressions (x * scale, then .to(float8_*)) give 0x7F for
// every NaN; writing 0x7F here keeps that whatever sign the product had.
template <int FMT> __device__ __forceinline__ uint32_t fix_code(float v, uint32_t c) {
    uint32_t u = __float_as_uint(v);
    uint32_t a = u & 0x7FFFFFFFu;
    uint32_t s = (u >> 24) & 0x80u;
    if (a > 0x7F800000u) return 0x7Fu;
    if (FMT == kE4M3) {
        if (a > 0x43E80000u) return 0x7Fu | s;
    } else {
        if (a >= 0x47700000u) return 0x7Cu | s;
    }
    return c;
}

template <int FMT, bool FIX>
__device__ __forceinline__ uint32_t enc2_sem(float lo, float hi) {
    uint32_t c = enc2<FMT>(lo, hi);
    if (FIX) {
        uint32_t c0 = fix_code<FMT>(lo, c & 0xFFu);
        uint32_t c1 = fix_code<FMT>(hi, c >> 8);
        c = c0 | (c1 << 8);
    }
    return c;
}

// two fp8 codes (lo byte, hi byte) -> two fp32 values, exact
template <int FMT> __device__ __forceinline__ float2 dec2(uint32_t two) {
    uint32_t h2;
    unsigned short t = (unsigned short)two;
    if (FMT == kE4M3)
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(t));
    else
        asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h2) : "h"(t));
    __half2 h = *reinterpret_cast<__half2*>(&h2);
    return __half22float2(h);
}

// two fp32 -> packed output pair of type YT (RNE); fp32 output returns via f
template <int YT> __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if (YT == kBF16) {
        __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&b);
    } else {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
}

// ---------------------------------------------------------------------------
// VB-byte vectors of high-precision elements (VB = 16 or 32)
// ---------------------------------------------------------------------------
template <int VB>
struct Vec {
    uint32_t w[VB / 4];
};

template <int VB>
__device__ __forceinline__ Vec<VB> load_vec(const uint8_t* p) {
    Vec<VB> v;
    if constexpr (VB == 32) {
        const U8x32 t = ld_stream_v8(p);
#pragma unroll
        for (int i = 0; i < 8; ++i) v.w[i] = t.w[i];
    } else {
        const uint4 t = ld_stream_v4(p);
        v.w[0] = t.x; v.w[1] = t.y; v.w[2] = t.z; v.w[3] = t.w;
    }
    return v;
}

template <int VB>
__device__ __forceinline__ Vec<VB> load_vec_policy(const uint8_t* p, uint64_t policy) {
    Vec<VB> v;
    if constexpr (VB == 32) {
        asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], %9;"
            : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]),
              "=r"(v.w[4]), "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7]) : "l"(p), "l"(policy));
    } else {
        const uint4 t = ld_stream_v4_policy(p, policy);
        v.w[0] = t.x; v.w[1] = t.y; v.w[2] = t.z; v.w[3] = t.w;
    }
    return v;
}

// unmasked NaN-propagating magnitude maximum over a vector (see absmax2)
template <int XT, int VB>
__device__ __forceinline__ uint32_t vec_absmax(const Vec<VB>& v) {
    uint32_t t = absmax2<XT>(v.w[0], v.w[1]);
#pragma unroll
    for (int i = 2; i < VB / 4; ++i) t = absmax2<XT>(t, v.w[i]);
    return t;
}

// result of absmax2 reductions -> fp32 magnitude bits
template <int XT>
__device__ __forceinline__ uint32_t absmax_bits(uint32_t m) {
    if (XT == kF32) return m & 0x7FFFFFFFu;
    return packed16_to_f32bits<XT>(m & 0x7FFF7FFFu);
}

// codes of one vector scaled by `scale`, stored in one access of VB / ES bytes;
// FIX applies the non-saturating NaN / Inf rules to every element
template <int XT, int FMT, int VB, bool FIX>
__device__ __forceinline__ void encode_store_vec(const Vec<VB>& v, float scale, uint8_t* dst) {
    constexpr int WPV = VB / 4;
    constexpr int NC = XT == kF32 ? WPV / 4 : WPV / 2;  // 32-bit words of codes
    uint32_t c[NC];
    if (XT == kF32) {
#pragma unroll
        for (int i = 0; i < NC; ++i) {
            const float a = __fmul_rn(__uint_as_float(v.w[4 * i]), scale);
            const float b = __fmul_rn(__uint_as_float(v.w[4 * i + 1]), scale);
            const float d = __fmul_rn(__uint_as_float(v.w[4 * i + 2]), scale);
            const float e = __fmul_rn(__uint_as_float(v.w[4 * i + 3]), scale);
            c[i] = FIX ? (enc2_sem<FMT, true>(a, b) | (enc2_sem<FMT, true>(d, e) << 16)) : enc4<FMT>(a, b, d, e);
        }
    } else {
#pragma unroll
        for (int i = 0; i < NC; ++i) {
            float a0, a1, b0, b1;
            widen2<XT>(v.w[2 * i], a0, a1);
            widen2<XT>(v.w[2 * i + 1], b0, b1);
            const float a = __fmul_rn(a0, scale), b = __fmul_rn(a1, scale);
            const float d = __fmul_rn(b0, scale), e = __fmul_rn(b1, scale);
            c[i] = FIX ? (enc2_sem<FMT, true>(a, b) | (enc2_sem<FMT, true>(d, e) << 16)) : enc4<FMT>(a, b, d, e);
        }
    }
    if constexpr (NC == 4) st_v4(dst, make_uint4(c[0], c[1], c[2], c[3]));
    else if constexpr (NC == 2) st_v2(dst, make_uint2(c[0], c[1]));
    else st_u32(dst, c[0]);
}

__host__ __device__ constexpr int ilog2c(int v) { return v <= 1 ? 0 : 1 + ilog2c(v / 2); }

}  // namespace fp8q
