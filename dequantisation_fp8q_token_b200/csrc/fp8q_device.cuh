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

namespace fp8q {

enum : int { kE4M3 = 0, kE5M2 = 1 };
enum : int { kF32 = 0, kF16 = 1, kBF16 = 2 };
enum : int { kGranTensor = 0, kGranRow = 1, kGranGroup = 2, kGranBlock = 3 };

template <int XT> struct ElemBytes { static constexpr int value = XT == kF32 ? 4 : 2; };

template <int FMT> __device__ __forceinline__ float fp8_max() {
    return FMT == kE4M3 ? 448.0f : 57344.0f;
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

// non-saturating semantics for one value given the hardware code c:
//   NaN -> NaN code (sign kept); e4m3fn: |v| > 464 (incl. Inf) -> NaN;
//   e5m2: |v| >= 61440 (incl. Inf) -> Inf.
template <int FMT> __device__ __forceinline__ uint32_t fix_code(float v, uint32_t c) {
    uint32_t u = __float_as_uint(v);
    uint32_t a = u & 0x7FFFFFFFu;
    uint32_t s = (u >> 24) & 0x80u;
    if (a > 0x7F800000u) return 0x7Fu | s;
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

__host__ __device__ constexpr int ilog2c(int v) { return v <= 1 ? 0 : 1 + ilog2c(v / 2); }

}  // namespace fp8q
