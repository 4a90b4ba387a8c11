// dequant.cu -- fp8 -> fp32/fp16/bf16 with per-granule scales:
//   y[r][c] = T(fl(float(q[r][c]) * s[granule(r, c)]))
// covering DeepSeek-V3 weight_dequant (B x B blocks, bf16 out) and ColossalAI
// cast_from_fp8 / DeepEP per_token_cast_back (tensor, row and 1 x G groups).
//
// Work decomposition: each problem is cut into tiles of 8 * U rows by
// 32 chunks of V consecutive elements (V = 32, 16, 8, 4, 2 or 1, the widest
// that the row length, granule edge and pointer alignment allow).  A CTA of 8
// warps owns one tile: warp w handles rows w, w + 8, ..., lane l the l-th
// chunk, so at V = 32 every warp-wide load is one 256-bit access per lane
// (1 KiB of contiguous codes) and each lane writes its 32 bf16 outputs with
// two 256-bit stores.  Each thread issues its U row loads before converting
// any of them.  U (rows per thread: 4, 2 or 1) is the largest that still
// gives the launch at least four waves of resident CTAs: large problems
// take long tiles, and a problem of a few waves keeps the last one short.
// Problems of one launch (a checkpoint's weights, a mixture-of-experts
// layer) share the grid through a descriptor table in kernel-parameter
// space; a CTA finds its problem by binary search over the first-tile
// prefix, so heterogeneous shapes need no device-side metadata.
//
// Arithmetic: two codes -> f16x2 (exact), widened to fp32, one fp32 multiply
// each, then one round-to-nearest-even into the output type.
#include "fp8q_device.cuh"
#include "fp8q_internal.h"

namespace fp8q {
namespace {

constexpr int kDqThreads = 256;
constexpr int kDqWarps = kDqThreads / 32;
#ifndef FP8Q_DQ_V32
#define FP8Q_DQ_V32 1  // 32-code chunks with 256-bit loads / stores where aligned
#endif
constexpr int kMinWaves = 4;            // waves of resident CTAs a launch should have at least
constexpr int kMaxGroupedDescs = 96;

struct DqDesc {
    const uint8_t* q;
    const float* s;
    void* y;
    int64_t rows;
    int64_t cols;
    int64_t tile_begin;     // first tile of this problem in the launch
    int32_t tiles_per_row;  // column tiles
    int32_t vshift;         // log2 V
};

template <int N>
struct DqParams {
    int32_t count;
    int32_t gb;          // group (GROUP) or block edge (BLOCK)
    int32_t gb_shift;    // log2(gb) when gb is a power of two, else -1
    DqDesc d[N];
};

// a / gb for the non-negative indices of one problem (rows, cols < 2^31)
__device__ __forceinline__ uint32_t div_gb(uint32_t a, int gb, int gb_shift) {
    return gb_shift >= 0 ? (a >> gb_shift) : a / (uint32_t)gb;
}

// V codes (V <= 32) in up to eight 32-bit words, code i in byte i
struct Chunk {
    uint32_t w[8];
};

template <int V>
__device__ __forceinline__ Chunk load_codes(const uint8_t* p) {
    Chunk c;
#pragma unroll
    for (int i = 0; i < 8; ++i) c.w[i] = 0u;
    if (V == 32) {
        const U8x32 t = ld_stream_v8(p);
#pragma unroll
        for (int i = 0; i < 8; ++i) c.w[i] = t.w[i];
    } else if (V == 16) {
        const uint4 t = ld_stream_v4(p);
        c.w[0] = t.x; c.w[1] = t.y; c.w[2] = t.z; c.w[3] = t.w;
    } else if (V == 8) {
        const uint2 t = ld_stream_v2(p);
        c.w[0] = t.x; c.w[1] = t.y;
    } else if (V == 4) {
        c.w[0] = ld_stream_u32(p);
    } else if (V == 2) {
        c.w[0] = *reinterpret_cast<const uint16_t*>(p);
    } else {
        c.w[0] = *p;
    }
    return c;
}

// convert and store V outputs starting at element offset e of y
template <int FMT, int YT, int V>
__device__ __forceinline__ void convert_store(const Chunk& c, float sc, void* y, int64_t e) {
    const uint32_t* w = c.w;
    if (YT == kF32) {
        float* yf = static_cast<float*>(y) + e;
        if (V == 32) {
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float2 a = dec2<FMT>(w[2 * h + i] & 0xFFFFu);
                    const float2 b = dec2<FMT>(w[2 * h + i] >> 16);
                    o[4 * i + 0] = __float_as_uint(__fmul_rn(a.x, sc));
                    o[4 * i + 1] = __float_as_uint(__fmul_rn(a.y, sc));
                    o[4 * i + 2] = __float_as_uint(__fmul_rn(b.x, sc));
                    o[4 * i + 3] = __float_as_uint(__fmul_rn(b.y, sc));
                }
                st_v8(yf + 8 * h, o);
            }
        } else if (V >= 4) {
#pragma unroll
            for (int i = 0; i < V / 4; ++i) {
                const float2 a = dec2<FMT>(w[i] & 0xFFFFu);
                const float2 b = dec2<FMT>(w[i] >> 16);
                st_v4(yf + 4 * i, make_uint4(__float_as_uint(__fmul_rn(a.x, sc)), __float_as_uint(__fmul_rn(a.y, sc)),
                                             __float_as_uint(__fmul_rn(b.x, sc)), __float_as_uint(__fmul_rn(b.y, sc))));
            }
        } else {
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const float2 a = dec2<FMT>((w[0] >> (8 * i)) & 0xFFu);
                yf[i] = __fmul_rn(a.x, sc);
            }
        }
    } else {
        uint16_t* yh = static_cast<uint16_t*>(y) + e;
        if (V == 32) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 a = dec2<FMT>(w[4 * h + i] & 0xFFFFu);
                    const float2 b = dec2<FMT>(w[4 * h + i] >> 16);
                    o[2 * i] = pack2<YT>(__fmul_rn(a.x, sc), __fmul_rn(a.y, sc));
                    o[2 * i + 1] = pack2<YT>(__fmul_rn(b.x, sc), __fmul_rn(b.y, sc));
                }
                st_v8(yh + 16 * h, o);
            }
        } else if (V >= 8) {
#pragma unroll
            for (int i = 0; i < V / 8; ++i) {
                uint32_t o[4];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float2 a = dec2<FMT>(w[2 * i + h] & 0xFFFFu);
                    const float2 b = dec2<FMT>(w[2 * i + h] >> 16);
                    o[2 * h] = pack2<YT>(__fmul_rn(a.x, sc), __fmul_rn(a.y, sc));
                    o[2 * h + 1] = pack2<YT>(__fmul_rn(b.x, sc), __fmul_rn(b.y, sc));
                }
                st_v4(yh + 8 * i, make_uint4(o[0], o[1], o[2], o[3]));
            }
        } else if (V == 4) {
            const float2 a = dec2<FMT>(w[0] & 0xFFFFu);
            const float2 b = dec2<FMT>(w[0] >> 16);
            st_v2(yh, make_uint2(pack2<YT>(__fmul_rn(a.x, sc), __fmul_rn(a.y, sc)),
                                 pack2<YT>(__fmul_rn(b.x, sc), __fmul_rn(b.y, sc))));
        } else if (V == 2) {
            const float2 a = dec2<FMT>(w[0] & 0xFFFFu);
            st_u32(yh, pack2<YT>(__fmul_rn(a.x, sc), __fmul_rn(a.y, sc)));
        } else {
            const float2 a = dec2<FMT>(w[0] & 0xFFu);
            yh[0] = (uint16_t)(pack2<YT>(__fmul_rn(a.x, sc), 0.0f) & 0xFFFFu);
        }
    }
}

template <int FMT, int YT, int GRAN, int V, int U>
__device__ __forceinline__ void dequant_tile(const DqDesc& D, int gb, int gb_shift, int64_t tr, int tc) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t cols = D.cols;
    const int64_t rows = D.rows;
    const int64_t c = ((int64_t)tc * 32 + lane) * V;  // first column of this thread's chunk
    const int64_t r0 = tr * (kDqWarps * U) + warp;
    const uint8_t* q = D.q;
    const float* s = D.s;
    if (c < cols) {
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int64_t r = r0 + (int64_t)k * kDqWarps;
            if (r < rows) prefetch_l2(q + r * cols + c);
        }
    }
    pdl_wait();
    if (c >= cols) return;
    Chunk codes[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
        const int64_t r = r0 + (int64_t)k * kDqWarps;
        if (r < rows) codes[k] = load_codes<V>(q + r * cols + c);
    }
    // scale index pieces that do not depend on the row
    int64_t s_cols = 0, s_col = 0;
    if (GRAN == kGranGroup) {
        s_cols = cols / gb;
        s_col = div_gb((uint32_t)c, gb, gb_shift);
    } else if (GRAN == kGranBlock) {
        s_cols = (cols + gb - 1) / gb;
        s_col = div_gb((uint32_t)c, gb, gb_shift);
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
        const int64_t r = r0 + (int64_t)k * kDqWarps;
        if (r < rows) {
            float sc;
            if (GRAN == kGranTensor) sc = __ldg(s);
            else if (GRAN == kGranRow) sc = __ldg(s + r);
            else if (GRAN == kGranGroup) sc = __ldg(s + r * s_cols + s_col);
            else sc = __ldg(s + (int64_t)div_gb((uint32_t)r, gb, gb_shift) * s_cols + s_col);
            convert_store<FMT, YT, V>(codes[k], sc, D.y, r * cols + c);
        }
    }
}

template <int FMT, int YT, int GRAN, int N, int U>
__global__ void __launch_bounds__(kDqThreads) dequant_kernel(const __grid_constant__ DqParams<N> p) {
    pdl_trigger();     // the tile's codes are prefetched into L2 before pdl_wait (in dequant_tile)
    const int64_t tile = blockIdx.x;
    int lo = 0;
    if (N > 1) {
        int hi = p.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.d[mid].tile_begin <= tile) lo = mid;
            else hi = mid - 1;
        }
    }
    const DqDesc& D = p.d[lo];
    const int64_t t = tile - D.tile_begin;
    const int64_t tr = t / D.tiles_per_row;
    const int tc = (int)(t - tr * D.tiles_per_row);
    switch (D.vshift) {
#if FP8Q_DQ_V32
    case 5: dequant_tile<FMT, YT, GRAN, 32, U>(D, p.gb, p.gb_shift, tr, tc); break;
#endif
    case 4: dequant_tile<FMT, YT, GRAN, 16, U>(D, p.gb, p.gb_shift, tr, tc); break;
    case 3: dequant_tile<FMT, YT, GRAN, 8, U>(D, p.gb, p.gb_shift, tr, tc); break;
    case 2: dequant_tile<FMT, YT, GRAN, 4, U>(D, p.gb, p.gb_shift, tr, tc); break;
    case 1: dequant_tile<FMT, YT, GRAN, 2, U>(D, p.gb, p.gb_shift, tr, tc); break;
    default: dequant_tile<FMT, YT, GRAN, 1, U>(D, p.gb, p.gb_shift, tr, tc); break;
    }
}

// widest chunk V such that rows start V-aligned, the chunk never crosses a
// granule, and loads / stores of the chunk are naturally aligned
int choose_vshift(const DequantProblem& P, int gran, int gb, int ybytes) {
    for (int vs = FP8Q_DQ_V32 ? 5 : 4; vs > 0; --vs) {
        const int V = 1 << vs;
        if (P.cols % V) continue;
        if ((gran == kGranGroup || gran == kGranBlock) && gb % V) continue;
        if ((uintptr_t)P.q % V) continue;
        const int widest = V == 32 ? 32 : 16;  // 256-bit stores only at V = 32
        const int ystore = V * ybytes < widest ? V * ybytes : widest;
        if ((uintptr_t)P.y % ystore) continue;
        return vs;
    }
    return 0;
}

// resident CTAs of one instantiation across the GPU (cached)
template <int FMT, int YT, int GRAN, int N, int U>
int64_t resident_ctas() {
    static const int64_t n = [] {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dequant_kernel<FMT, YT, GRAN, N, U>, kDqThreads,
                                                          0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        return (int64_t)per_sm * sm_count();
    }();
    return n;
}

template <int FMT, int YT, int GRAN, int N, int U>
// each problem's first tile with U rows per thread (8 * U rows per tile)
cudaError_t assign_tiles(DqParams<N>& p, int64_t& tiles) {
    tiles = 0;
    for (int i = 0; i < p.count; ++i) {
        DqDesc& D = p.d[i];
        D.tile_begin = tiles;
        tiles += ((D.rows + kDqWarps * U - 1) / (kDqWarps * U)) * D.tiles_per_row;
    }
    if (tiles > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    return cudaSuccess;
}

template <int FMT, int YT, int GRAN, int N>
fp8q_status run_batch(const DequantProblem* probs, int count, int gb, cudaStream_t s) {
    DqParams<N> p;
    p.count = 0;
    p.gb = gb;
    p.gb_shift = -1;
    if (gb > 0 && (gb & (gb - 1)) == 0) {
        p.gb_shift = 0;
        while ((1 << p.gb_shift) < gb) ++p.gb_shift;
    }
    const int ybytes = YT == kF32 ? 4 : 2;
    for (int i = 0; i < count; ++i) {
        const DequantProblem& P = probs[i];
        if (P.rows == 0 || P.cols == 0) continue;
        if (P.rows > 0x7FFFFFFFLL || P.cols > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
        DqDesc& D = p.d[p.count++];
        D.q = P.q;
        D.s = P.s;
        D.y = P.y;
        D.rows = P.rows;
        D.cols = P.cols;
        D.vshift = choose_vshift(P, GRAN, gb, ybytes);
        const int64_t span = (int64_t)32 << D.vshift;
        D.tiles_per_row = (int32_t)((P.cols + span - 1) / span);
    }
    if (p.count == 0) return FP8Q_OK;
    // rows per thread: the largest of 4, 2, 1 that leaves at least kMinWaves
    // waves of resident CTAs
    int64_t tiles = 0;
    cudaError_t err;
    if (assign_tiles<FMT, YT, GRAN, N, 4>(p, tiles) == cudaSuccess &&
        tiles >= kMinWaves * resident_ctas<FMT, YT, GRAN, N, 4>()) {
        err = launch_kernel(dequant_kernel<FMT, YT, GRAN, N, 4>, dim3((unsigned)tiles), dim3(kDqThreads), s, p);
    } else if (assign_tiles<FMT, YT, GRAN, N, 2>(p, tiles) == cudaSuccess &&
               tiles >= kMinWaves * resident_ctas<FMT, YT, GRAN, N, 2>()) {
        err = launch_kernel(dequant_kernel<FMT, YT, GRAN, N, 2>, dim3((unsigned)tiles), dim3(kDqThreads), s, p);
    } else {
        if (assign_tiles<FMT, YT, GRAN, N, 1>(p, tiles) != cudaSuccess) return FP8Q_ERR_BAD_SHAPE;
        err = launch_kernel(dequant_kernel<FMT, YT, GRAN, N, 1>, dim3((unsigned)tiles), dim3(kDqThreads), s, p);
    }
    return cuda_status(err);
}

template <int FMT, int YT, int GRAN>
fp8q_status run_all(const DequantProblem* probs, int count, int gb, cudaStream_t s) {
    if constexpr (GRAN != kGranBlock) {
        // only block dequant takes several problems per call
        fp8q_status st = FP8Q_OK;
        for (int i = 0; i < count && st == FP8Q_OK; ++i) st = run_batch<FMT, YT, GRAN, 1>(probs + i, 1, gb, s);
        return st;
    } else {
        if (count == 1) return run_batch<FMT, YT, GRAN, 1>(probs, 1, gb, s);
        for (int i = 0; i < count; i += kMaxGroupedDescs) {
            const int n = count - i < kMaxGroupedDescs ? count - i : kMaxGroupedDescs;
            fp8q_status st = run_batch<FMT, YT, GRAN, kMaxGroupedDescs>(probs + i, n, gb, s);
            if (st != FP8Q_OK) return st;
        }
        return FP8Q_OK;
    }
}

template <int FMT, int YT>
fp8q_status by_gran(const DequantProblem* probs, int count, int gran, int gb, cudaStream_t s) {
    switch (gran) {
    case kGranTensor: return run_all<FMT, YT, kGranTensor>(probs, count, gb, s);
    case kGranRow: return run_all<FMT, YT, kGranRow>(probs, count, gb, s);
    case kGranGroup: return run_all<FMT, YT, kGranGroup>(probs, count, gb, s);
    default: return run_all<FMT, YT, kGranBlock>(probs, count, gb, s);
    }
}

template <int FMT>
fp8q_status by_yt(const DequantProblem* probs, int count, int gran, int gb, int yt, cudaStream_t s) {
    switch (yt) {
    case kF32: return by_gran<FMT, kF32>(probs, count, gran, gb, s);
    case kF16: return by_gran<FMT, kF16>(probs, count, gran, gb, s);
    default: return by_gran<FMT, kBF16>(probs, count, gran, gb, s);
    }
}

}  // namespace

fp8q_status launch_dequant(const DequantProblem* probs, int count, int fmt, int gran, int gb,
                           int yt, cudaStream_t s) {
    if (count <= 0) return FP8Q_OK;
    return fmt == kE4M3 ? by_yt<kE4M3>(probs, count, gran, gb, yt, s)
                        : by_yt<kE5M2>(probs, count, gran, gb, yt, s);
}

}  // namespace fp8q
