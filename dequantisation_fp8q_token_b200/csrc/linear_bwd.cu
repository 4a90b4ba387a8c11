// linear_bwd.cu -- the two data movements of ColossalAI _LinearFp8.backward
// that are not fp8 products:
//   transpose_kernel   the .t().contiguous() copies of the fp8 operands
//                      (dst[c][r] = src[r][c], bytes), with the destination
//                      rows padded with zeros up to a pitch of the caller's
//                      choosing, so that a token count that is not a multiple
//                      of 16 still gives a legal row pitch to the products
//   sum_rows_kernel    bias_grad = out_grad.sum(0): out[c] = T(sum_r x[r][c]),
//                      summed in fp32 in a fixed order (a column's rows are
//                      split into 64 interleaved subsets, r % 64, each summed
//                      in ascending row order; the 64 partial sums are then
//                      added in subset order), so the result does not depend
//                      on timing.
// Both are streaming passes bound by HBM bandwidth.
#include "fp8q_device.cuh"
#include "fp8q_internal.h"

namespace fp8q {
namespace {

// ---------------------------------------------------------------------------
// transpose: 128 x 128 byte tiles through shared memory
// ---------------------------------------------------------------------------
constexpr int kT = 128;                // tile edge (bytes): full 128-byte lines on both sides
constexpr int kTW = kT / 4;            // words per tile row
constexpr int kTThreads = 256;

// 4 x 4 byte transpose of four words (a[i] = row i, bytes = columns 0..3):
// returns o[j] = column j, bytes = rows 0..3
__device__ __forceinline__ void transpose4x4(const uint32_t (&a)[4], uint32_t (&o)[4]) {
    const uint32_t t0 = __byte_perm(a[0], a[1], 0x5140), t1 = __byte_perm(a[0], a[1], 0x7362);
    const uint32_t t2 = __byte_perm(a[2], a[3], 0x5140), t3 = __byte_perm(a[2], a[3], 0x7362);
    o[0] = __byte_perm(t0, t2, 0x5410);
    o[1] = __byte_perm(t0, t2, 0x7632);
    o[2] = __byte_perm(t1, t3, 0x5410);
    o[3] = __byte_perm(t1, t3, 0x7632);
}

// The transposed tile in shared memory: 128 destination rows of 32 words.
// Word w of row d sits at word w ^ (4 * ((d / 16) % 8)): the XOR moves whole
// groups of four words, so a row still leaves as 16-byte chunks, and the
// word stores of the transpose step (a warp = 4 source row quads x the 8
// chunks of a row) touch 32 different banks.
__device__ __forceinline__ int tb_word(int d, int w) { return w ^ (4 * ((d >> 4) & 7)); }

// One CTA per 128 x 128 tile of the destination [cols][ld] (the padding
// columns r in [rows, ld) are written as zeros).  Interior tiles with 16-byte
// aligned pitches and bases: each thread loads a 4-row x 16-byte block of the
// source straight into registers, transposes its four 4 x 4 byte blocks there,
// and stores the sixteen 4-byte words into the transposed tile; after one
// barrier the destination rows leave as 16-byte stores.  Other tiles move
// bytes.
__global__ void __launch_bounds__(kTThreads)
transpose_kernel(const uint8_t* __restrict__ src, int64_t rows, int64_t cols, uint8_t* __restrict__ dst,
                 int64_t ld, int64_t tiles_r, int vec_ok) {
    __shared__ __align__(16) uint32_t tb[kT][kTW];         // transposed tile, swizzled words
    pdl_begin();
    const int64_t t = blockIdx.x;
    const int64_t tr = t % tiles_r;            // tile index along src rows (= dst columns)
    const int64_t tc = t / tiles_r;            // tile index along src columns (= dst rows)
    const int64_t r0 = tr * kT, c0 = tc * kT;
    const int tid = threadIdx.x;
    if (vec_ok && r0 + kT <= rows && c0 + kT <= cols) {
        // thread -> (row quad q: source rows 4q..4q+3, chunk j: source bytes 16j..16j+15);
        // a warp holds 4 row quads x the 8 chunks of a row, so each load
        // instruction reads four whole 128-byte lines
        const int lane = tid & 31, wid = tid >> 5;
        const int q = 4 * wid + (lane >> 3);
        const int j = lane & 7;
        uint4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = ld_stream_v4(src + (r0 + 4 * q + k) * cols + c0 + 16 * j);
#pragma unroll
        for (int w = 0; w < 4; ++w) {                            // source bytes 16j + 4w .. 16j + 4w + 3
            const uint32_t a[4] = {(&v[0].x)[w], (&v[1].x)[w], (&v[2].x)[w], (&v[3].x)[w]};
            uint32_t o[4];
            transpose4x4(a, o);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int d = 16 * j + 4 * w + k;                // destination row in the tile
                tb[d][tb_word(d, q)] = o[k];                     // bytes = source rows 4q .. 4q + 3
            }
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kT * (kT / 16) / kTThreads; ++k) {       // 128 dst rows x 8 chunks of 16 bytes
            const int i = tid + k * kTThreads;
            const int d = i >> 3, seg = i & 7;
            const uint4 w = *reinterpret_cast<const uint4*>(&tb[d][tb_word(d, 4 * seg)]);
            st_v4(dst + (c0 + d) * ld + r0 + 16 * seg, w);
        }
        return;
    }
    uint8_t* tile = reinterpret_cast<uint8_t*>(tb);          // bytes [kT][kT]
    for (int i = tid; i < kT * kT; i += kTThreads) {
        const int r = i / kT, c = i % kT;
        tile[r * kT + c] = (r0 + r < rows && c0 + c < cols) ? src[(r0 + r) * cols + c0 + c] : 0;
    }
    __syncthreads();
    for (int i = tid; i < kT * kT; i += kTThreads) {
        const int c = i / kT, r = i % kT;
        if (c0 + c < cols && r0 + r < ld) dst[(c0 + c) * ld + r0 + r] = tile[r * kT + c];
    }
}

// ---------------------------------------------------------------------------
// column sums
// ---------------------------------------------------------------------------
// Rows are split into kSubsets interleaved subsets (row r belongs to subset
// r % kSubsets); each subset is summed in ascending row order and the
// partial sums are added in subset order.  Both kernels below keep exactly
// this order.
constexpr int kSubsets = 64;
constexpr int kSThreads = 512;

template <int XT> __device__ __forceinline__ float load_elem(const void* x, int64_t i) {
    if constexpr (XT == kF32) return __ldg(static_cast<const float*>(x) + i);
    else if constexpr (XT == kF16) return __half2float(__ldg(static_cast<const __half*>(x) + i));
    else return __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(x) + i));
}
template <int XT> __device__ __forceinline__ void store_elem(void* y, int64_t i, float v) {
    if constexpr (XT == kF32) static_cast<float*>(y)[i] = v;
    else if constexpr (XT == kF16) static_cast<__half*>(y)[i] = __float2half_rn(v);
    else static_cast<__nv_bfloat16*>(y)[i] = __float2bfloat16_rn(v);
}
// the VEC elements of a 16-byte word, widened exactly to fp32
template <int XT> __device__ __forceinline__ void widen16(const uint4& w, float (&v)[16 / (XT == kF32 ? 4 : 2)]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
    if constexpr (XT == kF32) {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(u[i]);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) widen2<XT>(u[i], v[2 * i], v[2 * i + 1]);
    }
}

// Vector path (16-byte aligned rows): a CTA owns 8 x VEC columns (64 for
// 16-bit types, 32 for fp32); 8 threads cover one row of them with 16-byte
// loads, so the 512 threads form 64 row lanes, one per subset.  Each lane
// keeps kUnroll rows in flight (128 bytes per thread).
constexpr int kUnroll = 8;
template <int XT>
__global__ void __launch_bounds__(kSThreads)
sum_rows_vec_kernel(const uint8_t* __restrict__ x, int64_t rows, int64_t cols, void* __restrict__ out) {
    constexpr int kEs = XT == kF32 ? 4 : 2;
    constexpr int VEC = 16 / kEs;
    constexpr int W = 8 * VEC;                          // columns per CTA
    static_assert(kSThreads / 8 == kSubsets, "one row lane per subset");
    __shared__ float part[kSubsets][W + 1];
    pdl_begin();
    const int seg = threadIdx.x & 7, lane_r = threadIdx.x >> 3;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * W + seg * VEC;
    const bool col_ok = c0 < cols;                      // cols % VEC == 0: a segment is all in or all out
    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] = 0.0f;
    const int64_t pitch = cols * kEs;
    for (int64_t r = lane_r; r < rows; r += kSubsets * kUnroll) {
        uint4 w[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            w[u] = (col_ok && r + u * kSubsets < rows) ? ld_stream_v4(x + (r + u * kSubsets) * pitch + c0 * kEs)
                                                        : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (r + u * kSubsets < rows) {
                float v[VEC];
                widen16<XT>(w[u], v);
#pragma unroll
                for (int i = 0; i < VEC; ++i) acc[i] = __fadd_rn(acc[i], v[i]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < VEC; ++i) part[lane_r][seg * VEC + i] = acc[i];
    __syncthreads();
    if (threadIdx.x < W) {
        float t = 0.0f;
#pragma unroll 8
        for (int l = 0; l < kSubsets; ++l) t = __fadd_rn(t, part[l][threadIdx.x]);
        const int64_t cc = static_cast<int64_t>(blockIdx.x) * W + threadIdx.x;
        if (cc < cols) store_elem<XT>(out, cc, t);
    }
}

// Any alignment: one CTA per 8 columns, 64 row lanes x 8 columns, element loads.
template <int XT>
__global__ void __launch_bounds__(kSThreads)
sum_rows_kernel(const void* __restrict__ x, int64_t rows, int64_t cols, void* __restrict__ out) {
    __shared__ float part[kSubsets][9];
    pdl_begin();
    const int cl = threadIdx.x & 7, lane_r = threadIdx.x >> 3;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * 8 + cl;
    float acc = 0.0f;
    if (c < cols)
        for (int64_t r = lane_r; r < rows; r += kSubsets) acc = __fadd_rn(acc, load_elem<XT>(x, r * cols + c));
    part[lane_r][cl] = acc;
    __syncthreads();
    if (threadIdx.x < 8) {
        float t = 0.0f;
        for (int l = 0; l < kSubsets; ++l) t = __fadd_rn(t, part[l][threadIdx.x]);
        if (c < cols) store_elem<XT>(out, c, t);
    }
}

}  // namespace

fp8q_status launch_transpose(const uint8_t* src, int64_t rows, int64_t cols, uint8_t* dst, int64_t ld,
                             cudaStream_t s) {
    const int64_t tiles_r = (ld + kT - 1) / kT;
    const int64_t tiles_c = (cols + kT - 1) / kT;
    const int64_t tiles = tiles_r * tiles_c;
    if (tiles > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
    const int vec_ok = (cols % 16 == 0) && (ld % 16 == 0) && (reinterpret_cast<uintptr_t>(src) % 16 == 0) &&
                       (reinterpret_cast<uintptr_t>(dst) % 16 == 0);
    return cuda_status(launch_kernel(transpose_kernel, dim3(static_cast<unsigned>(tiles)), dim3(kTThreads), s, src,
                                     rows, cols, dst, ld, tiles_r, vec_ok));
}

fp8q_status launch_sum_rows(const void* x, int xt, int64_t rows, int64_t cols, void* out, cudaStream_t s) {
    const int es = xt == kF32 ? 4 : 2;
    const int vec = 16 / es;
    const bool vec_ok = cols % vec == 0 && reinterpret_cast<uintptr_t>(x) % 16 == 0;
    const int64_t width = vec_ok ? 8 * vec : 8;
    const int64_t ctas = (cols + width - 1) / width;
    if (ctas > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
    const dim3 grid(static_cast<unsigned>(ctas)), block(kSThreads);
    const uint8_t* xb = static_cast<const uint8_t*>(x);
    cudaError_t e;
    if (vec_ok) {
        if (xt == kF32) e = launch_kernel(sum_rows_vec_kernel<kF32>, grid, block, s, xb, rows, cols, out);
        else if (xt == kF16) e = launch_kernel(sum_rows_vec_kernel<kF16>, grid, block, s, xb, rows, cols, out);
        else e = launch_kernel(sum_rows_vec_kernel<kBF16>, grid, block, s, xb, rows, cols, out);
    } else {
        if (xt == kF32) e = launch_kernel(sum_rows_kernel<kF32>, grid, block, s, x, rows, cols, out);
        else if (xt == kF16) e = launch_kernel(sum_rows_kernel<kF16>, grid, block, s, x, rows, cols, out);
        else e = launch_kernel(sum_rows_kernel<kBF16>, grid, block, s, x, rows, cols, out);
    }
    return cuda_status(e);
}

}  // namespace fp8q
