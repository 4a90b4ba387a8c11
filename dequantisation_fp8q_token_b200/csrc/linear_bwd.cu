// linear_bwd.cu -- the two data movements of ColossalAI _LinearFp8.backward
// that are not fp8 products:
//   transpose_kernel   the .t().contiguous() copies of the fp8 operands
//                      (dst[c][r] = src[r][c], bytes), with the destination
//                      rows padded with zeros up to a pitch of the caller's
//                      choosing, so that a token count that is not a multiple
//                      of 16 still gives a legal row pitch to the products
//   sum_rows_kernel    bias_grad = out_grad.sum(0): out[c] = T(sum_r x[r][c]),
//                      summed in fp32 in a fixed order (each thread owns two
//                      columns and walks its share of the rows in ascending
//                      order; the 16 warps' partial sums are then added in
//                      warp order), so the result does not depend on timing.
// Both are streaming passes bound by HBM bandwidth.
#include "fp8q_device.cuh"
#include "fp8q_internal.h"

namespace fp8q {
namespace {

// ---------------------------------------------------------------------------
// transpose: 64 x 64 byte tiles through shared memory
// ---------------------------------------------------------------------------
constexpr int kT = 64;                 // tile edge (bytes)
constexpr int kTThreads = 256;

// One CTA per 64 x 64 tile of the destination [cols][ld] (the padding
// columns r in [rows, ld) are written as zeros).  Interior tiles move 4-byte
// words when both pitches and base pointers allow it; edge tiles move bytes.
__global__ void __launch_bounds__(kTThreads)
transpose_kernel(const uint8_t* __restrict__ src, int64_t rows, int64_t cols, uint8_t* __restrict__ dst,
                 int64_t ld, int64_t tiles_r, int words_ok) {
    __shared__ uint8_t tile[kT][kT + 4];
    pdl_begin();
    const int64_t t = blockIdx.x;
    const int64_t tr = t % tiles_r;            // tile index along src rows (= dst columns)
    const int64_t tc = t / tiles_r;            // tile index along src columns (= dst rows)
    const int64_t r0 = tr * kT, c0 = tc * kT;
    const bool full = words_ok && r0 + kT <= rows && c0 + kT <= cols;
    if (full) {
        // load 64 rows x 16 words
        for (int i = threadIdx.x; i < kT * (kT / 4); i += kTThreads) {
            const int r = i / (kT / 4), w = i % (kT / 4);
            const uint32_t v = ld_stream_u32(src + (r0 + r) * cols + c0 + 4 * w);
            tile[r][4 * w + 0] = static_cast<uint8_t>(v);
            tile[r][4 * w + 1] = static_cast<uint8_t>(v >> 8);
            tile[r][4 * w + 2] = static_cast<uint8_t>(v >> 16);
            tile[r][4 * w + 3] = static_cast<uint8_t>(v >> 24);
        }
    } else {
        for (int i = threadIdx.x; i < kT * kT; i += kTThreads) {
            const int r = i / kT, c = i % kT;
            tile[r][c] = (r0 + r < rows && c0 + c < cols) ? src[(r0 + r) * cols + c0 + c] : 0;
        }
    }
    __syncthreads();
    // dst row c0 + c holds src column c0 + c; its bytes r0 .. r0 + 63 come
    // from tile rows 0 .. 63 (zeros beyond `rows` pad the row up to ld)
    if (full && r0 + kT <= ld) {
        for (int i = threadIdx.x; i < kT * (kT / 4); i += kTThreads) {
            const int c = i / (kT / 4), w = i % (kT / 4);
            const uint32_t v = static_cast<uint32_t>(tile[4 * w + 0][c]) | (static_cast<uint32_t>(tile[4 * w + 1][c]) << 8)
                             | (static_cast<uint32_t>(tile[4 * w + 2][c]) << 16)
                             | (static_cast<uint32_t>(tile[4 * w + 3][c]) << 24);
            st_u32(dst + (c0 + c) * ld + r0 + 4 * w, v);
        }
    } else {
        for (int i = threadIdx.x; i < kT * kT; i += kTThreads) {
            const int c = i / kT, r = i % kT;
            if (c0 + c < cols && r0 + r < ld) dst[(c0 + c) * ld + r0 + r] = tile[r][c];
        }
    }
}

// ---------------------------------------------------------------------------
// column sums: one CTA per 64 columns, 16 warps splitting the rows
// ---------------------------------------------------------------------------
constexpr int kSWarps = 16;
constexpr int kSCols = 64;             // columns per CTA: 2 per lane

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

template <int XT>
__global__ void __launch_bounds__(32 * kSWarps)
sum_rows_kernel(const void* __restrict__ x, int64_t rows, int64_t cols, void* __restrict__ out) {
    __shared__ float part[kSWarps][kSCols];
    pdl_begin();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * kSCols + 2 * lane;
    float s0 = 0.0f, s1 = 0.0f;
    for (int64_t r = warp; r < rows; r += kSWarps) {
        const int64_t i = r * cols + c;
        if (c < cols) s0 = __fadd_rn(s0, load_elem<XT>(x, i));
        if (c + 1 < cols) s1 = __fadd_rn(s1, load_elem<XT>(x, i + 1));
    }
    part[warp][2 * lane] = s0;
    part[warp][2 * lane + 1] = s1;
    __syncthreads();
    if (threadIdx.x < kSCols) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kSWarps; ++w) s = __fadd_rn(s, part[w][threadIdx.x]);
        const int64_t cc = static_cast<int64_t>(blockIdx.x) * kSCols + threadIdx.x;
        if (cc < cols) store_elem<XT>(out, cc, s);
    }
}

}  // namespace

fp8q_status launch_transpose(const uint8_t* src, int64_t rows, int64_t cols, uint8_t* dst, int64_t ld,
                             cudaStream_t s) {
    const int64_t tiles_r = (ld + kT - 1) / kT;
    const int64_t tiles_c = (cols + kT - 1) / kT;
    const int64_t tiles = tiles_r * tiles_c;
    if (tiles > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
    const int words_ok = (cols % 4 == 0) && (ld % 4 == 0) && (reinterpret_cast<uintptr_t>(src) % 4 == 0) &&
                         (reinterpret_cast<uintptr_t>(dst) % 4 == 0);
    return cuda_status(launch_kernel(transpose_kernel, dim3(static_cast<unsigned>(tiles)), dim3(kTThreads), s, src,
                                     rows, cols, dst, ld, tiles_r, words_ok));
}

fp8q_status launch_sum_rows(const void* x, int xt, int64_t rows, int64_t cols, void* out, cudaStream_t s) {
    const int64_t ctas = (cols + kSCols - 1) / kSCols;
    if (ctas > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
    const dim3 grid(static_cast<unsigned>(ctas)), block(32 * kSWarps);
    cudaError_t e;
    if (xt == kF32) e = launch_kernel(sum_rows_kernel<kF32>, grid, block, s, x, rows, cols, out);
    else if (xt == kF16) e = launch_kernel(sum_rows_kernel<kF16>, grid, block, s, x, rows, cols, out);
    else e = launch_kernel(sum_rows_kernel<kBF16>, grid, block, s, x, rows, cols, out);
    return cuda_status(e);
}

}  // namespace fp8q
