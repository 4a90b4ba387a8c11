// fp8q_internal.h -- host-side launchers behind the C ABI (validated arguments only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fp8q.h"

#ifndef FP8Q_PDL
#define FP8Q_PDL 1
#endif

namespace fp8q {

// per-CTA partial maxima of the per-tensor amax pass
constexpr int kMaxPartials = 2048;
constexpr size_t kPerTensorWorkspaceBytes = kMaxPartials * sizeof(uint32_t);

// number of SMs of the current device (cached per device)
int sm_count();

// CTAs of `kernel` with `threads` threads that fit on one SM at once (>= 1)
template <typename Kernel>
int resident_blocks_per_sm(Kernel kernel, int threads) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1) n = 1;
    return n;
}

// Launch `kernel` on `s`; with FP8Q_PDL the launch may overlap the previous
// kernel's tail (programmatic stream serialization: the kernel's own
// pdl_begin() waits for that kernel to finish before touching memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
#if FP8Q_PDL
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
#else
    (void)attr;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
#endif
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// `rule` is an fp8q_scale_rule: 0 one IEEE division, 1 torch's evaluation order
fp8q_status launch_per_token(const void* x, int xt, int64_t m, int64_t n, int group, int fmt,
                             uint8_t* q, float* sinv, int rule, cudaStream_t s);
fp8q_status launch_per_channel(const void* x, int xt, int64_t rows, int64_t cols, int fmt,
                               uint8_t* q, float* sinv, int rule, cudaStream_t s);
fp8q_status launch_per_tensor(const void* x, int xt, int64_t numel, int fmt, uint8_t* q,
                              float* sinv, uint32_t* partials, int rule, cudaStream_t s);
fp8q_status launch_fill(float* dst, int64_t count, float value, cudaStream_t s);
fp8q_status launch_cast_pipeline(const void* x, int xt, int64_t numel, uint8_t* q, float* sinv,
                                 int32_t* fmt_out, uint32_t* partials, int rule, cudaStream_t s);
fp8q_status launch_tensor_amax(const void* x, int xt, int64_t numel, uint32_t* partials, uint32_t* amax_bits,
                               cudaStream_t s);
fp8q_status launch_cast_with_amax(const void* x, int xt, int64_t numel, int fmt, const uint32_t* amax_bits,
                                  uint8_t* q, float* sinv, int rule, cudaStream_t s);
fp8q_status launch_cast_from_pipeline(const uint8_t* q, int64_t numel, const float* sinv, const int32_t* fmt_in,
                                      int yt, void* y, cudaStream_t s);

// one dequantisation problem: y = T(scale(r, c) * float(q)), validated shapes
struct DequantProblem {
    const uint8_t* q;
    const float* s;
    void* y;
    int64_t rows;
    int64_t cols;
};
fp8q_status launch_dequant(const DequantProblem* probs, int count, int fmt, int gran, int gb,
                           int yt, cudaStream_t s);

// fp8 x fp8 products on the tensor cores (scaled_mm.cu).  fine = false: sa and
// sb are one scale each; fine = true: sa[M][sa_ld] per 1 x 128 group of A,
// sb[ceil(N/128)][sb_ld] per 128 x 128 block of B.  Shapes validated, K % 16
// == 0 for a K-major operand, M (N) % 16 == 0 for an MN-major A (B), a and b
// 16-byte aligned.  wait_limit_ns: bound of every wait inside the kernel (0:
// the default of a few seconds); stall_kb >= 0 leaves out the copies of that
// k-block of each CTA's first tile (the test of the bounded waits).
fp8q_status launch_scaled_mm(const uint8_t* a, int fa, const uint8_t* b, int fb, int64_t M, int64_t N, int64_t K,
                             const float* sa, int sa_ld, const float* sb, int sb_ld, bool fine, const void* bias,
                             int yt, void* d, uint32_t* status, cudaStream_t s, int a_mn = 0, int b_mn = 0,
                             uint64_t wait_limit_ns = 0, int stall_kb = -1);

// _LinearFp8.backward's data movements (linear_bwd.cu): validated shapes
fp8q_status launch_transpose(const uint8_t* src, int64_t rows, int64_t cols, uint8_t* dst, int64_t ld,
                             cudaStream_t s);
fp8q_status launch_sum_rows(const void* x, int xt, int64_t rows, int64_t cols, void* out, cudaStream_t s);

inline fp8q_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA; }

}  // namespace fp8q
