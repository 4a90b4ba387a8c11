// fp8q_api.cu -- the extern "C" entry points of libfp8q: argument checks on
// the host (enums, then shapes, then null pointers, then alignment), then the
// launchers.  Nothing is enqueued when a check fails.
#include <atomic>

#include "fp8q.h"
#include "fp8q_device.cuh"
#include "fp8q_internal.h"

namespace fp8q {

int sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64) {
        const int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

namespace {

bool fmt_ok(int f) { return f == FP8Q_E4M3FN || f == FP8Q_E5M2; }
bool rule_ok(int r) { return r == FP8Q_SCALE_IEEE || r == FP8Q_SCALE_TORCH; }
bool dtype_ok(int t) { return t == FP8Q_F32 || t == FP8Q_F16 || t == FP8Q_BF16; }
int dtype_bytes(int t) { return t == FP8Q_F32 ? 4 : 2; }
bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// product of two non-negative sizes, or -1 when it would not fit in int64
int64_t checked_mul(int64_t a, int64_t b) {
    if (a == 0 || b == 0) return 0;
    if (a > INT64_MAX / b) return -1;
    return a * b;
}

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" {

const char* fp8q_status_string(fp8q_status status) {
    switch (status) {
    case FP8Q_OK: return "FP8Q_OK";
    case FP8Q_ERR_NULL_POINTER: return "FP8Q_ERR_NULL_POINTER: a non-empty tensor pointer is NULL";
    case FP8Q_ERR_BAD_DTYPE: return "FP8Q_ERR_BAD_DTYPE: only float32, float16 and bfloat16 are allowed";
    case FP8Q_ERR_BAD_FORMAT: return "FP8Q_ERR_BAD_FORMAT: only float8_e4m3fn and float8_e5m2 are allowed";
    case FP8Q_ERR_BAD_SHAPE: return "FP8Q_ERR_BAD_SHAPE: size, group or block edge not allowed";
    case FP8Q_ERR_MISALIGNED: return "FP8Q_ERR_MISALIGNED: pointer not aligned to its element size";
    case FP8Q_ERR_WORKSPACE: return "FP8Q_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case FP8Q_ERR_CUDA: return "FP8Q_ERR_CUDA: the CUDA runtime refused a launch";
    case FP8Q_ERR_BAD_GRANULARITY: return "FP8Q_ERR_BAD_GRANULARITY: unknown scale granularity";
    case FP8Q_ERR_TOO_MANY: return "FP8Q_ERR_TOO_MANY: descriptor count out of range";
    case FP8Q_ERR_BAD_RULE: return "FP8Q_ERR_BAD_RULE: unknown scale rule";
    }
    return "FP8Q_ERR_UNKNOWN";
}

int fp8q_version(void) { return 10100; }

fp8q_status fp8q_per_token_group_quant(const void* x, fp8q_dtype xt, int64_t m, int64_t n, int group,
                                       fp8q_format fmt, uint8_t* q, float* scale_inv,
                                       fp8q_stream_t stream) {
    return fp8q_per_token_group_quant_ex(x, xt, m, n, group, fmt, q, scale_inv, FP8Q_SCALE_IEEE, stream);
}

fp8q_status fp8q_per_token_group_quant_ex(const void* x, fp8q_dtype xt, int64_t m, int64_t n, int group,
                                          fp8q_format fmt, uint8_t* q, float* scale_inv,
                                          fp8q_scale_rule rule, fp8q_stream_t stream) {
    if (!dtype_ok(xt)) return FP8Q_ERR_BAD_DTYPE;
    if (!rule_ok(rule)) return FP8Q_ERR_BAD_RULE;
    if (!fmt_ok(fmt)) return FP8Q_ERR_BAD_FORMAT;
    if (m < 0 || n < 0 || group < 1 || n % group != 0) return FP8Q_ERR_BAD_SHAPE;
    const int64_t numel = checked_mul(m, n);
    if (numel < 0 || checked_mul(numel, dtype_bytes(xt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    if (numel == 0) return FP8Q_OK;
    if (!x || !q || !scale_inv) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(x, dtype_bytes(xt)) || !aligned(scale_inv, 4)) return FP8Q_ERR_MISALIGNED;
    return launch_per_token(x, xt, m, n, group, fmt, q, scale_inv, rule, reinterpret_cast<cudaStream_t>(stream));
}

fp8q_status fp8q_cast_per_channel(const void* x, fp8q_dtype xt, int64_t rows, int64_t cols,
                                  fp8q_format fmt, uint8_t* q, float* scale_inv, fp8q_stream_t stream) {
    return fp8q_cast_per_channel_ex(x, xt, rows, cols, fmt, q, scale_inv, FP8Q_SCALE_IEEE, stream);
}

fp8q_status fp8q_cast_per_channel_ex(const void* x, fp8q_dtype xt, int64_t rows, int64_t cols,
                                     fp8q_format fmt, uint8_t* q, float* scale_inv, fp8q_scale_rule rule,
                                     fp8q_stream_t stream) {
    if (!dtype_ok(xt)) return FP8Q_ERR_BAD_DTYPE;
    if (!rule_ok(rule)) return FP8Q_ERR_BAD_RULE;
    if (!fmt_ok(fmt)) return FP8Q_ERR_BAD_FORMAT;
    if (rows < 0 || cols < 0 || rows > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
    const int64_t numel = checked_mul(rows, cols);
    if (numel < 0 || checked_mul(numel, dtype_bytes(xt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!scale_inv) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(scale_inv, 4)) return FP8Q_ERR_MISALIGNED;
    if (numel == 0) return launch_fill(scale_inv, rows > 0 ? rows : 1, 1.0f, s);
    if (!x || !q) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(x, dtype_bytes(xt))) return FP8Q_ERR_MISALIGNED;
    return launch_per_channel(x, xt, rows, cols, fmt, q, scale_inv, rule, s);
}

size_t fp8q_cast_per_tensor_workspace_bytes(void) { return kPerTensorWorkspaceBytes; }

fp8q_status fp8q_cast_per_tensor(const void* x, fp8q_dtype xt, int64_t numel, fp8q_format fmt,
                                 uint8_t* q, float* scale_inv, void* workspace, size_t workspace_bytes,
                                 fp8q_stream_t stream) {
    return fp8q_cast_per_tensor_ex(x, xt, numel, fmt, q, scale_inv, workspace, workspace_bytes, FP8Q_SCALE_IEEE,
                                   stream);
}

fp8q_status fp8q_cast_per_tensor_ex(const void* x, fp8q_dtype xt, int64_t numel, fp8q_format fmt,
                                    uint8_t* q, float* scale_inv, void* workspace, size_t workspace_bytes,
                                    fp8q_scale_rule rule, fp8q_stream_t stream) {
    if (!dtype_ok(xt)) return FP8Q_ERR_BAD_DTYPE;
    if (!rule_ok(rule)) return FP8Q_ERR_BAD_RULE;
    if (!fmt_ok(fmt)) return FP8Q_ERR_BAD_FORMAT;
    if (numel < 0 || checked_mul(numel, dtype_bytes(xt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!scale_inv) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(scale_inv, 4)) return FP8Q_ERR_MISALIGNED;
    if (numel == 0) return launch_fill(scale_inv, 1, 1.0f, s);
    if (!x || !q) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(x, dtype_bytes(xt))) return FP8Q_ERR_MISALIGNED;
    if (!workspace || workspace_bytes < kPerTensorWorkspaceBytes || !aligned(workspace, 16))
        return FP8Q_ERR_WORKSPACE;
    return launch_per_tensor(x, xt, numel, fmt, q, scale_inv, static_cast<uint32_t*>(workspace), rule, s);
}

fp8q_status fp8q_tensor_amax(const void* x, fp8q_dtype xt, int64_t numel, uint32_t* amax_bits, void* workspace,
                             size_t workspace_bytes, fp8q_stream_t stream) {
    if (!dtype_ok(xt)) return FP8Q_ERR_BAD_DTYPE;
    if (numel < 0 || checked_mul(numel, dtype_bytes(xt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!amax_bits) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(amax_bits, 4)) return FP8Q_ERR_MISALIGNED;
    if (numel == 0) return cuda_status(cudaMemsetAsync(amax_bits, 0, sizeof(uint32_t), s));
    if (!x) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(x, dtype_bytes(xt))) return FP8Q_ERR_MISALIGNED;
    if (!workspace || workspace_bytes < kPerTensorWorkspaceBytes || !aligned(workspace, 16))
        return FP8Q_ERR_WORKSPACE;
    return launch_tensor_amax(x, xt, numel, static_cast<uint32_t*>(workspace), amax_bits, s);
}

fp8q_status fp8q_cast_per_tensor_with_amax(const void* x, fp8q_dtype xt, int64_t numel, fp8q_format fmt,
                                           const uint32_t* amax_bits, uint8_t* q, float* scale_inv,
                                           fp8q_scale_rule rule, fp8q_stream_t stream) {
    if (!dtype_ok(xt)) return FP8Q_ERR_BAD_DTYPE;
    if (!rule_ok(rule)) return FP8Q_ERR_BAD_RULE;
    if (!fmt_ok(fmt)) return FP8Q_ERR_BAD_FORMAT;
    if (numel < 0 || checked_mul(numel, dtype_bytes(xt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!scale_inv || !amax_bits) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(scale_inv, 4) || !aligned(amax_bits, 4)) return FP8Q_ERR_MISALIGNED;
    // an empty shard still takes the shared scale from the global amax
    if (numel > 0 && (!x || !q)) return FP8Q_ERR_NULL_POINTER;
    if (numel > 0 && !aligned(x, dtype_bytes(xt))) return FP8Q_ERR_MISALIGNED;
    return launch_cast_with_amax(x, xt, numel, fmt, amax_bits, q, scale_inv, rule, s);
}

fp8q_status fp8q_cast_pipeline(const void* x, fp8q_dtype xt, int64_t numel, uint8_t* q, float* scale_inv,
                               int32_t* fmt_tag, void* workspace, size_t workspace_bytes, fp8q_scale_rule rule,
                               fp8q_stream_t stream) {
    if (!dtype_ok(xt)) return FP8Q_ERR_BAD_DTYPE;
    if (!rule_ok(rule)) return FP8Q_ERR_BAD_RULE;
    if (numel < 0 || checked_mul(numel, dtype_bytes(xt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!scale_inv || !fmt_tag) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(scale_inv, 4) || !aligned(fmt_tag, 4)) return FP8Q_ERR_MISALIGNED;
    if (numel == 0) {
        fp8q_status st = launch_fill(scale_inv, 1, 1.0f, s);
        if (st != FP8Q_OK) return st;
        return cuda_status(cudaMemsetAsync(fmt_tag, 0, sizeof(int32_t), s));
    }
    if (!x || !q) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(x, dtype_bytes(xt))) return FP8Q_ERR_MISALIGNED;
    if (!workspace || workspace_bytes < kPerTensorWorkspaceBytes || !aligned(workspace, 16))
        return FP8Q_ERR_WORKSPACE;
    return launch_cast_pipeline(x, xt, numel, q, scale_inv, fmt_tag, static_cast<uint32_t*>(workspace), rule, s);
}

fp8q_status fp8q_cast_from_pipeline(const uint8_t* q, int64_t numel, const float* scale_inv,
                                    const int32_t* fmt_tag, fp8q_dtype yt, void* y, fp8q_stream_t stream) {
    if (!dtype_ok(yt)) return FP8Q_ERR_BAD_DTYPE;
    if (numel < 0 || checked_mul(numel, dtype_bytes(yt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    if (numel == 0) return FP8Q_OK;
    if (!q || !scale_inv || !fmt_tag || !y) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(scale_inv, 4) || !aligned(fmt_tag, 4) || !aligned(y, dtype_bytes(yt))) return FP8Q_ERR_MISALIGNED;
    return launch_cast_from_pipeline(q, numel, scale_inv, fmt_tag, yt, y, reinterpret_cast<cudaStream_t>(stream));
}

static bool layout_ok(int layout) { return layout == FP8Q_RECORD_PACKED4 || layout == FP8Q_RECORD_ALIGNED16; }

size_t fp8q_record_bytes_ex(int64_t numel, fp8q_record_layout layout) {
    if (numel < 0 || !layout_ok(layout)) return 0;
    if (layout == FP8Q_RECORD_PACKED4) return (size_t)(4 + numel);
    return (size_t)(16 + ((numel + 15) / 16) * 16);
}

size_t fp8q_record_bytes(int64_t numel) { return fp8q_record_bytes_ex(numel, FP8Q_RECORD_ALIGNED16); }

fp8q_status fp8q_pack_record_ex(const void* x, fp8q_dtype xt, int64_t numel, fp8q_format fmt, uint8_t* record,
                                void* workspace, size_t workspace_bytes, fp8q_scale_rule rule,
                                fp8q_record_layout layout, fp8q_stream_t stream) {
    if (!dtype_ok(xt)) return FP8Q_ERR_BAD_DTYPE;
    if (!rule_ok(rule)) return FP8Q_ERR_BAD_RULE;
    if (!fmt_ok(fmt)) return FP8Q_ERR_BAD_FORMAT;
    if (!layout_ok(layout)) return FP8Q_ERR_BAD_SHAPE;
    if (numel < 0 || checked_mul(numel, dtype_bytes(xt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    if (!record) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(record, layout == FP8Q_RECORD_PACKED4 ? 4 : 16)) return FP8Q_ERR_MISALIGNED;
    // every check of the cast below, before the header memsets are enqueued
    if (numel > 0) {
        if (!x) return FP8Q_ERR_NULL_POINTER;
        if (!aligned(x, dtype_bytes(xt))) return FP8Q_ERR_MISALIGNED;
        if (!workspace || workspace_bytes < kPerTensorWorkspaceBytes || !aligned(workspace, 16))
            return FP8Q_ERR_WORKSPACE;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int head = layout == FP8Q_RECORD_PACKED4 ? 4 : 16;
    if (layout == FP8Q_RECORD_ALIGNED16) {
        // header padding and the payload's last partial 16-byte block start at zero
        if (cudaMemsetAsync(record, 0, 16, s) != cudaSuccess) return FP8Q_ERR_CUDA;
        if (numel % 16 && cudaMemsetAsync(record + 16 + (numel / 16) * 16, 0, 16, s) != cudaSuccess)
            return FP8Q_ERR_CUDA;
    }
    return fp8q_cast_per_tensor_ex(x, xt, numel, fmt, record + head, reinterpret_cast<float*>(record), workspace,
                                   workspace_bytes, rule, stream);
}

fp8q_status fp8q_pack_record(const void* x, fp8q_dtype xt, int64_t numel, fp8q_format fmt, uint8_t* record,
                             void* workspace, size_t workspace_bytes, fp8q_scale_rule rule, fp8q_stream_t stream) {
    return fp8q_pack_record_ex(x, xt, numel, fmt, record, workspace, workspace_bytes, rule, FP8Q_RECORD_ALIGNED16,
                               stream);
}

fp8q_status fp8q_unpack_records_ex(const uint8_t* records, int count, int64_t numel, fp8q_format fmt,
                                   fp8q_dtype yt, void* y, fp8q_record_layout layout, fp8q_stream_t stream) {
    if (!fmt_ok(fmt)) return FP8Q_ERR_BAD_FORMAT;
    if (!dtype_ok(yt)) return FP8Q_ERR_BAD_DTYPE;
    if (!layout_ok(layout)) return FP8Q_ERR_BAD_SHAPE;
    if (count < 0) return FP8Q_ERR_TOO_MANY;
    if (numel < 0 || checked_mul(checked_mul(numel, count), dtype_bytes(yt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    if (count == 0 || numel == 0) return FP8Q_OK;
    if (!records || !y) return FP8Q_ERR_NULL_POINTER;
    const bool packed = layout == FP8Q_RECORD_PACKED4;
    if (!aligned(records, packed ? 4 : 16) || !aligned(y, dtype_bytes(yt))) return FP8Q_ERR_MISALIGNED;
    if (packed && count > 1 && numel % 4) return FP8Q_ERR_MISALIGNED;   // record r's scale at r * (4 + numel)
    // each record's payload as a [numel / 4096][4096] matrix plus a one-row
    // tail, both with the header's single scale: a block edge above any size
    // makes every element's scale index 0
    constexpr int64_t kCols = 4096;
    const int64_t body_rows = numel / kCols, tail = numel % kCols;
    const size_t rec = fp8q_record_bytes_ex(numel, layout);
    const int head = packed ? 4 : 16;
    const int yb = dtype_bytes(yt);
    // up to 48 records (96 problems) per launch; nothing is allocated
    constexpr int kBatch = 96;
    DequantProblem probs[kBatch];
    int n = 0;
    for (int r = 0; r < count; ++r) {
        const uint8_t* base = records + (size_t)r * rec;
        const float* sc = reinterpret_cast<const float*>(base);
        uint8_t* yr = static_cast<uint8_t*>(y) + (size_t)r * numel * yb;
        if (body_rows) probs[n++] = DequantProblem{base + head, sc, yr, body_rows, kCols};
        if (tail) probs[n++] = DequantProblem{base + head + body_rows * kCols, sc, yr + body_rows * kCols * yb, 1, tail};
        if (n > kBatch - 2 || r == count - 1) {
            const fp8q_status st = launch_dequant(probs, n, fmt, kGranBlock, 1 << 30, yt,
                                                  reinterpret_cast<cudaStream_t>(stream));
            if (st != FP8Q_OK) return st;
            n = 0;
        }
    }
    return FP8Q_OK;
}

fp8q_status fp8q_unpack_records(const uint8_t* records, int count, int64_t numel, fp8q_format fmt, fp8q_dtype yt,
                                void* y, fp8q_stream_t stream) {
    return fp8q_unpack_records_ex(records, count, numel, fmt, yt, y, FP8Q_RECORD_ALIGNED16, stream);
}

fp8q_status fp8q_block_dequant(const uint8_t* w, fp8q_format fmt, int64_t M, int64_t N,
                               const float* scale_inv, int block, fp8q_dtype yt, void* y,
                               fp8q_stream_t stream) {
    fp8q_block_desc d = {w, scale_inv, y, M, N};
    return fp8q_block_dequant_grouped(&d, 1, fmt, block, yt, stream);
}

fp8q_status fp8q_block_dequant_grouped(const fp8q_block_desc* descs, int count, fp8q_format fmt, int block,
                                       fp8q_dtype yt, fp8q_stream_t stream) {
    if (!fmt_ok(fmt)) return FP8Q_ERR_BAD_FORMAT;
    if (!dtype_ok(yt)) return FP8Q_ERR_BAD_DTYPE;
    if (count < 0) return FP8Q_ERR_TOO_MANY;
    if (block < 1) return FP8Q_ERR_BAD_SHAPE;
    if (count == 0) return FP8Q_OK;
    if (!descs) return FP8Q_ERR_NULL_POINTER;
    for (int i = 0; i < count; ++i) {
        const fp8q_block_desc& d = descs[i];
        if (d.M < 0 || d.N < 0 || d.M > 0x7FFFFFFFLL || d.N > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
        const int64_t numel = checked_mul(d.M, d.N);
        if (numel < 0 || checked_mul(numel, dtype_bytes(yt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    }
    for (int i = 0; i < count; ++i) {
        const fp8q_block_desc& d = descs[i];
        if (d.M * d.N == 0) continue;
        if (!d.w || !d.scale_inv || !d.y) return FP8Q_ERR_NULL_POINTER;
    }
    for (int i = 0; i < count; ++i) {
        const fp8q_block_desc& d = descs[i];
        if (d.M * d.N == 0) continue;
        if (!aligned(d.scale_inv, 4) || !aligned(d.y, dtype_bytes(yt))) return FP8Q_ERR_MISALIGNED;
    }
    // problems on the stack in batches; each batch is one launch
    constexpr int kBatch = 96;
    DequantProblem probs[kBatch];
    for (int i = 0; i < count; i += kBatch) {
        const int nb = count - i < kBatch ? count - i : kBatch;
        for (int j = 0; j < nb; ++j) {
            const fp8q_block_desc& d = descs[i + j];
            probs[j] = DequantProblem{d.w, d.scale_inv, d.y, d.M, d.N};
        }
        fp8q_status st = launch_dequant(probs, nb, fmt, kGranBlock, block, yt,
                                        reinterpret_cast<cudaStream_t>(stream));
        if (st != FP8Q_OK) return st;
    }
    return FP8Q_OK;
}

fp8q_status fp8q_cast_from_fp8(const uint8_t* q, fp8q_format fmt, int64_t rows, int64_t cols,
                               const float* scale_inv, fp8q_granularity gran, int group_or_block,
                               fp8q_dtype yt, void* y, fp8q_stream_t stream) {
    if (!fmt_ok(fmt)) return FP8Q_ERR_BAD_FORMAT;
    if (!dtype_ok(yt)) return FP8Q_ERR_BAD_DTYPE;
    if (gran < FP8Q_GRAN_TENSOR || gran > FP8Q_GRAN_BLOCK) return FP8Q_ERR_BAD_GRANULARITY;
    if (rows < 0 || cols < 0 || rows > 0x7FFFFFFFLL || cols > 0x7FFFFFFFLL) return FP8Q_ERR_BAD_SHAPE;
    const bool sized = gran == FP8Q_GRAN_GROUP || gran == FP8Q_GRAN_BLOCK;
    if (sized && group_or_block < 1) return FP8Q_ERR_BAD_SHAPE;
    if (gran == FP8Q_GRAN_GROUP && cols % group_or_block != 0) return FP8Q_ERR_BAD_SHAPE;
    const int64_t numel = checked_mul(rows, cols);
    if (numel < 0 || checked_mul(numel, dtype_bytes(yt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    if (numel == 0) return FP8Q_OK;
    if (!q || !scale_inv || !y) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(scale_inv, 4) || !aligned(y, dtype_bytes(yt))) return FP8Q_ERR_MISALIGNED;
    DequantProblem p{q, scale_inv, y, rows, cols};
    return launch_dequant(&p, 1, fmt, gran, sized ? group_or_block : 1, yt,
                          reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// shared checks of the two fp8 products; returns FP8Q_OK to go on
fp8q_status check_scaled_mm(const uint8_t* a, int fa, const uint8_t* b, int fb, int64_t M, int64_t N, int64_t K,
                            const float* sa, const float* sb, const void* bias, int yt, const void* d,
                            const uint32_t* status, bool* nothing, int a_mn = 0, int b_mn = 0) {
    *nothing = false;
    if (!dtype_ok(yt)) return FP8Q_ERR_BAD_DTYPE;
    if (!fmt_ok(fa) || !fmt_ok(fb)) return FP8Q_ERR_BAD_FORMAT;
    const int64_t lim = 0x7FFFFFFFLL - 512;
    if (M < 0 || N < 0 || K < 0 || M > lim || N > lim || K > lim) return FP8Q_ERR_BAD_SHAPE;
    // the row pitch of every operand is a multiple of 16 bytes (TMA)
    if ((!(a_mn && b_mn) && K % 16 != 0) || (a_mn && M % 16 != 0) || (b_mn && N % 16 != 0))
        return FP8Q_ERR_BAD_SHAPE;
    const int64_t mn = checked_mul(M, N);
    if (mn < 0 || checked_mul(mn, dtype_bytes(yt)) < 0 || checked_mul(M, K) < 0 || checked_mul(N, K) < 0)
        return FP8Q_ERR_BAD_SHAPE;
    if (mn == 0) {
        *nothing = true;
        return FP8Q_OK;
    }
    if (!d) return FP8Q_ERR_NULL_POINTER;
    if (K > 0 && (!a || !b || !sa || !sb)) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(d, dtype_bytes(yt)) || (bias && !aligned(bias, dtype_bytes(yt))) || (status && !aligned(status, 4)))
        return FP8Q_ERR_MISALIGNED;
    if (K > 0 && (!aligned(a, 16) || !aligned(b, 16) || !aligned(sa, 4) || !aligned(sb, 4)))
        return FP8Q_ERR_MISALIGNED;
    return FP8Q_OK;
}

}  // namespace

extern "C" {

fp8q_status fp8q_scaled_mm(const uint8_t* a, fp8q_format fa, const uint8_t* b, fp8q_format fb, int64_t M,
                           int64_t N, int64_t K, const float* scale_a, const float* scale_b, const void* bias,
                           fp8q_dtype yt, void* d, uint32_t* status, fp8q_stream_t stream) {
    bool nothing = false;
    fp8q_status st = check_scaled_mm(a, fa, b, fb, M, N, K, scale_a, scale_b, bias, yt, d, status, &nothing);
    if (st != FP8Q_OK || nothing) return st;
    // the per-tensor epilogue reads both scales even when K == 0
    if (!scale_a || !scale_b) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(scale_a, 4) || !aligned(scale_b, 4)) return FP8Q_ERR_MISALIGNED;
    return launch_scaled_mm(a, fa, b, fb, M, N, K, scale_a, 0, scale_b, 0, false, bias, yt, d, status,
                            reinterpret_cast<cudaStream_t>(stream));
}

fp8q_status fp8q_scaled_mm_wait_test(const uint8_t* a, const uint8_t* b, int64_t M, int64_t N, int64_t K,
                                     const float* scale_a, const float* scale_b, void* d, uint32_t* status,
                                     uint64_t wait_limit_ns, int stall_kb, fp8q_stream_t stream) {
    bool nothing = false;
    fp8q_status st = check_scaled_mm(a, FP8Q_E4M3FN, b, FP8Q_E4M3FN, M, N, K, scale_a, scale_b, nullptr, FP8Q_BF16, d,
                                     status, &nothing);
    if (st != FP8Q_OK) return st;
    if (nothing || K == 0 || wait_limit_ns == 0 || wait_limit_ns > 4000000000ull || stall_kb < -1 ||
        stall_kb >= (K + 127) / 128)
        return FP8Q_ERR_BAD_SHAPE;
    if (!status || !scale_a || !scale_b) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(scale_a, 4) || !aligned(scale_b, 4)) return FP8Q_ERR_MISALIGNED;
    return launch_scaled_mm(a, FP8Q_E4M3FN, b, FP8Q_E4M3FN, M, N, K, scale_a, 0, scale_b, 0, false, nullptr, FP8Q_BF16,
                            d, status, reinterpret_cast<cudaStream_t>(stream), 0, 0, wait_limit_ns, stall_kb);
}

fp8q_status fp8q_scaled_mm_blockwise_wait_test(const uint8_t* a, const float* scale_a, const uint8_t* b,
                                               const float* scale_b, int64_t M, int64_t N, int64_t K, void* d,
                                               uint32_t* status, uint64_t wait_limit_ns, int stall_kb,
                                               fp8q_stream_t stream) {
    bool nothing = false;
    fp8q_status st = check_scaled_mm(a, FP8Q_E4M3FN, b, FP8Q_E4M3FN, M, N, K, scale_a, scale_b, nullptr, FP8Q_BF16, d,
                                     status, &nothing);
    if (st != FP8Q_OK) return st;
    if (nothing || K == 0 || wait_limit_ns == 0 || wait_limit_ns > 4000000000ull || stall_kb < -1 ||
        stall_kb >= (K + 127) / 128)
        return FP8Q_ERR_BAD_SHAPE;
    if (!status) return FP8Q_ERR_NULL_POINTER;
    const int kb = static_cast<int>((K + 127) / 128);
    return launch_scaled_mm(a, FP8Q_E4M3FN, b, FP8Q_E4M3FN, M, N, K, scale_a, kb, scale_b, kb, true, nullptr, FP8Q_BF16,
                            d, status, reinterpret_cast<cudaStream_t>(stream), 0, 0, wait_limit_ns, stall_kb);
}

fp8q_status fp8q_scaled_mm_blockwise(const uint8_t* a, fp8q_format fa, const float* scale_a, const uint8_t* b,
                                     fp8q_format fb, const float* scale_b, int64_t M, int64_t N, int64_t K,
                                     const void* bias, fp8q_dtype yt, void* d, uint32_t* status,
                                     fp8q_stream_t stream) {
    bool nothing = false;
    fp8q_status st = check_scaled_mm(a, fa, b, fb, M, N, K, scale_a, scale_b, bias, yt, d, status, &nothing);
    if (st != FP8Q_OK || nothing) return st;
    const int kb = static_cast<int>((K + 127) / 128);
    return launch_scaled_mm(a, fa, b, fb, M, N, K, scale_a, kb, scale_b, kb, true, bias, yt, d, status,
                            reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

extern "C" {

fp8q_status fp8q_transpose_fp8(const uint8_t* src, int64_t rows, int64_t cols, uint8_t* dst, int64_t ld,
                               fp8q_stream_t stream) {
    if (rows < 0 || cols < 0 || ld < rows) return FP8Q_ERR_BAD_SHAPE;
    if (checked_mul(rows, cols) < 0 || checked_mul(cols, ld) < 0) return FP8Q_ERR_BAD_SHAPE;
    if (checked_mul(cols, ld) == 0) return FP8Q_OK;
    if (!dst || (rows > 0 && !src)) return FP8Q_ERR_NULL_POINTER;
    return launch_transpose(src, rows, cols, dst, ld, reinterpret_cast<cudaStream_t>(stream));
}

fp8q_status fp8q_sum_rows(const void* x, fp8q_dtype xt, int64_t rows, int64_t cols, void* out,
                          fp8q_stream_t stream) {
    if (!dtype_ok(xt)) return FP8Q_ERR_BAD_DTYPE;
    if (rows < 0 || cols < 0) return FP8Q_ERR_BAD_SHAPE;
    const int64_t numel = checked_mul(rows, cols);
    if (numel < 0 || checked_mul(numel, dtype_bytes(xt)) < 0) return FP8Q_ERR_BAD_SHAPE;
    if (cols == 0) return FP8Q_OK;
    if (!out || (rows > 0 && !x)) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(out, dtype_bytes(xt)) || (x && !aligned(x, dtype_bytes(xt)))) return FP8Q_ERR_MISALIGNED;
    return launch_sum_rows(x, xt, rows, cols, out, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

extern "C" {

fp8q_status fp8q_scaled_mm_ex(const uint8_t* a, fp8q_format fa, fp8q_layout a_layout, const uint8_t* b,
                              fp8q_format fb, fp8q_layout b_layout, int64_t M, int64_t N, int64_t K,
                              const float* scale_a, const float* scale_b, const void* bias, fp8q_dtype yt, void* d,
                              uint32_t* status, fp8q_stream_t stream) {
    if ((a_layout != FP8Q_K_MAJOR && a_layout != FP8Q_MN_MAJOR) || (b_layout != FP8Q_K_MAJOR && b_layout != FP8Q_MN_MAJOR))
        return FP8Q_ERR_BAD_SHAPE;
    const int a_mn = a_layout == FP8Q_MN_MAJOR, b_mn = b_layout == FP8Q_MN_MAJOR;
    bool nothing = false;
    fp8q_status st = check_scaled_mm(a, fa, b, fb, M, N, K, scale_a, scale_b, bias, yt, d, status, &nothing, a_mn, b_mn);
    if (st != FP8Q_OK || nothing) return st;
    if (!scale_a || !scale_b) return FP8Q_ERR_NULL_POINTER;
    if (!aligned(scale_a, 4) || !aligned(scale_b, 4)) return FP8Q_ERR_MISALIGNED;
    return launch_scaled_mm(a, fa, b, fb, M, N, K, scale_a, 0, scale_b, 0, false, bias, yt, d, status,
                            reinterpret_cast<cudaStream_t>(stream), a_mn, b_mn);
}

}  // extern "C"
