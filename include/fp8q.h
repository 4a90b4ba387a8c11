/*
 * fp8q.h -- C ABI of libfp8q, scaled FP8 casting on NVIDIA B200 (sm_100a).
 *
 * Operations (each entry point cites the passage that defines it):
 *   fp8q_per_token_group_quant  DeepEP "5 Utils", per_token_cast_to_fp8
 *   fp8q_cast_per_channel       ColossalAI colossalai/quantization/fp8.py,
 *                               cast_to_fp8 (per_channel_scale=True)
 *   fp8q_cast_per_tensor        ColossalAI cast_to_fp8 (per-tensor branch)
 *   fp8q_block_dequant(_grouped) DeepSeek-V3 fp8_cast_bf16 blog,
 *                               weight_dequant / weight_dequant_kernel
 *   fp8q_cast_from_fp8          ColossalAI cast_from_fp8; DeepEP
 *                               per_token_cast_back
 *   fp8q_scaled_mm              ColossalAI _LinearFp8.forward (torch._scaled_mm)
 *   fp8q_scaled_mm_ex           the same with either operand stored MN-major
 *                               (_LinearFp8.backward's transposed operands)
 *   fp8q_scaled_mm_blockwise    DeepEP per-token activations x DeepSeek-V3
 *                               block-scaled weight
 *   fp8q_transpose_fp8,         ColossalAI _LinearFp8.backward (the operand
 *   fp8q_sum_rows               transposes and the bias gradient)
 *   fp8q_tensor_amax,           the per-tensor cast of a tensor sharded over
 *   fp8q_cast_per_tensor_with_amax  ranks (ColossalAI FSDP params hook)
 *   fp8q_cast_pipeline,         ColossalAI cast_to_fp8_pipeline /
 *   fp8q_cast_from_pipeline     cast_from_fp8_pipeline
 *   fp8q_pack_record(_ex),      ColossalAI all_gather_fp8: the [scale |
 *   fp8q_unpack_records(_ex)    payload] records (_ex: the page's packed
 *                               4-byte-header layout as well)
 *   fp8q_*_ex                   torch's rounding of the scale expressions
 *   fp8q_scaled_mm_wait_test,   tests of the products' bounded waits
 *   fp8q_scaled_mm_blockwise_wait_test
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors are caller-owned DEVICE pointers to contiguous row-major data.
 *   fp8 tensors are raw bytes (uint8_t codes); high-precision tensors are
 *   fp32, fp16 or bf16 as named by an fp8q_dtype argument.
 * - The library never allocates or frees memory, never synchronises, keeps
 *   no state between calls and enqueues all work on the given stream (NULL =
 *   the legacy default stream).  Calls on different streams are independent.
 *   Calls return as soon as the work is enqueued; outputs are valid once the
 *   stream reaches that point.  The stream must belong to the current device
 *   and the tensors must live on it: launch shapes are sized from the
 *   current device's SM count.
 * - Arithmetic is IEEE binary32 with round-to-nearest-even: scales are
 *   computed with true division (fl(FMAX / amax)), products are single
 *   fp32 multiplies, narrowing to fp8 / bf16 / fp16 rounds to nearest-even.
 *   The fp8 cast does not saturate: a magnitude that rounds above the
 *   format's maximum becomes NaN (e4m3fn) or Inf (e5m2), as torch's
 *   .to(float8_*) does.  Denormals are kept (no flush to zero).
 *   FMAX is 448 (e4m3fn) or 57344 (e5m2).
 * - Every argument is validated on the host before anything is enqueued, in
 *   this order: enums, sizes and shape rules, null pointers, alignment.  A
 *   pointer may be NULL only when its tensor has no elements.  On any error
 *   nothing is enqueued.  Errors reported by the CUDA runtime while
 *   enqueueing map to FP8Q_ERR_CUDA.  The library never aborts and never
 *   traps on the device.
 * - Alignment: each pointer must be aligned to its element size
 *   (FP8Q_ERR_MISALIGNED otherwise).  16-byte aligned pointers and row
 *   strides take the vectorised paths; other layouts are still accepted and
 *   take narrower loads.
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so this header needs no CUDA include. */
typedef struct CUstream_st* fp8q_stream_t;

typedef enum {
    FP8Q_E4M3FN = 0, /* float8_e4m3fn: bias 7, 3 mantissa bits, no Inf, max 448 */
    FP8Q_E5M2 = 1    /* float8_e5m2:   bias 15, 2 mantissa bits, max 57344 */
} fp8q_format;

typedef enum { FP8Q_F32 = 0, FP8Q_F16 = 1, FP8Q_BF16 = 2 } fp8q_dtype;

typedef enum {
    FP8Q_GRAN_TENSOR = 0, /* one scale for the whole tensor: scale_inv[0] */
    FP8Q_GRAN_ROW = 1,    /* one scale per row: scale_inv[r] */
    FP8Q_GRAN_GROUP = 2,  /* 1 x G groups along a row: scale_inv[r * (cols/G) + c/G] */
    FP8Q_GRAN_BLOCK = 3   /* B x B blocks: scale_inv[(r/B) * ceil(cols/B) + c/B] */
} fp8q_granularity;

/*
 * How the scale and scale_inv divisions are rounded (the pages write them as
 * `FMAX / amax` and `amax / FMAX` without saying more):
 *   FP8Q_SCALE_IEEE   one IEEE binary32 division each: scale = fl(FMAX / amax),
 *                     scale_inv = fl(amax / FMAX).  The default of every call.
 *   FP8Q_SCALE_TORCH  the order in which torch evaluates those expressions on
 *                     a CUDA tensor, for byte parity with outputs torch
 *                     produced: a Python number divided by a tensor is the
 *                     tensor's reciprocal times the number, scale =
 *                     fl(fl(1 / amax) * FMAX); a CUDA tensor divided by a
 *                     Python number is a multiply by the number's reciprocal,
 *                     scale_inv = fl(amax * fl(1 / FMAX)).  The per-tensor
 *                     scale_inv = fl(1 / scale) is the same under both rules.
 */
typedef enum { FP8Q_SCALE_IEEE = 0, FP8Q_SCALE_TORCH = 1 } fp8q_scale_rule;

typedef enum {
    FP8Q_OK = 0,
    FP8Q_ERR_NULL_POINTER = 1,    /* a non-empty tensor was given as NULL */
    FP8Q_ERR_BAD_DTYPE = 2,       /* dtype not fp32/fp16/bf16 (the pages' TypeError) */
    FP8Q_ERR_BAD_FORMAT = 3,      /* format not e4m3fn/e5m2 (the pages' TypeError) */
    FP8Q_ERR_BAD_SHAPE = 4,       /* negative size, n % group != 0, bad group/block edge */
    FP8Q_ERR_MISALIGNED = 5,      /* pointer not aligned to its element size */
    FP8Q_ERR_WORKSPACE = 6,       /* workspace missing or too small */
    FP8Q_ERR_CUDA = 7,            /* the CUDA runtime refused a launch */
    FP8Q_ERR_BAD_GRANULARITY = 8, /* granularity enum out of range */
    FP8Q_ERR_TOO_MANY = 9,        /* grouped call: count < 0 */
    FP8Q_ERR_BAD_RULE = 10        /* scale rule enum out of range */
} fp8q_status;

/* Human-readable name of a status code (static storage; never NULL). */
const char* fp8q_status_string(fp8q_status status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int fp8q_version(void);

/*
 * Per-token group quantisation -- DeepEP "5 Utils", per_token_cast_to_fp8:
 *   for each row r and group g of `group` consecutive elements,
 *     amax      = max(max_k |float(x[r][g*group + k])|, fl32(1e-4))  (clamp)
 *     scale     = fl(FMAX / amax)
 *     q[r][c]   = fp8(fl(float(x[r][c]) * scale))
 *     scale_inv[r][g] = fl(amax / FMAX)
 *   A NaN in a group makes its amax, scales and codes NaN (torch's amax and
 *   clamp keep NaN).  The pages fix group = 128 and e4m3fn; any group that
 *   divides n is accepted (powers of two from 16 to 1024 take the vector path).
 * x:         [m][n] elements of type xt (fp32, fp16 or bf16).
 * q:         [m][n] fp8 codes (output).
 * scale_inv: [m][n/group] fp32 (output).
 * Errors: n % group != 0 or group < 1 -> FP8Q_ERR_BAD_SHAPE (the page's
 *   assert on x.size(1) % 128).  m == 0 or n == 0 writes nothing.
 */
fp8q_status fp8q_per_token_group_quant(const void* x, fp8q_dtype xt, int64_t m, int64_t n,
                                       int group, fp8q_format fmt, uint8_t* q,
                                       float* scale_inv, fp8q_stream_t stream);

/* The same with an explicit scale rule (fp8q_scale_rule). */
fp8q_status fp8q_per_token_group_quant_ex(const void* x, fp8q_dtype xt, int64_t m, int64_t n,
                                          int group, fp8q_format fmt, uint8_t* q,
                                          float* scale_inv, fp8q_scale_rule rule,
                                          fp8q_stream_t stream);

/*
 * Per-channel cast -- ColossalAI cast_to_fp8 with per_channel_scale=True:
 *   amax[r]      = max_c |x[r][c]|, then amax[r] := amax[r] > 0 ? amax[r] : 1
 *                  (a NaN amax fails the test and becomes 1)
 *   scale[r]     = fl(FMAX / amax[r]);  scale_inv[r] = fl(amax[r] / FMAX)
 *   q[r][c]      = fp8(fl(float(x[r][c]) * scale[r]))
 *   Row r dequantises with scale_inv[r].
 * x: [rows][cols] of type xt; q: [rows][cols]; scale_inv: [max(rows, 1)].
 * Empty tensor (rows * cols == 0): scale_inv[0 .. max(rows,1)) = 1.0 (the
 *   page returns tensor([1.0]) for an empty input); q is not touched.
 */
fp8q_status fp8q_cast_per_channel(const void* x, fp8q_dtype xt, int64_t rows, int64_t cols,
                                  fp8q_format fmt, uint8_t* q, float* scale_inv,
                                  fp8q_stream_t stream);

/* The same with an explicit scale rule (fp8q_scale_rule). */
fp8q_status fp8q_cast_per_channel_ex(const void* x, fp8q_dtype xt, int64_t rows, int64_t cols,
                                     fp8q_format fmt, uint8_t* q, float* scale_inv,
                                     fp8q_scale_rule rule, fp8q_stream_t stream);

/*
 * Per-tensor cast -- ColossalAI cast_to_fp8 per-tensor branch:
 *   amax = max |x| over all numel elements, amax := amax > 0 ? amax : 1
 *   scale = fl(FMAX / amax);  scale_inv[0] = fl(1 / scale)
 *   q[i] = fp8(fl(float(x[i]) * scale))
 * Two passes over x (an amax reduction, then the scaled cast) in two kernels;
 * the first writes per-CTA partial maxima into `workspace`, the second
 * reduces them.  No atomics, no spin-waits, deterministic.
 * workspace: device memory of at least fp8q_cast_per_tensor_workspace_bytes()
 *   bytes, 16-byte aligned, owned by the caller; its contents need no
 *   initialisation and are scratch after the call.  Calls that share one
 *   workspace must be ordered (same stream, or synchronised).
 * Empty tensor (numel == 0): scale_inv[0] = 1.0 is written on the stream.
 */
size_t fp8q_cast_per_tensor_workspace_bytes(void);
fp8q_status fp8q_cast_per_tensor(const void* x, fp8q_dtype xt, int64_t numel, fp8q_format fmt,
                                 uint8_t* q, float* scale_inv, void* workspace,
                                 size_t workspace_bytes, fp8q_stream_t stream);
/* The same with an explicit scale rule (fp8q_scale_rule). */
fp8q_status fp8q_cast_per_tensor_ex(const void* x, fp8q_dtype xt, int64_t numel, fp8q_format fmt,
                                    uint8_t* q, float* scale_inv, void* workspace,
                                    size_t workspace_bytes, fp8q_scale_rule rule,
                                    fp8q_stream_t stream);

/*
 * Per-tensor cast without a caller workspace.  The paper has no counterpart:
 * this entry point is a convenience of this library, not part of the method.
 * Same computation and bytes as fp8q_cast_per_tensor, for callers that
 * cannot allocate device memory -- for example code running under an
 * allocator that owns all of the GPU's memory, or code that must not call
 * cudaMalloc because that call may synchronise the device.  The scratch for
 * the amax pass lives in a file-scope __device__ array inside the library:
 * 8 KiB (2048 per-CTA partial maxima), present on every GPU that loads the
 * library until the process exits.  Every tensor size fits: the amax pass
 * clamps its grid to 2048 CTAs, one partial maximum each, so no size is
 * refused for want of scratch (FP8Q_ERR_WORKSPACE is never returned).
 * - The call allocates nothing (no cudaMalloc / cudaFree).  The first call on
 *   a device looks up the array's device address on that device (with it
 *   current) and caches it; make that first call before any stream capture.
 *   The cached address is the primary context's: after cudaDeviceReset do
 *   not call this entry point again in the same process.
 * - `stream` must belong to the current device, and x, q and scale_inv must
 *   live on it (the scratch used is the current device's).
 * - All calls share the one array per device, and it keeps the last call's
 *   contents; nothing needs clearing, since each call writes every slot it
 *   reads.  Calls whose work overlaps on the GPU (different streams, no
 *   ordering between them) race on the array and may give wrong results;
 *   order them on one stream or synchronise.
 * Arguments, errors and empty-tensor rule as fp8q_cast_per_tensor.
 */
fp8q_status fp8q_cast_per_tensor_noalloc(const void* x, fp8q_dtype xt, int64_t numel, fp8q_format fmt,
                                         uint8_t* q, float* scale_inv, fp8q_stream_t stream);

/*
 * Per-tensor cast of a tensor sharded across ranks, in two calls with a
 * 4-byte exchange between them -- the pattern of ColossalAI
 * fp8_compress_fsdp_params_comm_hook (all_reduce(MAX) of the per-tensor max,
 * then scale = fp8_max / max on every rank):
 *   fp8q_tensor_amax:   amax_bits[0] = fp32 bit pattern of max |x| over this
 *                       rank's numel elements (0 for an empty shard).  The
 *                       sign bit is clear, so as int32 the words of all
 *                       ranks order like the magnitudes and every NaN lies
 *                       above +Inf: an integer MAX over ranks (e.g. NCCL
 *                       all_reduce MAX on int32) gives the amax of the whole
 *                       tensor with NaN propagating.
 *   fp8q_cast_per_tensor_with_amax: the per-tensor cast of this shard with the
 *                       amax read from amax_bits[0] (zero or NaN replaced by
 *                       1, scale and scale_inv as in fp8q_cast_per_tensor).
 * Every rank then holds the bytes the one-tensor cast gives for its slice,
 * and every rank -- one with an empty shard too -- the same scale_inv, derived
 * from the global amax.  (The one-tensor calls return scale_inv = 1.0 for an
 * empty tensor; a sharded tensor that is empty on every rank has amax 0,
 * which becomes 1 as for any zero tensor, so its scale_inv is fl(1 / FMAX).)
 * amax_bits: device uint32 [1]; workspace as fp8q_cast_per_tensor.
 */
fp8q_status fp8q_tensor_amax(const void* x, fp8q_dtype xt, int64_t numel, uint32_t* amax_bits,
                             void* workspace, size_t workspace_bytes, fp8q_stream_t stream);
fp8q_status fp8q_cast_per_tensor_with_amax(const void* x, fp8q_dtype xt, int64_t numel, fp8q_format fmt,
                                           const uint32_t* amax_bits, uint8_t* q, float* scale_inv,
                                           fp8q_scale_rule rule, fp8q_stream_t stream);

/*
 * Pipeline cast -- ColossalAI cast_to_fp8_pipeline: a per-tensor cast whose
 * fp8 format follows the data, for activations sent between pipeline stages.
 *   amax  = max |x| over all numel elements (NaN propagates)
 *   fmt   = amax > 448 (the e4m3fn maximum) ? e5m2 : e4m3fn
 *           (a NaN amax fails the test and gives e4m3fn)
 *   scale = amax == 0 ? 1 : FMAX(fmt) / amax        (rounded per `rule`)
 *   q[i]  = fmt(fl(float(x[i]) * scale)); scale_inv[0] = fl(1 / scale)
 *   fmt_tag[0] = the chosen fp8q_format (0 e4m3fn, 1 e5m2)
 * The page carries the format in the view dtype of the payload; here it is
 * a device int32 written on the stream, so the call needs no host round
 * trip and the decode reads it on the device.  Two kernels, as
 * fp8q_cast_per_tensor, with the same workspace rules.
 * Empty tensor (numel == 0): scale_inv[0] = 1.0 and fmt_tag[0] = e4m3fn.
 */
fp8q_status fp8q_cast_pipeline(const void* x, fp8q_dtype xt, int64_t numel, uint8_t* q,
                               float* scale_inv, int32_t* fmt_tag, void* workspace,
                               size_t workspace_bytes, fp8q_scale_rule rule, fp8q_stream_t stream);

/*
 * Pipeline decode -- ColossalAI cast_from_fp8_pipeline:
 *   y[i] = T(fl(float(q[i]) * scale_inv[0])), the codes read in the format
 *   fmt_tag[0] names (a device int32 as fp8q_cast_pipeline writes it: 1 is
 *   e5m2, any other value e4m3fn).
 * q: numel codes; scale_inv: [1]; y: numel elements of yt (output).
 */
fp8q_status fp8q_cast_from_pipeline(const uint8_t* q, int64_t numel, const float* scale_inv,
                                    const int32_t* fmt_tag, fp8q_dtype yt, void* y,
                                    fp8q_stream_t stream);

/*
 * fp8-compressed all-gather records -- ColossalAI all_gather_fp8_lagacy (and
 * _all_gather_fp8): every rank casts its tensor with its own per-tensor
 * scale and sends [scale | fp8 payload]; every rank then dequantises each
 * received chunk with the scale in its header.  A record here is
 *   bytes [0, 4)            fp32 scale_inv (fl(1 / scale) of the per-tensor cast)
 *   bytes [4, 16)           zero
 *   bytes [16, 16 + numel)  fp8 codes, then zero padding to a multiple of 16
 * (the page uses a 4-byte header, offered by the _ex calls below; 16 keeps
 * the payload 16-byte aligned), so
 * records of equal numel can be gathered back to back by any byte-level
 * all-gather (NCCL all_gather_into_tensor on uint8).
 *   fp8q_record_bytes:   the record size for numel codes.
 *   fp8q_pack_record:    the per-tensor cast of x into `record` (scale rule as
 *                        fp8q_cast_per_tensor_ex; workspace likewise).
 *   fp8q_unpack_records: `count` records of numel codes each, laid out
 *                        back to back (records 16-byte aligned), dequantised
 *                        into y[count][numel] (type yt, element-aligned):
 *                        y[r][i] = T(fl(float(code) * scale_inv of record r)),
 *                        one launch per 48 records.  count == 0 or numel == 0
 *                        enqueues nothing.
 * Ownership and errors as for the calls above: caller-owned device buffers,
 * host-side checks before any launch, nothing allocated.
 */
size_t fp8q_record_bytes(int64_t numel);
fp8q_status fp8q_pack_record(const void* x, fp8q_dtype xt, int64_t numel, fp8q_format fmt, uint8_t* record,
                             void* workspace, size_t workspace_bytes, fp8q_scale_rule rule,
                             fp8q_stream_t stream);
fp8q_status fp8q_unpack_records(const uint8_t* records, int count, int64_t numel, fp8q_format fmt,
                                fp8q_dtype yt, void* y, fp8q_stream_t stream);

/*
 * The same records in either layout:
 *   FP8Q_RECORD_PACKED4    the page's own layout (ColossalAI
 *                          all_gather_fp8_lagacy, SCALE_BYTES = 4): bytes
 *                          [0, 4) the fp32 scale_inv, bytes [4, 4 + numel)
 *                          the codes, no padding; record r of a gathered
 *                          buffer starts at r * (4 + numel).
 *   FP8Q_RECORD_ALIGNED16  the layout above (16-byte header, payload padded
 *                          to a multiple of 16); the calls without _ex.
 * A packed record's scale is read and written as an fp32, so it must be
 * 4-byte aligned: pack wants `record` 4-byte aligned, and unpack wants
 * `records` 4-byte aligned and, when count > 1, numel a multiple of 4 (so
 * that every record's scale is); otherwise FP8Q_ERR_MISALIGNED.  Its payload
 * starts 4 bytes in and takes the narrower accesses of an unaligned tensor.
 * fp8q_record_bytes_ex returns 0 for numel < 0 or an unknown layout; the
 * other two return FP8Q_ERR_BAD_SHAPE for an unknown layout.  Everything
 * else as fp8q_pack_record / fp8q_unpack_records.
 */
typedef enum { FP8Q_RECORD_PACKED4 = 4, FP8Q_RECORD_ALIGNED16 = 16 } fp8q_record_layout;
size_t fp8q_record_bytes_ex(int64_t numel, fp8q_record_layout layout);
fp8q_status fp8q_pack_record_ex(const void* x, fp8q_dtype xt, int64_t numel, fp8q_format fmt, uint8_t* record,
                                void* workspace, size_t workspace_bytes, fp8q_scale_rule rule,
                                fp8q_record_layout layout, fp8q_stream_t stream);
fp8q_status fp8q_unpack_records_ex(const uint8_t* records, int count, int64_t numel, fp8q_format fmt,
                                   fp8q_dtype yt, void* y, fp8q_record_layout layout, fp8q_stream_t stream);

/*
 * Block dequantisation -- DeepSeek-V3 weight_dequant / weight_dequant_kernel:
 *   y[i][j] = T(fl(float(w[i][j]) * scale_inv[i / B][j / B]))
 *   with scale_inv row-major [ceil(M/B)][ceil(N/B)] (the kernel's
 *   pid_m * cdiv(N, B) + pid_n index); partial edge blocks use their own
 *   scale.  T is bf16 on the pages (the default dtype the converter sets);
 *   fp16 and fp32 outputs are also offered.  The pages fix B = 128 and
 *   e4m3fn weights; e5m2 weights are also accepted.
 * w: [M][N] fp8 codes; scale_inv as above; y: [M][N] of type yt (output).
 * Errors: block < 1 -> FP8Q_ERR_BAD_SHAPE.
 */
fp8q_status fp8q_block_dequant(const uint8_t* w, fp8q_format fmt, int64_t M, int64_t N,
                               const float* scale_inv, int block, fp8q_dtype yt, void* y,
                               fp8q_stream_t stream);

/*
 * Many block dequantisations in one launch (the converter's loop over every
 * fp8 weight of a checkpoint, e.g. a mixture-of-experts layer).  `descs` is a
 * HOST array of `count` descriptors, read during the call only; each entry
 * is one fp8q_block_dequant problem with its own shape and pointers; fmt,
 * block and yt are shared.  Bytes written are identical to calling
 * fp8q_block_dequant once per entry.  Entries with M * N == 0 are skipped.
 * Large counts are split into several launches internally.
 */
typedef struct {
    const uint8_t* w;       /* [M][N] fp8 codes */
    const float* scale_inv; /* [ceil(M/B)][ceil(N/B)] fp32 */
    void* y;                /* [M][N] of the shared output type */
    int64_t M;
    int64_t N;
} fp8q_block_desc;

fp8q_status fp8q_block_dequant_grouped(const fp8q_block_desc* descs, int count,
                                       fp8q_format fmt, int block, fp8q_dtype yt,
                                       fp8q_stream_t stream);

/*
 * Dequantising cast -- ColossalAI cast_from_fp8 (ret = scale_inv * q.float(),
 * then .to(ret_type)), and DeepEP per_token_cast_back for 1 x G groups:
 *   y[r][c] = T(fl(scale_inv[granule(r, c)] * float(q[r][c])))
 * granule per fp8q_granularity above; group_or_block is G (GROUP) or B
 * (BLOCK) and is ignored for TENSOR and ROW.  For a per-channel cast the
 * intended row scaling is used (row r by scale_inv[r]).
 * q: [rows][cols] codes; scale_inv: granule-count fp32; y: [rows][cols] of yt.
 * Errors: GROUP with cols % G != 0, or G / B < 1 -> FP8Q_ERR_BAD_SHAPE.
 */
fp8q_status fp8q_cast_from_fp8(const uint8_t* q, fp8q_format fmt, int64_t rows, int64_t cols,
                               const float* scale_inv, fp8q_granularity gran, int group_or_block,
                               fp8q_dtype yt, void* y, fp8q_stream_t stream);

/*
 * fp8 matrix product with per-tensor scales -- ColossalAI
 * colossalai/quantization/fp8.py, _LinearFp8.forward: both operands cast
 * with cast_to_fp8 (one scale_inv each), then torch._scaled_mm(x_fp8,
 * w_fp8.t(), scale_a, scale_b, bias, out_dtype):
 *   acc[m][n] = sum over k of float(a[m][k]) * float(b[n][k])   (tensor cores, fp32)
 *   d[m][n]   = T(fl(fl(acc[m][n] * fl(scale_a[0] * scale_b[0])) + bias[n]))
 * a: [M][K] fp8 codes (format fa), row-major (the activations x_fp8).
 * b: [N][K] fp8 codes (format fb), row-major: the weight as stored
 *    ([out features][in features]); the product uses its transpose.
 *    e4m3fn and e5m2 mix freely (the page's backward multiplies an e5m2
 *    gradient by an e4m3 weight).
 * scale_a, scale_b: device fp32 [1] each (the scale_inv the casts return).
 * bias: NULL or [N] of the output type yt (the page requires the input's dtype).
 * d: [M][N] of type yt (bf16, fp16 or fp32), row-major (output).
 * status: NULL or a device uint32 word.  Every internal wait of the kernel
 *    is bounded; if one runs out (a hardware fault, never in normal use) the
 *    kernel ORs a nonzero code into *status, leaves d incomplete and returns
 *    instead of hanging.  The caller clears the word; the library never
 *    reads it.
 * The fp32 sum is the tensor cores' own (its rounding is not IEEE-sequential);
 * tests hold it to an error bound relative to sum |a*b|, not to bit equality.
 * Errors: K % 16 != 0 (the row pitch of a and b must be a multiple of 16
 *   bytes), M, N or K above 2^31 - 512 -> FP8Q_ERR_BAD_SHAPE; a or b not
 *   16-byte aligned -> FP8Q_ERR_MISALIGNED.  M == 0 or N == 0 writes
 *   nothing; K == 0 writes the bias (or zeros).
 */
fp8q_status fp8q_scaled_mm(const uint8_t* a, fp8q_format fa, const uint8_t* b, fp8q_format fb,
                           int64_t M, int64_t N, int64_t K, const float* scale_a, const float* scale_b,
                           const void* bias, fp8q_dtype yt, void* d, uint32_t* status,
                           fp8q_stream_t stream);

/* Bits that a product kernel ORs into its status word when a wait runs out:
 * the copy producer, the tensor-core issuer, the epilogue (each of these
 * also stops the others), and the final wait for work still in flight. */
#define FP8Q_WAIT_PRODUCER 1u
#define FP8Q_WAIT_MMA      2u
#define FP8Q_WAIT_EPILOGUE 4u
#define FP8Q_WAIT_DRAIN    8u

/*
 * Test of the bounded waits (not for production use): fp8q_scaled_mm with
 * e4m3fn operands, no bias and bf16 output, run with every internal wait
 * bounded by wait_limit_ns (1 ns .. 4 s) instead of the default of a few
 * seconds.  stall_kb >= 0 leaves out the shared-memory copies of k-block
 * stall_kb of each CTA's first tile (on CTA pairs: the leading CTA's half of
 * its pair's first tile), so the barrier those copies would complete never
 * does: the waits that depend on it run out, the kernel ORs
 * FP8Q_WAIT_* bits into *status, waits (again bounded) for its own copies
 * and tensor-core work in flight, frees its tensor memory and returns, with
 * d left incomplete.  Every access stays inside the operands.  stall_kb = -1
 * runs the product normally under the given limit.
 * status: a device uint32 word, required.
 * Errors: as fp8q_scaled_mm; also K == 0, M or N == 0, wait_limit_ns outside
 *   1 .. 4e9 or stall_kb outside -1 .. ceil(K / 128) - 1 -> FP8Q_ERR_BAD_SHAPE.
 */
fp8q_status fp8q_scaled_mm_wait_test(const uint8_t* a, const uint8_t* b, int64_t M, int64_t N, int64_t K,
                                     const float* scale_a, const float* scale_b, void* d, uint32_t* status,
                                     uint64_t wait_limit_ns, int stall_kb, fp8q_stream_t stream);
/* The same test for the fine-grained product: fp8q_scaled_mm_blockwise with
 * e4m3fn operands, no bias and bf16 output (scale_a [M][ceil(K/128)],
 * scale_b [ceil(N/128)][ceil(K/128)]), every wait bounded by wait_limit_ns,
 * stall_kb as above.  Errors as fp8q_scaled_mm_blockwise and as above. */
fp8q_status fp8q_scaled_mm_blockwise_wait_test(const uint8_t* a, const float* scale_a, const uint8_t* b,
                                               const float* scale_b, int64_t M, int64_t N, int64_t K, void* d,
                                               uint32_t* status, uint64_t wait_limit_ns, int stall_kb,
                                               fp8q_stream_t stream);

/*
 * Operand layouts of fp8q_scaled_mm_ex.  With A the [M][K] operand and B the
 * [N][K] operand of the product (D = A B^T):
 *   FP8Q_K_MAJOR   stored [M][K] (resp. [N][K]) row-major: k is contiguous
 *   FP8Q_MN_MAJOR  stored [K][M] (resp. [K][N]) row-major: m (n) is contiguous,
 *                  i.e. the operand is the transpose of a row-major matrix
 */
typedef enum { FP8Q_K_MAJOR = 0, FP8Q_MN_MAJOR = 1 } fp8q_layout;

/*
 * fp8q_scaled_mm with a layout per operand, so that transposed operands
 * need no copy -- ColossalAI _LinearFp8.backward multiplies the output
 * gradient g [T][N] by the weight w [N][K] (input gradient: A = g K-major,
 * B = w MN-major) and g^T by x [T][K] (weight gradient: A = g MN-major,
 * B = x MN-major).  Same arithmetic, scales, bias, status and errors as
 * fp8q_scaled_mm; the row pitch rule becomes: K % 16 == 0 unless both
 * operands are MN-major, M % 16 == 0 for an MN-major A, N % 16 == 0 for an
 * MN-major B (FP8Q_ERR_BAD_SHAPE otherwise, also for an unknown layout).
 */
fp8q_status fp8q_scaled_mm_ex(const uint8_t* a, fp8q_format fa, fp8q_layout a_layout, const uint8_t* b,
                              fp8q_format fb, fp8q_layout b_layout, int64_t M, int64_t N, int64_t K,
                              const float* scale_a, const float* scale_b, const void* bias, fp8q_dtype yt, void* d,
                              uint32_t* status, fp8q_stream_t stream);

/*
 * fp8 matrix product with fine-grained scales: activations quantised by
 * per_token_cast_to_fp8 (DeepEP "5 Utils": one scale_inv per 1 x 128 group
 * of a row) times a weight stored with one scale_inv per 128 x 128 block
 * (DeepSeek-V3 fp8_cast_bf16 blog, weight_dequant) -- the product of the
 * two dequantised operands without materialising either:
 *   acc_kb[m][n] = sum over k in [128 kb, 128 kb + 128) of float(a[m][k]) * float(b[n][k])
 *   d[m][n]      = T(fl(sum over kb, ascending, of fl(scale_a[m][kb] * scale_b[n/128][kb]) * acc_kb[m][n])
 *                    + bias[n])     (each step one fused multiply-add)
 * a: [M][K] codes; scale_a: fp32 [M][ceil(K/128)] (per_token_cast_to_fp8's
 *    second output).  b: [N][K] codes; scale_b: fp32 [ceil(N/128)][ceil(K/128)]
 *    (the weight's scale_inv).  bias, d, status, formats and errors as
 *    fp8q_scaled_mm.
 */
fp8q_status fp8q_scaled_mm_blockwise(const uint8_t* a, fp8q_format fa, const float* scale_a,
                                     const uint8_t* b, fp8q_format fb, const float* scale_b,
                                     int64_t M, int64_t N, int64_t K, const void* bias, fp8q_dtype yt,
                                     void* d, uint32_t* status, fp8q_stream_t stream);

/*
 * Byte transpose of an fp8 matrix -- the .t().contiguous() copies that
 * ColossalAI _LinearFp8.backward makes of its fp8 operands (the weight for
 * the input gradient; the gradient and the input for the weight gradient):
 *   dst[c][r] = src[r][c]   for r < rows, c < cols
 *   dst[c][r] = 0           for rows <= r < ld  (zero padding of each dst row)
 * src: [rows][cols] bytes, row-major.  dst: [cols][ld] bytes, ld >= rows.
 * A pitch ld that is a multiple of 16 makes dst a legal operand of the fp8
 * products with K = ld (the zero padding adds nothing to the sums).
 * Errors: ld < rows or a negative size -> FP8Q_ERR_BAD_SHAPE.  rows == 0 or
 * cols == 0 with ld == 0 writes nothing.
 */
fp8q_status fp8q_transpose_fp8(const uint8_t* src, int64_t rows, int64_t cols, uint8_t* dst, int64_t ld,
                               fp8q_stream_t stream);

/*
 * Column sums -- the bias gradient of ColossalAI _LinearFp8.backward,
 * out_grad.sum(0):
 *   out[c] = T(sum over r of float(x[r][c]))
 * accumulated in fp32 in a fixed order (each column's rows split into 64
 * interleaved subsets, row r in subset r % 64, each summed in ascending row
 * order, then the 64 partial sums added in subset order), so repeated calls
 * give the same bits.
 * x: [rows][cols] of type xt; out: [cols] of type xt.  rows == 0 writes zeros.
 */
fp8q_status fp8q_sum_rows(const void* x, fp8q_dtype xt, int64_t rows, int64_t cols, void* out,
                          fp8q_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* FP8Q_H */
