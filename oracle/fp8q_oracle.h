/*
 * fp8q_oracle.h -- plain, slow CPU definition of scaled FP8 casting.
 *
 * TEST INFRASTRUCTURE ONLY.  This oracle exists so that tests, the smoke
 * check and the benchmark's CPU-baseline leg can check the CUDA library
 * against an independent, obviously-correct restatement of the method.  No
 * product code path may link, load or call it.  It shares no header, table or
 * helper with the CUDA library.
 *
 * Every floating-point step is one IEEE-754 binary32 operation with
 * round-to-nearest-even (built with -ffp-contract=off, SSE arithmetic, no
 * fast-math).  The fp8 / fp16 / bf16 codecs are written from the format
 * definitions (sign, biased exponent, mantissa, RNE), not from any library.
 *
 * Sources (the web pages this method is described on):
 *   [CAI]  ColossalAI colossalai/quantization/fp8.py (v0.4.4):
 *          cast_to_fp8 (per-channel and per-tensor branches, empty-tensor
 *          rule, dtype guard) and cast_from_fp8.
 *   [DEP]  DeepEP "5 Utils" blog: per_token_cast_to_fp8 (input check,
 *          128-element grouping, amax with clamp(1e-4), 448/amax scaling,
 *          amax/448 scales returned); per_token_cast_back named as the
 *          inverse.
 *   [DSV3] DeepSeek-V3 fp8_cast_bf16 blog ("FP8 (8 bits) & FP16 (16 bits)"):
 *          weight_dequant and weight_dequant_kernel (one fp32 scale per
 *          B x B block, y = fp32(x) * s stored as the default dtype, bf16).
 *
 * Parity status: every function below is pinned by the CPU tests in tests/
 * (exhaustive code tables, library cross-checks, hand-worked tensors,
 * closed-form constants, invariants and a second naive formulation), with
 * one exception: the NaN/Inf propagation rules (NaN amax, Inf inputs) follow
 * a chosen reading of torch semantics that the pages never state; those
 * cases are "parity unpinned" beyond hand-worked IEEE consequences.
 */
#ifndef FP8Q_ORACLE_H
#define FP8Q_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* fp8 formats: 0 = float8_e4m3fn (bias 7, 3 mantissa bits, no Inf, max 448),
 *              1 = float8_e5m2   (bias 15, 2 mantissa bits, IEEE-like, max 57344) */
enum { ORC_E4M3FN = 0, ORC_E5M2 = 1 };
/* element types of high-precision tensors */
enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2 };
/* scale rules (see fp8q_oracle.c): one IEEE division, or torch's evaluation
 * order for the pages' expressions on a CUDA tensor */
enum { ORC_RULE_IEEE = 0, ORC_RULE_TORCH = 1 };
/* scale granularity for the dequantising cast */
enum { ORC_GRAN_TENSOR = 0, ORC_GRAN_ROW = 1, ORC_GRAN_GROUP = 2, ORC_GRAN_BLOCK = 3 };

/* ---- scalar codecs ---------------------------------------------------- */
float    orc_fp8_max(int fmt);                 /* torch.finfo(fp8).max */
float    orc_fp8_decode(uint8_t code, int fmt);/* exact */
uint8_t  orc_fp8_encode(float v, int fmt);     /* RNE, non-saturating */
uint16_t orc_bf16_encode(float v);             /* RNE */
float    orc_bf16_decode(uint16_t h);          /* exact */
uint16_t orc_f16_encode(float v);              /* RNE, overflow -> Inf */
float    orc_f16_decode(uint16_t h);           /* exact */

/* ---- bulk codecs (loops over the scalar codecs; used by the pins) ------ */
void orc_fp8_encode_n(const float* v, int64_t n, int fmt, uint8_t* out);
void orc_fp8_decode_n(const uint8_t* c, int64_t n, int fmt, float* out);
void orc_bf16_encode_n(const float* v, int64_t n, uint16_t* out);
void orc_f16_encode_n(const float* v, int64_t n, uint16_t* out);

/*
 * ---- the method --------------------------------------------------------
 * All tensors are contiguous row-major host arrays.  Row-structured
 * operations compute only rows [r0, r1) (so callers may sample rows or split
 * work across threads); every other output byte is left untouched.
 * Return 0 on success, -1 on an argument the method rejects.
 */

/* [DEP] per_token_cast_to_fp8: x[m][n] (bf16/f32/f16), n % group == 0.
 * q[m][n] fp8 codes; scale_inv[m][n/group] fp32. */
int orc_per_token_group_quant(const void* x, int xt, int64_t m, int64_t n,
                              int group, int fmt, uint8_t* q, float* scale_inv,
                              int64_t r0, int64_t r1);

int orc_per_token_group_quant_rule(const void* x, int xt, int64_t m, int64_t n,
                                   int group, int fmt, uint8_t* q, float* scale_inv,
                                   int64_t r0, int64_t r1, int rule);

/* [CAI] cast_to_fp8, per-channel branch: one scale per row of x[rows][cols].
 * scale_inv[rows]. */
int orc_cast_per_channel(const void* x, int xt, int64_t rows, int64_t cols,
                         int fmt, uint8_t* q, float* scale_inv,
                         int64_t r0, int64_t r1);

int orc_cast_per_channel_rule(const void* x, int xt, int64_t rows, int64_t cols,
                              int fmt, uint8_t* q, float* scale_inv,
                              int64_t r0, int64_t r1, int rule);

/* [CAI] cast_to_fp8, per-tensor branch over numel elements.  The amax is
 * always taken over all numel elements; only q[e0..e1) is written.
 * scale_inv[0]. */
int orc_cast_per_tensor(const void* x, int xt, int64_t numel, int fmt,
                        uint8_t* q, float* scale_inv, int64_t e0, int64_t e1);

int orc_cast_per_tensor_rule(const void* x, int xt, int64_t numel, int fmt,
                             uint8_t* q, float* scale_inv, int64_t e0, int64_t e1, int rule);

/* [CAI] cast_to_fp8_pipeline: per-tensor cast with the format chosen by the
 * amax (e5m2 above 448, else e4m3fn); scale 1 for an all-zero tensor;
 * scale_inv[0] = 1 / scale; *fmt_out = the chosen format. */
int orc_cast_pipeline(const void* x, int xt, int64_t numel, uint8_t* q, float* scale_inv,
                      int* fmt_out, int rule, int64_t e0, int64_t e1);

/* [CAI] cast_from_fp8_pipeline: y = T(float(q) * scale_inv[0]) in format fmt. */
int orc_cast_from_pipeline(const uint8_t* q, int fmt, int64_t numel, const float* scale_inv,
                           int yt, void* y, int64_t e0, int64_t e1);

/* [DSV3] weight_dequant: w[M][N] codes, s[ceil(M/B)][ceil(N/B)] fp32,
 * y[M][N] in yt. */
int orc_block_dequant(const uint8_t* w, int fmt, int64_t M, int64_t N,
                      const float* s, int block, int yt, void* y,
                      int64_t r0, int64_t r1);

/* [CAI] cast_from_fp8 (and [DEP] per_token_cast_back): q[rows][cols] codes,
 * scale_inv per granule, y[rows][cols] in yt.  gb = group (GROUP) or block
 * edge (BLOCK); ignored otherwise. */
int orc_cast_from_fp8(const uint8_t* q, int fmt, int64_t rows, int64_t cols,
                      const float* scale_inv, int gran, int gb, int yt,
                      void* y, int64_t r0, int64_t r1);

/* [CAI] linear_fp8 forward, torch._scaled_mm with per-tensor scales:
 * out[m][n] = (sum_k dec(a[m][k]) * dec(b[n][k])) * sa * sb + bias[n], in
 * binary64 (exact sums for e4m3fn operands); a [M][K], b [N][K]; bias NULL
 * or [N]; rows [r0, r1) of out[M][N]. */
int orc_scaled_mm(const uint8_t* a, int fa, const uint8_t* b, int fb, int64_t M, int64_t N, int64_t K,
                  float sa, float sb, const double* bias, double* out, int64_t r0, int64_t r1);

/* [DEP] x [DSV3] the same product with per-token-group activation scales
 * sa[M][ceil(K/ga)] and per-block weight scales sb[ceil(N/bb)][ceil(K/bb)]:
 * out[m][n] = sum_k (dec(a[m][k]) * sa[m][k/ga]) * (dec(b[n][k]) * sb[n/bb][k/bb])
 *             + bias[n], in binary64; rows [r0, r1) of out[M][N]. */
int orc_scaled_mm_blockwise(const uint8_t* a, int fa, const float* sa, int64_t ga,
                            const uint8_t* b, int fb, const float* sb, int64_t bb,
                            int64_t M, int64_t N, int64_t K, const double* bias,
                            double* out, int64_t r0, int64_t r1);

/* The same two products with the library's single-precision rounding:
 * per-tensor d = T(fl(fl(acc * fl(sa * sb)) + bias[n])); fine-grained
 * acc = fma(acc_kb, fl(sa[m][kb] * sb[n/bb][kb]), acc) over kb ascending,
 * d = T(fl(acc + bias[n])); acc and acc_kb the exact sums rounded once to
 * binary32.  bias NULL or fp32 [N]; out [M][N] of type yt. */
int orc_scaled_mm_rounded(const uint8_t* a, int fa, const uint8_t* b, int fb, int64_t M, int64_t N, int64_t K,
                          float sa, float sb, const float* bias, int yt, void* out, int64_t r0, int64_t r1);
int orc_scaled_mm_blockwise_rounded(const uint8_t* a, int fa, const float* sa, const uint8_t* b, int fb,
                                    const float* sb, int64_t bb, int64_t M, int64_t N, int64_t K,
                                    const float* bias, int yt, void* out, int64_t r0, int64_t r1);

/* [CAI] _LinearFp8.backward: the operand transpose dst[c][r] = src[r][c]
 * (zero for rows <= r < ld) and the bias gradient out[c] = sum_r x[r][c]
 * in binary64, ascending r. */
int orc_transpose_u8(const uint8_t* src, int64_t rows, int64_t cols, uint8_t* dst, int64_t ld);
int orc_sum_rows(const void* x, int xt, int64_t rows, int64_t cols, double* out);

#ifdef __cplusplus
}
#endif
#endif
