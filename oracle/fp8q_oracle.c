/*
 * fp8q_oracle.c -- plain CPU definition of scaled FP8 casting.
 *
 * TEST INFRASTRUCTURE ONLY (see fp8q_oracle.h): tests, the smoke check and
 * the benchmark's CPU-baseline leg are the only callers.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared
 * Each `float` expression below is one binary32 operation, rounded to
 * nearest-even; nothing is fused, reordered or blocked.
 */
#include "fp8q_oracle.h"

#include <math.h>
#include <string.h>

/* ------------------------------------------------------------------------
 * Bit access
 * ---------------------------------------------------------------------- */
static uint32_t f2u(float v) { uint32_t u; memcpy(&u, &v, 4); return u; }
static float    u2f(uint32_t u) { float v; memcpy(&v, &u, 4); return v; }

/* ------------------------------------------------------------------------
 * Rounding a finite fp32 magnitude onto a narrower binary format.
 *
 * The target format has `mbits` stored mantissa bits and exponent bias
 * `bias`; its smallest normal exponent is 1 - bias and below it the spacing
 * of representable values stays 2^(1 - bias - mbits) (gradual underflow).
 *
 * For |v| = sig * 2^(e - 23) (sig includes the hidden bit for normal fp32),
 * the representable neighbours are multiples of the quantum 2^qexp with
 * qexp = max(e, 1 - bias) - mbits.  n = RNE(|v| / 2^qexp) is found by a
 * right shift of sig with an exact remainder test; ties go to the even n.
 * The magnitude code is then ((max(e, 1-bias) + bias) << mbits) + n - 2^mbits,
 * which also covers the subnormal range (exponent field 0, mantissa n) and
 * the carry into the next binade when n reaches 2^(mbits+1).  The caller
 * decides what an out-of-range code means (NaN, Inf).
 * ---------------------------------------------------------------------- */
static uint32_t round_magnitude(uint32_t a, int mbits, int bias)
{
    int      efield = (int)(a >> 23);
    uint32_t sig    = a & 0x7FFFFFu;
    int      e;
    if (efield == 0) {
        e = -126;                 /* fp32 subnormal: no hidden bit */
    } else {
        e = efield - 127;
        sig |= 0x800000u;
    }
    int emin = 1 - bias;
    int ee   = e < emin ? emin : e;
    int qexp = ee - mbits;
    int k    = 23 + qexp - e;     /* bits of sig below the quantum, >= 23 - mbits */
    uint32_t n;
    if (k > 24) {
        n = 0;                    /* |v| < quantum / 2 */
    } else {
        uint32_t kept = sig >> k;
        uint32_t rem  = sig & ((1u << k) - 1u);
        uint32_t half = 1u << (k - 1);
        n = kept;
        if (rem > half || (rem == half && (kept & 1u)))
            n += 1u;
    }
    return ((uint32_t)(ee + bias) << mbits) + n - (1u << mbits);
}

/* ------------------------------------------------------------------------
 * fp8 codecs.  Format facts are torch.finfo's, which the ColossalAI page
 * reads through torch.finfo(fp8_type).max and the DeepEP page hard-codes
 * as 448 for float8_e4m3fn:
 *   e4m3fn: S EEEE MMM, bias 7; exponent field 0 is subnormal (m * 2^-9);
 *           S 1111 111 is NaN; there is no Inf; max 0x7E = 448.
 *   e5m2:   S EEEEE MM, bias 15; exponent field 31 is Inf (m == 0) or NaN;
 *           max 0x7B = 57344.
 * Encoding is round-to-nearest-even and does not saturate: a value whose
 * rounded magnitude exceeds the maximum becomes NaN (e4m3fn) or Inf (e5m2),
 * as torch's .to(float8_*) does -- the cast every page calls.  A NaN input
 * encodes to the NaN code with its sign bit kept.
 * ---------------------------------------------------------------------- */
float orc_fp8_max(int fmt)
{
    return fmt == ORC_E4M3FN ? 448.0f : 57344.0f;
}

uint8_t orc_fp8_encode(float v, int fmt)
{
    uint32_t b    = f2u(v);
    uint8_t  sign = (uint8_t)((b >> 24) & 0x80u);
    uint32_t a    = b & 0x7FFFFFFFu;
    if (a > 0x7F800000u)                       /* NaN */
        return (uint8_t)(0x7Fu | sign);
    if (fmt == ORC_E4M3FN) {
        if (a == 0x7F800000u)                  /* Inf has no e4m3fn code */
            return (uint8_t)(0x7Fu | sign);
        uint32_t c = round_magnitude(a, 3, 7);
        return (uint8_t)((c > 0x7Eu ? 0x7Fu : c) | sign);
    } else {
        if (a == 0x7F800000u)
            return (uint8_t)(0x7Cu | sign);
        uint32_t c = round_magnitude(a, 2, 15);
        return (uint8_t)((c > 0x7Bu ? 0x7Cu : c) | sign);
    }
}

float orc_fp8_decode(uint8_t code, int fmt)
{
    int   neg   = code >> 7;
    int   mag   = code & 0x7F;
    int   mbits = fmt == ORC_E4M3FN ? 3 : 2;
    int   bias  = fmt == ORC_E4M3FN ? 7 : 15;
    int   e     = mag >> mbits;
    int   m     = mag & ((1 << mbits) - 1);
    float v;
    if (fmt == ORC_E4M3FN && mag == 0x7F)
        return u2f(0x7FC00000u | ((uint32_t)neg << 31));
    if (fmt == ORC_E5M2 && e == 31) {
        if (m != 0)
            return u2f(0x7FC00000u | ((uint32_t)neg << 31));
        v = INFINITY;
    } else if (e == 0) {
        v = ldexpf((float)m, 1 - bias - mbits);
    } else {
        v = ldexpf((float)((1 << mbits) + m), e - bias - mbits);
    }
    return neg ? -v : v;
}

/* ------------------------------------------------------------------------
 * 16-bit codecs (bf16: bias 127, 7 mantissa bits; fp16: bias 15, 10 bits).
 * RNE from fp32; overflow becomes Inf; NaN stays a quiet NaN with its sign.
 * ---------------------------------------------------------------------- */
uint16_t orc_bf16_encode(float v)
{
    uint32_t b    = f2u(v);
    uint16_t sign = (uint16_t)((b >> 16) & 0x8000u);
    uint32_t a    = b & 0x7FFFFFFFu;
    if (a > 0x7F800000u)
        return (uint16_t)((b >> 16) | 0x0040u);
    if (a == 0x7F800000u)
        return (uint16_t)(0x7F80u | sign);
    uint32_t c = round_magnitude(a, 7, 127);
    return (uint16_t)((c > 0x7F7Fu ? 0x7F80u : c) | sign);
}

float orc_bf16_decode(uint16_t h)
{
    return u2f((uint32_t)h << 16);
}

uint16_t orc_f16_encode(float v)
{
    uint32_t b    = f2u(v);
    uint16_t sign = (uint16_t)((b >> 16) & 0x8000u);
    uint32_t a    = b & 0x7FFFFFFFu;
    if (a > 0x7F800000u)
        return (uint16_t)(0x7E00u | sign);
    if (a == 0x7F800000u)
        return (uint16_t)(0x7C00u | sign);
    uint32_t c = round_magnitude(a, 10, 15);
    return (uint16_t)((c > 0x7BFFu ? 0x7C00u : c) | sign);
}

float orc_f16_decode(uint16_t h)
{
    int   neg = h >> 15;
    int   e   = (h >> 10) & 31;
    int   m   = h & 0x3FF;
    float v;
    if (e == 31) {
        if (m != 0)
            return u2f(0x7FC00000u | ((uint32_t)neg << 31));
        v = INFINITY;
    } else if (e == 0) {
        v = ldexpf((float)m, -24);
    } else {
        v = ldexpf((float)(1024 + m), e - 25);
    }
    return neg ? -v : v;
}

void orc_fp8_encode_n(const float* v, int64_t n, int fmt, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_fp8_encode(v[i], fmt);
}
void orc_fp8_decode_n(const uint8_t* c, int64_t n, int fmt, float* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_fp8_decode(c[i], fmt);
}
void orc_bf16_encode_n(const float* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_encode(v[i]);
}
void orc_f16_encode_n(const float* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f16_encode(v[i]);
}

/* ------------------------------------------------------------------------
 * Element load / store in the high-precision types.  Widening to fp32 is
 * exact (the pages' `.float()`); narrowing is the RNE of the target type
 * (the pages' `.to(ret_type)` and the implicit conversion of a Triton store).
 * ---------------------------------------------------------------------- */
static float load_elem(const void* x, int xt, int64_t i)
{
    switch (xt) {
    case ORC_F32:  return ((const float*)x)[i];
    case ORC_F16:  return orc_f16_decode(((const uint16_t*)x)[i]);
    default:       return orc_bf16_decode(((const uint16_t*)x)[i]);
    }
}

static void store_elem(void* y, int yt, int64_t i, float v)
{
    switch (yt) {
    case ORC_F32:  ((float*)y)[i] = v; break;
    case ORC_F16:  ((uint16_t*)y)[i] = orc_f16_encode(v); break;
    default:       ((uint16_t*)y)[i] = orc_bf16_encode(v); break;
    }
}

static int valid_fmt(int fmt) { return fmt == ORC_E4M3FN || fmt == ORC_E5M2; }
static int valid_dtype(int t) { return t == ORC_F32 || t == ORC_F16 || t == ORC_BF16; }
static int valid_dt(int t)    { return t == ORC_F32 || t == ORC_F16 || t == ORC_BF16; }

/* max |x| over x[i0 .. i0+count), NaN-propagating like torch's max/amax:
 * once a NaN is seen the result stays NaN. */
static float abs_max(const void* x, int xt, int64_t i0, int64_t count)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < count; ++k) {
        float a = fabsf(load_elem(x, xt, i0 + k));
        if (isnan(a) || a > amax)
            amax = a;
    }
    return amax;
}

/* ------------------------------------------------------------------------
 * Scale rules: how FMAX / amax and amax / FMAX are rounded.
 *   ORC_RULE_IEEE  one IEEE binary32 division each (the reading used by
 *                  every operation unless a rule is given).
 *   ORC_RULE_TORCH the order in which torch evaluates the pages' own
 *                  expressions on a CUDA tensor: a Python number divided by
 *                  a tensor is the tensor's reciprocal times the number,
 *                  fl(fl(1 / amax) * FMAX); a tensor divided by a Python
 *                  number on the GPU is a multiply by the number's
 *                  reciprocal, fl(amax * fl(1 / FMAX)).
 * ---------------------------------------------------------------------- */
static float scale_of(float amax, float fmax, int rule)
{
    if (rule == ORC_RULE_TORCH) {
        float r = 1.0f / amax;
        return r * fmax;
    }
    return fmax / amax;
}

static float scale_inv_of(float amax, float fmax, int rule)
{
    if (rule == ORC_RULE_TORCH) {
        float inv = 1.0f / fmax;
        return amax * inv;
    }
    return amax / fmax;
}

static int valid_rule(int rule) { return rule == ORC_RULE_IEEE || rule == ORC_RULE_TORCH; }

/* ------------------------------------------------------------------------
 * [DEP] per_token_cast_to_fp8.
 *   view x[m][n] as x[m][n/G][G];
 *   amax[r][g]      = clamp(max_k |float(x[r][g][k])|, min = 1e-4)
 *   q[r][g][k]      = fp8( float(x[r][g][k]) * (FMAX / amax[r][g]) )
 *   scale_inv[r][g] = amax[r][g] / FMAX
 * The clamp bound is the fp32 value nearest 1e-4 (the clamp acts on an fp32
 * tensor); clamp keeps a NaN amax.  FMAX is 448 for e4m3fn (the page's
 * constant) and torch.finfo(...).max for e5m2.  Both quotients are IEEE fp32
 * divisions.
 * ---------------------------------------------------------------------- */
int orc_per_token_group_quant(const void* x, int xt, int64_t m, int64_t n,
                              int group, int fmt, uint8_t* q, float* scale_inv,
                              int64_t r0, int64_t r1)
{
    return orc_per_token_group_quant_rule(x, xt, m, n, group, fmt, q, scale_inv, r0, r1,
                                          ORC_RULE_IEEE);
}

int orc_per_token_group_quant_rule(const void* x, int xt, int64_t m, int64_t n,
                                   int group, int fmt, uint8_t* q, float* scale_inv,
                                   int64_t r0, int64_t r1, int rule)
{
    if (!valid_rule(rule) || !valid_fmt(fmt) || !valid_dt(xt) || group <= 0 || m < 0 || n < 0 ||
        n % group != 0 || r0 < 0 || r1 > m || r0 > r1)
        return -1;
    const float fmax     = orc_fp8_max(fmt);
    const float clampmin = 1e-4f;
    const int64_t G      = n / group;
    for (int64_t r = r0; r < r1; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            int64_t base = r * n + g * group;
            float amax = abs_max(x, xt, base, group);
            if (amax < clampmin)
                amax = clampmin;
            float scale = scale_of(amax, fmax, rule);
            scale_inv[r * G + g] = scale_inv_of(amax, fmax, rule);
            for (int64_t k = 0; k < group; ++k) {
                float v = load_elem(x, xt, base + k) * scale;
                q[base + k] = orc_fp8_encode(v, fmt);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * [CAI] cast_to_fp8, per-channel branch.
 *   amax[r]      = max_c |x[r][c]|;  amax[r] := amax[r] > 0 ? amax[r] : 1
 *   scale[r]     = FMAX / amax[r];   scale_inv[r] = amax[r] / FMAX
 *   q[r][c]      = fp8( float(x[r][c]) * scale[r] )
 * A NaN amax fails `> 0` and is replaced by 1 (torch.where).  Row r of the
 * dequant uses scale_inv[r].  An empty tensor returns scale_inv = 1.0.
 * ---------------------------------------------------------------------- */
int orc_cast_per_channel(const void* x, int xt, int64_t rows, int64_t cols,
                         int fmt, uint8_t* q, float* scale_inv,
                         int64_t r0, int64_t r1)
{
    return orc_cast_per_channel_rule(x, xt, rows, cols, fmt, q, scale_inv, r0, r1, ORC_RULE_IEEE);
}

int orc_cast_per_channel_rule(const void* x, int xt, int64_t rows, int64_t cols,
                              int fmt, uint8_t* q, float* scale_inv,
                              int64_t r0, int64_t r1, int rule)
{
    if (!valid_rule(rule) || !valid_fmt(fmt) || !valid_dt(xt) || rows < 0 || cols < 0 ||
        r0 < 0 || r1 > rows || r0 > r1)
        return -1;
    const float fmax = orc_fp8_max(fmt);
    if (rows == 0 || cols == 0) {
        /* empty tensor: the page returns scale_inv = [1.0] */
        int64_t ns = rows > 0 ? rows : 1;
        for (int64_t r = 0; r < ns; ++r) scale_inv[r] = 1.0f;
        return 0;
    }
    for (int64_t r = r0; r < r1; ++r) {
        float amax = abs_max(x, xt, r * cols, cols);
        amax = amax > 0.0f ? amax : 1.0f;
        float scale = scale_of(amax, fmax, rule);
        scale_inv[r] = scale_inv_of(amax, fmax, rule);
        for (int64_t c = 0; c < cols; ++c) {
            float v = load_elem(x, xt, r * cols + c) * scale;
            q[r * cols + c] = orc_fp8_encode(v, fmt);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * [CAI] cast_to_fp8, per-tensor branch.
 *   amax      = max |x|;  amax := amax > 0 ? amax : 1
 *   scale     = FMAX / amax;  scale_inv = 1 / scale   (as the page writes it)
 *   q         = fp8( float(x) * scale )
 * An empty tensor returns scale_inv = 1.0.
 * ---------------------------------------------------------------------- */
int orc_cast_per_tensor(const void* x, int xt, int64_t numel, int fmt,
                        uint8_t* q, float* scale_inv, int64_t e0, int64_t e1)
{
    return orc_cast_per_tensor_rule(x, xt, numel, fmt, q, scale_inv, e0, e1, ORC_RULE_IEEE);
}

int orc_cast_per_tensor_rule(const void* x, int xt, int64_t numel, int fmt,
                             uint8_t* q, float* scale_inv, int64_t e0, int64_t e1, int rule)
{
    if (!valid_rule(rule) || !valid_fmt(fmt) || !valid_dt(xt) || numel < 0 || e0 < 0 ||
        e1 > numel || e0 > e1)
        return -1;
    if (numel == 0) {
        scale_inv[0] = 1.0f;
        return 0;
    }
    const float fmax = orc_fp8_max(fmt);
    float amax = abs_max(x, xt, 0, numel);
    amax = amax > 0.0f ? amax : 1.0f;
    float scale = scale_of(amax, fmax, rule);
    scale_inv[0] = 1.0f / scale;   /* `1.0 / scale` is one rounding under both rules */
    for (int64_t i = e0; i < e1; ++i) {
        float v = load_elem(x, xt, i) * scale;
        q[i] = orc_fp8_encode(v, fmt);
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * [CAI] cast_to_fp8_pipeline: per-tensor cast whose fp8 format is chosen by
 * the amax, for activations sent between pipeline stages.
 *   amax  = max |x|  (the page takes max(|min|, |max|) from aminmax; NaN
 *           propagates)
 *   fmt   = amax > 448 (the e4m3fn maximum) ? e5m2 : e4m3fn
 *           (a NaN amax fails the test and gives e4m3fn)
 *   scale = amax == 0 ? 1 : FMAX(fmt) / amax       (scale rule as above)
 *   q     = fp8_fmt(fl(float(x) * scale)); scale_inv[0] = fl(1 / scale)
 *           (the page keeps scale.reciprocal()); *fmt_out = fmt
 * Only q[e0..e1) is written; amax is always over all numel elements.
 * ---------------------------------------------------------------------- */
int orc_cast_pipeline(const void* x, int xt, int64_t numel, uint8_t* q, float* scale_inv,
                      int* fmt_out, int rule, int64_t e0, int64_t e1)
{
    if (!valid_rule(rule) || !valid_dt(xt) || numel < 0 || e0 < 0 || e1 > numel || e0 > e1)
        return -1;
    float amax = abs_max(x, xt, 0, numel);
    int fmt = amax > orc_fp8_max(ORC_E4M3FN) ? ORC_E5M2 : ORC_E4M3FN;
    float scale = amax == 0.0f ? 1.0f : scale_of(amax, orc_fp8_max(fmt), rule);
    scale_inv[0] = 1.0f / scale;
    *fmt_out = fmt;
    for (int64_t i = e0; i < e1; ++i) {
        float v = load_elem(x, xt, i) * scale;
        q[i] = orc_fp8_encode(v, fmt);
    }
    return 0;
}

/* [CAI] cast_from_fp8_pipeline: y = T(fl(float(q) * scale_inv[0])), the
 * codes read in the format the tag names. */
int orc_cast_from_pipeline(const uint8_t* q, int fmt, int64_t numel, const float* scale_inv,
                           int yt, void* y, int64_t e0, int64_t e1)
{
    if (!valid_fmt(fmt) || !valid_dt(yt) || numel < 0 || e0 < 0 || e1 > numel || e0 > e1)
        return -1;
    for (int64_t i = e0; i < e1; ++i) {
        float v = orc_fp8_decode(q[i], fmt) * scale_inv[0];
        store_elem(y, yt, i, v);
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * [DSV3] weight_dequant / weight_dequant_kernel.
 *   y[i][j] = T( float(w[i][j]) * s[i / B][j / B] )
 * s is row-major [ceil(M/B)][ceil(N/B)] (the kernel's pid_m * cdiv(N, B) +
 * pid_n index); a partial edge block uses its own scale.  The product is an
 * fp32 multiply; the store into the bf16 output rounds to nearest-even.
 * ---------------------------------------------------------------------- */
int orc_block_dequant(const uint8_t* w, int fmt, int64_t M, int64_t N,
                      const float* s, int block, int yt, void* y,
                      int64_t r0, int64_t r1)
{
    if (!valid_fmt(fmt) || !valid_dt(yt) || block <= 0 || M < 0 || N < 0 ||
        r0 < 0 || r1 > M || r0 > r1)
        return -1;
    const int64_t nb = (N + block - 1) / block;
    for (int64_t i = r0; i < r1; ++i) {
        for (int64_t j = 0; j < N; ++j) {
            float sc = s[(i / block) * nb + j / block];
            float v  = orc_fp8_decode(w[i * N + j], fmt) * sc;
            store_elem(y, yt, i * N + j, v);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * [CAI] cast_from_fp8: y = T( scale_inv[granule] * float(q) ).
 *   TENSOR: scale_inv[0]
 *   ROW:    scale_inv[r]                       (per-channel: row r of x)
 *   GROUP:  scale_inv[r * (cols/G) + c / G]    ([DEP] per-token groups)
 *   BLOCK:  scale_inv[(r/B) * ceil(cols/B) + c / B]
 * ---------------------------------------------------------------------- */
int orc_cast_from_fp8(const uint8_t* q, int fmt, int64_t rows, int64_t cols,
                      const float* scale_inv, int gran, int gb, int yt,
                      void* y, int64_t r0, int64_t r1)
{
    if (!valid_fmt(fmt) || !valid_dt(yt) || rows < 0 || cols < 0 ||
        r0 < 0 || r1 > rows || r0 > r1)
        return -1;
    if ((gran == ORC_GRAN_GROUP || gran == ORC_GRAN_BLOCK) && gb <= 0)
        return -1;
    if (gran == ORC_GRAN_GROUP && cols % gb != 0)
        return -1;
    if (gran < ORC_GRAN_TENSOR || gran > ORC_GRAN_BLOCK)
        return -1;
    for (int64_t r = r0; r < r1; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            float sc;
            switch (gran) {
            case ORC_GRAN_TENSOR: sc = scale_inv[0]; break;
            case ORC_GRAN_ROW:    sc = scale_inv[r]; break;
            case ORC_GRAN_GROUP:  sc = scale_inv[r * (cols / gb) + c / gb]; break;
            default:              sc = scale_inv[(r / gb) * ((cols + gb - 1) / gb) + c / gb]; break;
            }
            float v = sc * orc_fp8_decode(q[r * cols + c], fmt);
            store_elem(y, yt, r * cols + c, v);
        }
    }
    return 0;
}

/*
 * [CAI] linear_fp8 forward (_LinearFp8.forward): both operands are cast to
 * fp8 with per-tensor scales and multiplied by torch._scaled_mm(x_fp8,
 * w_fp8.t(), scale_a = scale_inv of x, scale_b = scale_inv of w, bias):
 *     out[m][n] = (sum over k of dec(a[m][k]) * dec(b[n][k])) * sa * sb + bias[n]
 * a is [M][K] (the activations), b is [N][K] (the weight, as stored; the
 * product uses its transpose).  Evaluated in binary64: every product of two
 * fp8 values is exact, and for e4m3fn operands every partial sum is exact
 * too (products span 2^-18 .. 2^17.6 with 8 significant bits, and K < 2^20
 * keeps the sums inside 53 bits), so for e4m3fn the sum is the exact one.
 * bias may be NULL.  Only rows [r0, r1) of out are written.
 */
int orc_scaled_mm(const uint8_t* a, int fa, const uint8_t* b, int fb, int64_t M, int64_t N, int64_t K,
                  float sa, float sb, const double* bias, double* out, int64_t r0, int64_t r1)
{
    if (!valid_fmt(fa) || !valid_fmt(fb) || M < 0 || N < 0 || K < 0 || r0 < 0 || r1 > M || r0 > r1)
        return -1;
    double da[256], db[256];
    for (int c = 0; c < 256; ++c) {
        da[c] = (double)orc_fp8_decode((uint8_t)c, fa);
        db[c] = (double)orc_fp8_decode((uint8_t)c, fb);
    }
    for (int64_t m = r0; m < r1; ++m) {
        const uint8_t* ar = a + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* br = b + n * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += da[ar[k]] * db[br[k]];
            double v = acc * (double)sa * (double)sb;
            if (bias) v += bias[n];
            out[m * N + n] = v;
        }
    }
    return 0;
}

/*
 * The same product with fine-grained scales: the activations quantised by
 * [DEP] per_token_cast_to_fp8 (one scale_inv per 1 x ga group of a row,
 * sa[M][ceil(K/ga)]) times a weight stored as [DSV3] weight_dequant expects
 * it (one scale_inv per bb x bb block, sb[ceil(N/bb)][ceil(K/bb)]):
 *     out[m][n] = sum over k of (dec(a[m][k]) * sa[m][k/ga])
 *                             * (dec(b[n][k]) * sb[n/bb][k/bb])  + bias[n]
 * i.e. the product of the two dequantised operands, each element taken at
 * its exact value (no rounding to bf16 in between).  Evaluated in binary64,
 * k ascending: each dequantised element is exact in binary64 (4 + 24
 * significant bits), so only the products and the running sum round, each
 * at 2^-53 relative.  bias may be NULL.  Only rows [r0, r1) are written.
 */
int orc_scaled_mm_blockwise(const uint8_t* a, int fa, const float* sa, int64_t ga,
                            const uint8_t* b, int fb, const float* sb, int64_t bb,
                            int64_t M, int64_t N, int64_t K, const double* bias,
                            double* out, int64_t r0, int64_t r1)
{
    if (!valid_fmt(fa) || !valid_fmt(fb) || M < 0 || N < 0 || K < 0 || ga < 1 || bb < 1 ||
        r0 < 0 || r1 > M || r0 > r1)
        return -1;
    double da[256], db[256];
    for (int c = 0; c < 256; ++c) {
        da[c] = (double)orc_fp8_decode((uint8_t)c, fa);
        db[c] = (double)orc_fp8_decode((uint8_t)c, fb);
    }
    int64_t ka = (K + ga - 1) / ga;          /* groups per activation row */
    int64_t kb = (K + bb - 1) / bb;          /* blocks per weight block-row */
    for (int64_t m = r0; m < r1; ++m) {
        const uint8_t* ar = a + m * K;
        const float* sar = sa + m * ka;
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* br = b + n * K;
            const float* sbr = sb + (n / bb) * kb;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double x = da[ar[k]] * (double)sar[k / ga];
                double w = db[br[k]] * (double)sbr[k / bb];
                acc += x * w;
            }
            if (bias) acc += bias[n];
            out[m * N + n] = acc;
        }
    }
    return 0;
}

/*
 * The two products as the library rounds them.  The pages leave the
 * rounding inside torch._scaled_mm to the GEMM library; the reading taken
 * here is the plainest single-precision one:
 *   per-tensor:    d = T(fl(fl(acc * fl(sa * sb)) + bias[n]))
 *   fine-grained:  acc = 0; for kb ascending: acc = fma(acc_kb, fl(sa[m][kb] * sb[n/bb][kb]), acc)
 *                  d = T(fl(acc + bias[n]))
 * where acc (per-tensor) and acc_kb (one 128-deep block) are the binary64
 * sums above rounded once to binary32 -- the correctly rounded fp32 sum.
 * Whenever every partial sum of the products is an fp32 number (for
 * example all operand values multiples of 1/8 of magnitude <= 4, K <= 16384:
 * products are multiples of 2^-6 below 2^4, sums below 2^18), any fp32
 * accumulation order gives that same acc, so d is fixed bit for bit.
 * Other inputs differ from the tensor cores' sum only by its own rounding.
 * fmaf is the C library's correctly rounded fused multiply-add; bias is
 * NULL or binary32 values (bf16 / fp16 biases widen exactly); out is yt.
 */
static double dot_exact(const uint8_t* ar, const uint8_t* br, const double* da, const double* db,
                        int64_t k0, int64_t k1)
{
    double acc = 0.0;
    for (int64_t k = k0; k < k1; ++k) acc += da[ar[k]] * db[br[k]];
    return acc;
}

int orc_scaled_mm_rounded(const uint8_t* a, int fa, const uint8_t* b, int fb, int64_t M, int64_t N, int64_t K,
                          float sa, float sb, const float* bias, int yt, void* out, int64_t r0, int64_t r1)
{
    if (!valid_fmt(fa) || !valid_fmt(fb) || M < 0 || N < 0 || K < 0 || r0 < 0 || r1 > M || r0 > r1)
        return -1;
    double da[256], db[256];
    for (int c = 0; c < 256; ++c) {
        da[c] = (double)orc_fp8_decode((uint8_t)c, fa);
        db[c] = (double)orc_fp8_decode((uint8_t)c, fb);
    }
    const float s = sa * sb;
    for (int64_t m = r0; m < r1; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float acc = (float)dot_exact(a + m * K, b + n * K, da, db, 0, K);
            float v = acc * s;
            if (bias) v = v + bias[n];
            store_elem(out, yt, m * N + n, v);
        }
    return 0;
}

int orc_scaled_mm_blockwise_rounded(const uint8_t* a, int fa, const float* sa, const uint8_t* b, int fb,
                                    const float* sb, int64_t bb, int64_t M, int64_t N, int64_t K,
                                    const float* bias, int yt, void* out, int64_t r0, int64_t r1)
{
    if (!valid_fmt(fa) || !valid_fmt(fb) || M < 0 || N < 0 || K < 0 || bb < 1 || r0 < 0 || r1 > M || r0 > r1)
        return -1;
    double da[256], db[256];
    for (int c = 0; c < 256; ++c) {
        da[c] = (double)orc_fp8_decode((uint8_t)c, fa);
        db[c] = (double)orc_fp8_decode((uint8_t)c, fb);
    }
    const int64_t kb = (K + bb - 1) / bb;
    for (int64_t m = r0; m < r1; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float acc = 0.0f;
            for (int64_t j = 0; j < kb; ++j) {
                const int64_t k1 = (j + 1) * bb < K ? (j + 1) * bb : K;
                const float part = (float)dot_exact(a + m * K, b + n * K, da, db, j * bb, k1);
                const float s = sa[m * kb + j] * sb[(n / bb) * kb + j];
                acc = fmaf(part, s, acc);
            }
            if (bias) acc = acc + bias[n];
            store_elem(out, yt, m * N + n, acc);
        }
    return 0;
}

/*
 * [CAI] _LinearFp8.backward's data movements.
 * orc_transpose_u8: the .t().contiguous() copy of an fp8 operand, dst[c][r] =
 * src[r][c] for r < rows, zero for rows <= r < ld (the zero-padded pitch).
 * orc_sum_rows: bias_grad = out_grad.sum(0), out[c] = sum over r of x[r][c],
 * added in binary64 in ascending r (every bf16 / fp16 / fp32 value is exact
 * in binary64, so for up to 2^24 rows of values within a few binades the sum
 * is exact or within 2^-53 relative).
 */
int orc_transpose_u8(const uint8_t* src, int64_t rows, int64_t cols, uint8_t* dst, int64_t ld)
{
    if (rows < 0 || cols < 0 || ld < rows) return -1;
    for (int64_t c = 0; c < cols; ++c) {
        for (int64_t r = 0; r < rows; ++r) dst[c * ld + r] = src[r * cols + c];
        for (int64_t r = rows; r < ld; ++r) dst[c * ld + r] = 0;
    }
    return 0;
}

int orc_sum_rows(const void* x, int xt, int64_t rows, int64_t cols, double* out)
{
    if (!valid_dtype(xt) || rows < 0 || cols < 0) return -1;
    for (int64_t c = 0; c < cols; ++c) {
        double acc = 0.0;
        for (int64_t r = 0; r < rows; ++r) acc += (double)load_elem(x, xt, r * cols + c);
        out[c] = acc;
    }
    return 0;
}
