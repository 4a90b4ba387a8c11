/*
 * c_abi_check.c -- a plain C99 caller of libfp8q: include/fp8q.h compiles as
 * C, every entry point it declares links, and the host-side rules answer as
 * the header states.  Nothing here reaches the GPU: every call below returns
 * from argument validation before the library makes a CUDA call, so it runs
 * on a machine without one.  Built and run by tests/test_c_abi.py.
 */
#include <stdio.h>
#include <string.h>

#include "fp8q.h"

static int failures = 0;

#define EXPECT(cond)                                                    \
    do {                                                                \
        if (!(cond)) {                                                  \
            fprintf(stderr, "%s:%d: failed: %s\n", __FILE__, __LINE__, #cond); \
            ++failures;                                                 \
        }                                                               \
    } while (0)

typedef void (*any_fn)(void);

int main(void) {
    /* every declared entry point, resolved by the linker */
    const any_fn entry_points[] = {
        (any_fn)fp8q_block_dequant, (any_fn)fp8q_block_dequant_grouped, (any_fn)fp8q_cast_from_fp8,
        (any_fn)fp8q_cast_from_pipeline, (any_fn)fp8q_cast_per_channel, (any_fn)fp8q_cast_per_channel_ex,
        (any_fn)fp8q_cast_per_tensor, (any_fn)fp8q_cast_per_tensor_ex, (any_fn)fp8q_cast_per_tensor_noalloc,
        (any_fn)fp8q_cast_per_tensor_with_amax, (any_fn)fp8q_cast_per_tensor_workspace_bytes,
        (any_fn)fp8q_cast_pipeline, (any_fn)fp8q_pack_record, (any_fn)fp8q_pack_record_ex,
        (any_fn)fp8q_per_token_group_quant, (any_fn)fp8q_per_token_group_quant_ex, (any_fn)fp8q_record_bytes,
        (any_fn)fp8q_record_bytes_ex, (any_fn)fp8q_scaled_mm, (any_fn)fp8q_scaled_mm_blockwise,
        (any_fn)fp8q_scaled_mm_ex, (any_fn)fp8q_scaled_mm_wait_test, (any_fn)fp8q_scaled_mm_blockwise_wait_test,
        (any_fn)fp8q_status_string,
        (any_fn)fp8q_sum_rows, (any_fn)fp8q_tensor_amax, (any_fn)fp8q_transpose_fp8,
        (any_fn)fp8q_unpack_records, (any_fn)fp8q_unpack_records_ex, (any_fn)fp8q_version};
    const size_t n_entry = sizeof(entry_points) / sizeof(entry_points[0]);
    size_t i;
    for (i = 0; i < n_entry; ++i) EXPECT(entry_points[i] != NULL);

    /* constants and sizes */
    EXPECT(fp8q_version() == 10100);
    EXPECT(fp8q_cast_per_tensor_workspace_bytes() == 8192);
    EXPECT(fp8q_record_bytes(100) == 16 + 112);                              /* 16-byte header, payload to 16 */
    EXPECT(fp8q_record_bytes_ex(100, FP8Q_RECORD_ALIGNED16) == 16 + 112);
    EXPECT(fp8q_record_bytes_ex(100, FP8Q_RECORD_PACKED4) == 4 + 100);         /* the page's 4-byte header */
    EXPECT(fp8q_record_bytes_ex(100, (fp8q_record_layout)7) == 0);             /* unknown layout */
    {
        int code;
        for (code = 0; code <= 10; ++code) {
            const char* s = fp8q_status_string((fp8q_status)code);
            EXPECT(s != NULL && strncmp(s, "FP8Q_", 5) == 0);
        }
        EXPECT(strstr(fp8q_status_string((fp8q_status)99), "UNKNOWN") != NULL);
    }

    /* host validation (fake, never-dereferenced pointers) */
    {
        const void* P = (const void*)0x10000;
        uint8_t* Q = (uint8_t*)0x10000;
        float* S = (float*)0x10000;
        EXPECT(fp8q_per_token_group_quant(P, (fp8q_dtype)7, 4, 128, 128, FP8Q_E4M3FN, Q, S, NULL) ==
               FP8Q_ERR_BAD_DTYPE);
        EXPECT(fp8q_per_token_group_quant(P, FP8Q_BF16, 4, 128, 128, (fp8q_format)9, Q, S, NULL) ==
               FP8Q_ERR_BAD_FORMAT);
        EXPECT(fp8q_per_token_group_quant(P, FP8Q_BF16, 4, 130, 128, FP8Q_E4M3FN, Q, S, NULL) ==
               FP8Q_ERR_BAD_SHAPE);                                              /* n % group */
        EXPECT(fp8q_per_token_group_quant(NULL, FP8Q_BF16, 4, 128, 128, FP8Q_E4M3FN, Q, S, NULL) ==
               FP8Q_ERR_NULL_POINTER);
        EXPECT(fp8q_per_token_group_quant((const char*)P + 1, FP8Q_BF16, 4, 128, 128, FP8Q_E4M3FN, Q, S,
                                          NULL) == FP8Q_ERR_MISALIGNED);         /* bf16 on an odd address */
        EXPECT(fp8q_per_token_group_quant(NULL, FP8Q_BF16, 0, 128, 128, FP8Q_E4M3FN, NULL, NULL, NULL) ==
               FP8Q_OK);                                                         /* empty: nothing to do */
        EXPECT(fp8q_per_token_group_quant_ex(P, FP8Q_BF16, 4, 128, 128, FP8Q_E4M3FN, Q, S,
                                             (fp8q_scale_rule)2, NULL) == FP8Q_ERR_BAD_RULE);
        EXPECT(fp8q_cast_per_channel(P, FP8Q_F32, -4, 4, FP8Q_E4M3FN, Q, S, NULL) == FP8Q_ERR_BAD_SHAPE);
        EXPECT(fp8q_cast_per_tensor(P, FP8Q_F32, 16, FP8Q_E4M3FN, Q, S, NULL, 8192, NULL) == FP8Q_ERR_WORKSPACE);
        EXPECT(fp8q_cast_per_tensor(P, FP8Q_F32, 16, FP8Q_E4M3FN, Q, S, (void*)0x10000, 100, NULL) ==
               FP8Q_ERR_WORKSPACE);                                              /* too small */
        EXPECT(fp8q_block_dequant(Q, FP8Q_E4M3FN, 4, 4, S, 0, FP8Q_BF16, (void*)0x10000, NULL) ==
               FP8Q_ERR_BAD_SHAPE);                                              /* block < 1 */
        EXPECT(fp8q_block_dequant_grouped(NULL, -1, FP8Q_E4M3FN, 128, FP8Q_BF16, NULL) == FP8Q_ERR_TOO_MANY);
        EXPECT(fp8q_block_dequant_grouped(NULL, 0, FP8Q_E4M3FN, 128, FP8Q_BF16, NULL) == FP8Q_OK);
        EXPECT(fp8q_cast_from_fp8(Q, FP8Q_E4M3FN, 4, 4, S, (fp8q_granularity)4, 0, FP8Q_BF16, (void*)0x10000,
                                  NULL) == FP8Q_ERR_BAD_GRANULARITY);
        EXPECT(fp8q_scaled_mm(Q, FP8Q_E4M3FN, Q, FP8Q_E4M3FN, 8, 8, 24, S, S, NULL, FP8Q_BF16,
                              (void*)0x10000, NULL, NULL) == FP8Q_ERR_BAD_SHAPE);    /* K % 16 */
        EXPECT(fp8q_scaled_mm(NULL, FP8Q_E4M3FN, Q, FP8Q_E4M3FN, 8, 8, 32, S, S, NULL, FP8Q_BF16,
                              (void*)0x10000, NULL, NULL) == FP8Q_ERR_NULL_POINTER);
    }

    if (failures == 0) printf("ok: %zu entry points, every host rule as declared\n", n_entry);
    return failures == 0 ? 0 : 1;
}
