/*
 * A C (not C++) consumer of include/fp8bq.h: the header compiles as C99, the
 * descriptor layouts are the documented sizes, every declared entry point
 * links, and the calls that need no device behave as the header says
 * (argument errors are reported before any device is touched).
 */
#include <stdio.h>
#include <string.h>

#include "fp8bq.h"

#define CHECK(cond)                                                         \
    do {                                                                    \
        if (!(cond)) {                                                      \
            fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
            return 1;                                                       \
        }                                                                   \
    } while (0)

int main(void) {
    /* every entry point, taken by address so that the link resolves it */
    typedef void (*fn)(void);
    const fn entry[] = {
        (fn)fp8bq_quantize,       (fn)fp8bq_quantize_batched, (fn)fp8bq_dequantize,
        (fn)fp8bq_dequantize_batched, (fn)fp8bq_tensor_scale, (fn)fp8bq_status_string,
        (fn)fp8bq_sync_status,    (fn)fp8bq_version,          (fn)fp8bq_set_path,
        (fn)fp8bq_get_path,       (fn)fp8bq_path_for,         (fn)fp8bq_set_pdl,
        (fn)fp8bq_get_pdl,        (fn)fp8bq_debug_set_wait_limit_ns,
        (fn)fp8bq_debug_set_inject, (fn)fp8bq_launch_count, (fn)fp8bq_checked_build,
        (fn)fp8bq_debug_take_bounds,
    };
    size_t i;
    for (i = 0; i < sizeof entry / sizeof entry[0]; ++i) CHECK(entry[i] != NULL);

    CHECK(sizeof(fp8bq_desc) == 96);
    CHECK(sizeof(fp8bq_dequant_desc) == 80);
    CHECK(sizeof(fp8bq_scale_desc) == 24);
    CHECK(fp8bq_version() == FP8BQ_VERSION);
    CHECK(strlen(fp8bq_status_string(FP8BQ_ERR_SHAPE)) > 0);

    /* argument errors: reported before any device is touched */
    {
        float s[1];
        unsigned char y[1];
        CHECK(fp8bq_quantize(NULL, FP8BQ_BF16, 1, 1, 1, 128, 128, y, s, 0) == FP8BQ_ERR_NULL);
        CHECK(fp8bq_quantize((const void *)0x1000, FP8BQ_BF16, 1, 1, 1, 0, 128, y, s, 0) ==
              FP8BQ_ERR_BLOCK);
        CHECK(fp8bq_quantize((const void *)0x1000, FP8BQ_BF16, 4, 8, 7, 128, 128, y, s, 0) ==
              FP8BQ_ERR_SHAPE);
        CHECK(fp8bq_quantize_batched(NULL, -1, 0) == FP8BQ_ERR_ARG);
        CHECK(fp8bq_launch_count(NULL, -1) == -1);
        CHECK(fp8bq_quantize_batched(NULL, 0, 0) == FP8BQ_OK); /* nothing to do */
    }

    /* process-wide switches */
    CHECK(fp8bq_get_path() == FP8BQ_PATH_AUTO);
    CHECK(fp8bq_set_path(FP8BQ_PATH_GENERIC) == FP8BQ_OK);
    CHECK(fp8bq_get_path() == FP8BQ_PATH_GENERIC);
    CHECK(fp8bq_set_path((fp8bq_path)9) == FP8BQ_ERR_ARG);
    CHECK(fp8bq_set_path(FP8BQ_PATH_AUTO) == FP8BQ_OK);
    CHECK(fp8bq_get_pdl() == 1);
    CHECK(fp8bq_set_pdl(0) == FP8BQ_OK && fp8bq_get_pdl() == 0);
    CHECK(fp8bq_set_pdl(1) == FP8BQ_OK && fp8bq_get_pdl() == 1);
    /* the default build: no bounds record, and the trimming knob is refused */
    CHECK(fp8bq_checked_build() == 0);
    CHECK(fp8bq_debug_set_inject(FP8BQ_INJECT_TRIM_OUTPUTS) == FP8BQ_ERR_ARG);
    {
        uint64_t count = 1, first = 1;
        CHECK(fp8bq_debug_take_bounds(&count, &first) == FP8BQ_OK && count == 0 && first == 0);
    }
    CHECK(strlen(fp8bq_status_string(FP8BQ_ERR_DEVICE_BOUNDS)) > 0);

    printf("abi consumer ok\n");
    return 0;
}
