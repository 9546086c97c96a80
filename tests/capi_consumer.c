/* A plain C99 consumer of include/mea.h: compiled with gcc -std=c99
 * -pedantic -Werror and linked against libmea.so by test_capi_c.py.  It
 * makes only calls that the library refuses (or serves as no-ops) during
 * argument validation, so it runs without a GPU.  Pointer arguments are fake
 * addresses that no call dereferences.  Prints "ok" and exits 0 when every
 * check holds; otherwise prints the first failed check and exits 1. */
#include <stdio.h>
#include <string.h>

#include "mea.h"

#define CHECK(cond)                                                          \
    do {                                                                     \
        if (!(cond)) {                                                       \
            printf("failed: %s (line %d): %s\n", #cond, __LINE__,            \
                   mea_last_error());                                        \
            return 1;                                                        \
        }                                                                    \
    } while (0)

int main(void)
{
    void *x = (void *)0x100000, *y = (void *)0x200000, *dy = (void *)0x300000, *dx = (void *)0x400000;
    float *dparam = (float *)0x500000;
    void *ws = (void *)0x600000;
    const int64_t shape[4] = {2, 144, 3, 3};
    const int64_t bad_shape[4] = {2, -1, 3, 3};
    size_t need;

    CHECK(mea_version() > 0);
    CHECK(strcmp(mea_status_string(MEA_OK), "") != 0);
    CHECK(strcmp(mea_status_string(MEA_ERR_CUDA), "") != 0);

    /* n = 0 is a no-op, NULL pointers included, and clears the last error */
    CHECK(mea_act_fwd(MEA_SWISH, MEA_BF16, NULL, NULL, 0, 1.0f, NULL, NULL) == MEA_OK);
    CHECK(mea_last_error()[0] == '\0');

    /* bad enums, negative sizes, NULL pointers, overlapping outputs */
    CHECK(mea_act_fwd((mea_act_t)7, MEA_BF16, x, y, 10, 1.0f, NULL, NULL) == MEA_ERR_INVALID_ARG);
    CHECK(mea_last_error()[0] != '\0');
    CHECK(mea_act_fwd(MEA_SWISH, (mea_dtype_t)2, x, y, 10, 1.0f, NULL, NULL) == MEA_ERR_INVALID_ARG);
    CHECK(mea_act_fwd(MEA_SWISH, MEA_BF16, x, y, -1, 1.0f, NULL, NULL) == MEA_ERR_INVALID_ARG);
    CHECK(mea_act_fwd(MEA_SWISH, MEA_BF16, NULL, y, 10, 1.0f, NULL, NULL) == MEA_ERR_INVALID_ARG);
    CHECK(mea_act_fwd(MEA_SWISH, MEA_BF16, x, (char *)x + 2, 10, 1.0f, NULL, NULL) == MEA_ERR_INVALID_ARG);

    /* the d alpha backward needs a workspace of the advertised size */
    need = mea_act_bwd_workspace_bytes(MEA_SWISH, 1000, 1);
    CHECK(need >= 8);
    CHECK(mea_act_bwd(MEA_SWISH, MEA_BF16, x, dy, dx, 1000, 1.0f, NULL, dparam, NULL, need, NULL) ==
          MEA_ERR_WORKSPACE);
    CHECK(mea_act_bwd(MEA_SWISH, MEA_BF16, x, dy, dx, 1000, 1.0f, NULL, dparam, ws, need - 1, NULL) ==
          MEA_ERR_WORKSPACE);
    CHECK(mea_act_bwd(MEA_RELU, MEA_BF16, x, dy, dx, 1000, 1.0f, NULL, dparam, ws, need, NULL) ==
          MEA_ERR_UNSUPPORTED);

    /* grouped calls: counts, NULL tables, overlapping segments, d alpha in
     * some segments only, workspace size */
    {
        mea_act_segment_t segs[3];
        memset(segs, 0, sizeof(segs));
        segs[0].x = x; segs[0].dy = dy; segs[0].out = dx; segs[0].n = 1000; segs[0].param = 1.0f;
        segs[1].x = y; segs[1].dy = (char *)dy + 8192; segs[1].out = (char *)dx + 8192; segs[1].n = 10;
        segs[2].x = (char *)x + 8192; segs[2].dy = (char *)dy + 16384; segs[2].out = (char *)dx + 16384;
        segs[2].n = 0;
        CHECK(mea_act_fwd_grouped(MEA_SWISH, MEA_BF16, 0, NULL, NULL) == MEA_OK);
        CHECK(mea_act_fwd_grouped(MEA_SWISH, MEA_BF16, -1, segs, NULL) == MEA_ERR_INVALID_ARG);
        CHECK(mea_act_fwd_grouped(MEA_SWISH, MEA_BF16, 2, NULL, NULL) == MEA_ERR_INVALID_ARG);
        CHECK(mea_act_bwd_grouped((mea_act_t)8, MEA_BF16, 2, segs, NULL, 0, NULL) == MEA_ERR_INVALID_ARG);
        segs[1].out = (char *)dx + 100;   /* overlaps segment 0's dx */
        CHECK(mea_act_bwd_grouped(MEA_SWISH, MEA_BF16, 2, segs, NULL, 0, NULL) == MEA_ERR_INVALID_ARG);
        segs[1].out = (char *)dx + 8192;
        segs[0].dparam_dev = dparam;      /* d alpha in one segment only */
        CHECK(mea_act_bwd_grouped(MEA_SWISH, MEA_BF16, 2, segs, ws, 1 << 20, NULL) == MEA_ERR_INVALID_ARG);
        segs[1].dparam_dev = dparam + 1;
        segs[2].dparam_dev = dparam + 2;
        need = mea_act_bwd_grouped_workspace_bytes(MEA_SWISH, 3, segs);
        CHECK(need >= 3 * 256 && need % 256 == 0);
        CHECK(mea_act_bwd_grouped(MEA_SWISH, MEA_BF16, 3, segs, ws, need - 1, NULL) == MEA_ERR_WORKSPACE);
        CHECK(mea_act_bwd_grouped(MEA_SWISH, MEA_BF16, 3, segs, (char *)ws + 16, need, NULL) ==
              MEA_ERR_WORKSPACE);
        CHECK(mea_act_bwd_grouped(MEA_RELU, MEA_BF16, 3, segs, ws, need, NULL) == MEA_ERR_UNSUPPORTED);
    }

    /* per-channel entry points */
    need = mea_affine_swish_bwd_workspace_bytes(MEA_BF16, MEA_NHWC, shape);
    CHECK(need > 0);
    CHECK(mea_affine_swish_bwd_workspace_bytes(MEA_BF16, MEA_NHWC, bad_shape) == 0);
    CHECK(mea_affine_swish_fwd(MEA_BF16, MEA_NHWC, bad_shape, x, (float *)dy, (float *)dx, y, NULL) ==
          MEA_ERR_INVALID_ARG);
    CHECK(mea_affine_act_fwd((mea_act_t)9, MEA_BF16, MEA_NHWC, shape, x, (float *)dy, (float *)dx, 1.0f, y,
                             NULL) == MEA_ERR_INVALID_ARG);
    CHECK(mea_swish_channel_fwd(MEA_F32, (mea_layout_t)3, shape, x, (float *)dy, y, NULL) ==
          MEA_ERR_INVALID_ARG);
    {
        /* grouped per-channel Swish: the C struct, the size query, refusals */
        mea_channel_segment_t cs[2];
        memset(cs, 0, sizeof(cs));
        cs[0].x = x;
        cs[0].out = y;
        cs[0].alpha = (float *)dy;
        cs[0].shape[0] = 2;
        cs[0].shape[1] = 16;
        cs[0].shape[2] = 7;
        cs[0].shape[3] = 7;
        cs[1] = cs[0];
        cs[1].shape[1] = -1;
        CHECK(mea_swish_channel_fwd_grouped(MEA_BF16, 0, NULL, NULL) == MEA_OK);
        CHECK(mea_swish_channel_fwd_grouped(MEA_BF16, 2, cs, NULL) == MEA_ERR_INVALID_ARG);
        CHECK(mea_swish_channel_bwd_grouped_workspace_bytes(MEA_BF16, 2, cs) == 0);
        CHECK(mea_swish_channel_bwd_grouped_workspace_bytes(MEA_BF16, 1, cs) % 256 == 0);
        CHECK(mea_swish_channel_bwd_grouped_workspace_bytes(MEA_BF16, 1, cs) >=
              mea_swish_channel_bwd_workspace_bytes(MEA_BF16, MEA_NCHW, cs[0].shape));
        CHECK(mea_swish_channel_bwd_grouped(MEA_BF16, 1, cs, ws, 1 << 20, NULL) == MEA_ERR_INVALID_ARG);
    }

    /* matmul: K = 0 is not served, N must be a multiple of 8 */
    CHECK(mea_matmul_act_fwd(MEA_SWISH, 256, 256, 0, x, y, 1.0f, dy, dx, NULL) == MEA_ERR_UNSUPPORTED);
    CHECK(mea_matmul_act_fwd(MEA_SWISH, 256, 250, 64, x, y, 1.0f, dy, dx, NULL) == MEA_ERR_UNSUPPORTED);

    /* batch normalization: 1..128 pieces are served */
    CHECK(mea_concat_bn_relu_workspace_bytes(64, 224) > 0);
    CHECK(mea_concat_bn_relu_apply(MEA_BF16, 0, NULL, NULL, 64, 3136, (float *)dy, (float *)dx, (float *)dy,
                                   (float *)dx, y, NULL) == MEA_ERR_UNSUPPORTED);

    printf("ok\n");
    return 0;
}
