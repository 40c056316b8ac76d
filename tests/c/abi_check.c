/* Compiled as C (not C++) against include/hyb_attn.h and linked with
 * libhyb_attn.so: the header is usable from C and every call below resolves.
 * Only host-side paths run (sizes, status strings, argument validation), so
 * no GPU is needed.  Prints "ok" and exits 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "hyb_attn.h"

static int fails = 0;
#define CHECK(cond)                                              \
    do {                                                         \
        if (!(cond)) {                                           \
            fprintf(stderr, "check failed line %d: %s\n", __LINE__, #cond); \
            ++fails;                                             \
        }                                                        \
    } while (0)

int main(void) {
    hyb_attn_desc d;
    memset(&d, 0, sizeof(d));
    d.B = 1; d.H = 12; d.T = 1560; d.d_k = 128; d.d_v = 128; d.dtype = HYB_BF16;
    d.sm_scale = 0.0f; d.l2_eps = 1e-6f;
    size_t ws = hyb_attn_workspace_bytes(&d);
    CHECK(ws >= 256 && ws % 256 == 0);
    hyb_attn_desc bad = d;
    bad.d_k = bad.d_v = 64;
    CHECK(hyb_attn_workspace_bytes(&bad) == 0);

    void* p = (void*)(uintptr_t)0x10000; /* aligned, never dereferenced on these paths */
    /* argument errors are reported before anything is launched */
    CHECK(hyb_attn_forward(NULL, p, p, p, p, p, p, (const float*)p, (const float*)p, (float*)p, 1, p, p, ws, NULL) ==
          HYB_ERR_INVALID);
    CHECK(hyb_attn_forward(&d, p, p, p, p, p, p, (const float*)p, (const float*)p, (float*)p, 2, p, p, ws, NULL) ==
          HYB_ERR_INVALID);
    CHECK(hyb_attn_forward(&d, (char*)p + 2, p, p, p, p, p, (const float*)p, (const float*)p, (float*)p, 1, p, p,
                           ws, NULL) == HYB_ERR_ALIGN);
    CHECK(hyb_attn_forward(&d, p, p, p, p, p, p, (const float*)p, (const float*)p, (float*)p, 1, p, p, ws - 1,
                           NULL) == HYB_ERR_WORKSPACE);
    CHECK(hyb_attn_forward_mixed(&d, p, p, p, p, p, p, (const float*)p, (const float*)p, (float*)p, 1, NULL, p, p,
                                 ws, NULL) == HYB_ERR_INVALID);
    CHECK(hyb_kvcache_attn_forward(&d, p, p, p, p, p, 2 * 1560, 1560 + 1, p, p, 256, NULL) == HYB_ERR_INVALID);
    CHECK(hyb_attn_get_device_status(NULL, NULL) == HYB_ERR_INVALID);
    CHECK(strncmp(hyb_attn_status_string(HYB_ERR_TIMEOUT), "HYB_", 4) == 0);
    CHECK(hyb_attn_kernel_name(1) != NULL && hyb_attn_kernel_name(HYB_NUM_KERNELS) == NULL);
    if (fails) return 1;
    printf("ok\n");
    return 0;
}
