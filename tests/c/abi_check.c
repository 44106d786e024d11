/*
 * abi_check.c -- calls libmmscan through its C header from a plain C
 * program, with no CUDA or Python involved: every call below is rejected by
 * a host-side check (or by the launch-failure hook), so no GPU is needed.
 * Exit status 0 when every status matches; prints the first mismatch.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "mm_scan.h"

#define FAKE(k) ((void *)(uintptr_t)((uintptr_t)(k + 1) << 20)) /* 16-byte aligned, never dereferenced */

static int expect(const char *what, mm_status got, mm_status want)
{
    if (got != want) {
        printf("%s: got %d (%s), want %d\n", what, (int)got, mm_last_error(), (int)want);
        return 1;
    }
    return 0;
}

int main(void)
{
    int bad = 0;
    mm_scan_dims d = {2, 64, 16, 16, MM_F32};
    float *A = (float *)FAKE(2), *h = (float *)FAKE(6);

    bad |= expect("null dims", mm_scan_fwd(FAKE(0), FAKE(1), A, FAKE(3), FAKE(4), NULL, NULL, 0.9f, 1.0f,
                                           FAKE(5), NULL, NULL, NULL, NULL), MM_ERR_NULL);
    bad |= expect("beta >= 1", mm_scan_fwd(FAKE(0), FAKE(1), A, FAKE(3), FAKE(4), NULL, NULL, 1.0f, 1.0f,
                                           FAKE(5), NULL, NULL, &d, NULL), MM_ERR_SCALAR);
    bad |= expect("y over x", mm_scan_fwd(FAKE(0), FAKE(1), A, FAKE(3), FAKE(4), NULL, NULL, 0.9f, 1.0f,
                                          FAKE(0), NULL, NULL, &d, NULL), MM_ERR_ALIAS);
    d.dstate = 17;
    bad |= expect("dstate 17", mm_scan_fwd(FAKE(0), FAKE(1), A, FAKE(3), FAKE(4), NULL, NULL, 0.9f, 1.0f,
                                           FAKE(5), NULL, NULL, &d, NULL), MM_ERR_UNSUPPORTED);
    d.dstate = 16;
    d.io = 7;
    bad |= expect("dtype", mm_scan_fwd(FAKE(0), FAKE(1), A, FAKE(3), FAKE(4), NULL, NULL, 0.9f, 1.0f,
                                       FAKE(5), NULL, NULL, &d, NULL), MM_ERR_DTYPE);
    d.io = MM_F32;

    size_t bytes = 0;
    bad |= expect("ckpt size", mm_scan_ckpt_size(&d, &bytes), MM_OK);
    if (bytes != (size_t)2 * 16 * 4 * 2 * 16 * 4) {
        printf("ckpt size %zu\n", bytes);
        bad = 1;
    }
    mm_scan_dims one = {2, 1, 16, 16, MM_F32};
    bad |= expect("step: h and v on one buffer",
                  mm_scan_step(FAKE(0), FAKE(1), A, FAKE(3), FAKE(4), NULL, NULL, NULL, 0, h, h, 0.9f, 1.0f,
                               FAKE(7), &one, NULL), MM_ERR_ALIAS);
    mm_ssd_dims sd = {1, 128, 4, 64, 128, 1, 256};
    bad |= expect("ssd momentum: headdim 128",
                  (sd.headdim = 128, mm_ssd_fwd_momentum(FAKE(0), (float *)FAKE(1), A, FAKE(3), FAKE(4), NULL,
                                                         NULL, 0.9f, 1.0f, FAKE(5), NULL, NULL, &sd, NULL)),
                  MM_ERR_UNSUPPORTED);
    if (strlen(mm_status_string(MM_ERR_ALIAS)) == 0 || mm_version() <= 0) bad = 1;
    if (!bad) printf("abi ok\n");
    return bad;
}
