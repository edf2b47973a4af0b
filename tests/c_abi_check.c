/*
 * c_abi_check.c -- a plain C99 caller of the library's C ABI (include/nvq.h),
 * built and run by tests/test_c_abi_host.py on a host without a GPU.  It
 * calls only what needs no device: the size helpers, the status strings,
 * the wait-limit hook, and host-side argument checks, which return before
 * any CUDA call.  Prints "C ABI OK" and exits 0, else names the first
 * failed check and exits 1.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "nvq.h"

#define CHECK(cond)                                               \
    do {                                                          \
        if (!(cond)) {                                            \
            fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__); \
            return 1;                                             \
        }                                                         \
    } while (0)

int main(void) {
    static uint8_t buf[4096] __attribute__((aligned(16)));
    void* p = buf;

    /* sizes: NVFP4 [4608, 3072] codes K/2 bytes per row, scales 128x4 tiles */
    CHECK(nvq_codes_bytes(NVQ_NVFP4, 4608, 3072) == (size_t)4608 * 1536);
    CHECK(nvq_scale_bytes(NVQ_NVFP4, 4608, 3072) == (size_t)(4608 / 128) * (3072 / 16 / 4) * 512);
    CHECK(nvq_codes_bytes(NVQ_MXFP8, 100, 256) == (size_t)100 * 256);
    CHECK(nvq_scale_bytes(NVQ_MXFP8_E5M2, 100, 256) == (size_t)1 * 2 * 512);   /* rows padded to 128 */
    CHECK(nvq_codes_bytes(7, 128, 64) == 0);                                    /* unknown format */
    CHECK(nvq_workspace_bytes() == 256 * 128 + 1024 * 4 + 128);

    /* every return code has a name */
    {
        const int codes[] = {NVQ_OK, NVQ_ERR_NULL, NVQ_ERR_SHAPE, NVQ_ERR_ALIGN, NVQ_ERR_ARCH, NVQ_ERR_CUDA,
                             NVQ_ERR_FORMAT};
        size_t i;
        for (i = 0; i < sizeof codes / sizeof codes[0]; ++i) {
            const char* s = nvq_status_string(codes[i]);
            CHECK(s != NULL && strcmp(s, "unknown status") != 0);
        }
    }

    /* the wait-limit hook stores a process-wide value; no device needed */
    CHECK(nvq_set_wait_limit(4000000001ull) == NVQ_ERR_SHAPE);
    CHECK(nvq_set_wait_limit(1000) == NVQ_OK);
    CHECK(nvq_wait_limit() == 1000);
    CHECK(nvq_set_wait_limit(0) == NVQ_OK);
    CHECK(nvq_wait_limit() == 0);

    /* host-side argument checks return before any CUDA call */
    CHECK(nvfp4_quantize(NULL, 128, 64, 64, buf, buf, (float*)p, NULL, buf, NULL) == NVQ_ERR_NULL);
    CHECK(nvfp4_quantize(buf, 128, 48, 48, buf, buf, (float*)p, NULL, buf, NULL) == NVQ_ERR_SHAPE);
    CHECK(nvfp4_quantize(buf + 1, 128, 64, 64, buf, buf, (float*)p, NULL, buf, NULL) == NVQ_ERR_ALIGN);
    CHECK(mxfp8_quantize(buf, 128, 64, 64, buf, buf, NULL) == NVQ_ERR_SHAPE);      /* K % 128 != 0 */

    printf("C ABI OK\n");
    return 0;
}
