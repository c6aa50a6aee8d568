/* c_abi_check.c -- a plain C11 caller of libkda: the header compiles as C, the
 * library links without any C++ or Python, and host-side validation answers
 * through the C ABI alone (no device is needed: every call below is rejected
 * or answered before any CUDA work).  Run by tests/test_c_abi.py. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "kda.h"

#define CHECK(cond)                                                   \
    do {                                                              \
        if (!(cond)) {                                                \
            fprintf(stderr, "c_abi_check: failed at line %d: %s\n",   \
                    __LINE__, #cond);                                 \
            return 1;                                                 \
        }                                                             \
    } while (0)

int main(void) {
    void* const fake = (void*)(uintptr_t)0x10000; /* never dereferenced */
    size_t lo = 0, hi = 0, n = 0;

    CHECK(kda_version() >= 100);
    CHECK(strncmp(kda_status_string(KDA_ERR_WORKSPACE), "KDA_ERR_WORKSPACE", 17) == 0);

    /* workspace queries are pure host arithmetic */
    CHECK(kda_chunk_fwd_workspace_size(8192, 32, 128, 128, 1, 8192, &lo, &hi) == KDA_OK);
    CHECK(lo > 0 && hi > lo);
    CHECK(kda_chunk_fwd_workspace_size(8192, 32, 64, 128, 1, 8192, &lo, &hi) == KDA_ERR_UNSUPPORTED);
    CHECK(kda_kcp_workspace_size(8192, 32, 128, 128, 1, 8192, &n) == KDA_OK && n == hi);
    CHECK(kda_chunk_bwd_workspace_size(8192, 32, 128, 128, 1, 8192, &n) == KDA_OK && n > hi);

    /* rejected before any launch */
    CHECK(kda_chunk_fwd(NULL, fake, fake, fake, fake, NULL, fake, NULL, 1, 128, 2, 128, 128, NULL, 1, 128,
                        KDA_BF16, KDA_BF16, 1.0f, NULL, NULL, 1e-6f, fake, (size_t)1 << 40, NULL)
          == KDA_ERR_INVALID_ARG);
    CHECK(kda_chunk_fwd(fake, fake, fake, fake, fake, NULL, fake, NULL, 1, 128, 2, 128, 128, NULL, 1, 128,
                        KDA_BF16, KDA_BF16, 1.0f, NULL, NULL, 1e-6f, (char*)fake + 16, (size_t)1 << 40, NULL)
          == KDA_ERR_MISALIGNED);
    CHECK(kda_decode_step(fake, fake, fake, fake, fake, fake, fake, 4, 2, 128, 96, KDA_BF16, KDA_BF16, 1.0f,
                          NULL, NULL, 1e-6f, NULL) == KDA_ERR_UNSUPPORTED);
    CHECK(kda_kcp_compose(NULL, 2, NULL, fake, 1, 2, 128, 128, NULL) == KDA_ERR_INVALID_ARG);
    CHECK(kda_query_status(NULL, NULL) == KDA_ERR_INVALID_ARG);
    puts("c_abi_check ok");
    return 0;
}
