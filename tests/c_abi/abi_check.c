/* A plain C11 client of the libgdn ABI (include/libgdn.h): compiled with gcc, linked against
 * libgdn.so and run without a GPU.  It calls the paths that enqueue nothing: version, status
 * strings, workspace sizing, argument rejection and empty-input no-ops.  The device pointers
 * are aligned fake addresses that a rejecting call never dereferences. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "libgdn.h"

#define CHECK(cond)                                                          \
    do {                                                                     \
        if (!(cond)) {                                                       \
            fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
            return 1;                                                        \
        }                                                                    \
    } while (0)

#define A(n) ((void *)(uintptr_t)((uintptr_t)(n) << 20))

int main(void) {
    CHECK(gdn_api_version() == GDN_API_VERSION);
    for (int s = GDN_OK; s <= GDN_ERR_TIMEOUT; ++s) {
        const char *t = gdn_status_string((gdn_status)s);
        CHECK(t != NULL && strlen(t) > 0);
    }

    gdn_config cfg = {16, 48, 128, 128, 4, 1.0f, 1e-6f, GDN_ACT_NONE};
    size_t bytes = 0;
    CHECK(gdn_prefill_workspace_size(&cfg, GDN_BF16, 8192, 1, 0, &bytes) == GDN_OK && bytes > 0);
    /* with the longest sequence known, the size follows the chunk ranges, not the tokens */
    size_t b1 = 0, b2 = 0;
    CHECK(gdn_prefill_workspace_size(&cfg, GDN_BF16, 1 << 20, 16, 65536, &b1) == GDN_OK);
    CHECK(gdn_prefill_workspace_size(&cfg, GDN_BF16, 1 << 21, 16, 65536, &b2) == GDN_OK);
    CHECK(b1 == b2);
    gdn_config bad = cfg;
    bad.conv_activation = 7;
    CHECK(gdn_prefill_workspace_size(&bad, GDN_BF16, 8192, 1, 0, &bytes) == GDN_ERR_INVALID_ARG);
    bad = cfg;
    bad.d_k = 64;
    CHECK(gdn_prefill_workspace_size(&bad, GDN_BF16, 8192, 1, 0, &bytes) == GDN_ERR_UNSUPPORTED);
    CHECK(gdn_prefill_workspace_size(NULL, GDN_BF16, 8192, 1, 0, &bytes) == GDN_ERR_INVALID_ARG);
    CHECK(gdn_prefill_workspace_size(&cfg, GDN_BF16, -1, 1, 0, &bytes) == GDN_ERR_INVALID_ARG);
    CHECK(gdn_prefill_workspace_size(&cfg, GDN_BF16, 100, 1, -1, &bytes) == GDN_ERR_INVALID_ARG);

    /* prefill: rejected arguments, then an empty call */
    CHECK(gdn_prefill(&cfg, GDN_BF16, GDN_F32, NULL, A(2), A(3), A(4), A(5), A(6), A(7), A(8), A(9), 1, 100, 0,
                      NULL, NULL, NULL, NULL, A(10), A(11), (size_t)1 << 40, 0) == GDN_ERR_INVALID_ARG);
    CHECK(gdn_prefill(&cfg, GDN_BF16, GDN_F32, A(1), A(2), A(3), A(4), A(5), A(6), A(7), A(8), A(9), 1, 100, 0,
                      NULL, NULL, NULL, NULL, A(10), A(11), 16, 0) == GDN_ERR_WORKSPACE);
    CHECK(gdn_prefill(&cfg, GDN_BF16, GDN_F32, NULL, NULL, NULL, A(4), A(5), A(6), A(7), A(8), A(9), 0, 100, 0,
                      NULL, NULL, NULL, NULL, NULL, NULL, 0, 0) == GDN_OK);

    /* the no-allocation prefill: a problem whose tiles cannot fit GDN_STATIC_SCRATCH_BYTES even
     * with one chunk per sequence per range (more sequences than one chunk slot each fits) is
     * rejected on the host, before any device call */
    {
        const size_t slot = (size_t)16 * (65536 + 16384) + (size_t)48 * (16384 + 8192 + 16384 + 8192 + 640);
        const int n = (int)(GDN_STATIC_SCRATCH_BYTES / slot) + 1;
        CHECK(gdn_prefill_static_scratch(&cfg, GDN_BF16, GDN_F32, A(1), A(2), A(3), A(4), A(5), A(6), A(7), A(8),
                                         A(9), n, 64 * n, NULL, NULL, NULL, NULL, A(10), 0) == GDN_ERR_WORKSPACE);
        /* fp32 input keeps 40 KB of rows per token */
        const int64_t T = (int64_t)GDN_STATIC_SCRATCH_BYTES / (80 * 128 * 4) + 1;
        CHECK(gdn_prefill_static_scratch(&cfg, GDN_F32, GDN_F32, A(1), A(2), A(3), A(4), A(5), A(6), A(7), A(8),
                                         A(9), 1, T, NULL, NULL, NULL, NULL, A(10), 0) == GDN_ERR_WORKSPACE);
        printf("GDN_STATIC_SCRATCH_BYTES %zu\n", (size_t)GDN_STATIC_SCRATCH_BYTES);
    }

    /* decode (single and multi-token) and the output tail */
    CHECK(gdn_decode_step(&cfg, GDN_BF16, GDN_F32, A(1), A(2), A(3), A(4), A(5), A(6), A(7), A(8), NULL, A(10),
                          NULL, 4, A(11), 4, 0) == GDN_ERR_INVALID_ARG);
    CHECK(gdn_decode_step(&cfg, GDN_BF16, GDN_F32, NULL, A(2), A(3), A(4), A(5), A(6), A(7), A(8), A(9), A(10),
                          NULL, 4, A(11), 0, 0) == GDN_OK);
    CHECK(gdn_decode_multi(&cfg, GDN_BF16, GDN_F32, A(1), A(2), A(3), A(4), A(5), A(6), A(7), A(8), A(9), A(10),
                           NULL, 4, NULL, NULL, A(11), 4, 9, 0) == GDN_ERR_UNSUPPORTED);
    CHECK(gdn_decode_multi(&cfg, GDN_BF16, GDN_F32, NULL, A(2), A(3), A(4), A(5), A(6), A(7), A(8), A(9), A(10),
                           NULL, 4, NULL, NULL, A(11), 0, 4, 0) == GDN_OK);
    CHECK(gdn_output_gate(&cfg, GDN_F32, GDN_BF16, GDN_BF16, A(1), A(2), A(3), -1.0f, A(4), 10, 0) ==
          GDN_ERR_INVALID_ARG);
    CHECK(gdn_output_gate(&cfg, GDN_F32, GDN_BF16, GDN_BF16, NULL, A(2), A(3), 1e-6f, NULL, 0, 0) == GDN_OK);

    /* QSA indexer */
    CHECK(gdn_qsa_select_workspace_size(1, 8192, 16384, &bytes) == GDN_OK);
    CHECK(bytes == (size_t)8192 * 16384 * 4);
    CHECK(gdn_qsa_select_workspace_size(2, 3, 100, &bytes) == GDN_OK && bytes == 3072);
    CHECK(gdn_qsa_block_keys(A(1), A(2), A(3), 1, 6, 1e-6f, 1e4f, A(4), 16, 0) == GDN_ERR_INVALID_ARG);
    CHECK(gdn_qsa_block_keys(NULL, A(2), A(3), 0, 8, 1e-6f, 1e4f, NULL, 16, 0) == GDN_OK);
    CHECK(gdn_qsa_block_scores(A(1), A(2), A(3), A(4), A(5), 1, 2, 16, 1e-6f, -1.0f, A(6), 0) ==
          GDN_ERR_INVALID_ARG);
    CHECK(gdn_qsa_select(A(1), A(2), A(3), A(4), A(5), 1, 2, 16, 1e-6f, 1e4f, A(6), NULL, A(8), 16, 0) ==
          GDN_ERR_WORKSPACE);
    CHECK(gdn_qsa_select(NULL, A(2), A(3), A(4), A(5), 1, 0, 16, 1e-6f, 1e4f, NULL, NULL, NULL, 0, 0) == GDN_OK);

    /* a launch trace with nothing launched */
    gdn_trace_begin(NULL, 0);
    CHECK(gdn_trace_end() == 0);
    CHECK(gdn_last_cuda_error() == 0);

    puts("libgdn C ABI ok");
    return 0;
}
