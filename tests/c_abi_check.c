/*
 * A plain C99 consumer of libpkm.so (no Python, no torch, no CUDA headers):
 * include/pkm.h compiles as C, the library links, and the host-side paths
 * of the entry points behave as the header states.  No device memory is
 * touched: every call here either validates its arguments or is an empty
 * batch, both of which return before any CUDA call.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "pkm.h"

static int failures = 0;

#define EXPECT(cond, what)                                   \
    do {                                                     \
        if (!(cond)) {                                       \
            fprintf(stderr, "FAILED: %s (line %d)\n", what, __LINE__); \
            failures++;                                      \
        }                                                    \
    } while (0)

int main(void) {
    void *fake = (void *)(uintptr_t)(1u << 20); /* aligned, never dereferenced */
    EXPECT(pkm_version() >= 100, "version");
    for (int s = 0; s <= 6; s++)
        EXPECT(pkm_status_string((pkm_status)s) != NULL &&
                   strlen(pkm_status_string((pkm_status)s)) > 0,
               "status strings");

    pkm_fwd_args a;
    memset(&a, 0, sizeof a);
    a.T = 64;
    a.H = 2;
    a.d_half = 64;
    a.n_sub = 32;
    a.k = 8;
    a.d_v = 64;
    a.dtype = PKM_BF16;
    a.query = a.subkeys = a.values = fake;
    a.out = fake;
    a.idx = (int32_t *)fake;
    a.weights = (float *)fake;
    const size_t need = pkm_forward_workspace_size(&a);
    EXPECT(need > 0, "workspace size");
    a.workspace = fake;
    a.workspace_bytes = need - 1;
    EXPECT(pkm_forward(&a, NULL) == PKM_ERR_WORKSPACE, "short workspace");
    a.workspace_bytes = need;
    a.k = 0;
    EXPECT(pkm_forward(&a, NULL) == PKM_ERR_INVALID_ARG, "k = 0");
    EXPECT(pkm_select(&a, NULL) == PKM_ERR_INVALID_ARG, "select k = 0");
    a.k = 8;
    a.T = 0;
    EXPECT(pkm_forward(&a, NULL) == PKM_OK, "empty forward");
    EXPECT(pkm_select(&a, NULL) == PKM_OK, "empty selection");

    EXPECT(embbag_forward(fake, 10, 16, PKM_BF16, (const int32_t *)fake, (const float *)fake, 0, 4,
                          NULL, fake, NULL) == PKM_OK,
           "empty bag batch");
    EXPECT(embbag_forward(fake, 10, 12, PKM_BF16, (const int32_t *)fake, (const float *)fake, 1, 4,
                          NULL, fake, NULL) == PKM_ERR_INVALID_ARG,
           "bag width not a multiple of 8");
    EXPECT(embbag_forward_range(fake, 0, 0, 16, PKM_BF16, (const int32_t *)fake,
                                (const float *)fake, 1, 4, (float *)fake, NULL) ==
               PKM_ERR_INVALID_ARG,
           "empty shard");

    int32_t orders[2] = {2, 3};
    uint64_t seeds[4] = {1, 2, 3, 4};
    int64_t M[4] = {7, 11, 13, 17};
    pkm_engram_args e;
    memset(&e, 0, sizeof e);
    e.n_seq = 0;
    e.L = 8;
    e.n_orders = 2;
    e.K = 2;
    e.orders = orders;
    e.seeds = seeds;
    e.rows_per_head = M;
    e.d = 64;
    e.dtype = PKM_BF16;
    EXPECT(pkm_engram_forward(&e, NULL) == PKM_OK, "empty engram batch");
    orders[1] = 9;
    EXPECT(pkm_engram_forward(&e, NULL) == PKM_ERR_INVALID_ARG, "engram order 9");
    orders[1] = 3;
    EXPECT(pkm_check_wait_timeout(0, (int32_t *)fake, NULL) == PKM_ERR_INVALID_ARG,
           "timeout check with no polls");

    if (failures) return 1;
    printf("c abi ok\n");
    return 0;
}
