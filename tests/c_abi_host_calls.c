/* The C ABI from plain C (no C++, no torch): the header compiles as C99 and the
 * host-only calls answer without a GPU.  Built and run by tests/test_abi_c.py.
 * Prints "ok" and exits 0 when every check passes. */
#include <stdio.h>
#include <string.h>

#include "rma.h"

static int fails = 0;
#define CHECK(cond)                                                   \
    do {                                                              \
        if (!(cond)) {                                                \
            printf("check failed: %s (line %d)\n", #cond, __LINE__);  \
            ++fails;                                                  \
        }                                                             \
    } while (0)

int main(void) {
    rma_config cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.batch = 2;
    cfg.n_layers = 8;
    cfg.n_groups = 4;
    cfg.q_per_group = 4;
    cfg.head_dim = 256;
    cfg.ring_slots = 1023;
    cfg.bank_slots = 1024;
    cfg.pend_slots = 256;
    cfg.softmax_scale = 1.0f / 16.0f;

    /* the state size grows with the batch and nothing else */
    const size_t one = rma_state_bytes(&cfg);
    cfg.batch = 4;
    const size_t two = rma_state_bytes(&cfg);
    CHECK(one > 0);
    CHECK(two > one && two < 2 * one + 4096);
    cfg.batch = 2;

    /* FP8 storage: one byte per K/V element plus an exponent per row, about half the bytes */
    cfg.kv_format = RMA_KV_FP8_E4M3;
    const size_t fp8 = rma_state_bytes(&cfg);
    CHECK(fp8 > one / 2 && fp8 < one / 2 + one / 50);
    cfg.kv_format = 7;
    CHECK(rma_state_bytes(&cfg) == 0);
    cfg.kv_format = RMA_KV_BF16;

    /* an invalid configuration is refused with size 0 and a reason */
    cfg.head_dim = 128;
    CHECK(rma_state_bytes(&cfg) == 0);
    CHECK(strlen(rma_last_error()) > 0);
    cfg.head_dim = 256;

    /* argument errors are found on the host, before any CUDA call */
    rma_state* st = NULL;
    CHECK(rma_state_alloc(&cfg, NULL, one, NULL, &st) == RMA_ERR_INVALID_ARG);
    CHECK(st == NULL);
    CHECK(rma_state_alloc(NULL, NULL, one, NULL, &st) == RMA_ERR_INVALID_ARG);
    rma_state_free(NULL);   /* a no-op */

    /* every code has a text */
    CHECK(strlen(rma_strerror(RMA_OK)) > 0);
    CHECK(strlen(rma_strerror(RMA_ERR_INVALID_ARG)) > 0);
    CHECK(strlen(rma_strerror(RMA_ERR_MISALIGNED)) > 0);

    if (fails == 0) printf("ok\n");
    return fails == 0 ? 0 : 1;
}
