/*
 * Plain C11 user of libminikv.so: compiles against include/minikv.h alone and
 * exercises the calls that need no GPU (sizes, binding a cache descriptor,
 * ragged state, the decode cut, argument errors).  Exit status 0 = every check held.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "minikv.h"

static int failures = 0;
#define CHECK(cond)                                                        \
    do {                                                                   \
        if (!(cond)) {                                                     \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
            ++failures;                                                    \
        }                                                                  \
    } while (0)

int main(void)
{
    /* one layer of the Mistral-7B decode workload: B=16, Hkv=8, G=32, Gv=128, R=128, cap=6656 */
    size_t n = minikv_cache_bytes(16, 8, 128, 32, 128, 128, 6656);
    CHECK(n == 2u * 27262976u + 2u * 6815744u + 2u * 1703936u + 2u * 5242880u);
    CHECK(minikv_cache_bytes(16, 8, 64, 32, 128, 128, 6656) == 0);      /* D != 128 */

    minikv_cache c;
    memset(&c, 0xff, sizeof c);
    uintptr_t base = (uintptr_t)1 << 20;                                /* never dereferenced */
    CHECK(minikv_cache_bind(&c, (void *)base, n, 16, 8, 128, 32, 128, 128, 6656) == MINIKV_OK);
    CHECK((uintptr_t)c.k_codes == base && c.n_packed == 0 && c.n_res == 0 && c.seq == NULL && c.dseq == NULL);
    CHECK(minikv_cache_bind(&c, (void *)(base + 8), n, 16, 8, 128, 32, 128, 128, 6656) == MINIKV_ERR_INVALID_ARG);
    CHECK(minikv_last_error_string()[0] != '\0');

    /* ragged state: reset to empty; one row outside the batch is refused */
    int seq[3 * 16];
    for (int i = 0; i < 3 * 16; ++i) seq[i] = 7;
    CHECK(minikv_cache_set_ragged(&c, seq) == MINIKV_OK);
    for (int i = 0; i < 3 * 16; ++i) CHECK(seq[i] == 0);
    CHECK(minikv_quant_pack_seq(&c, 16, (const uint16_t *)base, (const uint16_t *)base, 10, NULL) ==
          MINIKV_ERR_INVALID_ARG);
    CHECK(minikv_cache_set_ragged(&c, NULL) == MINIKV_OK && c.seq == NULL);

    /* decode argument errors, before anything reaches the device */
    const uint16_t *p = (const uint16_t *)((uintptr_t)1 << 24);
    uint16_t *o = (uint16_t *)((uintptr_t)1 << 24);
    CHECK(minikv_decode_attn(&c, p, p, p, 12, 0.1f, o, (void *)p, 1 << 20, NULL) == MINIKV_ERR_INVALID_ARG);
    CHECK(minikv_decode_attn(&c, p, p, p, 48, 0.1f, o, (void *)p, 1 << 20, NULL) == MINIKV_ERR_UNSUPPORTED);
    CHECK(minikv_decode_attn_mass(&c, p, p, p, 32, 0.1f, o, NULL, (void *)p, 1 << 20, NULL) ==
          MINIKV_ERR_INVALID_ARG);

    /* the decode cut of the Mistral-7B step (6400 packed + 153 residual tokens per unit): one CTA
     * per unit of 31 residual + 200 packed items, boundary weight 2^20 */
    c.n_packed = 6400;
    c.n_res = 153;
    int ctas = 0, wu = 0, first[160];
    CHECK(minikv_decode_plan(&c, &ctas, &wu, first, 160) == MINIKV_OK);
    CHECK(ctas == 128 && wu == (1 << 20) && first[0] == 0 && first[1] == 231 && first[128] == 128 * 231);
    CHECK(minikv_decode_plan(&c, &ctas, &wu, first, 10) == MINIKV_ERR_INVALID_ARG);
    c.n_packed = 0;
    c.n_res = 0;

    /* workspace sizes */
    CHECK(minikv_workspace_size(MINIKV_OP_TOPK_EVICT, 1, 32, 32, 4096, 128, 32) == 0);
    CHECK(minikv_workspace_size(MINIKV_OP_DECODE_ATTN_MASS, 16, 32, 8, 6656 + 160, 128, 0) >
          minikv_workspace_size(MINIKV_OP_DECODE_ATTN, 16, 32, 8, 6656 + 160, 128, 0));

    if (failures == 0) printf("abi_check: all checks passed\n");
    return failures == 0 ? 0 : 1;
}
