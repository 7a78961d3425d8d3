/* Calls libnvkv through its C header from plain C (no Python, no GPU): the
 * size functions and the host-side argument checks, which return before any
 * kernel is launched.  Exit status 0 when every expectation holds; prints
 * the first failed one otherwise. */
#include <stdint.h>
#include <stdio.h>

#include "nvkv.h"

#define EXPECT(cond)                                                    \
    do {                                                                \
        if (!(cond)) {                                                  \
            fprintf(stderr, "%s:%d: expectation failed: %s\n", __FILE__, \
                    __LINE__, #cond);                                   \
            return 1;                                                   \
        }                                                               \
    } while (0)

int main(void) {
    EXPECT(nvkv_page_bytes(4, 256) == 18432);
    EXPECT(nvkv_page_bytes(0, 256) == 0);
    EXPECT(nvkv_k8v4_page_bytes(4, 256) == 4 * (25 * 256 + 64));

    /* Workspace of a 3-sequence, T=1, 24/4-head, d=256 decode with 296
     * splits: (S + B*Hkv - 1) slots of R rows, o and lse, 256-B aligned. */
    size_t slots = 296 + 3 * 4 - 1, R = 6;
    size_t o = (slots * R * 256 * 4 + 255) / 256 * 256;
    size_t l = (slots * R * 4 + 255) / 256 * 256;
    EXPECT(nvkv_decode_workspace_bytes(3, 1, 24, 4, 256, 296) == o + l);

    /* The split plan of two sequences (130 and 0 tokens), one kv-head,
     * three splits: range c owns units [c*2/3, (c+1)*2/3), so range 0 owns
     * none, range 1 unit 0 and range 2 unit 1; the empty sequence has none. */
    int32_t lens[2] = {130, 0}, first[2], last[2];
    EXPECT(nvkv_split_plan(lens, 2, 1, 3, first, last) == NVKV_OK);
    EXPECT(first[0] == 1 && last[0] == 2);
    EXPECT(first[1] > last[1]);

    /* Argument checks (fake, never dereferenced addresses). */
    nvkv_cache cache = {(uint8_t *)(uintptr_t)0x10000, 8, 4, 256};
    nvkv_seqs seqs = {(const int32_t *)(uintptr_t)0x20000, 4, (const int32_t *)(uintptr_t)0x30000,
                      1, 64, NULL};
    const void *k = (const void *)(uintptr_t)0x40000, *v = (const void *)(uintptr_t)0x50000;
    const int32_t *cu = (const int32_t *)(uintptr_t)0x60000;
    EXPECT(nvkv_append(NULL, &seqs, k, v, cu, 1, 1, NULL) == NVKV_ERR_INVALID_ARG);
    EXPECT(nvkv_append(&cache, &seqs, k, v, cu, 0, 0, NULL) == NVKV_OK);
    nvkv_cache bad_d = cache;
    bad_d.head_dim = 64;
    EXPECT(nvkv_append_k8v4(&bad_d, &seqs, k, v, cu, 1, 1, NULL) == NVKV_ERR_UNSUPPORTED);
    size_t need = nvkv_decode_workspace_bytes(1, 1, 24, 4, 256, 8);
    void *ws = (void *)(uintptr_t)0x70000;
    EXPECT(nvkv_decode_attn(&cache, &seqs, k, 17, 24, 0.1f, 8, ws, need, NULL) ==
           NVKV_ERR_UNSUPPORTED);
    EXPECT(nvkv_decode_attn(&cache, &seqs, k, 1, 24, 0.1f, 8, ws, need - 1, NULL) ==
           NVKV_ERR_WORKSPACE);
    EXPECT(nvkv_decode_attn_k8v4(&cache, &seqs, k, 1, 25, 0.1f, 8, ws, need, NULL) ==
           NVKV_ERR_INVALID_ARG);
    EXPECT(nvkv_combine(&seqs, ws, 1, 24, 4, 256, 8, NULL, NULL) == NVKV_ERR_INVALID_ARG);
    EXPECT(nvkv_prefill_attn(&cache, &seqs, NULL, NULL, 0, 0, 24, 0.1f, NULL, NULL) == NVKV_OK);
    EXPECT(nvkv_rope_table(NULL, 16, 64, 1e4, 1.0, NULL) == NVKV_ERR_INVALID_ARG);
    EXPECT(nvkv_pages_spill(&cache, cu, cu, 0, ws, 4, NULL, NULL) == NVKV_OK);
    EXPECT(nvkv_status_string(NVKV_ERR_WORKSPACE)[0] != '\0');
    printf("ok\n");
    return 0;
}
