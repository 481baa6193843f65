/*
 * A plain C client of libpagedattn.so, built by tests/test_abi_c.py: it shows
 * that the boundary is usable from C alone (no Python, no torch) and prints
 * what the host-side entry points return, for the test to compare with the
 * Python binding.  Nothing here touches a GPU.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "pa.h"
#include "pa_block_manager.h"

int main(void)
{
    printf("version %d\n", (int)pa_version());
    for (int s = 0; s <= 5; ++s) printf("status %d %s\n", s, pa_status_string(s));

    /* argument errors come back before anything is launched */
    pa_status st = pa_store_kvcache(NULL, NULL, 64, 64, NULL, NULL, NULL, -1, 1, 64, 16, 4, NULL);
    printf("store_negative %d\n", (int)st);
    st = pa_decode(NULL, NULL, NULL, NULL, NULL, 1, NULL, 10, 1, 4, 2, 96, 16, 4, 0.125f, 0, NULL, 0, NULL);
    printf("decode_head_dim_96 %d %s\n", (int)st, pa_last_error());

    /* XXH64 of the empty input and of "abc" */
    printf("xxh64_empty %llu\n", (unsigned long long)pa_xxh64("", 0, 0));
    printf("xxh64_abc %llu\n", (unsigned long long)pa_xxh64("abc", 3, 0));

    /* a block manager: two requests behind a shared 8-token prompt, block size 4 */
    pa_block_manager* bm = pa_bm_create(16, 4);
    if (!bm) return 1;
    const int32_t a[10] = {1, 2, 3, 4, 5, 6, 7, 8, 9, 10};
    const int32_t b[9] = {1, 2, 3, 4, 5, 6, 7, 8, 11};
    if (pa_bm_add_sequence(bm, 100, a, 10) || pa_bm_add_sequence(bm, 200, b, 9)) return 2;
    if (pa_bm_allocate(bm, 100) || pa_bm_allocate(bm, 200)) return 3;
    int32_t n = 0, cached = 0, nb = 0;
    pa_bm_sequence_info(bm, 200, &n, &cached, &nb);
    printf("seq200 tokens %d cached %d blocks %d free %d\n", n, cached, nb, pa_bm_num_free_blocks(bm));
    int64_t ids[2] = {100, 200};
    int32_t tables[2 * 4], cq[3], ck[3], slots[32], pos[32], total = 0;
    if (pa_bm_prepare_prefill(bm, ids, 2, 4, 32, tables, cq, ck, slots, pos, &total)) return 4;
    printf("prefill total_q %d cu_q %d %d %d cu_k %d %d %d\n", total, cq[0], cq[1], cq[2], ck[0], ck[1], ck[2]);
    printf("tables");
    for (int i = 0; i < 8; ++i) printf(" %d", tables[i]);
    printf("\nslots");
    for (int i = 0; i < total; ++i) printf(" %d", slots[i]);
    printf("\n");
    if (pa_bm_append_token(bm, 100, 42) || pa_bm_may_append(bm, 100)) return 5;
    int32_t dt[2 * 4], ctx[2], ds[2], dp[2];
    if (pa_bm_prepare_decode(bm, ids, 2, 4, dt, ctx, ds, dp)) return 6;
    printf("decode ctx %d %d slots %d %d pos %d %d\n", ctx[0], ctx[1], ds[0], ds[1], dp[0], dp[1]);
    st = pa_bm_allocate(bm, 999);
    printf("unknown_sequence %d\n", (int)st);
    pa_bm_destroy(bm);
    return 0;
}
