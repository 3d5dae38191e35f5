/*
 * Plain C (C11) client of the library's C ABI: compiles against include/pa.h and
 * include/pa_block_manager.h with a C compiler and links libpa_b200.so.  It calls
 * only host-side functions (no GPU is needed): version, status strings, host
 * validation of device calls (which fail before any CUDA call), the copy-pair
 * checked mode and the block manager, including a snapshot round trip.
 * Exit status 0 when every check holds; otherwise the number of the first failed check.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "pa.h"
#include "pa_block_manager.h"

#define CHECK(n, cond)                                      \
    do {                                                    \
        if (!(cond)) {                                      \
            fprintf(stderr, "check %d failed: %s\n", n, #cond); \
            return n;                                       \
        }                                                   \
    } while (0)

int main(void) {
    CHECK(1, pa_abi_version() == 3);
    CHECK(2, strcmp(pa_status_string(PA_OK), "ok") == 0);

    /* host validation of a device call: an unsupported block size fails first */
    pa_cache_desc bad = {8, 2, 32, 128, PA_BF16, 1.0f, 1.0f};
    void *fake = (void *)(uintptr_t)0x10000;
    CHECK(3, pa_cache_write(fake, fake, (const int64_t *)fake, 1, fake, fake, &bad, NULL, NULL) ==
                 PA_ERR_UNSUPPORTED);
    pa_cache_desc fp8 = {8, 2, 16, 128, PA_FP8_E4M3, 0.0f, 1.0f};
    CHECK(4, pa_cache_write(fake, fake, (const int64_t *)fake, 1, fake, fake, &fp8, NULL, NULL) ==
                 PA_ERR_INVALID_ARG);
    CHECK(5, pa_decode_workspace_size(3, 4, 64, 100, 0) == 0);
    CHECK(6, pa_decode_launches(8, 32, 8, 128, PA_BF16, 0) == 1);

    /* copy pairs: one source may feed several destinations; a repeated dst may not */
    const int32_t ok_pairs[] = {0, 1, 0, 2, 5, 4};
    const int32_t bad_pairs[] = {0, 1, 2, 1};
    CHECK(7, pa_check_copy_pairs(ok_pairs, 3, 8) == PA_OK);
    CHECK(8, pa_check_copy_pairs(bad_pairs, 2, 8) == PA_ERR_INVALID_ARG);

    /* block manager: a parent with 37 tokens, two forks, one step over both children */
    pa_block_manager *bm = NULL;
    CHECK(9, pa_bm_create(64, 16, NULL, &bm) == PA_OK && bm != NULL);
    CHECK(10, pa_bm_add_seq(bm, 0) == PA_OK);
    int64_t slots[64];
    int32_t pairs[8], ncow = -1;
    CHECK(11, pa_bm_append_slots(bm, 0, 37, slots, pairs, 4, &ncow) == PA_OK && ncow == 0);
    CHECK(12, pa_bm_fork(bm, 0, 1) == PA_OK && pa_bm_fork(bm, 0, 2) == PA_OK);
    CHECK(13, pa_bm_free_seq(bm, 0) == PA_OK);
    const int64_t kids[] = {1, 2};
    CHECK(14, pa_bm_append_step(bm, kids, NULL, 2, slots, pairs, 4, &ncow) == PA_OK);
    CHECK(15, ncow == 1);                                   /* the first child copies */
    CHECK(16, pa_bm_max_seq_blocks(bm, kids, 2) == 3);
    int32_t tables[2 * 3], lens[2];
    CHECK(17, pa_bm_build_tables(bm, kids, 2, 3, tables, lens) == PA_OK);
    CHECK(18, lens[0] == 38 && lens[1] == 38 && tables[0] == tables[3] && tables[2] != tables[5]);

    /* snapshot round trip */
    size_t need = pa_bm_snapshot_size(bm), got = 0;
    unsigned char *buf = (unsigned char *)malloc(need);
    CHECK(19, buf != NULL && pa_bm_snapshot(bm, buf, need, &got) == PA_OK && got == need);
    pa_block_manager *copy = NULL;
    CHECK(20, pa_bm_restore(buf, got, &copy) == PA_OK && copy != NULL);
    CHECK(21, pa_bm_block_size(copy) == 16 && pa_bm_num_blocks(copy) == 64);
    CHECK(22, pa_bm_num_tokens(copy, 1) == 38 && pa_bm_refcount(copy, tables[0]) == 2);
    CHECK(23, pa_bm_restore(buf, got - 1, &copy) == PA_ERR_INVALID_ARG);
    free(buf);
    pa_bm_destroy(copy);
    pa_bm_destroy(bm);
    printf("c abi ok\n");
    return 0;
}
