/* A plain C11 program that uses libpagedkv's host entry points through include/pagedkv.h alone: no Python,
 * no C++.  It follows a short allocator trace whose every result is fixed by the allocate / append_token /
 * free semantics of the page "LLM 推理引擎 Continuous Batching 与 PagedAttention" (§3.2 BlockManager: the
 * free list is a stack popped at its end; a block is taken when the stored length is a multiple of the block
 * size; freed blocks are pushed back in table order) and by §4.1's shared prefix (whole blocks, refcounted),
 * then checks that a checkpoint reads back to the same bytes.  Prints "ok" and exits 0, or names the first
 * step that differs and exits 1. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "pagedkv.h"

static int failures = 0;

static void expect(int cond, const char* what) {
    if (!cond && failures++ == 0) fprintf(stderr, "step failed: %s (%s)\n", what, pa_last_error());
}

static int table_is(const pa_alloc* a, int64_t req, const int32_t* want, int32_t n) {
    int32_t got[16], len = -1;
    if (pa_alloc_get_block_table(a, req, got, 16, &len) != PA_OK || len != n) return 0;
    return memcmp(got, want, sizeof(int32_t) * (size_t)n) == 0;
}

int main(void) {
    pa_alloc* a = NULL;
    expect(pa_alloc_create(8, 4, NULL, &a) == PA_OK && a != NULL, "create 8 blocks of 4 tokens");

    /* 9 tokens -> ceil(9/4) = 3 blocks, popped from the end of 0..7 */
    expect(pa_alloc_allocate(a, 1, 9) == PA_OK, "allocate req 1 (9 tokens)");
    const int32_t t1[3] = {7, 6, 5};
    expect(table_is(a, 1, t1, 3), "req 1 table = 7 6 5");

    /* position 9 lives in logical block 2 (block 5), row 1: slot 21; no block is taken */
    int64_t slot = -1;
    expect(pa_alloc_append_token(a, 1, &slot) == PA_OK && slot == 21, "append at position 9 -> slot 21");
    int64_t slots[3] = {0, 0, 0};
    expect(pa_alloc_append_tokens(a, 1, 3, slots) == PA_OK, "append 3 more");
    expect(slots[0] == 22 && slots[1] == 23 && slots[2] == 16, "slots 22 23, then a new block 4 row 0");
    const int32_t t1b[4] = {7, 6, 5, 4};
    expect(table_is(a, 1, t1b, 4), "req 1 table = 7 6 5 4");

    /* a 9-token prefix shares floor(9/4) = 2 whole blocks */
    expect(pa_alloc_fork(a, 1, 2, 9) == PA_OK, "fork req 1 -> req 2 over 9 tokens");
    const int32_t t2[2] = {7, 6};
    expect(table_is(a, 2, t2, 2), "req 2 table = 7 6");
    int32_t rc = 0, len = 0;
    expect(pa_alloc_refcount(a, 7, &rc) == PA_OK && rc == 2, "block 7 held twice");
    expect(pa_alloc_seq_len(a, 2, &len) == PA_OK && len == 8, "req 2 stores 8 tokens");

    /* freeing req 1 drops 7 and 6 to one reference and pushes 5 then 4 */
    expect(pa_alloc_free(a, 1) == PA_OK, "free req 1");
    int32_t fl[8], nfl = 0;
    const int32_t want_fl[6] = {0, 1, 2, 3, 5, 4};
    expect(pa_alloc_free_list(a, fl, 8, &nfl) == PA_OK && nfl == 6 &&
               memcmp(fl, want_fl, sizeof want_fl) == 0, "free list = 0 1 2 3 5 4");
    expect(pa_alloc_allocate(a, 3, 1) == PA_OK, "allocate req 3 (1 token)");
    const int32_t t3[1] = {4};
    expect(table_is(a, 3, t3, 1), "req 3 takes block 4, the top of the stack");
    expect(pa_alloc_allocate(a, 3, 1) == PA_ERR_EXISTS, "a second allocate of req 3 is refused");
    expect(pa_alloc_allocate(a, 4, 100) == PA_ERR_OOM, "25 blocks do not fit");

    /* the form the kernels read: padded tables and lengths */
    const int64_t reqs[2] = {2, 3};
    int32_t tables[2][3], lens[2];
    expect(pa_alloc_pack(a, reqs, 2, 3, &tables[0][0], lens) == PA_OK, "pack reqs 2 and 3");
    const int32_t want_tables[2][3] = {{7, 6, -1}, {4, -1, -1}};
    expect(memcmp(tables, want_tables, sizeof tables) == 0 && lens[0] == 8 && lens[1] == 1, "packed tables");

    /* checkpoint: size query, write, read back, write again */
    size_t need = 0;
    expect(pa_alloc_serialize(a, NULL, 0, &need) == PA_OK && need > 0, "checkpoint size query");
    uint8_t* buf = (uint8_t*)malloc(need);
    uint8_t* buf2 = (uint8_t*)malloc(need);
    size_t got = 0, got2 = 0;
    expect(buf && buf2 && pa_alloc_serialize(a, buf, need, &got) == PA_OK && got == need, "checkpoint");
    pa_alloc* b = NULL;
    expect(pa_alloc_deserialize(buf, need, &b) == PA_OK && b != NULL, "resume from the checkpoint");
    expect(pa_alloc_serialize(b, buf2, need, &got2) == PA_OK && got2 == need && memcmp(buf, buf2, need) == 0,
           "the resumed allocator writes the same bytes");
    pa_alloc* c = NULL;
    expect(pa_alloc_deserialize(buf, need - 1, &c) == PA_ERR_INVALID_ARG && c == NULL,
           "a truncated checkpoint is refused");
    free(buf);
    free(buf2);
    pa_alloc_destroy(b);
    pa_alloc_destroy(a);
    expect(strcmp(pa_status_string(PA_ERR_OOM), "") != 0, "status names");
    if (failures) return 1;
    printf("ok\n");
    return 0;
}
