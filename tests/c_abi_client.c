/*
 * A plain C11 client of include/hisa.h: the header compiles as C, and the
 * library links and answers host-side queries from C without a GPU (every
 * call below returns before it would touch the device: workspace sizes,
 * argument checks, calls with nothing to do).  Prints "c abi ok" and exits 0
 * when every check holds; otherwise names the first failed check.
 */
#include <stdio.h>
#include <string.h>

#include "hisa.h"

static int failures = 0;

#define CHECK(cond)                                                  \
    do {                                                             \
        if (!(cond)) {                                               \
            fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
            ++failures;                                              \
        }                                                            \
    } while (0)

/* A cache descriptor with placeholder (never dereferenced) 256-aligned
 * addresses: the checks below stop before any device access. */
static hisa_kv make_kv(int cap, int B) {
    hisa_kv kv;
    memset(&kv, 0, sizeof kv);
    kv.keys = (void*)(uintptr_t)0x10000;
    kv.pooled = (float*)(uintptr_t)0x20000;
    kv.pooled_hl = (uint16_t*)(uintptr_t)0x30000;
    kv.len = (int32_t*)(uintptr_t)0x40000;
    kv.status = (uint32_t*)(uintptr_t)0x50000;
    kv.batch = 1;
    kv.cap = cap;
    kv.d = 128;
    kv.B = B;
    kv.dtype = HISA_KEY_BF16;
    kv.pool = HISA_POOL_MEAN;
    return kv;
}

int main(void) {
    const void* Q = (const void*)(uintptr_t)0x60000;
    const float* w = (const float*)(uintptr_t)0x70000;
    const int32_t* q_seq = (const int32_t*)(uintptr_t)0x80000;
    int32_t* idx = (int32_t*)(uintptr_t)0x90000;
    void* ws = (void*)(uintptr_t)0xA0000;

    CHECK(strcmp(hisa_status_string(HISA_OK), "ok") == 0);

    /* workspace of the 32K decode step: block keys, kept blocks, their
     * counts, row plans and token keys for 64 rows, B = 128, m = 64 */
    hisa_kv kv = make_kv(32768, 128);
    size_t sel = hisa_select_workspace_bytes(&kv, 64, 64, 64, 2048);
    CHECK(sel == 65536 + 16384 + 256 + 1024 + 2097152);
    CHECK(hisa_select_workspace_bytes(NULL, 1, 1, 1, 1) == 0);

    /* the search of any depth: one level is hisa_select's workspace, two
     * levels hisa_tree_select's, three levels more */
    hisa_kv kv1 = make_kv(32768, 1024), kv2 = make_kv(32768, 8192);
    const hisa_kv* one[1] = {&kv};
    const hisa_kv* two[2] = {&kv, &kv1};
    const hisa_kv* three[3] = {&kv, &kv1, &kv2};
    const int keep1[1] = {64}, keep2[2] = {64, 8}, keep3[3] = {64, 8, 2};
    CHECK(hisa_levels_workspace_bytes(one, 1, keep1, 64, 64, 2048) == sel);
    CHECK(hisa_levels_workspace_bytes(two, 2, keep2, 64, 64, 2048) ==
          hisa_tree_workspace_bytes(&kv, &kv1, 64, 64, 8, 64, 2048));
    CHECK(hisa_levels_workspace_bytes(three, 3, keep3, 64, 64, 2048) >
          hisa_levels_workspace_bytes(two, 2, keep2, 64, 64, 2048));

    /* argument checks, before any launch */
    CHECK(hisa_select(&kv, (const uint16_t*)Q, w, q_seq, NULL, 4, 64, 8, 0, idx, NULL, ws, sel, NULL) ==
          HISA_E_INVAL);
    CHECK(hisa_select(&kv, (const uint16_t*)Q, w, q_seq, NULL, 4, 129, 8, 16, idx, NULL, ws, sel, NULL) ==
          HISA_E_UNSUPPORTED);
    CHECK(hisa_select(&kv, (const uint16_t*)Q, w, q_seq, NULL, 4, 64, 8, 16, idx, NULL, ws, 16, NULL) ==
          HISA_E_WORKSPACE);
    CHECK(hisa_select(&kv, (const uint16_t*)Q, w, q_seq, NULL, 0, 64, 8, 16, idx, NULL, ws, sel, NULL) ==
          HISA_OK);
    hisa_kv other = make_kv(32768, 1024);
    other.keys = (void*)(uintptr_t)0x11000;       /* not kv's keys */
    const hisa_kv* mismatched[2] = {&kv, &other};
    CHECK(hisa_levels_select(mismatched, 2, keep2, (const uint16_t*)Q, w, q_seq, NULL, 4, 64, 16, idx,
                             NULL, NULL, NULL, NULL, ws, sel, NULL) == HISA_E_INVAL);
    CHECK(hisa_levels_select(three, 3, keep3, (const uint16_t*)Q, w, q_seq, NULL, 0, 64, 16, idx, NULL,
                             NULL, NULL, NULL, ws, sel, NULL) == HISA_OK);

    if (failures) return 1;
    printf("c abi ok\n");
    return 0;
}
