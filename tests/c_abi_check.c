/* A plain C11 program against include/kvq.h: the header compiles as C and the
 * host-only entry points link and run from C, with no GPU.  Exit code 0 on
 * success, the number of the failed check otherwise. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "kvq.h"

int main(void) {
    kvq_pool_desc d = {16, 4, 24, 256, 256, 1024, KVQ_Q4_0};
    uint64_t bytes = 0;
    if (kvq_pool_bytes(&d, &bytes) != KVQ_OK || bytes != 16ull * 1024 * 4 * 256 * 288) return 1;
    kvq_layout lay;
    if (kvq_pool_layout(&d, &lay) != KVQ_OK || lay.bytes_per_token_head != 288) return 2;

    int32_t lens[1] = {262144};
    kvq_plan_info info;
    memset(&info, 0, sizeof info);
    if (kvq_decode_plan(&d, 1, lens, 1024, 148, NULL, 0, &info) != KVQ_ESIZE || info.plan_len <= 0) return 3;
    static int32_t plan[4096];
    if (info.plan_len > 4096) return 4;
    if (kvq_decode_plan(&d, 1, lens, 1024, 148, plan, info.plan_len, &info) != KVQ_OK || info.n_units != 148) return 5;

    int n_split = 0;
    uint64_t ws = 0;
    if (kvq_prefill_split(&d, 32256, 512, 0, &n_split, &ws) != KVQ_OK || n_split != 3 || ws == 0) return 6;

    /* residency planning over descriptors whose memory is never touched */
    kvq_pool host = {(void *)0x100000, {2, 4, 24, 256, 256, 8, KVQ_Q4_0}};
    kvq_pool cache = {(void *)0x200000, {1, 4, 24, 256, 256, 4, KVQ_Q4_0}};
    static uint64_t state[1024];
    const uint64_t sb = kvq_resident_state_bytes(2, 8, 4);
    if (sb == 0 || sb > sizeof state) return 7;
    if (kvq_resident_init(state, sb, &host, &cache) != KVQ_OK) return 8;
    int32_t hpt[2] = {5, 2}, cpt[2], loads[8];
    int32_t sl[1] = {300};
    int n_loads = 0;
    if (kvq_resident_map(state, 1, hpt, 1, 2, sl, cpt, loads, 4, &n_loads) != KVQ_OK || n_loads != 2) return 9;
    int slot = -9;
    if (kvq_resident_query(state, 1, 5, &slot) != KVQ_OK || slot != cpt[0]) return 10;
    int64_t hits = -1, misses = -1, ev = -1;
    if (kvq_resident_stats(state, &hits, &misses, &ev) != KVQ_OK || hits != 0 || misses != 2 || ev != 0) return 11;

    if (kv_append(NULL, 0, NULL, NULL, 1, NULL, NULL, NULL, 1, 1, NULL, NULL) != KVQ_EINVAL) return 12;
    printf("%s\n", kvq_version());
    return 0;
}
