// Host-resident KV with a device page cache ([Strata] "KV 从显存搬进内存之后发生了
// 什么": the authoritative KV lives in pinned host memory, the GPU keeps only the
// pages attention reads, a residency table with CLOCK (second chance) eviction
// decides which, missing pages come over the bus straight into the cache, and
// the attention kernels are unchanged, so their results are the same bits).
//
// Residency is per (layer, host page); a cache slot holds one page (every KV
// head of it) of any layer, so the cache is a one-layer pool of n_slots pages.
// kvq_resident_map is host-only planning; kvq_resident_load runs the page-in
// kernel, which reads the pinned host pages through unified addressing (no
// staging buffer, no copy engine) and writes the cache slots.
#include <algorithm>
#include <cstring>

#include "kvq_internal.cuh"

using namespace kvq;

namespace {

constexpr uint32_t RES_MAGIC = 0x4B565253u;   // "KVRS"
constexpr int LOADS_PER_LAUNCH = 1024;        // page-in list travels in the launch parameters

// State layout (caller memory): header, then one ResSlot per cache slot, then
// the residency table (one int32 per (layer, host page): its slot or -1).
struct ResHeader {
    uint32_t magic;
    int32_t n_layers, n_host_pages, n_slots;
    int32_t hand;              // CLOCK hand
    int32_t epoch;             // map-call counter; slots a call uses are pinned for it
    int64_t slot_bytes;        // one page, every KV head
    int64_t host_layer_stride;
    const uint8_t *host_base;  // as the caller passed it
    const uint8_t *host_dev;   // the same memory as the device addresses it (resolved on first load)
    uint8_t *cache_base;
    int64_t hits, misses, evictions;
};
struct ResSlot {
    int32_t key;               // layer * n_host_pages + host page, or -1 when empty
    int32_t ref;               // second-chance bit
    int32_t pinned;            // epoch of the last map call that used the slot
};

uint64_t state_bytes_for(int n_layers, int n_host_pages, int n_slots) {
    return sizeof(ResHeader) + (uint64_t)n_slots * sizeof(ResSlot) + (uint64_t)n_layers * n_host_pages * 4;
}
ResSlot *slots_of(ResHeader *h) { return reinterpret_cast<ResSlot *>(h + 1); }
int32_t *table_of(ResHeader *h) { return reinterpret_cast<int32_t *>(slots_of(h) + h->n_slots); }

struct LoadList {
    int32_t n;
    int2 page_slot[LOADS_PER_LAUNCH];   // (host page, cache slot)
};

// One CTA per page: four independent 16-byte loads per thread in flight, so
// enough requests are outstanding to cover the bus latency.
__global__ void __launch_bounds__(512) page_in_kernel(const uint8_t *host_layer, uint8_t *cache_base, int64_t slot_bytes,
                                                      const __grid_constant__ LoadList list) {
    grid_dependency_wait();
    const int2 ps = list.page_slot[blockIdx.x];
    const uint4 *src = reinterpret_cast<const uint4 *>(host_layer + (int64_t)ps.x * slot_bytes);
    uint4 *dst = reinterpret_cast<uint4 *>(cache_base + (int64_t)ps.y * slot_bytes);
    const int64_t n = slot_bytes / 16;
    int64_t i = threadIdx.x;
    for (; i + 3 * 512 < n; i += 4 * 512) {
        uint4 a = src[i], b = src[i + 512], c = src[i + 1024], d = src[i + 1536];
        dst[i] = a;
        dst[i + 512] = b;
        dst[i + 1024] = c;
        dst[i + 1536] = d;
    }
    for (; i < n; i += 512) dst[i] = src[i];
}

}  // namespace

extern "C" {

uint64_t kvq_resident_state_bytes(int n_layers, int n_host_pages, int n_cache_slots) {
    if (n_layers <= 0 || n_host_pages <= 0 || n_cache_slots <= 0) return 0;
    return state_bytes_for(n_layers, n_host_pages, n_cache_slots);
}

int kvq_resident_init(void *state, uint64_t state_bytes, const kvq_pool *host_pool, const kvq_pool *cache_pool) {
    if (!state || !host_pool || !cache_pool || !host_pool->base || !cache_pool->base) return KVQ_EINVAL;
    const kvq_pool_desc &hd = host_pool->desc, &cd = cache_pool->desc;
    kvq_layout hl, cl;
    if (kvq_pool_layout(&hd, &hl) != KVQ_OK || kvq_pool_layout(&cd, &cl) != KVQ_OK) return KVQ_EINVAL;
    if (hd.fmt != cd.fmt || hd.n_kv_heads != cd.n_kv_heads || hd.n_q_heads != cd.n_q_heads ||
        hd.head_dim != cd.head_dim || cd.n_layers != 1)
        return KVQ_EINVAL;
    if (state_bytes < state_bytes_for(hd.n_layers, hd.n_pages, cd.n_pages)) return KVQ_ESIZE;
    if ((reinterpret_cast<uintptr_t>(host_pool->base) & 15u) || (reinterpret_cast<uintptr_t>(cache_pool->base) & 15u))
        return KVQ_EALIGN;
    ResHeader *h = static_cast<ResHeader *>(state);
    std::memset(h, 0, sizeof(ResHeader));
    h->magic = RES_MAGIC;
    h->n_layers = hd.n_layers;
    h->n_host_pages = hd.n_pages;
    h->n_slots = cd.n_pages;
    h->slot_bytes = hl.slot_stride;
    h->host_layer_stride = hl.layer_stride;
    h->host_base = static_cast<const uint8_t *>(host_pool->base);
    h->cache_base = static_cast<uint8_t *>(cache_pool->base);
    ResSlot *s = slots_of(h);
    for (int i = 0; i < h->n_slots; ++i) s[i] = ResSlot{-1, 0, -1};
    int32_t *t = table_of(h);
    for (int64_t i = 0; i < (int64_t)h->n_layers * h->n_host_pages; ++i) t[i] = -1;
    return KVQ_OK;
}

int kvq_resident_map(void *state, int layer, const int32_t *host_page_table, int n_seq, int max_pages,
                     const int32_t *seq_len, int32_t *cache_page_table, int32_t *loads, int loads_capacity,
                     int *n_loads) {
    ResHeader *h = static_cast<ResHeader *>(state);
    if (!h || h->magic != RES_MAGIC || !host_page_table || !seq_len || !cache_page_table || !n_loads ||
        n_seq <= 0 || max_pages <= 0 || layer < 0 || layer >= h->n_layers || loads_capacity < 0 ||
        (!loads && loads_capacity > 0))
        return KVQ_EINVAL;
    ResSlot *s = slots_of(h);
    int32_t *t = table_of(h);

    // Validate everything and size the call before changing the state: the
    // distinct pages it needs must fit in the cache at once, and the caller's
    // list must hold every page that is not resident.
    for (int b = 0; b < n_seq; ++b) {
        const int T = seq_len[b];
        if (T < 0 || (int64_t)T > (int64_t)max_pages * PAGE) return KVQ_EINVAL;
        for (int p = 0; p < (T + PAGE - 1) / PAGE; ++p) {
            const int hp = host_page_table[(int64_t)b * max_pages + p];
            if (hp < 0 || hp >= h->n_host_pages) return KVQ_EINVAL;
        }
    }
    // Count distinct pages with temporary marks in the table itself (no
    // allocation): a missing page -1 becomes -2, a resident page in slot v
    // becomes -(v + 3); the second pass puts every entry back.
    int64_t need = 0, resident = 0;
    for (int pass = 0; pass < 2; ++pass)
        for (int b = 0; b < n_seq; ++b)
            for (int p = 0; p < (seq_len[b] + PAGE - 1) / PAGE; ++p) {
                int32_t &e = t[layer * h->n_host_pages + host_page_table[(int64_t)b * max_pages + p]];
                if (pass == 0) {
                    if (e == -1) {
                        e = -2;
                        ++need;
                    } else if (e >= 0) {
                        e = -(e + 3);
                        ++resident;
                    }
                } else if (e == -2) {
                    e = -1;
                } else if (e <= -3) {
                    e = -(e + 3);
                }
            }
    if (need + resident > h->n_slots) return KVQ_ESIZE;
    if (need > loads_capacity) {
        *n_loads = (int)need;
        return KVQ_ESIZE;
    }

    // Pin the resident part of the batch first, so that no miss of this call
    // evicts a page the same call reads.
    const int epoch = ++h->epoch;
    for (int b = 0; b < n_seq; ++b)
        for (int p = 0; p < (seq_len[b] + PAGE - 1) / PAGE; ++p) {
            const int32_t e = t[layer * h->n_host_pages + host_page_table[(int64_t)b * max_pages + p]];
            if (e >= 0) {
                s[e].ref = 1;
                s[e].pinned = epoch;
            }
        }
    int nl = 0;
    for (int b = 0; b < n_seq; ++b) {
        const int np = (seq_len[b] + PAGE - 1) / PAGE;
        for (int p = 0; p < np; ++p) {
            const int hp = host_page_table[(int64_t)b * max_pages + p];
            const int key = layer * h->n_host_pages + hp;
            int slot = t[key];
            if (slot >= 0) {                          // hit: the page earns a second chance
                ++h->hits;
                s[slot].ref = 1;
                s[slot].pinned = epoch;
            } else {                                  // miss: sweep the hand to a victim
                int victim = -1;
                while (victim < 0) {                  // ends within two sweeps: fewer pages are pinned than slots
                    ResSlot &c = s[h->hand];
                    if (c.pinned != epoch) {
                        if (c.ref) c.ref = 0;
                        else victim = h->hand;
                    }
                    h->hand = (h->hand + 1) % h->n_slots;
                }
                if (s[victim].key >= 0) {
                    t[s[victim].key] = -1;
                    ++h->evictions;
                }
                ++h->misses;
                s[victim] = ResSlot{key, 1, epoch};
                t[key] = victim;
                slot = victim;
                loads[2 * nl] = hp;
                loads[2 * nl + 1] = victim;
                ++nl;
            }
            cache_page_table[(int64_t)b * max_pages + p] = slot;
        }
        for (int p = np; p < max_pages; ++p) cache_page_table[(int64_t)b * max_pages + p] = -1;
    }
    *n_loads = nl;
    return KVQ_OK;
}

int kvq_resident_query(const void *state, int layer, int host_page, int *slot) {
    const ResHeader *h = static_cast<const ResHeader *>(state);
    if (!h || h->magic != RES_MAGIC || !slot || layer < 0 || layer >= h->n_layers || host_page < 0 ||
        host_page >= h->n_host_pages)
        return KVQ_EINVAL;
    *slot = table_of(const_cast<ResHeader *>(h))[(int64_t)layer * h->n_host_pages + host_page];
    return KVQ_OK;
}

int kvq_resident_stats(const void *state, int64_t *hits, int64_t *misses, int64_t *evictions) {
    const ResHeader *h = static_cast<const ResHeader *>(state);
    if (!h || h->magic != RES_MAGIC) return KVQ_EINVAL;
    if (hits) *hits = h->hits;
    if (misses) *misses = h->misses;
    if (evictions) *evictions = h->evictions;
    return KVQ_OK;
}

int kvq_resident_load(void *state, int layer, const int32_t *loads, int n_loads, void *stream) {
    ResHeader *h = static_cast<ResHeader *>(state);
    if (!h || h->magic != RES_MAGIC || n_loads < 0 || layer < 0 || layer >= h->n_layers) return KVQ_EINVAL;
    if (n_loads == 0) return KVQ_OK;
    if (!loads) return KVQ_EINVAL;
    for (int i = 0; i < n_loads; ++i)
        if (loads[2 * i] < 0 || loads[2 * i] >= h->n_host_pages || loads[2 * i + 1] < 0 ||
            loads[2 * i + 1] >= h->n_slots)
            return KVQ_EINVAL;
    if (!h->host_dev) {                               // the host pool must be pinned and mapped
        cudaPointerAttributes attr;
        if (cudaPointerGetAttributes(&attr, h->host_base) != cudaSuccess) return KVQ_ECUDA;
        if (attr.type != cudaMemoryTypeHost || !attr.devicePointer) return KVQ_EINVAL;
        h->host_dev = static_cast<const uint8_t *>(attr.devicePointer);
    }
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint8_t *host_layer = h->host_dev + (int64_t)layer * h->host_layer_stride;
    LoadList list;
    for (int done = 0; done < n_loads; done += LOADS_PER_LAUNCH) {
        list.n = std::min(LOADS_PER_LAUNCH, n_loads - done);
        for (int i = 0; i < list.n; ++i) list.page_slot[i] = make_int2(loads[2 * (done + i)], loads[2 * (done + i) + 1]);
        if (launch_ex(page_in_kernel, dim3((unsigned)list.n), dim3(512), 0, s, false, host_layer, h->cache_base,
                      h->slot_bytes, list) != cudaSuccess)
            return KVQ_ECUDA;
    }
    return KVQ_OK;
}

}  // extern "C"
