// paged_decode_attn_q4_0_noalloc: the q4_0 decode with the merge fused in, for
// callers that cannot hand the library a workspace.  Some hosts own all device
// memory and give a library only the buffers of the call itself (for example a
// plugin interface of an inference server that forbids allocation while it
// runs, to keep its memory use fixed), so the caller has no way to obtain the
// partial-result buffer the split-K decode needs.  This entry point uses a
// scratch array that lives in the library image instead, and allocates nothing.
//
// The scratch array is a file-scope __device__ array of KVQ_NOALLOC_WS_BYTES.
// Every GPU that loads the library holds it until the process exits.  Host code
// cannot use the array's name as a device address, so the first call on each
// device, with that device current, asks the runtime for the address
// (cudaGetSymbolAddress) and keeps it.  That first call should therefore come
// before any stream capture.
#include <mutex>

#include "kvq_internal.cuh"

using namespace kvq;

namespace {

__device__ __align__(256) static unsigned char g_noalloc_ws[KVQ_NOALLOC_WS_BYTES];

std::mutex g_mutex;
void *g_addr[64];            // device address of g_noalloc_ws per device ordinal, once known

int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ECUDA;
    if (dev < 0 || dev >= 64) return KVQ_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_ws);
        if (e != cudaSuccess || !p) return KVQ_ECUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return KVQ_OK;
}

}  // namespace

extern "C" int paged_decode_attn_q4_0_noalloc(const kvq_pool *pool, int layer, const float *q,
                                              const int32_t *page_table, int max_pages, const int32_t *plan,
                                              const kvq_plan_info *info, uint16_t *out_bf16, float *out_f32,
                                              int32_t *status, void *stream) {
    if (!out_bf16) return KVQ_EINVAL;
    // Every argument check runs before the scratch array is touched: the
    // counter clear below is sized from info, so an info that does not match
    // its own plan sizes must be rejected first.
    PoolGeom geo;
    const int vrc = check_decode_args(KVQ_Q4_0, pool, layer, q, page_table, max_pages, plan, info,
                                      KVQ_NOALLOC_WS_BYTES, out_bf16, out_f32, &geo);
    if (vrc == KVQ_ESIZE) return KVQ_ESIZE;   // the plan needs more than the array holds
    if (vrc != KVQ_OK) return vrc;
    void *ws = nullptr;
    const int rc = scratch_address(&ws);
    if (rc != KVQ_OK) return rc;
    // The array keeps the previous call's contents.  The fused merge needs its
    // per-group arrival counters at zero, so clear them on the caller's stream.
    const uint64_t counters_off = (uint64_t)info->n_units * ws_unit_floats(info->group) * sizeof(float);
    if (counters_off > info->workspace_bytes) return KVQ_EINVAL;   // excluded by the checks above; kept as a guard
    const uint64_t counters_bytes = info->workspace_bytes - counters_off;
    if (cudaMemsetAsync(static_cast<unsigned char *>(ws) + counters_off, 0, counters_bytes,
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return KVQ_ECUDA;
    return paged_decode_attn_q4_0_combined(pool, layer, q, page_table, max_pages, plan, info,
                                           static_cast<float *>(ws), KVQ_NOALLOC_WS_BYTES, out_bf16, out_f32, status,
                                           stream);
}
