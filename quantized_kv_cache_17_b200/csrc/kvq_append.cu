// q_rotate and kv_append launches (the device code is in kvq_append_dev.cuh).
#include "kvq_append_dev.cuh"

namespace kvq {
namespace {

__global__ void __launch_bounds__(128) q_rotate_kernel(const float *q, float *q_rot, int64_t n_vec) {
    grid_dependency_wait();
    const int64_t vec = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (vec < n_vec) rotate_vec(q, q_rot, vec, threadIdx.x & 31);
}

template <int FMT>
__global__ void __launch_bounds__(128) append_kernel(uint8_t *pool, PoolGeom geo, int layer, const float *k,
                                                     const float *v, int64_t n_rows, const int32_t *row_seq,
                                                     const int32_t *row_pos, const int32_t *page_table,
                                                     int max_pages, int n_seq, int32_t *status) {
    grid_dependency_wait();
    append_item<FMT>(pool, geo, layer, k, v, n_rows, row_seq, row_pos, page_table, max_pages, n_seq, status,
                     (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5), threadIdx.x & 31);
}

// kv_append and q_rotate of one decode step in one launch: blocks below
// append_blocks encode (row, KV head) items, the rest rotate query vectors.
template <int FMT>
__global__ void __launch_bounds__(128) append_rotate_kernel(uint8_t *pool, PoolGeom geo, int layer, const float *k,
                                                            const float *v, int64_t n_rows, const int32_t *row_seq,
                                                            const int32_t *row_pos, const int32_t *page_table,
                                                            int max_pages, int n_seq, int32_t *status,
                                                            unsigned append_blocks, const float *q, float *q_rot,
                                                            int64_t n_vec) {
    grid_dependency_wait();
    const int lane = threadIdx.x & 31;
    if (blockIdx.x < append_blocks) {
        append_item<FMT>(pool, geo, layer, k, v, n_rows, row_seq, row_pos, page_table, max_pages, n_seq, status,
                         (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5), lane);
    } else {
        const int64_t vec = (int64_t)(blockIdx.x - append_blocks) * 4 + (threadIdx.x >> 5);
        if (vec < n_vec) rotate_vec(q, q_rot, vec, lane);
    }
}

}  // namespace

cudaError_t launch_q_rotate(const float *q, float *q_rot, int64_t n_vec, cudaStream_t s) {
    if (n_vec == 0) return cudaSuccess;
    const int64_t blocks = (n_vec + 3) / 4;
    return launch_ex(q_rotate_kernel, dim3((unsigned)blocks), dim3(128), 0, s, false, q, q_rot, n_vec);
}

cudaError_t launch_append_rotate(int fmt, uint8_t *pool, const PoolGeom &geo, int layer, const float *k,
                                 const float *v, int64_t n_rows, const int32_t *row_seq, const int32_t *row_pos,
                                 const int32_t *page_table, int max_pages, int n_seq, int32_t *status, const float *q,
                                 float *q_rot, int64_t n_vec, cudaStream_t s) {
    const int64_t items = n_rows * geo.n_kv_heads;
    const unsigned ablocks = (unsigned)((items + 3) / 4), rblocks = (unsigned)((n_vec + 3) / 4);
    if (ablocks + rblocks == 0) return cudaSuccess;
    auto kern = fmt == KVQ_INT8    ? append_rotate_kernel<KVQ_INT8>
                : fmt == KVQ_Q4_0  ? append_rotate_kernel<KVQ_Q4_0>
                : fmt == KVQ_K8V4  ? append_rotate_kernel<KVQ_K8V4>
                : fmt == KVQ_FP8   ? append_rotate_kernel<KVQ_FP8>
                                   : append_rotate_kernel<KVQ_NVFP4>;
    return launch_ex(kern, dim3(ablocks + rblocks), dim3(128), 0, s, false, pool, geo, layer, k, v, n_rows, row_seq,
                     row_pos, page_table, max_pages, n_seq, status, ablocks, q, q_rot, n_vec);
}

cudaError_t launch_append(int fmt, uint8_t *pool, const PoolGeom &geo, int layer, const float *k,
                          const float *v, int64_t n_rows, const int32_t *row_seq, const int32_t *row_pos,
                          const int32_t *page_table, int max_pages, int n_seq, int32_t *status, cudaStream_t s) {
    if (n_rows == 0) return cudaSuccess;
    const int64_t items = n_rows * geo.n_kv_heads;
    const unsigned blocks = (unsigned)((items + 3) / 4);
    auto kern = fmt == KVQ_INT8    ? append_kernel<KVQ_INT8>
                : fmt == KVQ_Q4_0  ? append_kernel<KVQ_Q4_0>
                : fmt == KVQ_K8V4  ? append_kernel<KVQ_K8V4>
                : fmt == KVQ_FP8   ? append_kernel<KVQ_FP8>
                                   : append_kernel<KVQ_NVFP4>;
    return launch_ex(kern, dim3(blocks), dim3(128), 0, s, false, pool, geo, layer, k, v, n_rows, row_seq, row_pos,
                     page_table, max_pages, n_seq, status);
}

}  // namespace kvq
