// C ABI of the library: argument validation, pool layout, split plan, and the
// launches.  See include/kvq.h for the contract of every entry point.
#include <algorithm>
#include <cstring>
#include <vector>

#include "kvq_internal.cuh"

using namespace kvq;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_desc(const kvq_pool_desc *d) {
    if (!d) return KVQ_EINVAL;
    if (d->n_layers <= 0 || d->n_kv_heads <= 0 || d->n_q_heads <= 0 || d->n_pages <= 0) return KVQ_EINVAL;
    if (!host_valid_format(d->fmt)) return KVQ_EINVAL;
    if (d->head_dim != KVQ_HEAD_DIM || d->page_tokens != KVQ_PAGE_TOKENS) return KVQ_EUNSUPPORTED;
    if (d->n_q_heads % d->n_kv_heads != 0) return KVQ_EINVAL;
    if (d->n_q_heads / d->n_kv_heads > KVQ_MAX_GROUP) return KVQ_EUNSUPPORTED;
    return KVQ_OK;
}

int64_t tile_bytes_for(int fmt) {
    const int kp = host_part_k(fmt), vp = host_part_v(fmt);
    return part_code_bytes(kp) + part_scale_bytes(kp) + part_code_bytes(vp) + part_scale_bytes(vp);
}

void fill_layout(const kvq_pool_desc *d, kvq_layout *L) {
    const int kp = host_part_k(d->fmt), vp = host_part_v(d->fmt);
    L->tile_bytes = tile_bytes_for(d->fmt);
    L->k_codes_off = 0;
    L->k_scales_off = part_code_bytes(kp);
    L->v_codes_off = L->k_scales_off + part_scale_bytes(kp);
    L->v_scales_off = L->v_codes_off + part_code_bytes(vp);
    L->page_bytes = L->tile_bytes * TILES_PER_PAGE;
    L->head_stride = L->page_bytes;
    L->slot_stride = (int64_t)d->n_kv_heads * L->page_bytes;
    L->layer_stride = (int64_t)d->n_pages * L->slot_stride;
    L->total_bytes = (int64_t)d->n_layers * L->layer_stride;
    L->bytes_per_token_head = L->tile_bytes / TILE;
}

int check_pool(const kvq_pool *pool, int layer, PoolGeom *geo) {
    if (!pool || !pool->base) return KVQ_EINVAL;
    const int rc = check_desc(&pool->desc);
    if (rc) return rc;
    if (!aligned16(pool->base)) return KVQ_EALIGN;
    if (layer < 0 || layer >= pool->desc.n_layers) return KVQ_EINVAL;
    kvq_layout L;
    fill_layout(&pool->desc, &L);
    geo->layer_stride = L.layer_stride;
    geo->slot_stride = L.slot_stride;
    geo->page_bytes = L.page_bytes;
    geo->n_pages = pool->desc.n_pages;
    geo->n_kv_heads = pool->desc.n_kv_heads;
    return KVQ_OK;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ECUDA; }

}  // namespace

// Host-side checks of a decode call, shared by every decode entry point (and
// by the workspace-free one, which must run them before it touches its
// scratch array).  Fills geo on success.
int kvq::check_decode_args(int fmt, const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                           int max_pages, const int32_t *plan, const kvq_plan_info *info, uint64_t workspace_bytes,
                           const uint16_t *out_bf16, const float *out_f32, PoolGeom *geo) {
    int rc = check_pool(pool, layer, geo);
    if (rc) return rc;
    if (pool->desc.fmt != fmt) return KVQ_EINVAL;
    if (!q || !page_table || !plan || !info || max_pages <= 0) return KVQ_EINVAL;
    if (!aligned16(q)) return KVQ_EALIGN;
    const int G = pool->desc.n_q_heads / pool->desc.n_kv_heads;
    if (info->group != G || info->n_kv_heads != pool->desc.n_kv_heads || info->n_units <= 0 || info->n_seq <= 0)
        return KVQ_EINVAL;
    if ((int64_t)max_pages * PAGE > INT32_MAX) return KVQ_EINVAL;
    if (info->workspace_bytes != ws_bytes_for(info->n_units, G, info->n_seq * info->n_kv_heads)) return KVQ_EINVAL;
    if (workspace_bytes < info->workspace_bytes) return KVQ_ESIZE;
    if ((out_bf16 && !aligned16(out_bf16)) || (out_f32 && !aligned16(out_f32))) return KVQ_EALIGN;
    if (!out_bf16 && out_f32) return KVQ_EINVAL;
    return KVQ_OK;
}

namespace {

int decode_common(int fmt, bool tc, const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                  int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                  uint64_t workspace_bytes, int32_t *status, void *stream, uint16_t *out_bf16 = nullptr,
                  float *out_f32 = nullptr, const float *k_new = nullptr, const float *v_new = nullptr) {
    PoolGeom geo;
    if (!workspace) return KVQ_EINVAL;
    if (!aligned16(workspace)) return KVQ_EALIGN;
    const int rc = check_decode_args(fmt, pool, layer, q, page_table, max_pages, plan, info, workspace_bytes,
                                     out_bf16, out_f32, &geo);
    if (rc) return rc;
    const int inverse = host_rotated_v(fmt) ? 1 : 0;
    return cuda_rc(launch_decode(fmt, tc, static_cast<const uint8_t *>(pool->base), geo, layer, q, page_table,
                                 max_pages, plan, *info, workspace, status, inverse, out_bf16, out_f32,
                                 static_cast<cudaStream_t>(stream), k_new, v_new));
}

}  // namespace

extern "C" {

const char *kvq_version(void) { return "kvq 0.1 (sm_100a)"; }

int kvq_pool_bytes(const kvq_pool_desc *desc, uint64_t *bytes) {
    const int rc = check_desc(desc);
    if (rc) return rc;
    if (!bytes) return KVQ_EINVAL;
    kvq_layout L;
    fill_layout(desc, &L);
    *bytes = (uint64_t)L.total_bytes;
    return KVQ_OK;
}

int kvq_pool_layout(const kvq_pool_desc *desc, kvq_layout *out) {
    const int rc = check_desc(desc);
    if (rc) return rc;
    if (!out) return KVQ_EINVAL;
    fill_layout(desc, out);
    return KVQ_OK;
}

int q_rotate(const float *q, float *q_rot, int64_t n_vec, void *stream) {
    if (n_vec < 0) return KVQ_EINVAL;
    if (n_vec == 0) return KVQ_OK;
    if (!q || !q_rot) return KVQ_EINVAL;
    if (!aligned16(q) || !aligned16(q_rot)) return KVQ_EALIGN;
    if (n_vec > ((int64_t)1 << 36)) return KVQ_EINVAL;
    return cuda_rc(launch_q_rotate(q, q_rot, n_vec, static_cast<cudaStream_t>(stream)));
}

int kv_append(const kvq_pool *pool, int layer, const float *k, const float *v, int64_t n_rows,
              const int32_t *row_seq, const int32_t *row_pos, const int32_t *page_table, int max_pages, int n_seq,
              int32_t *status, void *stream) {
    PoolGeom geo;
    int rc = check_pool(pool, layer, &geo);
    if (rc) return rc;
    if (n_rows < 0 || max_pages <= 0 || n_seq <= 0) return KVQ_EINVAL;
    if (n_rows == 0) return KVQ_OK;
    if (!k || !v || !row_pos || !page_table) return KVQ_EINVAL;
    if (!aligned16(k) || !aligned16(v)) return KVQ_EALIGN;
    if ((int64_t)max_pages * PAGE > INT32_MAX || n_rows * geo.n_kv_heads > ((int64_t)1 << 34)) return KVQ_EINVAL;
    return cuda_rc(launch_append(pool->desc.fmt, static_cast<uint8_t *>(pool->base), geo, layer, k, v, n_rows,
                                 row_seq, row_pos, page_table, max_pages, n_seq, status,
                                 static_cast<cudaStream_t>(stream)));
}

int kv_append_q_rotate(const kvq_pool *pool, int layer, const float *k, const float *v, int64_t n_rows,
                       const int32_t *row_seq, const int32_t *row_pos, const int32_t *page_table, int max_pages,
                       int n_seq, const float *q, float *q_rot, int64_t n_vec, int32_t *status, void *stream) {
    PoolGeom geo;
    int rc = check_pool(pool, layer, &geo);
    if (rc) return rc;
    if (n_rows < 0 || n_vec < 0 || max_pages <= 0 || n_seq <= 0) return KVQ_EINVAL;
    if (n_rows == 0 && n_vec == 0) return KVQ_OK;
    if (n_rows > 0 && (!k || !v || !row_pos || !page_table)) return KVQ_EINVAL;
    if (n_vec > 0 && (!q || !q_rot)) return KVQ_EINVAL;
    if ((n_rows > 0 && (!aligned16(k) || !aligned16(v))) || (n_vec > 0 && (!aligned16(q) || !aligned16(q_rot))))
        return KVQ_EALIGN;
    if ((int64_t)max_pages * PAGE > INT32_MAX || n_rows * geo.n_kv_heads > ((int64_t)1 << 34) ||
        n_vec > ((int64_t)1 << 34))
        return KVQ_EINVAL;
    return cuda_rc(launch_append_rotate(pool->desc.fmt, static_cast<uint8_t *>(pool->base), geo, layer, k, v, n_rows,
                                        row_seq, row_pos, page_table, max_pages, n_seq, status, q, q_rot, n_vec,
                                        static_cast<cudaStream_t>(stream)));
}

int kvq_decode_plan(const kvq_pool_desc *desc, int n_seq, const int32_t *seq_len, int max_pages, int n_ctas,
                    int32_t *plan, int plan_capacity, kvq_plan_info *info) {
    int rc = check_desc(desc);
    if (rc) return rc;
    if (n_seq <= 0 || !seq_len || !info || max_pages <= 0 || n_ctas < 0) return KVQ_EINVAL;
    if ((int64_t)max_pages * PAGE > INT32_MAX) return KVQ_EINVAL;
    const int n_kv = desc->n_kv_heads, G = desc->n_q_heads / desc->n_kv_heads;
    std::vector<int64_t> steps(n_seq);
    int64_t total = 0;
    for (int b = 0; b < n_seq; ++b) {
        if (seq_len[b] <= 0 || (int64_t)seq_len[b] > (int64_t)max_pages * PAGE) return KVQ_EINVAL;
        steps[b] = (seq_len[b] + STEP_TOKENS - 1) / STEP_TOKENS;
        total += steps[b] * n_kv;
    }
    if (n_ctas == 0) {
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return KVQ_ECUDA;
        n_ctas = sms;   // one decode CTA per SM
    }
    auto units_for = [&](int64_t c) {
        int64_t n = 0;
        for (int b = 0; b < n_seq; ++b) n += n_kv * ((steps[b] + c - 1) / c);
        return n;
    };
    int64_t maxsteps = *std::max_element(steps.begin(), steps.end());
    int64_t c = std::max<int64_t>(1, (total + n_ctas - 1) / n_ctas);
    if (c > maxsteps) c = maxsteps;
    while (c < maxsteps && units_for(c) > n_ctas) ++c;
    const int64_t n_units = units_for(c);
    if (n_units > (1 << 24)) return KVQ_EUNSUPPORTED;
    const int len = plan_len_for((int)n_units, n_seq, n_kv);
    info->n_units = (int32_t)n_units;
    info->n_seq = n_seq;
    info->n_kv_heads = n_kv;
    info->group = G;
    info->plan_len = len;
    info->chunk_tokens = (int32_t)(c * STEP_TOKENS);
    info->workspace_bytes = ws_bytes_for((int)n_units, G, n_seq * n_kv);
    if (!plan || plan_capacity < len) return KVQ_ESIZE;
    plan[0] = PLAN_MAGIC;
    plan[1] = (int32_t)n_units;
    plan[2] = n_seq;
    plan[3] = n_kv;
    plan[4] = G;
    plan[5] = (int32_t)(c * STEP_TOKENS);
    plan[6] = plan[7] = 0;
    int32_t *units = plan + PLAN_HEADER;
    int32_t *start = units + 4 * n_units;
    int u = 0;
    for (int b = 0; b < n_seq; ++b) {
        const int64_t nu = (steps[b] + c - 1) / c;
        const int64_t base = steps[b] / nu, rem = steps[b] % nu;
        for (int g = 0; g < n_kv; ++g) {
            start[b * n_kv + g] = u;
            int64_t s0 = 0;
            for (int64_t k = 0; k < nu; ++k) {
                const int64_t ns = base + (k < rem ? 1 : 0);
                units[4 * u + 0] = b;
                units[4 * u + 1] = g;
                units[4 * u + 2] = (int32_t)(s0 * STEP_TOKENS);
                units[4 * u + 3] = (int32_t)std::min<int64_t>((s0 + ns) * STEP_TOKENS, seq_len[b]);
                s0 += ns;
                ++u;
            }
        }
    }
    start[n_seq * n_kv] = u;
    return KVQ_OK;
}

int paged_decode_attn_int8(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table, int max_pages,
                           const int32_t *plan, const kvq_plan_info *info, float *workspace, uint64_t workspace_bytes,
                           int32_t *status, void *stream) {
    return decode_common(KVQ_INT8, true, pool, layer, q, page_table, max_pages, plan, info, workspace,
                         workspace_bytes, status, stream);
}

int paged_decode_attn_q4_0(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table, int max_pages,
                           const int32_t *plan, const kvq_plan_info *info, float *workspace, uint64_t workspace_bytes,
                           int32_t *status, void *stream) {
    return decode_common(KVQ_Q4_0, true, pool, layer, q, page_table, max_pages, plan, info, workspace,
                         workspace_bytes, status, stream);
}

int paged_decode_attn_k8v4(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table, int max_pages,
                           const int32_t *plan, const kvq_plan_info *info, float *workspace, uint64_t workspace_bytes,
                           int32_t *status, void *stream) {
    return decode_common(KVQ_K8V4, true, pool, layer, q, page_table, max_pages, plan, info, workspace,
                         workspace_bytes, status, stream);
}

int paged_decode_attn_fp8(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table, int max_pages,
                          const int32_t *plan, const kvq_plan_info *info, float *workspace, uint64_t workspace_bytes,
                          int32_t *status, void *stream) {
    return decode_common(KVQ_FP8, true, pool, layer, q, page_table, max_pages, plan, info, workspace,
                         workspace_bytes, status, stream);
}

int paged_decode_attn_nvfp4(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table, int max_pages,
                            const int32_t *plan, const kvq_plan_info *info, float *workspace, uint64_t workspace_bytes,
                            int32_t *status, void *stream) {
    return decode_common(KVQ_NVFP4, true, pool, layer, q, page_table, max_pages, plan, info, workspace,
                         workspace_bytes, status, stream);
}

int paged_decode_attn_cudacore(int fmt, const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                               int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                               uint64_t workspace_bytes, int32_t *status, void *stream) {
    if (!host_valid_format(fmt)) return KVQ_EINVAL;
    if (fmt == KVQ_FP8 || fmt == KVQ_NVFP4) return KVQ_EUNSUPPORTED;   // the control covers the three 2-part formats
    if (pool) {
        const int G = pool->desc.n_kv_heads > 0 ? pool->desc.n_q_heads / pool->desc.n_kv_heads : 0;
        if (G != 4 && G != 6 && G != 8) return KVQ_EUNSUPPORTED;
    }
    return decode_common(fmt, false, pool, layer, q, page_table, max_pages, plan, info, workspace, workspace_bytes,
                         status, stream);
}

#define KVQ_COMBINED(NAME, FMT)                                                                                 \
    int NAME(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table, int max_pages,              \
             const int32_t *plan, const kvq_plan_info *info, float *workspace, uint64_t workspace_bytes,             \
             uint16_t *out_bf16, float *out_f32, int32_t *status, void *stream) {                                    \
        if (!out_bf16) return KVQ_EINVAL;                                                                            \
        return decode_common(FMT, true, pool, layer, q, page_table, max_pages, plan, info, workspace,               \
                             workspace_bytes, status, stream, out_bf16, out_f32);                                   \
    }
KVQ_COMBINED(paged_decode_attn_int8_combined, KVQ_INT8)
KVQ_COMBINED(paged_decode_attn_q4_0_combined, KVQ_Q4_0)
KVQ_COMBINED(paged_decode_attn_k8v4_combined, KVQ_K8V4)
KVQ_COMBINED(paged_decode_attn_fp8_combined, KVQ_FP8)
KVQ_COMBINED(paged_decode_attn_nvfp4_combined, KVQ_NVFP4)
#undef KVQ_COMBINED

#define KVQ_STEP(NAME, FMT)                                                                                     \
    int NAME(const kvq_pool *pool, int layer, const float *q, const float *k_new, const float *v_new,              \
             const int32_t *page_table, int max_pages, const int32_t *plan, const kvq_plan_info *info,            \
             float *workspace, uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32, int32_t *status,      \
             void *stream) {                                                                                       \
        if (!out_bf16 || !k_new || !v_new) return KVQ_EINVAL;                                                      \
        if (!aligned16(k_new) || !aligned16(v_new)) return KVQ_EALIGN;                                             \
        return decode_common(FMT, true, pool, layer, q, page_table, max_pages, plan, info, workspace,             \
                             workspace_bytes, status, stream, out_bf16, out_f32, k_new, v_new);                   \
    }
KVQ_STEP(paged_decode_step_int8, KVQ_INT8)
KVQ_STEP(paged_decode_step_q4_0, KVQ_Q4_0)
KVQ_STEP(paged_decode_step_k8v4, KVQ_K8V4)
KVQ_STEP(paged_decode_step_fp8, KVQ_FP8)
KVQ_STEP(paged_decode_step_nvfp4, KVQ_NVFP4)
#undef KVQ_STEP

int kvq_prefill_split(const kvq_pool_desc *desc, int pos0, int n_tok, int n_sms, int *n_split,
                      uint64_t *workspace_bytes) {
    uint64_t pb = 0;
    if (!desc || !n_split || !workspace_bytes) return KVQ_EINVAL;
    const int rc = kvq_pool_bytes(desc, &pb);
    if (rc) return rc;
    if (n_tok <= 0 || pos0 < 0 || (int64_t)pos0 + n_tok > INT32_MAX || n_sms < 0) return KVQ_EINVAL;
    const int sms = n_sms ? n_sms : 148;
    const int G = desc->n_q_heads / desc->n_kv_heads;
    const int64_t n_rows = (int64_t)n_tok * G;
    const int64_t ctas = (n_rows + 63) / 64 * desc->n_kv_heads;    // CTAs of one part (64 rows each)
    const int64_t t_end = (int64_t)pos0 + n_tok;
    // cost of a choice: waves of CTAs times the longest part
    int best = 1;
    int64_t best_cost = (ctas + sms - 1) / sms * t_end;
    for (int s = 2; s <= PF_MAX_SPLIT; ++s) {
        const int st = prefill_split_tokens(pos0, n_tok, s);
        if (!st) break;
        const int64_t longest = std::max<int64_t>(st, t_end - (int64_t)(s - 1) * st);
        const int64_t cost = (ctas * s + sms - 1) / sms * longest;
        if (cost < best_cost) {
            best = s;
            best_cost = cost;
        }
    }
    *n_split = best;
    *workspace_bytes = best > 1 ? (uint64_t)best * desc->n_kv_heads * n_rows * PF_WS_STRIDE * sizeof(float) : 0;
    return KVQ_OK;
}

int paged_prefill_attn(const kvq_pool *pool, int layer, const float *q, int seq, int pos0, int n_tok,
                       const int32_t *page_table, int max_pages, int n_seq, int n_split, float *workspace,
                       uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32, int32_t *status, void *stream) {
    PoolGeom geo;
    const int rc = check_pool(pool, layer, &geo);
    if (rc) return rc;
    if (!q || !page_table || !out_bf16 || n_tok <= 0 || pos0 < 0 || max_pages <= 0 || seq < 0 || seq >= n_seq)
        return KVQ_EINVAL;
    if ((int64_t)max_pages * PAGE > INT32_MAX || (int64_t)pos0 + n_tok > (int64_t)max_pages * PAGE) return KVQ_EINVAL;
    if ((int64_t)n_tok * pool->desc.n_q_heads > ((int64_t)1 << 28)) return KVQ_EINVAL;
    if (n_split < 1 || n_split > PF_MAX_SPLIT) return KVQ_EINVAL;
    const int split_tokens = prefill_split_tokens(pos0, n_tok, n_split);
    if (n_split > 1) {
        if (!split_tokens || !workspace) return KVQ_EINVAL;
        const uint64_t need = (uint64_t)n_split * pool->desc.n_kv_heads * ((uint64_t)n_tok * pool->desc.n_q_heads /
                                                                            pool->desc.n_kv_heads) *
                              PF_WS_STRIDE * sizeof(float);
        if (workspace_bytes < need) return KVQ_ESIZE;
        if (!aligned16(workspace)) return KVQ_EALIGN;
    }
    if (!aligned16(q) || !aligned16(out_bf16) || (out_f32 && !aligned16(out_f32))) return KVQ_EALIGN;
    return cuda_rc(launch_prefill(pool->desc.fmt, static_cast<const uint8_t *>(pool->base), geo, layer, q, seq, pos0,
                                  n_tok, page_table, max_pages, pool->desc.n_q_heads, n_split, split_tokens,
                                  workspace, host_rotated_v(pool->desc.fmt) ? 1 : 0, out_bf16, out_f32, status,
                                  static_cast<cudaStream_t>(stream)));
}

int attn_combine(const float *workspace, const int32_t *plan, const kvq_plan_info *info, int inverse_fwht,
                 uint16_t *out_bf16, float *out_f32, void *stream) {
    if (!workspace || !plan || !info || !out_bf16) return KVQ_EINVAL;
    if (!aligned16(workspace) || !aligned16(out_bf16) || (out_f32 && !aligned16(out_f32))) return KVQ_EALIGN;
    if (info->n_seq <= 0 || info->n_kv_heads <= 0 || info->group <= 0 || info->group > KVQ_MAX_GROUP ||
        info->n_units <= 0)
        return KVQ_EINVAL;
    return cuda_rc(launch_combine(workspace, plan, *info, inverse_fwht, out_bf16, out_f32,
                                  static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
