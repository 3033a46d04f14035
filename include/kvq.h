/*
 * kvq.h - C ABI of the quantized paged decode-attention library (B200, sm_100a).
 *
 * One decode step of a full-attention GQA layer over a long KV cache held in
 * 4-bit or 8-bit form:
 *
 *   q_rotate                      rotate the query by the same transform as K
 *   kv_append                     rotate, quantise and scatter the step's new K/V
 *   paged_decode_attn_{int8,q4_0,k8v4,fp8,nvfp4}
 *                                 split-K attention over the page table
 *   attn_combine                  merge the splits, un-rotate, write bf16 + f32
 *   paged_decode_step_{int8,q4_0,k8v4,fp8,nvfp4}
 *                                 all of the above for one layer in one launch
 *   paged_prefill_attn            causal attention of a prompt chunk over the cache
 *   kvq_resident_*                KV kept in pinned host memory behind a device
 *                                 page cache (residency table, CLOCK eviction)
 *
 * Sources (web pages, cited by title and section):
 *  [Strata] "KV 沉进内存、显存减半：Strata 让 12 GB 显卡跑满 262K 上下文"
 *           (hotelren.com news 6161890).  Section "4-bit KV 缓存：先旋转，再压到
 *           4-bit": Q, K and V pass through a 256-point Walsh-Hadamard rotation
 *           before 4-bit storage, scores are unchanged because <Hq,Hk> = <q,k>,
 *           the output is mixed over rotated V and multiplied by H again.
 *           Section "三种 KV 格式横向对比": formats int8 (default), q4_0 and k8v4
 *           (K 8-bit, V rotated then 4-bit).  Section "KV 从显存搬进内存之后发生了
 *           什么": KV in fixed pages addressed through a residency table.
 *  [Guide]  anozoder wiki "qwen38-27b-quant-vram-2026", section "一": the 27B
 *           full-attention shape (24 Q heads, 4 KV heads, head_dim 256, 16
 *           layers) and the KV-size formula; section "二": the q4_0 block size.
 *
 * Conventions (all entry points):
 *  - Every function returns KVQ_OK (0) or a negative KVQ_E* code and never
 *    throws.  Argument errors are detected on the host before any launch.
 *  - The caller owns every buffer.  The library never allocates device or host
 *    memory.  Device pointers must be 16-byte aligned (KVQ_EALIGN otherwise).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream); all device
 *    work is enqueued asynchronously on it.  KVQ_ECUDA reports a launch error
 *    (cudaGetLastError after the launch).
 *  - `status` (nullable, device int32) receives OR-ed KVQ_STATUS_* bits from
 *    kernels that detect bad data (a page-table entry outside the pool, a plan
 *    entry out of range, an internal wait that gave up).  Affected tokens are
 *    skipped; nothing faults.  The caller clears it.
 *  - head_dim and page_tokens are both 256.
 *  - Results are deterministic: the same inputs give the same output bits on
 *    every run (paged_decode_attn_cudacore, a control, excepted: its last bits
 *    may vary).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_OK 0
#define KVQ_EINVAL (-1)        /* bad argument value (null, range, shape) */
#define KVQ_EUNSUPPORTED (-2)  /* shape or format this build does not handle */
#define KVQ_EALIGN (-3)        /* a device pointer is not 16-byte aligned */
#define KVQ_ECUDA (-4)         /* a CUDA runtime call or launch failed */
#define KVQ_ESIZE (-5)         /* a caller buffer is smaller than required */

#define KVQ_STATUS_BAD_SLOT 1u   /* page-table entry outside [0, n_pages) */
#define KVQ_STATUS_BAD_PLAN 2u   /* plan entry inconsistent with the pool */
#define KVQ_STATUS_TIMEOUT 4u    /* a pipeline wait exceeded its time limit */

#define KVQ_HEAD_DIM 256
#define KVQ_PAGE_TOKENS 256
#define KVQ_MAX_GROUP 8          /* query heads per KV head handled by one CTA */

/* KV formats ([Strata] "三种 KV 格式横向对比"; [Roundup] section 一 for the
 * two floating-point formats and their 516 / 288 bytes per position):
 *  KVQ_INT8  K and V int8, one fp16 scale per 64 values, no rotation.
 *  KVQ_Q4_0  K and V rotated by H/16, then q4_0: one fp16 scale per 32 values,
 *            codes 0..15 stored as nibbles ([Guide] "二" q4_0 block).
 *  KVQ_K8V4  K int8 unrotated, V rotated then q4_0.
 *  KVQ_FP8   K and V as FP8 E4M3 codes with one fp16 scale per 256-vector,
 *            d = fp16(max|x| / 448), code = E4M3(x / d) (round to nearest
 *            even, saturating); no rotation.
 *  KVQ_NVFP4 K and V as FP4 E2M1 codes with one E4M3 scale per 16 values,
 *            s = E4M3(max|x| / 6), code = E2M1(x / s) (round to nearest even,
 *            saturating); no per-tensor scale; no rotation. */
typedef enum { KVQ_INT8 = 0, KVQ_Q4_0 = 1, KVQ_K8V4 = 2, KVQ_FP8 = 3, KVQ_NVFP4 = 4 } kvq_format;

typedef struct {
    int32_t n_layers;     /* layers stored in the pool */
    int32_t n_kv_heads;   /* KV heads per layer */
    int32_t n_q_heads;    /* query heads per layer; a multiple of n_kv_heads */
    int32_t head_dim;     /* must be 256 */
    int32_t page_tokens;  /* must be 256 */
    int32_t n_pages;      /* page slots per layer */
    int32_t fmt;          /* kvq_format */
} kvq_pool_desc;

typedef struct {
    void *base;           /* device memory of kvq_pool_bytes() bytes, caller-owned */
    kvq_pool_desc desc;
} kvq_pool;

/* Byte layout of the pool.  The pool is [layer][slot][kv_head] page blocks;
 * a page block is 32 tiles of 8 tokens; a tile holds, in this order, K codes,
 * K scales, V codes and V scales of its 8 tokens (offsets below).  Inside a
 * tile, codes and scales are arranged in the register-fragment order of the
 * attention kernel; the exact element order is documented with the kernels and
 * reproduced by the tests' layout decoder. */
typedef struct {
    int64_t tile_bytes;      /* bytes of one 8-token tile */
    int64_t k_codes_off;     /* offsets of the four sections inside a tile */
    int64_t k_scales_off;
    int64_t v_codes_off;
    int64_t v_scales_off;
    int64_t page_bytes;      /* one (layer, slot, kv head) block = 32 tiles */
    int64_t head_stride;     /* = page_bytes */
    int64_t slot_stride;     /* = n_kv_heads * page_bytes */
    int64_t layer_stride;    /* = n_pages * slot_stride */
    int64_t total_bytes;     /* = n_layers * layer_stride */
    int64_t bytes_per_token_head; /* algorithmic K+V bytes of one token of one KV head */
} kvq_layout;

/* Pool size and layout for a descriptor ([Guide] "一": KV bytes = 2 x layers x
 * KV heads x head_dim x bytes per element x context, here with the per-block
 * scales counted: 288 B (q4_0), 528 B (int8) and 408 B (k8v4) per token of one
 * KV head, so the 27B shape at 262,144 tokens in q4_0 needs the 4.8 GB the
 * guide quotes; [Strata] "KV 从显存搬进内存之后发生了什么": KV kept in fixed
 * pages reached through a table).  KVQ_EINVAL / KVQ_EUNSUPPORTED on a bad
 * descriptor.  Host only; no CUDA call. */
int kvq_pool_bytes(const kvq_pool_desc *desc, uint64_t *bytes);
int kvq_pool_layout(const kvq_pool_desc *desc, kvq_layout *out);

/* q_rotate: q_rot[i] = (H_256 / 16) q[i] for n_vec vectors of 256 fp32
 * ([Strata] "4-bit KV 缓存": Q takes the same rotation as K so that
 * <Hq, Hk> = <q, k>).  H is the Sylvester Hadamard matrix in natural order;
 * the transform is eight butterfly stages h = 1, 2, ..., 128 mapping
 * (x[i], x[i+h]) to (x[i] + x[i+h], x[i] - x[i+h]) in fp32 round-to-nearest
 * without fused multiply-add, then an exact multiply by 1/16, so the result is
 * bit-reproducible.  q and q_rot: device [n_vec][256] fp32, may alias.
 * n_vec == 0 is a no-op. */
int q_rotate(const float *q, float *q_rot, int64_t n_vec, void *stream);

/* kv_append: encode n_rows new tokens into the pool of one layer ([Strata]
 * "4-bit KV 缓存：先旋转，再压到 4-bit": K and V are rotated by the
 * Walsh-Hadamard transform, then stored as 4-bit codes with a scale per block;
 * [Guide] "二": the q4_0 block of 32 values; [Strata] "三种 KV 格式横向对比":
 * the int8 and k8v4 variants).
 *  k, v      device fp32 [n_rows][n_kv_heads][256]
 *  row_seq   device int32 [n_rows] sequence of each row, or NULL (row i -> seq i)
 *  row_pos   device int32 [n_rows] token position of each row in its sequence
 *  page_table device int32 [n_seq][max_pages]: slot of page p of sequence s
 * Per (row, kv head): rotate by H/16 where the format stores rotated data
 * (q4_0: K and V; k8v4: V), quantise per block with the fp16 scale rounded to
 * nearest and codes from round-half-even of a true division (q4_0: d =
 * signed-max/-8, code = clamp(rint(x/d)+8, 0, 15); int8: d = max|x|/127, code =
 * clamp(rint(x/d), -127, 127); a zero scale gives code 8 / 0), and store at
 * slot page_table[seq][pos/256], token pos%256.  Codes and scales are
 * bit-exact functions of the input.  A slot outside [0, n_pages) or a position
 * outside [0, max_pages*256) sets KVQ_STATUS_BAD_SLOT and skips the row.
 * Two rows writing the same (sequence, position) race. */
int kv_append(const kvq_pool *pool, int layer, const float *k, const float *v, int64_t n_rows,
              const int32_t *row_seq, const int32_t *row_pos, const int32_t *page_table,
              int max_pages, int n_seq, int32_t *status, void *stream);

/* kv_append_q_rotate: kv_append (arguments as there) and q_rotate of n_vec
 * query vectors (q -> q_rot, device [n_vec][256] fp32, may alias) in one kernel
 * launch.  The results are bit-identical to the two separate calls; the only
 * difference is one launch fewer per decode step.  Either part may be empty
 * (n_rows == 0 or n_vec == 0).  The pages have no such combined call: it
 * merges the two steps that precede the decode. */
int kv_append_q_rotate(const kvq_pool *pool, int layer, const float *k, const float *v, int64_t n_rows,
                       const int32_t *row_seq, const int32_t *row_pos, const int32_t *page_table,
                       int max_pages, int n_seq, const float *q, float *q_rot, int64_t n_vec,
                       int32_t *status, void *stream);

/* Split plan for a batch of sequences (host only).  A plan partitions every
 * (sequence, KV head) token range into work units of whole 64-token steps so
 * that the number of units does not exceed n_ctas (0 = one per SM of the
 * current device) and units are as even as possible; it also records, per
 * (sequence, KV head), the first unit.  seq_len: host int32 [n_seq], the
 * attended length of each sequence including this step's token, 1 <=
 * seq_len <= max_pages*256.  plan: host int32 array of plan_capacity entries,
 * filled with the plan (copy it to the device as is).  info receives the
 * sizes, including the workspace bytes the decode/combine pair needs.
 * KVQ_ESIZE if plan_capacity is too small (info->plan_len then holds the
 * needed length). */
typedef struct {
    int32_t n_units;        /* work units = CTAs of the decode launch */
    int32_t n_seq;
    int32_t n_kv_heads;
    int32_t group;          /* query heads per KV head */
    int32_t plan_len;       /* int32 entries used in the plan array */
    int32_t chunk_tokens;   /* largest unit, in tokens */
    uint64_t workspace_bytes;
} kvq_plan_info;

int kvq_decode_plan(const kvq_pool_desc *desc, int n_seq, const int32_t *seq_len, int max_pages, int n_ctas,
                    int32_t *plan, int plan_capacity, kvq_plan_info *info);

/* paged_decode_attn_<fmt>: per work unit of the plan, single-token attention
 * of the G query heads of one KV head over the unit's tokens, reading the
 * quantised codes through the page table and dequantising inside the score
 * and value loops ([Strata] "4-bit KV 缓存": scores on the rotated q and k,
 * values mixed in the rotated space).  Scores are q.k_hat/16 with k_hat =
 * (c-8)d (q4_0) or c d (int8); the softmax is online in fp32; all G heads of
 * a group share one read of each K/V tile.  Writes, per unit, the unnormalised
 * partial output and its running max and sum to the workspace.
 *  q          device fp32 [n_seq][n_q_heads][256]; for q4_0 the output of
 *             q_rotate, for the other formats the plain query
 *  page_table device int32 [n_seq][max_pages]
 *  plan       device copy of the kvq_decode_plan array; info its host info
 *             (an info whose workspace size differs from the one
 *             kvq_decode_plan computes for its own unit and group counts is
 *             rejected with KVQ_EINVAL)
 *  workspace  device, at least info->workspace_bytes; it ends with one int32
 *             arrival counter per (sequence, KV head) group that the
 *             *_combined entry points use: zero-fill the workspace once before
 *             its first use with them (every call leaves the counters at zero)
 * The pool's format must match the entry point (KVQ_EINVAL otherwise). */
int paged_decode_attn_int8(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                           int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                           uint64_t workspace_bytes, int32_t *status, void *stream);
int paged_decode_attn_q4_0(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                           int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                           uint64_t workspace_bytes, int32_t *status, void *stream);
int paged_decode_attn_k8v4(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                           int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                           uint64_t workspace_bytes, int32_t *status, void *stream);
int paged_decode_attn_fp8(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                          int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                          uint64_t workspace_bytes, int32_t *status, void *stream);
int paged_decode_attn_nvfp4(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                            int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                            uint64_t workspace_bytes, int32_t *status, void *stream);

/* paged_decode_attn_<fmt>_combined: the same decode with attn_combine fused
 * into it; out_bf16 / out_f32 are written exactly as attn_combine would (merge,
 * un-rotation for q4_0 and k8v4).  Saves the combine launch; otherwise the
 * same contract.  How the group merge runs:
 *  - When every CTA of the launch can be resident at once (info->n_units not
 *    above what the device holds; the default plan has one unit per SM), the
 *    launch is cooperative.  The CTAs of a (sequence, KV head) group count
 *    themselves in on the group's counter in the workspace and wait for one
 *    another (2 s limit; past it KVQ_STATUS_TIMEOUT and no output for the
 *    group).  CTA r of the group then merges heads r, r + n, ... of it.
 *  - Otherwise the last CTA of a group to finish, found with the same counter
 *    (no wait), merges the whole group.
 * Every call leaves the counters at zero, except after a TIMEOUT status: then
 * zero-fill them again.  Calls on the same workspace must not overlap on the
 * GPU. */
int paged_decode_attn_int8_combined(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                                    int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                                    uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32, int32_t *status,
                                    void *stream);
int paged_decode_attn_q4_0_combined(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                                    int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                                    uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32, int32_t *status,
                                    void *stream);
int paged_decode_attn_k8v4_combined(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                                    int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                                    uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32, int32_t *status,
                                    void *stream);
int paged_decode_attn_fp8_combined(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                                   int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                                   uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32, int32_t *status,
                                   void *stream);
int paged_decode_attn_nvfp4_combined(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                                     int max_pages, const int32_t *plan, const kvq_plan_info *info, float *workspace,
                                     uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32, int32_t *status,
                                     void *stream);

/* paged_decode_step_<fmt>: one whole decode step of one layer in a single
 * launch: kv_append of every sequence's newest token, q_rotate of the raw
 * query (q4_0; the other formats take the query as it is) and
 * paged_decode_attn_<fmt>_combined over the updated cache.  The results, pool
 * bytes and outputs, are bit-identical to those three calls.
 *  q         device fp32 [n_seq][n_q_heads][256], the raw query
 *  k_new, v_new device fp32 [n_seq][n_kv_heads][256]: the token at position
 *            seq_len - 1 of each sequence (seq_len as given to kvq_decode_plan)
 * The CTA whose unit ends each (sequence, KV head) range encodes that range's
 * token into the pool at its start, and writes the same codes into its copy of
 * the token's tile when the tile lands in shared memory (the copy may predate
 * the pool write); the pool bytes of the tile's other tokens are untouched.  A
 * page slot out of range sets KVQ_STATUS_BAD_SLOT as in kv_append.  Other
 * arguments, contract and errors as paged_decode_attn_<fmt>_combined.  The
 * pages describe the three steps separately; this entry only merges their
 * launches. */
int paged_decode_step_int8(const kvq_pool *pool, int layer, const float *q, const float *k_new, const float *v_new,
                           const int32_t *page_table, int max_pages, const int32_t *plan, const kvq_plan_info *info,
                           float *workspace, uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32,
                           int32_t *status, void *stream);
int paged_decode_step_q4_0(const kvq_pool *pool, int layer, const float *q, const float *k_new, const float *v_new,
                           const int32_t *page_table, int max_pages, const int32_t *plan, const kvq_plan_info *info,
                           float *workspace, uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32,
                           int32_t *status, void *stream);
int paged_decode_step_k8v4(const kvq_pool *pool, int layer, const float *q, const float *k_new, const float *v_new,
                           const int32_t *page_table, int max_pages, const int32_t *plan, const kvq_plan_info *info,
                           float *workspace, uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32,
                           int32_t *status, void *stream);
int paged_decode_step_fp8(const kvq_pool *pool, int layer, const float *q, const float *k_new, const float *v_new,
                          const int32_t *page_table, int max_pages, const int32_t *plan, const kvq_plan_info *info,
                          float *workspace, uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32,
                          int32_t *status, void *stream);
int paged_decode_step_nvfp4(const kvq_pool *pool, int layer, const float *q, const float *k_new, const float *v_new,
                            const int32_t *page_table, int max_pages, const int32_t *plan, const kvq_plan_info *info,
                            float *workspace, uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32,
                            int32_t *status, void *stream);

/* paged_decode_attn_q4_0_noalloc: paged_decode_attn_q4_0_combined without a
 * workspace argument, for callers that cannot allocate device memory.  Some
 * hosts own all device memory and pass a library only the buffers of the call
 * (a plugin interface of an inference server that forbids allocation while it
 * runs, to keep memory use fixed, is one); such a caller has nowhere to get the
 * split-K partial buffer from.  The pages have no counterpart to this entry
 * point; it is a deployment convenience.
 *  - Scratch: a file-scope device array of KVQ_NOALLOC_WS_BYTES inside the
 *    library, held by every GPU that loads the library until the process
 *    exits.  The plan's info->workspace_bytes must not exceed it (KVQ_ESIZE
 *    otherwise).
 *  - The first call on each device, with that device current, looks up the
 *    array's device address (cudaGetSymbolAddress) and keeps it; make that first
 *    call before any stream capture.
 *  - Allocates nothing: no cudaMalloc, no cudaFree.  Each call checks all of
 *    its arguments first (KVQ_E* and no device work on a bad one), then clears
 *    the group arrival counters in the array (cudaMemsetAsync on `stream`) and
 *    runs the decode.
 *  - All calls share the one array: calls that overlap on the GPU (on
 *    different streams, or from different threads) race and give wrong output.
 *    Serialise them.
 * Other arguments and results as paged_decode_attn_q4_0_combined. */
#define KVQ_NOALLOC_WS_BYTES (8u << 20)
int paged_decode_attn_q4_0_noalloc(const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                                   int max_pages, const int32_t *plan, const kvq_plan_info *info, uint16_t *out_bf16,
                                   float *out_f32, int32_t *status, void *stream);

/* The same computation on CUDA cores only (fp32 FMA, no tensor cores).  Kept
 * as the measured control for the tensor-core kernels above; fmt selects the
 * format (KVQ_INT8, KVQ_Q4_0 or KVQ_K8V4; KVQ_EUNSUPPORTED for KVQ_FP8 and
 * KVQ_NVFP4, which only the tensor-core path decodes). */
int paged_decode_attn_cudacore(int fmt, const kvq_pool *pool, int layer, const float *q,
                               const int32_t *page_table, int max_pages, const int32_t *plan,
                               const kvq_plan_info *info, float *workspace, uint64_t workspace_bytes,
                               int32_t *status, void *stream);

/* paged_prefill_attn: chunked-prefill attention over the quantised cache
 * ([Strata] "能力速览": reading a long prompt is the step before decoding;
 * "三种 KV 格式横向对比": prompt speed is part of each format's cost).  The
 * n_tok tokens of sequence seq at positions pos0 .. pos0 + n_tok - 1 must
 * already be in the pool (kv_append of the chunk; that call already takes
 * several tokens per sequence).  Each token i attends, per query head, over
 * the keys 0 .. pos0 + i of the sequence, dequantised from the pool, with the
 * same softmax scale and output (un-rotated for q4_0 and k8v4) as the decode.
 *  q        device fp32 [n_tok][n_q_heads][256], prepared as for
 *           paged_decode_attn (q_rotate'd for q4_0)
 *  page_table device int32 [n_seq][max_pages]; row seq is used
 *  out_bf16 device [n_tok][n_q_heads][256] bf16 (required); out_f32 the same
 *           in fp32 (optional)
 *  n_split  1: one pass over the keys, results written directly.  2 .. 8: the
 *           key range is cut into n_split parts (cuts at multiples of 64 tokens,
 *           all at or below pos0), each part runs as its own CTAs and writes an
 *           unnormalised partial to workspace, and a second kernel merges the
 *           parts with the log-sum-exp rule before the output rotation; this
 *           fills the GPU when the chunk alone gives too few CTAs.
 *  workspace device fp32, at least the kvq_prefill_split bytes for n_split
 *           (NULL when n_split is 1); caller-owned, needs no initialisation
 * Any pool format.  One CTA per 64 (token, head) rows of one KV head (and part)
 * reads that range of the sequence's keys once for all its rows.  KVQ_EINVAL /
 * KVQ_EALIGN on bad arguments (also an n_split with no valid cut), KVQ_ESIZE if
 * the workspace is too small; KVQ_STATUS_* in *status as for the decode. */
int paged_prefill_attn(const kvq_pool *pool, int layer, const float *q, int seq, int pos0, int n_tok,
                       const int32_t *page_table, int max_pages, int n_seq, int n_split, float *workspace,
                       uint64_t workspace_bytes, uint16_t *out_bf16, float *out_f32, int32_t *status, void *stream);

/* The key-range split paged_prefill_attn should use for a chunk of n_tok tokens
 * at pos0 on a GPU with n_sms multiprocessors (0: the 148 of a B200): the n_split
 * in 1 .. 8 whose CTA waves times longest part is smallest (the smaller on a
 * tie), and the workspace bytes it needs (0 for 1).  Host only; no CUDA call. */
int kvq_prefill_split(const kvq_pool_desc *desc, int pos0, int n_tok, int n_sms, int *n_split,
                      uint64_t *workspace_bytes);

/* attn_combine: for each (sequence, query head), merge the partials of its
 * units with the log-sum-exp rule (M = max m_j, L = sum l_j 2^(m_j - M),
 * o' = sum 2^(m_j - M) o_j / L), then, if inverse_fwht is non-zero (q4_0 and
 * k8v4: V was stored rotated), apply H/16 once more ([Strata] "4-bit KV 缓存":
 * H is its own inverse).  Writes out_bf16 (device uint16 bf16 bits
 * [n_seq][n_q_heads][256], round to nearest even) and, if non-NULL, out_f32
 * (device fp32, same shape). */
int attn_combine(const float *workspace, const int32_t *plan, const kvq_plan_info *info, int inverse_fwht,
                 uint16_t *out_bf16, float *out_f32, void *stream);

/* Host-resident KV with a device page cache ([Strata] "KV 从显存搬进内存之后发生了
 * 什么": the authoritative copy of the KV cache sits in pinned host memory, the
 * GPU holds only the pages attention is about to read, a residency table with
 * CLOCK (second chance) eviction chooses them, missing pages are pulled over the
 * bus without a staging copy, and attention runs unchanged on the cached pages,
 * so its output is bit-identical to attention over a fully resident pool).
 *
 * host pool : a kvq_pool whose base is pinned, device-mapped host memory
 *             (cudaHostAlloc / cudaMallocHost; under unified addressing the
 *             device reaches it directly).  kv_append writes it like any pool.
 * cache pool: a device kvq_pool with n_layers = 1 and the same format and
 *             heads; its n_pages are the cache slots.  A slot holds one page
 *             (every KV head) of any layer.
 * state     : caller-owned host memory of kvq_resident_state_bytes() bytes
 *             (header, one record per slot, and a residency table with one
 *             entry per (layer, host page)); the library allocates nothing.
 *
 * Per decode step and layer: kvq_resident_map (host only) turns the host page
 * table into a cache page table and a list of pages to load; kvq_resident_load
 * enqueues the page-in; kv_append writes the new token into both pools (the same
 * kernel on the same input writes the same bytes, so the cached page stays equal
 * to the host page); the attention entry points then take the cache pool, layer
 * 0 and the cache page table.  The state is not thread-safe. */
uint64_t kvq_resident_state_bytes(int n_layers, int n_host_pages, int n_cache_slots);

/* Initialise the state for a host pool and a cache pool (both stay owned by the
 * caller and must outlive the state).  Every slot starts empty.  KVQ_EINVAL on
 * mismatched descriptors or a cache pool with n_layers != 1, KVQ_ESIZE if
 * state_bytes is too small, KVQ_EALIGN if a base is not 16-byte aligned.
 * Host only; no CUDA call. */
int kvq_resident_init(void *state, uint64_t state_bytes, const kvq_pool *host_pool, const kvq_pool *cache_pool);

/* Make resident, for layer `layer`, every page the n_seq sequences read:
 * pages 0 .. ceil(seq_len[b] / 256) - 1 of row b of host_page_table (host int32
 * [n_seq][max_pages], host page indices).  Writes cache_page_table (host int32
 * [n_seq][max_pages], slot indices, -1 past each sequence's pages) and, in
 * loads (host int32 [loads_capacity][2]), the (host page, slot) pairs that
 * kvq_resident_load must copy, *n_loads of them.
 * Policy: the distinct pages of the call form its batch.  Resident pages of the
 * batch get their reference bit set and are pinned for the call.  Each missing
 * page, in order of first reference (sequence by sequence, page by page), takes
 * the slot the CLOCK hand finds: the hand skips pinned slots, clears a set
 * reference bit and moves on, and stops at the first unpinned slot with a clear
 * bit; the page evicted from it (if any) leaves the table, the new page takes
 * the slot with its bit set and pinned, and the hand moves one past it.
 * Statistics count one hit or miss per page reference.
 * KVQ_EINVAL on a bad argument (the state is unchanged); KVQ_ESIZE, with the
 * state unchanged, if the batch has more pages than the cache has slots or if
 * loads_capacity is below the number of missing pages (*n_loads then holds
 * that number; loads may be NULL with loads_capacity 0 to ask for it).
 * Host only; no CUDA call. */
int kvq_resident_map(void *state, int layer, const int32_t *host_page_table, int n_seq, int max_pages,
                     const int32_t *seq_len, int32_t *cache_page_table, int32_t *loads, int loads_capacity,
                     int *n_loads);

/* Enqueue on `stream` the copy of each listed page of layer `layer` from the
 * host pool into its cache slot: one kernel reads the pinned host memory
 * directly (zero-copy) and writes the slot.  loads is host memory, read before
 * the call returns (the list travels in the launch parameters, so the caller may
 * reuse the array at once).  The host pool must not be written between the
 * map and the completion of this copy except by stream-ordered work.
 * KVQ_EINVAL on a bad argument or a host pool that is not device-mapped host
 * memory; KVQ_ECUDA on a launch error. */
int kvq_resident_load(void *state, int layer, const int32_t *loads, int n_loads, void *stream);

/* The slot holding (layer, host_page), or -1 in *slot.  Host only. */
int kvq_resident_query(const void *state, int layer, int host_page, int *slot);

/* Hit, miss and eviction counts since init (any pointer may be NULL).  Host only. */
int kvq_resident_stats(const void *state, int64_t *hits, int64_t *misses, int64_t *evictions);

/* Library version string. */
const char *kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
