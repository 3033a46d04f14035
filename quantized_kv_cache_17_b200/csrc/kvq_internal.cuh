// Internal definitions shared by the CUDA translation units of the library:
// pool layout constants, plan layout, and small PTX wrappers (mbarrier, bulk
// copy, mma.sync, bounded waits).  Nothing here is part of the C ABI.
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "kvq.h"

namespace kvq {

constexpr int D = 256;            // head_dim
constexpr int PAGE = 256;         // tokens per page
constexpr int TILE = 8;           // tokens per tile
constexpr int TILES_PER_PAGE = PAGE / TILE;
constexpr int STEP_TOKENS = 64;   // granularity of the split plan (one pipeline stage)
constexpr int PLAN_HEADER = 8;
constexpr int PLAN_MAGIC = 0x4B565131;  // "KVQ1"
constexpr int WS_TAIL = 16;       // m[8], l[8] after o[G][256] in one workspace unit

// ---------------------------------------------------------------------------
// Pool layout.
//
// pool = [layer][slot][kv_head] page blocks; page block = 32 tiles of 8 tokens;
// tile = [K codes | K scales | V codes | V scales].  Four kinds of part:
//
//   Q4 part (q4_0):  codes 1024 B (8 tok x 256 x 4 bit), scales 128 B (8 tok x 8 fp16)
//   I8 part (int8):  codes 2048 B (8 tok x 256 x 8 bit), scales  64 B (8 tok x 4 fp16)
//   F8 part (E4M3):  codes 2048 B (8 tok x 256 x 8 bit), scales  16 B (8 tok x 1 fp16)
//   F4 part (E2M1):  codes 1024 B (8 tok x 256 x 4 bit), scales 128 B (8 tok x 16 E4M3)
//
// Formats: INT8 = (K I8, V I8); Q4_0 = (K Q4, V Q4); K8V4 = (K I8, V Q4);
// FP8 = (K F8, V F8); NVFP4 = (K F4, V F4).
//
// Code arrangement inside a tile (r = token in tile 0..7).  Each is the
// register-fragment order of mma.sync.m16n8k16 so that lane (g = lane/4,
// t = lane%4) finds its operands in 16-byte words at lane*16 of 512-byte rows:
//
//  K side, Q4: 32-bit word W(r, b, j) (block b = 32 dims, j 0..3) at
//      (b>>2)*512 + (r*4 + j)*16 + (b&3)*4; nibble n holds dim
//      32b + 8(n&3) + (n>>2) + 2j.
//  V side, Q4: word W(p, b, g) (token pair p: tokens 2p, 2p+1; g 0..7) at
//      (b>>2)*512 + (g*4 + p)*16 + (b&3)*4; nibble n holds token 2p + (n>>2),
//      dim 32b + g + 8(n&3).
//  K side, I8: word W(r, s, j) (k-step s = 16 dims) at
//      (s>>2)*512 + (r*4 + j)*16 + (s&3)*4; byte n holds dim 16s + 2j + {0,1,8,9}[n].
//  V side, I8: word W(p, m, g) (m-tile m = 16 dims) at
//      (m>>2)*512 + (g*4 + p)*16 + (m&3)*4; byte n holds token 2p + (n&1),
//      dim 16m + g + 8(n>>1).
//  F8 codes (one byte each) sit where I8 codes would: E4M3 bytes of dims
//      (2j, 2j+1) and (2j+8, 2j+9) of a k-step, or of tokens (2p, 2p+1) at one
//      dim, are adjacent, as one cvt.e4m3x2 converts them.
//  K side, F4: word W(r, b, j) where Q4 puts it; byte q holds the dims
//      (32b + 2j + 8q', +1) with q' = {0, 1, 2, 3}[q] -> {0, 8, 16, 24}: low
//      nibble the even dim, high nibble the odd one (one cvt.e2m1x2 per byte).
//  V side, F4: as Q4 (each token fills its own 16-bit half of a word, so two
//      tokens of a pair never share a byte and appends never overwrite each
//      other); the PV warp pairs the nibbles of tokens 2p, 2p+1 itself.
//  Scales: Q4 (fp16) token r, block b at (r>>1)*32 + b*4 + (r&1)*2;
//          I8 (fp16) token r, group q at (r>>1)*16 + q*4 + (r&1)*2;
//          F8 (fp16) token r at 2r;
//          F4 (E4M3) token r, block b (16 dims) at (r>>1)*32 + b*2 + (r&1).
// int8 codes are stored as two's complement bytes.
// ---------------------------------------------------------------------------
enum Part : int { PART_Q4 = 0, PART_I8 = 1, PART_F8 = 2, PART_F4 = 3 };

__host__ __device__ constexpr bool part_nibbles(int p) { return p == PART_Q4 || p == PART_F4; }
__host__ __device__ constexpr int part_code_bytes(int p) { return part_nibbles(p) ? 1024 : 2048; }
__host__ __device__ constexpr int part_scale_bytes(int p) {
    return p == PART_Q4 ? 128 : (p == PART_I8 ? 64 : (p == PART_F8 ? 16 : 128));
}

template <int FMT> struct Fmt;
template <> struct Fmt<KVQ_INT8> {
    static constexpr int KP = PART_I8, VP = PART_I8;
    static constexpr bool KROT = false, VROT = false;
};
template <> struct Fmt<KVQ_Q4_0> {
    static constexpr int KP = PART_Q4, VP = PART_Q4;
    static constexpr bool KROT = true, VROT = true;
};
template <> struct Fmt<KVQ_K8V4> {
    static constexpr int KP = PART_I8, VP = PART_Q4;
    static constexpr bool KROT = false, VROT = true;
};
template <> struct Fmt<KVQ_FP8> {
    static constexpr int KP = PART_F8, VP = PART_F8;
    static constexpr bool KROT = false, VROT = false;
};
template <> struct Fmt<KVQ_NVFP4> {
    static constexpr int KP = PART_F4, VP = PART_F4;
    static constexpr bool KROT = false, VROT = false;
};

template <int FMT> struct TileLayout {
    static constexpr int KP = Fmt<FMT>::KP, VP = Fmt<FMT>::VP;
    static constexpr int KC = 0;
    static constexpr int KS = KC + part_code_bytes(KP);
    static constexpr int VC = KS + part_scale_bytes(KP);
    static constexpr int VS = VC + part_code_bytes(VP);
    static constexpr int BYTES = VS + part_scale_bytes(VP);
    static constexpr int PAGE_BYTES = BYTES * TILES_PER_PAGE;
};

inline int host_part_k(int fmt) {
    return fmt == KVQ_Q4_0 ? PART_Q4 : (fmt == KVQ_FP8 ? PART_F8 : (fmt == KVQ_NVFP4 ? PART_F4 : PART_I8));
}
inline int host_part_v(int fmt) {
    return fmt == KVQ_INT8 ? PART_I8 : (fmt == KVQ_FP8 ? PART_F8 : (fmt == KVQ_NVFP4 ? PART_F4 : PART_Q4));
}
inline bool host_valid_format(int fmt) { return fmt >= KVQ_INT8 && fmt <= KVQ_NVFP4; }
inline bool host_rotated_v(int fmt) { return fmt == KVQ_Q4_0 || fmt == KVQ_K8V4; }

// ---------------------------------------------------------------------------
// FP8 E4M3 / FP4 E2M1 conversions (PTX cvt; round to nearest even, and
// saturating to the largest finite value on the way down).
// ---------------------------------------------------------------------------
// Two E4M3 bytes (low byte -> low half) as an exact fp16 pair.
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t v16) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "r"(v16));
    return r;
}
// Two E2M1 nibbles of one byte (low nibble -> low half) as an exact fp16 pair.
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t v8) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "r"(v8));
    return r;
}
// One value to E4M3 (the byte) / E2M1 (the nibble).
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(x));
    return r & 0xFFu;
}
__device__ __forceinline__ uint32_t f32_to_e2m1(float x) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %1;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(r) : "f"(x));
    return r & 0xFu;
}

struct PoolGeom {
    int64_t layer_stride, slot_stride, page_bytes;
    int n_pages, n_kv_heads;
};

// Launch with programmatic stream serialisation (and, with coop, as a
// cooperative launch: every block resident at once).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool coop,
                      Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (coop) {
        attr[n].id = cudaLaunchAttributeCooperative;
        attr[n].val.cooperative = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// Plan (int32): [magic, n_units, n_seq, n_kv_heads, group, chunk, 0, 0]
//               units[n_units][4] = {seq, kv_head, t_begin, t_end}
//               start[n_seq * n_kv_heads + 1]  (first unit of each (seq, kv head))
// ---------------------------------------------------------------------------
__host__ __device__ inline int plan_len_for(int n_units, int n_seq, int n_kv) {
    return PLAN_HEADER + 4 * n_units + n_seq * n_kv + 1;
}
__host__ __device__ inline int ws_unit_floats(int G) { return G * D + WS_TAIL; }
// Workspace = partials of every unit, then one int32 arrival counter per
// (sequence, KV head) group (used by the fused combine), padded to 16 bytes.
__host__ __device__ inline uint64_t ws_bytes_for(int n_units, int G, int n_groups) {
    return (uint64_t)n_units * ws_unit_floats(G) * 4 + (((uint64_t)n_groups * 4 + 15) & ~(uint64_t)15);
}

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that lets the hardware suspend the thread (up to hint_ns) until the
// phase completes, instead of returning at once: waiting warps do not spin.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Wait on an mbarrier phase with a time limit.  Returns false (and the caller
// records KVQ_STATUS_TIMEOUT) if the phase did not complete within limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// Programmatic dependent launch: every kernel of the library is launched with
// programmatic stream serialisation, so its launch overlaps the exit of the
// previous kernel in the stream; it then waits here, before reading anything
// that kernel may have written, until that kernel has completed and its writes
// are visible.  (No kernel signals early completion, so a dependent kernel
// starts only as the previous one's blocks exit.)  A no-op for a kernel
// launched without the attribute.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// 2^x on the special-function unit (inputs <= 0 here; -inf gives +0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier.
// src, dst 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint4 lds128(const void *p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ uint32_t lds32(const void *p) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));  // (a & b) | c
    return d;
}

// D = A * B + C, m16n8k16, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void status_or(int32_t *status, uint32_t bits) {
    if (status) atomicOr(reinterpret_cast<unsigned int *>(status), bits);
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
    return *reinterpret_cast<__half2 *>(&u);
}

// Host-side checks of a decode call (kvq_abi.cu): pool, format, shapes, plan
// info (its workspace size must be the one kvq_decode_plan computes) and the
// given workspace size; KVQ_OK or a KVQ_E* code, with geo filled on success.
int check_decode_args(int fmt, const kvq_pool *pool, int layer, const float *q, const int32_t *page_table,
                      int max_pages, const int32_t *plan, const kvq_plan_info *info, uint64_t workspace_bytes,
                      const uint16_t *out_bf16, const float *out_f32, PoolGeom *geo);

// Host launchers (defined in the .cu files).
cudaError_t launch_q_rotate(const float *q, float *q_rot, int64_t n_vec, cudaStream_t s);
cudaError_t launch_append(int fmt, uint8_t *pool, const PoolGeom &geo, int layer, const float *k,
                          const float *v, int64_t n_rows, const int32_t *row_seq, const int32_t *row_pos,
                          const int32_t *page_table, int max_pages, int n_seq, int32_t *status, cudaStream_t s);
cudaError_t launch_append_rotate(int fmt, uint8_t *pool, const PoolGeom &geo, int layer, const float *k,
                                 const float *v, int64_t n_rows, const int32_t *row_seq, const int32_t *row_pos,
                                 const int32_t *page_table, int max_pages, int n_seq, int32_t *status, const float *q,
                                 float *q_rot, int64_t n_vec, cudaStream_t s);
cudaError_t launch_prefill(int fmt, const uint8_t *pool, const PoolGeom &geo, int layer, const float *q, int seq,
                           int pos0, int n_tok, const int32_t *page_table, int max_pages, int n_q_heads,
                           int n_split, int split_tokens, float *ws, int inverse_fwht, uint16_t *out_bf16,
                           float *out_f32, int32_t *status, cudaStream_t s);

// Split prefill: floats per (part, KV head, row) partial: o[256], m, l, padding.
constexpr int PF_WS_STRIDE = 260;
constexpr int PF_MAX_SPLIT = 8;

// Length of every part but the last when the key range [0, pos0 + n_tok) of a
// prefill is cut into n_split parts: a multiple of 64 tokens (the copy step),
// about an equal share, and small enough that every cut lies at or below pos0
// (so each row of the chunk sees the first key of every part).  0 when no such
// cut exists.
inline int prefill_split_tokens(int pos0, int n_tok, int n_split) {
    if (n_split <= 1) return 0;
    const int64_t t_end = (int64_t)pos0 + n_tok;
    const int64_t share = (t_end + 64LL * n_split - 1) / (64LL * n_split) * 64;
    const int64_t cap = ((int64_t)(pos0 & ~63) / (n_split - 1)) & ~63LL;
    const int64_t st = share < cap ? share : cap;
    return st >= 64 ? (int)st : 0;
}
cudaError_t launch_decode(int fmt, bool tensor_cores, const uint8_t *pool, const PoolGeom &geo, int layer,
                          const float *q, const int32_t *page_table, int max_pages, const int32_t *plan,
                          const kvq_plan_info &info, float *ws, int32_t *status, int inverse_fwht,
                          uint16_t *out_bf16, float *out_f32, cudaStream_t s, const float *k_new = nullptr,
                          const float *v_new = nullptr);
cudaError_t launch_combine(const float *ws, const int32_t *plan, const kvq_plan_info &info, int inverse_fwht,
                           uint16_t *out_bf16, float *out_f32, cudaStream_t s);

}  // namespace kvq
