// paged_decode_attn_{int8,q4_0,k8v4}: split-K single-token attention over the
// quantised, paged KV cache, one CTA per work unit of the plan; attn_combine:
// the merge of a (sequence, KV head) group's partials, either as its own
// launch or fused into the decode (all CTAs of the group merging one head each
// under a cooperative launch, else the group's last CTA).
//
// [Strata] "4-bit KV 缓存：先旋转，再压到 4-bit": scores are taken on the rotated
// query and rotated keys (<Hq, Hk> = <q, k>), values are mixed in the rotated
// space and the merged output is rotated back (H/16 is its own inverse).
// [Guide] "一": 24 query heads share 4 KV heads (groups of 6), so every K/V
// tile read from HBM serves the whole group.
//
// Data path (both kernels): a copy warp streams the unit's tokens in 64-token
// steps (8 tiles, contiguous inside one page block) with 1-D bulk copies into
// a ring of shared-memory stages guarded by full/empty mbarriers.  At the end
// the CTA merges its warps' softmax states in shared memory and writes one
// partial (o[G][256] unnormalised, m[8], l[8]; scores in log2 units), then,
// with the combine fused in, takes part in the merge of its group.
//
// Tensor-core kernel (the product), warp-specialised:
//  - QK warps: the query of the group as mma.sync m16n8k16 A fragments in
//    registers (rows = [8 heads, fp16 hi | same 8 heads, fp16 lo], k = 16
//    dims), K codes as stored placed in fp16 words as B (cols = 8 tokens;
//    exact subnormals, the code offset removed by one m16n8k8 per tile), the
//    per-block K scale applied to the fp32 block sums; online softmax; hands
//    p (and the rescale factor of each head) to its PV warp through a 2-slot
//    shared-memory ring.
//  - PV warps: the output accumulators o[dims][heads] in registers; rows = 16
//    dims of V codes (exact in fp16), k = [8 tokens with P'hi | the same 8
//    tokens with P'lo], P' = p * dV formed as an exact fp16 pair.  The score
//    fragment layout of QK is exactly the P fragment layout PV needs.
//  - a scale warp converts each stage's fp16 K scales to fp32 once.
// Before the loop the QK warps stage the group's query through the (still
// unused) hand-over ring, one head per warp.
// paged_decode_step_*: the same kernel with the step enabled also rotates the
// raw query on its way into the ring, and in the CTA whose unit ends each
// (sequence, KV head) range the scale warp encodes the range's new token into
// the pool (as kv_append would) and writes its codes into the last stage when
// that lands.
// CUDA-core kernel (the measured control): the same computation with fp32
// FMAs only.
#include <mutex>
#include <type_traits>

#include "kvq_internal.cuh"
#include "kvq_append_dev.cuh"

namespace kvq {
namespace {

constexpr float QSCALE = 0.09016844005556021f;  // log2(e) / sqrt(256)
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr int COMBINE_MAX_UNITS = 256;            // units per group merged in one pass of the combine
constexpr int COMBINE_SMEM = 8 * D + 8 * COMBINE_MAX_UNITS + 24;   // floats of combine scratch

__device__ __forceinline__ __half2 q4_lo_pair(uint32_t w) {     // nibbles 0 / 4 of each half -> c - 8
    return __hsub2(u32_as_h2(lop3_and_or(w, 0x000F000Fu, 0x64006400u)), u32_as_h2(0x64086408u));
}
__device__ __forceinline__ __half2 q4_hi_pair(uint32_t w) {     // nibbles 1 / 5 -> c - 8
    return __hfma2(u32_as_h2(lop3_and_or(w, 0x00F000F0u, 0x64006400u)), u32_as_h2(0x2C002C00u),
                   u32_as_h2(0xD480D480u));
}
__device__ __forceinline__ __half2 i8_pair(uint32_t wb, uint32_t sel) {  // wb = codes ^ 0x80808080
    return __hsub2(u32_as_h2(__byte_perm(wb, 0x64646464u, sel)), u32_as_h2(0x64806480u));
}

// fp32 pair -> (hi, lo) fp16 pairs with hi + lo = x to ~22 bits.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    const __half2 h = __floats2half2_rn(x0, x1);
    const float2 hf = __half22float2(h);
    hi = h2_as_u32(h);
    lo = h2_as_u32(__floats2half2_rn(x0 - hf.x, x1 - hf.y));
}

// D = A * B (C = 0), A fragment from a 16-byte shared-memory word.
__device__ __forceinline__ void mma_z(float (&d)[4], const uint4 &a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1), "f"(0.f));
}
// D = A * B + D
__device__ __forceinline__ void mma_acc(float (&d)[4], const uint4 &a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}
// D = A * B (C = 0), m16n8k8: A = rows g / g+8, k 2t, 2t+1; B = k 2t, 2t+1 of column g.
__device__ __forceinline__ void mma_k8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%7,%7,%7,%7};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(b0), "f"(0.f));
}
__device__ __forceinline__ uint32_t u4_at(const uint4 &v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}
__device__ __forceinline__ float4 lds128f(const float *p) {
    const uint4 v = lds128(p);
    return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w));
}
// (v0, v1) = 8 floats; pair i = floats 2i, 2i+1
__device__ __forceinline__ float2 f2_at(const float4 &v0, const float4 &v1, int i) {
    return i == 0 ? make_float2(v0.x, v0.y)
                  : (i == 1 ? make_float2(v0.z, v0.w) : (i == 2 ? make_float2(v1.x, v1.y) : make_float2(v1.z, v1.w)));
}
__device__ __forceinline__ uint2 lds64(const void *p) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_u32(p)));
    return v;
}
__device__ __forceinline__ void sts128(void *p, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(smem_u32(p)), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Warpgroup register budgets (every warp of the warpgroup executes the same
// instruction; .inc waits until .dec has returned enough registers).
template <int N> __device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N> __device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------------------
// Tensor-core kernel: configuration
// ---------------------------------------------------------------------------
// Warp roles, in warpgroups of four: NQK QK warps, NQK PV warps, then one
// producer warpgroup: the copy warp and N_SCALE scale warps.  Each SM
// sub-partition (warp index mod 4) then holds two pairs and one producer; the
// scale work is split by ring slot so that no sub-partition carries all of it
// (a sub-partition whose producer did all the conversions ran its pairs about
// a quarter slower, and every pair waits for the slowest through the ring).  The
// launch gives every thread REG_LAUNCH registers; at the start the producer
// warpgroup gives registers back (setmaxnreg.dec) and the QK and PV
// warpgroups take them (setmaxnreg.inc), so that eight pairs fit on the SM:
// two per SM sub-partition, where seven pairs loaded two of the four with an
// extra pair's work.
template <int FMT> struct TcCfg {
    using L = TileLayout<FMT>;
    static constexpr int NQK = 8;
    static constexpr int COPY_WARP = 2 * NQK;
    static constexpr int SCALE_WARP = 2 * NQK + 1;               // the first of N_SCALE
    static constexpr int N_SCALE = 3;
    static constexpr int NTHREADS = (2 * NQK + 4) * 32;
    static constexpr int REG_LAUNCH = 65536 / NTHREADS / 8 * 8;     // 96
    static constexpr int REG_COMPUTE = 112, REG_PROD = 32;
    static_assert(NQK % 4 == 0, "QK and PV warps fill whole warpgroups");
    // the warpgroups' budgets after the split add up to what the launch holds
    static_assert(2 * NQK * REG_COMPUTE + 4 * REG_PROD <= NTHREADS / 32 * REG_LAUNCH,
                  "register split exceeds the launch's registers");
    static_assert(SCALE_WARP + N_SCALE == NTHREADS / 32, "producer warpgroup: copy warp + scale warps");
    // tiles per work item (measured best for int8 and q4_0; the 8-bit fp8 tiles follow int8)
    static constexpr int TPI = (FMT == KVQ_INT8 || FMT == KVQ_FP8) ? 2 : 4;
    static constexpr int ITEMS_PER_STAGE = 8 / TPI;
    static constexpr int STAGE_BYTES = 8 * L::BYTES;
    static constexpr int NS = (FMT == KVQ_Q4_0 || FMT == KVQ_NVFP4) ? 8 : ((FMT == KVQ_INT8 || FMT == KVQ_FP8) ? 5 : 6);
    static constexpr int DP = 2;                                // slots of each QK -> PV ring
    // fp32 K scales of a stage: per tile, token pair t at float t*KSTRIDE (block
    // or group j of tokens 2t, 2t+1 at 2j, 2j+1); the stride pads rows so the
    // four pairs fall into different banks
    static constexpr int KSTRIDE = L::KP == PART_Q4 ? 20 : (L::KP == PART_I8 ? 12 : (L::KP == PART_F8 ? 2 : 36));
    static constexpr int SF_TILE = 4 * KSTRIDE;                 // floats
    static constexpr int SF_STAGE_BYTES = 8 * SF_TILE * 4;
    static constexpr int PA = 32 * 2 * TPI;                     // alpha[8] in a slot, after p of 32 lanes x 2 TPI
    static constexpr int PSLOT = PA + 16;                       // floats: p, alpha[8], item
    static constexpr int PITEM = PA + 8;                        // the item index (int) in a slot
    static constexpr int OSTRIDE = D + 4;                       // row stride of the PV warps' o buffers
    static constexpr int RING = NS * STAGE_BYTES;
    static constexpr int OBUF = NQK * 8 * OSTRIDE + 2 * NQK * 8;   // floats of the CTA merge
    static constexpr int MERGE = (COMBINE_SMEM > OBUF ? COMBINE_SMEM : OBUF) * 4;
    static constexpr int DATA = RING > MERGE ? RING : MERGE;
    static constexpr int SFOFF = (DATA + 127) & ~127;
    static constexpr int POFF = SFOFF + NS * SF_STAGE_BYTES;
    // the QK -> PV rings; before the loop, the group's query (KVQ_MAX_GROUP heads)
    static constexpr int PRING_FLOATS = NQK * DP * PSLOT > KVQ_MAX_GROUP * D ? NQK * DP * PSLOT : KVQ_MAX_GROUP * D;
    // the group's query as MMA A fragments: [16 k-steps][32 lanes] x 16 bytes
    static constexpr int QOFF = POFF + PRING_FLOATS * 4;
    static constexpr int BAR_OFF = QOFF + 16 * 32 * 16;
    // full, ready, empty [NS]; p_full, p_empty [NQK * DP]; stage_ok [NS]; then,
    // for a decode step, the newest token's codes and scales (5 words per lane)
    static constexpr int TKV_OFF = (BAR_OFF + (3 * NS + 2 * NQK * DP) * 8 + NS * 4 + 15) & ~15;
    static constexpr int TOTAL = TKV_OFF + 32 * 5 * 4;
    static_assert(TOTAL <= 227 * 1024, "shared memory budget");
    // A QK warp waits on the ready barrier of the stage of its next item, which
    // lies (NQK items later) at most this many stages ahead of its last one; a
    // wait more than one lap of the ring ahead of the barrier's pending phase
    // would be satisfied by an older phase of the same parity.
    static_assert((NQK + ITEMS_PER_STAGE - 1) / ITEMS_PER_STAGE < NS, "QK item stride must stay within one ring lap");
};

// Scores are formed from the codes as stored (q4_0 nibbles 0..15, int8 codes
// + 128 as 0..255) placed directly in the low bits of fp16 words: as fp16
// subnormals they are the exact values code * 2^-24 (or 16 code * 2^-24 for a
// nibble in bits 4-7), so unpacking costs one AND per two values and no
// subtraction.  The constant offset (8 or 128) is removed by one extra small
// MMA per tile: -OFF * sum_b dK[t][b] * Q[b], Q[b] = the query's sum over block
// b.  Two power-of-two scales keep every fp16 operand in its normal range: the
// query fragments carry 2^kq (kq puts the group's largest |q| in [2^12, 2^13)),
// and scores are produced in units of 2^kb, kb = kq - KBS, removed inside the
// softmax.  The fp32 K scales are therefore stored multiplied by 2^(24 - KBS).
template <int FMT> struct QkCodes {
    static constexpr bool Q4 = TileLayout<FMT>::KP == PART_Q4;
    // fp8 / fp4 keys convert to exact fp16 values: no offset, no 2^-24 units
    static constexpr bool FP = TileLayout<FMT>::KP == PART_F8 || TileLayout<FMT>::KP == PART_F4;
    static constexpr float OFF = Q4 ? 8.f : 128.f;
    static constexpr int KBS = FP ? 0 : (Q4 ? 6 : 11);
    static constexpr float KSF = FP ? 1.f : (Q4 ? 262144.f : 8192.f);     // 2^(24 - KBS)
};

// Scale warp: convert the K scales of one stage (8 tiles) to fp32 rows (times
// 2^(24 - KBS) for the 4/8-bit integer codes).  fp8: one fp16 per token, row
// of pair t = (d[2t], d[2t+1]); nvfp4: 16 E4M3 per token, row of pair t =
// (d[2t][b], d[2t+1][b]) for b = 0..15.
template <int FMT>
__device__ __forceinline__ void convert_stage_scales(const uint8_t *stage, float *sf, int lane) {
    using L = TileLayout<FMT>;
    if constexpr (L::KP == PART_F8) {
        const int tile = lane >> 2, pair = lane & 3;
        const uint32_t w = *reinterpret_cast<const uint32_t *>(stage + tile * L::BYTES + L::KS + pair * 4);
        const float2 d = __half22float2(u32_as_h2(w));
        *reinterpret_cast<float2 *>(sf + tile * TcCfg<FMT>::SF_TILE + pair * TcCfg<FMT>::KSTRIDE) = d;
        return;
    } else if constexpr (L::KP == PART_F4) {
        // lane: tile lane / 4, tokens 2 (lane % 4) and 2 (lane % 4) + 1; word 16 r + b of
        // the tile's row = the scale of token r, block b as the fp16 pair (s, s)
        const int tile = lane >> 2, pair = lane & 3;
        uint32_t *dst = reinterpret_cast<uint32_t *>(sf) + tile * TcCfg<FMT>::SF_TILE + 32 * pair;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint4 h = lds128(stage + tile * L::BYTES + L::KS + pair * 32 + half * 16);
            uint32_t ev[8], od[8];                          // blocks 8 half .. 8 half + 7
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t w = u4_at(h, i);             // bytes: (b, even), (b, odd), (b + 1, even), (b + 1, odd)
                const uint32_t x = e4m3x2_to_h2(w), y = e4m3x2_to_h2(w >> 16);
                ev[2 * i] = __byte_perm(x, 0, 0x1010);
                od[2 * i] = __byte_perm(x, 0, 0x3232);
                ev[2 * i + 1] = __byte_perm(y, 0, 0x1010);
                od[2 * i + 1] = __byte_perm(y, 0, 0x3232);
            }
            sts128(dst + 8 * half, make_uint4(ev[0], ev[1], ev[2], ev[3]));
            sts128(dst + 8 * half + 4, make_uint4(ev[4], ev[5], ev[6], ev[7]));
            sts128(dst + 16 + 8 * half, make_uint4(od[0], od[1], od[2], od[3]));
            sts128(dst + 16 + 8 * half + 4, make_uint4(od[4], od[5], od[6], od[7]));
        }
        return;
    }
    constexpr int KSB = part_scale_bytes(L::KP);        // fp16 bytes per tile: 4 token pairs
    constexpr int PAIR_B = KSB / 4;                     // 32 (q4) or 16 (i8) bytes per pair
    constexpr int KSTRIDE = TcCfg<FMT>::KSTRIDE;
    constexpr int CPT = KSB / 16;                       // 16-byte chunks per tile
    constexpr float F = QkCodes<FMT>::KSF;
    for (int c = lane; c < 8 * CPT; c += 32) {
        const int tile = c / CPT, o = (c % CPT) * 16;
        const int pair = o / PAIR_B, within = (o % PAIR_B) / 2;
        const uint4 h = lds128(stage + tile * L::BYTES + L::KS + o);
        float *dst = sf + tile * 4 * KSTRIDE + pair * KSTRIDE + within;
        const float2 a = __half22float2(u32_as_h2(h.x)), b = __half22float2(u32_as_h2(h.y));
        const float2 cc = __half22float2(u32_as_h2(h.z)), d = __half22float2(u32_as_h2(h.w));
        sts128(dst, make_uint4(__float_as_uint(a.x * F), __float_as_uint(a.y * F), __float_as_uint(b.x * F),
                               __float_as_uint(b.y * F)));
        sts128(dst + 4, make_uint4(__float_as_uint(cc.x * F), __float_as_uint(cc.y * F), __float_as_uint(d.x * F),
                                   __float_as_uint(d.y * F)));
    }
}

// ---------------------------------------------------------------------------
// QK warp: scores and online softmax for one work item (tiles A, B = 16 tokens)
// ---------------------------------------------------------------------------
// The PV warp multiplies p by the fp16 V scale in fp16 arithmetic (an exact
// hi/lo pair, see PvWarp::pscale), so p dV must stay in fp16's normal range
// even when every V scale of a sequence is tiny (down to subnormal).  The QK
// warp therefore hands over p' = p 2^sigma instead of p, with sigma a power of
// two set from e, the largest biased fp16 exponent of the V scales its items
// have held so far: sigma = min(15, 29 - max(e, 1)) keeps p' and p' dV below
// 2^14 (p <= 1/2), and the weights of the largest-scale tokens get the pair's
// full precision.  sigma only enters the softmax reference point: the warp
// keeps m' = m - sigma as its running max, so its l and o carry 2^sigma and
// every merge (rescale on a new max, CTA merge, split-K combine) cancels it
// like any other shift of the reference.  e only grows, so m' never falls.
__device__ __forceinline__ int pv_sigma(int e) { return min(15, 29 - (e > 1 ? e : 1)); }

// The largest |V scale| of the TPI tiles at tp, as fp16 bits (warp-uniform).
// fp16 (and E4M3) magnitudes order as integers.  Tokens past the sequence end
// count too (their bytes are stale or zero): that can only lower sigma, never
// overflow.
template <int FMT> __device__ __forceinline__ uint32_t item_v_scale_max(const uint8_t *tp, int lane) {
    using L = TileLayout<FMT>;
    if constexpr (L::VP == PART_F8) {                         // one fp16 per token: TPI x 8 of them
        const uint32_t m = lane < 8 * TcCfg<FMT>::TPI
                               ? *reinterpret_cast<const uint16_t *>(tp + (lane >> 3) * L::BYTES + L::VS + (lane & 7) * 2) &
                                     0x7FFFu
                               : 0u;
        return __reduce_max_sync(0xffffffffu, m);
    } else if constexpr (L::VP == PART_F4) {                  // E4M3 bytes, 16 per lane
        static_assert(TcCfg<FMT>::TPI == 4, "nvfp4: four tiles per item");
        const uint4 h = lds128(tp + (lane >> 3) * L::BYTES + L::VS + (lane & 7) * 16);
        uint32_t m = __vmaxu4(__vmaxu4(h.x & 0x7F7F7F7Fu, h.y & 0x7F7F7F7Fu), __vmaxu4(h.z & 0x7F7F7F7Fu, h.w & 0x7F7F7F7Fu));
        m = max(max(m & 0xFFu, (m >> 8) & 0xFFu), max((m >> 16) & 0xFFu, m >> 24));
        m = __reduce_max_sync(0xffffffffu, m);
        return e4m3x2_to_h2(m) & 0xFFFFu;                      // its fp16 bits (exact)
    } else {
        constexpr int VSB = part_scale_bytes(L::VP);          // bytes per tile
        constexpr int PER_LANE = TcCfg<FMT>::TPI * VSB / 32;  // 16 (q4) or 4 (int8) bytes
        constexpr int LPT = VSB / PER_LANE;                   // lanes per tile
        const uint8_t *src = tp + (lane / LPT) * L::BYTES + L::VS + (lane % LPT) * PER_LANE;
        uint32_t m;
        if constexpr (PER_LANE == 16) {
            const uint4 h = lds128(src);
            m = __vmaxu2(__vmaxu2(h.x & 0x7FFF7FFFu, h.y & 0x7FFF7FFFu), __vmaxu2(h.z & 0x7FFF7FFFu, h.w & 0x7FFF7FFFu));
        } else {
            static_assert(PER_LANE == 4, "V scale bytes per lane");
            m = *reinterpret_cast<const uint32_t *>(src) & 0x7FFF7FFFu;
        }
        return __reduce_max_sync(0xffffffffu, max(m & 0xFFFFu, m >> 16));
    }
}

template <int FMT> struct QkWarp {
    using L = TileLayout<FMT>;
    using C = TcCfg<FMT>;
    using K = QkCodes<FMT>;
    const uint8_t *qf;     // A fragments of the 16 k-steps (scaled by 2^kq), shared by the QK warps
    uint32_t qb_hi, qb_lo; // A fragment of the offset MMA: -OFF 2^-KBS Q[2t], Q[2t+1] of head g, hi / lo rows
    float inv_sb;          // 2^-kb
    float m_run, l_run;    // head g (the four lanes of a group agree)
    float sg;              // sigma of the hand-over weights (warp-uniform); m_run is m - sigma
    uint32_t vmax;         // largest |V scale| (fp16 bits) of the items seen

    // Fragments of head g (rows g: fp16 hi, g+8: fp16 lo), k-step ks: dims
    // 16ks + 2t, +1 (x, y) and 16ks + 2t + 8, +9 (z, w).  For 4-bit keys the
    // second pair is divided by 16, matching its codes' 16 code * 2^-24.
    __device__ __forceinline__ uint4 qa(int ks, int lane) const { return lds128(qf + (ks * 32 + lane) * 16); }

    // Every QK warp computes the fragments (and its own offset fragment);
    // `writer` stores them to q_frag.  qrow: the query vector of this lane's
    // row g = lane / 4 (read only when row_ok; otherwise the row is zero).
    __device__ __forceinline__ void init(const float *qrow, bool row_ok, int lane, uint8_t *q_frag, bool writer) {
        const int t = lane & 3;
        qf = q_frag;
        float mx = 0.f;
        if (row_ok) {
#pragma unroll
            for (int ks = 0; ks < 16; ++ks) {
                const float *p = qrow + 16 * ks + 2 * t;
                mx = fmaxf(mx, fmaxf(fmaxf(fabsf(p[0] * QSCALE), fabsf(p[1] * QSCALE)),
                                     fmaxf(fabsf(p[8] * QSCALE), fabsf(p[9] * QSCALE))));
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int kq = 0;
        if (mx > 0.f) kq = min(max(12 - ((int)((__float_as_uint(mx) >> 23) & 255u) - 127), -60), 60);
        const float s_lo = __int_as_float((127 + kq) << 23);
        const float s_hi = K::Q4 ? __int_as_float((127 + kq - 4) << 23) : s_lo;
        constexpr float M_HI = K::Q4 ? 16.f : 1.f;
        float S[8];            // sum of the represented query over block b (units 2^kq)
#pragma unroll
        for (int b = 0; b < 8; ++b) S[b] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 16; ++ks) {
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            if (row_ok) {
                const float *p = qrow + 16 * ks + 2 * t;
                x[0] = (p[0] * QSCALE) * s_lo; x[1] = (p[1] * QSCALE) * s_lo;
                x[2] = (p[8] * QSCALE) * s_hi; x[3] = (p[9] * QSCALE) * s_hi;
            }
            uint4 f;
            split_pair(x[0], x[1], f.x, f.y);
            split_pair(x[2], x[3], f.z, f.w);
            if (writer) sts128(q_frag + (ks * 32 + lane) * 16, f);
            const float2 h0 = __half22float2(u32_as_h2(f.x)), l0 = __half22float2(u32_as_h2(f.y));
            const float2 h1 = __half22float2(u32_as_h2(f.z)), l1 = __half22float2(u32_as_h2(f.w));
            const float r = ((h0.x + l0.x) + (h0.y + l0.y)) + M_HI * ((h1.x + l1.x) + (h1.y + l1.y));
            S[K::Q4 ? ks >> 1 : ks >> 2] += r;
        }
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            S[b] += __shfl_xor_sync(0xffffffffu, S[b], 1);
            S[b] += __shfl_xor_sync(0xffffffffu, S[b], 2);
        }
        constexpr float CA = -K::OFF / (float)(1 << K::KBS);
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int b = 0; b < 8; b += 2)
            if (b == 2 * t && !K::FP && (K::Q4 || b < 4)) {
                a0 = CA * S[b];
                a1 = CA * S[b + 1];
            }
        split_pair(a0, a1, qb_hi, qb_lo);
        inv_sb = __int_as_float((127 - (kq - K::KBS)) << 23);
        m_run = -INFINITY;
        l_run = 0.f;
        sg = 0.f;
        vmax = 0u;
    }

    // B fragment of the offset MMA for one tile: fp16 K scales of token g,
    // blocks (groups) 2t, 2t+1; zero for the missing groups of int8 keys.
    __device__ __forceinline__ static uint32_t kscale_frag(const uint8_t *tp, int lane) {
        const int g = lane >> 2, t = lane & 3;
        if constexpr (K::Q4) {
            const uint2 w = lds64(tp + L::KS + (g >> 1) * 32 + 8 * t);
            return __byte_perm(w.x, w.y, (g & 1) ? 0x7632u : 0x5410u);
        } else {
            const uint2 w = lds64(tp + L::KS + (g >> 1) * 16 + 8 * (t & 1));
            return t < 2 ? __byte_perm(w.x, w.y, (g & 1) ? 0x7632u : 0x5410u) : 0u;
        }
    }

    // S[head g][tokens 2t, 2t+1] of tiles A (s[0], s[1]) and B (s[2], s[3]), in
    // units of 2^kb.
    __device__ __forceinline__ void scores(const uint8_t *tA, const float *fA, int lane, float (&s)[4]) const {
        const uint8_t *tB = tA + L::BYTES;
        const float *fB = fA + C::SF_TILE;
        const int t = lane & 3;
        if constexpr (L::KP == PART_F8) {
            // E4M3 keys: the 16 k-steps accumulate in two chains per tile; the
            // token's one scale multiplies the sum
            float a[2][4], c[2][4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 kA = lds128(tA + L::KC + q * 512 + lane * 16);
                const uint4 kB = lds128(tB + L::KC + q * 512 + lane * 16);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t wA = u4_at(kA, j), wB = u4_at(kB, j);
                    const uint4 qj = qa(4 * q + j, lane);
                    float(&ra)[4] = a[q & 1];
                    float(&rc)[4] = c[q & 1];
                    if (q < 2 && j == 0) {
                        mma_z(ra, qj, e4m3x2_to_h2(wA), e4m3x2_to_h2(wA >> 16));
                        mma_z(rc, qj, e4m3x2_to_h2(wB), e4m3x2_to_h2(wB >> 16));
                    } else {
                        mma_acc(ra, qj, e4m3x2_to_h2(wA), e4m3x2_to_h2(wA >> 16));
                        mma_acc(rc, qj, e4m3x2_to_h2(wB), e4m3x2_to_h2(wB >> 16));
                    }
                }
            }
            const float2 dA = *reinterpret_cast<const float2 *>(fA + t * C::KSTRIDE);
            const float2 dB = *reinterpret_cast<const float2 *>(fB + t * C::KSTRIDE);
            s[0] = ((a[0][0] + a[0][2]) + (a[1][0] + a[1][2])) * dA.x;
            s[1] = ((a[0][1] + a[0][3]) + (a[1][1] + a[1][3])) * dA.y;
            s[2] = ((c[0][0] + c[0][2]) + (c[1][0] + c[1][2])) * dB.x;
            s[3] = ((c[0][1] + c[0][3]) + (c[1][1] + c[1][3])) * dB.y;
            return;
        } else if constexpr (L::KP == PART_F4) {
            // E2M1 keys: a value times its E4M3 scale has at most 6 significant
            // bits and lies in [2^-10, 2688], so the fp16 product is the exact key
            // and the 16 k-steps of a tile accumulate in one product (two chains)
            const int g = lane >> 2;
            const uint32_t *sfA = reinterpret_cast<const uint32_t *>(fA) + 16 * g;     // token g's 16 scale pairs
            const uint32_t *sfB = reinterpret_cast<const uint32_t *>(fB) + 16 * g;
            float a[2][4], c[2][4];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint4 kA = lds128(tA + L::KC + hf * 512 + lane * 16);
                const uint4 kB = lds128(tB + L::KC + hf * 512 + lane * 16);
                const uint4 sA0 = lds128(sfA + 8 * hf), sA1 = lds128(sfA + 8 * hf + 4);
                const uint4 sB0 = lds128(sfB + 8 * hf), sB1 = lds128(sfB + 8 * hf + 4);
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) {
                    const int b = 4 * hf + bb;              // 32 dims: k-steps 2b, 2b + 1
                    const uint32_t wA = u4_at(kA, bb), wB = u4_at(kB, bb);
                    const uint32_t xA0 = u4_at(bb < 2 ? sA0 : sA1, (2 * bb) & 3), xA1 = u4_at(bb < 2 ? sA0 : sA1, (2 * bb + 1) & 3);
                    const uint32_t xB0 = u4_at(bb < 2 ? sB0 : sB1, (2 * bb) & 3), xB1 = u4_at(bb < 2 ? sB0 : sB1, (2 * bb + 1) & 3);
                    const uint4 q0 = qa(2 * b, lane), q1 = qa(2 * b + 1, lane);
                    float(&ra)[4] = a[b & 1];
                    float(&rc)[4] = c[b & 1];
                    const uint32_t kA0 = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2(wA)), u32_as_h2(xA0)));
                    const uint32_t kA1 = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2(wA >> 8)), u32_as_h2(xA0)));
                    const uint32_t kA2 = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2(wA >> 16)), u32_as_h2(xA1)));
                    const uint32_t kA3 = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2(wA >> 24)), u32_as_h2(xA1)));
                    const uint32_t kB0 = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2(wB)), u32_as_h2(xB0)));
                    const uint32_t kB1 = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2(wB >> 8)), u32_as_h2(xB0)));
                    const uint32_t kB2 = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2(wB >> 16)), u32_as_h2(xB1)));
                    const uint32_t kB3 = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2(wB >> 24)), u32_as_h2(xB1)));
                    if (b < 2) {
                        mma_z(ra, q0, kA0, kA1);
                        mma_z(rc, q0, kB0, kB1);
                    } else {
                        mma_acc(ra, q0, kA0, kA1);
                        mma_acc(rc, q0, kB0, kB1);
                    }
                    mma_acc(ra, q1, kA2, kA3);
                    mma_acc(rc, q1, kB2, kB3);
                }
            }
            s[0] = (a[0][0] + a[0][2]) + (a[1][0] + a[1][2]);
            s[1] = (a[0][1] + a[0][3]) + (a[1][1] + a[1][3]);
            s[2] = (c[0][0] + c[0][2]) + (c[1][0] + c[1][2]);
            s[3] = (c[0][1] + c[0][3]) + (c[1][1] + c[1][3]);
            return;
        }
        {
            float ca[4], cb[4];
            mma_k8(ca, qb_hi, qb_lo, kscale_frag(tA, lane));
            mma_k8(cb, qb_hi, qb_lo, kscale_frag(tB, lane));
            s[0] = ca[0] + ca[2];
            s[1] = ca[1] + ca[3];
            s[2] = cb[0] + cb[2];
            s[3] = cb[1] + cb[3];
        }
        if constexpr (K::Q4) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint4 kA = lds128(tA + L::KC + hf * 512 + lane * 16);
                const uint4 kB = lds128(tB + L::KC + hf * 512 + lane * 16);
                const float4 dA0 = lds128f(fA + t * C::KSTRIDE + 8 * hf), dA1 = lds128f(fA + t * C::KSTRIDE + 8 * hf + 4);
                const float4 dB0 = lds128f(fB + t * C::KSTRIDE + 8 * hf), dB1 = lds128f(fB + t * C::KSTRIDE + 8 * hf + 4);
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) {
                    const int b = 4 * hf + bb;
                    const uint32_t wA = u4_at(kA, bb), wB = u4_at(kB, bb);
                    const uint32_t wA2 = wA >> 8, wB2 = wB >> 8;
                    float a[4], c[4];
                    const uint4 q0 = qa(2 * b, lane), q1 = qa(2 * b + 1, lane);
                    mma_z(a, q0, wA & 0x000F000Fu, wA & 0x00F000F0u);
                    mma_z(c, q0, wB & 0x000F000Fu, wB & 0x00F000F0u);
                    mma_acc(a, q1, wA2 & 0x000F000Fu, wA2 & 0x00F000F0u);
                    mma_acc(c, q1, wB2 & 0x000F000Fu, wB2 & 0x00F000F0u);
                    const float2 da = f2_at(dA0, dA1, bb), db = f2_at(dB0, dB1, bb);
                    s[0] = fmaf(a[0] + a[2], da.x, s[0]);
                    s[1] = fmaf(a[1] + a[3], da.y, s[1]);
                    s[2] = fmaf(c[0] + c[2], db.x, s[2]);
                    s[3] = fmaf(c[1] + c[3], db.y, s[3]);
                }
            }
        } else {
            const float4 dA0 = lds128f(fA + t * C::KSTRIDE), dA1 = lds128f(fA + t * C::KSTRIDE + 4);
            const float4 dB0 = lds128f(fB + t * C::KSTRIDE), dB1 = lds128f(fB + t * C::KSTRIDE + 4);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 kA = lds128(tA + L::KC + q * 512 + lane * 16);
                const uint4 kB = lds128(tB + L::KC + q * 512 + lane * 16);
                float a[4], c[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t wA = u4_at(kA, j) ^ 0x80808080u, wB = u4_at(kB, j) ^ 0x80808080u;
                    const uint32_t a0 = __byte_perm(wA, 0u, 0x4140u), a1 = __byte_perm(wA, 0u, 0x4342u);
                    const uint32_t b0 = __byte_perm(wB, 0u, 0x4140u), b1 = __byte_perm(wB, 0u, 0x4342u);
                    const uint4 qj = qa(4 * q + j, lane);
                    if (j == 0) {
                        mma_z(a, qj, a0, a1);
                        mma_z(c, qj, b0, b1);
                    } else {
                        mma_acc(a, qj, a0, a1);
                        mma_acc(c, qj, b0, b1);
                    }
                }
                const float2 da = f2_at(dA0, dA1, q), db = f2_at(dB0, dB1, q);
                s[0] = fmaf(a[0] + a[2], da.x, s[0]);
                s[1] = fmaf(a[1] + a[3], da.y, s[1]);
                s[2] = fmaf(c[0] + c[2], db.x, s[2]);
                s[3] = fmaf(c[1] + c[3], db.y, s[3]);
            }
        }
    }

    // Scores of the TPI tiles of an item, softmax update, and the hand-over
    // slot: p' of tile j, tokens 2t, 2t+1 at lane*2TPI + 2j, +1, and the
    // rescale factor of head g at [PA + g].  The running max keeps one binade of
    // headroom (it moves to max + 1 only when a score exceeds it), so the rescale
    // factor is rarely different from 1 and p stays <= 1/2 (p' <= 2^(sigma - 1)).
    // lim (CAUSAL only): index, from the item's first token, of the last key
    // this lane's row may see (a prefill row sees keys up to its own position).
    template <bool MASK, bool CAUSAL = false>
    __device__ __forceinline__ void item(const uint8_t *tp, const float *fp, const int (&v)[C::TPI], int lane,
                                         float *slot, int lim = 0) {
        constexpr int NS2 = 2 * C::TPI;       // scores per lane: tokens 2t, 2t+1 of each tile
        const int g = lane >> 2, t = lane & 3;
        float s[NS2];
#pragma unroll
        for (int h = 0; h < C::TPI / 2; ++h) {
            float a[4];
            scores(tp + 2 * h * L::BYTES, fp + 2 * h * C::SF_TILE, lane, a);
#pragma unroll
            for (int i = 0; i < 4; ++i) s[4 * h + i] = a[i];
        }
        if (MASK) {
#pragma unroll
            for (int j = 0; j < C::TPI; ++j) {
                if (2 * t >= v[j]) s[2 * j] = -INFINITY;
                if (2 * t + 1 >= v[j]) s[2 * j + 1] = -INFINITY;
            }
        }
        if (CAUSAL) {
#pragma unroll
            for (int j = 0; j < C::TPI; ++j) {
                if (8 * j + 2 * t > lim) s[2 * j] = -INFINITY;
                if (8 * j + 2 * t + 1 > lim) s[2 * j + 1] = -INFINITY;
            }
        }
        float mx = s[0];
#pragma unroll
        for (int i = 1; i < NS2; ++i) mx = fmaxf(mx, s[i]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        mx *= inv_sb;                                          // log2 units
        if constexpr (L::VP != PART_F4) vmax = max(vmax, item_v_scale_max<FMT>(tp, lane));
        const float m_true = m_run + sg;
        // mx is finite on the first item (every row sees key 0); later a row may
        // see none of an item's keys (mx = -inf): nothing moves then
        const float m_new = mx > m_true ? mx + 1.f : m_true;
        // (nvfp4 values enter the product already scaled, exactly: no shift needed)
        if constexpr (L::VP != PART_F4) sg = (float)pv_sigma((int)(vmax >> 10));
        const float alpha = ex2(m_run - (m_new - sg));        // 1 when unchanged; 0 on the first item
        l_run *= alpha;
        m_run = m_new - sg;
        float p[NS2];
#pragma unroll
        for (int i = 0; i < NS2; ++i) p[i] = ex2(fmaf(s[i], inv_sb, -m_run));
        float ls = 0.f;
#pragma unroll
        for (int i = 0; i < NS2; i += 4) {
            ls += (p[i] + p[i + 1]) + (p[i + 2] + p[i + 3]);
            sts128(slot + lane * NS2 + i, make_uint4(__float_as_uint(p[i]), __float_as_uint(p[i + 1]),
                                                     __float_as_uint(p[i + 2]), __float_as_uint(p[i + 3])));
        }
        l_run += ls;
        slot[C::PA + g] = alpha;        // the four lanes of group g store the same value
    }
    // An item whose page could not be read: nothing to add, nothing to rescale.
    __device__ __forceinline__ void skip(int lane, float *slot) {
        if (lane < 8) slot[C::PA + lane] = 1.f;
    }
};

// ---------------------------------------------------------------------------
// PV warp: o[dims][heads] += V^T P for one work item
// ---------------------------------------------------------------------------
template <int FMT> struct PvWarp {
    using L = TileLayout<FMT>;
    float o[16][4];        // m-tile mt: o[16 mt + g (+8)][heads 2t, 2t+1]

    __device__ __forceinline__ void init() {
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    }

    // B operand of the value product for one block: P' = p * dV as an exact
    // fp16 pair (hi, lo): hi = rn(p_hi dV), r = p_hi dV - hi (exact, from the
    // fused multiply-add), lo = rn(p_lo dV + r).
    __device__ __forceinline__ static void pscale(uint32_t dv2, uint32_t ph, uint32_t pl, uint32_t &hi, uint32_t &lo) {
        const __half2 d = u32_as_h2(dv2);
        const __half2 h = __hmul2(u32_as_h2(ph), d);
        const __half2 r = __hfma2(u32_as_h2(ph), d, __hneg2(h));
        hi = h2_as_u32(h);
        lo = h2_as_u32(__hfma2(u32_as_h2(pl), d, r));
    }
    // Block b of both tiles: A = [V of tile A tokens 2t, 2t+1 | of tile B], k =
    // 16 tokens; B = P' of the same tokens, once with the hi and once with the
    // lo halves of the exact fp16 pair.
    __device__ __forceinline__ void pv_q4(int b, uint32_t wA, uint32_t wB, uint32_t dA, uint32_t dB,
                                          uint32_t phA, uint32_t plA, uint32_t phB, uint32_t plB) {
        uint32_t hA, lA, hB, lB;
        pscale(dA, phA, plA, hA, lA);
        pscale(dB, phB, plB, hB, lB);
        const uint4 m0 = make_uint4(h2_as_u32(q4_lo_pair(wA)), h2_as_u32(q4_hi_pair(wA)),
                                    h2_as_u32(q4_lo_pair(wB)), h2_as_u32(q4_hi_pair(wB)));
        const uint4 m1 = make_uint4(h2_as_u32(q4_lo_pair(wA >> 8)), h2_as_u32(q4_hi_pair(wA >> 8)),
                                    h2_as_u32(q4_lo_pair(wB >> 8)), h2_as_u32(q4_hi_pair(wB >> 8)));
        mma_acc(o[2 * b], m0, hA, hB);
        mma_acc(o[2 * b + 1], m1, hA, hB);
        mma_acc(o[2 * b], m0, lA, lB);
        mma_acc(o[2 * b + 1], m1, lA, lB);
    }
    __device__ __forceinline__ void pv_i8(int q, const uint4 &wvA, const uint4 &wvB, uint32_t dA, uint32_t dB,
                                          uint32_t phA, uint32_t plA, uint32_t phB, uint32_t plB) {
        uint32_t hA, lA, hB, lB;
        pscale(dA, phA, plA, hA, lA);
        pscale(dB, phB, plB, hB, lB);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t xa = u4_at(wvA, j) ^ 0x80808080u, xb = u4_at(wvB, j) ^ 0x80808080u;
            const uint4 m = make_uint4(h2_as_u32(i8_pair(xa, 0x4140u)), h2_as_u32(i8_pair(xa, 0x4342u)),
                                       h2_as_u32(i8_pair(xb, 0x4140u)), h2_as_u32(i8_pair(xb, 0x4342u)));
            mma_acc(o[4 * q + j], m, hA, hB);
            mma_acc(o[4 * q + j], m, lA, lB);
        }
    }

    // E4M3 values: the token's one scale gives one P' pair per tile for every
    // m-tile; bytes (2t, 2t+1) of a word are one token pair at one dim.
    __device__ __forceinline__ void pv_f8(int q, const uint4 &wvA, const uint4 &wvB, uint32_t hA, uint32_t lA,
                                          uint32_t hB, uint32_t lB) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t xa = u4_at(wvA, j), xb = u4_at(wvB, j);
            const uint4 m = make_uint4(e4m3x2_to_h2(xa), e4m3x2_to_h2(xa >> 16), e4m3x2_to_h2(xb), e4m3x2_to_h2(xb >> 16));
            mma_acc(o[4 * q + j], m, hA, hB);
            mma_acc(o[4 * q + j], m, lA, lB);
        }
    }
    // E2M1 values in the q4_0 word order (token 2t in nibbles 0-3, token 2t+1
    // in nibbles 4-7, dims g, g+8, g+16, g+24): pair the nibbles of the two
    // tokens per dim into bytes, one cvt.e2m1x2 each.  dv0 / dv1: E4M3 scale
    // pairs (tokens 2t, 2t+1) of the two 16-dim blocks of 32-dim block b.
    __device__ __forceinline__ static void f4_pairs(uint32_t w, uint32_t &d0, uint32_t &d8, uint32_t &d16,
                                                    uint32_t &d24) {
        const uint32_t a = w & 0x0F0F0F0Fu, b = (w >> 4) & 0x0F0F0F0Fu;
        const uint32_t u = a | (a >> 12), v = b | (b >> 12);   // bytes: (dim g, dim g+16) and (g+8, g+24)
        d0 = e2m1x2_to_h2(u);
        d16 = e2m1x2_to_h2(u >> 8);
        d8 = e2m1x2_to_h2(v);
        d24 = e2m1x2_to_h2(v >> 8);
    }
    // The values enter exactly (E2M1 times its E4M3 scale: at most 6 significant
    // bits, within fp16's normal range), so B is p itself as an fp16 hi/lo pair.
    __device__ __forceinline__ void pv_f4(int b, uint32_t wA, uint32_t wB, uint32_t eA, uint32_t eB, uint32_t mA,
                                          uint32_t mB, uint32_t phA, uint32_t plA, uint32_t phB, uint32_t plB) {
        uint32_t a0, a8, a16, a24, b0, b8, b16, b24;
        f4_pairs(wA, a0, a8, a16, a24);
        f4_pairs(wB, b0, b8, b16, b24);
        const __half2 sA = u32_as_h2(e4m3x2_to_h2(eA) & mA), sB = u32_as_h2(e4m3x2_to_h2(eB) & mB);   // block 2b
        const uint4 m0 = make_uint4(h2_as_u32(__hmul2(u32_as_h2(a0), sA)), h2_as_u32(__hmul2(u32_as_h2(a8), sA)),
                                    h2_as_u32(__hmul2(u32_as_h2(b0), sB)), h2_as_u32(__hmul2(u32_as_h2(b8), sB)));
        mma_acc(o[2 * b], m0, phA, phB);
        mma_acc(o[2 * b], m0, plA, plB);
        const __half2 tA = u32_as_h2(e4m3x2_to_h2(eA >> 16) & mA), tB = u32_as_h2(e4m3x2_to_h2(eB >> 16) & mB);
        const uint4 m1 = make_uint4(h2_as_u32(__hmul2(u32_as_h2(a16), tA)), h2_as_u32(__hmul2(u32_as_h2(a24), tA)),
                                    h2_as_u32(__hmul2(u32_as_h2(b16), tB)), h2_as_u32(__hmul2(u32_as_h2(b24), tB)));
        mma_acc(o[2 * b + 1], m1, phA, phB);
        mma_acc(o[2 * b + 1], m1, plA, plB);
    }

    // Tiles A, B (consecutive) with p of their tokens 2t, 2t+1.
    template <bool MASK>
    __device__ __forceinline__ void two_tiles(const uint8_t *tA, int vA, int vB, int t, int lane, float pA0, float pA1,
                                              float pB0, float pB1) {
        const uint8_t *tB = tA + L::BYTES;
        uint32_t phA, plA, phB, plB;     // p of tokens 2t, 2t+1 as fp16 hi + lo pairs
        split_pair(pA0, pA1, phA, plA);
        split_pair(pB0, pB1, phB, plB);
        // zero the scales of tokens past the end (their bytes may hold anything)
        const uint32_t mA = MASK ? ((2 * t < vA ? 0xFFFFu : 0u) | (2 * t + 1 < vA ? 0xFFFF0000u : 0u)) : 0xFFFFFFFFu;
        const uint32_t mB = MASK ? ((2 * t < vB ? 0xFFFFu : 0u) | (2 * t + 1 < vB ? 0xFFFF0000u : 0u)) : 0xFFFFFFFFu;
        if constexpr (L::VP == PART_Q4) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint4 wvA = lds128(tA + L::VC + hf * 512 + lane * 16);
                const uint4 wvB = lds128(tB + L::VC + hf * 512 + lane * 16);
                const uint4 eA = lds128(tA + L::VS + t * 32 + hf * 16);   // (dV[2t][b], dV[2t+1][b]), b = 4 hf + bb
                const uint4 eB = lds128(tB + L::VS + t * 32 + hf * 16);
#pragma unroll
                for (int bb = 0; bb < 4; ++bb)
                    pv_q4(4 * hf + bb, u4_at(wvA, bb), u4_at(wvB, bb), u4_at(eA, bb) & mA, u4_at(eB, bb) & mB, phA,
                          plA, phB, plB);
            }
        } else if constexpr (L::VP == PART_F4) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint4 wvA = lds128(tA + L::VC + hf * 512 + lane * 16);
                const uint4 wvB = lds128(tB + L::VC + hf * 512 + lane * 16);
                // E4M3 pairs (dV[2t][blk], dV[2t+1][blk]) for the 16-dim blocks 8 hf .. 8 hf + 7
                const uint4 eA = lds128(tA + L::VS + t * 32 + hf * 16);
                const uint4 eB = lds128(tB + L::VS + t * 32 + hf * 16);
#pragma unroll
                for (int bb = 0; bb < 4; ++bb)
                    pv_f4(4 * hf + bb, u4_at(wvA, bb), u4_at(wvB, bb), u4_at(eA, bb), u4_at(eB, bb), mA, mB, phA, plA,
                          phB, plB);
            }
        } else if constexpr (L::VP == PART_F8) {
            uint32_t hA, lA, hB, lB;
            pscale(*reinterpret_cast<const uint32_t *>(tA + L::VS + t * 4) & mA, phA, plA, hA, lA);
            pscale(*reinterpret_cast<const uint32_t *>(tB + L::VS + t * 4) & mB, phB, plB, hB, lB);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 wvA = lds128(tA + L::VC + q * 512 + lane * 16);
                const uint4 wvB = lds128(tB + L::VC + q * 512 + lane * 16);
                pv_f8(q, wvA, wvB, hA, lA, hB, lB);
            }
        } else {
            const uint4 eA = lds128(tA + L::VS + t * 16);                 // (dV[2t][q], dV[2t+1][q]), q = 0..3
            const uint4 eB = lds128(tB + L::VS + t * 16);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 wvA = lds128(tA + L::VC + q * 512 + lane * 16);
                const uint4 wvB = lds128(tB + L::VC + q * 512 + lane * 16);
                pv_i8(q, wvA, wvB, u4_at(eA, q) & mA, u4_at(eB, q) & mB, phA, plA, phB, plB);
            }
        }
    }

    // Rescale (factors of heads 2t, 2t+1 from the slot) and accumulate the four
    // tiles of an item.
    template <bool MASK>
    __device__ __forceinline__ void item(const uint8_t *tp, const int (&v)[TcCfg<FMT>::TPI], bool ok, int lane,
                                         const float4 (&pv)[TcCfg<FMT>::TPI / 2], float2 al) {
        const int t = lane & 3;
        if (__any_sync(0xffffffffu, al.x != 1.f || al.y != 1.f)) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                o[i][0] *= al.x; o[i][2] *= al.x;
                o[i][1] *= al.y; o[i][3] *= al.y;
            }
        }
        if (!ok) return;
#pragma unroll
        for (int h = 0; h < TcCfg<FMT>::TPI / 2; ++h)
            two_tiles<MASK>(tp + 2 * h * L::BYTES, v[2 * h], v[2 * h + 1], t, lane, pv[h].x, pv[h].y, pv[h].z, pv[h].w);
    }

    // Write this warp's o, heads 2t, 2t+1 scaled by sc0, sc1, to b[8][OSTRIDE]
    // (a row stride of 260 floats keeps the stores of a warp on distinct banks).
    __device__ __forceinline__ void store_scaled(float *b, float sc0, float sc1, int lane) const {
        const int g = lane >> 2, t = lane & 3;
        float *r0 = b + (2 * t) * TcCfg<FMT>::OSTRIDE + g, *r1 = r0 + TcCfg<FMT>::OSTRIDE;
#pragma unroll
        for (int mt = 0; mt < 16; ++mt) {
            r0[16 * mt] = o[mt][0] * sc0;
            r1[16 * mt] = o[mt][1] * sc1;
            r0[16 * mt + 8] = o[mt][2] * sc0;
            r1[16 * mt + 8] = o[mt][3] * sc1;
        }
    }
};

// ---------------------------------------------------------------------------
// CUDA-core compute policy (control).  Lane l owns 8 dims of K and 8 dims of V
// for all heads; partial scores are reduced across the warp by a butterfly
// reduce-scatter so that lane l ends with tokens l/4, heads 2(l%4), 2(l%4)+1.
// ---------------------------------------------------------------------------
template <int FMT, int GT> struct AluCompute {
    using L = TileLayout<FMT>;
    static constexpr int TPI = 1;
    float qr[GT][8];
    float o[GT][8];
    float m_run[2], l_run[2];   // heads 2(l%4), 2(l%4)+1
    float *p_s;                 // warp-private [8 tokens][8 heads]

    __device__ __forceinline__ static int kdim(int lane, int n) {   // dim of this lane's K element n
        if (L::KP == PART_Q4) {
            const int b = lane >> 2, j = lane & 3;
            return 32 * b + 8 * (n & 3) + (n >> 2) + 2 * j;
        } else {
            const int s = 2 * (lane >> 2) + (n >> 2), j = lane & 3;
            const int nb = n & 3;
            return 16 * s + 2 * j + (nb & 1) + 8 * (nb >> 1);
        }
    }
    __device__ __forceinline__ static int vdim(int lane, int e) {   // dim of this lane's V element e
        if (L::VP == PART_Q4) {
            const int b = lane >> 2, g = 2 * (lane & 3) + (e >> 2);
            return 32 * b + g + 8 * (e & 3);
        } else {
            const int m = 2 * (lane >> 2) + (e >> 2), g = 2 * (lane & 3) + ((e >> 1) & 1);
            return 16 * m + g + 8 * (e & 1);
        }
    }

    __device__ __forceinline__ void init(const float *qg, int G, int lane, float *pbuf) {
#pragma unroll
        for (int h = 0; h < GT; ++h)
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                qr[h][n] = h < G ? qg[h * D + kdim(lane, n)] * QSCALE : 0.f;
                o[h][n] = 0.f;
            }
        m_run[0] = m_run[1] = -INFINITY;
        l_run[0] = l_run[1] = 0.f;
        p_s = pbuf;
    }

    __device__ __forceinline__ static float q4f(uint32_t w, int n) {
        return __uint_as_float(0x4B000000u | ((w >> (4 * n)) & 15u)) - 8388616.0f;   // 2^23 + c - (2^23 + 8)
    }
    __device__ __forceinline__ static float i8f(uint32_t w, int n) {
        return (float)(int8_t)((w >> (8 * n)) & 0xFFu);
    }

    template <bool MASK>
    __device__ __forceinline__ void tile(const uint8_t *tp, int valid, int lane) {
        float part[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) part[i] = 0.f;
        // ---- partial scores over this lane's 8 dims ---------------------------
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            float kv[8];
            float dk;
            if constexpr (L::KP == PART_Q4) {
                const int b = lane >> 2, j = lane & 3;
                const uint32_t w = lds32(tp + L::KC + (b >> 2) * 512 + (r * 4 + j) * 16 + (b & 3) * 4);
#pragma unroll
                for (int n = 0; n < 8; ++n) kv[n] = q4f(w, n);
                dk = __half2float(*reinterpret_cast<const __half *>(tp + L::KS + (r >> 1) * 32 + b * 4 + (r & 1) * 2));
            } else {
                const int j = lane & 3;
#pragma unroll
                for (int hs = 0; hs < 2; ++hs) {
                    const int s = 2 * (lane >> 2) + hs;
                    const uint32_t w = lds32(tp + L::KC + (s >> 2) * 512 + (r * 4 + j) * 16 + (s & 3) * 4);
#pragma unroll
                    for (int n = 0; n < 4; ++n) kv[4 * hs + n] = i8f(w, n);
                }
                const int q = (lane >> 2) >> 1;
                dk = __half2float(*reinterpret_cast<const __half *>(tp + L::KS + (r >> 1) * 16 + q * 4 + (r & 1) * 2));
            }
#pragma unroll
            for (int h = 0; h < GT; ++h) {
                float acc = 0.f;
#pragma unroll
                for (int n = 0; n < 8; ++n) acc = fmaf(qr[h][n], kv[n], acc);
                part[r * 8 + h] = acc * dk;
            }
        }
        // ---- reduce-scatter across the warp: lane keeps slots 2l, 2l+1 ----------
#pragma unroll
        for (int step = 0; step < 5; ++step) {
            const int off = 16 >> step;
            const int n = 64 >> step;       // current length
            const bool upper = (lane & off) != 0;
#pragma unroll
            for (int i = 0; i < n / 2; ++i) {
                const float send = upper ? part[i] : part[i + n / 2];
                const float keep = upper ? part[i + n / 2] : part[i];
                part[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
            }
        }
        const int r = lane >> 2, h0 = 2 * (lane & 3);
        float s[2] = {part[0], part[1]};
        if (MASK && r >= valid) s[0] = s[1] = -INFINITY;
        float mx[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            mx[k] = s[k];
            mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 4));
            mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 8));
            mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 16));
        }
        const bool grow = mx[0] > m_run[0] || mx[1] > m_run[1];
        if (__any_sync(0xffffffffu, grow)) {
            float alpha[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const float m_new = fmaxf(m_run[k], mx[k]);
                alpha[k] = exp2f(m_run[k] - m_new);
                l_run[k] *= alpha[k];
                m_run[k] = m_new;
            }
#pragma unroll
            for (int h = 0; h < GT; ++h) {
                const float a = __shfl_sync(0xffffffffu, alpha[h & 1], h >> 1);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[h][e] *= a;
            }
        }
        float p[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            p[k] = exp2f(s[k] - m_run[k]);
            l_run[k] += p[k];
        }
        __syncwarp();
        p_s[r * 8 + h0] = p[0];
        p_s[r * 8 + h0 + 1] = p[1];
        __syncwarp();
        // ---- values ------------------------------------------------------------
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            float vv[8];
            float dv;
            if constexpr (L::VP == PART_Q4) {
                const int b = lane >> 2;
#pragma unroll
                for (int gg = 0; gg < 2; ++gg) {
                    const int g = 2 * (lane & 3) + gg;
                    const uint32_t w = lds32(tp + L::VC + (b >> 2) * 512 + (g * 4 + (rr >> 1)) * 16 + (b & 3) * 4);
#pragma unroll
                    for (int k = 0; k < 4; ++k) vv[4 * gg + k] = q4f(w, 4 * (rr & 1) + k);
                }
                dv = __half2float(*reinterpret_cast<const __half *>(tp + L::VS + (rr >> 1) * 32 + b * 4 + (rr & 1) * 2));
            } else {
#pragma unroll
                for (int mm = 0; mm < 2; ++mm)
#pragma unroll
                    for (int gg = 0; gg < 2; ++gg) {
                        const int m = 2 * (lane >> 2) + mm, g = 2 * (lane & 3) + gg;
                        const uint32_t w = lds32(tp + L::VC + (m >> 2) * 512 + (g * 4 + (rr >> 1)) * 16 + (m & 3) * 4);
                        vv[4 * mm + 2 * gg + 0] = i8f(w, 0 + (rr & 1));
                        vv[4 * mm + 2 * gg + 1] = i8f(w, 2 + (rr & 1));
                    }
                const int q = (lane >> 2) >> 1;
                dv = __half2float(*reinterpret_cast<const __half *>(tp + L::VS + (rr >> 1) * 16 + q * 4 + (rr & 1) * 2));
            }
            if (MASK && rr >= valid) dv = 0.f;
#pragma unroll
            for (int h = 0; h < GT; ++h) {
                const float pp = p_s[rr * 8 + h] * dv;
#pragma unroll
                for (int e = 0; e < 8; ++e) o[h][e] = fmaf(pp, vv[e], o[h][e]);
            }
        }
    }

    template <bool MASK>
    __device__ __forceinline__ void item(const uint8_t *tp, const float *, int vA, int, int lane) {
        tile<MASK>(tp, vA, lane);
    }

    __device__ __forceinline__ void report(int lane, float *m_s, float *l_s) {
        float l0 = l_run[0], l1 = l_run[1];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, off);
            l1 += __shfl_xor_sync(0xffffffffu, l1, off);
        }
        if (lane < 4) {
            m_s[2 * lane] = m_run[0];
            m_s[2 * lane + 1] = m_run[1];
            l_s[2 * lane] = l0;
            l_s[2 * lane + 1] = l1;
        }
    }
    __device__ __forceinline__ void accumulate(float *o_s, const float *scale, int lane) {
#pragma unroll
        for (int h = 0; h < GT; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) atomicAdd(o_s + h * D + vdim(lane, e), o[h][e] * scale[h]);
    }
};

// One output row (256 dims, lane holds dims 8 lane .. 8 lane + 7, already
// divided by L): H/16 if V was stored rotated (butterflies inside the lane for
// the low three index bits, then across lanes), then fp32 and bf16 stores.
__device__ __forceinline__ void finish_row(float (&x)[8], int lane, int inverse_fwht, int64_t row, uint16_t *out_bf16,
                                           float *out_f32) {
    if (inverse_fwht) {
#pragma unroll
        for (int hh = 1; hh < 8; hh <<= 1)
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if ((i & hh) == 0) {
                    const float a = x[i], b = x[i + hh];
                    x[i] = a + b;
                    x[i + hh] = a - b;
                }
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float other = __shfl_xor_sync(0xffffffffu, x[i], m);
                x[i] = upper ? other - x[i] : x[i] + other;
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] *= 0.0625f;
    }
    const size_t off = (size_t)row * D + lane * 8;
    if (out_f32) {
        float4 *o = reinterpret_cast<float4 *>(out_f32 + off);
        o[0] = make_float4(x[0], x[1], x[2], x[3]);
        o[1] = make_float4(x[4], x[5], x[6], x[7]);
    }
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        pk[i] = *reinterpret_cast<const uint32_t *>(&v);
    }
    *reinterpret_cast<uint4 *>(out_bf16 + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
}

// ---------------------------------------------------------------------------
// Merge of one (sequence, KV head) group: units [u0, u1) of the workspace ->
// the G output rows starting at out_row.  M = max m_u, L = sum l_u 2^(m_u - M),
// o = sum 2^(m_u - M) o_u / L, then H/16 if V was stored rotated.  Runs on the
// first NTH threads of the CTA (named barrier bar_id); sm: COMBINE_SMEM floats.
// Warp h computes head h's weights from all units' (m, l) at once (warp max
// and sum); then every lane keeps 2 UB independent 16-byte loads in flight,
// and the warps that share a head add their sums in a fixed order.  Out of
// line, so that it does not shape the register allocation of the decode's
// main loop.
// ---------------------------------------------------------------------------
template <int NTH>
__device__ __noinline__ void combine_group(const float *ws, int G, int u0, int u1, int64_t out_row,
                                           int inverse_fwht, uint16_t *out_bf16, float *out_f32, float *sm,
                                           int bar_id) {
    constexpr int NWARP = NTH / 32;
    static_assert(NWARP >= 8, "the weight pass takes one warp per head");
    constexpr int UB = 8;                         // units whose loads are in flight together (16 float4 / lane)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int stride = ws_unit_floats(G);
    float *o_s = sm;                              // [8][256] accumulated outputs
    float *f_s = sm + 8 * D;                      // [units][8] weights 2^(m_u - M)
    float *Ms = f_s + 8 * COMBINE_MAX_UNITS;      // [8] running max
    float *Ls = Ms + 8;                           // [8] running sum
    float *Cs = Ls + 8;                           // [8] factor for what is accumulated so far
    for (int i = tid; i < 8 * D; i += NTH) o_s[i] = 0.f;
    for (int c0 = u0; c0 < u1; c0 += COMBINE_MAX_UNITS) {     // chunks of units (one pass in practice)
        const int n = min(COMBINE_MAX_UNITS, u1 - c0);
        // weights: warp h reads (m, l) of every unit for head h, all loads first
        if (warp < G) {
            const int h = warp;
            float m[COMBINE_MAX_UNITS / 32], l[COMBINE_MAX_UNITS / 32];
#pragma unroll
            for (int j = 0; j < COMBINE_MAX_UNITS / 32; ++j) {
                const int uu = lane + 32 * j;
                const float *p = ws + (size_t)(c0 + uu) * stride + G * D;
                m[j] = uu < n ? __ldcg(p + h) : -INFINITY;
                l[j] = uu < n ? __ldcg(p + 8 + h) : 0.f;
            }
            float M = -INFINITY;
#pragma unroll
            for (int j = 0; j < COMBINE_MAX_UNITS / 32; ++j) M = fmaxf(M, m[j]);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            const float M_old = c0 == u0 ? -INFINITY : Ms[h];
            M = fmaxf(M, M_old);
            float L = 0.f;
#pragma unroll
            for (int j = 0; j < COMBINE_MAX_UNITS / 32; ++j) {
                const float f = m[j] == -INFINITY ? 0.f : exp2f(m[j] - M);
                if (lane + 32 * j < n) f_s[(lane + 32 * j) * 8 + h] = f;
                L = fmaf(l[j], f, L);
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
            __syncwarp();
            if (lane == 0) {
                const float c = M_old == -INFINITY ? 0.f : exp2f(M_old - M);
                Cs[h] = c;
                Ls[h] = (c0 == u0 ? 0.f : Ls[h] * c) + L;
                Ms[h] = M;
            }
        }
        asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(NTH));
        if (c0 > u0) {                                  // rescale earlier chunks
            for (int i = tid; i < G * D; i += NTH) o_s[i] *= Cs[i >> 8];
            asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(NTH));
        }
        // warps per head: warp w takes head w % G and every wph-th unit, UB units
        // (2 UB independent 16-byte loads per lane) at a time
        const int wph = NWARP / G;
        const int h = warp % G, part = warp / G;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (warp < wph * G) {
            for (int ub = part; ub < n; ub += UB * wph) {
                float4 a[UB], b[UB];
#pragma unroll
                for (int j = 0; j < UB; ++j) {
                    const int uu = ub + j * wph;
                    const float4 *p = reinterpret_cast<const float4 *>(ws + (size_t)(c0 + min(uu, n - 1)) * stride +
                                                                       h * D + lane * 8);
                    a[j] = __ldcg(p);
                    b[j] = __ldcg(p + 1);
                }
#pragma unroll
                for (int j = 0; j < UB; ++j) {
                    const int uu = ub + j * wph;
                    const float f = uu < n ? f_s[uu * 8 + h] : 0.f;
                    acc[0] = fmaf(a[j].x, f, acc[0]); acc[1] = fmaf(a[j].y, f, acc[1]);
                    acc[2] = fmaf(a[j].z, f, acc[2]); acc[3] = fmaf(a[j].w, f, acc[3]);
                    acc[4] = fmaf(b[j].x, f, acc[4]); acc[5] = fmaf(b[j].y, f, acc[5]);
                    acc[6] = fmaf(b[j].z, f, acc[6]); acc[7] = fmaf(b[j].w, f, acc[7]);
                }
            }
        }
        // the parts of a head add their sums in part order, so that the result
        // does not depend on which warp finishes first
        for (int p = 0; p < wph; ++p) {
            if (warp < wph * G && part == p) {
#pragma unroll
                for (int i = 0; i < 8; ++i) o_s[h * D + lane * 8 + i] += acc[i];
            }
            asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(NTH));
        }
    }
    // warp h finishes head h
    for (int h = warp; h < G; h += NWARP) {
        float x[8];
        const float inv = 1.0f / Ls[h];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = o_s[h * D + lane * 8 + i] * inv;
        finish_row(x, lane, inverse_fwht, out_row + h, out_bf16, out_f32);
    }
}

// ---------------------------------------------------------------------------
// Merge of head h of one (sequence, KV head) group by one CTA, used when every
// CTA of the launch is resident at once (cooperative launch): each CTA of the
// group takes its own heads, so the group's partials are read by up to G CTAs
// in parallel instead of by the last one alone.  Units [u0, u0 + n); NTH
// threads (named barrier bar_id); sm: MH_SMEM floats.
// ---------------------------------------------------------------------------
constexpr int MH_MAX_UNITS = 256;                 // units per group on this path
constexpr int MH_BATCH = 8;                       // float4 loads in flight per thread
template <int NTH>
__device__ void merge_head(const float *ws, int G, int u0, int n, int h, int64_t out_row, int inverse_fwht,
                           uint16_t *out_bf16, float *out_f32, float *sm, int bar_id) {
    constexpr int NPART = NTH / 64;               // threads per float4 column of the head
    static_assert(NPART >= 1 && NTH % 64 == 0, "threads");
    const int tid = threadIdx.x, lane = tid & 31, c = tid & 63, part = tid >> 6;
    const int stride = ws_unit_floats(G);
    float *f_s = sm;                              // [n] weights 2^(m_u - M)
    float *red = f_s + MH_MAX_UNITS;              // [NPART][256] partial sums
    float *o_s = red + NPART * D;                 // [256]
    float *L_s = o_s + D;                         // [1]
    const float *base = ws + (size_t)u0 * stride + h * D + 4 * c;
    // first batch of this thread's loads, issued before the weights are known
    float4 v[MH_BATCH];
#pragma unroll
    for (int j = 0; j < MH_BATCH; ++j) {
        const int uu = part + j * NPART;
        v[j] = uu < n ? __ldcg(reinterpret_cast<const float4 *>(base + (size_t)uu * stride)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (tid < 32) {
        float m[MH_MAX_UNITS / 32], l[MH_MAX_UNITS / 32];
#pragma unroll
        for (int j = 0; j < MH_MAX_UNITS / 32; ++j) {
            const int uu = lane + 32 * j;
            const float *p = ws + (size_t)(u0 + uu) * stride + G * D;
            m[j] = uu < n ? __ldcg(p + h) : -INFINITY;
            l[j] = uu < n ? __ldcg(p + 8 + h) : 0.f;
        }
        float M = -INFINITY;
#pragma unroll
        for (int j = 0; j < MH_MAX_UNITS / 32; ++j) M = fmaxf(M, m[j]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float L = 0.f;
#pragma unroll
        for (int j = 0; j < MH_MAX_UNITS / 32; ++j) {
            const float f = m[j] == -INFINITY ? 0.f : exp2f(m[j] - M);
            if (lane + 32 * j < n) f_s[lane + 32 * j] = f;
            L = fmaf(l[j], f, L);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        if (lane == 0) *L_s = L;
    }
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(NTH));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int b0 = 0;; b0 += MH_BATCH * NPART) {
#pragma unroll
        for (int j = 0; j < MH_BATCH; ++j) {
            const int uu = b0 + part + j * NPART;
            const float f = uu < n ? f_s[uu] : 0.f;
            acc.x = fmaf(v[j].x, f, acc.x); acc.y = fmaf(v[j].y, f, acc.y);
            acc.z = fmaf(v[j].z, f, acc.z); acc.w = fmaf(v[j].w, f, acc.w);
        }
        if (b0 + MH_BATCH * NPART >= n) break;
#pragma unroll
        for (int j = 0; j < MH_BATCH; ++j) {
            const int uu = b0 + MH_BATCH * NPART + part + j * NPART;
            v[j] = uu < n ? __ldcg(reinterpret_cast<const float4 *>(base + (size_t)uu * stride)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    reinterpret_cast<float4 *>(red + part * D)[c] = acc;
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(NTH));
    for (int i = tid; i < D; i += NTH) {
        float s = 0.f;
#pragma unroll
        for (int p = 0; p < NPART; ++p) s += red[p * D + i];
        o_s[i] = s;
    }
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(NTH));
    if (tid < 32) {
        float x[8];
        const float inv = 1.0f / *L_s;
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = o_s[lane * 8 + i] * inv;
        finish_row(x, lane, inverse_fwht, out_row + h, out_bf16, out_f32);
    }
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(NTH));
}

// Spin (with a time limit) until *p >= target; acquire ordering on success.
__device__ __forceinline__ bool wait_count_at_least(const int *p, int target, uint64_t limit_ns) {
    uint64_t t0 = 0;
    for (;;) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        if (v >= target) return true;
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) t0 = now;
        else if (now - t0 > limit_ns) return false;
        __nanosleep(128);
    }
}

struct DecodeArgs {
    const uint8_t *pool;
    PoolGeom geo;
    int layer;
    const float *q;
    const int32_t *page_table;
    int max_pages;
    const int32_t *plan;
    int n_q_heads;
    int G;
    float *ws;
    int32_t *status;
    int inverse_fwht;      // fused combine: un-rotate the output
    uint16_t *out_bf16;    // fused combine outputs (NULL: write partials only)
    float *out_f32;
    int coop;              // fused combine: every CTA is resident (cooperative launch); merge heads in parallel
    // decode step (tensor-core kernel only): q is the raw query, rotated in the
    // kernel where the format rotates; k_new / v_new [n_seq][n_kv][256] are the
    // sequences' newest tokens (position seq_len - 1), appended by the last
    // CTA of each (sequence, KV head) group before it fetches that position
    const float *k_new;
    const float *v_new;
};

// ---------------------------------------------------------------------------
// Shared pieces of both kernels
// ---------------------------------------------------------------------------
// Plan entry check; on failure write an empty partial so that the merge ignores
// the unit.
__device__ __forceinline__ bool unit_ok(const DecodeArgs &A, int seq, int kvh, int t0, int t1, float *wsu) {
    const bool ok = A.plan[0] == PLAN_MAGIC && seq >= 0 && seq < A.plan[2] && kvh >= 0 &&
                    kvh < A.geo.n_kv_heads && t0 >= 0 && t0 < t1 && (t0 % STEP_TOKENS) == 0 &&
                    t1 <= A.max_pages * PAGE;
    if (!ok) {
        if (threadIdx.x == 0) status_or(A.status, KVQ_STATUS_BAD_PLAN);
        for (int i = threadIdx.x; i < A.G * D; i += blockDim.x) wsu[i] = 0.f;
        if (threadIdx.x < 8) {
            wsu[A.G * D + threadIdx.x] = -INFINITY;
            wsu[A.G * D + 8 + threadIdx.x] = 0.f;
        }
    }
    return ok;
}

// Copy warp: stream the unit's 64-token steps into the stage ring.  All 32
// lanes fetch the page slots of 32 pages at a time (one load round trip per 32
// pages instead of one per step); lane 0 waits for free stages and issues the
// bulk copies.  Before the warp exits, every copy it issued has landed.
struct NoHook {
    __device__ __forceinline__ void operator()(int, int) const {}
};
template <int NS, int STAGE_BYTES, int TILE_BYTES, class Hook = NoHook>
__device__ __forceinline__ void copy_loop(const DecodeArgs &A, uint8_t *smem, uint64_t *full, uint64_t *empty,
                                          int *stage_ok, int seq, int kvh, int t0, int n_steps, int lane,
                                          Hook hook = Hook()) {
    const uint8_t *head_base = A.pool + (int64_t)A.layer * A.geo.layer_stride + (int64_t)kvh * A.geo.page_bytes;
    const int32_t *pt = A.page_table + (int64_t)seq * A.max_pages;
    const uint64_t pol = policy_evict_first();
    const int page0 = t0 >> 8;
    int chunk = -1, my_slot = -1, issued = 0;
    bool stop = false;
    for (int i = 0; i < n_steps; ++i) {
        const int tok = t0 + i * STEP_TOKENS;
        const int rel = (tok >> 8) - page0;
        if ((rel >> 5) != chunk) {
            chunk = rel >> 5;
            const int pg = page0 + 32 * chunk + lane;
            my_slot = pg < A.max_pages ? __ldg(pt + pg) : -1;
        }
        const int slot = __shfl_sync(0xffffffffu, my_slot, rel & 31);
        hook(i, lane);                 // whole warp, before step i is requested
        // the whole warp waits for the free stage (a warp whose lane 0 waits
        // alone while the rest sit at the warp barrier slowed the other warps
        // of its SM sub-partition)
        bool free_stage = stop || i < NS || mbar_wait_bounded(&empty[i % NS], ((i / NS) - 1) & 1, WAIT_LIMIT_NS);
        free_stage = __all_sync(0xffffffffu, free_stage);
        if (!free_stage) {                       // a stage never came free: issue nothing more
            if (lane == 0) status_or(A.status, KVQ_STATUS_TIMEOUT);
            stop = true;
        }
        if (lane == 0 && !stop) {
            ++issued;
            const int si = i % NS;
            if (slot < 0 || slot >= A.geo.n_pages) {
                status_or(A.status, KVQ_STATUS_BAD_SLOT);
                stage_ok[si] = 0;
                mbar_arrive(&full[si]);
            } else {
                stage_ok[si] = 1;
                const uint8_t *src = head_base + (int64_t)slot * A.geo.slot_stride + ((tok & 255) >> 3) * TILE_BYTES;
                mbar_arrive_expect_tx(&full[si], STAGE_BYTES);
                bulk_g2s(smem + si * STAGE_BYTES, src, STAGE_BYTES, &full[si], pol);
            }
        }
        __syncwarp();
    }
    // every copy this warp issued has landed before it exits (the consumers may
    // have stopped early on a timeout)
    if (lane == 0) {
        for (int i = issued > NS ? issued - NS : 0; i < issued; ++i)
            if (!mbar_wait_bounded(&full[i % NS], (i / NS) & 1, WAIT_LIMIT_NS)) status_or(A.status, KVQ_STATUS_TIMEOUT);
    }
    __syncwarp();
}

// The unit's partial is in the workspace: with FUSED, count the unit in and let
// the last CTA of the (sequence, KV head) group merge the group.  Runs on the
// NCT merge threads (bar 1).
template <bool FUSED, int NCT>
__device__ __forceinline__ void publish_unit(const DecodeArgs &A, int seq, int kvh, int n_units, int *s_last,
                                             uint8_t *smem) {
    if constexpr (FUSED) {
        const int G = A.G;
        const int32_t *start = A.plan + PLAN_HEADER + 4 * n_units;
        const int grp = seq * A.geo.n_kv_heads + kvh;
        int *counter = reinterpret_cast<int *>(A.ws + (size_t)n_units * ws_unit_floats(G)) + grp;
        __threadfence();
        asm volatile("bar.sync 1, %0;" ::"r"(NCT));
        if (A.coop) {
            // every CTA of the group counts in, waits for the others, merges its
            // heads (rank, rank + n_grp, ...) and counts out; the last one out
            // resets the counter for the next launch
            const int n_grp = start[grp + 1] - start[grp];
            if (threadIdx.x == 0) {
                atomicAdd(counter, 1);
                *s_last = wait_count_at_least(counter, n_grp, WAIT_LIMIT_NS);
                if (!*s_last) status_or(A.status, KVQ_STATUS_TIMEOUT);
                __threadfence();
            }
            asm volatile("bar.sync 1, %0;" ::"r"(NCT));
            if (*s_last) {
                const int64_t row0 = (int64_t)seq * A.n_q_heads + (int64_t)kvh * G;
                for (int h = blockIdx.x - start[grp]; h < G; h += n_grp)
                    merge_head<NCT>(A.ws, G, start[grp], n_grp, h, row0, A.inverse_fwht, A.out_bf16, A.out_f32,
                                    reinterpret_cast<float *>(smem), 1);
            }
            if (threadIdx.x == 0 && atomicAdd(counter, 1) == 2 * n_grp - 1) *counter = 0;
            return;
        }
        if (threadIdx.x == 0) {
            const int n_grp = start[grp + 1] - start[grp];
            const int old = atomicAdd(counter, 1);
            *s_last = old == n_grp - 1;
            if (*s_last) *counter = 0;         // every unit of the group has arrived: reset for the next launch
        }
        asm volatile("bar.sync 1, %0;" ::"r"(NCT));
        if (*s_last) {
            __threadfence();
            combine_group<NCT>(A.ws, G, start[grp], start[grp + 1], (int64_t)seq * A.n_q_heads + (int64_t)kvh * G,
                               A.inverse_fwht, A.out_bf16, A.out_f32, reinterpret_cast<float *>(smem), 1);
        }
    }
}

// After the warps' states are in m_s/l_s [n_rep][8] and o_s [8][256] (scaled to
// M_s): write the unit's partial, then publish it.
template <bool FUSED, int NCT>
__device__ __forceinline__ void finish_unit(const DecodeArgs &A, const float *o_s, const float *m_s, const float *l_s,
                                            const float *M_s, int n_rep, float *wsu, int seq, int kvh, int n_units,
                                            int *s_last, uint8_t *smem) {
    const int G = A.G;
    for (int i = threadIdx.x; i < G * D; i += NCT) wsu[i] = o_s[i];
    if (threadIdx.x < 8) {
        const int h = threadIdx.x;
        float Lh = 0.f;
        for (int w = 0; w < n_rep; ++w) {
            const float mw = m_s[w * 8 + h];
            if (mw != -INFINITY) Lh += l_s[w * 8 + h] * exp2f(mw - M_s[h]);
        }
        wsu[G * D + h] = M_s[h];
        wsu[G * D + 8 + h] = Lh;
    }
    publish_unit<FUSED, NCT>(A, seq, kvh, n_units, s_last, smem);
}

// Helpers kept out of line so that their registers do not shape the allocation
// of the kernel's main loop.  In a decode step, in the CTA whose unit ends the
// group, the scale warp encodes the newest token into the pool while the first
// stages land, and keeps its codes in shared memory, to write them into the
// last stage when it lands.  The QK warps copy the query heads h = first,
// first + stride, ... into q_s, rotating them (ROTATE) in a decode step.
// Encode the newest token into the pool and keep its codes and scales in
// shared memory (5 words per lane).
template <int FMT>
__device__ __noinline__ void step_encode_token(const DecodeArgs &A, int seq, int kvh, int pos, uint32_t *stash,
                                               int lane) {
    const int64_t row = ((int64_t)seq * A.geo.n_kv_heads + kvh) * D;
    float xk[8], xv[8];
    load8(A.k_new + row + lane * 8, xk);
    load8(A.v_new + row + lane * 8, xv);
    const bool in_range = pos >= 0 && pos < A.max_pages * PAGE;
    const int slot = in_range ? A.page_table[(int64_t)seq * A.max_pages + (pos >> 8)] : -1;
    TokenCodes t;
    quant_token<FMT>(xk, xv, lane, t);
    uint8_t *gtile = token_tile<FMT>(const_cast<uint8_t *>(A.pool), A.geo, A.layer, slot, kvh, pos, A.status, lane);
    if (gtile) store_token<FMT>(t, lane, pos & 7, gtile);
    uint32_t w[5];
    w[4] = (uint32_t)__half_as_ushort(t.dk) | ((uint32_t)__half_as_ushort(t.dv) << 16);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        w[h] = w[2 + h] = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            w[h] |= (uint32_t)(t.k[4 * h + e] & 0xFF) << (8 * e);
            w[2 + h] |= (uint32_t)(t.v[4 * h + e] & 0xFF) << (8 * e);
        }
    }
#pragma unroll
    for (int i = 0; i < 5; ++i) stash[lane * 5 + i] = w[i];
    __syncwarp();
}
// Write the stashed token into the landed stage that holds it, over the bytes
// the copy brought (which may predate the pool store above).
template <int FMT>
__device__ __noinline__ void step_patch_stage(int pos, const uint32_t *stash, uint8_t *stage, int lane) {
    TokenCodes t;
    uint32_t w[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) w[i] = stash[lane * 5 + i];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            t.k[4 * h + e] = (w[h] >> (8 * e)) & 0xFF;
            t.v[4 * h + e] = (w[2 + h] >> (8 * e)) & 0xFF;
        }
    t.dk = __ushort_as_half((unsigned short)(w[4] & 0xFFFF));
    t.dv = __ushort_as_half((unsigned short)(w[4] >> 16));
    store_token<FMT>(t, lane, pos & 7, stage + ((pos & 63) >> 3) * TileLayout<FMT>::BYTES);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // before the stage's next bulk fill
    __syncwarp();
}
template <bool ROTATE>
__device__ __noinline__ void step_stage_query(const float *qg, float *q_s, int G, int first, int stride, int lane) {
    for (int h = first; h < G; h += stride) {
        float x[8];
        load8(qg + h * D + lane * 8, x);
        if (ROTATE) fwht256_lane(x, lane);
#pragma unroll
        for (int i = 0; i < 8; ++i) q_s[h * D + lane * 8 + i] = x[i];
    }
}

// ---------------------------------------------------------------------------
// Tensor-core kernel
// ---------------------------------------------------------------------------
template <int FMT, bool FUSED, bool STEP = false>
__global__ void __launch_bounds__(TcCfg<FMT>::NTHREADS, 1) decode_tc_kernel(const __grid_constant__ DecodeArgs A) {
    static_assert(!STEP || FUSED, "the decode step merges in the kernel");
    using L = TileLayout<FMT>;
    using C = TcCfg<FMT>;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *ready = full + C::NS;            // fp32 K scales of the stage are written
    uint64_t *empty = ready + C::NS;           // every item of the stage is done
    uint64_t *p_full = empty + C::NS;          // QK -> PV slot written
    uint64_t *p_empty = p_full + C::NQK * C::DP;
    int *stage_ok = reinterpret_cast<int *>(p_empty + C::NQK * C::DP);
    __shared__ int s_last;

    grid_dependency_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.x;
    const int32_t *U = A.plan + PLAN_HEADER + 4 * u;
    const int seq = U[0], kvh = U[1], t0 = U[2], t1 = U[3];
    const int G = A.G;
    const int n_units = A.plan[1];
    float *wsu = A.ws + (size_t)u * ws_unit_floats(G);
    if (!unit_ok(A, seq, kvh, t0, t1, wsu)) return;
    const int n_steps = (t1 - t0 + STEP_TOKENS - 1) / STEP_TOKENS;
    const int n_items = (t1 - t0 + C::TPI * TILE - 1) / (C::TPI * TILE);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&ready[i], 32);                    // every lane of the scale warp arrives
            mbar_init(&empty[i], 32 * C::ITEMS_PER_STAGE);
        }
        for (int i = 0; i < C::NQK * C::DP; ++i) {      // every lane of the QK / PV warp arrives
            mbar_init(&p_full[i], 32);
            mbar_init(&p_empty[i], 32);
        }
        fence_mbar_init();
    }
    __syncthreads();
    // decode step: the last CTA of the group appends the group's newest token
    const bool appends = STEP && u == A.plan[PLAN_HEADER + 4 * n_units + seq * A.geo.n_kv_heads + kvh + 1] - 1;

    if (warp >= 2 * C::NQK) {                   // the producer warpgroup
        setmaxnreg_dec<C::REG_PROD>();
        if (warp == C::COPY_WARP)
            copy_loop<C::NS, C::STAGE_BYTES, L::BYTES>(A, smem, full, empty, stage_ok, seq, kvh, t0, n_steps, lane);
        if (warp < C::SCALE_WARP) return;
        // scale warp c owns the ring slots si with si % N_SCALE == c, so each
        // slot's phases are awaited by one warp, in order.  The stages still
        // become ready in order: a QK warp waits on the ready barrier of a stage
        // up to NQK items past its last one, and a barrier two phases behind
        // would answer that wait with an older phase of the same parity.  So a
        // scale warp converts as soon as its stage lands, but announces it only
        // after the previous stage's announcement.
        const int c = warp - C::SCALE_WARP;
        uint32_t *stash = reinterpret_cast<uint32_t *>(smem + C::TKV_OFF);
        const bool encodes = appends && ((n_steps - 1) % C::NS) % C::N_SCALE == c;   // owns the newest token's stage
        if (encodes) step_encode_token<FMT>(A, seq, kvh, t1 - 1, stash, lane);
        for (int i = 0; i < n_steps; ++i) {
            const int si = i % C::NS;
            if (si % C::N_SCALE != c) continue;
            if (!mbar_wait_bounded(&full[si], (i / C::NS) & 1, WAIT_LIMIT_NS)) {
                if (lane == 0) status_or(A.status, KVQ_STATUS_TIMEOUT);
                break;
            }
            if (encodes && i == n_steps - 1 && stage_ok[si])    // the stage that holds the newest token
                step_patch_stage<FMT>(t1 - 1, stash, smem + si * C::STAGE_BYTES, lane);
            if (stage_ok[si])
                convert_stage_scales<FMT>(smem + si * C::STAGE_BYTES,
                                          reinterpret_cast<float *>(smem + C::SFOFF + si * C::SF_STAGE_BYTES), lane);
            // (the ready barrier of stage i - 1 is at most one phase behind,
            // since stage i's copy waited for the consumers of stage i - NS)
            if (i > 0 && !mbar_wait_bounded(&ready[(i - 1) % C::NS], ((i - 1) / C::NS) & 1, WAIT_LIMIT_NS)) {
                if (lane == 0) status_or(A.status, KVQ_STATUS_TIMEOUT);
                break;
            }
            __syncwarp();
            mbar_arrive(&ready[si]);
        }
        return;
    }
    setmaxnreg_inc<C::REG_COMPUTE>();          // QK and PV warpgroups

    float *pring = reinterpret_cast<float *>(smem + C::POFF);
    constexpr int NCT = 2 * C::NQK * 32;       // merge threads: QK + PV warps
    const bool is_qk = warp < C::NQK;
    const int pw = is_qk ? warp : warp - C::NQK;    // pair index
    QkWarp<FMT> qk;
    PvWarp<FMT> pv;
    // Pair pw takes items pw, pw + NQK, ... (item `it` = tiles 4 it .. 4 it + 3 =
    // half of stage it / 2); the QK warp passes the item index, or -1 at the end,
    // to its PV warp with the scores.  (Handing items out from a shared counter
    // instead measured slower on long units.)
    if (is_qk) {
        const float *qg = A.q + ((int64_t)seq * A.n_q_heads + (int64_t)kvh * G) * D;
        // The group's query goes through the (still unused) hand-over ring, one
        // head per QK warp: a warp that loads all G heads itself waits longer
        // while the first stages flood the memory system.  A decode step
        // rotates the raw query on the way, as q_rotate would.
        step_stage_query<STEP && Fmt<FMT>::KROT>(qg, pring, G, pw, C::NQK, lane);
        asm volatile("bar.sync 2, %0;" ::"r"(C::NQK * 32));
        qk.init(pring + (lane >> 2) * D, (lane >> 2) < G, lane, smem + C::QOFF, pw == 0);
        asm volatile("bar.sync 2, %0;" ::"r"(C::NQK * 32));
        for (int k = 0;; ++k) {
            const int slot = k % C::DP;
            float *ps = pring + (pw * C::DP + slot) * C::PSLOT;
            if (k >= C::DP && !mbar_wait_bounded(&p_empty[pw * C::DP + slot], ((k / C::DP) - 1) & 1, WAIT_LIMIT_NS)) {
                if (lane == 0) status_or(A.status, KVQ_STATUS_TIMEOUT);
                break;
            }
            const int it = pw + C::NQK * k;
            if (it >= n_items) {                       // no work left: tell the PV warp
                if (lane == 0) reinterpret_cast<int *>(ps)[C::PITEM] = -1;
                mbar_arrive(&p_full[pw * C::DP + slot]);
                break;
            }
            const int st = it / C::ITEMS_PER_STAGE, si = st % C::NS, within = it % C::ITEMS_PER_STAGE;
            // ready implies the stage's bulk copy has landed (the scale warp waited for it)
            if (!mbar_wait_bounded(&ready[si], (st / C::NS) & 1, WAIT_LIMIT_NS)) {
                if (lane == 0) status_or(A.status, KVQ_STATUS_TIMEOUT);
                break;
            }
            const int tok = t0 + it * C::TPI * TILE;
            int v[C::TPI];
#pragma unroll
            for (int j = 0; j < C::TPI; ++j) v[j] = max(0, min(TILE, t1 - tok - j * TILE));
            if (stage_ok[si]) {
                const uint8_t *tp = smem + si * C::STAGE_BYTES + within * C::TPI * L::BYTES;
                const float *fp = reinterpret_cast<const float *>(smem + C::SFOFF + si * C::SF_STAGE_BYTES) +
                                  within * C::TPI * C::SF_TILE;
                if (v[C::TPI - 1] == TILE) qk.template item<false>(tp, fp, v, lane, ps);
                else qk.template item<true>(tp, fp, v, lane, ps);
            } else {
                qk.skip(lane, ps);
            }
            if (lane == 0) reinterpret_cast<int *>(ps)[C::PITEM] = it;
            mbar_arrive(&p_full[pw * C::DP + slot]);
        }
    } else {
        pv.init();
        for (int k = 0;; ++k) {
            const int slot = k % C::DP;
            const float *ps = pring + (pw * C::DP + slot) * C::PSLOT;
            // p_full implies the QK warp saw the stage ready, hence landed
            if (!mbar_wait_bounded(&p_full[pw * C::DP + slot], (k / C::DP) & 1, WAIT_LIMIT_NS)) {
                if (lane == 0) status_or(A.status, KVQ_STATUS_TIMEOUT);
                break;
            }
            const int it = reinterpret_cast<const int *>(ps)[C::PITEM];
            if (it < 0) break;
            float4 pp[C::TPI / 2];
#pragma unroll
            for (int h = 0; h < C::TPI / 2; ++h) pp[h] = lds128f(ps + lane * 2 * C::TPI + 4 * h);
            const float2 al = make_float2(ps[C::PA + 2 * (lane & 3)], ps[C::PA + 2 * (lane & 3) + 1]);
            mbar_arrive(&p_empty[pw * C::DP + slot]);
            const int st = it / C::ITEMS_PER_STAGE, si = st % C::NS, within = it % C::ITEMS_PER_STAGE;
            const int tok = t0 + it * C::TPI * TILE;
            int v[C::TPI];
#pragma unroll
            for (int j = 0; j < C::TPI; ++j) v[j] = max(0, min(TILE, t1 - tok - j * TILE));
            const uint8_t *tp = smem + si * C::STAGE_BYTES + within * C::TPI * L::BYTES;
            const bool ok = stage_ok[si] != 0;
            if (v[C::TPI - 1] == TILE) pv.template item<false>(tp, v, ok, lane, pp, al);
            else pv.template item<true>(tp, v, ok, lane, pp, al);
            mbar_arrive(&empty[si]);
        }
    }

    // ---- CTA merge: QK warps report (m, l); PV warps write o scaled to the CTA
    // max into their own buffer; the merge threads sum the buffers into the
    // partial -----------------------------------------------------------------
    asm volatile("bar.sync 1, %0;" ::"r"(NCT));               // every consumer is done with the ring
    float *obuf = reinterpret_cast<float *>(smem);            // [NQK][8][OSTRIDE]
    float *m_s = obuf + C::NQK * 8 * C::OSTRIDE;              // [NQK][8]
    float *l_s = m_s + C::NQK * 8;                            // [NQK][8]
    if (is_qk) {
        float lr = qk.l_run;
        lr += __shfl_xor_sync(0xffffffffu, lr, 1);
        lr += __shfl_xor_sync(0xffffffffu, lr, 2);
        if ((lane & 3) == 0) {
            m_s[pw * 8 + (lane >> 2)] = qk.m_run;
            l_s[pw * 8 + (lane >> 2)] = lr;
        }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(NCT));
    if (!is_qk) {
        const int t = lane & 3;
        float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
        for (int w = 0; w < C::NQK; ++w) {
            M0 = fmaxf(M0, m_s[w * 8 + 2 * t]);
            M1 = fmaxf(M1, m_s[w * 8 + 2 * t + 1]);
        }
        const float m0 = m_s[pw * 8 + 2 * t], m1 = m_s[pw * 8 + 2 * t + 1];
        const float sc0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M0), sc1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M1);
        pv.store_scaled(obuf + pw * 8 * C::OSTRIDE, sc0, sc1, lane);
    } else if (pw == 0 && lane < 8) {
        const int h = lane;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < C::NQK; ++w) M = fmaxf(M, m_s[w * 8 + h]);
        float Lh = 0.f;
#pragma unroll
        for (int w = 0; w < C::NQK; ++w) {
            const float mw = m_s[w * 8 + h];
            if (mw != -INFINITY) Lh += l_s[w * 8 + h] * exp2f(mw - M);
        }
        wsu[G * D + h] = M;
        wsu[G * D + 8 + h] = Lh;
    }
    asm volatile("bar.sync 1, %0;" ::"r"(NCT));
    for (int i = threadIdx.x; i < G * D; i += NCT) {
        const float *b = obuf + (i >> 8) * C::OSTRIDE + (i & 255);
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < C::NQK; ++w) acc += b[w * 8 * C::OSTRIDE];
        wsu[i] = acc;
    }
    publish_unit<FUSED, NCT>(A, seq, kvh, n_units, &s_last, smem);
}

// ---------------------------------------------------------------------------
// Chunked prefill attention over the quantised cache
// ---------------------------------------------------------------------------
// A chunk of n_tok new tokens of one sequence at positions pos0 .. pos0 +
// n_tok - 1 (already appended to the pool) attends, each token over the keys
// 0 .. its own position.  For one KV head, the chunk's query rows are
// r = i * G + h (token i, head h of the group); a CTA takes ROWS of them, and
// each of its NW compute warps takes 8 rows and runs the decode's QK and PV
// products for them over every item of the key range: the stage ring, the
// scale conversion and the fragments are the decode's, and each stage is read
// from HBM once for all ROWS rows (the decode reads it for 6 or 8).
struct PrefillArgs {
    DecodeArgs d;            // pool, geometry, layer, page table, status (the copy loop's view)
    int seq, pos0, n_tok, n_rows;
    int n_split, split_tokens;   // key range cut at multiples of split_tokens (blockIdx.z = part)
    float *ws;                   // n_split > 1: partials [part][kv head][row][PF_WS_STRIDE]
};

template <int FMT> struct PfCfg {
    using L = TileLayout<FMT>;
    using T = TcCfg<FMT>;
    static constexpr int NW = 8;                          // compute warps, 8 query rows each
    static constexpr int ROWS = 8 * NW;
    static constexpr int COPY_WARP = NW, SCALE_WARP = NW + 1;
    static constexpr int NTHREADS = (NW + 2) * 32;
    static constexpr int TPI = T::TPI, IPS = 8 / TPI;
    static constexpr int STAGE_BYTES = 8 * L::BYTES;
    static constexpr int NS = (FMT == KVQ_Q4_0 || FMT == KVQ_NVFP4) ? 6 : 4;
    static constexpr int RING = NS * STAGE_BYTES;
    static constexpr int OBUF = NW * 8 * T::OSTRIDE * 4;   // the epilogue's rows (after the loop, over the ring)
    static constexpr int DATA = RING > OBUF ? RING : OBUF;
    static constexpr int SFOFF = (DATA + 127) & ~127;
    static constexpr int QOFF = SFOFF + NS * T::SF_STAGE_BYTES;      // per warp: 16 k-steps x 32 lanes x 16 B
    static constexpr int POFF = QOFF + NW * 16 * 32 * 16;            // per warp: one p slot
    static constexpr int BAR_OFF = (POFF + NW * T::PSLOT * 4 + 15) & ~15;
    static constexpr int TOTAL = BAR_OFF + 3 * NS * 8 + NS * 4;      // full, ready, empty; stage_ok
    static_assert(TOTAL <= 227 * 1024, "shared memory budget");
};

template <int FMT>
__global__ void __launch_bounds__(PfCfg<FMT>::NTHREADS, 1) prefill_tc_kernel(const __grid_constant__ PrefillArgs P) {
    using L = TileLayout<FMT>;
    using C = PfCfg<FMT>;
    using T = TcCfg<FMT>;
    const DecodeArgs &A = P.d;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *ready = full + C::NS;
    uint64_t *empty = ready + C::NS;
    int *stage_ok = reinterpret_cast<int *>(empty + C::NS);

    grid_dependency_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kvh = blockIdx.y, G = A.G;
    const int r0 = blockIdx.x * C::ROWS;
    if (r0 >= P.n_rows) return;
    // keys 0 .. pos0 + (last token of the CTA's rows)
    const int i_last = min(P.n_tok - 1, (r0 + C::ROWS - 1) / G);
    const int t_end = P.pos0 + i_last + 1;
    // this CTA's part of the key range: [t0, t1).  Every cut lies at or below
    // pos0, so every row sees the first key of its part.
    const int part = blockIdx.z;
    const int t0 = part * P.split_tokens;
    const int t1 = part == P.n_split - 1 ? t_end : min(t_end, t0 + P.split_tokens);
    if (t1 <= t0) {                            // excluded by the host; kept as a guard
        if (threadIdx.x == 0) status_or(A.status, KVQ_STATUS_BAD_PLAN);
        return;
    }
    const int n_steps = (t1 - t0 + STEP_TOKENS - 1) / STEP_TOKENS;
    const int n_items = (t1 - t0 + C::TPI * TILE - 1) / (C::TPI * TILE);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&ready[i], 32);
            mbar_init(&empty[i], 32 * C::NW * C::IPS);     // every compute warp, every item of the stage
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == C::COPY_WARP) {
        copy_loop<C::NS, C::STAGE_BYTES, L::BYTES>(A, smem, full, empty, stage_ok, P.seq, kvh, t0, n_steps, lane);
        return;
    }
    if (warp == C::SCALE_WARP) {
        for (int i = 0; i < n_steps; ++i) {
            const int si = i % C::NS;
            if (!mbar_wait_bounded(&full[si], (i / C::NS) & 1, WAIT_LIMIT_NS)) {
                if (lane == 0) status_or(A.status, KVQ_STATUS_TIMEOUT);
                break;
            }
            if (stage_ok[si])
                convert_stage_scales<FMT>(smem + si * C::STAGE_BYTES,
                                          reinterpret_cast<float *>(smem + C::SFOFF + si * T::SF_STAGE_BYTES), lane);
            __syncwarp();
            mbar_arrive(&ready[si]);
        }
        return;
    }

    // compute warp: rows r0 + 8 warp + g, g = lane / 4
    const int r = r0 + 8 * warp + (lane >> 2);
    const bool row_ok = r < P.n_rows;
    const int tok_i = row_ok ? r / G : 0, head = row_ok ? r % G : 0;
    const int lim = row_ok ? P.pos0 + tok_i : t_end - 1;        // last key the row sees
    const float *qrow = A.q + ((int64_t)tok_i * A.n_q_heads + (int64_t)kvh * G + head) * D;
    QkWarp<FMT> qk;
    PvWarp<FMT> pv;
    qk.init(qrow, row_ok, lane, smem + C::QOFF + warp * (16 * 32 * 16), true);
    __syncwarp();
    pv.init();
    float *ps = reinterpret_cast<float *>(smem + C::POFF) + warp * T::PSLOT;
    for (int it = 0; it < n_items; ++it) {
        const int st = it / C::IPS, si = st % C::NS, within = it % C::IPS;
        if (!mbar_wait_bounded(&ready[si], (st / C::NS) & 1, WAIT_LIMIT_NS)) {
            if (lane == 0) status_or(A.status, KVQ_STATUS_TIMEOUT);
            break;
        }
        const int tok = t0 + it * C::TPI * TILE;
        int v[C::TPI];
#pragma unroll
        for (int j = 0; j < C::TPI; ++j) v[j] = max(0, min(TILE, t1 - tok - j * TILE));
        const uint8_t *tp = smem + si * C::STAGE_BYTES + within * C::TPI * L::BYTES;
        const bool ok = stage_ok[si] != 0;
        if (ok) {
            const float *fp = reinterpret_cast<const float *>(smem + C::SFOFF + si * T::SF_STAGE_BYTES) +
                              within * C::TPI * T::SF_TILE;
            if (v[C::TPI - 1] == TILE) qk.template item<false, true>(tp, fp, v, lane, ps, lim - tok);
            else qk.template item<true, true>(tp, fp, v, lane, ps, lim - tok);
        } else {
            qk.skip(lane, ps);
        }
        __syncwarp();
        float4 pp[C::TPI / 2];
#pragma unroll
        for (int h = 0; h < C::TPI / 2; ++h) pp[h] = lds128f(ps + lane * 2 * C::TPI + 4 * h);
        const float2 al = make_float2(ps[T::PA + 2 * (lane & 3)], ps[T::PA + 2 * (lane & 3) + 1]);
        if (v[C::TPI - 1] == TILE) pv.template item<false>(tp, v, ok, lane, pp, al);
        else pv.template item<true>(tp, v, ok, lane, pp, al);
        __syncwarp();                               // the slot is rewritten by the next item
        mbar_arrive(&empty[si]);
    }

    // ---- epilogue: o / l per row, un-rotated where the format rotates V ----
    asm volatile("bar.sync 1, %0;" ::"r"(C::NW * 32));   // every warp is done with the ring
    float lr = qk.l_run;
    lr += __shfl_xor_sync(0xffffffffu, lr, 1);
    lr += __shfl_xor_sync(0xffffffffu, lr, 2);            // row g's sum on lanes 4g .. 4g+3
    const int t = lane & 3;
    float *b = reinterpret_cast<float *>(smem) + warp * 8 * T::OSTRIDE;
    if (P.ws) {
        // a part of the key range: o unnormalised with its (m, l), merged later
        pv.store_scaled(b, 1.f, 1.f, lane);
        __syncwarp();
        float *wsp = P.ws + ((size_t)part * A.geo.n_kv_heads + kvh) * (size_t)P.n_rows * PF_WS_STRIDE;
        const int rh = r0 + 8 * warp + (lane >> 2);
        if ((lane & 3) == 0 && rh < P.n_rows) {
            wsp[(size_t)rh * PF_WS_STRIDE + D] = qk.m_run;
            wsp[(size_t)rh * PF_WS_STRIDE + D + 1] = lr;
        }
        for (int h = 0; h < 8; ++h) {
            const int rr = r0 + 8 * warp + h;
            if (rr >= P.n_rows) break;
            const float *src = b + h * T::OSTRIDE + lane * 8;
            float4 *dst = reinterpret_cast<float4 *>(wsp + (size_t)rr * PF_WS_STRIDE + lane * 8);
            dst[0] = make_float4(src[0], src[1], src[2], src[3]);
            dst[1] = make_float4(src[4], src[5], src[6], src[7]);
        }
        return;
    }
    const float l0 = __shfl_sync(0xffffffffu, lr, 8 * t), l1 = __shfl_sync(0xffffffffu, lr, 8 * t + 4);
    pv.store_scaled(b, l0 > 0.f ? 1.f / l0 : 0.f, l1 > 0.f ? 1.f / l1 : 0.f, lane);
    __syncwarp();
    for (int h = 0; h < 8; ++h) {
        const int rr = r0 + 8 * warp + h;
        if (rr >= P.n_rows) break;
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = b[h * T::OSTRIDE + lane * 8 + i];
        const int ti = rr / G, hh = rr % G;
        finish_row(x, lane, A.inverse_fwht, (int64_t)ti * A.n_q_heads + (int64_t)kvh * G + hh, A.out_bf16, A.out_f32);
    }
}

// Merge of the key-range parts of a split prefill: one warp per (KV head, row),
// the log-sum-exp rule over the parts, then 1/L and the output rotation.
__global__ void __launch_bounds__(256) prefill_merge_kernel(const float *__restrict__ ws, int n_split, int n_kv,
                                                            int n_rows, int G, int n_q_heads, int inverse_fwht,
                                                            uint16_t *out_bf16, float *out_f32) {
    grid_dependency_wait();
    const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (w >= n_kv * n_rows) return;            // warp-uniform
    const int kvh = w / n_rows, r = w - kvh * n_rows;
    const size_t part_stride = (size_t)n_kv * n_rows * PF_WS_STRIDE;
    const float *row = ws + ((size_t)kvh * n_rows + r) * PF_WS_STRIDE;
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, row[s * part_stride + D]);
    float L = 0.f, x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < n_split; ++s) {
        const float *p = row + s * part_stride;
        const float m = p[D];
        if (m == -INFINITY) continue;
        const float f = exp2f(m - M);
        L += f * p[D + 1];
        const float4 a = reinterpret_cast<const float4 *>(p + lane * 8)[0];
        const float4 b = reinterpret_cast<const float4 *>(p + lane * 8)[1];
        x[0] += f * a.x; x[1] += f * a.y; x[2] += f * a.z; x[3] += f * a.w;
        x[4] += f * b.x; x[5] += f * b.y; x[6] += f * b.z; x[7] += f * b.w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] *= inv;
    const int ti = r / G, hh = r - ti * G;
    finish_row(x, lane, inverse_fwht, (int64_t)ti * n_q_heads + (int64_t)kvh * G + hh, out_bf16, out_f32);
}

// ---------------------------------------------------------------------------
// CUDA-core kernel (control): 8 consumer warps, one tile per item, + copy warp
// ---------------------------------------------------------------------------
template <int FMT> struct AluCfg {
    static constexpr int NCW = 8;
    static constexpr int NTHREADS = (NCW + 1) * 32;
    static constexpr int STAGE_BYTES = 8 * TileLayout<FMT>::BYTES;
    static constexpr int NS = FMT == KVQ_Q4_0 ? 5 : (FMT == KVQ_INT8 ? 3 : 4);
    static constexpr int RING = NS * STAGE_BYTES;
    static constexpr int MERGE = (COMBINE_SMEM > 8 * D + 2 * NCW * 8 + 16 ? COMBINE_SMEM : 8 * D + 2 * NCW * 8 + 16) * 4;
    static constexpr int DATA = RING > MERGE ? RING : MERGE;
    static constexpr int BAR_OFF = (DATA + 127) & ~127;
    static constexpr int TOTAL = BAR_OFF + 2 * NS * 8 + NS * 4 + 16;
};

template <int FMT, int GT, bool FUSED>
__global__ void __launch_bounds__(AluCfg<FMT>::NTHREADS, 1) decode_alu_kernel(const DecodeArgs A) {
    using L = TileLayout<FMT>;
    using C = AluCfg<FMT>;
    extern __shared__ __align__(128) uint8_t smem[];
    grid_dependency_wait();
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *empty = full + C::NS;
    int *stage_ok = reinterpret_cast<int *>(empty + C::NS);
    __shared__ int s_last;
    __shared__ float p_bufs[C::NCW * 64];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.x;
    const int32_t *U = A.plan + PLAN_HEADER + 4 * u;
    const int seq = U[0], kvh = U[1], t0 = U[2], t1 = U[3];
    const int G = A.G;
    const int n_units = A.plan[1];
    float *wsu = A.ws + (size_t)u * ws_unit_floats(G);
    if (!unit_ok(A, seq, kvh, t0, t1, wsu)) return;
    const int n_steps = (t1 - t0 + STEP_TOKENS - 1) / STEP_TOKENS;
    const int n_tiles = (t1 - t0 + TILE - 1) / TILE;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 8);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == C::NCW) {
        copy_loop<C::NS, C::STAGE_BYTES, L::BYTES>(A, smem, full, empty, stage_ok, seq, kvh, t0, n_steps, lane);
        return;
    }
    AluCompute<FMT, GT> comp;
    comp.init(A.q + ((int64_t)seq * A.n_q_heads + (int64_t)kvh * G) * D, G, lane, p_bufs + warp * 64);
    for (int it = warp; it < n_tiles; it += C::NCW) {
        const int st = it >> 3, si = st % C::NS;
        if (!mbar_wait_bounded(&full[si], (st / C::NS) & 1, WAIT_LIMIT_NS)) {
            if (lane == 0) status_or(A.status, KVQ_STATUS_TIMEOUT);
            break;
        }
        const int valid = min(TILE, t1 - (t0 + it * TILE));
        if (stage_ok[si]) {
            const uint8_t *tp = smem + si * C::STAGE_BYTES + (it & 7) * L::BYTES;
            if (valid == TILE) comp.template item<false>(tp, nullptr, valid, 0, lane);
            else comp.template item<true>(tp, nullptr, valid, 0, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[si]);
    }
    constexpr int NCT = C::NCW * 32;
    asm volatile("bar.sync 1, %0;" ::"r"(NCT));
    float *o_s = reinterpret_cast<float *>(smem);
    float *m_s = o_s + 8 * D;
    float *l_s = m_s + C::NCW * 8;
    float *M_s = l_s + C::NCW * 8;
    for (int i = threadIdx.x; i < 8 * D; i += NCT) o_s[i] = 0.f;
    comp.report(lane, m_s + warp * 8, l_s + warp * 8);
    asm volatile("bar.sync 1, %0;" ::"r"(NCT));
    if (threadIdx.x < 8) {
        float M = -INFINITY;
        for (int w = 0; w < C::NCW; ++w) M = fmaxf(M, m_s[w * 8 + threadIdx.x]);
        M_s[threadIdx.x] = M;
    }
    asm volatile("bar.sync 1, %0;" ::"r"(NCT));
    float scale[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        const float mw = m_s[warp * 8 + h];
        scale[h] = mw == -INFINITY ? 0.f : exp2f(mw - M_s[h]);
    }
    comp.accumulate(o_s, scale, lane);
    asm volatile("bar.sync 1, %0;" ::"r"(NCT));
    finish_unit<FUSED, NCT>(A, o_s, m_s, l_s, M_s, C::NCW, wsu, seq, kvh, n_units, &s_last, smem);
}

__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ ws, const int32_t *__restrict__ plan,
                                                      int n_kv, int G, int inverse_fwht, uint16_t *out_bf16,
                                                      float *out_f32) {
    __shared__ float sm[COMBINE_SMEM];
    grid_dependency_wait();
    const int grp = blockIdx.x;
    const int seq = grp / n_kv, kvh = grp - seq * n_kv;
    const int n_units = plan[1];
    const int32_t *start = plan + PLAN_HEADER + 4 * n_units;
    combine_group<256>(ws, G, start[grp], start[grp + 1], (int64_t)seq * n_kv * G + (int64_t)kvh * G, inverse_fwht,
                       out_bf16, out_f32, sm, 1);
}

// Launch one decode kernel.  The first launch on each device sets the kernel's
// shared-memory limit and counts how many of its CTAs fit on the device at
// once (for this very kernel, so the cooperative decision matches what is
// launched); both happen once per (kernel, device) under a lock, so threads
// may launch concurrently.  A kernel that moves registers between warpgroups
// (regs > 0) is launched only if it was built with exactly that many
// registers per thread: with fewer, its setmaxnreg.inc could never be met.
template <auto KERNEL>
cudaError_t launch_decode_kernel(int smem_bytes, int threads, const DecodeArgs &a, int n_units, bool fused,
                                 cudaStream_t s, int regs = 0) {
    static std::mutex mu;
    static int cap[64];                  // resident CTAs per device ordinal; 0 = not yet known
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int c = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (cap[dev] == 0) {
            if (regs > 0) {
                cudaFuncAttributes fa;
                cudaError_t e = cudaFuncGetAttributes(&fa, KERNEL);
                if (e != cudaSuccess) return e;
                if (fa.numRegs != regs) return cudaErrorInvalidConfiguration;
            }
            cudaError_t e = cudaFuncSetAttribute(KERNEL, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
            if (e != cudaSuccess) return e;
            int sms = 0, per_sm = 0;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, KERNEL, threads, smem_bytes);
            if (e != cudaSuccess) return e;
            if (per_sm <= 0) return cudaErrorInvalidConfiguration;
            cap[dev] = sms * per_sm;
        }
        c = cap[dev];
    }
    DecodeArgs b = a;
    b.coop = fused && n_units <= c && n_units <= MH_MAX_UNITS ? 1 : 0;
    return launch_ex(KERNEL, dim3(n_units), dim3(threads), smem_bytes, s, b.coop != 0, b);
}

template <int FMT, bool FUSED>
cudaError_t launch_fmt(bool tc, const DecodeArgs &a, int n_units, cudaStream_t s) {
    if (tc) {
        using C = TcCfg<FMT>;
        if constexpr (FUSED) {
            if (a.k_new)
                return launch_decode_kernel<decode_tc_kernel<FMT, true, true>>(C::TOTAL, C::NTHREADS, a, n_units, true,
                                                                               s, C::REG_LAUNCH);
        }
        return launch_decode_kernel<decode_tc_kernel<FMT, FUSED>>(C::TOTAL, C::NTHREADS, a, n_units, FUSED, s,
                                                                  C::REG_LAUNCH);
    }
    if constexpr (FMT == KVQ_FP8 || FMT == KVQ_NVFP4) {
        return cudaErrorNotSupported;          // the CUDA-core control covers the integer-code formats only
    } else {
        using C = AluCfg<FMT>;
        switch (a.G) {
        case 4: return launch_decode_kernel<decode_alu_kernel<FMT, 4, FUSED>>(C::TOTAL, C::NTHREADS, a, n_units, FUSED, s);
        case 6: return launch_decode_kernel<decode_alu_kernel<FMT, 6, FUSED>>(C::TOTAL, C::NTHREADS, a, n_units, FUSED, s);
        default:
            return launch_decode_kernel<decode_alu_kernel<FMT, 8, FUSED>>(C::TOTAL, C::NTHREADS, a, n_units, FUSED, s);
        }
    }
}

template <bool FUSED>
cudaError_t launch_fused(int fmt, bool tc, const DecodeArgs &a, int n_units, cudaStream_t s) {
    switch (fmt) {
    case KVQ_INT8: return launch_fmt<KVQ_INT8, FUSED>(tc, a, n_units, s);
    case KVQ_Q4_0: return launch_fmt<KVQ_Q4_0, FUSED>(tc, a, n_units, s);
    case KVQ_K8V4: return launch_fmt<KVQ_K8V4, FUSED>(tc, a, n_units, s);
    case KVQ_FP8: return launch_fmt<KVQ_FP8, FUSED>(tc, a, n_units, s);
    default: return launch_fmt<KVQ_NVFP4, FUSED>(tc, a, n_units, s);
    }
}

}  // namespace

cudaError_t launch_decode(int fmt, bool tensor_cores, const uint8_t *pool, const PoolGeom &geo, int layer,
                          const float *q, const int32_t *page_table, int max_pages, const int32_t *plan,
                          const kvq_plan_info &info, float *ws, int32_t *status, int inverse_fwht, uint16_t *out_bf16,
                          float *out_f32, cudaStream_t s, const float *k_new, const float *v_new) {
    DecodeArgs a{pool, geo, layer, q, page_table, max_pages, plan, info.n_kv_heads * info.group, info.group, ws,
                 status, inverse_fwht, out_bf16, out_f32, 0, k_new, v_new};
    if (out_bf16) return launch_fused<true>(fmt, tensor_cores, a, info.n_units, s);
    return launch_fused<false>(fmt, tensor_cores, a, info.n_units, s);
}

template <int FMT>
cudaError_t launch_prefill_fmt(const PrefillArgs &p, cudaStream_t s) {
    using C = PfCfg<FMT>;
    static std::mutex mu;
    static bool configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev]) {
            cudaError_t e =
                cudaFuncSetAttribute(prefill_tc_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::TOTAL);
            if (e != cudaSuccess) return e;
            configured[dev] = true;
        }
    }
    const dim3 grid((unsigned)((p.n_rows + C::ROWS - 1) / C::ROWS), (unsigned)p.d.geo.n_kv_heads,
                    (unsigned)p.n_split);
    cudaError_t e = launch_ex(prefill_tc_kernel<FMT>, grid, dim3(C::NTHREADS), C::TOTAL, s, false, p);
    if (e != cudaSuccess || !p.ws) return e;
    const int warps = p.d.geo.n_kv_heads * p.n_rows;
    return launch_ex(prefill_merge_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, s, false,
                     (const float *)p.ws, p.n_split, p.d.geo.n_kv_heads, p.n_rows, p.d.G, p.d.n_q_heads,
                     p.d.inverse_fwht, p.d.out_bf16, p.d.out_f32);
}

cudaError_t launch_prefill(int fmt, const uint8_t *pool, const PoolGeom &geo, int layer, const float *q, int seq,
                           int pos0, int n_tok, const int32_t *page_table, int max_pages, int n_q_heads,
                           int n_split, int split_tokens, float *ws, int inverse_fwht, uint16_t *out_bf16,
                           float *out_f32, int32_t *status, cudaStream_t s) {
    const int G = n_q_heads / geo.n_kv_heads;
    PrefillArgs p{};
    p.d = DecodeArgs{pool, geo, layer, q, page_table, max_pages, nullptr, n_q_heads, G, nullptr,
                     status, inverse_fwht, out_bf16, out_f32, 0, nullptr, nullptr};
    p.seq = seq;
    p.pos0 = pos0;
    p.n_tok = n_tok;
    p.n_rows = n_tok * G;
    p.n_split = n_split;
    p.split_tokens = split_tokens;
    p.ws = n_split > 1 ? ws : nullptr;
    switch (fmt) {
    case KVQ_INT8: return launch_prefill_fmt<KVQ_INT8>(p, s);
    case KVQ_Q4_0: return launch_prefill_fmt<KVQ_Q4_0>(p, s);
    case KVQ_K8V4: return launch_prefill_fmt<KVQ_K8V4>(p, s);
    case KVQ_FP8: return launch_prefill_fmt<KVQ_FP8>(p, s);
    default: return launch_prefill_fmt<KVQ_NVFP4>(p, s);
    }
}

cudaError_t launch_combine(const float *ws, const int32_t *plan, const kvq_plan_info &info, int inverse_fwht,
                           uint16_t *out_bf16, float *out_f32, cudaStream_t s) {
    const int groups = info.n_seq * info.n_kv_heads;
    if (groups == 0) return cudaSuccess;
    return launch_ex(combine_kernel, dim3(groups), dim3(256), 0, s, false, ws, plan, info.n_kv_heads, info.group,
                     inverse_fwht, out_bf16, out_f32);
}

}  // namespace kvq
