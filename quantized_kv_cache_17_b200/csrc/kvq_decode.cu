// paged_decode_attn_{int8,q4_0,k8v4}: split-K single-token attention over the
// quantised, paged KV cache, one CTA per work unit of the plan.
//
// [Strata] "4-bit KV 缓存：先旋转，再压到 4-bit": scores are taken on the rotated
// query and rotated keys (<Hq, Hk> = <q, k>), values are mixed in the rotated
// space and the output is rotated back afterwards (attn_combine).  [Guide]
// "一": 24 query heads share 4 KV heads (groups of 6), so every K/V tile read
// from HBM serves the whole group.
//
// CTA = 8 consumer warps + 1 producer warp.  The producer streams the unit's
// tokens in 64-token steps (8 tiles, contiguous inside one page block) with
// 1-D bulk copies into a ring of shared-memory stages (full/empty mbarriers);
// consumer warp w takes tile w of every step.  Each warp keeps its own online
// softmax state; at the end the warps are merged in shared memory and the CTA
// writes one partial (o[G][256] unnormalised, m[G], l[G], scores in log2 units).
//
// Two compute policies share the scaffold:
//  MmaCompute  - tensor cores (mma.sync m16n8k16, fp16 x fp16 -> fp32).  Codes
//                are exact in fp16; the query and the probabilities are split
//                into fp16 hi + lo parts so the products keep ~22 bits.
//                QK^T: rows = [8 heads hi | 8 heads lo], cols = 8 tokens,
//                k = 16 dims; the per-block K scale is applied to the fp32
//                block sums.  PV: rows = 16 dims, cols = 8 heads, k = [8 tokens
//                hi-P | same 8 tokens lo-P]; the per-block V scale is folded
//                into P before the split.  The score fragment of QK^T is exactly
//                the P fragment PV needs, so no data moves between lanes.
//  AluCompute  - the same computation with fp32 FMAs on CUDA cores only; the
//                measured control for the tensor-core version.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int NW = 8;                         // consumer warps
constexpr int NTHREADS = (NW + 1) * 32;
constexpr float QSCALE = 0.09016844005556021f;  // log2(e) / sqrt(256)
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

template <int FMT> struct Stages { static constexpr int N = 4; };
template <> struct Stages<KVQ_Q4_0> { static constexpr int N = 5; };
template <> struct Stages<KVQ_INT8> { static constexpr int N = 3; };
template <> struct Stages<KVQ_K8V4> { static constexpr int N = 4; };

template <int FMT> struct Smem {
    static constexpr int STAGE_BYTES = NW * TileLayout<FMT>::BYTES;
    static constexpr int NS = Stages<FMT>::N;
    static constexpr int RING = NS * STAGE_BYTES;
    static constexpr int MERGE = (8 * D + 2 * NW * 8 + 2 * 8) * 4;   // o[8][256], m/l per warp, M/L
    static constexpr int DATA = RING > MERGE ? RING : MERGE;
    static constexpr int BAR_OFF = (DATA + 15) & ~15;
    static constexpr int TOTAL = BAR_OFF + NS * 16 + NS * 4 + 16;
};

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

// ---------------------------------------------------------------------------
// Tensor-core compute policy
// ---------------------------------------------------------------------------
template <int FMT> struct MmaCompute {
    using L = TileLayout<FMT>;
    uint32_t qa[16][4];
    float o[16][4];
    float m_run, l_run;

    __device__ __forceinline__ void init(const float *qg, int G, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int ks = 0; ks < 16; ++ks) {
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            if (g < G) {
                const float *p = qg + g * D + 16 * ks + 2 * t;
                x[0] = p[0] * QSCALE; x[1] = p[1] * QSCALE; x[2] = p[8] * QSCALE; x[3] = p[9] * QSCALE;
            }
            split_pair(x[0], x[1], qa[ks][0], qa[ks][1]);
            split_pair(x[2], x[3], qa[ks][2], qa[ks][3]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        m_run = -INFINITY;
        l_run = 0.f;
    }

    template <bool MASK>
    __device__ __forceinline__ void tile(const uint8_t *tp, int valid, int lane) {
        const int t = lane & 3;
        // ---- scores S[head g][tokens 2t, 2t+1] ------------------------------
        float s0 = 0.f, s1 = 0.f;
        if constexpr (L::KP == PART_Q4) {
            const uint4 kw0 = lds128(tp + L::KC + lane * 16);
            const uint4 kw1 = lds128(tp + L::KC + 512 + lane * 16);
            const uint4 ks0 = lds128(tp + L::KS + t * 32);
            const uint4 ks1 = lds128(tp + L::KS + t * 32 + 16);
            const uint32_t kw[8] = {kw0.x, kw0.y, kw0.z, kw0.w, kw1.x, kw1.y, kw1.z, kw1.w};
            const uint32_t kd[8] = {ks0.x, ks0.y, ks0.z, ks0.w, ks1.x, ks1.y, ks1.z, ks1.w};
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                const uint32_t w = kw[b], w2 = kw[b] >> 8;
                mma16816(acc, qa[2 * b], h2_as_u32(q4_lo_pair(w)), h2_as_u32(q4_hi_pair(w)));
                mma16816(acc, qa[2 * b + 1], h2_as_u32(q4_lo_pair(w2)), h2_as_u32(q4_hi_pair(w2)));
                const float2 d = __half22float2(u32_as_h2(kd[b]));
                s0 = fmaf(acc[0] + acc[2], d.x, s0);
                s1 = fmaf(acc[1] + acc[3], d.y, s1);
            }
        } else {
            uint4 kwv[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) kwv[c] = lds128(tp + L::KC + c * 512 + lane * 16);
            const uint4 ks = lds128(tp + L::KS + t * 16);
            const uint32_t kd[4] = {ks.x, ks.y, ks.z, ks.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                const uint32_t ws[4] = {kwv[q].x, kwv[q].y, kwv[q].z, kwv[q].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t wb = ws[j] ^ 0x80808080u;
                    mma16816(acc, qa[4 * q + j], h2_as_u32(i8_pair(wb, 0x4140u)), h2_as_u32(i8_pair(wb, 0x4342u)));
                }
                const float2 d = __half22float2(u32_as_h2(kd[q]));
                s0 = fmaf(acc[0] + acc[2], d.x, s0);
                s1 = fmaf(acc[1] + acc[3], d.y, s1);
            }
        }
        if (MASK) {
            if (2 * t >= valid) s0 = -INFINITY;
            if (2 * t + 1 >= valid) s1 = -INFINITY;
        }
        // ---- online softmax for head g ---------------------------------------
        float mx = fmaxf(s0, s1);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const bool grow = mx > m_run;
        if (__any_sync(0xffffffffu, grow)) {
            const float m_new = grow ? mx : m_run;
            const float alpha = exp2f(m_run - m_new);     // 0 on the first tile (m_run = -inf)
            l_run *= alpha;
            m_run = m_new;
            const float a_lo = __shfl_sync(0xffffffffu, alpha, 8 * t);       // head 2t
            const float a_hi = __shfl_sync(0xffffffffu, alpha, 8 * t + 4);   // head 2t+1
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                o[i][0] *= a_lo; o[i][2] *= a_lo;
                o[i][1] *= a_hi; o[i][3] *= a_hi;
            }
        }
        const float p0 = exp2f(s0 - m_run), p1 = exp2f(s1 - m_run);
        l_run += p0 + p1;
        // ---- values: o[dims][heads] += V^T P ------------------------------------
        if constexpr (L::VP == PART_Q4) {
            const uint4 vw0 = lds128(tp + L::VC + lane * 16);
            const uint4 vw1 = lds128(tp + L::VC + 512 + lane * 16);
            const uint4 vs0 = lds128(tp + L::VS + t * 32);
            const uint4 vs1 = lds128(tp + L::VS + t * 32 + 16);
            const uint32_t vw[8] = {vw0.x, vw0.y, vw0.z, vw0.w, vw1.x, vw1.y, vw1.z, vw1.w};
            const uint32_t vd[8] = {vs0.x, vs0.y, vs0.z, vs0.w, vs1.x, vs1.y, vs1.z, vs1.w};
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                const float2 d = __half22float2(u32_as_h2(vd[b]));
                float x0 = p0 * d.x, x1 = p1 * d.y;
                if (MASK) {           // scales of tokens past the end may hold anything
                    if (2 * t >= valid) x0 = 0.f;
                    if (2 * t + 1 >= valid) x1 = 0.f;
                }
                uint32_t hi, lo;
                split_pair(x0, x1, hi, lo);
                const uint32_t w = vw[b], w2 = vw[b] >> 8;
                const uint32_t a0 = h2_as_u32(q4_lo_pair(w)), a1 = h2_as_u32(q4_hi_pair(w));
                const uint32_t c0 = h2_as_u32(q4_lo_pair(w2)), c1 = h2_as_u32(q4_hi_pair(w2));
                const uint32_t A0[4] = {a0, a1, a0, a1};
                const uint32_t A1[4] = {c0, c1, c0, c1};
                mma16816(o[2 * b], A0, hi, lo);
                mma16816(o[2 * b + 1], A1, hi, lo);
            }
        } else {
            const uint4 vs = lds128(tp + L::VS + t * 16);
            const uint32_t vd[4] = {vs.x, vs.y, vs.z, vs.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 vw = lds128(tp + L::VC + q * 512 + lane * 16);
                const uint32_t ws[4] = {vw.x, vw.y, vw.z, vw.w};
                const float2 d = __half22float2(u32_as_h2(vd[q]));
                float x0 = p0 * d.x, x1 = p1 * d.y;
                if (MASK) {
                    if (2 * t >= valid) x0 = 0.f;
                    if (2 * t + 1 >= valid) x1 = 0.f;
                }
                uint32_t hi, lo;
                split_pair(x0, x1, hi, lo);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t wb = ws[j] ^ 0x80808080u;
                    const uint32_t a0 = h2_as_u32(i8_pair(wb, 0x4140u)), a1 = h2_as_u32(i8_pair(wb, 0x4342u));
                    const uint32_t A[4] = {a0, a1, a0, a1};
                    mma16816(o[4 * q + j], A, hi, lo);
                }
            }
        }
    }

    // Per-warp result into the CTA merge buffers.
    __device__ __forceinline__ void warp_stats(int lane, float &m, float &l) {
        float lr = l_run;
        lr += __shfl_xor_sync(0xffffffffu, lr, 1);
        lr += __shfl_xor_sync(0xffffffffu, lr, 2);
        m = m_run;
        l = lr;
    }
    // Add this warp's o (scaled per head) into o_s[8][256].
    __device__ __forceinline__ void accumulate(float *o_s, const float *scale, int lane) {
        const int g = lane >> 2, t = lane & 3;
        const float sc0 = scale[2 * t], sc1 = scale[2 * t + 1];
#pragma unroll
        for (int mt = 0; mt < 16; ++mt) {
            const int d0 = 16 * mt + g;
            atomicAdd(o_s + (2 * t) * D + d0, o[mt][0] * sc0);
            atomicAdd(o_s + (2 * t + 1) * D + d0, o[mt][1] * sc1);
            atomicAdd(o_s + (2 * t) * D + d0 + 8, o[mt][2] * sc0);
            atomicAdd(o_s + (2 * t + 1) * D + d0 + 8, o[mt][3] * sc1);
        }
    }
    // head whose (m, l) this lane reports; -1 if none
    __device__ __forceinline__ int stats_head(int lane) { return (lane & 3) == 0 ? (lane >> 2) : -1; }
};

// ---------------------------------------------------------------------------
// CUDA-core compute policy (control).  Lane l owns 8 dims of K and 8 dims of V
// for all heads; partial scores are reduced across the warp by a butterfly
// reduce-scatter so that lane l ends with tokens l/4, heads 2(l%4), 2(l%4)+1.
// ---------------------------------------------------------------------------
template <int FMT, int GT> struct AluCompute {
    using L = TileLayout<FMT>;
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

    __device__ __forceinline__ void warp_stats(int lane, float &m, float &l) {
        // lanes 0..3 report heads 2l, 2l+1 via the caller; reduce l over tokens
        float l0 = l_run[0], l1 = l_run[1];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, off);
            l1 += __shfl_xor_sync(0xffffffffu, l1, off);
        }
        l_run[0] = l0;
        l_run[1] = l1;
        m = m_run[0];
        l = l0;
    }
    __device__ __forceinline__ void accumulate(float *o_s, const float *scale, int lane) {
#pragma unroll
        for (int h = 0; h < GT; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) atomicAdd(o_s + h * D + vdim(lane, e), o[h][e] * scale[h]);
    }
};

// ---------------------------------------------------------------------------
// Kernel scaffold
// ---------------------------------------------------------------------------
template <int FMT, bool TC, int GT>
__global__ void __launch_bounds__(NTHREADS, 1)
decode_kernel(const uint8_t *__restrict__ pool, PoolGeom geo, int layer, const float *__restrict__ q,
              const int32_t *__restrict__ page_table, int max_pages, const int32_t *__restrict__ plan, int n_q_heads,
              int G, float *__restrict__ ws, int32_t *status) {
    using L = TileLayout<FMT>;
    using S = Smem<FMT>;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + S::BAR_OFF);
    uint64_t *empty = full + S::NS;
    int *stage_ok = reinterpret_cast<int *>(empty + S::NS);
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.x;
    const int32_t *U = plan + PLAN_HEADER + 4 * u;
    const int seq = U[0], kvh = U[1], t0 = U[2], t1 = U[3];
    float *wsu = ws + (size_t)u * ws_unit_floats(G);

    const bool plan_ok = plan[0] == PLAN_MAGIC && seq >= 0 && seq < plan[2] && kvh >= 0 && kvh < geo.n_kv_heads &&
                         t0 >= 0 && t0 < t1 && (t0 % STEP_TOKENS) == 0 && t1 <= max_pages * PAGE;
    if (!plan_ok) {   // write an empty partial so that the merge ignores this unit
        if (threadIdx.x == 0) status_or(status, KVQ_STATUS_BAD_PLAN);
        for (int i = threadIdx.x; i < G * D; i += blockDim.x) wsu[i] = 0.f;
        if (threadIdx.x < 8) {
            wsu[G * D + threadIdx.x] = -INFINITY;
            wsu[G * D + 8 + threadIdx.x] = 0.f;
        }
        return;
    }
    const int n_steps = (t1 - t0 + STEP_TOKENS - 1) / STEP_TOKENS;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S::NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], NW);
        }
        s_abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const uint8_t *head_base = pool + (int64_t)layer * geo.layer_stride + (int64_t)kvh * geo.page_bytes;
    const int32_t *pt = page_table + (int64_t)seq * max_pages;

    if (warp == NW) {
        // ------------------------------ producer --------------------------------
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            for (int i = 0; i < n_steps; ++i) {
                const int si = i % S::NS;
                if (i >= S::NS) {
                    if (!mbar_wait_bounded(&empty[si], ((i / S::NS) - 1) & 1, WAIT_LIMIT_NS)) {
                        status_or(status, KVQ_STATUS_TIMEOUT);
                        atomicExch(&s_abort, 1);
                        break;
                    }
                }
                const int tok = t0 + i * STEP_TOKENS;
                const int slot = pt[tok >> 8];
                if (slot < 0 || slot >= geo.n_pages) {
                    status_or(status, KVQ_STATUS_BAD_SLOT);
                    stage_ok[si] = 0;
                    mbar_arrive(&full[si]);
                    continue;
                }
                stage_ok[si] = 1;
                const uint8_t *src = head_base + (int64_t)slot * geo.slot_stride + ((tok & 255) >> 3) * L::BYTES;
                mbar_arrive_expect_tx(&full[si], S::STAGE_BYTES);
                bulk_g2s(smem + si * S::STAGE_BYTES, src, S::STAGE_BYTES, &full[si], pol);
            }
        }
    } else {
        // ------------------------------ consumers -------------------------------
        float *pbuf = reinterpret_cast<float *>(smem + S::BAR_OFF + S::NS * 16 + S::NS * 4 + 16);  // unused by MMA
        (void)pbuf;
        const float *qg = q + ((int64_t)seq * n_q_heads + (int64_t)kvh * G) * D;
        __shared__ float p_bufs[TC ? 1 : NW * 64];
        typename std::conditional<TC, MmaCompute<FMT>, AluCompute<FMT, GT>>::type C;
        if constexpr (TC) C.init(qg, G, lane);
        else C.init(qg, G, lane, p_bufs + warp * 64);

        for (int i = 0; i < n_steps; ++i) {
            const int si = i % S::NS;
            if (!mbar_wait_bounded(&full[si], (i / S::NS) & 1, WAIT_LIMIT_NS)) {
                if (lane == 0) { status_or(status, KVQ_STATUS_TIMEOUT); atomicExch(&s_abort, 1); }
                break;
            }
            const int tile_tok = t0 + i * STEP_TOKENS + warp * TILE;
            const int valid = t1 - tile_tok;
            if (stage_ok[si] && valid > 0) {
                const uint8_t *tp = smem + si * S::STAGE_BYTES + warp * L::BYTES;
                if (valid >= TILE) C.template tile<false>(tp, TILE, lane);
                else C.template tile<true>(tp, valid, lane);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[si]);
        }

        // ------------------------------ CTA merge -------------------------------
        asm volatile("bar.sync 1, %0;" ::"r"(NW * 32));           // all consumers done with the ring
        float *o_s = reinterpret_cast<float *>(smem);             // [8][256]
        float *m_s = o_s + 8 * D;                                 // [NW][8]
        float *l_s = m_s + NW * 8;                                // [NW][8]
        float *M_s = l_s + NW * 8;                                // [8]
        float *sc_s = M_s + 8;                                    // [8] (unused slot)
        (void)sc_s;
        for (int i = threadIdx.x; i < 8 * D; i += NW * 32) o_s[i] = 0.f;
        {
            float m, l;
            C.warp_stats(lane, m, l);
            if constexpr (TC) {
                const int h = C.stats_head(lane);
                if (h >= 0) { m_s[warp * 8 + h] = m; l_s[warp * 8 + h] = l; }
            } else {
                if (lane < 4) {
                    m_s[warp * 8 + 2 * lane] = C.m_run[0];
                    m_s[warp * 8 + 2 * lane + 1] = C.m_run[1];
                    l_s[warp * 8 + 2 * lane] = C.l_run[0];
                    l_s[warp * 8 + 2 * lane + 1] = C.l_run[1];
                }
            }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(NW * 32));
        if (threadIdx.x < 8) {
            float M = -INFINITY;
            for (int w = 0; w < NW; ++w) M = fmaxf(M, m_s[w * 8 + threadIdx.x]);
            M_s[threadIdx.x] = M;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(NW * 32));
        float scale[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            const float mw = m_s[warp * 8 + h];
            scale[h] = mw == -INFINITY ? 0.f : exp2f(mw - M_s[h]);
        }
        C.accumulate(o_s, scale, lane);
        asm volatile("bar.sync 1, %0;" ::"r"(NW * 32));
        // partial: o[G][256], m[8], l[8]
        for (int i = threadIdx.x; i < G * D; i += NW * 32) wsu[i] = o_s[i];
        if (threadIdx.x < 8) {
            const int h = threadIdx.x;
            float Lh = 0.f;
            for (int w = 0; w < NW; ++w) {
                const float mw = m_s[w * 8 + h];
                if (mw != -INFINITY) Lh += l_s[w * 8 + h] * exp2f(mw - M_s[h]);
            }
            wsu[G * D + h] = M_s[h];
            wsu[G * D + 8 + h] = Lh;
        }
    }
}

template <int FMT, bool TC, int GT>
cudaError_t launch_one(const uint8_t *pool, const PoolGeom &geo, int layer, const float *q, const int32_t *pt,
                       int max_pages, const int32_t *plan, const kvq_plan_info &info, float *ws, int32_t *status,
                       cudaStream_t s) {
    constexpr int SMEM = Smem<FMT>::TOTAL;
    auto k = decode_kernel<FMT, TC, GT>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    k<<<info.n_units, NTHREADS, SMEM, s>>>(pool, geo, layer, q, pt, max_pages, plan,
                                           info.n_kv_heads * info.group, info.group, ws, status);
    return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_fmt(bool tc, const uint8_t *pool, const PoolGeom &geo, int layer, const float *q,
                       const int32_t *pt, int max_pages, const int32_t *plan, const kvq_plan_info &info, float *ws,
                       int32_t *status, cudaStream_t s) {
    if (tc) return launch_one<FMT, true, 8>(pool, geo, layer, q, pt, max_pages, plan, info, ws, status, s);
    switch (info.group) {
    case 4: return launch_one<FMT, false, 4>(pool, geo, layer, q, pt, max_pages, plan, info, ws, status, s);
    case 6: return launch_one<FMT, false, 6>(pool, geo, layer, q, pt, max_pages, plan, info, ws, status, s);
    default: return launch_one<FMT, false, 8>(pool, geo, layer, q, pt, max_pages, plan, info, ws, status, s);
    }
}

}  // namespace

cudaError_t launch_decode(int fmt, bool tensor_cores, const uint8_t *pool, const PoolGeom &geo, int layer,
                          const float *q, const int32_t *page_table, int max_pages, const int32_t *plan,
                          const kvq_plan_info &info, float *ws, int32_t *status, cudaStream_t s) {
    switch (fmt) {
    case KVQ_INT8:
        return launch_fmt<KVQ_INT8>(tensor_cores, pool, geo, layer, q, page_table, max_pages, plan, info, ws, status, s);
    case KVQ_Q4_0:
        return launch_fmt<KVQ_Q4_0>(tensor_cores, pool, geo, layer, q, page_table, max_pages, plan, info, ws, status, s);
    default:
        return launch_fmt<KVQ_K8V4>(tensor_cores, pool, geo, layer, q, page_table, max_pages, plan, info, ws, status, s);
    }
}

}  // namespace kvq
