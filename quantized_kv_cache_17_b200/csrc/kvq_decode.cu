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
// The product kernel (decode_umma_kernel) runs the two contractions on the
// fifth-generation tensor cores (tcgen05): K and V codes are unpacked once into
// tensor memory as exact fp16 values, the query and the softmax weights are
// the shared-memory operands, and the score and output accumulators live in
// tensor memory; the per-block scales are applied to the fp32 block sums
// (scores) and folded into the weights (values).  A CUDA-core kernel with the
// same data path (decode_alu_kernel) is kept as the measured control.
//
// Data path (both kernels): a copy warp streams the unit's tokens in 64-token
// steps (8 tiles, contiguous inside one page block) with 1-D bulk copies into
// a ring of shared-memory stages guarded by full/empty mbarriers.  Each unit
// writes one partial (o[G][256] unnormalised, m[8], l[8]; scores in log2
// units), then, with the combine fused in, takes part in the merge of its
// group.
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
constexpr int MH_MAX_UNITS = 256;                 // units per group on the cooperative merge path
// floats of the cooperative merge's scratch for NTH threads (merge_head)
__host__ __device__ constexpr int mh_smem_floats(int nth) { return MH_MAX_UNITS + (nth / 64) * D + D + 1; }
constexpr int MH_SMEM_MAX = mh_smem_floats(16 * 32);

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

__device__ __forceinline__ uint32_t u4_at(const uint4 &v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
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

    // Lane l owns dims 8l .. 8l+7 of K and of V.  Dim of K element n (nibble n
    // of the lane's q4 word, byte n of its int8 bytes) and of V element e.
    __device__ __forceinline__ static int kdim(int lane, int n) {
        return L::KP == PART_Q4 ? 8 * lane + 2 * (n & 3) + (n >> 2) : 8 * lane + n;
    }
    __device__ __forceinline__ static int vdim(int lane, int e) { return 8 * lane + e; }

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
                const int b = lane >> 2;
                const uint32_t w = lds32(tp + L::KC + 128 * r + 16 * (b ^ r) + 4 * (lane & 3));
#pragma unroll
                for (int n = 0; n < 8; ++n) kv[n] = q4f(w, n);
                dk = __half2float(*reinterpret_cast<const __half *>(tp + L::KS + 16 * r + 2 * b));
            } else {
                const uint2 w = lds64(tp + L::KC + 256 * r + 16 * ((lane >> 1) ^ r) + 8 * (lane & 1));
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    kv[n] = i8f(w.x, n);
                    kv[4 + n] = i8f(w.y, n);
                }
                dk = __half2float(*reinterpret_cast<const __half *>(tp + L::KS + 8 * r + 2 * (lane >> 3)));
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
        // ---- values: the lane's 8 dims hold the tile's 8 tokens each ------------
        uint32_t vw[8];
        if constexpr (L::VP == PART_Q4) {
            const uint4 a = lds128(tp + L::VC + 32 * lane), b = lds128(tp + L::VC + 32 * lane + 16);
            vw[0] = a.x; vw[1] = a.y; vw[2] = a.z; vw[3] = a.w; vw[4] = b.x; vw[5] = b.y; vw[6] = b.z; vw[7] = b.w;
        }
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            float vv[8];
            float dv;
            if constexpr (L::VP == PART_Q4) {
#pragma unroll
                for (int e = 0; e < 8; ++e) vv[e] = q4f(vw[e], 4 * (rr & 1) + (rr >> 1));
                dv = __half2float(*reinterpret_cast<const __half *>(tp + L::VS + 16 * rr + 2 * (lane >> 2)));
            } else {
                if ((rr & 3) == 0) {          // tokens 0-3, then 4-7: word rr / 4 of each dim's 8 bytes
#pragma unroll
                    for (int e = 0; e < 8; ++e) vw[e] = lds32(tp + L::VC + 64 * lane + 8 * e + 4 * (rr >> 2));
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) vv[e] = i8f(vw[e], rr & 3);
                dv = __half2float(*reinterpret_cast<const __half *>(tp + L::VS + 8 * rr + 2 * (lane >> 3)));
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
                    kvh < A.geo.n_kv_heads && t0 >= 0 && t0 < t1 && (t0 % PLAN_TOKENS) == 0 &&
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
// bulk copies.  before_last (optional): an mbarrier phase to wait for before
// the last step is requested (in a decode step, the pool write of the newest
// token, which that step holds).  Before the warp exits, every copy it issued
// has landed.
template <int NS, int STAGE_BYTES, int TILE_BYTES>
__device__ __forceinline__ void copy_loop(const DecodeArgs &A, uint8_t *smem, uint64_t *full, uint64_t *empty,
                                          int *stage_ok, int seq, int kvh, int t0, int n_steps, int lane,
                                          uint64_t *before_last = nullptr) {
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
        if (lane == 0 && !stop) {
            const int si = i % NS;
            if (i == n_steps - 1 && before_last && !mbar_wait_bounded(before_last, 0, WAIT_LIMIT_NS))
                status_or(A.status, KVQ_STATUS_TIMEOUT);
            if (i >= NS && !mbar_wait_bounded(&empty[si], ((i / NS) - 1) & 1, WAIT_LIMIT_NS)) {
                status_or(A.status, KVQ_STATUS_TIMEOUT);
                stop = true;
            } else if (slot < 0 || slot >= A.geo.n_pages) {
                status_or(A.status, KVQ_STATUS_BAD_SLOT);
                stage_ok[si] = 0;
                mbar_arrive(&full[si]);
                ++issued;
            } else {
                stage_ok[si] = 1;
                const uint8_t *src = head_base + (int64_t)slot * A.geo.slot_stride + ((tok & 255) >> 3) * TILE_BYTES;
                mbar_arrive_expect_tx(&full[si], STAGE_BYTES);
                bulk_g2s(smem + si * STAGE_BYTES, src, STAGE_BYTES, &full[si], pol);
                ++issued;
            }
        }
        __syncwarp();
    }
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
// In a decode step, one warp of the CTA whose unit ends a (sequence, KV head)
// range encodes the range's newest token into the pool, as kv_append would,
// and makes the write visible to the bulk copies that read the pool later (the
// copy of the step that holds the token waits for it).  Out of line, so that
// its registers do not shape the allocation of the warp's main loop.
template <int FMT>
__device__ __noinline__ void step_encode_token(const DecodeArgs &A, int seq, int kvh, int pos, int lane) {
    const int64_t row = ((int64_t)seq * A.geo.n_kv_heads + kvh) * D;
    append_token<FMT>(const_cast<uint8_t *>(A.pool), A.geo, A.layer, A.k_new + row, A.v_new + row, seq, kvh, pos,
                      A.page_table, A.max_pages, A.status, lane);
    __threadfence();
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncwarp();
}
// Warps of the softmax group copy the query heads h = first, first + stride, ... into
// q_s, rotating them (ROTATE) in a decode step.
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
// Tensor-core kernel (tcgen05): configuration
// ---------------------------------------------------------------------------
template <int FMT> struct UmCfg {
    using L = TileLayout<FMT>;
    static constexpr bool KQ4 = L::KP == PART_Q4, VQ4 = L::VP == PART_Q4;
    static constexpr int NKB = KQ4 ? 8 : 4;              // K scale blocks per token (32 or 64 dims each)
    static constexpr int NVB = VQ4 ? 8 : 4;              // V scale blocks per token
    static constexpr int KSPB = 16 / NKB;                // 16-dim MMA k-steps per K block
    static constexpr int VBM = NVB / 2;                  // V blocks per 128-dim M-tile
    static constexpr int NPV = VBM * 16;                 // value columns per M-tile: (group, block, hi/lo, 4 heads)
    static constexpr float KOFF = KQ4 ? 8.f : 128.f;     // code offset of the K codes as stored
    static constexpr int STEP_BYTES = 8 * L::BYTES;      // one 64-token copy step (8 tiles)
#ifndef KVQ_UMMA_STAGES
    static constexpr int NS = FMT == KVQ_Q4_0 ? 6 : (FMT == KVQ_INT8 ? 4 : 5);   // copy ring steps
#else
    static constexpr int NS = KVQ_UMMA_STAGES;
#endif
    // warp roles: softmax groups 0-3 (heads 0-3) and 4-7 (heads 4-7), K 8-11, V 12-15, then
    // the copy warp and the two MMA issuers (warp 19 idles)
    static constexpr int W_K = 8, W_V = 12, W_COPY = 16, W_QK = 17, W_PV = 18;
    static constexpr int NTHREADS = 20 * 32;
    static constexpr int NCT = 16 * 32;                  // threads of the unit's merge: warps 0-15
    // tensor memory columns
    static constexpr int T_KOP = 0;                      // K of a 128-token stage: lane = token, col = dim pair
    static constexpr int T_SQK = 128;                    // scores: 16 columns per K block
    static constexpr int T_VOP = T_SQK + 16 * NKB;       // 2 slots x 64: V of 64 tokens, lane = dim
    static constexpr int T_O = T_VOP + 128;              // output accumulators: 2 M-tiles x NPV
    static constexpr int TMEM_COLS = 512;
    static_assert(T_O + 2 * NPV <= TMEM_COLS, "tensor memory budget");
    // shared memory
    static constexpr int RING = NS * STEP_BYTES;
    static constexpr int MERGE = (COMBINE_SMEM > MH_SMEM_MAX ? COMBINE_SMEM : MH_SMEM_MAX) * 4;
    static constexpr int DATA = RING > MERGE ? RING : MERGE;
    static constexpr int BQK_OFF = (DATA + 1023) & ~1023;     // query operand: 16 k-steps x [16 x 16] fp16
    static constexpr int BPV_OFF = BQK_OFF + 16 * 512;
    static constexpr int BPV_SLOT = 2 * NPV * 256;            // (2 NPV / 8) n-groups x 128 tokens x 16 B
    static constexpr int SIDE_OFF = BPV_OFF + 2 * BPV_SLOT;   // [2 slots][dK | dV][128 tokens] x 16 B
    static constexpr int RED_OFF = SIDE_OFF + 2 * 2 * 128 * 16;
    static constexpr int RED_FLOATS = 2 * 2 * 4 * 4 + 2 * 2 * 4 + 8;   // per group [2][4 warps][4] + [2][4] ints, query max
    static constexpr int KC_OFF = RED_OFF + RED_FLOATS * 4;   // K offset terms [8 blocks][8 heads] floats
    static constexpr int BAR_OFF = KC_OFF + 64 * 4;
    static constexpr int NBAR = 2 * NS + 20;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;       // stage_ok[NS], step_ok[2][2], tmem base, s_last
    static constexpr int TOTAL = MISC_OFF + NS * 4 + 4 * 4 + 8;
    static_assert(TOTAL <= 227 * 1024, "shared memory budget");
    static_assert(2 * BPV_SLOT >= KVQ_MAX_GROUP * D * 4, "the query is staged in the value-operand buffers");
    // instruction descriptors: scores (M = 128 tokens, N = 16) and values (M = 128 dims, N = NPV, B MN-major)
    static constexpr uint32_t IDESC_QK = umma_idesc_f16(128, 16, 0);
    static constexpr uint32_t IDESC_PV = umma_idesc_f16(128, NPV, 1);
};

// mbarriers of the tensor-core kernel
struct UmBars {
    uint64_t *full, *empty;          // [NS] copy ring
    uint64_t *kop_full;              // [2] K dims 0-127 / 128-255 of the stage are in TMEM (K warps)
    uint64_t *kq_done;               // [2] the score MMAs of those dims are complete (commit)
    uint64_t *sqk_free;              // [2] both softmax groups have read those scores
    uint64_t *side_full;             // [2] a stage's scales and step flags are in shared memory (K warps)
    uint64_t *vop_full, *vop_free;   // [2] V of a 64-token half in TMEM / its MMAs are complete
    uint64_t *bpv_full, *bpv_free;   // [2] P' of a stage in shared memory / its MMAs are complete
    uint64_t *bqk_ready;             // the query operand is in shared memory
    uint64_t *enc_done;              // decode step: the newest token is in the pool
    uint64_t *drain;                 // [2] final commits of the two MMA issuers
};

// 4-bit codes as exact fp16 subnormals (code x 2^-24) from a word whose nibble
// n holds element 2(n&3) + (n>>2): pairs (0,1), (2,3), (4,5), (6,7), the second
// and fourth at 16 x code x 2^-24.
__device__ __forceinline__ void q4_word_sub(uint32_t w, uint32_t *o) {
    o[0] = w & 0x000F000Fu;
    o[1] = w & 0x00F000F0u;
    o[2] = (w >> 8) & 0x000F000Fu;
    o[3] = (w >> 8) & 0x00F000F0u;
}
// int8 codes (two's complement) as exact fp16 subnormals (code + 128) x 2^-24:
// two pairs of consecutive bytes.
__device__ __forceinline__ void i8_word_sub(uint32_t w, uint32_t *o) {
    const uint32_t wb = w ^ 0x80808080u;
    o[0] = __byte_perm(wb, 0u, 0x4140u);
    o[1] = __byte_perm(wb, 0u, 0x4342u);
}
// (c - 8) and c as exact fp16 values (V operand, normal numbers)
__device__ __forceinline__ void q4_word_pairs(uint32_t w, uint32_t *o) {
    o[0] = h2_as_u32(q4_lo_pair(w));
    o[1] = h2_as_u32(q4_hi_pair(w));
    o[2] = h2_as_u32(q4_lo_pair(w >> 8));
    o[3] = h2_as_u32(q4_hi_pair(w >> 8));
}
__device__ __forceinline__ void i8_word_pairs(uint32_t w, uint32_t *o) {
    const uint32_t wb = w ^ 0x80808080u;
    o[0] = h2_as_u32(i8_pair(wb, 0x4140u));
    o[1] = h2_as_u32(i8_pair(wb, 0x4342u));
}

// p' = 2^(x - m - PSHIFT): the running max m moves only when a score exceeds it
// by more than RESCALE_SLACK (log2 units), so p' <= 2^(RESCALE_SLACK - PSHIFT) = 8.
constexpr float RESCALE_SLACK = 8.f;
constexpr float PSHIFT = 5.f;

// The value weights P' = p' dV 2^sigma go to the tensor cores as fp16 (hi, lo)
// pairs.  sigma is a power of two for the whole unit (per softmax group), set
// from the largest V scale exponent e seen so far (sigma = 26 - max(e, 1)), so
// that every |P'| < 8 * 2^12 stays in fp16 range and the weights of the tokens
// with the largest scales keep the full pair precision even when all V values
// are tiny; the output is multiplied by 2^-sigma at the end.  When a later
// stage brings a larger scale, sigma drops and the accumulators are rescaled
// like a moved running max.
__device__ __forceinline__ int um_sigma(int e) { return 26 - (e > 1 ? e : 1); }
// (2^a, 2^a) and (2^b, 2^b) as fp16 pairs with a + b = sigma, each factor in range
__device__ __forceinline__ void um_sigma_factors(int sig, uint32_t &fa, uint32_t &fb) {
    const int a = sig > 15 ? 15 : (sig < -14 ? -14 : sig);
    const uint32_t ha = (uint32_t)(a + 15) << 10, hb = (uint32_t)(sig - a + 15) << 10;
    fa = ha | (ha << 16);
    fb = hb | (hb << 16);
}

// ---------------------------------------------------------------------------
// Tensor-core kernel.  One CTA per plan unit, 20 warps:
//  warps 0-7   (S) two softmax warp groups, heads 0-3 and 4-7: thread t of a
//              group owns token t of each 128-token stage (TMEM lane t); it
//              reads its scores from TMEM, applies the K scales and removes the
//              code offset, runs the online softmax of its 4 heads (a running
//              max shared by the group, moved only in steps larger than
//              RESCALE_SLACK, the output accumulators rescaled in TMEM when it
//              moves) and writes its part of P' = p dV (fp16 hi/lo) to shared
//              memory.
//  warps 8-11  (K) unpack the stage's K codes (thread = token) into TMEM as
//              exact fp16 subnormals, dims 0-127 and 128-255 as two halves with
//              their own barriers, and hand the token's scales to S.
//  warps 12-15 (V) unpack the V codes of each 64-token half (thread = dims d
//              and 128 + d) into TMEM as exact fp16 (c - offset).
//  warp 16     copy: 64-token steps from the pool into a ring of shared-memory
//              stages (1-D bulk copies, full / empty mbarriers).
//  warp 17     issues the score MMAs: per K block, S[128 tokens x (group, hi/lo,
//              4 heads)] = K (TMEM) x Q (shared memory), 8 per half stage.
//  warp 18     issues the value MMAs: per 128-dim M-tile, O[128 dims x (group,
//              block, hi/lo, 4 heads)] += V (TMEM) x P' (shared memory), 8 per
//              64-token half; in a decode step it first encodes the newest token.
// Every wait has a time limit; past it the kernel records KVQ_STATUS_TIMEOUT,
// drains its MMAs, frees its tensor memory and finishes.
// ---------------------------------------------------------------------------

// S (both groups, 256 threads): the group's query as the score MMA's B operand,
// [k-step][16 rows][16 dims] fp16, row n = 8 g + 4 hl + (h & 3) for head h of
// group g = h / 4 and half hl (0 = fp16 value, 1 = residual), K-major without
// swizzle: element (n, k) of k-step ks at ks*512 + (n/8)*256 + (k/8)*128 +
// (n%8)*16 + (k%8)*2.  Values are q * log2(e)/16 * 2^kq / f, kq putting the
// group's largest |value| into [2^12, 2^13) so that the fp16 residual keeps its
// precision and f = 16 for the dims whose 4-bit codes sit at 16 x code (dim % 8
// in {2, 3, 6, 7}), else 1.  Also the K offset terms kc[b][h] = OFF 2^-24
// sum over block b of the represented query, which the scores subtract.
// Returns 2^(24 - kq), the factor from the score accumulators (codes x 2^-24,
// query x 2^kq) to log2 units.
template <int FMT>
__device__ __noinline__ float um_build_query(const float *q_s, int G, uint8_t *bqk, float *kc, float *red, int t) {
    using C = UmCfg<FMT>;
    const int warp = t >> 5, lane = t & 31;
    float mx = 0.f;
    for (int i = t; i < G * D; i += 256) mx = fmaxf(mx, fabsf(q_s[i] * QSCALE));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    asm volatile("bar.sync 5, 256;" ::: "memory");
    mx = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) mx = fmaxf(mx, red[w]);
    int kq = 0;
    if (mx > 0.f) kq = min(max(12 - ((int)((__float_as_uint(mx) >> 23) & 255u) - 127), -60), 60);
    const float sc = __int_as_float((127 + kq) << 23);
    for (int wi = t; wi < 16 * 16 * 8; wi += 256) {        // 32-bit words: (k-step, row n, dim pair kp)
        const int ks = wi >> 7, n = (wi >> 3) & 15, kp = wi & 7;
        const int h = 4 * (n >> 3) + (n & 3), hl = (n >> 2) & 1;
        const float f = (C::KQ4 && (kp & 1)) ? 0.0625f : 1.f;
        float x0 = 0.f, x1 = 0.f;
        if (h < G) {
            x0 = ((q_s[h * D + 16 * ks + 2 * kp] * QSCALE) * sc) * f;
            x1 = ((q_s[h * D + 16 * ks + 2 * kp + 1] * QSCALE) * sc) * f;
        }
        uint32_t hi, lo;
        split_pair(x0, x1, hi, lo);
        *reinterpret_cast<uint32_t *>(bqk + ks * 512 + (n >> 3) * 256 + (kp >> 2) * 128 + (n & 7) * 16 +
                                      (kp & 3) * 4) = hl ? lo : hi;
    }
    // offset terms, summed in a fixed order from the same represented values
    if (t < 8 * 8) {
        const int b = t >> 3, h = t & 7;
        float sum = 0.f;
        if (h < G && b < C::NKB) {
            const int bd = D / C::NKB;
            for (int d = b * bd; d < (b + 1) * bd; d += 2) {
                const float f = (C::KQ4 && ((d >> 1) & 1)) ? 0.0625f : 1.f;
                uint32_t hi, lo;
                split_pair(((q_s[h * D + d] * QSCALE) * sc) * f, ((q_s[h * D + d + 1] * QSCALE) * sc) * f, hi, lo);
                const float2 a = __half22float2(u32_as_h2(hi)), c = __half22float2(u32_as_h2(lo));
                sum += ((a.x + c.x) + (a.y + c.y)) / f;
            }
        }
        kc[b * 8 + h] = C::KOFF * 5.9604644775390625e-08f * sum;     // OFF 2^-24 sum
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic writes -> tensor-core reads
    asm volatile("bar.sync 5, 256;" ::: "memory");
    return __int_as_float((127 + 24 - kq) << 23);
}

// Bounded wait by one thread; a wait past its limit records
// KVQ_STATUS_TIMEOUT and sets `to`, and every later wait then fails at once.
__device__ __forceinline__ bool um_wait(uint64_t *bar, uint32_t parity, const DecodeArgs &A, bool &to) {
    if (to) return false;
    if (!mbar_wait_bounded(bar, parity, WAIT_LIMIT_NS)) {
        status_or(A.status, KVQ_STATUS_TIMEOUT);
        to = true;
        return false;
    }
    return true;
}
// The same by all 32 lanes of a warp, with one outcome for the whole warp (the
// tensor-memory loads and stores that follow are warp-collective).
__device__ __forceinline__ bool um_wait_warp(uint64_t *bar, uint32_t parity, const DecodeArgs &A, bool &to) {
    bool ok = !to && mbar_wait_bounded(bar, parity, WAIT_LIMIT_NS);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
        if (!to && (threadIdx.x & 31) == 0) status_or(A.status, KVQ_STATUS_TIMEOUT);
        to = true;
    }
    return ok;
}

// K: thread t unpacks token t of each stage: dims 0-127 (words [0, NW/2)) then
// 128-255, each half into its TMEM columns once the previous stage's score MMAs
// of that half are complete.
template <int FMT>
__device__ __forceinline__ void um_k_role(const DecodeArgs &A, uint8_t *smem, const UmBars &B, const int *stage_ok,
                                          int *step_ok, uint32_t tmem, int n_steps, int n_stages, int t, bool &to) {
    using L = TileLayout<FMT>;
    using C = UmCfg<FMT>;
    constexpr int NW = C::KQ4 ? 32 : 64;              // code words per token
    constexpr int HW = NW / 2;                        // words per half (dims 0-127 / 128-255)
    constexpr int TB = C::KQ4 ? 128 : 256;            // bytes per token
    const int lane = t & 31, r = t & 7;
    const uint32_t tl = tmem + ((uint32_t)(t & ~31) << 16);
    for (int s = 0; s < n_stages; ++s) {
        const int step = 2 * s + (t >> 6);
        const bool has = step < n_steps;
        const int slot = step % C::NS;
        uint4 sk = make_uint4(0u, 0u, 0u, 0u), sv = make_uint4(0u, 0u, 0u, 0u);
        int ok = 0;
        const uint8_t *tile = smem + slot * C::STEP_BYTES + ((t & 63) >> 3) * L::BYTES;
        if (has) {
            if (!um_wait_warp(&B.full[slot], (step / C::NS) & 1, A, to)) break;
            ok = reinterpret_cast<const volatile int *>(stage_ok)[slot];
            if (C::KQ4) sk = lds128(tile + L::KS + 16 * r);
            else { const uint2 x = lds64(tile + L::KS + 8 * r); sk = make_uint4(x.x, x.y, 0u, 0u); }
            if (C::VQ4) sv = lds128(tile + L::VS + 16 * r);
            else { const uint2 x = lds64(tile + L::VS + 8 * r); sv = make_uint4(x.x, x.y, 0u, 0u); }
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            // the chunk of 16 dims-group j sits at 16 (j ^ r): conflict-free for the warp
            uint32_t w[HW];
            if (has) {
#pragma unroll
                for (int j = 0; j < HW / 4; ++j) {
                    const int jj = hf * (HW / 4) + j;
                    const uint4 v = lds128(tile + L::KC + TB * r + 16 * (jj ^ r));
                    w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
                }
                if (hf == 1) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&B.empty[slot]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < HW; ++j) w[j] = 0u;
            }
            // the previous stage's score MMAs of this half are done with its columns
            if (s > 0 && !um_wait_warp(&B.kq_done[hf], (s - 1) & 1, A, to)) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t o[32];
                if constexpr (C::KQ4) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) q4_word_sub(w[8 * c + i], o + 4 * i);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) i8_word_sub(w[16 * c + i], o + 2 * i);
                }
                Tmem<32>::st(tl + C::T_KOP + 64 * hf + 32 * c, o);
            }
            if (hf == 1) {
                // scales of the token, and the validity of its step, for the softmax warps
                uint8_t *side = smem + C::SIDE_OFF + (s & 1) * 2 * 128 * 16;
                sts128(side + 16 * t, sk);
                sts128(side + 128 * 16 + 16 * t, sv);
                if ((t & 63) == 0) step_ok[2 * (s & 1) + (t >> 6)] = has && ok;
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (hf == 1) mbar_arrive(&B.side_full[s & 1]);
                mbar_arrive(&B.kop_full[hf]);
            }
        }
        if (to) break;
    }
}

// V: thread tq unpacks dims tq (M-tile 0) and 128 + tq (M-tile 1) of every
// 64-token half into the V slot of that half.
template <int FMT>
__device__ __forceinline__ void um_v_role(const DecodeArgs &A, uint8_t *smem, const UmBars &B, uint32_t tmem,
                                          int n_steps, int tq, bool &to) {
    using L = TileLayout<FMT>;
    using C = UmCfg<FMT>;
    constexpr int WPD = C::VQ4 ? 1 : 2;               // code words per dim per tile
    const int lane = tq & 31;
    const uint32_t tl = tmem + ((uint32_t)(tq & ~31) << 16);
    for (int i = 0; i < n_steps; ++i) {
        const int slot = i % C::NS;
        if (!um_wait_warp(&B.full[slot], (i / C::NS) & 1, A, to)) break;
        const uint8_t *stage = smem + slot * C::STEP_BYTES;
        uint32_t w0[8 * WPD], w1[8 * WPD];
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) {
            const uint8_t *v = stage + tt * L::BYTES + L::VC;
            if constexpr (C::VQ4) {
                w0[tt] = lds32(v + 4 * tq);
                w1[tt] = lds32(v + 4 * (128 + tq));
            } else {
                const uint2 a = lds64(v + 8 * tq), b = lds64(v + 8 * (128 + tq));
                w0[2 * tt] = a.x; w0[2 * tt + 1] = a.y;
                w1[2 * tt] = b.x; w1[2 * tt + 1] = b.y;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.empty[slot]);
        if (i >= 2 && !um_wait_warp(&B.vop_free[i & 1], ((i - 2) >> 1) & 1, A, to)) break;
        tc_fence_after();
        uint32_t o[32];
#pragma unroll
        for (int j = 0; j < 8 * WPD; ++j) {
            if constexpr (C::VQ4) q4_word_pairs(w0[j], o + 4 * j);
            else i8_word_pairs(w0[j], o + 2 * j);
        }
        Tmem<32>::st(tl + C::T_VOP + 64 * (i & 1), o);
#pragma unroll
        for (int j = 0; j < 8 * WPD; ++j) {
            if constexpr (C::VQ4) q4_word_pairs(w1[j], o + 4 * j);
            else i8_word_pairs(w1[j], o + 2 * j);
        }
        Tmem<32>::st(tl + C::T_VOP + 64 * (i & 1) + 32, o);
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.vop_full[i & 1]);
    }
}

// Score MMA issuer (one thread): per stage, the 8 k-steps of dims 0-127 as soon
// as K warps have written them, then the 8 of dims 128-255.
template <int FMT>
__device__ __forceinline__ void um_qk_issue(const DecodeArgs &A, uint8_t *smem, const UmBars &B, uint32_t tmem,
                                            int n_stages, bool &to) {
    using C = UmCfg<FMT>;
    if (!um_wait(B.bqk_ready, 0, A, to)) return;
    const uint32_t bqk = smem_u32(smem + C::BQK_OFF);
    for (int s = 0; s < n_stages; ++s) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            if (!um_wait(&B.kop_full[hf], s & 1, A, to)) return;
            if (s > 0 && !um_wait(&B.sqk_free[hf], (s - 1) & 1, A, to)) return;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int ks = 8 * hf + k;
                umma_f16_ts(tmem + C::T_SQK + 16 * (ks / C::KSPB), tmem + C::T_KOP + 8 * ks,
                            umma_sdesc(bqk + ks * 512, 128, 256), C::IDESC_QK, (ks % C::KSPB) != 0);
            }
            tc_commit(&B.kq_done[hf]);
        }
    }
}

// Value MMA issuer (one thread).  P' of stage s: slot s & 1, n-group g (8
// consecutive accumulator columns) at g*2048, token k of the stage at k*16.
template <int FMT>
__device__ __forceinline__ void um_pv_issue(const DecodeArgs &A, uint8_t *smem, const UmBars &B, uint32_t tmem,
                                            int n_steps, bool &to) {
    using C = UmCfg<FMT>;
    const uint32_t bpv = smem_u32(smem + C::BPV_OFF);
    bool first = true;
    for (int i = 0; i < n_steps; ++i) {
        const int s = i >> 1;
        if ((i & 1) == 0 && !um_wait(&B.bpv_full[s & 1], (s >> 1) & 1, A, to)) return;
        if (!um_wait(&B.vop_full[i & 1], (i >> 1) & 1, A, to)) return;
        tc_fence_after();
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t b = bpv + (s & 1) * C::BPV_SLOT + mt * (C::NPV / 8) * 2048 + ((i & 1) * 8 + 2 * kk) * 128;
                umma_f16_ts(tmem + C::T_O + C::NPV * mt, tmem + C::T_VOP + 64 * (i & 1) + 32 * mt + 8 * kk,
                            umma_sdesc(b, 128, 2048), C::IDESC_PV, !(first && kk == 0));
            }
        first = false;
        tc_commit(&B.vop_free[i & 1]);
        if ((i & 1) == 1 || i == n_steps - 1) tc_commit(&B.bpv_free[s & 1]);
    }
}

// Group-wide OR over the 128 threads of softmax group g (named barrier 2 + g).
__device__ __forceinline__ bool um_group_any(int g, bool v) {
    uint32_t r;
    if (g == 0)
        asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 2, 128, p;\n\t"
                     "selp.u32 %0, 1, 0, q;\n\t}" : "=r"(r) : "r"((uint32_t)v) : "memory");
    else
        asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 3, 128, p;\n\t"
                     "selp.u32 %0, 1, 0, q;\n\t}" : "=r"(r) : "r"((uint32_t)v) : "memory");
    return r != 0;
}
__device__ __forceinline__ void um_group_sync(int g) {
    if (g == 0) asm volatile("bar.sync 2, 128;" ::: "memory");
    else asm volatile("bar.sync 3, 128;" ::: "memory");
}

// S: one softmax group (g = 0: heads 0-3, 1: heads 4-7).  Returns, for the
// unit's partial, the reference m + PSHIFT of its heads (log2 units; p' =
// 2^(x - reference)), this thread's sum of p' per head, and 2^-sigma.
template <int FMT>
__device__ __forceinline__ void um_s_role(const DecodeArgs &A, uint8_t *smem, const UmBars &B, const int *step_ok,
                                          uint32_t tmem, float qsc, int t0, int t1, int n_stages, int g, int t,
                                          float (&m)[4], float (&l)[4], float &unsig, bool &to) {
    using C = UmCfg<FMT>;
    const int warp = t >> 5, lane = t & 31;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    float *red = reinterpret_cast<float *>(smem + C::RED_OFF) + g * (2 * 4 * 4 + 2 * 4);
    int *red_e = reinterpret_cast<int *>(red + 2 * 4 * 4);          // [2][4] exponent maxima
    const float *kc = reinterpret_cast<const float *>(smem + C::KC_OFF);
    float mref[4];        // m + PSHIFT, or 0 while m is still -inf (no valid token yet)
#pragma unroll
    for (int h = 0; h < 4; ++h) { m[h] = -INFINITY; l[h] = 0.f; mref[h] = 0.f; }
    int e_cur = 0;
    uint32_t fa, fb;
    um_sigma_factors(um_sigma(0), fa, fb);
    for (int s = 0; s < n_stages; ++s) {
        bool ok = um_wait_warp(&B.side_full[s & 1], (s >> 1) & 1, A, to);
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        uint4 skk = make_uint4(0u, 0u, 0u, 0u), svv = make_uint4(0u, 0u, 0u, 0u);
        bool valid = false;
        if (ok) {
            const uint8_t *side = smem + C::SIDE_OFF + (s & 1) * 2 * 128 * 16;
            skk = lds128(side + 16 * t);
            svv = lds128(side + 128 * 16 + 16 * t);
            valid = step_ok[2 * (s & 1) + (t >> 6)] != 0 && t0 + 128 * s + t < t1;
        }
        // scores of the group's heads: x_h = sum_b dK_b 2^-kq (S_b[hi h] + S_b[lo h] - kc[b][h])
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            ok = ok && um_wait_warp(&B.kq_done[hf], s & 1, A, to);
            if (ok) {
                tc_fence_after();
                constexpr int NB = C::NKB / 2;                 // K blocks per half
                uint32_t r[NB][8];
#pragma unroll
                for (int bb = 0; bb < NB; ++bb) {
                    uint32_t (&rb)[8] = r[bb];
                    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                                 : "=r"(rb[0]), "=r"(rb[1]), "=r"(rb[2]), "=r"(rb[3]), "=r"(rb[4]), "=r"(rb[5]),
                                   "=r"(rb[6]), "=r"(rb[7])
                                 : "r"(tl + C::T_SQK + 16 * (NB * hf + bb) + 8 * g)
                                 : "memory");
                }
                tc_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&B.sqk_free[hf]);
#pragma unroll
                for (int bb = 0; bb < NB; ++bb) {
                    const int b = NB * hf + bb;
                    const float dk = __half2float(__ushort_as_half((unsigned short)(u4_at(skk, b >> 1) >> (16 * (b & 1))))) * qsc;
                    const float4 c = *reinterpret_cast<const float4 *>(kc + 8 * b + 4 * g);
                    x[0] = fmaf((__uint_as_float(r[bb][0]) + __uint_as_float(r[bb][4])) - c.x, dk, x[0]);
                    x[1] = fmaf((__uint_as_float(r[bb][1]) + __uint_as_float(r[bb][5])) - c.y, dk, x[1]);
                    x[2] = fmaf((__uint_as_float(r[bb][2]) + __uint_as_float(r[bb][6])) - c.z, dk, x[2]);
                    x[3] = fmaf((__uint_as_float(r[bb][3]) + __uint_as_float(r[bb][7])) - c.w, dk, x[3]);
                }
            } else {
                __syncwarp();
                if (lane == 0) mbar_arrive(&B.sqk_free[hf]);
            }
        }
        if (!valid) {
            svv = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int h = 0; h < 4; ++h) x[h] = -INFINITY;
        }
        // largest V scale exponent of the token (fp16 magnitudes order as integers)
        uint32_t vm = __vmaxu2(__vmaxu2(svv.x & 0x7FFF7FFFu, svv.y & 0x7FFF7FFFu),
                               __vmaxu2(svv.z & 0x7FFF7FFFu, svv.w & 0x7FFF7FFFu));
        vm = max(vm & 0xFFFFu, vm >> 16);
        const int e_tok = (int)(vm >> 10);
        // the running max moves only past the slack, sigma only for a larger
        // scale exponent; both checks, and a timed-out wait, are decided for the
        // whole group
        bool need = e_tok > e_cur;
#pragma unroll
        for (int h = 0; h < 4; ++h) need |= x[h] > m[h] + RESCALE_SLACK;
        if (um_group_any(g, need || to)) {
            if (um_group_any(g, to)) { to = true; break; }
            float mx[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                mx[h] = x[h];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
            }
            const int ew = (int)__reduce_max_sync(0xffffffffu, (unsigned)e_tok);
            float *rr = red + (s & 1) * 16;
            if (lane < 4) rr[warp * 4 + lane] = lane == 0 ? mx[0] : (lane == 1 ? mx[1] : (lane == 2 ? mx[2] : mx[3]));
            if (lane == 0) red_e[(s & 1) * 4 + warp] = ew;
            um_group_sync(g);
            const int *re = red_e + (s & 1) * 4;
            const int e_new = max(e_cur, max(max(re[0], re[1]), max(re[2], re[3])));
            const int sig_old = um_sigma(e_cur), sig_new = um_sigma(e_new);
            const float sc = __int_as_float((127 + sig_new - sig_old) << 23);   // 2^(sigma_new - sigma_old) <= 1
            e_cur = e_new;
            um_sigma_factors(sig_new, fa, fb);
            float alpha[4];
            bool moved = sig_new != sig_old;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float M = fmaxf(fmaxf(rr[h], rr[4 + h]), fmaxf(rr[8 + h], rr[12 + h]));
                const float mn = M > m[h] ? M : m[h];
                alpha[h] = m[h] == -INFINITY ? 0.f : ex2(m[h] - mn);
                moved |= mn != m[h] && m[h] != -INFINITY;
                m[h] = mn;
                mref[h] = mn == -INFINITY ? 0.f : mn + PSHIFT;
                l[h] *= alpha[h];
                alpha[h] *= sc;              // the accumulators also carry 2^sigma
            }
            // rescale the group's output columns once every earlier value MMA is
            // complete (the first stage has nothing accumulated yet)
            if (s > 0 && moved) {
                um_wait_warp(&B.bpv_free[(s - 1) & 1], ((s - 1) >> 1) & 1, A, to);   // a timeout ends the loop at the next stage
                tc_fence_after();
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    const uint32_t ta = tl + C::T_O + C::NPV * mt + g * (C::NPV / 2);
                    if constexpr (C::NPV / 2 == 32) {
                        uint32_t r[32];
                        Tmem<32>::ld(ta, r);
                        tc_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha[j & 3]);
                        Tmem<32>::st(ta, r);
                    } else {
                        uint32_t r[16];
                        Tmem<16>::ld(ta, r);
                        tc_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha[j & 3]);
                        Tmem<16>::st(ta, r);
                    }
                }
                tc_wait_st();
            }
            um_group_sync(g);            // the reduction slots are read before the next stage writes them
        }
        // p' = 2^(x - m - PSHIFT); masked tokens give 0
        float p[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            p[h] = ex2(x[h] - mref[h]);
            l[h] += p[h];
        }
        // the token's V scales times 2^sigma (exact: two power-of-two products)
        svv.x = h2_as_u32(__hmul2(__hmul2(u32_as_h2(svv.x), u32_as_h2(fa)), u32_as_h2(fb)));
        svv.y = h2_as_u32(__hmul2(__hmul2(u32_as_h2(svv.y), u32_as_h2(fa)), u32_as_h2(fb)));
        if (C::NVB > 4) {
            svv.z = h2_as_u32(__hmul2(__hmul2(u32_as_h2(svv.z), u32_as_h2(fa)), u32_as_h2(fb)));
            svv.w = h2_as_u32(__hmul2(__hmul2(u32_as_h2(svv.w), u32_as_h2(fa)), u32_as_h2(fb)));
        }
        // P' = p' dV 2^sigma as exact fp16 (hi, lo) pairs into slot s & 1
        if (s >= 2) um_wait_warp(&B.bpv_free[s & 1], ((s - 2) >> 1) & 1, A, to);   // a timeout ends the loop next stage
        uint32_t ph0, pl0, ph1, pl1;
        split_pair(p[0], p[1], ph0, pl0);
        split_pair(p[2], p[3], ph1, pl1);
        uint8_t *bp = smem + C::BPV_OFF + (s & 1) * C::BPV_SLOT + 16 * t;
#pragma unroll
        for (int b = 0; b < C::NVB; ++b) {
            const uint32_t dvw = u4_at(svv, b >> 1);
            const __half2 dv = u32_as_h2(__byte_perm(dvw, dvw, (b & 1) ? 0x3232u : 0x1010u));    // (dV_b, dV_b)
            const __half2 h0 = __hmul2(u32_as_h2(ph0), dv), h1 = __hmul2(u32_as_h2(ph1), dv);
            const __half2 l0 = __hfma2(u32_as_h2(pl0), dv, __hfma2(u32_as_h2(ph0), dv, __hneg2(h0)));
            const __half2 l1 = __hfma2(u32_as_h2(pl1), dv, __hfma2(u32_as_h2(ph1), dv, __hneg2(h1)));
            const int mt = b / C::VBM, bl = b % C::VBM;
            const int ng = mt * (C::NPV / 8) + g * C::VBM + bl;          // n-group (group, block): hi h0-3, lo h0-3
            sts128(bp + ng * 2048, make_uint4(h2_as_u32(h0), h2_as_u32(h1), h2_as_u32(l0), h2_as_u32(l1)));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");    // generic writes -> tensor-core reads
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.bpv_full[s & 1]);
    }
    unsig = __int_as_float((127 - um_sigma(e_cur)) << 23);
}

template <int FMT, bool FUSED, bool STEP = false>
__global__ void __launch_bounds__(UmCfg<FMT>::NTHREADS, 1) decode_umma_kernel(const __grid_constant__ DecodeArgs A) {
    static_assert(!STEP || FUSED, "the decode step merges in the kernel");
    using L = TileLayout<FMT>;
    using C = UmCfg<FMT>;
    extern __shared__ __align__(1024) uint8_t smem[];
    grid_dependency_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.x;
    const int32_t *U = A.plan + PLAN_HEADER + 4 * u;
    const int seq = U[0], kvh = U[1], t0 = U[2], t1 = U[3];
    const int G = A.G;
    const int n_units = A.plan[1];
    float *wsu = A.ws + (size_t)u * ws_unit_floats(G);
    if (!unit_ok(A, seq, kvh, t0, t1, wsu)) return;           // the whole CTA, before anything is allocated
    const int n_steps = (t1 - t0 + STEP_TOKENS - 1) / STEP_TOKENS;
    const int n_stages = (n_steps + 1) / 2;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    UmBars B;
    B.full = bars;
    B.empty = bars + C::NS;
    uint64_t *nb = bars + 2 * C::NS;
    B.kop_full = nb;
    B.kq_done = nb + 2;
    B.sqk_free = nb + 4;
    B.side_full = nb + 6;
    B.vop_full = nb + 8;
    B.vop_free = nb + 10;
    B.bpv_full = nb + 12;
    B.bpv_free = nb + 14;
    B.drain = nb + 16;
    B.bqk_ready = nb + 18;
    B.enc_done = nb + 19;
    int *stage_ok = reinterpret_cast<int *>(smem + C::MISC_OFF);
    int *step_ok = stage_ok + C::NS;                           // [2 stage slots][2 halves]
    uint32_t *tmem_base = reinterpret_cast<uint32_t *>(step_ok + 4);
    int *s_last = reinterpret_cast<int *>(tmem_base + 1);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(&B.full[i], 1);
            mbar_init(&B.empty[i], 6);                       // 2 K warps + 4 V warps read each step
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&B.kop_full[i], 4);
            mbar_init(&B.kq_done[i], 1);
            mbar_init(&B.sqk_free[i], 8);
            mbar_init(&B.side_full[i], 4);
            mbar_init(&B.vop_full[i], 4);
            mbar_init(&B.vop_free[i], 1);
            mbar_init(&B.bpv_full[i], 8);
            mbar_init(&B.bpv_free[i], 1);
            mbar_init(&B.drain[i], 1);
        }
        mbar_init(B.bqk_ready, 8);
        mbar_init(B.enc_done, 1);
        fence_mbar_init();
    }
    if (warp == C::W_QK) tmem_alloc(tmem_base, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base;
    // decode step: the CTA whose unit ends the (sequence, KV head) range appends its newest token
    const bool appends = STEP && u == A.plan[PLAN_HEADER + 4 * n_units + seq * A.geo.n_kv_heads + kvh + 1] - 1;
    bool to = false;

    if (warp == C::W_COPY) {
        copy_loop<C::NS, C::STEP_BYTES, L::BYTES>(A, smem, B.full, B.empty, stage_ok, seq, kvh, t0, n_steps, lane,
                                                  appends ? B.enc_done : nullptr);
        return;
    }
    if (warp > C::W_PV) return;                                  // spare warp
    if (warp == C::W_QK || warp == C::W_PV) {
        if (warp == C::W_PV && appends) {
            step_encode_token<FMT>(A, seq, kvh, t1 - 1, lane);
            if (lane == 0) mbar_arrive(B.enc_done);
        }
        if (lane == 0) {
            if (warp == C::W_QK) um_qk_issue<FMT>(A, smem, B, tmem, n_stages, to);
            else um_pv_issue<FMT>(A, smem, B, tmem, n_steps, to);
            // every MMA this thread issued is complete before the memory is freed
            tc_commit(&B.drain[warp - C::W_QK]);
            bool dto = false;
            um_wait(&B.drain[warp - C::W_QK], 0, A, dto);
        }
        __syncwarp();
        asm volatile("bar.sync 4, 320;" ::: "memory");       // with the softmax warps: tensor memory is idle
        if (warp == C::W_QK) {
            tc_fence_after();
            tmem_dealloc(tmem, C::TMEM_COLS);
        }
        return;
    }

    if (warp < C::W_K) {
        const int g = warp >> 2, t = threadIdx.x & 127;
        const float *qg = A.q + ((int64_t)seq * A.n_q_heads + (int64_t)kvh * G) * D;
        float *q_s = reinterpret_cast<float *>(smem + C::BPV_OFF);       // free until the first P'
        step_stage_query<STEP && Fmt<FMT>::KROT>(qg, q_s, G, warp, 8, lane);
        asm volatile("bar.sync 5, 256;" ::: "memory");
        const float qsc = um_build_query<FMT>(q_s, G, smem + C::BQK_OFF, reinterpret_cast<float *>(smem + C::KC_OFF),
                                              reinterpret_cast<float *>(smem + C::RED_OFF) + 2 * (2 * 4 * 4 + 2 * 4),
                                              threadIdx.x);
        if (lane == 0) mbar_arrive(B.bqk_ready);
        float m[4], l[4], unsig;
        um_s_role<FMT>(A, smem, B, step_ok, tmem, qsc, t0, t1, n_stages, g, t, m, l, unsig, to);
        // the unit's partial: o from the accumulators once the last value MMA is done
        const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        um_wait_warp(&B.bpv_free[(n_stages - 1) & 1], ((n_stages - 1) >> 1) & 1, A, to);
        tc_fence_after();
        float o0[4], o1[4];
        {
            const int bl = ((warp & 3) * 32) / (256 / C::NVB);      // V block of dim t inside its M-tile
            uint32_t r[8];
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                         : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                           "=r"(r[7])
                         : "r"(tl + C::T_O + g * (C::NPV / 2) + 8 * bl)
                         : "memory");
            tc_wait_ld();
#pragma unroll
            for (int h = 0; h < 4; ++h) o0[h] = (__uint_as_float(r[h]) + __uint_as_float(r[4 + h])) * unsig;
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                         : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                           "=r"(r[7])
                         : "r"(tl + C::T_O + C::NPV + g * (C::NPV / 2) + 8 * bl)
                         : "memory");
            tc_wait_ld();
#pragma unroll
            for (int h = 0; h < 4; ++h) o1[h] = (__uint_as_float(r[h]) + __uint_as_float(r[4 + h])) * unsig;
        }
        tc_fence_before();
        asm volatile("bar.arrive 4, 320;" ::: "memory");       // tensor memory may be freed
        // l: sum over the 128 tokens of the group
        float *red = reinterpret_cast<float *>(smem + C::RED_OFF) + g * (2 * 4 * 4 + 2 * 4);
#pragma unroll
        for (int h = 0; h < 4; ++h)
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
        um_group_sync(g);
        if (lane < 4) red[(warp & 3) * 4 + lane] = lane == 0 ? l[0] : (lane == 1 ? l[1] : (lane == 2 ? l[2] : l[3]));
        um_group_sync(g);
#pragma unroll
        for (int h = 0; h < 4; ++h)
            if (4 * g + h < G) {
                wsu[(4 * g + h) * D + t] = o0[h];
                wsu[(4 * g + h) * D + 128 + t] = o1[h];
            }
        if (t < 4) {
            const float mv = t == 0 ? m[0] : (t == 1 ? m[1] : (t == 2 ? m[2] : m[3]));
            wsu[G * D + 4 * g + t] = mv + PSHIFT;
            wsu[G * D + 8 + 4 * g + t] = (red[t] + red[4 + t]) + (red[8 + t] + red[12 + t]);
        }
    } else if (warp < C::W_V) {
        um_k_role<FMT>(A, smem, B, stage_ok, step_ok, tmem, n_steps, n_stages, threadIdx.x - 32 * C::W_K, to);
    } else {
        um_v_role<FMT>(A, smem, B, tmem, n_steps, threadIdx.x - 32 * C::W_V, to);
    }
    publish_unit<FUSED, C::NCT>(A, seq, kvh, n_units, s_last, smem);
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
    extern __shared__ __align__(1024) uint8_t smem[];
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
// may launch concurrently.
template <auto KERNEL>
cudaError_t launch_decode_kernel(int smem_bytes, int threads, const DecodeArgs &a, int n_units, bool fused,
                                 cudaStream_t s) {
    static std::mutex mu;
    static int cap[64];                  // resident CTAs per device ordinal; 0 = not yet known
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int c = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (cap[dev] == 0) {
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
        using C = UmCfg<FMT>;
        if constexpr (FUSED) {
            if (a.k_new)
                return launch_decode_kernel<decode_umma_kernel<FMT, true, true>>(C::TOTAL, C::NTHREADS, a, n_units,
                                                                                 true, s);
        }
        return launch_decode_kernel<decode_umma_kernel<FMT, FUSED>>(C::TOTAL, C::NTHREADS, a, n_units, FUSED, s);
    }
    using C = AluCfg<FMT>;
    switch (a.G) {
    case 4: return launch_decode_kernel<decode_alu_kernel<FMT, 4, FUSED>>(C::TOTAL, C::NTHREADS, a, n_units, FUSED, s);
    case 6: return launch_decode_kernel<decode_alu_kernel<FMT, 6, FUSED>>(C::TOTAL, C::NTHREADS, a, n_units, FUSED, s);
    default: return launch_decode_kernel<decode_alu_kernel<FMT, 8, FUSED>>(C::TOTAL, C::NTHREADS, a, n_units, FUSED, s);
    }
}

template <bool FUSED>
cudaError_t launch_fused(int fmt, bool tc, const DecodeArgs &a, int n_units, cudaStream_t s) {
    switch (fmt) {
    case KVQ_INT8: return launch_fmt<KVQ_INT8, FUSED>(tc, a, n_units, s);
    case KVQ_Q4_0: return launch_fmt<KVQ_Q4_0, FUSED>(tc, a, n_units, s);
    default: return launch_fmt<KVQ_K8V4, FUSED>(tc, a, n_units, s);
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

cudaError_t launch_combine(const float *ws, const int32_t *plan, const kvq_plan_info &info, int inverse_fwht,
                           uint16_t *out_bf16, float *out_f32, cudaStream_t s) {
    const int groups = info.n_seq * info.n_kv_heads;
    if (groups == 0) return cudaSuccess;
    return launch_ex(combine_kernel, dim3(groups), dim3(256), 0, s, false, ws, plan, info.n_kv_heads, info.group,
                     inverse_fwht, out_bf16, out_f32);
}

}  // namespace kvq
