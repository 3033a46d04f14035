// Device code of q_rotate and kv_append, shared by the launches that run them
// on their own and by the decode-step kernel that runs them inside the decode:
// the 256-point Walsh-Hadamard rotation and the q4_0 / int8 / fp8 / nvfp4 block
// quantisers ([Roundup] section 一 for the last two),
// written into the fragment-ordered pool layout.
//
// [Strata] "4-bit KV 缓存：先旋转，再压到 4-bit": K, V (and the query) are rotated
// by a 256-point Hadamard transform before 4-bit storage; [Strata] "三种 KV 格式
// 横向对比": int8 stores K and V unrotated, k8v4 rotates only V.
//
// Bit-exactness: every fp32 operation is an explicit round-to-nearest
// intrinsic (__fadd_rn, __fsub_rn, __fmul_rn, __fdiv_rn), so no multiply-add
// contraction can change a result whatever the translation unit's flags, and
// the butterfly pairs the same operands in the same order as the definition:
// stage h = 1, 2, ..., 128 maps (x[i], x[i+h]) with (i & h) == 0 to
// (x[i] + x[i+h], x[i] - x[i+h]).
//
// One warp per 256-vector: lane l holds elements 8l .. 8l+7, so stages 1, 2, 4
// stay inside a thread and stages 8 .. 128 pair lanes l and l ^ (h/8).
#pragma once

#include "kvq_internal.cuh"

namespace kvq {
namespace {

__device__ __forceinline__ void fwht256_lane(float (&x)[8], int lane) {
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if ((i & h) == 0) {
                const float a = x[i], b = x[i + h];
                x[i] = __fadd_rn(a, b);
                x[i + h] = __fsub_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float other = __shfl_xor_sync(0xffffffffu, x[i], m);
            // lower element a = x[i] of the lane without bit m, upper b = the partner's
            x[i] = upper ? __fsub_rn(other, x[i]) : __fadd_rn(x[i], other);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = __fmul_rn(x[i], 0.0625f);
}

__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// One warp rotates query vector `vec` of 256 values.
__device__ __forceinline__ void rotate_vec(const float *q, float *q_rot, int64_t vec, int lane) {
    float x[8];
    load8(q + vec * D + lane * 8, x);
    fwht256_lane(x, lane);
    float4 *o = reinterpret_cast<float4 *>(q_rot + vec * D + lane * 8);
    o[0] = make_float4(x[0], x[1], x[2], x[3]);
    o[1] = make_float4(x[4], x[5], x[6], x[7]);
}


// ---- q4_0: blocks of 32 = 4 lanes (lanes 4b .. 4b+3 hold block b) ----------
// d = fp16(signed max / -8), first index wins a tie in |x|; code =
// clamp(rint(x / d) + 8, 0, 15); all codes 8 when d rounds to zero.
__device__ __forceinline__ void quant_q4_lane(const float (&x)[8], int lane, int (&c)[8], __half &d16) {
    float amax = fabsf(x[0]), sv = x[0];
    int idx = lane * 8;
#pragma unroll
    for (int i = 1; i < 8; ++i)
        if (fabsf(x[i]) > amax) { amax = fabsf(x[i]); sv = x[i]; idx = lane * 8 + i; }
#pragma unroll
    for (int m = 1; m < 4; m <<= 1) {
        const float oa = __shfl_xor_sync(0xffffffffu, amax, m);
        const float os = __shfl_xor_sync(0xffffffffu, sv, m);
        const int oi = __shfl_xor_sync(0xffffffffu, idx, m);
        if (oa > amax || (oa == amax && oi < idx)) { amax = oa; sv = os; idx = oi; }
    }
    const float d32 = __fdiv_rn(sv, -8.0f);
    d16 = __float2half_rn(d32);
    const float df = __half2float(d16);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int v = 8;
        if (df != 0.0f) {
            v = (int)rintf(__fdiv_rn(x[i], df)) + 8;
            v = v < 0 ? 0 : (v > 15 ? 15 : v);
        }
        c[i] = v;
    }
}

// ---- int8: groups of 64 = 8 lanes --------------------------------------------
// d = fp16(max|x| / 127); code = clamp(rint(x / d), -127, 127); 0 when d == 0.
__device__ __forceinline__ void quant_i8_lane(const float (&x)[8], int (&c)[8], __half &d16) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const float d32 = __fdiv_rn(amax, 127.0f);
    d16 = __float2half_rn(d32);
    const float df = __half2float(d16);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int v = 0;
        if (df != 0.0f) {
            v = (int)rintf(__fdiv_rn(x[i], df));
            v = v < -127 ? -127 : (v > 127 ? 127 : v);
        }
        c[i] = v;
    }
}

// ---- fp8: one E4M3 code per value, one fp16 scale per 256-vector ------------
// d = fp16(max|x| / 448); code = E4M3(x / d) (round to nearest even,
// saturating); all codes +0 when d rounds to zero.
__device__ __forceinline__ void quant_f8_lane(const float (&x)[8], int (&c)[8], __half &d16) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    d16 = __float2half_rn(__fdiv_rn(amax, 448.0f));
    const float df = __half2float(d16);
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = df != 0.0f ? (int)f32_to_e4m3(__fdiv_rn(x[i], df)) : 0;
}

// ---- nvfp4: blocks of 16 = 2 lanes, E2M1 codes, one E4M3 scale per block ------
// s = E4M3(max|x| / 6); code = E2M1(x / s) (round to nearest even,
// saturating); all codes +0 when s is zero.  The scale byte travels in d16's
// bits.
__device__ __forceinline__ void quant_f4_lane(const float (&x)[8], int (&c)[8], __half &d16) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    const uint32_t sb = f32_to_e4m3(__fdiv_rn(amax, 6.0f));
    d16 = __ushort_as_half((unsigned short)sb);
    const float sd = __half2float(__ushort_as_half((unsigned short)(e4m3x2_to_h2(sb) & 0xFFFFu)));
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = sd != 0.0f ? (int)f32_to_e2m1(__fdiv_rn(x[i], sd)) : 0;
}

// ---- stores into the fragment-ordered tile ---------------------------------
// K side, Q4: lane (block b = lane>>2, jl = lane&3) holds dims 32b + 8jl + e.
// Dim 32b + 8(n&3) + (n>>2) + 2j lives in word W(r,b,j) nibble n, so element
// e goes to word j = e>>1, nibble jl + 4(e&1).
__device__ __forceinline__ void store_q4_kside(uint8_t *tile, int r, int lane, const int (&c)[8]) {
    const int b = lane >> 2, jl = lane & 3;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        w[j] = ((uint32_t)c[2 * j] << (4 * jl)) | ((uint32_t)c[2 * j + 1] << (4 * jl + 16));
#pragma unroll
    for (int m = 1; m < 4; m <<= 1)
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] |= __shfl_xor_sync(0xffffffffu, w[j], m);
    uint32_t mine = w[0];
#pragma unroll
    for (int j = 1; j < 4; ++j) if (jl == j) mine = w[j];
    *reinterpret_cast<uint32_t *>(tile + (b >> 2) * 512 + (r * 4 + jl) * 16 + (b & 3) * 4) = mine;
}

// V side, Q4: word W(p,b,g) nibble n holds token 2p + (n>>2), dim 32b + g + 8(n&3).
// Lane jl holds dims 32b + 8jl + e, i.e. g = e, n&3 = jl.  Token r fills the
// 16-bit half (r&1) of words (r>>1, b, g) for g = 0..7.
__device__ __forceinline__ void store_q4_vside(uint8_t *tile, int r, int lane, const int (&c)[8]) {
    const int b = lane >> 2, jl = lane & 3;
    uint32_t w[4];  // w[k] = half(g=2k) | half(g=2k+1) << 16
#pragma unroll
    for (int k = 0; k < 4; ++k)
        w[k] = ((uint32_t)c[2 * k] << (4 * jl)) | ((uint32_t)c[2 * k + 1] << (4 * jl + 16));
#pragma unroll
    for (int m = 1; m < 4; m <<= 1)
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] |= __shfl_xor_sync(0xffffffffu, w[k], m);
    uint32_t mine = w[0];
#pragma unroll
    for (int k = 1; k < 4; ++k) if (jl == k) mine = w[k];
    const int p = r >> 1, half = r & 1;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int g = 2 * jl + t;
        const uint16_t hv = (uint16_t)(mine >> (16 * t));
        *reinterpret_cast<uint16_t *>(tile + (b >> 2) * 512 + (g * 4 + p) * 16 + (b & 3) * 4 + half * 2) = hv;
    }
}

// K side, I8: word W(r,s,j) byte n holds dim 16s + 2j + {0,1,8,9}[n].  Lane
// (s = lane>>1, hl = lane&1) holds dims 16s + 8hl + e: word j = e>>1, byte
// 2hl + (e&1).
__device__ __forceinline__ void store_i8_kside(uint8_t *tile, int r, int lane, const int (&c)[8]) {
    const int s = lane >> 1, hl = lane & 1;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        w[j] = (((uint32_t)(c[2 * j] & 0xFF)) | ((uint32_t)(c[2 * j + 1] & 0xFF) << 8)) << (16 * hl);
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] |= __shfl_xor_sync(0xffffffffu, w[j], 1);
    uint8_t *base = tile + (s >> 2) * 512 + (s & 3) * 4;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int j = 2 * hl + t;
        *reinterpret_cast<uint32_t *>(base + (r * 4 + j) * 16) = hl ? w[2 + t] : w[t];
    }
}

// V side, I8: word W(p,m,g) byte n holds token 2p + (n&1), dim 16m + g + 8(n>>1).
// Lane (m = lane>>1, hl = lane&1) holds dims 16m + 8hl + e: g = e, byte 2hl + (r&1).
__device__ __forceinline__ void store_i8_vside(uint8_t *tile, int r, int lane, const int (&c)[8]) {
    const int m = lane >> 1, hl = lane & 1;
    uint8_t *base = tile + (m >> 2) * 512 + (m & 3) * 4 + 2 * hl + (r & 1) + (r >> 1) * 16;
#pragma unroll
    for (int g = 0; g < 8; ++g) base[g * 64] = (uint8_t)(c[g] & 0xFF);
}

// K side, F4: word W(r,b,j) (where Q4 puts it) byte q holds dims 32b + 8q + 2j
// (low nibble) and + 1 (high nibble).  Lane (b = lane>>2, jl = lane&3) holds
// dims 32b + 8jl + e: byte q = jl of word j = e>>1, nibble e&1.
__device__ __forceinline__ void store_f4_kside(uint8_t *tile, int r, int lane, const int (&c)[8]) {
    const int b = lane >> 2, jl = lane & 3;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = ((uint32_t)c[2 * j] | ((uint32_t)c[2 * j + 1] << 4)) << (8 * jl);
#pragma unroll
    for (int m = 1; m < 4; m <<= 1)
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] |= __shfl_xor_sync(0xffffffffu, w[j], m);
    uint32_t mine = w[0];
#pragma unroll
    for (int j = 1; j < 4; ++j) if (jl == j) mine = w[j];
    *reinterpret_cast<uint32_t *>(tile + (b >> 2) * 512 + (r * 4 + jl) * 16 + (b & 3) * 4) = mine;
}

__device__ __forceinline__ void store_scale_q4(uint8_t *sc, int r, int lane, __half d) {
    if ((lane & 3) == 0)
        *reinterpret_cast<__half *>(sc + (r >> 1) * 32 + (lane >> 2) * 4 + (r & 1) * 2) = d;
}
__device__ __forceinline__ void store_scale_i8(uint8_t *sc, int r, int lane, __half d) {
    if ((lane & 7) == 0)
        *reinterpret_cast<__half *>(sc + (r >> 1) * 16 + (lane >> 3) * 4 + (r & 1) * 2) = d;
}
__device__ __forceinline__ void store_scale_f8(uint8_t *sc, int r, int lane, __half d) {
    if (lane == 0) *reinterpret_cast<__half *>(sc + 2 * r) = d;
}
// the E4M3 byte of block lane/2 (both lanes of the block hold it)
__device__ __forceinline__ void store_scale_f4(uint8_t *sc, int r, int lane, __half d) {
    if ((lane & 1) == 0) sc[(r >> 1) * 32 + (lane >> 1) * 2 + (r & 1)] = (uint8_t)__half_as_ushort(d);
}

// A token's codes and block scales as one lane of the encoding warp holds them
// (lane l: elements 8l .. 8l+7 of the rotated or plain K and V rows); an E4M3
// scale rides in the low byte of the __half's bits.
struct TokenCodes {
    int k[8], v[8];
    __half dk, dv;
};

template <int P> __device__ __forceinline__ void quant_part(const float (&x)[8], int lane, int (&c)[8], __half &d) {
    if constexpr (P == PART_Q4) quant_q4_lane(x, lane, c, d);
    else if constexpr (P == PART_I8) quant_i8_lane(x, c, d);
    else if constexpr (P == PART_F8) quant_f8_lane(x, c, d);
    else quant_f4_lane(x, c, d);
}

// One warp quantises one token of one KV head: xk / xv = its 256 K and V values
// (lane l holds 8l .. 8l+7), rotated first where the format stores them rotated.
template <int FMT>
__device__ __forceinline__ void quant_token(float (&xk)[8], float (&xv)[8], int lane, TokenCodes &t) {
    using L = TileLayout<FMT>;
    if (Fmt<FMT>::KROT) fwht256_lane(xk, lane);
    quant_part<L::KP>(xk, lane, t.k, t.dk);
    if (Fmt<FMT>::VROT) fwht256_lane(xv, lane);
    quant_part<L::VP>(xv, lane, t.v, t.dv);
}

// The warp writes the token as row r of the tile at `tile`.
template <int FMT>
__device__ __forceinline__ void store_token(const TokenCodes &t, int lane, int r, uint8_t *tile) {
    using L = TileLayout<FMT>;
    if constexpr (L::KP == PART_Q4) {
        store_q4_kside(tile + L::KC, r, lane, t.k);
        store_scale_q4(tile + L::KS, r, lane, t.dk);
    } else if constexpr (L::KP == PART_I8) {
        store_i8_kside(tile + L::KC, r, lane, t.k);
        store_scale_i8(tile + L::KS, r, lane, t.dk);
    } else if constexpr (L::KP == PART_F8) {
        store_i8_kside(tile + L::KC, r, lane, t.k);
        store_scale_f8(tile + L::KS, r, lane, t.dk);
    } else {
        store_f4_kside(tile + L::KC, r, lane, t.k);
        store_scale_f4(tile + L::KS, r, lane, t.dk);
    }
    if constexpr (L::VP == PART_Q4) {
        store_q4_vside(tile + L::VC, r, lane, t.v);
        store_scale_q4(tile + L::VS, r, lane, t.dv);
    } else if constexpr (L::VP == PART_I8) {
        store_i8_vside(tile + L::VC, r, lane, t.v);
        store_scale_i8(tile + L::VS, r, lane, t.dv);
    } else if constexpr (L::VP == PART_F8) {
        store_i8_vside(tile + L::VC, r, lane, t.v);
        store_scale_f8(tile + L::VS, r, lane, t.dv);
    } else {
        store_q4_vside(tile + L::VC, r, lane, t.v);
        store_scale_f4(tile + L::VS, r, lane, t.dv);
    }
}

// The tile of the pool that holds position pos of the sequence whose page slot
// is `slot`, or null (and KVQ_STATUS_BAD_SLOT) when the slot is out of range.
template <int FMT>
__device__ __forceinline__ uint8_t *token_tile(uint8_t *pool, const PoolGeom &geo, int layer, int slot, int head,
                                               int pos, int32_t *status, int lane) {
    if (slot < 0 || slot >= geo.n_pages) {
        if (lane == 0) status_or(status, KVQ_STATUS_BAD_SLOT);
        return nullptr;
    }
    return pool + layer * geo.layer_stride + (int64_t)slot * geo.slot_stride + (int64_t)head * geo.page_bytes +
           (int64_t)((pos & 255) >> 3) * TileLayout<FMT>::BYTES;
}

// One warp encodes the token at position pos of sequence seq for one KV head:
// k_row, v_row = its 256 values.  Returns false (and sets KVQ_STATUS_BAD_SLOT)
// when the position or its page slot is out of range; nothing is written then.
template <int FMT>
__device__ __forceinline__ bool append_token(uint8_t *pool, const PoolGeom &geo, int layer, const float *k_row,
                                             const float *v_row, int seq, int head, int pos,
                                             const int32_t *page_table, int max_pages, int32_t *status, int lane) {
    if (pos < 0 || pos >= max_pages * PAGE) {
        if (lane == 0) status_or(status, KVQ_STATUS_BAD_SLOT);
        return false;
    }
    // the three loads are independent: issue them together
    const int slot = page_table[(int64_t)seq * max_pages + (pos >> 8)];
    float xk[8], xv[8];
    load8(k_row + lane * 8, xk);
    load8(v_row + lane * 8, xv);
    uint8_t *tile = token_tile<FMT>(pool, geo, layer, slot, head, pos, status, lane);
    if (!tile) return false;
    TokenCodes t;
    quant_token<FMT>(xk, xv, lane, t);
    store_token<FMT>(t, lane, pos & 7, tile);
    return true;
}

// One warp encodes (row, KV head) `item` of a kv_append call.
template <int FMT>
__device__ __forceinline__ void append_item(uint8_t *pool, const PoolGeom &geo, int layer, const float *k,
                                            const float *v, int64_t n_rows, const int32_t *row_seq,
                                            const int32_t *row_pos, const int32_t *page_table, int max_pages,
                                            int n_seq, int32_t *status, int64_t item, int lane) {
    const int64_t row = item / geo.n_kv_heads;
    const int head = (int)(item - row * geo.n_kv_heads);
    if (row >= n_rows) return;
    const int seq = row_seq ? row_seq[row] : (int)row;
    if (seq < 0 || seq >= n_seq) {
        if (lane == 0) status_or(status, KVQ_STATUS_BAD_SLOT);
        return;
    }
    const int64_t off = (row * geo.n_kv_heads + head) * D;
    append_token<FMT>(pool, geo, layer, k + off, v + off, seq, head, row_pos[row], page_table, max_pages, status,
                      lane);
}

}  // namespace
}  // namespace kvq
