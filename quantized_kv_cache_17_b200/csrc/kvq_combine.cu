// attn_combine: merge the split partials of every (sequence, query head) and
// rotate the result back ([Strata] "4-bit KV 缓存": the output, mixed over the
// rotated V, is multiplied by H again since the normalised Hadamard matrix is
// its own inverse).
//
// One warp per (sequence, query head); lane l owns dims 8l .. 8l+7.  Partials
// hold scores in log2 units: M = max_j m_j, L = sum_j l_j 2^(m_j - M),
// o = sum_j 2^(m_j - M) o_j / L.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

__device__ __forceinline__ void fwht256_lane_f32(float (&x)[8], int lane) {
#pragma unroll
    for (int h = 1; h < 8; h <<= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if ((i & h) == 0) {
                const float a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
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

__global__ void __launch_bounds__(128) combine_kernel(const float *__restrict__ ws, const int32_t *__restrict__ plan,
                                                      int n_seq, int n_kv, int G, int inverse_fwht,
                                                      uint16_t *__restrict__ out_bf16, float *__restrict__ out_f32) {
    const int lane = threadIdx.x & 31;
    const int item = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int n_q = n_kv * G;
    if (item >= n_seq * n_q) return;
    const int seq = item / n_q, h = item - seq * n_q;
    const int kvh = h / G, hh = h - kvh * G;
    const int n_units = plan[1];
    const int32_t *start = plan + PLAN_HEADER + 4 * n_units;
    const int u0 = start[seq * n_kv + kvh], u1 = start[seq * n_kv + kvh + 1];
    const int stride = ws_unit_floats(G);

    float M = -INFINITY;
    for (int u = u0; u < u1; ++u) M = fmaxf(M, __ldg(ws + (size_t)u * stride + G * D + hh));
    float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float Lsum = 0.f;
    for (int u = u0; u < u1; ++u) {
        const float *p = ws + (size_t)u * stride;
        const float m = __ldg(p + G * D + hh);
        if (m == -INFINITY) continue;
        const float f = exp2f(m - M);
        Lsum = fmaf(__ldg(p + G * D + 8 + hh), f, Lsum);
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p + hh * D + lane * 8));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(p + hh * D + lane * 8) + 1);
        x[0] = fmaf(a.x, f, x[0]); x[1] = fmaf(a.y, f, x[1]); x[2] = fmaf(a.z, f, x[2]); x[3] = fmaf(a.w, f, x[3]);
        x[4] = fmaf(b.x, f, x[4]); x[5] = fmaf(b.y, f, x[5]); x[6] = fmaf(b.z, f, x[6]); x[7] = fmaf(b.w, f, x[7]);
    }
    const float inv = 1.0f / Lsum;
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] *= inv;
    if (inverse_fwht) fwht256_lane_f32(x, lane);
    const size_t off = (size_t)item * D + lane * 8;
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

}  // namespace

cudaError_t launch_combine(const float *ws, const int32_t *plan, const kvq_plan_info &info, int inverse_fwht,
                           uint16_t *out_bf16, float *out_f32, cudaStream_t s) {
    const int items = info.n_seq * info.n_kv_heads * info.group;
    if (items == 0) return cudaSuccess;
    combine_kernel<<<(items + 3) / 4, 128, 0, s>>>(ws, plan, info.n_seq, info.n_kv_heads, info.group, inverse_fwht,
                                                   out_bf16, out_f32);
    return cudaGetLastError();
}

}  // namespace kvq
