// Device twin of the seeded input generator in kvq_inputs/__init__.py.
//
// Produces rows [row0, row0 + n_rows) of a [rows][H][256] fp32 tensor with the
// same element definition as the numpy generator: SplitMix64 draws at explicit
// counters, an Irwin-Hall normal converted to fp32 once (round to nearest),
// Student-t(3) from four normals with correctly rounded fp32 operations, then
// a per-channel multiplier and a final scale.  Every fp32 step uses an explicit
// round-to-nearest intrinsic, so the output is bit-identical to numpy's.
// This is input generation only; it holds none of the method's arithmetic.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t GAMMA = 0x9E3779B97F4A7C15ull;
constexpr uint64_t MIX1 = 0xBF58476D1CE4E5B9ull;
constexpr uint64_t MIX2 = 0x94D049BB133111EBull;
constexpr uint64_t TKEY = 0xD1B54A32D192ED03ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * MIX1;
    z = (z ^ (z >> 27)) * MIX2;
    return z ^ (z >> 31);
}

__device__ __forceinline__ float normal_at(uint64_t key, uint64_t j) {
    int64_t acc = 0;
#pragma unroll
    for (int r = 0; r < 6; ++r) {
        const uint64_t u = mix64(key + (j * 6 + r + 1) * GAMMA);
        acc += (int64_t)(u >> 40) + (int64_t)((u >> 16) & 0xFFFFFFull);
    }
    acc -= 6ll * (1ll << 24);
    return __fmul_rn(__ll2float_rn(acc), 5.9604644775390625e-08f);   // 2^-24
}

__device__ __forceinline__ float student_t3_at(uint64_t key, uint64_t e) {
    const uint64_t kt = mix64(key ^ TKEY);
    const float z0 = normal_at(key, e);
    const float z1 = normal_at(kt, 3 * e), z2 = normal_at(kt, 3 * e + 1), z3 = normal_at(kt, 3 * e + 2);
    float s = __fadd_rn(__fmul_rn(z1, z1), __fmul_rn(z2, z2));
    s = __fadd_rn(s, __fmul_rn(z3, z3));
    s = __fdiv_rn(s, 3.0f);
    const float r = __fsqrt_rn(s);
    float t = r > 0.f ? __fdiv_rn(z0, r) : 0.f;
    t = fminf(fmaxf(t, -4096.0f), 4096.0f);
    return t;
}

__global__ void gen_rows_kernel(float *out, int64_t row0, int64_t n, int H, uint64_t key, const float *mul,
                                const uint8_t *kind, float post) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int hc = (int)(i % (H * 256));
    const uint64_t e = (uint64_t)(row0 * H * 256) + (uint64_t)i;
    const float z = kind[hc] ? student_t3_at(key, e) : normal_at(key, e);
    out[i] = __fmul_rn(__fmul_rn(z, mul[hc]), post);
}

}  // namespace

extern "C" int kvq_gen_rows(float *out, int64_t row0, int64_t n_rows, int n_heads, uint64_t key, const float *mul,
                            const uint8_t *kind, float post, void *stream) {
    if (!out || !mul || !kind || n_rows < 0 || n_heads <= 0 || row0 < 0) return -1;
    const int64_t n = n_rows * n_heads * 256;
    if (n == 0) return 0;
    const int threads = 256;
    const int64_t blocks = (n + threads - 1) / threads;
    if (blocks > 0x7FFFFFFFll) return -1;
    gen_rows_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(out, row0, n, n_heads, key,
                                                                                         mul, kind, post);
    return cudaGetLastError() == cudaSuccess ? 0 : -4;
}
