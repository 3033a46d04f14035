/*
 * Reference oracle for quantized paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant generator with the CUDA path; the CUDA path never
 * loads it.
 *
 * Plain C11, single threaded, no vector intrinsics.  Built with
 * -ffp-contract=off so that every fp32 expression below is the sequence of
 * correctly rounded IEEE operations written in the source (no fused
 * multiply-add), which is what "bit exact" is measured against.
 *
 * Sources (web pages; cited by title and section):
 *  [Strata]  "KV 沉进内存、显存减半：Strata 让 12 GB 显卡跑满 262K 上下文"
 *            (hotelren.com news 6161890), sections "4-bit KV 缓存：先旋转，再压到
 *            4-bit" and "三种 KV 格式横向对比": 256-point Walsh-Hadamard
 *            rotation of Q, K and V before 4-bit storage; scores unchanged
 *            because <Hq,Hk> = <q,k>; output mixed over rotated V and multiplied
 *            by H again (self-inverse); formats int8 / q4_0 / k8v4 with 1,056 /
 *            576 / (-23%) bytes per token per layer for two KV heads.
 *  [Guide]   anozoder wiki "qwen38-27b-quant-vram-2026", section
 *            "一、为什么 256K 上下文的显存这么吓人": the KV-size formula and the
 *            27B shape (24 Q heads, 4 KV heads, head_dim 256, 16 full-attention
 *            layers); section "二、核心组合表": q4_0 / q8_0 / fp16 KV sizes.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - H_n = H_256 / 16 (Sylvester order, H[i][j] = (-1)^popcount(i&j)), applied
 *    as eight butterfly stages h = 1,2,...,128, pair (i, i+h) -> (a+b, a-b),
 *    then an exact multiply by 1/16.
 *  - q4_0: blocks of 32, d = fp16(signed max / -8) (first index wins a tie in
 *    |x|), code = clamp(rint(x / d) + 8, 0, 15) with true division and
 *    round-half-even, all codes 8 when d rounds to zero.
 *  - int8: groups of 64, d = fp16(max|x| / 127), code = clamp(rint(x / d),
 *    -127, 127), all codes 0 when d rounds to zero.
 *  - Softmax scale 1/sqrt(256) = 1/16.  Q is rotated (q4_0) but never quantised.
 *  - q4_0: K and V rotated; k8v4: V rotated, K not; int8: nothing rotated.
 *  - fp8 ([Roundup] section 一: 516 bytes per position = 2 x (256 + 2)): each
 *    256-vector as OCP FP8 E4M3 codes with one fp16 scale d = fp16(max|x| / 448)
 *    (448 = the largest finite E4M3 value); code = E4M3(x / d), round to
 *    nearest even, saturating to +-448; all codes +0 when d rounds to zero.
 *    Not rotated.
 *  - nvfp4 ([Roundup] section 一: 288 bytes per position = 2 x (128 + 16)):
 *    blocks of 16 values as E2M1 codes (values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and
 *    their negatives) with one E4M3 scale per block, s = E4M3(max|x| / 6)
 *    (round to nearest even, saturating); code = E2M1(x / s), round to nearest
 *    even, saturating to +-6; all codes +0 when s is zero.  No per-tensor
 *    scale (it is not in the 288 bytes).  Not rotated.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define D 256

enum { ORACLE_INT8 = 0, ORACLE_Q4_0 = 1, ORACLE_K8V4 = 2, ORACLE_FP8 = 3, ORACLE_NVFP4 = 4 };
/* how one half (K or V) of a token-kvhead is stored */
enum { PART_INT8 = 0, PART_Q4_0 = 1, PART_E4M3 = 2, PART_E2M1 = 3 };

static int part_n_scales(int part)
{
    switch (part) {
    case PART_INT8: return 4;
    case PART_Q4_0: return 8;
    case PART_E4M3: return 1;
    default: return 16;
    }
}

/* ---------------------------------------------------------------------------
 * IEEE 754 binary32 -> binary16 / bfloat16, round to nearest, ties to even.
 * Written from the format definitions: sign, biased exponent, fraction.
 * ------------------------------------------------------------------------- */
uint16_t oracle_f32_to_f16(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t expf = (x >> 23) & 0xFFu;
    uint32_t frac = x & 0x7FFFFFu;
    if (expf == 0xFFu)                       /* inf / NaN */
        return frac ? (uint16_t)0x7FFFu : (uint16_t)(sign | 0x7C00u);
    if (expf == 0)                           /* fp32 zero or subnormal: < 2^-126, rounds to 0 */
        return (uint16_t)sign;
    int e = (int)expf - 127;                 /* value = 1.frac * 2^e */
    uint64_t mant = (uint64_t)(frac | 0x800000u);   /* 24-bit significand, value = mant * 2^(e-23) */
    /* binary16 quantum: 2^(e-10) for normal results (e >= -14), 2^-24 below */
    int shift = (e >= -14) ? 13 : 13 + (-14 - e);
    if (shift > 25)
        return (uint16_t)sign;               /* below half the smallest subnormal */
    uint64_t q = mant >> shift;
    uint64_t rem = mant & ((1ull << shift) - 1);
    uint64_t half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (q & 1u)))
        q += 1;
    if (e >= -14) {
        /* q in [1024, 2048]; 2048 carries into the exponent field */
        uint32_t bits = ((uint32_t)(e + 15) << 10) + (uint32_t)(q - 1024);
        if (bits >= 0x7C00u)
            return (uint16_t)(sign | 0x7C00u);
        return (uint16_t)(sign | bits);
    }
    return (uint16_t)(sign | (uint32_t)q);   /* subnormal (q == 1024 is the smallest normal) */
}

float oracle_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1Fu;
    uint32_t m = h & 0x3FFu;
    float v;
    if (e == 0)
        v = (float)m * 0x1p-24f;             /* exact: m < 2^10 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexpf((float)(m | 0x400u), (int)e - 25);
    uint32_t bits;
    memcpy(&bits, &v, 4);
    bits |= sign;
    memcpy(&v, &bits, 4);
    return v;
}

uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    if ((x & 0x7F800000u) == 0x7F800000u)
        return (x & 0x7FFFFFu) ? (uint16_t)0x7FFFu : (uint16_t)(x >> 16);
    uint32_t q = x >> 16;                    /* keep sign, exponent, 7 fraction bits */
    uint32_t rem = x & 0xFFFFu;
    if (rem > 0x8000u || (rem == 0x8000u && (q & 1u)))
        q += 1;                              /* a carry into the exponent is the correct result */
    return (uint16_t)q;
}

/* ---------------------------------------------------------------------------
 * OCP 8-bit floating point E4M3 (1 sign, 4 exponent bits with bias 7, 3
 * fraction bits; no infinities; S.1111.111 is NaN; largest finite 448) and
 * 4-bit E2M1 (1 sign, 2 exponent bits with bias 1, 1 fraction bit; values
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6), decoded from the field definitions.
 * ------------------------------------------------------------------------- */
float oracle_e4m3_to_f32(uint8_t b)
{
    int e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);                    /* m/8 * 2^(1-7) */
    else
        v = ldexp(8.0 + m, e - 10);                  /* (1 + m/8) * 2^(e-7) */
    return (float)((b & 0x80) ? -v : v);
}

float oracle_e2m1_to_f32(uint8_t c)
{
    int e = (c >> 1) & 3, m = c & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(2.0 + m, e - 2);   /* (1 + m/2) * 2^(e-1) */
    return (float)((c & 8) ? -v : v);
}

/* |x| rounded to nearest, ties to even, on the grid of a small binary format
 * with `mbits` fraction bits, smallest normal exponent emin and largest finite
 * value vmax; the result saturates at vmax.  Inside the binade [2^e, 2^(e+1))
 * (or below 2^emin) the representable values are the multiples of the quantum
 * 2^(max(e, emin) - mbits), and the binade's first value is an even multiple, so
 * ties to the even multiple are ties to the even code. */
static double round_small_format(double a, int mbits, int emin, double vmax)
{
    if (a == 0.0)
        return 0.0;
    int e;
    frexp(a, &e);                                    /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;                                          /* a in [2^e, 2^(e+1)) */
    if (e < emin)
        e = emin;
    double quantum = ldexp(1.0, e - mbits);
    double r = rint(a / quantum) * quantum;          /* a / quantum is exact (power of two) */
    return r > vmax ? vmax : r;
}

/* Field encoding of a value already on the grid (and within range). */
static uint8_t encode_small_format(double r, int sign, int mbits, int ebits, int bias)
{
    int emin = 1 - bias;
    uint32_t code;
    if (r < ldexp(1.0, emin)) {                      /* subnormal (or zero) */
        code = (uint32_t)(r / ldexp(1.0, emin - mbits));
    } else {
        int e;
        frexp(r, &e);
        e -= 1;
        uint32_t frac = (uint32_t)((r / ldexp(1.0, e) - 1.0) * (double)(1 << mbits));
        code = ((uint32_t)(e + bias) << mbits) | frac;
    }
    return (uint8_t)((sign ? 1u << (ebits + mbits) : 0u) | code);
}

uint8_t oracle_f32_to_e4m3(float x)
{
    int sign = signbit(x) != 0;
    double r = round_small_format(fabs((double)x), 3, -6, 448.0);
    return encode_small_format(r, sign, 3, 4, 7);
}

uint8_t oracle_f32_to_e2m1(float x)
{
    int sign = signbit(x) != 0;
    double r = round_small_format(fabs((double)x), 1, 0, 6.0);
    return encode_small_format(r, sign, 1, 2, 1);
}

/* ---------------------------------------------------------------------------
 * 256-point Walsh-Hadamard transform, normalised (H/16), fp32, fixed order.
 * [Strata] "4-bit KV 缓存": the rotation applied to Q, K and V.
 * ------------------------------------------------------------------------- */
void oracle_fwht256_f32(const float *x, float *y)
{
    float t[D];
    memcpy(t, x, sizeof t);
    for (int h = 1; h < D; h <<= 1)
        for (int i = 0; i < D; ++i)
            if ((i & h) == 0) {
                float a = t[i], b = t[i + h];
                t[i] = a + b;
                t[i + h] = a - b;
            }
    for (int i = 0; i < D; ++i)
        y[i] = t[i] * 0.0625f;
}

/* The same transform in fp64, used to un-rotate the fp64 attention output. */
void oracle_fwht256_f64(const double *x, double *y)
{
    double t[D];
    memcpy(t, x, sizeof t);
    for (int h = 1; h < D; h <<= 1)
        for (int i = 0; i < D; ++i)
            if ((i & h) == 0) {
                double a = t[i], b = t[i + h];
                t[i] = a + b;
                t[i + h] = a - b;
            }
    for (int i = 0; i < D; ++i)
        y[i] = t[i] * 0.0625;
}

/* ---------------------------------------------------------------------------
 * Block quantisers.  One 256-vector in, one code per element out
 * (q4_0: 0..15, stored unpacked; int8: -127..127), fp16 scale bits per block.
 * ------------------------------------------------------------------------- */
void oracle_quant_q4_0(const float *x, uint8_t *codes, uint16_t *scales)
{
    for (int blk = 0; blk < D / 32; ++blk) {
        const float *xb = x + 32 * blk;
        int imax = 0;
        float amax = fabsf(xb[0]);
        for (int j = 1; j < 32; ++j)
            if (fabsf(xb[j]) > amax) {
                amax = fabsf(xb[j]);
                imax = j;
            }
        float d32 = xb[imax] / -8.0f;
        uint16_t d16 = oracle_f32_to_f16(d32);
        float df = oracle_f16_to_f32(d16);
        scales[blk] = d16;
        for (int j = 0; j < 32; ++j) {
            int c = 8;
            if (df != 0.0f) {
                float r = rintf(xb[j] / df);
                c = (int)r + 8;
                if (c < 0) c = 0;
                if (c > 15) c = 15;
            }
            codes[32 * blk + j] = (uint8_t)c;
        }
    }
}

void oracle_quant_int8(const float *x, int8_t *codes, uint16_t *scales)
{
    for (int grp = 0; grp < D / 64; ++grp) {
        const float *xg = x + 64 * grp;
        float amax = 0.0f;
        for (int j = 0; j < 64; ++j)
            if (fabsf(xg[j]) > amax)
                amax = fabsf(xg[j]);
        float d32 = amax / 127.0f;
        uint16_t d16 = oracle_f32_to_f16(d32);
        float df = oracle_f16_to_f32(d16);
        scales[grp] = d16;
        for (int j = 0; j < 64; ++j) {
            int c = 0;
            if (df != 0.0f) {
                float r = rintf(xg[j] / df);
                c = (int)r;
                if (c < -127) c = -127;
                if (c > 127) c = 127;
            }
            codes[64 * grp + j] = (int8_t)c;
        }
    }
}

/* fp8: one 256-vector -> 256 E4M3 codes and one fp16 scale.  [Roundup]
 * section 一 fixes 516 bytes per (layer, KV head) position; the reading is one
 * fp16 scale per vector for K and for V. */
void oracle_quant_fp8(const float *x, uint8_t *codes, uint16_t *scale)
{
    float amax = 0.0f;
    for (int j = 0; j < D; ++j)
        if (fabsf(x[j]) > amax)
            amax = fabsf(x[j]);
    float dq = amax / 448.0f;
    uint16_t dh = oracle_f32_to_f16(dq);
    *scale = dh;
    float d = oracle_f16_to_f32(dh);
    for (int j = 0; j < D; ++j)
        codes[j] = (d == 0.0f) ? 0 : oracle_f32_to_e4m3(x[j] / d);
}

/* nvfp4: one 256-vector -> 256 E2M1 codes (0..15, unpacked) and 16 E4M3 block
 * scales (stored in the low byte of each uint16).  [Roundup] section 一:
 * 288 bytes per position = 2 x (128 code bytes + 16 scale bytes). */
void oracle_quant_nvfp4(const float *x, uint8_t *codes, uint16_t *scales)
{
    for (int b = 0; b < 16; ++b) {
        const float *xb = x + 16 * b;
        float amax = 0.0f;
        for (int j = 0; j < 16; ++j)
            if (fabsf(xb[j]) > amax)
                amax = fabsf(xb[j]);
        uint8_t sb = oracle_f32_to_e4m3(amax / 6.0f);
        scales[b] = sb;
        float sd = oracle_e4m3_to_f32(sb);
        for (int j = 0; j < 16; ++j)
            codes[16 * b + j] = (sd == 0.0f) ? 0 : oracle_f32_to_e2m1(xb[j] / sd);
    }
}

static void quant_part(int part, const float *x, uint8_t *codes, uint16_t *scales)
{
    switch (part) {
    case PART_INT8: oracle_quant_int8(x, (int8_t *)codes, scales); break;
    case PART_Q4_0: oracle_quant_q4_0(x, codes, scales); break;
    case PART_E4M3: oracle_quant_fp8(x, codes, scales); break;
    default: oracle_quant_nvfp4(x, codes, scales); break;
    }
}

/* Layout of one token-kvhead in the oracle's own (unpacked) representation:
 * K codes [256] (one byte per value: q4_0 0..15, int8 two's complement, E4M3
 * bits, E2M1 bits 0..15), K scales [8, 4, 1 or 16] (fp16 bits; E4M3 bits for
 * nvfp4), then the same for V.  Returns 0, or -1 for an unknown format. */
int oracle_format_parts(int fmt, int *k_part, int *v_part, int *k_rot, int *v_rot)
{
    switch (fmt) {
    case ORACLE_INT8: *k_part = PART_INT8; *v_part = PART_INT8; *k_rot = 0; *v_rot = 0; return 0;
    case ORACLE_Q4_0: *k_part = PART_Q4_0; *v_part = PART_Q4_0; *k_rot = 1; *v_rot = 1; return 0;
    case ORACLE_K8V4: *k_part = PART_INT8; *v_part = PART_Q4_0; *k_rot = 0; *v_rot = 1; return 0;
    case ORACLE_FP8: *k_part = PART_E4M3; *v_part = PART_E4M3; *k_rot = 0; *v_rot = 0; return 0;
    case ORACLE_NVFP4: *k_part = PART_E2M1; *v_part = PART_E2M1; *k_rot = 0; *v_rot = 0; return 0;
    default: return -1;
    }
}

/* Encode one token of one KV head: optional rotation, then quantisation.
 * kc/vc: 256 bytes each (q4_0 codes 0..15 or int8 codes as two's complement),
 * ks/vs: 8 (q4_0) or 4 (int8) fp16 scale bits. */
int oracle_append_token(int fmt, const float *k, const float *v,
                        uint8_t *kc, uint16_t *ks, uint8_t *vc, uint16_t *vs)
{
    int kpart, vpart, krot, vrot;
    if (oracle_format_parts(fmt, &kpart, &vpart, &krot, &vrot))
        return -1;
    float tk[D], tv[D];
    if (krot) oracle_fwht256_f32(k, tk); else memcpy(tk, k, sizeof tk);
    if (vrot) oracle_fwht256_f32(v, tv); else memcpy(tv, v, sizeof tv);
    quant_part(kpart, tk, kc, ks);
    quant_part(vpart, tv, vc, vs);
    return 0;
}

/* Batched form: n tokens, row-major [n][256] inputs and outputs. */
int oracle_append_rows(int fmt, long n, const float *k, const float *v,
                       uint8_t *kc, uint16_t *ks, uint8_t *vc, uint16_t *vs)
{
    int kpart, vpart, krot, vrot;
    if (oracle_format_parts(fmt, &kpart, &vpart, &krot, &vrot))
        return -1;
    int nks = part_n_scales(kpart), nvs = part_n_scales(vpart);
    for (long i = 0; i < n; ++i)
        oracle_append_token(fmt, k + D * i, v + D * i, kc + D * i, ks + nks * i, vc + D * i, vs + nvs * i);
    return 0;
}

/* Query preparation: the same rotation as K (q4_0 only), never quantised. */
int oracle_q_prepare(int fmt, const float *q, float *qp, long n_vec)
{
    int kpart, vpart, krot, vrot;
    if (oracle_format_parts(fmt, &kpart, &vpart, &krot, &vrot))
        return -1;
    for (long i = 0; i < n_vec; ++i) {
        if (krot) oracle_fwht256_f32(q + D * i, qp + D * i);
        else memcpy(qp + D * i, q + D * i, D * sizeof(float));
    }
    return 0;
}

/* Dequantisation to fp64: q4_0 (c - 8) * d, int8 c * d, fp8 E4M3(c) * d
 * (d the fp16 scale), nvfp4 E2M1(c) * E4M3(s) per block of 16. */
static void dequant_row(int part, const uint8_t *c, const uint16_t *s, double *out)
{
    if (part == PART_Q4_0) {
        for (int j = 0; j < D; ++j)
            out[j] = (double)((int)c[j] - 8) * (double)oracle_f16_to_f32(s[j / 32]);
    } else if (part == PART_INT8) {
        const int8_t *ci = (const int8_t *)c;
        for (int j = 0; j < D; ++j)
            out[j] = (double)ci[j] * (double)oracle_f16_to_f32(s[j / 64]);
    } else if (part == PART_E4M3) {
        for (int j = 0; j < D; ++j)
            out[j] = (double)oracle_e4m3_to_f32(c[j]) * (double)oracle_f16_to_f32(s[0]);
    } else {
        for (int j = 0; j < D; ++j)
            out[j] = (double)oracle_e2m1_to_f32(c[j]) * (double)oracle_e4m3_to_f32((uint8_t)s[j / 16]);
    }
}

void oracle_dequant_rows(int part, long n, const uint8_t *c, const uint16_t *s, double *out)
{
    int ns = part_n_scales(part);
    for (long i = 0; i < n; ++i)
        dequant_row(part, c + D * i, s + ns * i, out + D * i);
}

/* Partial attention over tokens [t0, t1) of one KV head for G query heads:
 * m[h] = max score, l[h] = sum exp(s - m), o[h][:] = sum exp(s - m) * v_hat
 * (unnormalised), all in fp64 natural-log units.  Scores are q'.k_hat / 16.
 * [Strata] "4-bit KV 缓存": scores on the rotated q and k, mix over rotated V. */
int oracle_attn_partial(int fmt, const float *qp, int G, long t0, long t1,
                        const uint8_t *kc, const uint16_t *ks,
                        const uint8_t *vc, const uint16_t *vs,
                        double *m, double *l, double *o)
{
    int kpart, vpart, krot, vrot;
    if (oracle_format_parts(fmt, &kpart, &vpart, &krot, &vrot) || G <= 0 || t1 <= t0)
        return -1;
    int nks = part_n_scales(kpart), nvs = part_n_scales(vpart);
    long T = t1 - t0;
    double *s = (double *)malloc(sizeof(double) * (size_t)G * (size_t)T);
    if (!s)
        return -2;
    double row[D];
    for (long t = 0; t < T; ++t) {
        dequant_row(kpart, kc + D * (t0 + t), ks + nks * (t0 + t), row);
        for (int h = 0; h < G; ++h) {
            double acc = 0.0;
            for (int j = 0; j < D; ++j)
                acc += (double)qp[D * h + j] * row[j];
            s[(size_t)h * T + t] = acc / 16.0;
        }
    }
    for (int h = 0; h < G; ++h) {
        double mx = -INFINITY;
        for (long t = 0; t < T; ++t)
            if (s[(size_t)h * T + t] > mx)
                mx = s[(size_t)h * T + t];
        m[h] = mx;
        double sum = 0.0;
        for (long t = 0; t < T; ++t) {
            double p = exp(s[(size_t)h * T + t] - mx);
            s[(size_t)h * T + t] = p;
            sum += p;
        }
        l[h] = sum;
        for (int j = 0; j < D; ++j)
            o[D * h + j] = 0.0;
    }
    for (long t = 0; t < T; ++t) {
        dequant_row(vpart, vc + D * (t0 + t), vs + nvs * (t0 + t), row);
        for (int h = 0; h < G; ++h) {
            double p = s[(size_t)h * T + t];
            for (int j = 0; j < D; ++j)
                o[D * h + j] += p * row[j];
        }
    }
    free(s);
    return 0;
}

/* Merge of two partial results (the log-sum-exp rule), in place into a. */
void oracle_merge_partials(int G, double *ma, double *la, double *oa,
                           const double *mb, const double *lb, const double *ob)
{
    for (int h = 0; h < G; ++h) {
        double M = ma[h] > mb[h] ? ma[h] : mb[h];
        double fa = exp(ma[h] - M), fb = exp(mb[h] - M);
        for (int j = 0; j < D; ++j)
            oa[D * h + j] = oa[D * h + j] * fa + ob[D * h + j] * fb;
        la[h] = la[h] * fa + lb[h] * fb;
        ma[h] = M;
    }
}

/* Final output from a (merged) partial: o / l, then H_n o for rotated V. */
int oracle_finish(int fmt, int G, const double *l, const double *o, double *out)
{
    int kpart, vpart, krot, vrot;
    if (oracle_format_parts(fmt, &kpart, &vpart, &krot, &vrot))
        return -1;
    for (int h = 0; h < G; ++h) {
        double tmp[D];
        for (int j = 0; j < D; ++j)
            tmp[j] = o[D * h + j] / l[h];
        if (vrot) oracle_fwht256_f64(tmp, out + D * h);
        else memcpy(out + D * h, tmp, sizeof tmp);
    }
    return 0;
}

/* Split-free single-token decode attention over T tokens of one KV head,
 * G query heads sharing it (GQA).  qp: prepared query [G][256] (rotated for
 * q4_0).  Output [G][256] fp64, un-rotated. */
int oracle_attn_decode(int fmt, const float *qp, int G, long T,
                       const uint8_t *kc, const uint16_t *ks,
                       const uint8_t *vc, const uint16_t *vs, double *out)
{
    if (G <= 0 || G > 64 || T <= 0)
        return -1;
    double m[64], l[64];
    double *o = (double *)malloc(sizeof(double) * (size_t)G * D);
    if (!o)
        return -2;
    int rc = oracle_attn_partial(fmt, qp, G, 0, T, kc, ks, vc, vs, m, l, o);
    if (rc == 0)
        rc = oracle_finish(fmt, G, l, o, out);
    free(o);
    return rc;
}

/* ---------------------------------------------------------------------------
 * Sizes.  [Guide] "一、为什么 256K 上下文的显存这么吓人": KV bytes =
 * 2 x full-attention layers x KV heads x head_dim x bytes per element x context.
 * ------------------------------------------------------------------------- */
double oracle_kv_cache_bytes(int layers, int kv_heads, int head_dim, double bytes_per_elem, double context)
{
    return 2.0 * layers * kv_heads * head_dim * bytes_per_elem * context;
}

/* Bytes of K and V (codes + scales) per token per KV head per layer.
 * int8: 2 x (256 + 4 x 2) = 528; q4_0: 2 x (128 + 8 x 2) = 288;
 * k8v4: (256 + 4 x 2) + (128 + 8 x 2) = 408; fp8: 2 x (256 + 2) = 516;
 * nvfp4: 2 x (128 + 16 x 1) = 288. */
long oracle_format_bytes_per_token_head(int fmt)
{
    switch (fmt) {
    case ORACLE_INT8: return 2 * (256 + 4 * 2);
    case ORACLE_Q4_0: return 2 * (128 + 8 * 2);
    case ORACLE_K8V4: return (256 + 4 * 2) + (128 + 8 * 2);
    case ORACLE_FP8: return 2 * (256 + 1 * 2);
    case ORACLE_NVFP4: return 2 * (128 + 16 * 1);
    default: return -1;
    }
}
