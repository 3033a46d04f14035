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
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define D 256

enum { ORACLE_INT8 = 0, ORACLE_Q4_0 = 1, ORACLE_K8V4 = 2 };

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

/* Layout of one token-kvhead in the oracle's own (unpacked) representation:
 * K codes [256] (uint8 for q4_0, int8 for int8), K scales [8 or 4],
 * V codes [256], V scales [8 or 4].  Returns 0, or -1 for an unknown format. */
int oracle_format_parts(int fmt, int *k_is_q4, int *v_is_q4, int *k_rot, int *v_rot)
{
    switch (fmt) {
    case ORACLE_INT8: *k_is_q4 = 0; *v_is_q4 = 0; *k_rot = 0; *v_rot = 0; return 0;
    case ORACLE_Q4_0: *k_is_q4 = 1; *v_is_q4 = 1; *k_rot = 1; *v_rot = 1; return 0;
    case ORACLE_K8V4: *k_is_q4 = 0; *v_is_q4 = 1; *k_rot = 0; *v_rot = 1; return 0;
    default: return -1;
    }
}

/* Encode one token of one KV head: optional rotation, then quantisation.
 * kc/vc: 256 bytes each (q4_0 codes 0..15 or int8 codes as two's complement),
 * ks/vs: 8 (q4_0) or 4 (int8) fp16 scale bits. */
int oracle_append_token(int fmt, const float *k, const float *v,
                        uint8_t *kc, uint16_t *ks, uint8_t *vc, uint16_t *vs)
{
    int kq4, vq4, krot, vrot;
    if (oracle_format_parts(fmt, &kq4, &vq4, &krot, &vrot))
        return -1;
    float tk[D], tv[D];
    if (krot) oracle_fwht256_f32(k, tk); else memcpy(tk, k, sizeof tk);
    if (vrot) oracle_fwht256_f32(v, tv); else memcpy(tv, v, sizeof tv);
    if (kq4) oracle_quant_q4_0(tk, kc, ks); else oracle_quant_int8(tk, (int8_t *)kc, ks);
    if (vq4) oracle_quant_q4_0(tv, vc, vs); else oracle_quant_int8(tv, (int8_t *)vc, vs);
    return 0;
}

/* Batched form: n tokens, row-major [n][256] inputs and outputs. */
int oracle_append_rows(int fmt, long n, const float *k, const float *v,
                       uint8_t *kc, uint16_t *ks, uint8_t *vc, uint16_t *vs)
{
    int kq4, vq4, krot, vrot;
    if (oracle_format_parts(fmt, &kq4, &vq4, &krot, &vrot))
        return -1;
    int nks = kq4 ? 8 : 4, nvs = vq4 ? 8 : 4;
    for (long i = 0; i < n; ++i)
        oracle_append_token(fmt, k + D * i, v + D * i, kc + D * i, ks + nks * i, vc + D * i, vs + nvs * i);
    return 0;
}

/* Query preparation: the same rotation as K (q4_0 only), never quantised. */
int oracle_q_prepare(int fmt, const float *q, float *qp, long n_vec)
{
    int kq4, vq4, krot, vrot;
    if (oracle_format_parts(fmt, &kq4, &vq4, &krot, &vrot))
        return -1;
    for (long i = 0; i < n_vec; ++i) {
        if (krot) oracle_fwht256_f32(q + D * i, qp + D * i);
        else memcpy(qp + D * i, q + D * i, D * sizeof(float));
    }
    return 0;
}

/* Dequantisation to fp64: q4_0 (c - 8) * d, int8 c * d, d the fp16 scale. */
static void dequant_row(int is_q4, const uint8_t *c, const uint16_t *s, double *out)
{
    if (is_q4) {
        for (int j = 0; j < D; ++j)
            out[j] = (double)((int)c[j] - 8) * (double)oracle_f16_to_f32(s[j / 32]);
    } else {
        const int8_t *ci = (const int8_t *)c;
        for (int j = 0; j < D; ++j)
            out[j] = (double)ci[j] * (double)oracle_f16_to_f32(s[j / 64]);
    }
}

void oracle_dequant_rows(int is_q4, long n, const uint8_t *c, const uint16_t *s, double *out)
{
    int ns = is_q4 ? 8 : 4;
    for (long i = 0; i < n; ++i)
        dequant_row(is_q4, c + D * i, s + ns * i, out + D * i);
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
    int kq4, vq4, krot, vrot;
    if (oracle_format_parts(fmt, &kq4, &vq4, &krot, &vrot) || G <= 0 || t1 <= t0)
        return -1;
    int nks = kq4 ? 8 : 4, nvs = vq4 ? 8 : 4;
    long T = t1 - t0;
    double *s = (double *)malloc(sizeof(double) * (size_t)G * (size_t)T);
    if (!s)
        return -2;
    double row[D];
    for (long t = 0; t < T; ++t) {
        dequant_row(kq4, kc + D * (t0 + t), ks + nks * (t0 + t), row);
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
        dequant_row(vq4, vc + D * (t0 + t), vs + nvs * (t0 + t), row);
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
    int kq4, vq4, krot, vrot;
    if (oracle_format_parts(fmt, &kq4, &vq4, &krot, &vrot))
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

/* Bytes of K and V (codes + fp16 scales) per token per KV head per layer.
 * int8: 2 x (256 + 4 x 2) = 528; q4_0: 2 x (128 + 8 x 2) = 288;
 * k8v4: (256 + 4 x 2) + (128 + 8 x 2) = 408. */
long oracle_format_bytes_per_token_head(int fmt)
{
    switch (fmt) {
    case ORACLE_INT8: return 2 * (256 + 4 * 2);
    case ORACLE_Q4_0: return 2 * (128 + 8 * 2);
    case ORACLE_K8V4: return (256 + 4 * 2) + (128 + 8 * 2);
    default: return -1;
    }
}
