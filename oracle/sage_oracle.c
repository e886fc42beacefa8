/*
 * CPU oracle for 8-bit quantized softmax attention (SageAttention).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library and its Python binding) never calls into it, and the two
 * share no code, headers, tables or constants.
 *
 * It follows the SageAttention article ("又快又准，即插即用！清华8比特量化
 * Attention"), method section, whose three steps are:
 *   - K smoothing: K <- K - mean(K), which leaves softmax(QK^T) unchanged;
 *   - per-block INT8 quantization of Q and K at FlashAttention block size,
 *     with an INT8 matmul accumulating in INT32;
 *   - P and V kept in FP16 for the P V product.
 *
 * Readings where the article is silent (each is a plain choice, listed with
 * its reason in the design notes of the repository):
 *   mean axis   the mean runs over the token axis, one value per channel and
 *               per (batch, kv head), over all Lk tokens.  Only a vector that
 *               is constant across tokens leaves each softmax row unchanged.
 *   mean value  sum = sum_t int64(K[t,c] * 2^24) (exact, fp16 values are
 *               multiples of 2^-24), m = float(double(sum) * 2^-24 / double(Lk)).
 *   quantizer   symmetric, range +-127, per block a = max|x|,
 *               r = fl32(127 / a), q = clamp(rne(fl32(x * r)), -127, 127),
 *               scale = fl32(a / 127).  An all-zero block gives q = 0 and
 *               scale = 0.  For K, x = fl32(float(K) - m).
 *   blocks      Q blocks are 128 rows, K blocks 64 rows, each spanning all d
 *               channels of one (batch, head); the last block holds the
 *               remaining rows only.
 *   sm_scale    folded into Q's scale together with log2(e):
 *               c = fl32(double(sm_scale) * log2(e)), q_scale = fl32(scale * c),
 *               so the softmax runs in base 2.
 *   P rounding  the quantized-path simulation rounds every
 *               p = exp2(s - rowmax) to fp16 and accumulates in fp64.
 *   causal      bottom-right aligned: key j is visible to query i iff
 *               j <= i + Lk - Lq; a row with no visible key outputs 0.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 * All float arithmetic below is IEEE binary32/binary64 with round-to-nearest.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ fp16 */

/* fp16 bit pattern -> exact double. */
double oracle_half_to_double(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);               /* subnormal or zero */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m | 0x400), e - 25);  /* (1.m) * 2^(e-15) */
    return sign ? -v : v;
}

/* double -> fp16 bit pattern, round to nearest, ties to even. */
uint16_t oracle_double_to_half(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x))
        return 0x7e00;
    double a = fabs(x);
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: value = n * 2^-24, n in [0, 1024]; n = 1024 is
           the smallest normal, whose encoding is exactly 0x0400 */
        double n = nearbyint(ldexp(a, 24));
        return sign | (uint16_t)n;
    }
    int e2;
    frexp(a, &e2);              /* a in [2^(e2-1), 2^e2) */
    int E = e2 - 1;             /* unbiased exponent */
    double n = nearbyint(ldexp(a, 10 - E));   /* significand in [1024, 2048] */
    if (n == 2048.0) {
        n = 1024.0;
        E += 1;
    }
    if (E > 15)
        return sign | 0x7c00;   /* overflow to infinity */
    return sign | (uint16_t)(((E + 15) << 10) | ((int)n - 1024));
}

/* --------------------------------------------------------------- K mean */

/* Per-(batch, kv head, channel) mean of K over all Lk tokens (smoothing
 * step).  k: fp16 bits [B, Hkv, Lk, d]; k_mean: float [B, Hkv, d]. */
void oracle_k_mean(const uint16_t *k, int B, int Hkv, int Lk, int d, float *k_mean)
{
    for (int bh = 0; bh < B * Hkv; ++bh) {
        for (int c = 0; c < d; ++c) {
            int64_t sum = 0;
            for (int t = 0; t < Lk; ++t) {
                double v = oracle_half_to_double(k[((int64_t)bh * Lk + t) * d + c]);
                sum += (int64_t)(v * 16777216.0);     /* exact integer */
            }
            double mean = ((double)sum * ldexp(1.0, -24)) / (double)Lk;
            k_mean[(int64_t)bh * d + c] = (float)mean;
        }
    }
}

/* ------------------------------------------------------- block quantizer */

/* Quantize one block of `rows` x `d` fp32 values to int8 with one scale.
 * Returns fl32(a / 127) (0 for an all-zero block). */
static float quant_block(const float *x, int rows, int d, int8_t *q)
{
    float a = 0.0f;
    for (int i = 0; i < rows * d; ++i) {
        float m = fabsf(x[i]);
        if (m > a)
            a = m;
    }
    if (a == 0.0f) {
        memset(q, 0, (size_t)rows * d);
        return 0.0f;
    }
    float r = 127.0f / a;
    for (int i = 0; i < rows * d; ++i) {
        float y = x[i] * r;
        float t = nearbyintf(y);               /* ties to even */
        if (t > 127.0f) t = 127.0f;
        if (t < -127.0f) t = -127.0f;
        q[i] = (int8_t)t;
    }
    return a / 127.0f;
}

/* Block quantization of Q and smoothed K.
 *   q  fp16 [B, H, Lq, d]     -> q_i8 [B, H, Lq, d],  q_scale [B, H, ceil(Lq/128)]
 *   k  fp16 [B, Hkv, Lk, d]   -> k_i8 [B, Hkv, Lk, d], k_scale [B, Hkv, ceil(Lk/64)]
 *   k_mean [B, Hkv, d]        (written)
 * smooth = 0 skips the mean subtraction (ablation only; k_mean is then 0). */
void oracle_quant_qk_blocks(const uint16_t *q, const uint16_t *k, int B, int H, int Hkv,
                            int Lq, int Lk, int d, double sm_scale, int smooth,
                            int BQ, int8_t *q_i8, int8_t *k_i8, float *q_scale,
                            float *k_scale, float *k_mean);

void oracle_quant_qk(const uint16_t *q, const uint16_t *k, int B, int H, int Hkv,
                     int Lq, int Lk, int d, double sm_scale, int smooth,
                     int8_t *q_i8, int8_t *k_i8, float *q_scale, float *k_scale,
                     float *k_mean)
{
    oracle_quant_qk_blocks(q, k, B, H, Hkv, Lq, Lk, d, sm_scale, smooth, 128, q_i8, k_i8,
                           q_scale, k_scale, k_mean);
}

/* Same with Q blocks of BQ rows (1 = one scale per query token); K blocks
 * stay 64 rows.  q_scale is [B, H, ceil(Lq / BQ)]. */
void oracle_quant_qk_blocks(const uint16_t *q, const uint16_t *k, int B, int H, int Hkv,
                            int Lq, int Lk, int d, double sm_scale, int smooth,
                            int BQ, int8_t *q_i8, int8_t *k_i8, float *q_scale,
                            float *k_scale, float *k_mean)
{
    const int BK = 64;
    const int nqb = (Lq + BQ - 1) / BQ, nkb = (Lk + BK - 1) / BK;
    const float c = (float)(sm_scale * 1.4426950408889634074);   /* log2(e) */

    if (smooth)
        oracle_k_mean(k, B, Hkv, Lk, d, k_mean);
    else
        for (int i = 0; i < B * Hkv * d; ++i) k_mean[i] = 0.0f;

    float *buf = (float *)malloc(sizeof(float) * (size_t)(BQ > BK ? BQ : BK) * d);
    for (int bh = 0; bh < B * H; ++bh) {
        for (int blk = 0; blk < nqb; ++blk) {
            int r0 = blk * BQ, rows = Lq - r0 < BQ ? Lq - r0 : BQ;
            const uint16_t *src = q + ((int64_t)bh * Lq + r0) * d;
            for (int i = 0; i < rows * d; ++i)
                buf[i] = (float)oracle_half_to_double(src[i]);
            float s = quant_block(buf, rows, d, q_i8 + ((int64_t)bh * Lq + r0) * d);
            q_scale[(int64_t)bh * nqb + blk] = s * c;
        }
    }
    for (int bh = 0; bh < B * Hkv; ++bh) {
        const float *m = k_mean + (int64_t)bh * d;
        for (int blk = 0; blk < nkb; ++blk) {
            int r0 = blk * BK, rows = Lk - r0 < BK ? Lk - r0 : BK;
            const uint16_t *src = k + ((int64_t)bh * Lk + r0) * d;
            for (int i = 0; i < rows; ++i)
                for (int ch = 0; ch < d; ++ch)
                    buf[i * d + ch] = (float)oracle_half_to_double(src[i * d + ch]) - m[ch];
            k_scale[(int64_t)bh * nkb + blk] =
                quant_block(buf, rows, d, k_i8 + ((int64_t)bh * Lk + r0) * d);
        }
    }
    free(buf);
}

/* ------------------------------------------------------------ attention */

static int64_t visible_keys(int i, int Lq, int Lk, int causal)
{
    if (!causal)
        return Lk;
    int64_t n = (int64_t)i + (Lk - Lq) + 1;
    if (n < 0) n = 0;
    if (n > Lk) n = Lk;
    return n;
}

/* Simulation of the quantized forward pass, in the article's order:
 * S = int32 sum of int8 products (exact), s = S * q_scale * k_scale (already
 * in base-2 units), p = fp16(exp2(s - max s)), O = sum p v / sum p in fp64.
 * rows: flat indices (b*H + h)*Lq + i to compute, or NULL for all rows.
 * out: [n_rows, d] doubles (unrounded output). */
void oracle_attn_quant_sim_blocks(const int8_t *q_i8, const int8_t *k_i8,
                                  const float *q_scale, const float *k_scale,
                                  const uint16_t *v, int B, int H, int Hkv, int Lq, int Lk,
                                  int d, int causal, int BQ, const int64_t *rows,
                                  int64_t n_rows, double *out);

void oracle_attn_quant_sim(const int8_t *q_i8, const int8_t *k_i8,
                           const float *q_scale, const float *k_scale,
                           const uint16_t *v, int B, int H, int Hkv, int Lq, int Lk,
                           int d, int causal, const int64_t *rows, int64_t n_rows,
                           double *out)
{
    oracle_attn_quant_sim_blocks(q_i8, k_i8, q_scale, k_scale, v, B, H, Hkv, Lq, Lk, d, causal,
                                 128, rows, n_rows, out);
}

/* Same for q_scale blocks of BQ rows. */
void oracle_attn_quant_sim_blocks(const int8_t *q_i8, const int8_t *k_i8,
                                  const float *q_scale, const float *k_scale,
                                  const uint16_t *v, int B, int H, int Hkv, int Lq, int Lk,
                                  int d, int causal, int BQ, const int64_t *rows,
                                  int64_t n_rows, double *out)
{
    const int nqb = (Lq + BQ - 1) / BQ, nkb = (Lk + 63) / 64;
    const int group = H / Hkv;
    if (!rows)
        n_rows = (int64_t)B * H * Lq;

#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t flat = rows ? rows[r] : r;
            int i = (int)(flat % Lq);
            int64_t bh = flat / Lq;
            int b = (int)(bh / H), h = (int)(bh % H);
            int64_t bhk = (int64_t)b * Hkv + h / group;
            double *o = out + r * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            int64_t nvis = visible_keys(i, Lq, Lk, causal);
            if (nvis == 0)
                continue;
            const int8_t *qi = q_i8 + (bh * Lq + i) * d;
            double sq = (double)q_scale[bh * nqb + i / BQ];
            double mx = -INFINITY;
            for (int64_t j = 0; j < nvis; ++j) {
                const int8_t *kj = k_i8 + (bhk * Lk + j) * d;
                int32_t acc = 0;
                for (int c = 0; c < d; ++c)
                    acc += (int32_t)qi[c] * (int32_t)kj[c];
                s[j] = (double)acc * sq * (double)k_scale[bhk * nkb + j / 64];
                if (s[j] > mx) mx = s[j];
            }
            double l = 0.0;
            for (int64_t j = 0; j < nvis; ++j) {
                double p = oracle_half_to_double(oracle_double_to_half(exp2(s[j] - mx)));
                l += p;
                const uint16_t *vj = v + (bhk * Lk + j) * d;
                for (int c = 0; c < d; ++c)
                    o[c] += p * oracle_half_to_double(vj[c]);
            }
            for (int c = 0; c < d; ++c) o[c] /= l;
        }
        free(s);
    }
}

/* Full-precision attention straight from the fp16 inputs, no smoothing and no
 * quantization: O = softmax(sm_scale * Q K^T + mask) V in fp64. */
void oracle_attn_fp64(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                      int B, int H, int Hkv, int Lq, int Lk, int d, int causal,
                      double sm_scale, const int64_t *rows, int64_t n_rows, double *out)
{
    const int group = H / Hkv;
    if (!rows)
        n_rows = (int64_t)B * H * Lq;

#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        double *qi = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t flat = rows ? rows[r] : r;
            int i = (int)(flat % Lq);
            int64_t bh = flat / Lq;
            int b = (int)(bh / H), h = (int)(bh % H);
            int64_t bhk = (int64_t)b * Hkv + h / group;
            double *o = out + r * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            int64_t nvis = visible_keys(i, Lq, Lk, causal);
            if (nvis == 0)
                continue;
            for (int c = 0; c < d; ++c)
                qi[c] = oracle_half_to_double(q[(bh * Lq + i) * d + c]);
            double mx = -INFINITY;
            for (int64_t j = 0; j < nvis; ++j) {
                const uint16_t *kj = k + (bhk * Lk + j) * d;
                double acc = 0.0;
                for (int c = 0; c < d; ++c)
                    acc += qi[c] * oracle_half_to_double(kj[c]);
                s[j] = acc * sm_scale;
                if (s[j] > mx) mx = s[j];
            }
            double l = 0.0;
            for (int64_t j = 0; j < nvis; ++j) {
                double p = exp(s[j] - mx);
                l += p;
                const uint16_t *vj = v + (bhk * Lk + j) * d;
                for (int c = 0; c < d; ++c)
                    o[c] += p * oracle_half_to_double(vj[c]);
            }
            for (int c = 0; c < d; ++c) o[c] /= l;
        }
        free(s);
        free(qi);
    }
}

/* ------------------------------------------------------ FP8 (E4M3) P V */

/* SageAttention2 as the pages describe it keeps P and V in FP8 (E4M3) for the
 * P V product.  E4M3 here is the finite-only format with 1 sign bit, 4
 * exponent bits (bias 7) and 3 mantissa bits: normals (1 + m/8) 2^(e-7) for
 * e = 1..15 (e = 15, m = 7 is not a number), subnormals m 2^-9, largest
 * finite value 448.  Conversion rounds to nearest, ties to even, and clamps
 * magnitudes above 448 to 448 (saturating). */
uint8_t oracle_e4m3_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0)
        return sign | 0x7E;
    if (a < 0.015625) {                       /* below 2^-6: subnormal grid 2^-9 */
        double t = a * 512.0;                 /* exact */
        double m = nearbyint(t);              /* ties to even (default rounding mode) */
        return sign | (uint8_t)m;             /* m = 8 is the smallest normal, code 0x08 */
    }
    int e = 0;
    double f = frexp(a, &e);                  /* a = f 2^e, f in [0.5, 1) */
    int ex = e - 1;                           /* a = (2f) 2^ex, 2f in [1, 2) */
    double m = nearbyint((2.0 * f - 1.0) * 8.0);
    if (m == 8.0) { m = 0.0; ++ex; }
    if (ex > 8 || (ex == 8 && m > 6.0))
        return sign | 0x7E;
    return sign | (uint8_t)(((ex + 7) << 3) | (int)m);
}

double oracle_e4m3_decode(uint8_t c)
{
    int e = (c >> 3) & 0xF, m = c & 7;
    double v = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (c & 0x80) ? -v : v;
}

/* V -> E4M3 with one scale per channel over all Lk tokens of a (batch, kv
 * head): a = max_t |V[t, c]|, r = fl32(448 / a), code = e4m3(fl32(V * r)),
 * scale = fl32(a / 448); a zero channel gives codes 0 and scale 0.  The codes
 * are stored channel-major, v8t [B, Hkv, d, Lk]. */
void oracle_quant_v_fp8(const uint16_t *v, int B, int Hkv, int Lk, int d, uint8_t *v8t,
                        float *v_scale)
{
#pragma omp parallel for schedule(static)
    for (int64_t bc = 0; bc < (int64_t)B * Hkv * d; ++bc) {
        int64_t bh = bc / d;
        int c = (int)(bc % d);
        const uint16_t *src = v + bh * Lk * d + c;
        float a = 0.0f;
        for (int t = 0; t < Lk; ++t) {
            float x = (float)fabs(oracle_half_to_double(src[(int64_t)t * d]));
            if (x > a) a = x;
        }
        float r = a > 0.0f ? 448.0f / a : 0.0f;
        uint8_t *dst = v8t + (bh * d + c) * (int64_t)Lk;
        for (int t = 0; t < Lk; ++t) {
            float x = (float)oracle_half_to_double(src[(int64_t)t * d]) * r;
            dst[t] = oracle_e4m3_encode(x);
        }
        v_scale[bh * d + c] = a > 0.0f ? a / 448.0f : 0.0f;
    }
}

/* Quantized forward pass with P and V in E4M3: S, s and the exact row max as
 * in oracle_attn_quant_sim; p = exp2(s - max) in fp64; P8 = e4m3(fl32(fl32(p)
 * * 448)) (p <= 1 maps onto the E4M3 range); O = sum_j e4m3(P8)/448 *
 * e4m3(V8[c][j]) * v_scale[c] / sum_j p (the row sum of the unquantized
 * probabilities). */
void oracle_attn_fp8pv_sim(const int8_t *q_i8, const int8_t *k_i8, const float *q_scale,
                           const float *k_scale, const uint8_t *v8t, const float *v_scale,
                           int B, int H, int Hkv, int Lq, int Lk, int d, int causal, int BQ,
                           const int64_t *rows, int64_t n_rows, double *out)
{
    const int nqb = (Lq + BQ - 1) / BQ, nkb = (Lk + 63) / 64;
    const int group = H / Hkv;
    if (!rows)
        n_rows = (int64_t)B * H * Lq;

#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        double *pq = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t flat = rows ? rows[r] : r;
            int i = (int)(flat % Lq);
            int64_t bh = flat / Lq;
            int b = (int)(bh / H), h = (int)(bh % H);
            int64_t bhk = (int64_t)b * Hkv + h / group;
            double *o = out + r * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            int64_t nvis = visible_keys(i, Lq, Lk, causal);
            if (nvis == 0)
                continue;
            const int8_t *qi = q_i8 + (bh * Lq + i) * d;
            double sq = (double)q_scale[bh * nqb + i / BQ];
            double mx = -INFINITY;
            for (int64_t j = 0; j < nvis; ++j) {
                const int8_t *kj = k_i8 + (bhk * Lk + j) * d;
                int32_t acc = 0;
                for (int c = 0; c < d; ++c)
                    acc += (int32_t)qi[c] * (int32_t)kj[c];
                s[j] = (double)acc * sq * (double)k_scale[bhk * nkb + j / 64];
                if (s[j] > mx) mx = s[j];
            }
            double l = 0.0;
            for (int64_t j = 0; j < nvis; ++j) {
                double p = exp2(s[j] - mx);
                l += p;
                float p448 = (float)p * 448.0f;
                pq[j] = oracle_e4m3_decode(oracle_e4m3_encode(p448)) / 448.0;
            }
            for (int c = 0; c < d; ++c) {
                const uint8_t *vc = v8t + (bhk * d + c) * (int64_t)Lk;
                double acc = 0.0;
                for (int64_t j = 0; j < nvis; ++j)
                    acc += pq[j] * oracle_e4m3_decode(vc[j]);
                o[c] = acc * (double)v_scale[bhk * d + c] / l;
            }
        }
        free(s);
        free(pq);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
