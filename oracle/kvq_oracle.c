/*
 * kvq_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, deliberately unoptimised CPU restatement of decode-phase
 * attention over a KIVI-style low-bit KV cache.  It exists so that tests,
 * the smoke check and the benchmark's CPU-baseline leg can compare the CUDA
 * library against an independent computation.  Nothing in the product
 * library includes, links or calls this file, and this file uses nothing
 * from the product library.
 *
 * Sources (web pages), followed step by step:
 *  - "KV Cache的Int4量化：如何解决Attention Sink导致的量化精度崩塌问题",
 *    section 2 (linear quantization: q = round(x/scale + zero_point),
 *    x' = (q - zero_point) * scale; min-max scale = (max-min)/(2^bits-1),
 *    zero_point = round(-min/scale)) and section 3 (scaled dot-product
 *    attention softmax(Q K^T / sqrt(d_k)) V).
 *  - "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving",
 *    section "核心公式 / 量化基础": asymmetric s = (max-min)/((2^n-1)c),
 *    z = round(-min/s), Xbar = clamp(round(X/s) + z, 0, 2^n-1); symmetric
 *    s = 2 max|X| / ((2^n-1)c), Xbar = clamp(round(X/s), -2^(n-1), 2^(n-1)-1).
 *    The clip factor c is taken as 1 for the KV cache.
 *  - "LLM系列：KVCache量化1 KIVI ...", section 1 (KIVI): keys quantized
 *    per channel in groups of G tokens, values per token; the newest tokens
 *    stay in a full-precision residual X_Kr that is quantized and appended
 *    when it reaches R tokens; A = Concat(A_g, A_r).
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *  - round() is round-half-to-even, evaluated in IEEE fp32, as are the
 *    divisions that feed it (codes are decided in fp32 exactly as written).
 *  - A constant group (max == min) would divide by zero.  Its scale is taken
 *    as |min| (1 when min == 0); the formulas are then applied unchanged,
 *    which gives z = -sign(min), code 0 and an exact reconstruction.
 *  - The symmetric variant stores the offset code u = q + 2^(n-1); an
 *    all-zero group has s = 0 and every u = 2^(n-1).
 *  - Dequantisation and attention are computed in fp64.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math
 *        [-fopenmp] -o liboracle.so kvq_oracle.c -lm
 * (no FMA contraction and no fast-math: every fp32 operation below is the
 *  single IEEE operation written.)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ERANGE 2

/* ------------------------------------------------------------------ */
/* Element widening (exact).                                           */
/* dtype 0 = IEEE fp16, 1 = bfloat16.                                  */
/* ------------------------------------------------------------------ */

float oracle_widen(uint16_t bits, int dtype)
{
    if (dtype == 1) {
        /* bfloat16 is the top half of an fp32 word. */
        uint32_t u = ((uint32_t)bits) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return f;
    }
    /* fp16: 1 sign bit, 5 exponent bits (bias 15), 10 mantissa bits. */
    int sign = (bits >> 15) & 1;
    int e = (bits >> 10) & 0x1f;
    int m = bits & 0x3ff;
    float v;
    if (e == 0)
        v = ldexpf((float)m, -24);              /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexpf((float)(1024 + m), e - 25);  /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* Supported input magnitudes: 0 or within [2^-60, 2^60] and finite. */
static int value_supported(float x)
{
    if (!isfinite(x)) return 0;
    float a = fabsf(x);
    if (a == 0.0f) return 1;
    return a >= 0x1p-60f && a <= 0x1p60f;
}

/* ------------------------------------------------------------------ */
/* Group parameters and codes for one group of values.                */
/* ------------------------------------------------------------------ */

/*
 * Asymmetric min-max parameters (Atom review, 核心公式: s = (max-min)/(2^n-1),
 * z = round(-min/s); zyxy section 2, Min-Max quantization).
 * x[i*stride], i < count.  Returns ORACLE_OK or an error code.
 */
int oracle_asym_params(const float *x, int64_t count, int64_t stride, int bits,
                       float *s_out, int32_t *z_out)
{
    if (count <= 0 || bits < 1 || bits > 8) return ORACLE_EINVAL;
    float mn = x[0], mx = x[0];
    for (int64_t i = 0; i < count; ++i) {
        float v = x[i * stride];
        if (!value_supported(v)) return ORACLE_ERANGE;
        if (v < mn) mn = v;
        if (v > mx) mx = v;
    }
    float L = (float)((1 << bits) - 1);
    float s;
    if (mx > mn)
        s = (mx - mn) / L;
    else
        s = (mn != 0.0f) ? fabsf(mn) : 1.0f;   /* constant group */
    float zf = rintf(-mn / s);
    if (zf < -32768.0f || zf > 32767.0f) return ORACLE_ERANGE;
    *s_out = s;
    *z_out = (int32_t)zf;
    return ORACLE_OK;
}

/* Asymmetric code: clamp(round(x/s) + z, 0, 2^n - 1) (Atom review, 核心公式). */
int oracle_asym_code(float x, float s, int32_t z, int bits)
{
    int32_t L = (1 << bits) - 1;
    int32_t q = (int32_t)rintf(x / s) + z;
    if (q < 0) q = 0;
    if (q > L) q = L;
    return q;
}

/*
 * Symmetric parameters (Atom review, 核心公式: s = 2 max|X| / (2^n - 1)).
 * An all-zero group gets s = 0.
 */
int oracle_sym_params(const float *x, int64_t count, int64_t stride, int bits,
                      float *s_out)
{
    if (count <= 0 || bits < 2 || bits > 8) return ORACLE_EINVAL;
    float A = 0.0f;
    for (int64_t i = 0; i < count; ++i) {
        float v = x[i * stride];
        if (!value_supported(v)) return ORACLE_ERANGE;
        float a = fabsf(v);
        if (a > A) A = a;
    }
    float L = (float)((1 << bits) - 1);
    *s_out = (2.0f * A) / L;
    return ORACLE_OK;
}

/*
 * Symmetric code, stored offset-binary: u = clamp(round(x/s), -2^(n-1),
 * 2^(n-1) - 1) + 2^(n-1)  (Atom review, 核心公式, symmetric form).
 */
int oracle_sym_code(float x, float s, int bits)
{
    int32_t half = 1 << (bits - 1);
    if (s == 0.0f) return half;
    int32_t q = (int32_t)rintf(x / s);
    if (q < -half) q = -half;
    if (q > half - 1) q = half - 1;
    return q + half;
}

/* ------------------------------------------------------------------ */
/* KIVI quantisation of a block of tokens.                             */
/* ------------------------------------------------------------------ */

/*
 * Quantise T tokens of K and V for every (batch, kv-head) slice.
 *   XK, XV : element bits [BH][T][d]   (row t of slice bh at (bh*T + t)*d)
 *   Keys   : per channel, groups of G consecutive tokens
 *            -> Kq [BH][T][d] codes, Ks/Kz [BH][T/G][d]
 *   Values : per token, groups of Gv consecutive channels
 *            -> Vq [BH][T][d] codes, Vs/Vz [BH][T][d/Gv]
 * (KIVI: Key per-channel, Value per-token.)  Symmetric mode writes no
 * zeros (Kz/Vz may be NULL).  T must be a multiple of G.
 */
int oracle_quantize_kv(const uint16_t *XK, const uint16_t *XV, int dtype,
                       int64_t BH, int64_t T, int d, int G, int Gv, int bits,
                       int symmetric,
                       uint8_t *Kq, float *Ks, int16_t *Kz,
                       uint8_t *Vq, float *Vs, int16_t *Vz)
{
    if (BH < 0 || T < 0 || d <= 0 || G <= 0 || Gv <= 0) return ORACLE_EINVAL;
    if (T % G != 0 || d % Gv != 0) return ORACLE_EINVAL;
    if (symmetric && bits < 2) return ORACLE_EINVAL;
    int status = ORACLE_OK;
    int64_t ngroups = T / G;
    int nvg = d / Gv;

#pragma omp parallel for schedule(dynamic)
    for (int64_t bh = 0; bh < BH; ++bh) {
        float *kx = (float *)malloc(sizeof(float) * (size_t)(G * d));
        float *vx = (float *)malloc(sizeof(float) * (size_t)d);
        if (!kx || !vx) {
            free(kx); free(vx);
#pragma omp atomic write
            status = ORACLE_EINVAL;
            continue;
        }
        /* Keys: one group = G tokens; one scale/zero per channel. */
        for (int64_t g = 0; g < ngroups; ++g) {
            for (int t = 0; t < G; ++t)
                for (int c = 0; c < d; ++c)
                    kx[t * d + c] =
                        oracle_widen(XK[((bh * T) + g * G + t) * d + c], dtype);
            for (int c = 0; c < d; ++c) {
                float s;
                int32_t z = 0;
                int rc = symmetric
                    ? oracle_sym_params(kx + c, G, d, bits, &s)
                    : oracle_asym_params(kx + c, G, d, bits, &s, &z);
                if (rc != ORACLE_OK) {
#pragma omp atomic write
                    status = rc;
                    s = 1.0f;
                    z = 0;
                }
                Ks[(bh * ngroups + g) * d + c] = s;
                if (!symmetric) Kz[(bh * ngroups + g) * d + c] = (int16_t)z;
                for (int t = 0; t < G; ++t) {
                    float x = kx[t * d + c];
                    int q = symmetric ? oracle_sym_code(x, s, bits)
                                      : oracle_asym_code(x, s, z, bits);
                    Kq[((bh * T) + g * G + t) * d + c] = (uint8_t)q;
                }
            }
        }
        /* Values: one group = Gv consecutive channels of one token. */
        for (int64_t t = 0; t < T; ++t) {
            for (int c = 0; c < d; ++c)
                vx[c] = oracle_widen(XV[(bh * T + t) * d + c], dtype);
            for (int j = 0; j < nvg; ++j) {
                float s;
                int32_t z = 0;
                int rc = symmetric
                    ? oracle_sym_params(vx + j * Gv, Gv, 1, bits, &s)
                    : oracle_asym_params(vx + j * Gv, Gv, 1, bits, &s, &z);
                if (rc != ORACLE_OK) {
#pragma omp atomic write
                    status = rc;
                    s = 1.0f;
                    z = 0;
                }
                Vs[(bh * T + t) * nvg + j] = s;
                if (!symmetric) Vz[(bh * T + t) * nvg + j] = (int16_t)z;
                for (int c = j * Gv; c < (j + 1) * Gv; ++c) {
                    int q = symmetric ? oracle_sym_code(vx[c], s, bits)
                                      : oracle_asym_code(vx[c], s, z, bits);
                    Vq[(bh * T + t) * d + c] = (uint8_t)q;
                }
            }
        }
        free(kx);
        free(vx);
    }
    return status;
}

/* ------------------------------------------------------------------ */
/* Packed layout of the codes.                                         */
/* ------------------------------------------------------------------ */

/*
 * Position of code (token t, channel c) of one (batch, kv-head) slice in
 * its packed uint32 array.  The layout is this library's own storage format
 * (the pages fix none); the CUDA side writes and reads the same format:
 *
 *  - tokens are cut into tiles of 16, channels into chunks of 16;
 *  - a tile holds 16*d*n bits = d*n/2 words, tile i at word i*d*n/2;
 *  - inside a tile, 32 "lanes" own W = d*n/64 consecutive words each;
 *  - within chunk j, a 16x16 block is indexed (row, col): keys use
 *    (row, col) = (t%16, c%16), values use (row, col) = (c%16, t%16);
 *  - lane = 4*(row%8) + col/4, byte = col%4, half = row/8;
 *  - a word holds B = 4/n blocks of a lane: block j sits in word j/B,
 *    slot s = 2*(j%B) + half, and the code at bit 8*byte + n*s.
 * So (word >> n*s) masked to the low n bits of every byte yields four codes
 * of one row, one per byte.
 */
void oracle_code_position(int64_t t, int c, int is_v, int d, int bits,
                          int64_t *word, int *bit)
{
    int64_t tile = t / 16;
    int row = is_v ? (c % 16) : (int)(t % 16);
    int col = is_v ? (int)(t % 16) : (c % 16);
    int j = c / 16;
    int lane = 4 * (row % 8) + col / 4;
    int byte = col % 4;
    int half = row / 8;
    int B = 4 / bits;
    int W = d * bits / 64;
    int slot = 2 * (j % B) + half;
    *word = tile * (int64_t)(d * bits / 2) + (int64_t)lane * W + j / B;
    *bit = 8 * byte + bits * slot;
}

/* Pack codes q [BH][T][d] (T a multiple of 16) into words [BH][T*d*n/32]. */
int oracle_pack(const uint8_t *q, int64_t BH, int64_t T, int d, int bits,
                int is_v, uint32_t *out)
{
    if ((bits != 2 && bits != 4) || T % 16 != 0 || d % 32 != 0)
        return ORACLE_EINVAL;
    int64_t words = T * d * bits / 32;
    memset(out, 0, sizeof(uint32_t) * (size_t)(BH * words));
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t t = 0; t < T; ++t)
            for (int c = 0; c < d; ++c) {
                int64_t w;
                int b;
                oracle_code_position(t, c, is_v, d, bits, &w, &b);
                uint32_t code = q[(bh * T + t) * d + c];
                out[bh * words + w] |= code << b;
            }
    return ORACLE_OK;
}

/* Inverse of oracle_pack. */
int oracle_unpack(const uint32_t *in, int64_t BH, int64_t T, int d, int bits,
                  int is_v, uint8_t *q)
{
    if ((bits != 2 && bits != 4) || T % 16 != 0 || d % 32 != 0)
        return ORACLE_EINVAL;
    int64_t words = T * d * bits / 32;
    uint32_t mask = (1u << bits) - 1u;
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t t = 0; t < T; ++t)
            for (int c = 0; c < d; ++c) {
                int64_t w;
                int b;
                oracle_code_position(t, c, is_v, d, bits, &w, &b);
                q[(bh * T + t) * d + c] =
                    (uint8_t)((in[bh * words + w] >> b) & mask);
            }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Dequantisation (fp64) and decode attention.                         */
/* ------------------------------------------------------------------ */

/* x' = (q - z) * s in fp64 (zyxy section 2; symmetric: z = 2^(n-1)). */
double oracle_dequant(int code, float s, int32_t z)
{
    return (double)(code - z) * (double)s;
}

/*
 * One decode step for every (batch, query head):
 *   keys   = [deq(K_g) for tokens 0..Tq-1 ; residual rows 0..r-1]
 *   values = [deq(V_g) ; residual]
 *   out    = softmax(q . keys^T / sqrt(d)) . values        (fp64)
 * KIVI section 1 (A = Concat(A_g, A_r), t_O = A X_V) with the 1/sqrt(d_k)
 * of zyxy section 3.  Query head i reads kv head i / (Hq/Hkv).
 *
 *   Kq, Vq  codes [B*Hkv][Tq][d];   Ks, Kz [B*Hkv][Tq/G][d];
 *   Vs, Vz  [B*Hkv][Tq][d/Gv];      Kr, Vr element bits [B*Hkv][Rcap][d]
 *   (first r rows valid);  Q element bits [B][Hq][d];  out [B][Hq][d].
 *   Symmetric mode: Kz/Vz ignored, z = 2^(n-1).
 *   max_out, denom_out [B][Hq] (each may be NULL): the largest scaled logit m
 *   and sum_t exp(logit_t - m), the statistics with which outputs over
 *   disjoint token sets merge into the output over their union (the order-free
 *   concatenation of the LogQuant summary, section 4).
 */
int oracle_decode_attention(const uint8_t *Kq, const float *Ks, const int16_t *Kz,
                            const uint8_t *Vq, const float *Vs, const int16_t *Vz,
                            int64_t Tq, const uint16_t *Kr, const uint16_t *Vr,
                            int64_t Rcap, int64_t r, const uint16_t *Q,
                            int dtype, int64_t B, int Hq, int Hkv, int d, int G,
                            int Gv, int bits, int symmetric, double *out,
                            double *max_out, double *denom_out)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0) return ORACLE_EINVAL;
    if (Tq < 0 || r < 0 || r > Rcap || (Tq > 0 && (Tq % G != 0 || d % Gv != 0)))
        return ORACLE_EINVAL;
    int64_t T = Tq + r;
    if (T == 0) return ORACLE_EINVAL;
    int grp = Hq / Hkv;
    int nvg = d / Gv;
    int64_t ngroups = Tq / G;
    int32_t symz = 1 << (bits - 1);
    int status = ORACLE_OK;

#pragma omp parallel for schedule(dynamic)
    for (int64_t bi = 0; bi < B * (int64_t)Hq; ++bi) {
        int64_t b = bi / Hq;
        int i = (int)(bi % Hq);
        int64_t bh = b * Hkv + i / grp;
        double *q = (double *)malloc(sizeof(double) * (size_t)d);
        double *logit = (double *)malloc(sizeof(double) * (size_t)T);
        if (!q || !logit) {
            free(q); free(logit);
#pragma omp atomic write
            status = ORACLE_EINVAL;
            continue;
        }
        for (int c = 0; c < d; ++c)
            q[c] = (double)oracle_widen(Q[(b * Hq + i) * d + c], dtype);
        double inv_sqrt_d = 1.0 / sqrt((double)d);

        /* A_g: logits against the dequantised quantised tokens. */
        for (int64_t t = 0; t < Tq; ++t) {
            int64_t g = t / G;
            double acc = 0.0;
            for (int c = 0; c < d; ++c) {
                float s = Ks[(bh * ngroups + g) * d + c];
                int32_t z = symmetric ? symz : Kz[(bh * ngroups + g) * d + c];
                acc += q[c] * oracle_dequant(Kq[(bh * Tq + t) * d + c], s, z);
            }
            logit[t] = acc * inv_sqrt_d;
        }
        /* A_r: logits against the full-precision residual rows. */
        for (int64_t t = 0; t < r; ++t) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += q[c] * (double)oracle_widen(Kr[(bh * Rcap + t) * d + c], dtype);
            logit[Tq + t] = acc * inv_sqrt_d;
        }
        /* softmax over the concatenation (max-subtracted). */
        double mx = logit[0];
        for (int64_t t = 1; t < T; ++t)
            if (logit[t] > mx) mx = logit[t];
        double denom = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            logit[t] = exp(logit[t] - mx);
            denom += logit[t];
        }
        /* t_O = A . X_V */
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            int j = c / Gv;
            for (int64_t t = 0; t < Tq; ++t) {
                float s = Vs[(bh * Tq + t) * nvg + j];
                int32_t z = symmetric ? symz : Vz[(bh * Tq + t) * nvg + j];
                acc += logit[t] * oracle_dequant(Vq[(bh * Tq + t) * d + c], s, z);
            }
            for (int64_t t = 0; t < r; ++t)
                acc += logit[Tq + t] *
                       (double)oracle_widen(Vr[(bh * Rcap + t) * d + c], dtype);
            out[(b * Hq + i) * d + c] = acc / denom;
        }
        /* the softmax statistics, for merging with other token sets (max_out, denom_out may be NULL) */
        if (max_out) max_out[b * Hq + i] = mx;
        if (denom_out) denom_out[b * Hq + i] = denom;
        free(q);
        free(logit);
    }
    return status;
}

/* Number of threads the parallel loops above use. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the later parallel sections (n >= 1); returns the previous count.
 * Only the timing of the oracle depends on it, never a result. */
int oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    const int old = omp_get_max_threads();
    if (n >= 1) omp_set_num_threads(n);
    return old;
#else
    (void)n;
    return 1;
#endif
}
