/*
 * vc_oracle.c - plain, slow CPU oracle for VC-Attention (the FP8 path and the
 * NVFP4-residual variant).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the library's product path may link,
 * load or call this file; only tests, the smoke check and the bench's CPU
 * baseline do. It shares no code with the CUDA path (no common headers,
 * helpers, tables or constant generators).
 *
 * Every function restates one step of the method as the pages describe it,
 * in the pages' order, in double precision where the step is a sum, and
 * with each rounding written out where the method rounds. It is compiled
 * with -ffp-contract=off so that the compiler fuses nothing: the only fused
 * multiply-adds are the explicit fmaf() calls, which are the method's.
 *
 * Sources (web pages, cited by title and section):
 *  [VCA]  "VC-Attention acelera atenção em modelos de vídeo de IA em até
 *          3,58× sem retreinamento" (noticiai.com.br)
 *          - "Por que a atenção é o gargalo": low-bit tensor cores for QK and
 *            PV; prior methods smooth queries and keys.
 *          - "V-Smooth: corrigindo outliers de valor": Group / Demean / Restore.
 *          - "ExpCast-FP8: eliminando o gargalo do softmax": byte ~ 8 log2 v + 56.
 *  [IP73] "VC-Attention et FLUX 3 accélèrent la génération d'images sur
 *          Blackwell" (ip73.fr), section "Le compromis entre vitesse et
 *          fidélité": repair budget rho = 0.005 for the tokens with the largest
 *          quantization error.
 *
 * Readings where the pages leave a step open are marked [R] and listed in
 * the design notes; the main ones:
 *  - Frames: the online softmax keeps its running max m (in "byte units",
 *    1/8 of a log2 step) and writes bytes against the frame F = 8*ceil(m/8),
 *    so frame changes rescale by exact powers of two.
 *  - ExpCast bias C (default 120): the row maximum maps to value 2^8, the
 *    pages' constant 56 is the E4M3 encoding offset of the identity.
 *  - V residual scale: per (b,h,channel) over all tokens, a power of two.
 *  - Repair adds bf16(residual error) to the selected tokens' values.
 *
 * Parity pins live in tests/test_oracle_*.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define TILE 128

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

/* bf16 bit pattern -> value (bf16 is the top half of an IEEE binary32). */
float orc_bf16_value(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* binary32 -> bf16, round to nearest, ties to even (finite inputs). */
uint16_t orc_bf16_round(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    uint32_t kept = u & 0xFFFF0000u;
    uint32_t dropped = u & 0x0000FFFFu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 0x10000u)))
        kept += 0x10000u; /* carries into the exponent when the mantissa overflows */
    return (uint16_t)(kept >> 16);
}

/* OCP FP8 E4M3 ("E4M3FN"): 1 sign, 4 exponent bits (bias 7), 3 mantissa
 * bits; no infinities; S.1111.111 is NaN; largest finite 448 = 1.75*2^8;
 * exponent field 0 is subnormal with value m/8 * 2^-6. */
double orc_e4m3_value(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);          /* m/8 * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* binary32 -> E4M3, round to nearest, ties to even, saturating to +/-448
 * ("satfinite"). The grid spacing in the binade [2^E, 2^(E+1)) is 2^(E-3);
 * below 2^-6 the grid is the subnormal spacing 2^-9. */
uint8_t orc_e4m3_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    int E, ex, code;
    double q, r, val;
    if (isnan(x))
        return (uint8_t)(sign | 0x7F);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);
    if (a == 0.0)
        return sign;
    frexp(a, &E);      /* a = f * 2^E, f in [0.5, 1): floor(log2 a) = E - 1 */
    ex = E - 1;
    if (ex < -6)
        ex = -6;
    q = ldexp(1.0, ex - 3);
    r = nearbyint(a / q); /* a/q is exact; default mode rounds ties to even */
    val = r * q;          /* in [0, 448]: a < 448 keeps r <= 14 in the top binade */
    if (val == 0.0)
        return sign;
    frexp(val, &E);
    ex = E - 1;
    if (ex < -6)
        code = (int)(val / ldexp(1.0, -9));                   /* subnormal m */
    else
        code = ((ex + 7) << 3) | ((int)(val / ldexp(1.0, ex - 3)) - 8);
    return (uint8_t)(sign | code);
}

/* OCP FP4 E2M1, defined with the NVFP4 variant below. */
double orc_e2m1_value(uint8_t code);
uint8_t orc_e2m1_encode(float x);

/* ------------------------------------------------------------------ */
/* ExpCast-FP8 ([VCA] "ExpCast-FP8: eliminando o gargalo do softmax")   */
/* ------------------------------------------------------------------ */
/* An E4M3 byte read as an integer is close to 8*log2(v) + 56. With the
 * score already in byte units (acc*alpha, alpha folding 8*log2(e)*scale and
 * the Q/K dequantization scales) the byte is written by ONE fused
 * multiply-add against the frame offset c = C - F, then taken to the nearest
 * integer (ties to even) and clamped to the finite non-negative codes
 * [0, 126]. */
int orc_expcast_byte(float acc, float alpha, float c)
{
    float v = fmaf(acc, alpha, c); /* single rounding to binary32 */
    float r = rintf(v);             /* nearest integer, ties to even */
    if (!(r > 0.0f))
        return 0;                   /* negatives, -0 and NaN */
    if (r > 126.0f)
        return 126;
    return (int)r;
}

/* kappa = 8 * log2(e) * softmax_scale, rounded once to binary32. */
float orc_kappa(float softmax_scale)
{
    return (float)(8.0 * 1.4426950408889634074 * (double)softmax_scale);
}

/* ------------------------------------------------------------------ */
/* V-Smooth, Group ([VCA] "V-Smooth…", item Group)                      */
/* ------------------------------------------------------------------ */
/* Lloyd k-means on the value tokens of one (b,h), deterministic:
 *  init   c_j = V[floor(j*N/k)]                                      [R]
 *  assign d(n,j) = sum_c (v_nc - c_jc)^2 accumulated by fmaf in channel
 *         order c = 0..d-1 from 0; label = argmin_j, ties to lowest j
 *  update c_j = fp32(sum_fp64 / count); an empty cluster keeps c_j
 * `iters` assign+update rounds, then one final assignment gives the labels. */
static void kmeans_assign(const uint16_t *V, int N, int d, int k, const float *cent, int32_t *labels)
{
    for (int n = 0; n < N; ++n) {
        const uint16_t *v = V + (size_t)n * d;
        int best = 0;
        float bestd = 0.0f;
        for (int j = 0; j < k; ++j) {
            float acc = 0.0f;
            for (int c = 0; c < d; ++c) {
                float x = orc_bf16_value(v[c]) - cent[(size_t)j * d + c];
                acc = fmaf(x, x, acc);
            }
            if (j == 0 || acc < bestd) {
                bestd = acc;
                best = j;
            }
        }
        labels[n] = best;
    }
}

/* warm != 0: the iterations start from the centroids already in `cent` (the
 * previous denoising step's, [VCA] "V-Smooth", Group: the grouping is online
 * and runs only in the first quarter of the steps) instead of the tokens
 * floor(j N / k). */
void orc_kmeans_head(const uint16_t *V, int N, int d, int k, int iters, float *cent, int32_t *labels, int warm)
{
    double *sum = (double *)calloc((size_t)k * d, sizeof(double));
    long long *cnt = (long long *)calloc((size_t)k, sizeof(long long));
    for (int j = 0; j < k && !warm; ++j) {
        int src = (int)(((long long)j * N) / k);
        for (int c = 0; c < d; ++c)
            cent[(size_t)j * d + c] = orc_bf16_value(V[(size_t)src * d + c]);
    }
    for (int it = 0; it < iters; ++it) {
        kmeans_assign(V, N, d, k, cent, labels);
        memset(sum, 0, (size_t)k * d * sizeof(double));
        memset(cnt, 0, (size_t)k * sizeof(long long));
        for (int n = 0; n < N; ++n) {
            int j = labels[n];
            cnt[j] += 1;
            for (int c = 0; c < d; ++c)
                sum[(size_t)j * d + c] += (double)orc_bf16_value(V[(size_t)n * d + c]);
        }
        for (int j = 0; j < k; ++j)
            if (cnt[j] > 0)
                for (int c = 0; c < d; ++c)
                    cent[(size_t)j * d + c] = (float)(sum[(size_t)j * d + c] / (double)cnt[j]);
    }
    kmeans_assign(V, N, d, k, cent, labels);
    free(sum);
    free(cnt);
}

/* The permutation: token indices stably sorted by cluster label, so that the
 * tokens of a cluster are contiguous and keep their original order.
 * perm[p] = original index of the token at permuted position p. K and V are
 * both read through perm ("chaves e valores são permutados juntos"). */
void orc_stable_sort_labels(const int32_t *labels, int N, int k, int32_t *perm)
{
    long long *start = (long long *)calloc((size_t)k + 1, sizeof(long long));
    for (int n = 0; n < N; ++n)
        start[labels[n] + 1] += 1;
    for (int j = 0; j < k; ++j)
        start[j + 1] += start[j];
    for (int n = 0; n < N; ++n)
        perm[start[labels[n]]++] = n;
    free(start);
}

/* ------------------------------------------------------------------ */
/* Q/K smoothing and 8-bit quantization ([VCA] "Por que a atenção é o   */
/* gargalo": low-bit tensor cores for QK; prior methods smooth Q and K) */
/* ------------------------------------------------------------------ */
/* [R] K smoothing subtracts the per-(b,h) channel mean of K (this shifts
 * every score of a query row by the same amount, which softmax ignores);
 * Q is not smoothed. Q (original order) and K' (permuted order) are
 * quantized per 128-row block: scale = amax/448, codes = E4M3(x * 448/amax). */
static void quant_block_rows(const float *X, int rows, int d, uint8_t *codes, float *scale)
{
    float amax = 0.0f, mult;
    for (int i = 0; i < rows * d; ++i) {
        float a = fabsf(X[i]);
        if (a > amax)
            amax = a;
    }
    if (amax == 0.0f) {
        *scale = 0.0f;
        mult = 0.0f;
    } else {
        *scale = amax / 448.0f;
        mult = 448.0f / amax;
    }
    for (int i = 0; i < rows * d; ++i)
        codes[i] = orc_e4m3_encode(X[i] * mult);
}

void orc_quant_qk_head(const uint16_t *Q, const uint16_t *K, const int32_t *perm, int N, int d, int ksmooth,
                       uint8_t *q8, float *sq, uint8_t *k8, float *sk, float *kbar)
{
    int Nb = (N + TILE - 1) / TILE;
    float *blk = (float *)malloc((size_t)TILE * d * sizeof(float));
    for (int c = 0; c < d; ++c) {
        double s = 0.0;
        for (int n = 0; n < N; ++n)
            s += (double)orc_bf16_value(K[(size_t)n * d + c]);
        kbar[c] = ksmooth ? (float)(s / (double)N) : 0.0f;
    }
    memset(q8, 0, (size_t)Nb * TILE * d);
    memset(k8, 0, (size_t)Nb * TILE * d);
    for (int t = 0; t < Nb; ++t) {
        int r0 = t * TILE, rows = (N - r0 < TILE) ? N - r0 : TILE;
        for (int i = 0; i < rows; ++i)
            for (int c = 0; c < d; ++c)
                blk[(size_t)i * d + c] = orc_bf16_value(Q[(size_t)(r0 + i) * d + c]);
        quant_block_rows(blk, rows, d, q8 + (size_t)r0 * d, &sq[t]);
        for (int i = 0; i < rows; ++i) {
            int src = perm[r0 + i];
            for (int c = 0; c < d; ++c)
                blk[(size_t)i * d + c] = orc_bf16_value(K[(size_t)src * d + c]) - kbar[c];
        }
        quant_block_rows(blk, rows, d, k8 + (size_t)r0 * d, &sk[t]);
    }
    free(blk);
}

/* NVFP4 Q and K' for the full 4-bit path [R]: the same smoothing and row
 * order as orc_quant_qk_head; per 128-row block a power-of-two global scale
 * g = 2^e, the least with amax <= 2688 * 2^e over the block (1 when the block
 * is all zero); per row and 16 consecutive channels the E4M3 scale
 * sf = E4M3(fl(fl(b * 2^-e) / 6)) of the block maximum b, and the codes
 * E2M1(fl(fl(x * 2^-e) * fl(1 / sf))) (every code 0 when sf is 0): the value
 * format of the NVFP4 residual, with the blocks along the channels (the K
 * dimension of QK^T). Outputs: codes [Nb*128][d] (padding rows 0),
 * sfc [Nb*128][d/16], g [Nb]. */
static void quant4_block_rows(const float *X, int rows, int d, uint8_t *codes, uint8_t *sfc, float *g)
{
    float amax = 0.0f;
    int e = 0, E, db = d / 16;
    for (int i = 0; i < rows * d; ++i)
        if (fabsf(X[i]) > amax)
            amax = fabsf(X[i]);
    if (amax > 0.0f) {
        float f = frexpf(amax, &E); /* 2688 = 0.65625 * 2^12 */
        e = (f > 0.65625f) ? E - 11 : E - 12;
    }
    *g = ldexpf(1.0f, e);
    for (int i = 0; i < rows; ++i)
        for (int jb = 0; jb < db; ++jb) {
            const float *x = X + (size_t)i * d + 16 * jb;
            float b = 0.0f, sfv, rcp;
            uint8_t sc;
            for (int c = 0; c < 16; ++c)
                if (fabsf(x[c]) > b)
                    b = fabsf(x[c]);
            sc = orc_e4m3_encode(ldexpf(b, -e) / 6.0f);
            sfv = (float)orc_e4m3_value(sc);
            rcp = (sfv == 0.0f) ? 0.0f : 1.0f / sfv;
            sfc[(size_t)i * db + jb] = sc;
            for (int c = 0; c < 16; ++c)
                codes[(size_t)i * d + 16 * jb + c] = (sfv == 0.0f) ? 0 : orc_e2m1_encode(ldexpf(x[c], -e) * rcp);
        }
}

void orc_quant_qk4_head(const uint16_t *Q, const uint16_t *K, const int32_t *perm, int N, int d, int ksmooth,
                        uint8_t *qcodes, uint8_t *qsfc, float *qg, uint8_t *kcodes, uint8_t *ksfc, float *kg,
                        float *kbar)
{
    int Nb = (N + TILE - 1) / TILE, db = d / 16;
    float *blk = (float *)malloc((size_t)TILE * d * sizeof(float));
    for (int c = 0; c < d; ++c) {
        double s = 0.0;
        for (int n = 0; n < N; ++n)
            s += (double)orc_bf16_value(K[(size_t)n * d + c]);
        kbar[c] = ksmooth ? (float)(s / (double)N) : 0.0f;
    }
    memset(qcodes, 0, (size_t)Nb * TILE * d);
    memset(kcodes, 0, (size_t)Nb * TILE * d);
    memset(qsfc, 0, (size_t)Nb * TILE * db);
    memset(ksfc, 0, (size_t)Nb * TILE * db);
    for (int t = 0; t < Nb; ++t) {
        int r0 = t * TILE, rows = (N - r0 < TILE) ? N - r0 : TILE;
        for (int i = 0; i < rows; ++i)
            for (int c = 0; c < d; ++c)
                blk[(size_t)i * d + c] = orc_bf16_value(Q[(size_t)(r0 + i) * d + c]);
        quant4_block_rows(blk, rows, d, qcodes + (size_t)r0 * d, qsfc + (size_t)r0 * db, &qg[t]);
        for (int i = 0; i < rows; ++i) {
            int src = perm[r0 + i];
            for (int c = 0; c < d; ++c)
                blk[(size_t)i * d + c] = orc_bf16_value(K[(size_t)src * d + c]) - kbar[c];
        }
        quant4_block_rows(blk, rows, d, kcodes + (size_t)r0 * d, ksfc + (size_t)r0 * db, &kg[t]);
    }
    free(blk);
}

/* ------------------------------------------------------------------ */
/* V-Smooth Demean + per-channel E4M3 residual ([VCA] "V-Smooth…", item */
/* Demean) and the rho-repair list ([IP73] "Le compromis…")             */
/* ------------------------------------------------------------------ */
/* Blocks are the 128-token hardware blocks of the permuted sequence; the
 * tail block holds the remaining tokens only.
 *   mu_t   = bf16(fp32(sum_fp64(v) / count))           (0 when demean is off)
 *   r      = fp32(v - mu_t)
 *   s_c    = 2^e_c, the least power of two with amax_c(r) <= 448 * 2^e_c [R]
 *            (1 when every residual of the channel is zero)
 *   code   = E4M3(r * 2^-e_c)                           (exact scaling)
 *   err    = fp32(r - value(code) * s_c)
 *   e_p    = sum_c err^2, fmaf-accumulated in channel order from 0
 *   repair = the R = ceil(rho*N) tokens of largest e_p (ties: lowest position),
 *            listed in ascending position; delta = bf16(err) for each.     */
static void pow2_scale(float amax, float *scale, int *expo)
{
    int E;
    float f;
    if (amax == 0.0f) {          /* all residuals zero: codes are 0, any scale works; take 1 */
        *scale = 1.0f;
        *expo = 0;
        return;
    }
    f = frexpf(amax, &E);     /* amax = f * 2^E, f in [0.5, 1); 448 = 0.875 * 2^9 */
    *expo = (f > 0.875f) ? E - 8 : E - 9;
    *scale = ldexpf(1.0f, *expo);
}

int orc_repair_count(float rho, int N)
{
    double r = ceil((double)rho * (double)N);
    if (r < 0)
        r = 0;
    if (r > N)
        r = N;
    return (int)r;
}

void orc_quant_v_head(const uint16_t *V, const int32_t *perm, int N, int d, int demean, int R,
                      uint8_t *v8, float *vscale, uint16_t *vmean, float *errsum,
                      int32_t *rep_idx, uint16_t *rep_delta)
{
    int Nb = (N + TILE - 1) / TILE;
    float *res = (float *)malloc((size_t)N * d * sizeof(float));
    float *amax = (float *)calloc((size_t)d, sizeof(float));
    int *expo = (int *)calloc((size_t)d, sizeof(int));
    for (int t = 0; t < Nb; ++t) {
        int p0 = t * TILE, cntb = (N - p0 < TILE) ? N - p0 : TILE;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            uint16_t mu = 0;
            float muf;
            for (int i = 0; i < cntb; ++i)
                s += (double)orc_bf16_value(V[(size_t)perm[p0 + i] * d + c]);
            if (demean)
                mu = orc_bf16_round((float)(s / (double)cntb));
            vmean[(size_t)t * d + c] = mu;
            muf = orc_bf16_value(mu);
            for (int i = 0; i < cntb; ++i) {
                float r = orc_bf16_value(V[(size_t)perm[p0 + i] * d + c]) - muf;
                res[(size_t)(p0 + i) * d + c] = r;
                if (fabsf(r) > amax[c])
                    amax[c] = fabsf(r);
            }
        }
    }
    for (int c = 0; c < d; ++c)
        pow2_scale(amax[c], &vscale[c], &expo[c]);
    memset(v8, 0, (size_t)Nb * TILE * d);
    for (int p = 0; p < N; ++p) {
        float acc = 0.0f;
        for (int c = 0; c < d; ++c) {
            float r = res[(size_t)p * d + c];
            uint8_t code = orc_e4m3_encode(ldexpf(r, -expo[c]));
            float deq = (float)(orc_e4m3_value(code) * (double)vscale[c]);
            float err = r - deq;
            v8[(size_t)p * d + c] = code;
            res[(size_t)p * d + c] = err; /* keep err for delta */
            acc = fmaf(err, err, acc);
        }
        errsum[p] = acc;
    }
    /* top-R selection by repeated maximum (plain and slow, ties to lowest p) */
    if (R > 0) {
        char *taken = (char *)calloc((size_t)N, 1);
        int *pick = (int *)malloc((size_t)R * sizeof(int));
        for (int r = 0; r < R; ++r) {
            int best = -1;
            for (int p = 0; p < N; ++p)
                if (!taken[p] && (best < 0 || errsum[p] > errsum[best]))
                    best = p;
            taken[best] = 1;
            pick[r] = best;
        }
        int w = 0;
        for (int p = 0; p < N; ++p)
            if (taken[p])
                rep_idx[w++] = p;
        for (int r = 0; r < R; ++r)
            for (int c = 0; c < d; ++c)
                rep_delta[(size_t)r * d + c] = orc_bf16_round(res[(size_t)rep_idx[r] * d + c]);
        free(taken);
        free(pick);
    }
    free(res);
    free(amax);
    free(expo);
}

/* ------------------------------------------------------------------ */
/* The attention forward of one (b,h) for selected query rows          */
/* ------------------------------------------------------------------ */
/* Online softmax over KV tiles of 128 permuted positions ([VCA] "V-Smooth…",
 * item Restore, and "ExpCast-FP8…"):
 *   acc_ij  = exact dot product of the E4M3 codes of q_i and k_j, to binary32
 *   alpha_t = fp32(fp32(sq_i * sk_t) * kappa)
 *   m      <- max(m, max_j fp32(acc_ij * alpha_t));   F = 8*ceil(m/8)   [R]
 *   on a frame change the running numerator and row sum are rescaled by the
 *   exact power of two 2^((F_old - F)/8)
 *   b_ij    = ExpCast(acc_ij, alpha_t, C - F);   p_ij = value(b_ij)
 *   l_t     = sum_j p_ij                    (the row sum the softmax keeps)
 *   num    += sum_j p_ij * value(v8_j) * s + l_t * mu_t    (Restore)
 *   l      += l_t
 * after the last tile, repair adds, for each listed token j, p'_ij * delta_j
 * with p'_ij = value(ExpCast(acc_ij, alpha_t(j), C - F_final)); then
 * O_i = num / l. Padded key positions (>= N) are not part of any row.
 * Output: out[nrows*d] in double (before any output rounding), the row sum
 * l and the final frame F for each requested row. */
void orc_attn_vc_rows(const uint8_t *q8, const float *sq, const uint8_t *k8, const float *sk,
                      const uint8_t *v8, const float *vscale, const uint16_t *vmean,
                      const int32_t *rep_idx, const uint16_t *rep_delta, int R,
                      int N, int d, float kappa, int C, const int32_t *rows, int nrows,
                      double *out, double *out_l, float *out_F)
{
    int Nb = (N + TILE - 1) / TILE;
    double *kd = (double *)malloc((size_t)N * d * sizeof(double));
    double *vd = (double *)malloc((size_t)N * d * sizeof(double));
    double *mud = (double *)malloc((size_t)Nb * d * sizeof(double));
    for (int j = 0; j < N; ++j)
        for (int c = 0; c < d; ++c) {
            kd[(size_t)j * d + c] = orc_e4m3_value(k8[(size_t)j * d + c]);
            vd[(size_t)j * d + c] = orc_e4m3_value(v8[(size_t)j * d + c]) * (double)vscale[c];
        }
    for (int t = 0; t < Nb; ++t)
        for (int c = 0; c < d; ++c)
            mud[(size_t)t * d + c] = (double)orc_bf16_value(vmean[(size_t)t * d + c]);

#pragma omp parallel for schedule(dynamic, 1)
    for (int ir = 0; ir < nrows; ++ir) {
        int i = rows[ir];
        double qd[TILE * 2];
        double *num = (double *)calloc((size_t)d, sizeof(double));
        double *numt = (double *)malloc((size_t)d * sizeof(double));
        float *acc = (float *)malloc((size_t)TILE * sizeof(float));
        double l = 0.0;
        float m = -INFINITY, F = -INFINITY;
        float sqi = sq[i / TILE];
        for (int c = 0; c < d; ++c)
            qd[c] = orc_e4m3_value(q8[(size_t)i * d + c]);
        for (int t = 0; t < Nb; ++t) {
            int j0 = t * TILE, j1 = (j0 + TILE < N) ? j0 + TILE : N;
            float alpha = (sqi * sk[t]) * kappa;
            float Fnew, cfr;
            double lt = 0.0;
            for (int j = j0; j < j1; ++j) {
                double s = 0.0;
                for (int c = 0; c < d; ++c)
                    s += qd[c] * kd[(size_t)j * d + c];
                acc[j - j0] = (float)s;
                float u = acc[j - j0] * alpha;
                if (u > m)
                    m = u;
            }
            Fnew = 8.0f * ceilf(m * 0.125f);
            if (t > 0 && Fnew != F) {
                double sc = ldexp(1.0, (int)((F - Fnew) / 8.0f));
                for (int c = 0; c < d; ++c)
                    num[c] *= sc;
                l *= sc;
            }
            F = Fnew;
            cfr = (float)C - F;
            for (int c = 0; c < d; ++c)
                numt[c] = 0.0;
            for (int j = j0; j < j1; ++j) {
                double p = orc_e4m3_value((uint8_t)orc_expcast_byte(acc[j - j0], alpha, cfr));
                lt += p;
                for (int c = 0; c < d; ++c)
                    numt[c] += p * vd[(size_t)j * d + c];
            }
            for (int c = 0; c < d; ++c)
                num[c] += numt[c] + lt * mud[(size_t)t * d + c];
            l += lt;
        }
        for (int r = 0; r < R; ++r) {
            int j = rep_idx[r], t = j / TILE;
            float alpha = (sqi * sk[t]) * kappa;
            double s = 0.0;
            for (int c = 0; c < d; ++c)
                s += qd[c] * kd[(size_t)j * d + c];
            double p = orc_e4m3_value((uint8_t)orc_expcast_byte((float)s, alpha, (float)C - F));
            for (int c = 0; c < d; ++c)
                num[c] += p * (double)orc_bf16_value(rep_delta[(size_t)r * d + c]);
        }
        for (int c = 0; c < d; ++c)
            out[(size_t)ir * d + c] = num[c] / l;
        out_l[ir] = l;
        out_F[ir] = F;
        free(num);
        free(numt);
        free(acc);
    }
    free(kd);
    free(vd);
    free(mud);
}

/* Diagnostic (not a step of the method): the same online softmax and the same
 * probability bytes as orc_attn_vc_rows, but the numerator uses the exact bf16
 * values v_j (no quantization, no demean, no repair). The difference between
 * the method's output and this one is the value-term error alone, which is the
 * error V-Smooth and repair act on ([VCA] "Por que a atenção é o gargalo":
 * after Q/K smoothing the value term dominates the output error). */
void orc_attn_exactv_rows(const uint8_t *q8, const float *sq, const uint8_t *k8, const float *sk,
                          const uint16_t *V, const int32_t *perm, int N, int d, float kappa, int C,
                          const int32_t *rows, int nrows, double *out)
{
    int Nb = (N + TILE - 1) / TILE;
    double *kd = (double *)malloc((size_t)N * d * sizeof(double));
    double *vx = (double *)malloc((size_t)N * d * sizeof(double));
    for (int j = 0; j < N; ++j)
        for (int c = 0; c < d; ++c) {
            kd[(size_t)j * d + c] = orc_e4m3_value(k8[(size_t)j * d + c]);
            vx[(size_t)j * d + c] = (double)orc_bf16_value(V[(size_t)perm[j] * d + c]);
        }
#pragma omp parallel for schedule(dynamic, 1)
    for (int ir = 0; ir < nrows; ++ir) {
        int i = rows[ir];
        double qd[TILE * 2];
        double *num = (double *)calloc((size_t)d, sizeof(double));
        float *acc = (float *)malloc((size_t)TILE * sizeof(float));
        double l = 0.0;
        float m = -INFINITY, F = -INFINITY;
        float sqi = sq[i / TILE];
        for (int c = 0; c < d; ++c)
            qd[c] = orc_e4m3_value(q8[(size_t)i * d + c]);
        for (int t = 0; t < Nb; ++t) {
            int j0 = t * TILE, j1 = (j0 + TILE < N) ? j0 + TILE : N;
            float alpha = (sqi * sk[t]) * kappa;
            float Fnew;
            for (int j = j0; j < j1; ++j) {
                double s = 0.0;
                for (int c = 0; c < d; ++c)
                    s += qd[c] * kd[(size_t)j * d + c];
                acc[j - j0] = (float)s;
                float u = acc[j - j0] * alpha;
                if (u > m)
                    m = u;
            }
            Fnew = 8.0f * ceilf(m * 0.125f);
            if (t > 0 && Fnew != F) {
                double sc = ldexp(1.0, (int)((F - Fnew) / 8.0f));
                for (int c = 0; c < d; ++c)
                    num[c] *= sc;
                l *= sc;
            }
            F = Fnew;
            for (int j = j0; j < j1; ++j) {
                double p = orc_e4m3_value((uint8_t)orc_expcast_byte(acc[j - j0], alpha, (float)C - F));
                l += p;
                for (int c = 0; c < d; ++c)
                    num[c] += p * vx[(size_t)j * d + c];
            }
        }
        for (int c = 0; c < d; ++c)
            out[(size_t)ir * d + c] = num[c] / l;
        free(num);
        free(acc);
    }
    free(kd);
    free(vx);
}

/* ------------------------------------------------------------------ */
/* NVFP4-residual variant ([VCA] "V-Smooth…", item Demean: the residual  */
/* is quantized per channel in E4M3 for the 8-bit kernel or in NVFP4 for */
/* the 4-bit one; "ExpCast-FP8…": ExpCast is 8-bit only, so the 4-bit   */
/* kernel takes the probabilities from an exp2 softmax)                 */
/* ------------------------------------------------------------------ */
/* OCP FP4 E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit, no
 * infinities or NaN. Exponent field 0 is subnormal (m * 0.5); otherwise the
 * value is (1 + m/2) * 2^(e-1). The eight magnitudes are 0, 0.5, 1, 1.5, 2,
 * 3, 4, 6. The code sits in the low 4 bits. */
double orc_e2m1_value(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* binary32 -> E2M1, round to nearest, ties to even, saturating to +/-6.
 * The grid spacing is 0.5 below 2 (the subnormal 0.5 and the binade [1, 2)),
 * 1 in [2, 4) and 2 in [4, 8); a rounded value past 6 saturates. An even
 * grid index is an even mantissa bit in every binade, so ties to an even
 * index are ties to even. The sign is kept (a negative value that rounds to
 * zero gives code 8, negative zero). */
uint8_t orc_e2m1_encode(float x)
{
    uint8_t sign = signbit(x) ? 8 : 0;
    double a = fabs((double)x), q, val;
    if (isnan(x))
        return 7; /* NaN converts to +6 */
    q = (a < 2.0) ? 0.5 : (a < 4.0) ? 1.0 : 2.0;
    val = nearbyint(a / q) * q; /* a/q is exact; ties to even */
    if (val > 6.0)
        val = 6.0;
    for (int c = 0; c < 8; ++c)
        if (orc_e2m1_value((uint8_t)c) == val)
            return (uint8_t)(sign | c);
    return (uint8_t)(sign | 7); /* unreachable: val is on the grid */
}

/* NVFP4 global/ block scale of the probabilities [R]: p <= 1 in the frame of
 * its tile, so the global decode scale is 1/2688 (2688 = 6 * 448, the E2M1
 * maximum times the E4M3 maximum) and a block of 16 keys with maximum a gets
 * the E4M3 scale sf = E4M3(fp32(a * 448)). The element code of p is
 * E2M1(fp32(p * fp32(2688 / sf))), with every code 0 when sf is 0. The value
 * the tensor core multiplies is value(code) * sf = 2688 * (dequantized p).
 *   x_j = fmaf(acc_j, alpha/8, -F/8)      (the exponent, one rounding)
 *   p_j = binary32(2^x_j)
 * n <= 16 valid keys; codes[] gets n codes, *sfc the scale code. */
void orc_nvfp4_p_block(const float *x, int n, uint8_t *codes, uint8_t *sfc)
{
    float p[16], a = 0.0f, sfv, rcp;
    for (int j = 0; j < n; ++j) {
        p[j] = (float)exp2((double)x[j]);
        if (p[j] > a)
            a = p[j];
    }
    *sfc = orc_e4m3_encode(a * 448.0f);
    sfv = (float)orc_e4m3_value(*sfc);
    rcp = (sfv == 0.0f) ? 0.0f : 2688.0f / sfv;
    for (int j = 0; j < n; ++j)
        codes[j] = orc_e2m1_encode(p[j] * rcp);
}

/* V residual in NVFP4 [R]. Demean and residual as in orc_quant_v_head; then
 *   g_c   = 2^e_c, the least power of two with amax_c(r) <= 2688 * 2^e_c
 *           (1 when every residual of the channel is zero), the per-channel
 *           fp32 global scale
 *   block = 16 consecutive permuted positions of one channel (the K-major
 *           scale block of the PV product); positions >= N count as zero
 *   sf    = E4M3(fp32(fp32(b * 2^-e_c) / 6)), b = max |r| over the block
 *   code  = E2M1(fp32(fp32(r * 2^-e_c) * fp32(1 / sf)))
 *           (the reciprocal of the block scale rounded once, the multiplier
 *           form of the probability codes too; every code 0 when sf is 0)
 *   deq   = value(code) * sf * g_c          (exact in binary32)
 *   err   = fp32(r - deq); e_p, the repair list and delta as in the 8-bit path.
 * Outputs: codes[N][d] (one per byte, low 4 bits), sfc[ceil(N/16)][d],
 * vscale[d] = g_c, vmean[Nb][d], errsum[N], rep_idx[R], rep_delta[R][d]. */
void orc_quant_v4_head(const uint16_t *V, const int32_t *perm, int N, int d, int demean, int R,
                       uint8_t *codes, uint8_t *sfc, float *vscale, uint16_t *vmean, float *errsum,
                       int32_t *rep_idx, uint16_t *rep_delta)
{
    int Nb = (N + TILE - 1) / TILE, N16 = (N + 15) / 16;
    float *res = (float *)malloc((size_t)N * d * sizeof(float));
    float *amax = (float *)calloc((size_t)d, sizeof(float));
    int *expo = (int *)calloc((size_t)d, sizeof(int));
    for (int t = 0; t < Nb; ++t) {
        int p0 = t * TILE, cntb = (N - p0 < TILE) ? N - p0 : TILE;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            uint16_t mu = 0;
            float muf;
            for (int i = 0; i < cntb; ++i)
                s += (double)orc_bf16_value(V[(size_t)perm[p0 + i] * d + c]);
            if (demean)
                mu = orc_bf16_round((float)(s / (double)cntb));
            vmean[(size_t)t * d + c] = mu;
            muf = orc_bf16_value(mu);
            for (int i = 0; i < cntb; ++i) {
                float r = orc_bf16_value(V[(size_t)perm[p0 + i] * d + c]) - muf;
                res[(size_t)(p0 + i) * d + c] = r;
                if (fabsf(r) > amax[c])
                    amax[c] = fabsf(r);
            }
        }
    }
    for (int c = 0; c < d; ++c) {
        int E;
        float f;
        if (amax[c] == 0.0f) {
            expo[c] = 0;
        } else {
            f = frexpf(amax[c], &E); /* amax = f 2^E; 2688 = 0.65625 * 2^12 */
            expo[c] = (f > 0.65625f) ? E - 11 : E - 12;
        }
        vscale[c] = ldexpf(1.0f, expo[c]);
    }
    for (int jb = 0; jb < N16; ++jb) {
        int p0 = 16 * jb, n = (N - p0 < 16) ? N - p0 : 16;
        for (int c = 0; c < d; ++c) {
            float b = 0.0f, sfv, rcpv;
            uint8_t sc;
            for (int i = 0; i < n; ++i) {
                float a = fabsf(res[(size_t)(p0 + i) * d + c]);
                if (a > b)
                    b = a;
            }
            sc = orc_e4m3_encode(ldexpf(b, -expo[c]) / 6.0f);
            sfc[(size_t)jb * d + c] = sc;
            sfv = (float)orc_e4m3_value(sc);
            rcpv = (sfv == 0.0f) ? 0.0f : 1.0f / sfv;
            for (int i = 0; i < n; ++i) {
                float r = res[(size_t)(p0 + i) * d + c];
                uint8_t code = (sfv == 0.0f) ? 0 : orc_e2m1_encode(ldexpf(r, -expo[c]) * rcpv);
                codes[(size_t)(p0 + i) * d + c] = code;
            }
        }
    }
    for (int p = 0; p < N; ++p) {
        float acc = 0.0f;
        for (int c = 0; c < d; ++c) {
            float r = res[(size_t)p * d + c];
            float sfv = (float)orc_e4m3_value(sfc[(size_t)(p / 16) * d + c]);
            float deq = (float)(orc_e2m1_value(codes[(size_t)p * d + c]) * (double)sfv * (double)vscale[c]);
            float err = r - deq;
            res[(size_t)p * d + c] = err;
            acc = fmaf(err, err, acc);
        }
        errsum[p] = acc;
    }
    if (R > 0) {
        char *taken = (char *)calloc((size_t)N, 1);
        for (int r = 0; r < R; ++r) {
            int best = -1;
            for (int p = 0; p < N; ++p)
                if (!taken[p] && (best < 0 || errsum[p] > errsum[best]))
                    best = p;
            taken[best] = 1;
        }
        int w = 0;
        for (int p = 0; p < N; ++p)
            if (taken[p])
                rep_idx[w++] = p;
        for (int r = 0; r < R; ++r)
            for (int c = 0; c < d; ++c)
                rep_delta[(size_t)r * d + c] = orc_bf16_round(res[(size_t)rep_idx[r] * d + c]);
        free(taken);
    }
    free(res);
    free(amax);
    free(expo);
}

/* The 4-bit attention forward of one (b,h) for selected query rows. The
 * scores, the running max and the frames are those of orc_attn_vc_rows; the
 * probabilities are 2^((u - F)/8) quantized per 16 keys by orc_nvfp4_p_block,
 * and the values are the NVFP4 residuals:
 *   x_ij   = fmaf(acc_ij, alpha_t/8, -F/8),  p_ij = binary32(2^x_ij)
 *   P_ij   = value(code_ij) * sf_i,kb          (2688 x the dequantized p)
 *   l_t    = sum_j P_ij
 *   num   += sum_j P_ij * value(vcode_j) * vsf_j * g + l_t * mu_t
 * after the last tile, repair adds P'_ij * delta_j for each listed token j,
 * with P'_ij = bf16(fp32(2^x'_ij * 2688)) and x'_ij the exponent against the
 * final frame [R]; then O_i = num / l. Inputs: vcodes[N][d], vsfc[ceil(N/16)][d]
 * and vscale[d] = g_c as orc_quant_v4_head writes them. */
static void attn_vc4_core(const double *qd_all, const float *sq, const double *kd, const float *sk,
                          const double *vd, const double *mud, const int32_t *rep_idx, const uint16_t *rep_delta,
                          int R, int N, int d, float kappa, const int32_t *rows, int nrows, double *out,
                          double *out_l, float *out_F)
{
    int Nb = (N + TILE - 1) / TILE;
#pragma omp parallel for schedule(dynamic, 1)
    for (int ir = 0; ir < nrows; ++ir) {
        int i = rows[ir];
        const double *qd = qd_all + (size_t)i * d;
        double *num = (double *)calloc((size_t)d, sizeof(double));
        float *acc = (float *)malloc((size_t)TILE * sizeof(float));
        double l = 0.0;
        float m = -INFINITY, F = -INFINITY;
        float sqi = sq[i / TILE];
        for (int t = 0; t < Nb; ++t) {
            int j0 = t * TILE, j1 = (j0 + TILE < N) ? j0 + TILE : N;
            float alpha = (sqi * sk[t]) * kappa;
            float Fnew;
            double lt = 0.0;
            for (int j = j0; j < j1; ++j) {
                double s = 0.0;
                for (int c = 0; c < d; ++c)
                    s += qd[c] * kd[(size_t)j * d + c];
                acc[j - j0] = (float)s;
                float u = acc[j - j0] * alpha;
                if (u > m)
                    m = u;
            }
            Fnew = 8.0f * ceilf(m * 0.125f);
            if (t > 0 && Fnew != F) {
                double sc = ldexp(1.0, (int)((F - Fnew) / 8.0f));
                for (int c = 0; c < d; ++c)
                    num[c] *= sc;
                l *= sc;
            }
            F = Fnew;
            for (int b0 = j0; b0 < j1; b0 += 16) {
                int n = (j1 - b0 < 16) ? j1 - b0 : 16;
                float x[16];
                uint8_t codes[16], sfc;
                double sfv;
                for (int e = 0; e < n; ++e)
                    x[e] = fmaf(acc[b0 + e - j0], alpha * 0.125f, -F * 0.125f);
                orc_nvfp4_p_block(x, n, codes, &sfc);
                sfv = orc_e4m3_value(sfc);
                for (int e = 0; e < n; ++e) {
                    double P = orc_e2m1_value(codes[e]) * sfv;
                    lt += P;
                    for (int c = 0; c < d; ++c)
                        num[c] += P * vd[(size_t)(b0 + e) * d + c];
                }
            }
            for (int c = 0; c < d; ++c)
                num[c] += lt * mud[(size_t)t * d + c];
            l += lt;
        }
        for (int r = 0; r < R; ++r) {
            int j = rep_idx[r], t = j / TILE;
            float alpha = (sqi * sk[t]) * kappa;
            double s = 0.0;
            for (int c = 0; c < d; ++c)
                s += qd[c] * kd[(size_t)j * d + c];
            float x = fmaf((float)s, alpha * 0.125f, -F * 0.125f);
            float P = orc_bf16_value(orc_bf16_round((float)exp2((double)x) * 2688.0f));
            for (int c = 0; c < d; ++c)
                num[c] += (double)P * (double)orc_bf16_value(rep_delta[(size_t)r * d + c]);
        }
        for (int c = 0; c < d; ++c)
            out[(size_t)ir * d + c] = num[c] / l;
        out_l[ir] = l;
        out_F[ir] = F;
        free(num);
        free(acc);
    }
}

/* The NVFP4 values and block means in the units the core multiplies. */
static void v4_dequant(const uint8_t *vcodes, const uint8_t *vsfc, const float *vscale, const uint16_t *vmean,
                       int N, int d, double *vd, double *mud)
{
    int Nb = (N + TILE - 1) / TILE;
    for (int j = 0; j < N; ++j)
        for (int c = 0; c < d; ++c)
            vd[(size_t)j * d + c] = orc_e2m1_value(vcodes[(size_t)j * d + c]) *
                                    orc_e4m3_value(vsfc[(size_t)(j / 16) * d + c]) * (double)vscale[c];
    for (int t = 0; t < Nb; ++t)
        for (int c = 0; c < d; ++c)
            mud[(size_t)t * d + c] = (double)orc_bf16_value(vmean[(size_t)t * d + c]);
}

void orc_attn_vc4_rows(const uint8_t *q8, const float *sq, const uint8_t *k8, const float *sk,
                       const uint8_t *vcodes, const uint8_t *vsfc, const float *vscale, const uint16_t *vmean,
                       const int32_t *rep_idx, const uint16_t *rep_delta, int R,
                       int N, int d, float kappa, const int32_t *rows, int nrows,
                       double *out, double *out_l, float *out_F)
{
    int Nb = (N + TILE - 1) / TILE;
    double *qd = (double *)malloc((size_t)N * d * sizeof(double));
    double *kd = (double *)malloc((size_t)N * d * sizeof(double));
    double *vd = (double *)malloc((size_t)N * d * sizeof(double));
    double *mud = (double *)malloc((size_t)Nb * d * sizeof(double));
    for (size_t i = 0; i < (size_t)N * d; ++i) {
        qd[i] = orc_e4m3_value(q8[i]);
        kd[i] = orc_e4m3_value(k8[i]);
    }
    v4_dequant(vcodes, vsfc, vscale, vmean, N, d, vd, mud);
    attn_vc4_core(qd, sq, kd, sk, vd, mud, rep_idx, rep_delta, R, N, d, kappa, rows, nrows, out, out_l, out_F);
    free(qd);
    free(kd);
    free(vd);
    free(mud);
}

/* Full 4-bit path [R]: Q and K' in NVFP4 as well (orc_quant_qk4_head); the
 * score is sum_c value(qcode) sfq value(kcode) sfk (exact, rounded once to
 * binary32, as the tensor core accumulates it) and its scale the product of
 * the two blocks' power-of-two global scales; the rest is orc_attn_vc4_rows. */
void orc_attn_vc44_rows(const uint8_t *qcodes, const uint8_t *qsfc, const float *qg, const uint8_t *kcodes,
                        const uint8_t *ksfc, const float *kg, const uint8_t *vcodes, const uint8_t *vsfc,
                        const float *vscale, const uint16_t *vmean, const int32_t *rep_idx,
                        const uint16_t *rep_delta, int R, int N, int d, float kappa, const int32_t *rows,
                        int nrows, double *out, double *out_l, float *out_F)
{
    int Nb = (N + TILE - 1) / TILE, db = d / 16;
    double *qd = (double *)malloc((size_t)N * d * sizeof(double));
    double *kd = (double *)malloc((size_t)N * d * sizeof(double));
    double *vd = (double *)malloc((size_t)N * d * sizeof(double));
    double *mud = (double *)malloc((size_t)Nb * d * sizeof(double));
    for (int j = 0; j < N; ++j)
        for (int c = 0; c < d; ++c) {
            qd[(size_t)j * d + c] = orc_e2m1_value(qcodes[(size_t)j * d + c]) *
                                    orc_e4m3_value(qsfc[(size_t)j * db + c / 16]);
            kd[(size_t)j * d + c] = orc_e2m1_value(kcodes[(size_t)j * d + c]) *
                                    orc_e4m3_value(ksfc[(size_t)j * db + c / 16]);
        }
    v4_dequant(vcodes, vsfc, vscale, vmean, N, d, vd, mud);
    attn_vc4_core(qd, qg, kd, kg, vd, mud, rep_idx, rep_delta, R, N, d, kappa, rows, nrows, out, out_l, out_F);
    free(qd);
    free(kd);
    free(vd);
    free(mud);
}

void orc_e2m1_encode_n(const float *x, long long n, uint8_t *out)
{
    for (long long i = 0; i < n; ++i)
        out[i] = orc_e2m1_encode(x[i]);
}

/* Thread control for the bench's CPU baseline (OpenMP over query rows). */
void orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int orc_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Vectorized helpers for the tests (plain loops over the scalar functions). */
void orc_e4m3_encode_n(const float *x, long long n, uint8_t *out)
{
    for (long long i = 0; i < n; ++i)
        out[i] = orc_e4m3_encode(x[i]);
}

void orc_e4m3_value_n(const uint8_t *c, long long n, double *out)
{
    for (long long i = 0; i < n; ++i)
        out[i] = orc_e4m3_value(c[i]);
}

void orc_bf16_round_n(const float *x, long long n, uint16_t *out)
{
    for (long long i = 0; i < n; ++i)
        out[i] = orc_bf16_round(x[i]);
}

void orc_expcast_n(const float *acc, const float *alpha, const float *c, long long n, uint8_t *out)
{
    for (long long i = 0; i < n; ++i)
        out[i] = (uint8_t)orc_expcast_byte(acc[i], alpha[i], c[i]);
}

/* ExpCast of a run of consecutive binary32 bit patterns, for the exhaustive
 * sweeps of the tests: acc = the float whose bit pattern is first + i (with
 * the sign bit set when `negative`), one alpha and c for the whole run. A
 * plain loop over orc_expcast_byte, split over threads. */
void orc_expcast_bits_n(uint32_t first, long long n, int negative, float alpha, float c, uint8_t *out)
{
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (long long i = 0; i < n; ++i) {
        uint32_t b = first + (uint32_t)i;
        float a;
        if (negative)
            b |= 0x80000000u;
        memcpy(&a, &b, 4);
        out[i] = (uint8_t)orc_expcast_byte(a, alpha, c);
    }
}
