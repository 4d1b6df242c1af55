/*
 * expcast_pin.c - test helper: an independent check of ExpCast bytes over
 * runs of consecutive binary32 scores.
 *
 * ExpCast (page "VC-Attention acelera atenção em modelos de vídeo de IA em
 * até 3,58× sem retreinamento", section "ExpCast-FP8: eliminando o gargalo do
 * softmax") writes the E4M3 byte of a probability from its log-domain score
 * with one fused multiply-add: an E4M3 byte read as an integer is close to
 * 8*log2(v) + 56. Here the score x = acc*alpha + c (byte units) stands for the
 * probability t = 2^((x - 56)/8). This file does not compute ExpCast. It
 * computes t with the C library's exp2 and rounds it to the nearest E4M3
 * value (ties to even) from the format's definition, then checks the byte
 * given to it:
 *   - where x >= 7.5 (normal codes) the decoded byte is that nearest E4M3
 *     value or the next code up (the piecewise-linear map 1 + f lies above
 *     2^f), and the ratio decoded / t stays within the bounds the caller
 *     checks;
 *   - along the run the bytes never increase as the score decreases, and
 *     every place where the byte changes is reported, so that the caller can
 *     check those points with exact rational arithmetic.
 * A t within 2^-44 (relative) of a rounding midpoint is counted as ambiguous
 * instead of decided (double exp2 is accurate to about 2^-52).
 * Built by the test with gcc -O2 -fopenmp -ffp-contract=off.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

typedef struct {
    long long n_normal, n_equal, n_next, n_bad, n_ambiguous, n_nonmono, n_trans;
    double min_ratio, max_ratio;
} pin_stats;

/* E4M3 value of a byte (sign 1, exponent 4 with bias 7, mantissa 3;
 * exponent field 0 is subnormal m * 2^-9). Bytes passed here are <= 0x7E. */
static double e4m3_decode(uint8_t b)
{
    int e = (b >> 3) & 15, m = b & 7;
    return e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
}

/* Spacing of the E4M3 grid at a magnitude v in [0, 448). */
static double e4m3_step(double v)
{
    int e;
    if (v < 0x1p-6)
        return 0x1p-9;
    frexp(v, &e); /* v = f 2^e, f in [0.5, 1): floor(log2 v) = e - 1 */
    return ldexp(1.0, e - 4);
}

static float bits_to_float(uint32_t b)
{
    float f;
    memcpy(&f, &b, 4);
    return f;
}

/* Check bytes[i] = ExpCast(acc_i, alpha, c) for acc_i = the float with bit
 * pattern first + i (sign bit set when negative). prev_byte is the byte just
 * before this run (-1 for none). Transitions (bit pattern of the first input
 * with the new byte, byte before, byte after) are appended to the trans_*
 * arrays at position st->n_trans, at most trans_cap of them in all. */
void pin_expcast_run(const uint8_t *bytes, uint32_t first, long long n, int negative, double alpha, double c,
                     int prev_byte, pin_stats *st, long long *trans_idx, int *trans_from, int *trans_to,
                     long long trans_cap)
{
    long long n_normal = 0, n_equal = 0, n_next = 0, n_bad = 0, n_amb = 0;
    double mn = st->min_ratio, mx = st->max_ratio;
#pragma omp parallel for schedule(static) reduction(+ : n_normal, n_equal, n_next, n_bad, n_amb) \
    reduction(min : mn) reduction(max : mx)
    for (long long i = 0; i < n; ++i) {
        uint32_t b = first + (uint32_t)i;
        if (negative)
            b |= 0x80000000u;
        const double acc = (double)bits_to_float(b);
        const double x = acc * alpha + c; /* the product is exact in double */
        if (!(x >= 7.5))
            continue;
        n_normal++;
        const double t = exp2((x - 56.0) / 8.0);
        const double s = e4m3_step(t);
        const double q = t / s;
        const double fl = floor(q);
        if (fabs(q - (fl + 0.5)) < 0x1p-44 * q) {
            n_amb++;
            continue;
        }
        const double r = nearbyint(q); /* default rounding mode: ties to even */
        const double near = r * s;
        const double next = near + e4m3_step(near);
        const double dv = e4m3_decode(bytes[i]);
        if (dv == near)
            n_equal++;
        else if (dv == next)
            n_next++;
        else
            n_bad++;
        const double ratio = dv / t;
        if (ratio < mn)
            mn = ratio;
        if (ratio > mx)
            mx = ratio;
    }
    st->n_normal += n_normal;
    st->n_equal += n_equal;
    st->n_next += n_next;
    st->n_bad += n_bad;
    st->n_ambiguous += n_amb;
    st->min_ratio = mn;
    st->max_ratio = mx;
    /* monotonicity and transitions, in order */
    int prev = prev_byte;
    for (long long i = 0; i < n; ++i) {
        const int cur = bytes[i];
        if (prev >= 0 && cur != prev) {
            /* acc moves away from zero along the run: with alpha > 0 the
             * score decreases for negative acc and increases for positive */
            const int wrong = negative ? (cur > prev) : (cur < prev);
            if (wrong)
                st->n_nonmono++;
            if (st->n_trans < trans_cap) {
                trans_idx[st->n_trans] = (long long)first + i; /* bit pattern without the sign */
                trans_from[st->n_trans] = prev;
                trans_to[st->n_trans] = cur;
            }
            st->n_trans++;
        }
        prev = cur;
    }
}
