/*
 * oracle.c -- plain fp64 CPU oracle for the fused group-wise
 * quantize/dequantize matrix multiply ("matmul_q").
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header or table with the CUDA
 * library.
 *
 * What it computes (each step cited to the page that defines it):
 *
 *   BITCRUSH BC-06, "Under the hood": matmul_q is group-wise affine
 *   round-to-nearest quantization computed inline as weights are read,
 *   with a separate per-group scale/zero precompute.
 *   BITCRUSH BC-06, "The machine" table, NAIVE / SMART row: one scale per
 *   output channel (naive) or one per 64-weight group (smart).
 *   Enargeia, "Four bits per weight" section: int4 weights in blocks of 64
 *   along the reduction axis, each block with its own scale and zero point.
 *
 * The pages fix neither the RTN arithmetic nor the rounding; the adopted
 * convention (scale = (max-min)/(2^b-1), zero = round(-min/scale),
 * q = clamp(round(w/scale)+zero, 0, 2^b-1), w' = (q-zero)*scale) is
 * written out step by step below, with these readings:
 *   - round() is round-half-to-even of the EXACT real quotient;
 *   - scale is IEEE fp32: fl32(fl32(max-min) / L);
 *   - fp16 storage (packed int4 mode) rounds that fp32 scale to fp16 (RNE,
 *     floored at the smallest fp16 subnormal), then derives zero and codes
 *     from the stored fp16 scale and stores zero as fp16 (RNE);
 *   - a constant group (max == min == c) takes scale |c| (1 when c == 0),
 *     so that it dequantizes to c exactly.
 *
 * Every function is a straight loop over the definition, in double.
 * Quotients are computed as fp64 divisions and then rounded: for an fp16
 * numerator and an fp32/fp16 denominator the fp64 quotient never crosses a
 * rounding boundary of the exact quotient (the distance from the exact
 * quotient to any half-integer it is not equal to exceeds 2^-41 times the
 * fp64 rounding error), so nearbyint() of it equals round-half-even of the
 * exact real quotient.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (see build.py).
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>

/* ---- IEEE binary16 <-> double (exact decode, RNE encode) ---------------- */

double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal or zero */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25);     /* 1.m * 2^(e-15) */
    return sign ? -v : v;
}

/* Round a double to the nearest binary16 value, ties to even. */
uint16_t oracle_double_to_half(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v)) return 0x7e00;
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);              /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;             /* a in [2^E, 2^(E+1)) */
    if (E < -14) E = -14;       /* subnormal range: quantum 2^-24 */
    double quantum = ldexp(1.0, E - 10);
    double n = nearbyint(a / quantum);   /* exact scaling, RNE */
    double r = n * quantum;
    if (r > 65504.0) return sign | 0x7c00;
    if (r < ldexp(1.0, -14)) {
        return sign | (uint16_t)(r / ldexp(1.0, -24));
    }
    frexp(r, &e2);
    E = e2 - 1;
    uint16_t mant = (uint16_t)((r / ldexp(1.0, E) - 1.0) * 1024.0);
    return sign | (uint16_t)((E + 15) << 10) | mant;
}

/* Round a double to the nearest binary32 value (C conversion, RNE). */
static double to_f32(double v) { return (double)(float)v; }

/* ---- step 1-4: per-group scale and zero -------------------------------- */
/*
 * W      : [N][K] binary16 bit patterns, row-major (PyTorch Linear layout)
 * group  : 64 (per-group, "SMART") or K (per-output-channel, "NAIVE")
 * f16    : 0 -> fp32 storage of scale and zero (runtime re-quantization)
 *          1 -> fp16 storage (pre-packed int4 mode)
 * s, z   : [N][K/group] stored values, returned as doubles (exact)
 */
void oracle_group_params(const uint16_t *W, int64_t N, int64_t K, int bits,
                         int64_t group, int f16, double *s, double *z)
{
    const double L = (double)((1 << bits) - 1);
    const int64_t G = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < G; ++j) {
            /* 1. group range, exact */
            double lo = INFINITY, hi = -INFINITY;
            for (int64_t k = j * group; k < (j + 1) * group; ++k) {
                double w = oracle_half_to_double(W[n * K + k]);
                if (w < lo) lo = w;
                if (w > hi) hi = w;
            }
            /* 2. scale in fp32: fl32(fl32(hi - lo) / L).  The fp64
             *    difference of two fp16 values is exact; the fp64 quotient
             *    rounded once to fp32 is the correctly rounded fp32 quotient
             *    (53 >= 2*24 + 2). */
            double sc;
            if (hi == lo) {
                sc = (lo == 0.0) ? 1.0 : fabs(lo);   /* constant group */
            } else {
                double d = to_f32(hi - lo);
                sc = to_f32(d / L);
            }
            /* 3. fp16 storage: round the fp32 scale to fp16, floored at the
             *    smallest positive fp16 subnormal. */
            if (f16) {
                sc = oracle_half_to_double(oracle_double_to_half(sc));
                if (sc < ldexp(1.0, -24)) sc = ldexp(1.0, -24);
            }
            /* 4. zero = round-half-even(-lo / scale), exact quotient */
            double zz = nearbyint(-lo / sc) + 0.0;   /* +0.0: no -0 */
            if (f16)
                zz = oracle_half_to_double(oracle_double_to_half(zz)) + 0.0;
            s[n * G + j] = sc;
            z[n * G + j] = zz;
        }
    }
}

/* ---- step 1 alone: the group range ---------------------------------------- */
/*
 * The bit-width-independent precompute (BITCRUSH BC-06, "Under the hood":
 * after the precompute a change of bit width costs one argument): the
 * exact (min, max) of every group, from which steps 2-4 give the scale and
 * zero of any bit width.
 * lo, hi : [N][K/group] doubles (exact fp16 values)
 */
void oracle_group_range(const uint16_t *W, int64_t N, int64_t K, int64_t group,
                        double *lo_out, double *hi_out)
{
    const int64_t G = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < G; ++j) {
            double lo = INFINITY, hi = -INFINITY;
            for (int64_t k = j * group; k < (j + 1) * group; ++k) {
                double w = oracle_half_to_double(W[n * K + k]);
                if (w < lo) lo = w;
                if (w > hi) hi = w;
            }
            lo_out[n * G + j] = lo;
            hi_out[n * G + j] = hi;
        }
    }
}

/* ---- step 5: codes ------------------------------------------------------ */
/* q = clamp(round-half-even(w / s) + z, 0, L) with the exact quotient. */
void oracle_codes(const uint16_t *W, const double *s, const double *z,
                  int64_t N, int64_t K, int bits, int64_t group, uint8_t *q)
{
    const double L = (double)((1 << bits) - 1);
    const int64_t G = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            double sc = s[n * G + k / group];
            double zz = z[n * G + k / group];
            double w = oracle_half_to_double(W[n * K + k]);
            double c = nearbyint(w / sc) + zz;
            if (c < 0.0) c = 0.0;
            if (c > L) c = L;
            q[n * K + k] = (uint8_t)c;
        }
    }
}

/* ---- step 6: dequantization w' = (q - z) * s (exact in fp64) ------------ */
void oracle_dequant(const uint8_t *q, const double *s, const double *z,
                    int64_t N, int64_t K, int64_t group, double *wq)
{
    const int64_t G = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            wq[n * K + k] = ((double)q[n * K + k] - z[n * G + k / group]) *
                            s[n * G + k / group];
}

/* ---- step 9: int4 packing ----------------------------------------------- */
/* byte[n][k/2] = q[n][k] | q[n][k+1] << 4 for even k (low nibble = even k). */
void oracle_pack_int4(const uint8_t *q, int64_t N, int64_t K, uint8_t *packed)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; k += 2)
            packed[n * (K / 2) + k / 2] =
                (uint8_t)((q[n * K + k] & 0xf) | ((q[n * K + k + 1] & 0xf) << 4));
}

/* ---- step 9, any width: packed codes of `bits` bits ------------------------ */
/*
 * Other packed widths (Enargeia, "Honestly": an int8 tied embedding;
 * BITCRUSH BC-06, "The machine", BRAIN SIZE: 2-bit weights): each row is one
 * little-endian bit string in which code k occupies bits [bits*k,
 * bits*k + bits).  For bits = 4 this is the int4 layout above (low nibble =
 * even k); for bits = 8 one byte per code; a 64-group takes 8*bits bytes.
 * packed : [N][K*bits/8]
 */
void oracle_pack_codes(const uint8_t *q, int64_t N, int64_t K, int bits, uint8_t *packed)
{
    const int64_t rb = K * bits / 8;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < rb; ++b) packed[n * rb + b] = 0;
        for (int64_t k = 0; k < K; ++k) {
            for (int i = 0; i < bits; ++i) {
                const int64_t bit = k * bits + i;               /* position in the row */
                if ((q[n * K + k] >> i) & 1)
                    packed[n * rb + bit / 8] |= (uint8_t)(1u << (bit % 8));
            }
        }
    }
}

/* ---- step 8: y = x . w'^T in fp64, plus the tolerance scale A ----------- */
/*
 * x  : [M][K] doubles (the fp32 or bf16 input values, exactly)
 * wq : [N][K] dequantized weights
 * y  : [M][N] sum_k x[m][k] * wq[n][k]
 * a  : [M][N] sum_k |x[m][k] * wq[n][k]|   (may be NULL)
 */
void oracle_matmul(const double *x, const double *wq, int64_t M, int64_t N,
                   int64_t K, double *y, double *a)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, acc_abs = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = x[m * K + k] * wq[n * K + k];
                acc += p;
                acc_abs += fabs(p);
            }
            y[m * N + n] = acc;
            if (a) a[m * N + n] = acc_abs;
        }
    }
}

/* Passthrough (bits = 16): w' = w, decoded exactly. */
void oracle_half_rows_to_double(const uint16_t *W, int64_t count, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i)
        out[i] = oracle_half_to_double(W[i]);
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
