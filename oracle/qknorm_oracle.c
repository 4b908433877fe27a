/*
 * Oracle for layerwise QK-RMSNorm — TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, double-precision CPU restatement of what the normalization
 * computes.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load this library; the product path never does.  It shares
 * no source, header, table or helper with the CUDA library.
 *
 * Source of every formula: "SwiftQK: Fast and Communication-Efficient Tensor
 * Parallelism for Query-Key Normalization" (arXiv 2608.09160, HTML version).
 *   - Background, the RMS-Norm definition (Equation 1; its typeset form was
 *     lost from the page, the reading used is y = x / sqrt(mean(x^2) + eps) * gamma,
 *     eps inside the square root, mean over the full width H).
 *   - Phase A: each hidden-dimension shard contributes only its squared sum;
 *     the partial sums are added to give the global squared sum, with the same
 *     normalization semantics as the unsharded form.
 *   - Phase B: the weight multiplication x*gamma does not depend on the
 *     reduction; the global RMS factor is applied to it afterwards.
 *   - Evaluation, Fig. 2(b): the accuracy reference is RMSNorm in FP64 over the
 *     full vector.  This file is that reference.
 *
 * Element types:
 *   dtype 0 = IEEE binary32;
 *   dtype 1 = bfloat16 (1 sign bit, 8 exponent bits with bias 127, 7 stored
 *             mantissa bits);
 *   dtype 2 = IEEE binary16 (1 sign, 5 exponent bits with bias 15, 10 stored
 *             mantissa bits);
 *   dtype 3 = FP8 E4M3 in its "fn" form (1 sign, 4 exponent bits with bias 7,
 *             3 stored mantissa bits; no infinities; exponent 15 with mantissa
 *             7 is NaN, so the largest finite value is 1.75 * 2^8 = 448).
 *             With dtype 3 the gamma vector is bfloat16 (an E4M3 gamma near 1
 *             would be spaced 0.125 apart); x and y are E4M3.
 * Inputs are decoded exactly into double; all arithmetic is in double in
 * plain left-to-right order; an output of a narrow type is produced by one
 * correctly rounded (round-to-nearest, ties-to-even) conversion from the
 * double result.  E4M3 outputs beyond the finite range saturate to +-448
 * (the reading taken for an 8-bit format without infinities).
 *
 * Build: gcc -O2 -std=c11 -fno-fast-math -ffp-contract=off -shared -fPIC -lm
 * (FMA contraction is disabled so every product and sum is rounded on its own.)
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1
#define ORACLE_F16 2
#define ORACLE_E4M3 3

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

int oracle_version(void) { return 1; }

/* bfloat16 bit pattern -> exact double, from the field definition. */
double oracle_bf16_decode(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int expo = (b >> 7) & 0xFF;
    int mant = b & 0x7F;
    double v;
    if (expo == 0xFF) {
        v = mant ? NAN : INFINITY;
    } else if (expo == 0) {
        /* subnormal: 0.mant * 2^-126 = mant * 2^-133 */
        v = ldexp((double)mant, -133);
    } else {
        /* normal: 1.mant * 2^(expo-127) = (128 + mant) * 2^(expo-134) */
        v = ldexp((double)(128 + mant), expo - 134);
    }
    return sign ? -v : v;
}

/*
 * double -> bfloat16 with round-to-nearest, ties-to-even, applied once to the
 * exact double value (no intermediate rounding through binary32).
 * A finite non-zero |y| in [2^E, 2^(E+1)) has representable neighbours spaced
 * 2^(E-7) apart (8 significant bits); below 2^-126 the spacing is fixed at
 * 2^-133 (subnormals).  The value is scaled by a power of two (exact), rounded
 * to an integer with nearbyint (the default rounding mode is to-nearest-even),
 * and scaled back.
 */
uint16_t oracle_bf16_encode_rne(double y)
{
    if (isnan(y))
        return 0x7FC0;
    uint16_t sign = signbit(y) ? 0x8000 : 0;
    double a = fabs(y);
    if (isinf(a))
        return sign | 0x7F80;
    if (a == 0.0)
        return sign;
    int e;
    (void)frexp(a, &e);          /* a = m * 2^e, m in [0.5, 1): floor(log2 a) = e - 1 */
    int q = (e - 1) - 7;         /* exponent of the spacing between neighbours */
    if (q < -133)
        q = -133;
    double n = nearbyint(ldexp(a, -q));
    double r = ldexp(n, q);      /* exact: n has at most 9 significant bits */
    if (r >= 0x1p128)
        return sign | 0x7F80;    /* rounds past the largest finite value */
    /* Encode r, which is exactly representable: find its fields. */
    if (r < 0x1p-126) {
        /* subnormal: r = mant * 2^-133 with mant in [1, 127] */
        long mant = lrint(ldexp(r, 133));
        return sign | (uint16_t)mant;
    }
    int er;
    double m = frexp(r, &er);    /* r = m * 2^er, m in [0.5, 1) */
    int expo = er - 1 + 127;     /* biased exponent of 1.f * 2^(er-1) */
    long frac = lrint(ldexp(m, 8)) - 128;   /* 1.f = 2m, 7 stored bits */
    return sign | (uint16_t)((expo << 7) | (int)frac);
}

/* binary16 bit pattern -> exact double, from the field definition. */
double oracle_f16_decode(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int expo = (b >> 10) & 0x1F;
    int mant = b & 0x3FF;
    double v;
    if (expo == 0x1F)
        v = mant ? NAN : INFINITY;
    else if (expo == 0)
        v = ldexp((double)mant, -24);                 /* 0.mant * 2^-14 */
    else
        v = ldexp((double)(1024 + mant), expo - 25);  /* 1.mant * 2^(expo-15) */
    return sign ? -v : v;
}

/* E4M3 ("fn") bit pattern -> exact double, from the field definition. */
double oracle_e4m3_decode(uint8_t b)
{
    int sign = (b >> 7) & 1;
    int expo = (b >> 3) & 0xF;
    int mant = b & 0x7;
    double v;
    if (expo == 0xF && mant == 0x7)
        v = NAN;
    else if (expo == 0)
        v = ldexp((double)mant, -9);                  /* 0.mant * 2^-6 */
    else
        v = ldexp((double)(8 + mant), expo - 10);     /* 1.mant * 2^(expo-7) */
    return sign ? -v : v;
}

/*
 * |y| rounded to nearest, ties to even, onto the grid of a binary format with
 * `sig` significant bits whose smallest normal exponent is `emin`: spacing
 * 2^(E - sig + 1) for |y| in [2^E, 2^(E+1)), never finer than the subnormal
 * spacing 2^(emin - sig + 1).  Exact scaling by powers of two, nearbyint in
 * the default (to-nearest-even) mode.  a > 0 and finite.
 */
static double round_to_grid(double a, int sig, int emin)
{
    int e;
    (void)frexp(a, &e);               /* a = m * 2^e, m in [0.5, 1) */
    int q = (e - 1) - (sig - 1);
    if (q < emin - (sig - 1))
        q = emin - (sig - 1);
    return ldexp(nearbyint(ldexp(a, -q)), q);
}

/* double -> binary16, one rounding (RNE); beyond the largest finite value
 * (65504) the rounded result is infinity. */
uint16_t oracle_f16_encode_rne(double y)
{
    if (isnan(y))
        return 0x7E00;
    uint16_t sign = signbit(y) ? 0x8000 : 0;
    double a = fabs(y);
    if (isinf(a))
        return sign | 0x7C00;
    if (a == 0.0)
        return sign;
    double r = round_to_grid(a, 11, -14);
    if (r >= 65536.0)
        return sign | 0x7C00;
    if (r < 0x1p-14)
        return sign | (uint16_t)lrint(ldexp(r, 24));  /* subnormal */
    int er;
    double m = frexp(r, &er);
    return sign | (uint16_t)(((er - 1 + 15) << 10) | (int)(lrint(ldexp(m, 11)) - 1024));
}

/* double -> E4M3 ("fn"), one rounding (RNE), saturating to +-448; NaN -> 0x7F. */
uint8_t oracle_e4m3_encode_rne_sat(double y)
{
    if (isnan(y))
        return 0x7F;
    uint8_t sign = signbit(y) ? 0x80 : 0;
    double a = fabs(y);
    if (a == 0.0)
        return sign;
    double r = isinf(a) ? 448.0 : round_to_grid(a, 4, -6);
    if (r > 448.0)
        r = 448.0;
    if (r < 0x1p-6)
        return sign | (uint8_t)lrint(ldexp(r, 9));    /* subnormal */
    int er;
    double m = frexp(r, &er);
    return sign | (uint8_t)(((er - 1 + 7) << 3) | (int)(lrint(ldexp(m, 4)) - 8));
}

static int elem_size(int dtype) { return dtype == ORACLE_F32 ? 4 : (dtype == ORACLE_E4M3 ? 1 : 2); }

/* gamma is stored in the element type, except with E4M3 data, where it is bfloat16 */
static int gamma_dtype(int dtype) { return dtype == ORACLE_E4M3 ? ORACLE_BF16 : dtype; }

static double load_elem(const void *base, int dtype, int64_t idx)
{
    const char *p = (const char *)base + idx * elem_size(dtype);
    if (dtype == ORACLE_F32) {
        float f;
        memcpy(&f, p, 4);
        return (double)f;
    }
    if (dtype == ORACLE_E4M3)
        return oracle_e4m3_decode(*(const uint8_t *)p);
    uint16_t b;
    memcpy(&b, p, 2);
    return dtype == ORACLE_F16 ? oracle_f16_decode(b) : oracle_bf16_decode(b);
}

static void store_elem(void *base, int dtype, int64_t idx, double v)
{
    char *p = (char *)base + idx * elem_size(dtype);
    if (dtype == ORACLE_F32) {
        float f = (float)v;      /* C conversion: round to nearest, ties to even */
        memcpy(p, &f, 4);
        return;
    }
    if (dtype == ORACLE_E4M3) {
        *(uint8_t *)p = oracle_e4m3_encode_rne_sat(v);
        return;
    }
    uint16_t b = dtype == ORACLE_F16 ? oracle_f16_encode_rne(v) : oracle_bf16_encode_rne(v);
    memcpy(p, &b, 2);
}

static int bad_dtype(int dtype) { return dtype < ORACLE_F32 || dtype > ORACLE_E4M3; }

/*
 * RMS-Norm of T rows of width H (Background, Equation 1):
 *   S_t = sum_j x_tj^2,  r_t = 1 / sqrt(S_t / H + eps),  y_tj = x_tj * gamma_j * r_t.
 * Row t of x starts at element t * x_stride.  Outputs (each optional, NULL to skip):
 *   y_out   : [T][y_stride] elements of the input's type, rounded once;
 *   y_exact : [T][H] doubles before rounding;
 *   sumsq   : [T] doubles, the squared sums S_t.
 */
int oracle_rmsnorm_rows(const void *x, int64_t x_stride, int64_t T, int32_t H,
                        const void *gamma, double eps, int dtype,
                        void *y_out, int64_t y_stride, double *y_exact, double *sumsq)
{
    if (T < 0 || H <= 0 || x_stride < H || bad_dtype(dtype) || !(eps >= 0.0))
        return ORACLE_BAD_ARG;
    if (T > 0 && (!x || !gamma))
        return ORACLE_BAD_ARG;
    if (y_out && y_stride < H)
        return ORACLE_BAD_ARG;
    for (int64_t t = 0; t < T; ++t) {
        double S = 0.0;
        for (int32_t j = 0; j < H; ++j) {
            double v = load_elem(x, dtype, t * x_stride + j);
            S += v * v;
        }
        double r = 1.0 / sqrt(S / (double)H + eps);
        for (int32_t j = 0; j < H; ++j) {
            double v = load_elem(x, dtype, t * x_stride + j);
            double g = load_elem(gamma, gamma_dtype(dtype), j);
            double yv = (v * g) * r;
            if (y_exact)
                y_exact[t * (int64_t)H + j] = yv;
            if (y_out)
                store_elem(y_out, dtype, t * y_stride + j, yv);
        }
        if (sumsq)
            sumsq[t] = S;
    }
    return ORACLE_OK;
}

/*
 * Layerwise QK-Norm of one batch: the full projected Q row and the full
 * projected K row of every token are normalized independently, each with its
 * own gamma (Background).  Outputs are contiguous [T][Hq] and [T][Hk].
 */
int oracle_qknorm_layerwise(const void *q, int64_t q_stride, const void *gamma_q, int32_t Hq,
                            const void *k, int64_t k_stride, const void *gamma_k, int32_t Hk,
                            int64_t T, double eps, int dtype, void *q_out, void *k_out)
{
    int st = oracle_rmsnorm_rows(q, q_stride, T, Hq, gamma_q, eps, dtype, q_out, Hq, NULL, NULL);
    if (st != ORACLE_OK)
        return st;
    return oracle_rmsnorm_rows(k, k_stride, T, Hk, gamma_k, eps, dtype, k_out, Hk, NULL, NULL);
}

/*
 * Headwise QK-Norm (Background: "headwise QK-Norm computes an independent
 * factor for each attention head"): token t's row of one tensor holds
 * n_heads heads of head_dim elements each, head h at columns
 * [h * head_dim, (h + 1) * head_dim).  Each head is RMS-normalized on its own
 * over head_dim elements, with one gamma of length head_dim shared by every
 * head (the reading taken: the pages do not say how gamma is laid out):
 *   S_th = sum_{j < head_dim} x_t,h*hd+j ^2,  r_th = 1 / sqrt(S_th / head_dim + eps),
 *   y_t,h*hd+j = (x_t,h*hd+j * gamma_j) * r_th.
 * Output is contiguous [T][n_heads * head_dim].
 */
int oracle_rmsnorm_heads(const void *x, int64_t x_stride, int64_t T, int32_t n_heads, int32_t head_dim,
                         const void *gamma, double eps, int dtype, void *y_out, double *y_exact)
{
    if (T < 0 || n_heads <= 0 || head_dim <= 0 || x_stride < (int64_t)n_heads * head_dim || bad_dtype(dtype) ||
        !(eps >= 0.0))
        return ORACLE_BAD_ARG;
    if (T > 0 && (!x || !gamma))
        return ORACLE_BAD_ARG;
    const int64_t W = (int64_t)n_heads * head_dim;
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t h = 0; h < n_heads; ++h) {
            const int64_t c0 = (int64_t)h * head_dim;
            double S = 0.0;
            for (int32_t j = 0; j < head_dim; ++j) {
                double v = load_elem(x, dtype, t * x_stride + c0 + j);
                S += v * v;
            }
            double r = 1.0 / sqrt(S / (double)head_dim + eps);
            for (int32_t j = 0; j < head_dim; ++j) {
                double v = load_elem(x, dtype, t * x_stride + c0 + j);
                double g = load_elem(gamma, gamma_dtype(dtype), j);
                double yv = (v * g) * r;
                if (y_exact)
                    y_exact[t * W + c0 + j] = yv;
                if (y_out)
                    store_elem(y_out, dtype, t * W + c0 + j, yv);
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Phase A, local step: the squared sum of each token's row restricted to one
 * hidden-dimension shard of width h_shard.  sumsq[t] = sum_{j < h_shard} x_tj^2.
 */
int oracle_partial_sumsq(const void *x, int64_t x_stride, int64_t T, int32_t h_shard,
                         int dtype, double *sumsq)
{
    if (T < 0 || h_shard <= 0 || x_stride < h_shard || bad_dtype(dtype))
        return ORACLE_BAD_ARG;
    if (T > 0 && (!x || !sumsq))
        return ORACLE_BAD_ARG;
    for (int64_t t = 0; t < T; ++t) {
        double S = 0.0;
        for (int32_t j = 0; j < h_shard; ++j) {
            double v = load_elem(x, dtype, t * x_stride + j);
            S += v * v;
        }
        sumsq[t] = S;
    }
    return ORACLE_OK;
}

/*
 * Phase A aggregation followed by Phase B on one shard: the P partial squared
 * sums of token t (sumsq_all[p * T + t], p = 0..P-1, added in that order) give
 * the global squared sum; the factor divides by the FULL width H_full; the
 * shard's elements are multiplied by their gamma slice and then by the factor.
 *   S_t = sum_p sumsq_all[p][t],  r_t = 1 / sqrt(S_t / H_full + eps),
 *   y_tj = (x_tj * gamma_j) * r_t  for j < h_shard.
 */
int oracle_combine_apply(const void *x, int64_t x_stride, int64_t T, int32_t h_shard,
                         const void *gamma_shard, const double *sumsq_all, int32_t P,
                         int32_t H_full, double eps, int dtype,
                         void *y_out, int64_t y_stride, double *y_exact)
{
    if (T < 0 || h_shard <= 0 || x_stride < h_shard || P < 1 || H_full < h_shard ||
        bad_dtype(dtype) || !(eps >= 0.0))
        return ORACLE_BAD_ARG;
    if (T > 0 && (!x || !gamma_shard || !sumsq_all))
        return ORACLE_BAD_ARG;
    if (y_out && y_stride < h_shard)
        return ORACLE_BAD_ARG;
    for (int64_t t = 0; t < T; ++t) {
        double S = 0.0;
        for (int32_t p = 0; p < P; ++p)
            S += sumsq_all[(int64_t)p * T + t];
        double r = 1.0 / sqrt(S / (double)H_full + eps);
        for (int32_t j = 0; j < h_shard; ++j) {
            double v = load_elem(x, dtype, t * x_stride + j);
            double g = load_elem(gamma_shard, gamma_dtype(dtype), j);
            double yv = (v * g) * r;
            if (y_exact)
                y_exact[t * (int64_t)h_shard + j] = yv;
            if (y_out)
                store_elem(y_out, dtype, t * y_stride + j, yv);
        }
    }
    return ORACLE_OK;
}

/*
 * The linear projection that produces the tensors QK-Norm normalizes
 * (Background: in a Pre-LN layer, linear projections of the hidden state give
 * Q, K and V; QK-Norm runs between the Q/K projections and attention).
 * W is stored one row per output column, [N][D] with row stride w_stride, so
 * for each requested token t = rows[i]:
 *   y_in = sum_{d < D} x_td * w_nd        (double, d from 0 to D-1 in order),
 * and y_out[i][n] is y_in rounded once to the element type (the projection's
 * output type).  y_exact (optional) receives the unrounded doubles, [n_rows][N].
 * Products of two bfloat16 or binary16 values are exact in double; the sum is
 * the only rounding before the final conversion.
 */
int oracle_project_rows(const void *x, int64_t x_stride, const int64_t *rows, int64_t n_rows, int64_t T,
                        int32_t D, const void *w, int64_t w_stride, int32_t N, int dtype,
                        void *y_out, double *y_exact)
{
    if (n_rows < 0 || T < 0 || D <= 0 || N <= 0 || x_stride < D || w_stride < D || bad_dtype(dtype))
        return ORACLE_BAD_ARG;
    if (n_rows > 0 && (!x || !w || !rows))
        return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < n_rows; ++i) {
        const int64_t t = rows[i];
        if (t < 0 || t >= T)
            return ORACLE_BAD_ARG;
        for (int32_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int32_t d = 0; d < D; ++d)
                acc += load_elem(x, dtype, t * x_stride + d) * load_elem(w, dtype, (int64_t)n * w_stride + d);
            if (y_exact)
                y_exact[i * (int64_t)N + n] = acc;
            if (y_out)
                store_elem(y_out, dtype, i * (int64_t)N + n, acc);
        }
    }
    return ORACLE_OK;
}
