/*
 * SharQ CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library. The CUDA path
 * never calls it, and it shares no code, header, table or helper with the
 * CUDA path.
 *
 * What it computes comes from the SharQ abstract ("SharQ: Bridging Activation
 * Sparsity and FP4 Quantization for LLM Inference", arXiv 2606.26587,
 * Abstract): LayerNorm; per row, an N:M mask chosen from the data that keeps
 * a sparse backbone S holding the large (outlier) values; FP4 quantization
 * of S; a dense residual R = X_ln - deq(Q(S)), measured from the quantized
 * backbone; FP4 quantization of R; and two FP4 GEMMs that use the same FP4
 * weight codes and whose outputs are added. The abstract leaves the arithmetic open; each
 * function below states the reading it implements.
 *
 * Formats: NVFP4 = E2M1 codes, one UE4M3 scale per 16 elements and one fp32
 * tensor scale (NVIDIA's NVFP4 description); MXFP4 = E2M1 codes and one E8M0
 * scale per 32 elements (OCP Microscaling Formats v1.0).
 *
 * Arithmetic: every float operation is one IEEE-754 binary32 (or binary64
 * where stated) operation rounded to nearest even. Build with
 * -ffp-contract=off so that no multiply-add is fused. Codecs are brute-force
 * nearest-value searches over the format's value table, the plainest
 * correct definition.
 *
 * Canonical layouts (row-major, one value per byte):
 *   codes   [rows][k]        E2M1 code, bit 3 = sign, bits 0-2 = magnitude
 *   scales  [rows][k / blk]  UE4M3 code (NVFP4) or E8M0 code (MXFP4)
 *   idx     [rows][k / m][n] kept positions inside each M-group, ascending
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef unsigned __int128 u128;
typedef __int128 i128;

#define FMT_NVFP4 0
#define FMT_MXFP4 1

/* Threads the row and output-element loops use: 1 in the plain build. */
int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* fp16 decode (IEEE-754 binary16), exact in binary64.                 */

double oracle_half_to_double(uint16_t h)
{
    int s = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f + 1024), e - 25);
    return s ? -v : v;
}

/* ------------------------------------------------------------------ */
/* Correctly rounded (nearest, ties to even) binary64 value of a       */
/* non-negative 128-bit integer, written as an integer routine.        */

static double u128_to_double_rn(u128 v)
{
    if (v == 0)
        return 0.0;
    int p = 127;
    while (!((v >> p) & 1))
        --p;
    if (p < 53)
        return (double)(uint64_t)v;
    int drop = p - 52; /* keep the top 53 bits */
    u128 q = v >> drop;
    u128 rem = v - (q << drop);
    u128 half = (u128)1 << (drop - 1);
    if (rem > half || (rem == half && (q & 1)))
        q += 1; /* q <= 2^53: still exact */
    return ldexp((double)(uint64_t)q, drop);
}

double oracle_u128_to_double(uint64_t hi, uint64_t lo)
{
    return u128_to_double_rn(((u128)hi << 64) | lo);
}

/* ------------------------------------------------------------------ */
/* LayerNorm statistics, exactly (reading: the abstract names "layer   */
/* normalization" inside the fused preparation operator; it does not   */
/* say how the statistics round, so they are defined from exact        */
/* integer sums, which makes them independent of summation order).     */
/*                                                                      */
/*   a_i  = x_i * 2^24                  integer, |a_i| < 2^40          */
/*   S1   = sum a_i,  S2 = sum a_i^2     exact                          */
/*   D    = K*S2 - S1^2                  exact, >= 0                    */
/*   mu   = RN32( RN64(S1) / (K*2^24) )                                 */
/*   var  = RN64(D) / (K^2 * 2^48)        (binary64 division)           */
/*   rstd = RN32( 1 / sqrt(var + eps) )   (binary64 sqrt and division)  */

void oracle_ln_stats(const uint16_t *x, int64_t rows, int64_t k, float eps,
                     float *mu, float *rstd)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t s1 = 0;
        u128 s2 = 0;
        for (int64_t i = 0; i < k; ++i) {
            int64_t a = (int64_t)ldexp(oracle_half_to_double(x[r * k + i]), 24);
            s1 += a;
            s2 += (u128)((i128)a * (i128)a);
        }
        i128 d = (i128)k * (i128)s2 - (i128)s1 * (i128)s1;
        double mean64 = (double)s1 / ((double)k * 16777216.0);
        double var64 = u128_to_double_rn((u128)d) /
                       ((double)k * (double)k * 281474976710656.0);
        mu[r] = (float)mean64;
        rstd[r] = (float)(1.0 / sqrt(var64 + (double)eps));
    }
}

/* RMSNorm statistics, exactly (reading: models that normalize by the    */
/* root mean square, without centring, use this form of the preparation */
/* operator's normalization; same exact sums as above):                 */
/*                                                                      */
/*   S2   = sum a_i^2                     exact                          */
/*   ms   = RN64(S2) / (K * 2^48)          (binary64 division)           */
/*   rstd = RN32( 1 / sqrt(ms + eps) )    (binary64 sqrt and division)  */
/*   mu   = 0, so the apply step below gives RN32(RN32(x * rstd) * g).   */

void oracle_rms_stats(const uint16_t *x, int64_t rows, int64_t k, float eps,
                      float *mu, float *rstd)
{
    for (int64_t r = 0; r < rows; ++r) {
        u128 s2 = 0;
        for (int64_t i = 0; i < k; ++i) {
            int64_t a = (int64_t)ldexp(oracle_half_to_double(x[r * k + i]), 24);
            s2 += (u128)((i128)a * (i128)a);
        }
        double ms64 = u128_to_double_rn(s2) / ((double)k * 281474976710656.0);
        mu[r] = 0.0f;
        rstd[r] = (float)(1.0 / sqrt(ms64 + (double)eps));
    }
}

/* LayerNorm apply, left to right, each step rounded to binary32:       */
/*   X_ln = RN32( RN32( RN32(x - mu) * rstd ) * gamma ) + beta           */
/* gamma == NULL skips the multiply, beta == NULL skips the add.        */
void oracle_ln_apply(const uint16_t *x, int64_t rows, int64_t k,
                     const uint16_t *gamma, const uint16_t *beta,
                     const float *mu, const float *rstd, float *x_ln)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < k; ++i) {
            float t = (float)oracle_half_to_double(x[r * k + i]) - mu[r];
            t = t * rstd[r];
            if (gamma)
                t = t * (float)oracle_half_to_double(gamma[i]);
            if (beta)
                t = t + (float)oracle_half_to_double(beta[i]);
            x_ln[r * k + i] = t;
        }
}

/* ------------------------------------------------------------------ */
/* Codecs.                                                              */

static const double E2M1_GRID[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* E2M1 value of a code (bit 3 = sign). */
double oracle_e2m1_value(int code)
{
    double v = E2M1_GRID[code & 7];
    return (code & 8) ? -v : v;
}

/* E2M1 code of y: nearest magnitude on the grid, equal distances go to the
 * even code, |y| beyond 6 gives 6 (saturating); the sign bit is y's sign, so
 * a small negative y gives -0 (code 8). */
int oracle_e2m1_encode(float y)
{
    double a = fabs((double)y);
    int best = 0;
    double bd = a;
    for (int c = 1; c < 8; ++c) {
        double dd = fabs(a - E2M1_GRID[c]);
        if (dd < bd || (dd == bd && (c & 1) == 0)) {
            best = c;
            bd = dd;
        }
    }
    return best | (signbit(y) ? 8 : 0);
}

/* UE4M3 value: e = code>>3 (bias 7), m = code&7; e == 0 is subnormal.
 * Code 127 is NaN in E4M3 and is never produced. */
double oracle_ue4m3_value(int code)
{
    int e = (code >> 3) & 15, m = code & 7;
    return e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
}

/* UE4M3 code of u >= 0: nearest finite value (0 .. 448), equal distances go
 * to the even code; values above 448 give 448 (saturating). */
int oracle_ue4m3_encode(float u)
{
    double a = (double)u;
    int best = 0;
    double bd = fabs(a);
    for (int c = 1; c < 127; ++c) {
        double dd = fabs(a - oracle_ue4m3_value(c));
        if (dd < bd || (dd == bd && (c & 1) == 0)) {
            best = c;
            bd = dd;
        }
    }
    return best;
}

/* E8M0 block exponent of OCP MX v1.0: for a block amax a > 0,
 * e = floor(log2 a) - emax(E2M1), emax(E2M1) = 2, clamped to [-127, 127]. */
int oracle_mx_exponent(float a)
{
    int ex;
    frexp((double)a, &ex); /* a = f * 2^ex, f in [0.5, 1): floor(log2 a) = ex-1 */
    int e = ex - 1 - 2;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return e;
}

/* ------------------------------------------------------------------ */
/* Block quantization of one row of values (used for S, R and W).       */
/*                                                                      */
/* NVFP4, blocks of 16:  a = max|v|;  u = a / RN32(6 * s_t);             */
/*   sb = UE4M3(u);  d = RN32(value(sb) * s_t);                          */
/*   code = d == 0 ? +0 : E2M1(RN32(v / d)).                             */
/* MXFP4, blocks of 32:  a == 0 gives scale code 0 and +0 codes;         */
/*   else e = mx_exponent(a), scale code e + 127, d = 2^e,               */
/*   code = E2M1(RN32(v / d)).                                           */
/* The per-value division (not a multiply by a reciprocal) is the reading */
/* of "quantizes it to FP4"; d doubles as the dequantization step.        */

/* blk: the block length; the format's own (16 or 32) everywhere except in
 * the pair-wise sparse mode below, whose backbone and weight blocks are
 * twice as long. */
static void quantize_row_blk(const float *v, int64_t k, int fmt, int blk, float s_t,
                             uint8_t *codes, uint8_t *scales)
{
    for (int64_t b = 0; b < k / blk; ++b) {
        const float *vb = v + b * blk;
        float a = 0.0f;
        for (int i = 0; i < blk; ++i)
            if (fabsf(vb[i]) > a)
                a = fabsf(vb[i]);
        float d;
        if (fmt == FMT_NVFP4) {
            float six_st = 6.0f * s_t;
            float u = a / six_st;
            int sb = oracle_ue4m3_encode(u);
            scales[b] = (uint8_t)sb;
            d = (float)oracle_ue4m3_value(sb) * s_t;
        } else {
            if (a == 0.0f) {
                scales[b] = 0;
                d = 0.0f;
            } else {
                int e = oracle_mx_exponent(a);
                scales[b] = (uint8_t)(e + 127);
                d = (float)ldexp(1.0, e);
            }
        }
        for (int i = 0; i < blk; ++i)
            codes[b * blk + i] = d == 0.0f ? 0 : (uint8_t)oracle_e2m1_encode(vb[i] / d);
    }
}

static void quantize_row(const float *v, int64_t k, int fmt, float s_t,
                         uint8_t *codes, uint8_t *scales)
{
    quantize_row_blk(v, k, fmt, fmt == FMT_NVFP4 ? 16 : 32, s_t, codes, scales);
}

/* Dequantized value of one code with step d (RN32 product). */
static float deq(int code, float d)
{
    return (float)oracle_e2m1_value(code) * d;
}

/* Step d of a block from its scale code. */
static float block_step(int fmt, int scale_code, float s_t)
{
    if (fmt == FMT_NVFP4)
        return (float)oracle_ue4m3_value(scale_code) * s_t;
    return (float)ldexp(1.0, scale_code - 127);
}

void oracle_quantize(const float *v, int64_t rows, int64_t k, int fmt, float s_t,
                     uint8_t *codes, uint8_t *scales)
{
    int blk = fmt == FMT_NVFP4 ? 16 : 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        quantize_row(v + r * k, k, fmt, s_t, codes + r * k, scales + r * (k / blk));
}

/* ------------------------------------------------------------------ */
/* Tensor scale (reading: NVFP4 carries one fp32 scale per tensor; the    */
/* abstract does not say how it is chosen, so it is one dynamic scale per  */
/* activation tensor from amax over the whole tensor:                      */
/* s_t = RN32(amax / 2688), 2688 = 448 * 6; s_t = 1 if amax == 0; MXFP4    */
/* has no tensor scale, s_t = 1).                                          */

float oracle_tensor_scale(const float *v, int64_t count, int fmt)
{
    if (fmt != FMT_NVFP4)
        return 1.0f;
    float a = 0.0f;
    for (int64_t i = 0; i < count; ++i)
        if (fabsf(v[i]) > a)
            a = fabsf(v[i]);
    return a == 0.0f ? 1.0f : a / 2688.0f;
}

/* ------------------------------------------------------------------ */
/* N:M mask: in every row, in every aligned group of m consecutive       */
/* values along K, keep the n largest |X_ln|; equal magnitudes go to the  */
/* lower index (so -0 and +0 tie). Exactly n survivors per group.         */
/* Writes the kept positions ascending, and a 0/1 keep map.               */

void oracle_mask(const float *x_ln, int64_t rows, int64_t k, int n, int m,
                 uint8_t *idx, uint8_t *keep)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < k / m; ++g) {
            const float *v = x_ln + r * k + g * m;
            uint8_t taken[16] = {0};
            for (int j = 0; j < n; ++j) { /* pick the j-th largest */
                int best = -1;
                for (int i = 0; i < m; ++i)
                    if (!taken[i] && (best < 0 || fabsf(v[i]) > fabsf(v[best])))
                        best = i;
                taken[best] = 1;
            }
            int w = 0;
            for (int i = 0; i < m; ++i) {
                if (taken[i])
                    idx[(r * (k / m) + g) * n + w++] = (uint8_t)i;
                if (keep)
                    keep[r * k + g * m + i] = taken[i];
            }
        }
}

/* ------------------------------------------------------------------ */
/* The preparation operator, step by step in the abstract's order:       */
/* LayerNorm -> N:M mask -> Q(S) -> R = X_ln - deq(Q(S)) -> Q(R).         */
/* S is X_ln on survivors and +0 elsewhere; deq(Q(S)) is 0 off the mask;  */
/* R = RN32(X_ln - deqS); Q(R) uses the same tensor scale as Q(S).        */
/* All arrays are required (rows*k floats / bytes as named).               */
/* s_t_in: NULL computes the tensor scale from these rows; otherwise the   */
/* given value is used, so that a sample of rows of a larger tensor can be */
/* prepared with that tensor's scale (the per-row steps do not depend on   */
/* other rows).                                                            */

/* norm: 0 = LayerNorm (oracle_ln_stats), 1 = RMSNorm (oracle_rms_stats,  */
/* no beta). The steps after the normalization are the same.               */
void oracle_prepare_norm(const uint16_t *x, int64_t rows, int64_t k,
                         const uint16_t *gamma, const uint16_t *beta, float eps,
                         int n, int m, int fmt, int norm,
                         float *mu, float *rstd, float *x_ln, float *s, float *deq_s, float *r,
                         uint8_t *idx, uint8_t *keep,
                         uint8_t *s_codes, uint8_t *s_scales,
                         uint8_t *r_codes, uint8_t *r_scales, float *s_t_out, const float *s_t_in)
{
    int blk = fmt == FMT_NVFP4 ? 16 : 32;
    if (norm)
        oracle_rms_stats(x, rows, k, eps, mu, rstd);
    else
        oracle_ln_stats(x, rows, k, eps, mu, rstd);
    oracle_ln_apply(x, rows, k, gamma, beta, mu, rstd, x_ln);
    float s_t = s_t_in ? *s_t_in : oracle_tensor_scale(x_ln, rows * k, fmt);
    *s_t_out = s_t;
    oracle_mask(x_ln, rows, k, n, m, idx, keep);
    for (int64_t i = 0; i < rows * k; ++i)
        s[i] = keep[i] ? x_ln[i] : 0.0f;
    oracle_quantize(s, rows, k, fmt, s_t, s_codes, s_scales);
    for (int64_t row = 0; row < rows; ++row)
        for (int64_t i = 0; i < k; ++i) {
            int64_t e = row * k + i;
            float d = block_step(fmt, s_scales[row * (k / blk) + i / blk], s_t);
            deq_s[e] = keep[e] ? deq(s_codes[e], d) : 0.0f;
            r[e] = x_ln[e] - deq_s[e];
        }
    oracle_quantize(r, rows, k, fmt, s_t, r_codes, r_scales);
}

void oracle_prepare(const uint16_t *x, int64_t rows, int64_t k,
                    const uint16_t *gamma, const uint16_t *beta, float eps,
                    int n, int m, int fmt,
                    float *mu, float *rstd, float *x_ln, float *s, float *deq_s, float *r,
                    uint8_t *idx, uint8_t *keep,
                    uint8_t *s_codes, uint8_t *s_scales,
                    uint8_t *r_codes, uint8_t *r_scales, float *s_t_out, const float *s_t_in)
{
    oracle_prepare_norm(x, rows, k, gamma, beta, eps, n, m, fmt, 0, mu, rstd, x_ln, s, deq_s, r, idx, keep,
                        s_codes, s_scales, r_codes, r_scales, s_t_out, s_t_in);
}

/* Weight quantization: the same block quantizer along K on every row of  */
/* W [n_out][k], with s_tW = RN32(amax(W) / 2688) (NVFP4) or 1 (MXFP4).   */
/* One code payload serves both GEMM paths.                               */
void oracle_quantize_weight(const uint16_t *w, int64_t n_out, int64_t k, int fmt,
                            float *w_f32, uint8_t *codes, uint8_t *scales, float *s_tw)
{
    for (int64_t i = 0; i < n_out * k; ++i)
        w_f32[i] = (float)oracle_half_to_double(w[i]);
    *s_tw = oracle_tensor_scale(w_f32, n_out * k, fmt);
    oracle_quantize(w_f32, n_out, k, fmt, *s_tw, codes, scales);
}

/* Dequantized value of element (row, i) in the factored form the GEMM uses:
 * value(code) * value(scale), without the tensor scale. Exact in binary64. */
static double block_value_blk(int fmt, int blk, const uint8_t *codes, const uint8_t *scales,
                              int64_t k, int64_t row, int64_t i)
{
    int sc = scales[row * (k / blk) + i / blk];
    double sv = fmt == FMT_NVFP4 ? oracle_ue4m3_value(sc) : ldexp(1.0, sc - 127);
    return oracle_e2m1_value(codes[row * k + i]) * sv;
}

static double block_value(int fmt, const uint8_t *codes, const uint8_t *scales,
                          int64_t k, int64_t row, int64_t i)
{
    return block_value_blk(fmt, fmt == FMT_NVFP4 ? 16 : 32, codes, scales, k, row, i);
}

/* Dual-path linear: the backbone GEMM on Q(S) and the residual GEMM on    */
/* Q(R) against the same Q(W), summed (SharQ, Abstract: a sparse GEMM for  */
/* the backbone, a dense one for the residual):                             */
/*   out[i][j] = s_t * s_tW * sum_k (aS[i][k] + aR[i][k]) * w[j][k]         */
/* with a, w the block-scaled code values, in binary64 (every product is    */
/* exact; only the sum rounds). bound[i][j] is the same sum over absolute   */
/* values, the scale of the acceptance tolerance. Either may be NULL.       */
void oracle_linear(const uint8_t *s_codes, const uint8_t *s_scales,
                   const uint8_t *r_codes, const uint8_t *r_scales, float s_t,
                   const uint8_t *w_codes, const uint8_t *w_scales, float s_tw,
                   int64_t rows, int64_t n_out, int64_t k, int fmt,
                   double *out, double *bound)
{
    double ts = (double)s_t * (double)s_tw;
    /* Output elements are independent: built with OpenMP (the all-cores
     * baseline build), they are split across threads; each is still the
     * same sequential sum, so the results are identical. */
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t j = 0; j < n_out; ++j) {
            double acc = 0.0, mag = 0.0;
            for (int64_t q = 0; q < k; ++q) {
                double a_s = block_value(fmt, s_codes, s_scales, k, i, q);
                double a_r = block_value(fmt, r_codes, r_scales, k, i, q);
                double w = block_value(fmt, w_codes, w_scales, k, j, q);
                acc += a_s * w + a_r * w;
                mag += fabs(a_s) * fabs(w) + fabs(a_r) * fabs(w);
            }
            if (out)
                out[i * n_out + j] = ts * acc;
            if (bound)
                bound[i * n_out + j] = ts * mag;
        }
}

/* ------------------------------------------------------------------ */
/* Pair-wise 4:8 sparse-backbone mode.                                  */
/*                                                                      */
/* The abstract's backbone GEMM is "sparse". The block-scaled FP4        */
/* tensor-core instructions with structured sparsity accept one pattern:  */
/* in every aligned group of 8 values along K, two of the four adjacent   */
/* pairs (2j, 2j+1) are kept, and the hardware then applies one scale     */
/* per 32 logical values along K (NVFP4) or per 64 (MXFP4), on both       */
/* operands. Reading for this opt-in mode:                                */
/*   mask: in every aligned group of 8, the two pairs with the largest    */
/*         pair magnitude max(|x_2j|, |x_2j+1|) are kept, equal pair      */
/*         magnitudes going to the lower pair; exactly 4 survivors;       */
/*   Q(S): blocks of 32 values along K (NVFP4; 64 for MXFP4), i.e. the    */
/*         16 (32) kept values of the block, with the rules above;       */
/*   R = X_ln - deq(Q(S)) and Q(R) exactly as in the default mode;       */
/*   W:    one code payload quantized with blocks of 32 (64): the         */
/*         backbone path reads one scale per 32 (64) values, the residual */
/*         path the same values once per 16 (32) (its scale view repeats  */
/*         each one), so deq(W) is the same on both paths.                */

/* Kept positions (ascending, 4 per group of 8) and the 0/1 keep map. */
void oracle_mask_pairs48(const float *x_ln, int64_t rows, int64_t k, uint8_t *idx, uint8_t *keep)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < k / 8; ++g) {
            const float *v = x_ln + r * k + g * 8;
            float key[4];
            for (int j = 0; j < 4; ++j)
                key[j] = fabsf(v[2 * j]) > fabsf(v[2 * j + 1]) ? fabsf(v[2 * j]) : fabsf(v[2 * j + 1]);
            uint8_t taken[4] = {0, 0, 0, 0};
            for (int t = 0; t < 2; ++t) { /* pick the t-th largest pair */
                int best = -1;
                for (int j = 0; j < 4; ++j)
                    if (!taken[j] && (best < 0 || key[j] > key[best]))
                        best = j;
                taken[best] = 1;
            }
            int w = 0;
            for (int j = 0; j < 4; ++j) {
                if (taken[j]) {
                    idx[(r * (k / 8) + g) * 4 + w++] = (uint8_t)(2 * j);
                    idx[(r * (k / 8) + g) * 4 + w++] = (uint8_t)(2 * j + 1);
                }
                if (keep) {
                    keep[r * k + g * 8 + 2 * j] = taken[j];
                    keep[r * k + g * 8 + 2 * j + 1] = taken[j];
                }
            }
        }
}

/* Block quantization with an explicit block length (canonical layout:
 * scales [rows][k / blk]). */
void oracle_quantize_blk(const float *v, int64_t rows, int64_t k, int fmt, int blk, float s_t,
                         uint8_t *codes, uint8_t *scales)
{
    for (int64_t r = 0; r < rows; ++r)
        quantize_row_blk(v + r * k, k, fmt, blk, s_t, codes + r * k, scales + r * (k / blk));
}

/* The preparation operator in the pair-wise mode, in the abstract's order.
 * Outputs as oracle_prepare_norm (s_scales: [rows][k / (2 blk)]). */
void oracle_prepare_sparse(const uint16_t *x, int64_t rows, int64_t k,
                           const uint16_t *gamma, const uint16_t *beta, float eps, int fmt, int norm,
                           float *mu, float *rstd, float *x_ln, float *s, float *deq_s, float *r,
                           uint8_t *idx, uint8_t *keep,
                           uint8_t *s_codes, uint8_t *s_scales,
                           uint8_t *r_codes, uint8_t *r_scales, float *s_t_out, const float *s_t_in)
{
    int blk = fmt == FMT_NVFP4 ? 16 : 32, sblk = 2 * blk;
    if (norm)
        oracle_rms_stats(x, rows, k, eps, mu, rstd);
    else
        oracle_ln_stats(x, rows, k, eps, mu, rstd);
    oracle_ln_apply(x, rows, k, gamma, beta, mu, rstd, x_ln);
    float s_t = s_t_in ? *s_t_in : oracle_tensor_scale(x_ln, rows * k, fmt);
    *s_t_out = s_t;
    oracle_mask_pairs48(x_ln, rows, k, idx, keep);
    for (int64_t i = 0; i < rows * k; ++i)
        s[i] = keep[i] ? x_ln[i] : 0.0f;
    oracle_quantize_blk(s, rows, k, fmt, sblk, s_t, s_codes, s_scales);
    for (int64_t row = 0; row < rows; ++row)
        for (int64_t i = 0; i < k; ++i) {
            int64_t e = row * k + i;
            float d = block_step(fmt, s_scales[row * (k / sblk) + i / sblk], s_t);
            deq_s[e] = keep[e] ? deq(s_codes[e], d) : 0.0f;
            r[e] = x_ln[e] - deq_s[e];
        }
    oracle_quantize(r, rows, k, fmt, s_t, r_codes, r_scales);
}

/* Weight quantization with an explicit block length (the pair-wise mode's
 * weights: 32 for NVFP4, 64 for MXFP4); s_tW as oracle_quantize_weight. */
void oracle_quantize_weight_blk(const uint16_t *w, int64_t n_out, int64_t k, int fmt, int blk,
                                float *w_f32, uint8_t *codes, uint8_t *scales, float *s_tw)
{
    for (int64_t i = 0; i < n_out * k; ++i)
        w_f32[i] = (float)oracle_half_to_double(w[i]);
    *s_tw = oracle_tensor_scale(w_f32, n_out * k, fmt);
    oracle_quantize_blk(w_f32, n_out, k, fmt, blk, *s_tw, codes, scales);
}

/* Dual-path linear with explicit block lengths of the backbone, residual
 * and weight scales (the formula of oracle_linear). */
void oracle_linear_blk(const uint8_t *s_codes, const uint8_t *s_scales, int blk_s,
                       const uint8_t *r_codes, const uint8_t *r_scales, int blk_r, float s_t,
                       const uint8_t *w_codes, const uint8_t *w_scales, int blk_w, float s_tw,
                       int64_t rows, int64_t n_out, int64_t k, int fmt,
                       double *out, double *bound)
{
    double ts = (double)s_t * (double)s_tw;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t j = 0; j < n_out; ++j) {
            double acc = 0.0, mag = 0.0;
            for (int64_t q = 0; q < k; ++q) {
                double a_s = block_value_blk(fmt, blk_s, s_codes, s_scales, k, i, q);
                double a_r = block_value_blk(fmt, blk_r, r_codes, r_scales, k, i, q);
                double w = block_value_blk(fmt, blk_w, w_codes, w_scales, k, j, q);
                acc += a_s * w + a_r * w;
                mag += fabs(a_s) * fabs(w) + fabs(a_r) * fabs(w);
            }
            if (out)
                out[i * n_out + j] = ts * acc;
            if (bound)
                bound[i * n_out + j] = ts * mag;
        }
}

/* ------------------------------------------------------------------ */
/* Residual add feeding the preparation operator (reading: in pre-norm  */
/* transformers the normalization's input is the residual stream after  */
/* the add x = h + d; the abstract's fused operator starts from x. The  */
/* add is IEEE binary16 addition: x = RN16(h + d), the exact sum         */
/* (exact in binary64) rounded to nearest even binary16, overflowing to  */
/* +-inf).                                                               */

/* Nearest binary16 (ties to even) of a binary64 value, as bits. */
uint16_t oracle_double_to_half_rn(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    /* a = q * 2^-24 in the subnormal range and below: the grid 2^-24 */
    int e;
    frexp(a, &e); /* a in [2^(e-1), 2^e) */
    int ulp_exp = e - 1 - 10; /* spacing of binary16 at this binade */
    if (ulp_exp < -24)
        ulp_exp = -24;
    double q = ldexp(a, -ulp_exp); /* a in units of the spacing */
    double f = floor(q);
    double rem = q - f;
    if (rem > 0.5 || (rem == 0.5 && fmod(f, 2.0) != 0.0))
        f += 1.0;
    double r = ldexp(f, ulp_exp);
    if (r > 65504.0)
        return sign | 0x7C00; /* overflow: infinity */
    /* encode r exactly */
    if (r < ldexp(1.0, -14))
        return sign | (uint16_t)ldexp(r, 24); /* subnormal (or the smallest normal reached by rounding) */
    frexp(r, &e);
    int be = e - 1 + 15;
    uint16_t mant = (uint16_t)(ldexp(r, -(e - 1)) * 1024.0 - 1024.0);
    return sign | (uint16_t)(be << 10) | mant;
}

void oracle_add_fp16(const uint16_t *h, const uint16_t *d, int64_t count, uint16_t *x)
{
    for (int64_t i = 0; i < count; ++i)
        x[i] = oracle_double_to_half_rn(oracle_half_to_double(h[i]) + oracle_half_to_double(d[i]));
}
