/*
 * CPU oracle for the NF4 + double-quantisation format (test infrastructure).
 *
 * This file is TEST INFRASTRUCTURE. Only the tests, the smoke check and the
 * CPU-baseline leg of the benchmark may load it. It shares no code, header,
 * table or constant generator with the CUDA library: the codebook is derived
 * here from its definition, independently of the library's own derivation.
 *
 * Source of the method: "QLoRA: put the large model in memory, then change it
 * with a small adapter" (wq-win.github.io/llm/074-qlora), section 2 (NF4
 * weight codes, quantisation constants, double quantisation; the 16384-weight
 * worked example) and section 3 (the procedure that quantises W first and the
 * first-level scales afterwards).
 *
 * Arithmetic conventions (the oracle fixes them; the CUDA path must agree):
 *   - every float operation is one IEEE-754 binary32 operation with
 *     round-to-nearest-even; the file is compiled with -ffp-contract=off so
 *     that no multiply-add is fused; denormals are kept;
 *   - bf16 rounding is round-to-nearest-even of the fp32 bit pattern;
 *   - int8 rounding uses rintf() in the default round-half-even mode.
 *
 * The OpenMP pragmas only split loops over independent blocks; every value is
 * computed by the same operations in the same order with or without them.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stddef.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_BLOCK1 64   /* weights per first-level absmax block (section 2) */
#define ORC_BLOCK2 256  /* first-level constants per second-level block (section 2) */

enum { ORC_OK = 0, ORC_NONFINITE = 1, ORC_BADARG = 2 };

/* ------------------------------------------------------------------------ */
/* Standard normal quantile by bisection on the complementary error function. */
/* Phi(x) = 0.5 * erfc(-x / sqrt 2). For p >= 0.5 we solve the upper tail      */
/* 0.5 * erfc(x / sqrt 2) = 1 - p (1 - p is exact for p in [0.5, 1]).          */
/* Bisection is slow but its correctness is plain to see.                      */
/* ------------------------------------------------------------------------ */
double orc_norm_quantile_upper(double p)
{
    if (!(p >= 0.5 && p < 1.0)) return NAN;
    const double q = 1.0 - p;
    double lo = 0.0, hi = 40.0;            /* 0.5*erfc(0) = 0.5 >= q > 0.5*erfc(40/sqrt2) */
    for (int it = 0; it < 2000; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;  /* interval can no longer shrink */
        double tail = 0.5 * erfc(mid / sqrt(2.0));
        if (tail > q) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* NF4 codebook (section 2: sixteen values taken from normal quantiles, finer
 * near zero, with an exact zero, normalised to [-1, 1] by the block absmax).
 * The pages do not print the values. We take the asymmetric construction of
 * the paper the page summarises (Dettmers et al. 2023): 8 positive quantiles,
 * 7 negative quantiles and zero, with end probability
 *   delta = 1 - (1/32 + 1/30) / 2,
 * positive probabilities 1/2 + j (delta - 1/2) / 8 (j = 1..8), negative
 * probabilities 1/2 + j (delta - 1/2) / 7 (j = 1..7, mirrored), every value
 * divided by the quantile at delta. Computed in double, rounded once to fp32.
 * Output in ascending order. */
void orc_codebook_f64(double out[16])
{
    const double delta = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
    const double zmax = orc_norm_quantile_upper(delta);
    /* negative half, most negative first: j = 7 .. 1 */
    for (int j = 7; j >= 1; --j) {
        double p = 0.5 + (delta - 0.5) * ((double)j / 7.0);
        out[7 - j] = -orc_norm_quantile_upper(p) / zmax;
    }
    out[7] = 0.0;
    for (int j = 1; j <= 8; ++j) {
        double p = 0.5 + (delta - 0.5) * ((double)j / 8.0);
        out[7 + j] = orc_norm_quantile_upper(p) / zmax;
    }
}

void orc_codebook(float Q[16])
{
    double d[16];
    orc_codebook_f64(d);
    for (int i = 0; i < 16; ++i) Q[i] = (float)d[i];
}

/* Decision thresholds between neighbouring codes: T[t] = fl(fl(Q[t]+Q[t+1]) * 0.5). */
void orc_midpoints(const float Q[16], float T[15])
{
    for (int t = 0; t < 15; ++t) {
        float s = Q[t] + Q[t + 1];
        T[t] = s * 0.5f;
    }
}

/* Nearest-code assignment by counting thresholds strictly below x.
 * A value exactly on a threshold goes to the lower code; -0.0 maps to the
 * zero code 7 because T[6] < 0 < T[7]. */
int orc_code_of(float x, const float T[15])
{
    int c = 0;
    for (int t = 0; t < 15; ++t) c += (x > T[t]) ? 1 : 0;
    return c;
}

/* Brute-force nearest code in double: argmin_k |x - Q[k]|, ties to the lower k.
 * Used only to check orc_code_of. */
int orc_code_bruteforce(float x, const float Q[16])
{
    int best = 0;
    double bd = fabs((double)x - (double)Q[0]);
    for (int k = 1; k < 16; ++k) {
        double d = fabs((double)x - (double)Q[k]);
        if (d < bd) { bd = d; best = k; }
    }
    return best;
}

/* Exhaustive check over every fp32 value in [-1, 1] (both signs of zero).
 * Returns the number of x where the threshold count and the brute-force
 * nearest code disagree and x is NOT exactly one of the thresholds; also
 * reports how many values were tested and how many disagreements fell on a
 * threshold. */
int64_t orc_sweep_codes(const float Q[16], int64_t *n_tested, int64_t *n_on_threshold)
{
    float T[15];
    orc_midpoints(Q, T);
    /* non-negative floats 0 .. 1.0f are bit patterns 0x00000000 .. 0x3f800000 */
    const uint32_t last = 0x3f800000u;
    int64_t bad = 0, tested = 0, onthr = 0;
    #pragma omp parallel for schedule(static) reduction(+:bad,tested,onthr)
    for (int64_t u = 0; u <= (int64_t)last; ++u) {
        for (int sign = 0; sign < 2; ++sign) {
            uint32_t bits = (uint32_t)u | (sign ? 0x80000000u : 0u);
            float x;
            memcpy(&x, &bits, 4);
            int a = orc_code_of(x, T);
            int b = orc_code_bruteforce(x, Q);
            tested += 1;
            if (a != b) {
                int on = 0;
                for (int t = 0; t < 15; ++t) if (x == T[t]) on = 1;
                if (on) onthr += 1; else bad += 1;
            }
        }
    }
    if (n_tested) *n_tested = tested;
    if (n_on_threshold) *n_on_threshold = onthr;
    return bad;
}

/* bf16 round-to-nearest-even of an fp32 value (NaN stays NaN). */
uint16_t orc_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

float orc_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ------------------------------------------------------------------------ */
/* Steps 1-4: blockwise absmax, normalisation, code search, nibble packing.   */
/* W is n fp32 values, flattened row-major from [rows, cols]; block b covers  */
/* elements 64b .. min(64b+64, n)-1. Outputs: c1[nb] (fp32 absmax) and       */
/* codes[ceil(n/2)]: byte k = (code[2k] << 4) | code[2k+1]; for odd n the     */
/* missing low nibble of the last byte is 7, the zero code.                   */
/* ------------------------------------------------------------------------ */
int orc_quantize_codes(const float *w, int64_t n, const float Q[16], float *c1, uint8_t *codes)
{
    if (n <= 0 || !w || !c1 || !codes) return ORC_BADARG;
    float T[15];
    orc_midpoints(Q, T);
    const int64_t nb = (n + ORC_BLOCK1 - 1) / ORC_BLOCK1;
    int nonfinite = 0;
    #pragma omp parallel for schedule(static) reduction(|:nonfinite)
    for (int64_t b = 0; b < nb; ++b) {
        const int64_t i0 = b * ORC_BLOCK1;
        const int64_t i1 = (i0 + ORC_BLOCK1 < n) ? i0 + ORC_BLOCK1 : n;
        float m = 0.0f;
        for (int64_t i = i0; i < i1; ++i) {
            if (!isfinite(w[i])) nonfinite = 1;
            float a = fabsf(w[i]);
            if (a > m) m = a;
        }
        c1[b] = m;
        /* element codes; blocks hold an even number of elements except the
         * very last block when n is odd, so each byte lies in one block */
        for (int64_t i = i0; i < i1; i += 2) {
            float x0 = (m == 0.0f) ? 0.0f : w[i] / m;
            int hi = orc_code_of(x0, T);
            int lo = 7;
            if (i + 1 < i1) {
                float x1 = (m == 0.0f) ? 0.0f : w[i + 1] / m;
                lo = orc_code_of(x1, T);
            }
            codes[i / 2] = (uint8_t)((hi << 4) | lo);
        }
    }
    return nonfinite ? ORC_NONFINITE : ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Step 5: the offset mu = mean of all first-level constants.                 */
/* Sum in fp64 by the pairwise tree over the constants in index order,        */
/* zero-padded to a power of two: level 0 holds the constants, each node of   */
/* level L+1 is the sum of nodes 2i and 2i+1 of level L. Adding a zero leaf   */
/* is exact, so the padding length does not change the result. Then          */
/* mu = (float)(S / nb).                                                      */
/* ------------------------------------------------------------------------ */
double orc_pairwise_sum_f64(const double *v, int64_t len, double *scratch)
{
    /* scratch holds at least len doubles; written level by level */
    if (len <= 0) return 0.0;
    for (int64_t i = 0; i < len; ++i) scratch[i] = v[i];
    int64_t cur = len;
    while (cur > 1) {
        int64_t next = (cur + 1) / 2;
        for (int64_t i = 0; i < next; ++i) {
            double a = scratch[2 * i];
            double b = (2 * i + 1 < cur) ? scratch[2 * i + 1] : 0.0;
            scratch[i] = a + b;
        }
        cur = next;
    }
    return scratch[0];
}

/* scratch: 2*nb doubles */
float orc_offset(const float *c1, int64_t nb, double *scratch)
{
    double *leaves = scratch;
    double *work = scratch + nb;
    for (int64_t b = 0; b < nb; ++b) leaves[b] = (double)c1[b];
    double S = orc_pairwise_sum_f64(leaves, nb, work);
    return (float)(S / (double)nb);
}

/* ------------------------------------------------------------------------ */
/* Step 6: double quantisation of the first-level constants (section 2:     */
/* 8-bit constants, one fp32 second-level constant per 256 constants, and   */
/* an offset). Reading: linear symmetric int8 about the offset.             */
/*   d_b  = fl(c1[b] - mu)                                                  */
/*   s2_j = max |d_b| over the group                                        */
/*   q8_b = 0 if s2_j == 0 else rint(fl(fl(d_b / s2_j) * 127))              */
/* ------------------------------------------------------------------------ */
void orc_double_quant(const float *c1, int64_t nb, float mu, int8_t *q8, float *s2)
{
    const int64_t nb2 = (nb + ORC_BLOCK2 - 1) / ORC_BLOCK2;
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nb2; ++j) {
        const int64_t b0 = j * ORC_BLOCK2;
        const int64_t b1 = (b0 + ORC_BLOCK2 < nb) ? b0 + ORC_BLOCK2 : nb;
        float m = 0.0f;
        for (int64_t b = b0; b < b1; ++b) {
            float d = c1[b] - mu;
            float a = fabsf(d);
            if (a > m) m = a;
        }
        s2[j] = m;
        for (int64_t b = b0; b < b1; ++b) {
            if (m == 0.0f) { q8[b] = 0; continue; }
            float d = c1[b] - mu;
            float r = d / m;
            float t = r * 127.0f;
            q8[b] = (int8_t)rintf(t);
        }
    }
}

/* Step 7: the dequantised first-level constant of block b.
 *   step_j = fl(s2_j / 127);  c^_b = fl(fl(q8_b * step_j) + mu) */
float orc_dequant_constant(int8_t q8, float s2, float mu)
{
    float step = s2 / 127.0f;
    float p = (float)q8 * step;
    return p + mu;
}

/* Step 8: the dequantised weight w^_i = bf16(fl(Q[code_i] * c^_b)), the
 * value the forward and backward products use (section 3: weights are
 * dequantised to BF16 on demand). Output: bf16 bit patterns. */
void orc_dequant(const uint8_t *codes, const int8_t *q8, const float *s2, float mu,
                 int64_t n, const float Q[16], uint16_t *out)
{
    const int64_t nb = (n + ORC_BLOCK1 - 1) / ORC_BLOCK1;
    #pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        const float c = orc_dequant_constant(q8[b], s2[b / ORC_BLOCK2], mu);
        const int64_t i0 = b * ORC_BLOCK1;
        const int64_t i1 = (i0 + ORC_BLOCK1 < n) ? i0 + ORC_BLOCK1 : n;
        for (int64_t i = i0; i < i1; ++i) {
            uint8_t byte = codes[i / 2];
            int code = (i % 2 == 0) ? (byte >> 4) : (byte & 15);
            float v = Q[code] * c;
            out[i] = orc_bf16_rne(v);
        }
    }
}

/* Decode of bf16 bit patterns to fp32 (exact widening), for callers that
 * hand bf16 inputs to orc_quantize_codes. */
void orc_bf16_array_to_f32(const uint16_t *in, int64_t n, float *out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_to_f32(in[i]);
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Adapter merge (the page's section 5 notes that merging the adapter into    */
/* the weight and re-quantising can change outputs; section 6 asks to check   */
/* it). Reading: the merge is done in BF16, the compute type:                  */
/*   d[n,k]  = A[k,0]*B[0,n] + ... + A[k,r-1]*B[r-1,n], one fused multiply-add */
/*             per term in increasing j, starting from 0 (fmaf: the exactly   */
/*             rounded a*b+c, not a contraction by the compiler);             */
/*   w'[n,k] = bf16( fl( w^[n,k] + fl(s * d[n,k]) ) ),                         */
/* with w^ the dequantised BF16 weight [rows, cols] (bf16 bits), A [cols, r]   */
/* and B [r, rows] widened exactly from bf16 to fp32. Output: bf16 bits.       */
void orc_merge_bf16(const uint16_t *w_hat, const float *A, const float *B, int64_t rows, int64_t cols,
                    int r, float s, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < rows; ++n) {
        for (int64_t k = 0; k < cols; ++k) {
            float d = 0.0f;
            for (int j = 0; j < r; ++j) d = fmaf(A[k * r + j], B[(int64_t)j * rows + n], d);
            const float t = s * d;
            const float w = orc_bf16_to_f32(w_hat[n * cols + k]) + t;
            out[n * cols + k] = orc_bf16_rne(w);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Optimizer step of the adapter (the page's section 3 procedure ends every   */
/* batch with "update LoRA with a paged optimizer"; section 2 says paged      */
/* optimizers keep their state in unified memory that moves between GPU and  */
/* CPU when needed). The optimizer is AdamW (decoupled weight decay) on fp32  */
/* master parameters theta with fp32 moments m, v. Reading: one step at       */
/* step count t >= 1 is, per element and in this order, every operation one   */
/* IEEE binary32 operation:                                                   */
/*   m     = fl( fl(b1 * m) + fl(fl(1 - b1) * g) )                            */
/*   v     = fl( fl(b2 * v) + fl(fl(1 - b2) * fl(g * g)) )                    */
/*   den   = fl( fl(sqrt(fl(v * ib2))) + eps )                                */
/*   upd   = fl( fl(m * ib1) / den )                                          */
/*   theta = fl( theta - fl(lr * fl(upd + fl(wd * theta))) )                  */
/* with the inverse bias corrections ib1 = 1 / (1 - b1^t) and                 */
/* ib2 = 1 / (1 - b2^t) computed by the caller in double and rounded once to  */
/* float (one division and one square root per element). theta_bf16          */
/* (optional) receives bf16(theta), the adapter copy the layer multiplies     */
/* with.                                                                      */
void orc_adamw_step(float *theta, const float *g, float *m, float *v, int64_t n, float lr, float b1,
                    float b2, float eps, float wd, float ib1, float ib2, uint16_t *theta_bf16)
{
    const float c1 = 1.0f - b1, c2 = 1.0f - b2;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const float gi = g[i];
        const float mi = b1 * m[i] + c1 * gi;
        const float gg = gi * gi;
        const float vi = b2 * v[i] + c2 * gg;
        const float den = sqrtf(vi * ib2) + eps;
        const float upd = (mi * ib1) / den;
        const float decay = wd * theta[i];
        const float step = lr * (upd + decay);
        theta[i] = theta[i] - step;
        m[i] = mi;
        v[i] = vi;
        if (theta_bf16) theta_bf16[i] = orc_bf16_rne(theta[i]);
    }
}

/* Inverse bias corrections of step t (double, rounded once to float). */
void orc_adamw_bias_corrections(float b1, float b2, int64_t t, float *ib1, float *ib2)
{
    *ib1 = (float)(1.0 / (1.0 - pow((double)b1, (double)t)));
    *ib2 = (float)(1.0 / (1.0 - pow((double)b2, (double)t)));
}
