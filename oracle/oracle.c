/*
 * oracle.c -- plain, slow, CPU reference for the INT8-quantised attention
 * forward pass.  TEST INFRASTRUCTURE ONLY: it is loaded by the tests, by the
 * smoke check and by the benchmark's CPU-baseline leg, never by the product
 * path.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes, and where each step comes from:
 *
 *   quantiser       IntAttention: A Fully Integer Attention Pipeline for
 *                   Efficient Edge Inference, section 2.1, eq. 3:
 *                   s_X = max|X| / 127, X ~= s_X * X_hat, zero-point 0.
 *                   Granularity: one scale per token row for Q and K
 *                   (INT-FlashAttention: Enabling Flash Attention for INT8
 *                   Quantization, abstract: "token-level" quantisation), one
 *                   scale per L x d tensor for V (IntAttention section 2.1
 *                   applies eq. 3 per tensor to V in R^{L x d}).
 *   integer logits  IntAttention section 2.1, eq. 4: A_hat = Q_hat K_hat^T in
 *                   INT8 x INT8 -> INT32; the rescale alpha is
 *                   s_Q[i] s_K[j] / sqrt(d) (section 3.1, eq. 8 gives
 *                   c_int = round(c / alpha) = round(c sqrt(d) / (s_Q s_K))).
 *   softmax         IntAttention section 2.2, eq. 6: row-max subtraction,
 *                   two passes over the full row (max, then exp and sum).
 *   P quantisation  IntAttention section 3.2: probabilities times 127 stored
 *                   as signed INT8; applied to the unnormalised
 *                   p = exp(t - m) in (0, 1].
 *   value path      IntAttention section 2.1, eq. 5: O ~= s_V P V_hat.
 *   online form     the same steps in FlashAttention's block-wise order
 *                   (running max and running sum, P codes against the
 *                   running max), see oracle_attention_online_rows.
 *   reference       IntAttention section 2.1, eq. 1: O = softmax(Q K^T /
 *                   sqrt(d)) V in fp64 from the unquantised inputs.
 *   decode          one query against a key / value cache with the keys cut
 *                   into ranges (split-KV), each range in the online order,
 *                   merged at the end; see oracle_decode.
 *   IndexSoftmax    IntAttention sections 3.1-3.2: integer clipping of the
 *                   row-max distance, a 2^b-entry UINT8 exponential table,
 *                   UINT8 P (times 255), integer row sums; see
 *                   oracle_index_attention_rows.
 *
 * Causal masking keeps keys j <= i (square, top-left aligned).
 *
 * Parity status: every function here is pinned by the CPU tests (closed
 * forms, invariants, brute force on tiny inputs); see tests/test_oracle_*.py.
 *
 * Built with plain gcc -O2 -fopenmp, no fast-math: fp32 divisions are IEEE
 * round-to-nearest-even, nearbyint() uses the default rounding mode (to
 * nearest, ties to even).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* threads                                                             */
/* ------------------------------------------------------------------ */

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* quantiser (IntAttention section 2.1, eq. 3)                         */
/* ------------------------------------------------------------------ */

/* One symmetric INT8 code: RNE(x / s) clamped to [-127, 127]; s == 0 -> 0.
 * x / s is one IEEE fp32 division. */
static int8_t quant_one(float x, float s) {
    if (s == 0.0f) return 0;
    float r = nearbyintf(x / s);
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/* Scale of a set of values: max|x| / 127, one IEEE fp32 division. */
static float scale_of(const float *x, int64_t n) {
    float amax = 0.0f;
    for (int64_t k = 0; k < n; ++k) {
        float a = fabsf(x[k]);
        if (a > amax) amax = a;
    }
    return amax / 127.0f;
}

/* Per-token: `rows` rows of `d` values, one scale per row. */
void oracle_quantize_per_token(const float *x, int64_t rows, int64_t d,
                               int8_t *xq, float *scale) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float *xr = x + r * d;
        float s = scale_of(xr, d);
        scale[r] = s;
        for (int64_t k = 0; k < d; ++k) xq[r * d + k] = quant_one(xr[k], s);
    }
}

/* Per-token with b-bit symmetric codes (the pages' INT4 remark, INT-FA
 * abstract; eq. 3 with 127 replaced by qmax = 2^(b-1) - 1): s = max|x| / qmax
 * (one IEEE fp32 division), codes RNE(x / s) clamped to [-qmax, qmax], stored
 * one per int8.  b = 8 is oracle_quantize_per_token. */
void oracle_quantize_per_token_bits(const float *x, int64_t rows, int64_t d, int bits,
                                    int8_t *xq, float *scale) {
    const float qmax = (float)((1 << (bits - 1)) - 1);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float *xr = x + r * d;
        float amax = 0.0f;
        for (int64_t k = 0; k < d; ++k) {
            float a = fabsf(xr[k]);
            if (a > amax) amax = a;
        }
        const float s = amax / qmax;
        scale[r] = s;
        for (int64_t k = 0; k < d; ++k) {
            float c = 0.0f;
            if (s != 0.0f) {
                c = nearbyintf(xr[k] / s);
                if (c > qmax) c = qmax;
                if (c < -qmax) c = -qmax;
            }
            xq[r * d + k] = (int8_t)c;
        }
    }
}

/* Per-tensor: `groups` contiguous groups of `group_len` values, one scale
 * per group (for V: groups = B*H, group_len = L*d). */
void oracle_quantize_per_tensor(const float *x, int64_t groups,
                                int64_t group_len, int8_t *xq, float *scale) {
    for (int64_t g = 0; g < groups; ++g) {
        const float *xg = x + g * group_len;
        float s = scale_of(xg, group_len);
        scale[g] = s;
#pragma omp parallel for schedule(static)
        for (int64_t k = 0; k < group_len; ++k) xq[g * group_len + k] = quant_one(xg[k], s);
    }
}

/* ------------------------------------------------------------------ */
/* integer logits (IntAttention section 2.1, eq. 4)                    */
/* ------------------------------------------------------------------ */

static int32_t dot_i8(const int8_t *a, const int8_t *b, int64_t d) {
    int32_t acc = 0;
    for (int64_t k = 0; k < d; ++k) acc += (int32_t)a[k] * (int32_t)b[k];
    return acc;
}

/* S[h][i][j] = sum_k Qq[h][i][k] * Kq[h][j][k] for `heads` heads of L x d. */
void oracle_qk_int32(const int8_t *Qq, const int8_t *Kq, int64_t heads,
                     int64_t L, int64_t d, int32_t *S) {
    for (int64_t h = 0; h < heads; ++h) {
        const int8_t *q = Qq + h * L * d, *k = Kq + h * L * d;
        int32_t *s = S + h * L * L;
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < L; ++i)
            for (int64_t j = 0; j < L; ++j) s[i * L + j] = dot_i8(q + i * d, k + j * d, d);
    }
}

/* ------------------------------------------------------------------ */
/* quantised attention, rows [r0, r1) of one head                       */
/* ------------------------------------------------------------------ */

/*
 * Qq, Kq, Vq: int8 [L][d] of one (b, h); sQ, sK: fp32 [L]; sV: the head's
 * per-tensor scale.  Writes O[(i - r0) * d + c] in fp64.  Optional outputs
 * (may be NULL): m_out / l_out [r1 - r0] (row max of t in natural-log units
 * and the row sum of p), P_out [(r1 - r0) * L] (the INT8 P codes, 0 for
 * masked keys).
 */
void oracle_attention_rows(const int8_t *Qq, const int8_t *Kq, const int8_t *Vq,
                           const float *sQ, const float *sK, float sV,
                           int64_t L, int64_t d, int causal, int64_t r0, int64_t r1,
                           double *O, double *m_out, double *l_out, int32_t *P_out) {
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = r0; i < r1; ++i) {
        const int64_t n = causal ? (i + 1) : L; /* keys j < n are visible */
        double *t = (double *)malloc((size_t)n * sizeof(double));
        int32_t *ph = (int32_t *)malloc((size_t)n * sizeof(int32_t));
        int64_t *acc = (int64_t *)calloc((size_t)d, sizeof(int64_t));
        /* step 1: integer logits and their float rescale (eq. 4, alpha) */
        for (int64_t j = 0; j < n; ++j) {
            int32_t sij = dot_i8(Qq + i * d, Kq + j * d, d);
            t[j] = (double)sij * (double)sQ[i] * (double)sK[j] * inv_sqrt_d;
        }
        /* step 2: pass 1, the row max (eq. 6) */
        double m = -INFINITY;
        for (int64_t j = 0; j < n; ++j) if (t[j] > m) m = t[j];
        /* step 3: pass 2, p = exp(t - m), the row sum, and P codes = RNE(127 p) */
        double l = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            double p = exp(t[j] - m);
            l += p;
            ph[j] = (int32_t)nearbyint(127.0 * p);
        }
        /* step 4: integer P V_hat (eq. 5, before the scale) */
        for (int64_t j = 0; j < n; ++j) {
            const int8_t *v = Vq + j * d;
            for (int64_t c = 0; c < d; ++c) acc[c] += (int64_t)ph[j] * (int64_t)v[c];
        }
        /* step 5: O = s_V * (P_hat V_hat) / (127 l) */
        double *o = O + (i - r0) * d;
        for (int64_t c = 0; c < d; ++c) o[c] = (double)sV * (double)acc[c] / (127.0 * l);
        if (m_out) m_out[i - r0] = m;
        if (l_out) l_out[i - r0] = l;
        if (P_out) {
            int32_t *pr = P_out + (i - r0) * L;
            for (int64_t j = 0; j < L; ++j) pr[j] = (j < n) ? ph[j] : 0;
        }
        free(t);
        free(ph);
        free(acc);
    }
}

/* ------------------------------------------------------------------ */
/* quantised attention in FlashAttention's block-wise online form       */
/* ------------------------------------------------------------------ */

/*
 * The same method as oracle_attention_rows, but in the order of
 * FlashAttention's forward workflow (INT-FlashAttention abstract: the INT8
 * architecture is compatible with that workflow; FlashAttention-3 abstract:
 * block-wise softmax interleaved with the two matmuls).  Keys are visited in
 * blocks of `block`; per block:
 *   m_new = max(m, max_j t_ij);  alpha = exp(m - m_new)  (0 for the first)
 *   p_ij  = exp(t_ij - m_new);   codes = RNE(127 p_ij)  (IntAttention 3.2)
 *   acc   = alpha acc + sum_j codes_ij V_hat_j   (integer block sum, fp64)
 *   l     = alpha l + sum_j p_ij
 * and finally O = s_V acc / (127 l) (IntAttention eq. 5).  With one block
 * this is exactly the two-pass function above.
 * lsum_codes != 0 takes the other reading of the row sum: l from the P codes,
 * l = alpha l + sum_j codes_ij / 127 (IntAttention section 3.2 quantises P
 * before the value product; the pages do not say which p the sum uses).
 * p_levels is the largest P code: 127 (P stored as INT8, the INT-FlashAttention
 * pipeline) or 255 (P stored as UINT8, codes RNE(255 p), the scheme that
 * IntAttention's Table 5 ablation favours); 127 above stands for p_levels.
 */
void oracle_attention_online_rows(const int8_t *Qq, const int8_t *Kq, const int8_t *Vq,
                                  const float *sQ, const float *sK, float sV,
                                  int64_t L, int64_t d, int causal, int64_t block,
                                  int64_t r0, int64_t r1, double *O, double *l_out, int lsum_codes,
                                  int p_levels) {
    const double levels = (double)p_levels;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = r0; i < r1; ++i) {
        const int64_t n = causal ? (i + 1) : L;
        double *t = (double *)malloc((size_t)block * sizeof(double));
        double *acc = (double *)calloc((size_t)d, sizeof(double));
        int64_t *blk = (int64_t *)malloc((size_t)d * sizeof(int64_t));
        double m = -INFINITY, l = 0.0;
        for (int64_t j0 = 0; j0 < n; j0 += block) {
            const int64_t nb = (n - j0 < block) ? (n - j0) : block;
            double bm = -INFINITY;
            for (int64_t jj = 0; jj < nb; ++jj) {
                const int64_t j = j0 + jj;
                int32_t sij = dot_i8(Qq + i * d, Kq + j * d, d);
                t[jj] = (double)sij * (double)sQ[i] * (double)sK[j] * inv_sqrt_d;
                if (t[jj] > bm) bm = t[jj];
            }
            const double m_new = (bm > m) ? bm : m;
            const double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
            double psum = 0.0;
            for (int64_t c = 0; c < d; ++c) blk[c] = 0;
            for (int64_t jj = 0; jj < nb; ++jj) {
                double p = exp(t[jj] - m_new);
                int64_t code = (int64_t)nearbyint(levels * p);
                psum += lsum_codes ? (double)code / levels : p;
                const int8_t *v = Vq + (j0 + jj) * d;
                for (int64_t c = 0; c < d; ++c) blk[c] += code * (int64_t)v[c];
            }
            for (int64_t c = 0; c < d; ++c) acc[c] = alpha * acc[c] + (double)blk[c];
            l = alpha * l + psum;
            m = m_new;
        }
        double *o = O + (i - r0) * d;
        for (int64_t c = 0; c < d; ++c) o[c] = (double)sV * acc[c] / (levels * l);
        if (l_out) l_out[i - r0] = l;
        free(t);
        free(acc);
        free(blk);
    }
}

/* ------------------------------------------------------------------ */
/* unquantised fp64 attention (IntAttention section 2.1, eq. 1)         */
/* ------------------------------------------------------------------ */

/* Q, K, V: fp32 [L][d] of one head (the exact widening of the fp16 inputs).
 * Writes O[(i - r0) * d + c] for rows [r0, r1). */
void oracle_attention_fp64_rows(const float *Q, const float *K, const float *V,
                                int64_t L, int64_t d, int causal, int64_t r0,
                                int64_t r1, double *O) {
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = r0; i < r1; ++i) {
        const int64_t n = causal ? (i + 1) : L;
        double *a = (double *)malloc((size_t)n * sizeof(double));
        double m = -INFINITY;
        for (int64_t j = 0; j < n; ++j) {
            double s = 0.0;
            for (int64_t k = 0; k < d; ++k) s += (double)Q[i * d + k] * (double)K[j * d + k];
            a[j] = s * inv_sqrt_d;
            if (a[j] > m) m = a[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            a[j] = exp(a[j] - m);
            l += a[j];
        }
        double *o = O + (i - r0) * d;
        for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
        for (int64_t j = 0; j < n; ++j)
            for (int64_t c = 0; c < d; ++c) o[c] += a[j] * (double)V[j * d + c];
        for (int64_t c = 0; c < d; ++c) o[c] /= l;
        free(a);
    }
}

/* ------------------------------------------------------------------ */
/* IndexSoftmax attention (IntAttention sections 3.1-3.2)               */
/* ------------------------------------------------------------------ */

/*
 * The exponential lookup table of IndexSoftmax (IntAttention section 3.1,
 * "LUT-based alternative", and section 3.2, "the float table is mapped
 * linearly onto an integer table"): 2^b UINT8 entries, entry k standing for
 * the clipped distance k c / (2^b - 1) (the index map of eq. 10 read
 * backwards), scaled by 255 (section 3.2: UINT8 probabilities times 255):
 *   LUT[k] = RNE(255 exp(-c k / (2^b - 1))),   k = 0 .. 2^b - 1.
 */
void oracle_index_lut(double c, int b, uint8_t *lut) {
    const int64_t n = (int64_t)1 << b;
    for (int64_t k = 0; k < n; ++k) {
        const double x = c * (double)k / (double)(n - 1);
        lut[k] = (uint8_t)nearbyint(255.0 * exp(-x));
    }
}

/*
 * The quantisation-aligned clipping threshold (IntAttention section 3.1,
 * eq. 8): c_int = round(c / alpha) with alpha = s_Q s_K / sqrt(d), the
 * per-tensor scales of the default configuration (section 3.3).  Evaluated
 * in fp64 as rint((c sqrt(d)) / (s_Q s_K)); at least 1 (a zero scale means
 * all logits are 0 and every distance is 0, so any positive threshold gives
 * the same result).
 */
int64_t oracle_index_cint(double c, int64_t d, float sQ, float sK) {
    const double den = (double)sQ * (double)sK;
    if (!(den > 0.0)) return 1;
    const double v = nearbyint((c * sqrt((double)d)) / den);
    if (v < 1.0) return 1;
    if (v > 4.0e18) return (int64_t)4e18;
    return (int64_t)v;
}

/*
 * IndexSoftmax attention for rows [r0, r1) of one head (IntAttention
 * section 3.1 eqs. 7-10, section 3.2), with the value path of eq. 5:
 *   A_hat    = Q_hat K_hat^T                       (INT32, eq. 4)
 *   Delta    = rowmax(A_hat) - A_hat               (eq. 7; over visible keys)
 *   Delta'   = min(Delta, c_int)                   (eq. 9)
 *   idx      = floor(Delta' (2^b - 1) / c_int)     (eq. 10, exact integers)
 *   E        = LUT[idx]                            (UINT8, ~ 255 exp(-alpha Delta'))
 *   O_i      = s_V sum_j E_ij V_hat_j / sum_j E_ij
 * Qq, Kq, Vq: int8 [L][d]; sQ, sK, sV: the head's per-tensor scales.
 * The normalisation by the integer row sum is applied after the P V
 * product (the same quotient as normalising P first, without rounding the
 * normalised probabilities to 8 bits).  Masked keys (causal, j > i) get
 * E = 0.  Optional outputs (may be NULL): m_out / l_out [r1 - r0] (the
 * integer row max of A_hat and the integer row sum of E), E_out
 * [(r1 - r0) * L] (E, 0 for masked keys).
 */
void oracle_index_attention_rows(const int8_t *Qq, const int8_t *Kq, const int8_t *Vq,
                                 float sQ, float sK, float sV, int64_t L, int64_t d,
                                 int causal, double c, int b, int64_t r0, int64_t r1,
                                 double *O, int64_t *m_out, int64_t *l_out, int32_t *E_out) {
    uint8_t lut[256];
    oracle_index_lut(c, b, lut);
    const int64_t nm1 = ((int64_t)1 << b) - 1;
    const int64_t cint = oracle_index_cint(c, d, sQ, sK);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = r0; i < r1; ++i) {
        const int64_t n = causal ? (i + 1) : L;
        int64_t *a = (int64_t *)malloc((size_t)n * sizeof(int64_t));
        int64_t *acc = (int64_t *)calloc((size_t)d, sizeof(int64_t));
        int32_t *e = (int32_t *)malloc((size_t)n * sizeof(int32_t));
        /* eq. 4: integer logits; eq. 7: the row max over visible keys */
        int64_t m = INT64_MIN;
        for (int64_t j = 0; j < n; ++j) {
            a[j] = dot_i8(Qq + i * d, Kq + j * d, d);
            if (a[j] > m) m = a[j];
        }
        /* eqs. 7-10: distance, clip, index, table */
        int64_t l = 0;
        for (int64_t j = 0; j < n; ++j) {
            int64_t delta = m - a[j];
            if (delta > cint) delta = cint;
            const int64_t idx = (delta * nm1) / cint;
            e[j] = lut[idx];
            l += e[j];
        }
        /* eq. 5: integer E V_hat, then the scale and the row-sum normalisation */
        for (int64_t j = 0; j < n; ++j) {
            const int8_t *v = Vq + j * d;
            for (int64_t cc = 0; cc < d; ++cc) acc[cc] += (int64_t)e[j] * (int64_t)v[cc];
        }
        double *o = O + (i - r0) * d;
        for (int64_t cc = 0; cc < d; ++cc) o[cc] = (double)sV * (double)acc[cc] / (double)l;
        if (m_out) m_out[i - r0] = m;
        if (l_out) l_out[i - r0] = l;
        if (E_out) {
            int32_t *er = E_out + (i - r0) * L;
            for (int64_t j = 0; j < L; ++j) er[j] = (j < n) ? e[j] : 0;
        }
        free(a);
        free(acc);
        free(e);
    }
}

/* ------------------------------------------------------------------ */
/* decode: one query against a key / value cache, split into ranges    */
/* ------------------------------------------------------------------ */

/*
 * One query row of the quantised attention against L keys (no mask), in the
 * block-wise online order of oracle_attention_online_rows, with the keys cut
 * into consecutive ranges of split_len keys (split_len a multiple of
 * `block`).  Each range runs the online steps on its own (running max, P
 * codes against that range's running max, integer block sums, alpha
 * rescales), and the ranges are merged at the end (FlashAttention's
 * block-wise softmax applied once more at range granularity):
 *   M = max_s m_s,  O = s_V sum_s e^(m_s - M) acc_s / (127 sum_s e^(m_s - M) l_s).
 * With split_len >= L this is exactly one row of oracle_attention_online_rows.
 * q: int8 [d] with scale sq; Kq, Vq: int8 [L][d]; sK: fp32 [L].
 */
void oracle_decode(const int8_t *q, float sq, const int8_t *Kq, const float *sK, const int8_t *Vq,
                   float sV, int64_t L, int64_t d, int64_t block, int64_t split_len, double *O) {
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    const int64_t nsplit = (L + split_len - 1) / split_len;
    double *ms = (double *)malloc((size_t)nsplit * sizeof(double));
    double *ls = (double *)malloc((size_t)nsplit * sizeof(double));
    double *accs = (double *)calloc((size_t)(nsplit * d), sizeof(double));
    double *t = (double *)malloc((size_t)block * sizeof(double));
    int64_t *blk = (int64_t *)malloc((size_t)d * sizeof(int64_t));
    for (int64_t s = 0; s < nsplit; ++s) {
        const int64_t s0 = s * split_len;
        const int64_t s1 = (s0 + split_len < L) ? s0 + split_len : L;
        double m = -INFINITY, l = 0.0;
        double *acc = accs + s * d;
        for (int64_t j0 = s0; j0 < s1; j0 += block) {
            const int64_t nb = (s1 - j0 < block) ? (s1 - j0) : block;
            double bm = -INFINITY;
            for (int64_t jj = 0; jj < nb; ++jj) {
                const int64_t j = j0 + jj;
                t[jj] = (double)dot_i8(q, Kq + j * d, d) * (double)sq * (double)sK[j] * inv_sqrt_d;
                if (t[jj] > bm) bm = t[jj];
            }
            const double m_new = (bm > m) ? bm : m;
            const double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
            double psum = 0.0;
            for (int64_t c = 0; c < d; ++c) blk[c] = 0;
            for (int64_t jj = 0; jj < nb; ++jj) {
                const double p = exp(t[jj] - m_new);
                psum += p;
                const int64_t code = (int64_t)nearbyint(127.0 * p);
                const int8_t *v = Vq + (j0 + jj) * d;
                for (int64_t c = 0; c < d; ++c) blk[c] += code * (int64_t)v[c];
            }
            for (int64_t c = 0; c < d; ++c) acc[c] = alpha * acc[c] + (double)blk[c];
            l = alpha * l + psum;
            m = m_new;
        }
        ms[s] = m;
        ls[s] = l;
    }
    double M = -INFINITY;
    for (int64_t s = 0; s < nsplit; ++s) if (ms[s] > M) M = ms[s];
    double den = 0.0;
    for (int64_t c = 0; c < d; ++c) O[c] = 0.0;
    for (int64_t s = 0; s < nsplit; ++s) {
        const double w = exp(ms[s] - M);
        den += w * ls[s];
        for (int64_t c = 0; c < d; ++c) O[c] += w * accs[s * d + c];
    }
    for (int64_t c = 0; c < d; ++c) O[c] = (double)sV * O[c] / (127.0 * den);
    free(ms);
    free(ls);
    free(accs);
    free(t);
    free(blk);
}
