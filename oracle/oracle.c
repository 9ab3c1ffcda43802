/*
 * oracle.c -- plain, slow CPU oracle for the BWTA / BiLLM hot path.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the benchmark's
 * CPU-baseline leg call this code; the product path (the CUDA library) never
 * does, and the two share no code, header, table or helper. The oracle works on
 * UNPACKED values: int8 arrays holding -1, 0 or +1 plus fp32 scales, and it
 * accumulates in int64 / fp64. Packing is a separate, naive bit-by-bit loop
 * (orc_pack_plane) whose output the CUDA packers must reproduce exactly.
 *
 * Sources (web pages) this follows:
 *  [BWTA]  "BWTA: Accurate and Efficient Binarized Transformer by
 *          Algorithm-Hardware Co-design" -- abstract and "Core claim": weights
 *          are binary, activations are ternary by projecting tiny values to
 *          zero; Figure 6: 32 fp16 values are packed into one 32-bit word.
 *  [BiLLM] "BiLLM: Pushing the Limit of Post-Training Quantization for LLMs"
 *          -- abstract and "Approach": salient weights are chosen structurally
 *          by column and binarized with a residual (second) binarization; the
 *          bell-shaped non-salient weights are split at a break-point into a
 *          concentrated and a sparse group, each binarized with its own
 *          scale; "Limitations": a 1-bit group identifier per weight; the
 *          block-size ablation: 128-column blocks.
 *  [XNOR]  XNOR-Net (cited by both pages): the scale of a binarized tensor is
 *          mean|w| (the L2-optimal scale for sign(w)).
 *
 * Readings where the pages are silent (each one is a stated convention):
 *  R1  ternary threshold: keep x iff |x| > 0.5 * mean|x|, the mean taken over
 *      all K entries of the row; equality projects to zero.
 *  R2  activation scale: the mean of |x| over the kept entries (0 if none).
 *  R3  weight scale: mean|w| per row, or per group of `group` consecutive
 *      columns; sign(0) = +1 (and -0.0 counts as 0).
 *  R4  BiLLM salient metric without calibration data: the Hessian is taken
 *      as the identity, so a column's saliency is sum_n w[n,k]^2; the n_sal
 *      largest per 128-column block are salient (ties: lower index).
 *  R5  BiLLM break-point: p = 0.5 * max|w| over the non-salient weights of
 *      one row inside one block; sparse group = {|w| > p}.
 *  R6  BiLLM scales are rounded to fp32 before any further use.
 *  R17 attention probabilities are ternarized like activations: kept iff
 *      p > 0.5 * mean(p) = 1/(2L) (a softmax row has mean 1/L); scale = mean
 *      of the kept p.
 *  R18 BiLLM's "optimal splitting search": the break-point is the non-salient
 *      magnitude of the row-block that minimizes the squared binarization
 *      error of the two groups (each scaled by its mean magnitude); ties go to
 *      the smaller break-point.
 *
 * Arithmetic of the fp16 magnitudes: every finite fp16 value is an integer
 * multiple of 2^-24, so |x| * 2^24 is an exact integer below 2^40 and sums of
 * them are exact in int64. The threshold test R1 then reads 2*K*v > S, where
 * v = |x|*2^24 and S = sum of v over the row: exact, with no rounding order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_OK = 0, ORC_ERR_ARG = 1, ORC_ERR_NONFINITE = 5 };

/* ------------------------------------------------------------ fp16 values */

static int half_is_finite(uint16_t h) { return ((h >> 10) & 31) != 31; }

/* exact value of a finite fp16 bit pattern (IEEE 754 binary16 definition) */
static double half_value(uint16_t h) {
  int e = (h >> 10) & 31;
  int f = h & 1023;
  double mag = (e == 0) ? ldexp((double)f, -24) : ldexp((double)(1024 + f), e - 25);
  return (h & 0x8000) ? -mag : mag;
}

/* |x| in units of 2^-24, an exact integer */
static int64_t half_mag_units(uint16_t h) { return (int64_t)ldexp(fabs(half_value(h)), 24); }

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ------------------------------------------------- activation quantization
 * [BWTA] abstract: activations are ternarized by projecting tiny values to
 * zero (readings R1, R2). Binary mode: a = sign(x) with sign(0) = +1 and scale
 * mean|x| over the whole row ([XNOR]).
 * Output a[m*K + k] in {-1, 0, +1}; scale[m] fp32.
 */
int orc_quantize_acts(const uint16_t *X, int64_t M, int64_t K, int64_t ldX, int ternary,
                      int8_t *a, float *scale) {
  if (M < 0 || K < 0 || ldX < K || K > (1LL << 22)) return ORC_ERR_ARG;
  for (int64_t m = 0; m < M; ++m) {
    const uint16_t *row = X + m * ldX;
    int64_t S = 0;
    for (int64_t k = 0; k < K; ++k) {
      if (!half_is_finite(row[k])) return ORC_ERR_NONFINITE;
      S += half_mag_units(row[k]);
    }
    if (ternary) {
      int64_t kept_sum = 0, kept = 0;
      for (int64_t k = 0; k < K; ++k) {
        double x = half_value(row[k]);
        int64_t v = half_mag_units(row[k]);
        int keep = (2 * K * v > S); /* |x| > 0.5 * (S / K): R1, strict */
        a[m * K + k] = keep ? (x < 0 ? -1 : 1) : 0;
        if (keep) {
          kept_sum += v;
          kept += 1;
        }
      }
      scale[m] = kept ? (float)(((double)kept_sum / (double)kept) * 0x1p-24) : 0.0f;
    } else {
      for (int64_t k = 0; k < K; ++k) a[m * K + k] = (half_value(row[k]) < 0) ? -1 : 1;
      scale[m] = K ? (float)(((double)S / (double)K) * 0x1p-24) : 0.0f;
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------ weight binarization
 * [BWTA] binary weights; [XNOR] scale = mean|w| (reading R3).
 * group == 0: one scale per row; otherwise ceil(K/group) scales per row, the
 * last group holding the K % group leftover columns when K is not a multiple.
 * b[n*K + k] in {-1, +1}; alpha[n*G + g] fp32.
 */
int orc_binarize_weights(const float *W, int64_t N, int64_t K, int64_t ldW, int64_t group,
                         int8_t *b, float *alpha) {
  if (N < 0 || K <= 0 || ldW < K || group < 0) return ORC_ERR_ARG;
  int64_t gs = group ? group : K;
  int64_t G = (K + gs - 1) / gs;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < G; ++g) {
      int64_t k0 = g * gs, k1 = k0 + gs < K ? k0 + gs : K;
      double sum = 0.0;
      for (int64_t k = k0; k < k1; ++k) {
        float w = W[n * ldW + k];
        if (isnan(w) || isinf(w)) return ORC_ERR_NONFINITE;
        b[n * K + k] = (w < 0.0f) ? -1 : 1;
        sum += fabs((double)w);
      }
      alpha[n * G + g] = (float)(sum / (double)(k1 - k0));
    }
  }
  return ORC_OK;
}

/* ---------------------------------------------------------------- packing
 * [BWTA] Figure 6: 32 values packed into one 32-bit word. Convention of this
 * library: bit i of word w is element k = 32*w + i (least significant bit
 * first). plane 0 = nonzero mask (v != 0), plane 1 = sign (v < 0). Words past
 * K, up to ld, are zero.
 */
int orc_pack_plane(const int8_t *v, int64_t R, int64_t K, int64_t ld, int plane, uint32_t *out) {
  if (ld * 32 < K || (plane != 0 && plane != 1)) return ORC_ERR_ARG;
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t w = 0; w < ld; ++w) {
      uint32_t word = 0;
      for (int i = 0; i < 32; ++i) {
        int64_t k = 32 * w + i;
        if (k >= K) break;
        int8_t x = v[r * K + k];
        int bit = plane == 0 ? (x != 0) : (x < 0);
        if (bit) word |= (uint32_t)1 << i;
      }
      out[r * ld + w] = word;
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------ integer dots
 * d[(m*N + n)*G + g] = sum over k in group g of a[m,k] * b[n,k], int64.
 * The plain definition of the binary-weight x ternary-activation product.
 */
int orc_int_dots(const int8_t *a, int64_t M, const int8_t *b, int64_t N, int64_t K, int64_t group,
                 int64_t *d) {
  if (M < 0 || N < 0 || K <= 0 || group < 0) return ORC_ERR_ARG;
  int64_t gs = group ? group : K;
  int64_t G = (K + gs - 1) / gs;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      for (int64_t g = 0; g < G; ++g) {
        int64_t k0 = g * gs, k1 = k0 + gs < K ? k0 + gs : K;
        int64_t acc = 0;
        for (int64_t k = k0; k < k1; ++k) acc += (int64_t)a[m * K + k] * (int64_t)b[n * K + k];
        d[(m * N + n) * G + g] = acc;
      }
    }
  }
  return ORC_OK;
}

/* --------------------------------------------------------- scaled outputs
 * y[m,n] = s[m] * sum_g alpha[n,g] * d[m,n,g]: the binarized weight is
 * alpha * b and the ternarized activation is s * a, so the product of the
 * dequantized operands factors this way.
 *   yref: fp64 value of that expression from the fp32 scales;
 *   mag : s * sum_g |alpha * d_g| (magnitude used for the tolerance when the
 *         group terms cancel);
 *   yrep: one fixed fp32 evaluation (acc = fma((float)d_g, alpha_g, acc) for
 *         g ascending, then acc * s), a diagnostic for kernels using that order.
 */
int orc_linear_out(const int64_t *d, int64_t M, int64_t N, int64_t G, const float *alpha,
                   const float *s, double *yref, double *mag, float *yrep) {
  if (M < 0 || N < 0 || G <= 0) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0, accmag = 0.0;
      float accf = 0.0f;
      for (int64_t g = 0; g < G; ++g) {
        int64_t dg = d[(m * N + n) * G + g];
        double t = (double)alpha[n * G + g] * (double)dg;
        acc += t;
        accmag += fabs(t);
        accf = fmaf((float)dg, alpha[n * G + g], accf);
      }
      if (yref) yref[m * N + n] = (double)s[m] * acc;
      if (mag) mag[m * N + n] = fabs((double)s[m]) * accmag;
      if (yrep) yrep[m * N + n] = accf * s[m];
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------- attention scores
 * [BWTA] abstract: binary/ternary MatMul for the attention operators. Here
 * Q . K^T with both sides ternary, per (batch*head):
 *   S[h,i,j] = sum_k q[h,i,k] * k[h,j,k]            (int64)
 *   fref     = S * sq[h,i] * sk[h,j]                 (fp64)
 *   frep     = ((float)S * sq) * sk                  (fp32, that order)
 * No 1/sqrt(d) and no softmax: the scores only.
 */
int orc_attn_scores(const int8_t *q, const int8_t *k, int64_t BH, int64_t Lq, int64_t Lk, int64_t D,
                    const float *sq, const float *sk, int64_t *S, double *fref, float *frep) {
  if (BH < 0 || Lq < 0 || Lk < 0 || D <= 0) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (int64_t h = 0; h < BH; ++h) {
    for (int64_t i = 0; i < Lq; ++i) {
      for (int64_t j = 0; j < Lk; ++j) {
        int64_t acc = 0;
        for (int64_t t = 0; t < D; ++t)
          acc += (int64_t)q[(h * Lq + i) * D + t] * (int64_t)k[(h * Lk + j) * D + t];
        int64_t o = (h * Lq + i) * Lk + j;
        float a = sq[h * Lq + i], c = sk[h * Lk + j];
        if (S) S[o] = acc;
        if (fref) fref[o] = (double)acc * (double)a * (double)c;
        if (frep) {
          float t1 = (float)acc * a;
          frep[o] = t1 * c;
        }
      }
    }
  }
  return ORC_OK;
}

/* ------------------------------------------ attention probabilities, A.V
 * [BWTA] abstract: the binary/ternary MatMul serves the attention operators,
 * so the attention probabilities, the activations that enter A . V, are
 * ternarized like any activation (reading R17): keep p iff p > 0.5 * mean(p)
 * over the row. A softmax row sums to 1, so its mean is exactly 1/L and the
 * test reads p > 1/(2L); every p is positive, so a kept value is +1. The row
 * scale is the mean of the kept p (0 if none).
 * Input: f fp32 [R][L], the scores of one query row each (the fp32 output of
 * the Q . K^T product), and the softmax factor c; x = f * c in fp32.
 * p = exp(x - max x) / sum exp(x - max x), in fp64 (exp of the math library).
 * Output: a int8 [R][L] in {0, 1}; scale fp32 [R] (fp64 sum of the kept p in
 * ascending column order, divided by the count, rounded once); p fp64 [R][L]
 * (may be NULL).
 * A . V itself is orc_attn_scores with the ternary probabilities as the query
 * side and the rows of V^T (one per output channel, ternarized over the
 * sequence) as the key side: the contraction runs over the L keys.
 */
int orc_softmax_ternarize(const float *f, int64_t R, int64_t L, float c, int8_t *a, float *scale,
                          double *p_out) {
  if (R < 0 || L <= 0) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < R; ++r) {
    const float *fr = f + r * L;
    double mx = -INFINITY;
    for (int64_t j = 0; j < L; ++j) {
      const float x = fr[j] * c;
      if ((double)x > mx) mx = (double)x;
    }
    double z = 0.0;
    for (int64_t j = 0; j < L; ++j) z += exp((double)(fr[j] * c) - mx);
    double kept = 0.0;
    int64_t n = 0;
    for (int64_t j = 0; j < L; ++j) {
      const double p = exp((double)(fr[j] * c) - mx) / z;
      if (p_out) p_out[r * L + j] = p;
      const int keep = p > 0.5 / (double)L;
      a[r * L + j] = (int8_t)keep;
      if (keep) {
        kept += p;
        ++n;
      }
    }
    scale[r] = n ? (float)(kept / (double)n) : 0.0f;
  }
  return ORC_OK;
}

/* ------------------------------------------------------- BiLLM quantizer
 * Salient columns ([BiLLM] Approach, reading R4): per block of `block`
 * columns, the n_sal columns with the largest sum_n w^2 (fp64, n ascending);
 * ties go to the lower column. Output sal_idx[j*n_sal + i], ascending within
 * each block.
 */
int orc_billm_salient(const float *W, int64_t N, int64_t K, int64_t ldW, int64_t block, int64_t n_sal,
                      int32_t *sal_idx) {
  if (N <= 0 || K <= 0 || block <= 0 || K % block || n_sal < 0 || n_sal > block || ldW < K)
    return ORC_ERR_ARG;
  int64_t nb = K / block;
  double *metric = (double *)calloc((size_t)K, sizeof(double));
  if (!metric) return ORC_ERR_ARG;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      double w = (double)W[n * ldW + k];
      metric[k] += w * w;
    }
  char *taken = (char *)malloc((size_t)block);
  for (int64_t j = 0; j < nb; ++j) {
    memset(taken, 0, (size_t)block);
    for (int64_t s = 0; s < n_sal; ++s) {
      int64_t best = -1;
      for (int64_t c = 0; c < block; ++c) {
        if (taken[c]) continue;
        if (best < 0 || metric[j * block + c] > metric[j * block + best]) best = c;
      }
      taken[best] = 1;
    }
    int64_t i = 0;
    for (int64_t c = 0; c < block; ++c)
      if (taken[c]) sal_idx[j * n_sal + i++] = (int32_t)c;
  }
  free(taken);
  free(metric);
  return ORC_OK;
}

/* The squared binarization error of the non-salient weights of one
 * row-block when split at break-point p ([BiLLM] "Approach": the bell-shaped
 * non-salient weights are split at a break-point into a concentrated and a
 * sparse group, each binarized with its own scale). With a group's scale the
 * mean of its magnitudes (the L2-optimal scale of a sign-binarized group) and
 * (w - a*sign(w))^2 = (|w| - a)^2:
 *   E(p) = sum_{|w| <= p} (|w| - a_c)^2 + sum_{|w| > p} (|w| - a_s)^2
 * Every sum in fp64, columns ascending; an empty group contributes 0. */
static double split_error(const float *w, const int8_t *cat, int64_t block, double p) {
  double sc = 0.0, ss = 0.0;
  int64_t nc = 0, ns = 0;
  for (int64_t c = 0; c < block; ++c) {
    if (cat[c] == 2) continue;
    const double aw = fabs((double)w[c]);
    if (aw <= p) {
      sc += aw;
      ++nc;
    } else {
      ss += aw;
      ++ns;
    }
  }
  const double ac = nc ? sc / (double)nc : 0.0, as = ns ? ss / (double)ns : 0.0;
  double e = 0.0;
  for (int64_t c = 0; c < block; ++c) {
    if (cat[c] == 2) continue;
    const double aw = fabs((double)w[c]);
    const double d = aw - (aw <= p ? ac : as);
    e += d * d;
  }
  return e;
}

/* Per-row BiLLM binarization of rows [n0, n1) ([BiLLM] Approach; R5, R6).
 * Inside block j of row n:
 *   salient columns:  alpha1 = mean|w|, b1 = sign(w);
 *                     r = w - alpha1*b1, alpha2 = mean|r|, b2 = sign(r)
 *                     (residual binarization: w ~ alpha1*b1 + alpha2*b2);
 *   other columns:    split == 1: p = 0.5 * max|w| (R5); split == 2: p is the
 *                     searched break-point (R18, split_error above);
 *                     sparse group = {|w| > p} (none when split == 0),
 *                     concentrated = the rest; each group: alpha = mean|w|
 *                     over its members (0 if empty), b = sign(w).
 * Outputs for row r = n - n0:
 *   cat[r*K + k]   0 concentrated, 1 sparse, 2 salient
 *   b1[r*K + k]    +-1 (b for non-salient, b1 for salient)
 *   b2[r*K + k]    +-1 at salient columns, 0 elsewhere
 *   scales[(r*nb + j)*4 + {0,1,2,3}] = alpha_c, alpha_sp, alpha1, alpha2
 */
int orc_billm_quantize_rows(const float *W, int64_t n0, int64_t n1, int64_t K, int64_t ldW,
                            int64_t block, int64_t n_sal, int split, const int32_t *sal_idx,
                            int8_t *cat, int8_t *b1, int8_t *b2, float *scales) {
  if (n0 < 0 || n1 < n0 || K <= 0 || block <= 0 || K % block || n_sal < 0 || n_sal > block)
    return ORC_ERR_ARG;
  int64_t nb = K / block;
  for (int64_t n = n0; n < n1; ++n) {
    int64_t r = n - n0;
    const float *row = W + n * ldW;
    for (int64_t j = 0; j < nb; ++j) {
      int64_t base = j * block;
      /* mark salient columns of this block */
      for (int64_t c = 0; c < block; ++c) cat[r * K + base + c] = 0;
      for (int64_t i = 0; i < n_sal; ++i) cat[r * K + base + sal_idx[j * n_sal + i]] = 2;
      /* salient: residual binarization */
      float alpha1 = 0.0f, alpha2 = 0.0f;
      if (n_sal > 0) {
        double s1 = 0.0;
        for (int64_t c = 0; c < block; ++c)
          if (cat[r * K + base + c] == 2) s1 += fabs((double)row[base + c]);
        alpha1 = (float)(s1 / (double)n_sal);
        double s2 = 0.0;
        for (int64_t c = 0; c < block; ++c) {
          if (cat[r * K + base + c] != 2) continue;
          double w = (double)row[base + c];
          int sgn1 = (row[base + c] < 0.0f) ? -1 : 1;
          double res = w - (double)alpha1 * (double)sgn1;
          s2 += fabs(res);
        }
        alpha2 = (float)(s2 / (double)n_sal);
        for (int64_t c = 0; c < block; ++c) {
          if (cat[r * K + base + c] != 2) continue;
          double w = (double)row[base + c];
          int sgn1 = (row[base + c] < 0.0f) ? -1 : 1;
          double res = w - (double)alpha1 * (double)sgn1;
          b1[r * K + base + c] = (int8_t)sgn1;
          b2[r * K + base + c] = (res < 0.0) ? -1 : 1;
        }
      }
      /* non-salient: break-point split into concentrated / sparse groups */
      double maxabs = 0.0;
      for (int64_t c = 0; c < block; ++c)
        if (cat[r * K + base + c] != 2) {
          double aw = fabs((double)row[base + c]);
          if (aw > maxabs) maxabs = aw;
        }
      /* split == 2: the searched break-point (reading R18). Candidates are the
       * block's non-salient magnitudes; the chosen p minimizes the squared
       * binarization error of the two groups; ties go to the smaller p. */
      double pbest = maxabs;
      if (split == 2) {
        double ebest = INFINITY;
        for (int64_t c0 = 0; c0 < block; ++c0) {
          if (cat[r * K + base + c0] == 2) continue;
          const double p = fabs((double)row[base + c0]);
          const double e = split_error(row + base, cat + r * K + base, block, p);
          if (e < ebest || (e == ebest && p < pbest)) {
            ebest = e;
            pbest = p;
          }
        }
      }
      double sum_c = 0.0, sum_s = 0.0;
      int64_t cnt_c = 0, cnt_s = 0;
      for (int64_t c = 0; c < block; ++c) {
        int64_t k = base + c;
        if (cat[r * K + k] == 2) continue;
        double aw = fabs((double)row[k]);
        /* |w| > 0.5 * max|w| (R5), or |w| above the searched break-point */
        int sparse = split == 2 ? (aw > pbest) : (split && (2.0 * aw > maxabs));
        cat[r * K + k] = sparse ? 1 : 0;
        b1[r * K + k] = (row[k] < 0.0f) ? -1 : 1;
        b2[r * K + k] = 0;
        if (sparse) {
          sum_s += aw;
          cnt_s++;
        } else {
          sum_c += aw;
          cnt_c++;
        }
      }
      float *sc = scales + (r * nb + j) * 4;
      sc[0] = cnt_c ? (float)(sum_c / (double)cnt_c) : 0.0f;
      sc[1] = cnt_s ? (float)(sum_s / (double)cnt_s) : 0.0f;
      sc[2] = alpha1;
      sc[3] = alpha2;
    }
  }
  return ORC_OK;
}

/* Dequantized BiLLM weight of one element, fp64 (from the fp32 scales). */
static double billm_what(int8_t c, int8_t s1, int8_t s2, const float *sc) {
  if (c == 2) return (double)sc[2] * s1 + (double)sc[3] * s2;
  return (double)sc[c] * s1;
}

/* BiLLM GEMM, rows [0, R) of the quantized weights against M fp16 rows of X:
 *   yref[m,n] = sum_j [ alpha_c  * sum_{k in C_j}   b  x
 *                     + alpha_sp * sum_{k in S_j}   b  x
 *                     + alpha1   * sum_{k in sal_j} b1 x
 *                     + alpha2   * sum_{k in sal_j} b2 x ]      (fp64)
 *   mag[m,n]  = sum_k |x_k * what_k|
 * Also checked (in the tests) against the dense product X . What^T.
 */
int orc_billm_gemm(const uint16_t *X, int64_t M, int64_t K, int64_t ldX, int64_t R, int64_t block,
                   const int8_t *cat, const int8_t *b1, const int8_t *b2, const float *scales,
                   double *yref, double *mag) {
  if (M < 0 || R < 0 || K <= 0 || block <= 0 || K % block) return ORC_ERR_ARG;
  int64_t nb = K / block;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k)
      if (!half_is_finite(X[m * ldX + k])) return ORC_ERR_NONFINITE;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t r = 0; r < R; ++r) {
      double y = 0.0, mg = 0.0;
      for (int64_t j = 0; j < nb; ++j) {
        const float *sc = scales + (r * nb + j) * 4;
        double tc = 0.0, ts = 0.0, t1 = 0.0, t2 = 0.0;
        for (int64_t c = 0; c < block; ++c) {
          int64_t k = j * block + c;
          double x = half_value(X[m * ldX + k]);
          int8_t ct = cat[r * K + k];
          if (ct == 0) tc += b1[r * K + k] * x;
          else if (ct == 1) ts += b1[r * K + k] * x;
          else {
            t1 += b1[r * K + k] * x;
            t2 += b2[r * K + k] * x;
          }
          mg += fabs(x * billm_what(ct, b1[r * K + k], b2[r * K + k], sc));
        }
        y += (double)sc[0] * tc + (double)sc[1] * ts + (double)sc[2] * t1 + (double)sc[3] * t2;
      }
      yref[m * R + r] = y;
      if (mag) mag[m * R + r] = mg;
    }
  }
  return ORC_OK;
}

/* Dense dequantized weights What[r*K + k] (fp64), for the dense cross-check. */
int orc_billm_dequant(int64_t R, int64_t K, int64_t block, const int8_t *cat, const int8_t *b1,
                      const int8_t *b2, const float *scales, double *what) {
  if (R < 0 || K <= 0 || block <= 0 || K % block) return ORC_ERR_ARG;
  int64_t nb = K / block;
  for (int64_t r = 0; r < R; ++r)
    for (int64_t k = 0; k < K; ++k)
      what[r * K + k] = billm_what(cat[r * K + k], b1[r * K + k], b2[r * K + k],
                                   scales + (r * nb + k / block) * 4);
  return ORC_OK;
}

/* BiLLM packed format, written naively element by element:
 *   sign[r*ldw + w]  bit i <-> column 32w+i: 1 if b (or b1) is negative
 *   gmap[r*ldw + w]  bit i: 1 if the column is in the sparse group
 *   res[r*nb + j]    bit i: 1 if b2 of salient column sal_idx[j][i] is negative
 *   sal[j*n_sal + i] salient column index inside block j (uint8)
 *   bscale           copied as is: [r][j][alpha_c, alpha_sp, alpha1, alpha2]
 */
int orc_billm_pack(int64_t R, int64_t K, int64_t block, int64_t n_sal, const int32_t *sal_idx,
                   const int8_t *cat, const int8_t *b1, const int8_t *b2, int64_t ldw,
                   uint32_t *sign, uint32_t *gmap, uint8_t *res, uint8_t *sal) {
  if (R < 0 || K <= 0 || block <= 0 || block > 256 || K % block || n_sal < 0 || n_sal > 8 ||
      ldw * 32 < K)
    return ORC_ERR_ARG;
  int64_t nb = K / block;
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t w = 0; w < ldw; ++w) {
      uint32_t s = 0, g = 0;
      for (int i = 0; i < 32; ++i) {
        int64_t k = 32 * w + i;
        if (k >= K) break;
        if (b1[r * K + k] < 0) s |= (uint32_t)1 << i;
        if (cat[r * K + k] == 1) g |= (uint32_t)1 << i;
      }
      sign[r * ldw + w] = s;
      gmap[r * ldw + w] = g;
    }
    for (int64_t j = 0; j < nb; ++j) {
      uint32_t byte = 0;
      for (int64_t i = 0; i < n_sal; ++i)
        if (b2[r * K + j * block + sal_idx[j * n_sal + i]] < 0) byte |= 1u << i;
      res[r * nb + j] = (uint8_t)byte;
    }
  }
  for (int64_t j = 0; j < nb; ++j)
    for (int64_t i = 0; i < n_sal; ++i) sal[j * n_sal + i] = (uint8_t)sal_idx[j * n_sal + i];
  return ORC_OK;
}
