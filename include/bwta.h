/*
 * bwta.h -- C ABI of libbwta.so: bit-packed binary weights x binary/ternary
 * activations (BWTA) and BiLLM-format binary weights x fp16 activations, as
 * hand-written CUDA kernels for NVIDIA B200 (sm_100a).
 *
 * Sources:
 *  "BWTA: Accurate and Efficient Binarized Transformer by Algorithm-Hardware
 *   Co-design" (abstract, "Core claim", Figure 6): binary weights, ternary
 *   activations made by projecting tiny values to zero, 32 fp16 values packed
 *   into one 32-bit word, binary/ternary MatMul for linear and attention.
 *  "BiLLM: Pushing the Limit of Post-Training Quantization for LLMs"
 *   (abstract, "Approach", "Limitations"): salient columns with residual
 *   binarization, non-salient weights split into two groups with their own
 *   scales, a 1-bit group map; 128-column blocks.
 *
 * Conventions shared by every call
 *  - Bit planes are uint32 words; bit i of word w is element k = 32*w + i.
 *    Rows of a plane are ld_words apart; ld_words >= ceil(K/32) and
 *    ld_words % 4 == 0 (16-byte rows). Packers write every word of the row,
 *    the padding words past K as zero.
 *  - Sign bit 1 means negative. Mask bit 1 means the ternary value is nonzero;
 *    sign bits are 0 wherever the mask bit is 0. sign(0) = +1 and -0.0 is 0.
 *  - Ternary activations: keep x iff |x| > 0.5 * mean|x| over the row (equal
 *    values are projected to zero); the row scale is the mean |x| over the kept
 *    entries (0 if none). The test is done exactly in integers (every fp16 is a
 *    multiple of 2^-24), so the planes do not depend on summation order.
 *  - Binary weights: b = sign(w); scale = mean|w| per row (group == 0) or per
 *    `group` consecutive columns (group a positive multiple of 128; the last
 *    group may be shorter when K is not a multiple of group).
 *  - Scales are fp32; fp16 data is passed as raw uint16 bit patterns.
 *  - Ownership: the caller allocates every buffer (device memory unless stated
 *    otherwise) and keeps it alive until the stream reaches the call. The
 *    library allocates no memory and keeps no state between calls.
 *  - Every call is asynchronous on `stream` (NULL = the legacy default stream)
 *    and returns a bwta_status. Argument checks happen on the host before any
 *    launch. Data-dependent conditions (non-finite inputs) are reported by
 *    OR-ing BWTA_STATUS_* flags into *d_status (a device int32, may be NULL);
 *    kernels never trap.
 *  - Pointers to bit planes, scales and outputs must be 16-byte aligned;
 *    fp16/fp32 input matrices must be 16-byte aligned with ld % 8 == 0 (fp16)
 *    or ld % 4 == 0 (fp32).
 */
#ifndef BWTA_H
#define BWTA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *bwta_stream_t; /* the same type as cudaStream_t */

typedef enum bwta_status {
  BWTA_OK = 0,
  BWTA_ERR_INVALID_ARG = 1, /* NULL where a buffer is required, negative size, ld too small */
  BWTA_ERR_UNSUPPORTED = 2, /* an option or size outside what this version implements */
  BWTA_ERR_ALIGNMENT = 3,   /* a pointer or leading dimension breaks the alignment rules */
  BWTA_ERR_CUDA = 4         /* the CUDA runtime reported an error at launch */
} bwta_status;

/* device-side status flags, OR-ed into *d_status */
#define BWTA_STATUS_NONFINITE 0x1 /* an input held Inf or NaN; outputs of that row are unspecified */
#define BWTA_STATUS_TIMEOUT 0x2   /* a bounded wait inside a kernel gave up; outputs are unspecified */
/* After a timeout a kernel lets its own copies and tensor-core operations in
 * flight finish (bounded at 1 s) before it releases tensor memory and exits.
 * This flag says that bound ran out as well: the kernel exited anyway, so work
 * of that launch may still have been running. Treat the CUDA context as
 * unreliable and reset it. */
#define BWTA_STATUS_DRAIN 0x4

#define BWTA_TERNARY 0
#define BWTA_BINARY 1

#define BWTA_MAX_K (1 << 22) /* exactness bound of the integer threshold test */

/* Binarize and pack weights (BWTA abstract: binary weights; scale mean|w|).
 *  W       fp32 [N][ldW] latent weights (read only)
 *  group   0 (one scale per row) or a positive multiple of 128
 *  wbits   uint32 [N][ldw_words] out: sign planes
 *  wscale  fp32 [N][G] out, G = group ? ceil(K/group) : 1; each scale is the
 *          fp64 sum of |w| in ascending column order divided by the count,
 *          rounded once to fp32
 *  Errors: INVALID_ARG, UNSUPPORTED (group), ALIGNMENT; NONFINITE flag. */
int bwta_pack_weights(const float *W, int64_t N, int64_t K, int64_t ldW, int64_t group,
                      uint32_t *wbits, int64_t ldw_words, float *wscale, int32_t *d_status,
                      bwta_stream_t stream);

/* Ternarize (or binarize) and pack activations, one fused pass per row
 * (BWTA abstract: tiny values projected to zero; Figure 6: 32 fp16 -> one word).
 *  X            fp16 bits [M][ldX]
 *  mode         BWTA_TERNARY or BWTA_BINARY (binary: mask all ones for k < K,
 *               scale = mean|x| over the row)
 *  thresh_ratio must be 0.5 (the threshold is thresh_ratio * mean|x|)
 *  mask, sign   uint32 [M][lda_words] out
 *  scale        fp32 [M] out
 *  Errors: INVALID_ARG, UNSUPPORTED (ratio, K > BWTA_MAX_K), ALIGNMENT;
 *  NONFINITE flag. */
int bwta_quantize_pack_acts(const uint16_t *X, int64_t M, int64_t K, int64_t ldX, int mode,
                            float thresh_ratio, uint32_t *mask, uint32_t *sign,
                            int64_t lda_words, float *scale, int32_t *d_status,
                            bwta_stream_t stream);

/* bwta_quantize_pack_acts that can also (or only) write the ternary values as
 * 8-bit floats for the tensor-core GEMM: one E4M3 byte per element, +1 = 0x38,
 * -1 = 0xB8, 0 = 0x00 (same keep/sign decisions, same scale). Byte order is
 * the tensor-core order: within each block of 32 elements (bytes 32b ..
 * 32b+31 of a row), byte 32b + 4k + j (k = 0..7, j = 0..3) holds element
 * 32b + 8j + k. bwta_gemm_tc expands the weight bits into the same order; a
 * dot product does not depend on the order its terms are listed in.
 *  mask, sign     both NULL or both valid (uint32 [M][lda_words])
 *  a_e4m3         uint8 [M][ld_e4m3] out, may be NULL (not together with mask);
 *                 bytes 0 .. 32*lda_words-1 of every row are written, those past
 *                 K as 0; ld_e4m3 >= 32*lda_words, ld_e4m3 % 16 == 0
 *  lda_words      row stride of the planes; also fixes how many E4M3 bytes
 *                 per row are written
 *  Errors: as bwta_quantize_pack_acts. */
int bwta_quantize_pack_acts_ex(const uint16_t *X, int64_t M, int64_t K, int64_t ldX, int mode,
                               float thresh_ratio, uint32_t *mask, uint32_t *sign,
                               int64_t lda_words, uint8_t *a_e4m3, int64_t ld_e4m3, float *scale,
                               int32_t *d_status, bwta_stream_t stream);

/* The same product as bwta_gemm on the tensor cores (tcgen05.mma, 8-bit
 * floating-point operands, fp32 accumulation). Every +-1 x {-1,0,+1} product
 * and partial sum is an integer below 2^24 and therefore exact, so the dots
 * are the same integers and Y follows the same fp32 order (group by group,
 * then the activation scale): the outputs equal bwta_gemm's tiled path bit
 * for bit. The weights stay bit-packed in memory and are expanded to E4M3
 * inside the kernel.
 *  a_e4m3, ld_e4m3  activations from bwta_quantize_pack_acts_ex
 *                   (ld_e4m3 >= 128 * ceil(K/128), % 16 == 0, 16-byte aligned)
 *  a_scale          fp32 [M] (may be NULL when Y is NULL)
 *  other arguments  as bwta_gemm (group 0 or a multiple of 128)
 *  d_status         BWTA_STATUS_TIMEOUT if a bounded barrier wait gave up
 *  Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA. */
int bwta_gemm_tc(const uint8_t *a_e4m3, int64_t ld_e4m3, const float *a_scale, int64_t M,
                 const uint32_t *wbits, const float *wscale, int64_t N, int64_t ldw_words, int64_t K,
                 int64_t group, float *Y, int64_t ldY, int32_t *dots, int64_t ldD,
                 int32_t *d_status, bwta_stream_t stream);

/* Bit-packed GEMM: Y = (s_a * A_ternary) x (alpha * B_binary)^T
 * (BWTA abstract: the bit-packed binary/ternary MatMul for linear layers).
 * Per output (m, n) and weight group g over the words of that group:
 *     d_g = sum popc(mask) - 2 * popc(mask & (a_sign ^ w_sign))
 *     Y[m][n] = fp32: acc = 0; for g ascending: acc = fma((float)d_g, alpha[n][g], acc);
 *               Y = acc * a_scale[m]
 *     dots[m][n] = sum_g d_g  (exact int32)
 * M <= 8 (and K <= 16384) runs the decode GEMV kernel, larger M the tiled
 * GEMM; both follow the serial order above, so Y is the same bit for bit.
 *  a_mask, a_sign  uint32 [M][lda_words]; a_scale fp32 [M]
 *  wbits           uint32 [N][ldw_words]; wscale fp32 [N][G]
 *  Y               fp32 [M][ldY] out, may be NULL
 *  dots            int32 [M][ldD] out, may be NULL (not both NULL); with group > 0
 *                  the full-K dots come from a second, ungrouped pass
 *  d_status        device int32, may be NULL: BWTA_STATUS_TIMEOUT if a bounded
 *                  wait on a shared-memory barrier gave up
 *  Errors: INVALID_ARG, UNSUPPORTED (group, K), ALIGNMENT, CUDA. */
int bwta_gemm(const uint32_t *a_mask, const uint32_t *a_sign, const float *a_scale, int64_t M,
              int64_t lda_words, const uint32_t *wbits, const float *wscale, int64_t N,
              int64_t ldw_words, int64_t K, int64_t group, float *Y, int64_t ldY, int32_t *dots,
              int64_t ldD, int32_t *d_status, bwta_stream_t stream);

/* bwta_gemm with flags. BWTA_GEMM_WEIGHTS_READY promises that `wbits` and
 * `wscale` were complete before this call was enqueued (e.g. packed at load
 * time, then the stream or device was synchronized). The kernels launch with
 * programmatic dependent launch: without the flag they read nothing before
 * the previous kernel in the stream has completed; with it the decode GEMV
 * starts streaming the weights while the previous kernel (typically the
 * activation packer) is still running, and waits only before it reads the
 * activation planes. Passing the flag for weights that a still-running kernel
 * writes is a race. Other flags bits must be 0. */
#define BWTA_GEMM_WEIGHTS_READY 0x1u
int bwta_gemm_ex(const uint32_t *a_mask, const uint32_t *a_sign, const float *a_scale, int64_t M,
                 int64_t lda_words, const uint32_t *wbits, const float *wscale, int64_t N,
                 int64_t ldw_words, int64_t K, int64_t group, float *Y, int64_t ldY,
                 int32_t *dots, int64_t ldD, uint32_t flags, int32_t *d_status,
                 bwta_stream_t stream);

/* Decode linear layer in one kernel: ternarize (or binarize) M <= 8 fp16 rows
 * and multiply them by packed binary weights, without writing the activation
 * planes to memory (BWTA abstract: ternary activations; bit-packed MatMul).
 * Equivalent to bwta_quantize_pack_acts followed by bwta_gemm: the same planes
 * and scales, the same integer dots and the same fp32 outputs, bit for bit.
 *  X          fp16 bits [M][ldX], any alignment
 *  mode, thresh_ratio   as bwta_quantize_pack_acts
 *  wbits, wscale, N, ldw_words, group, Y, ldY, dots, ldD   as bwta_gemm
 *  flags      0 or BWTA_GEMM_WEIGHTS_READY (see bwta_gemm_ex)
 *  Limits: M <= 8, ceil(K/128) <= 128 (K <= 16384); else UNSUPPORTED.
 *  Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA; NONFINITE flag. */
int bwta_linear_decode(const uint16_t *X, int64_t M, int64_t K, int64_t ldX, int mode,
                       float thresh_ratio, const uint32_t *wbits, const float *wscale, int64_t N,
                       int64_t ldw_words, int64_t group, float *Y, int64_t ldY, int32_t *dots,
                       int64_t ldD, uint32_t flags, int32_t *d_status, bwta_stream_t stream);

/* One projection of a batched decode call: the arguments of bwta_linear_decode. */
typedef struct bwta_decode_job {
  const uint16_t *X; /* fp16 bits [M][ldX] */
  int64_t M, K, ldX;
  const uint32_t *wbits; /* [N][ldw_words] */
  const float *wscale;   /* [N][G] */
  int64_t N, ldw_words, group;
  float *Y; /* [M][ldY], may be NULL */
  int64_t ldY;
  int32_t *dots; /* [M][ldD], may be NULL (not both) */
  int64_t ldD;
} bwta_decode_job;

/* Several independent decode projections in ONE launch (BWTA abstract: the
 * bit-packed MatMul, here at decode, where each product streams its weights
 * once and a launch per projection would cost more than the stream itself):
 * e.g. the q/k/v or gate/up projections of one layer, or projections of
 * different layers that do not depend on one another. Every job is computed
 * exactly as bwta_linear_decode computes it alone (same planes, dots and fp32
 * outputs, bit for bit); the jobs must not write overlapping outputs.
 *  jobs       host array of njobs descriptors (read during the call only)
 *  njobs      0 .. 8
 *  mode, thresh_ratio, flags   as bwta_linear_decode, for every job
 *  Limits: per job as bwta_linear_decode; the packed activations of all jobs
 *  (36 bytes per 128 elements per row, rounded to 16 bytes per job) must fit in
 *  48 KB of shared memory; else UNSUPPORTED.
 *  Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA; NONFINITE flag. */
int bwta_linear_decode_batched(const bwta_decode_job *jobs, int64_t njobs, int mode,
                               float thresh_ratio, uint32_t flags, int32_t *d_status,
                               bwta_stream_t stream);

/* Ternary attention scores Q . K^T per batch*head (BWTA abstract: binary /
 * ternary MatMul for the attention operators). Both operands come from
 * bwta_quantize_pack_acts over rows of length D.
 *  q_mask, q_sign [BH*Lq][ld_words], q_scale [BH*Lq]
 *  k_mask, k_sign [BH*Lk][ld_words], k_scale [BH*Lk]
 *  S_i32 int32 [BH][Lq][Lk] out (may be NULL): S = popc(mq & mk) - 2*popc(mq & mk & (sq ^ sk))
 *  S_f32 fp32  [BH][Lq][Lk] out (may be NULL): ((float)S * q_scale) * k_scale
 *  No 1/sqrt(D) and no softmax. Errors: INVALID_ARG, ALIGNMENT, CUDA. */
int bwta_attn_scores(const uint32_t *q_mask, const uint32_t *q_sign, const float *q_scale,
                     const uint32_t *k_mask, const uint32_t *k_sign, const float *k_scale,
                     int64_t BH, int64_t Lq, int64_t Lk, int64_t D, int64_t ld_words,
                     int32_t *S_i32, float *S_f32, bwta_stream_t stream);

/* Attention probabilities as ternary planes, straight from the ternary Q and
 * K planes (BWTA abstract: binary/ternary MatMul for the attention operators;
 * the probabilities are the activations of the A . V product and are
 * ternarized like any activation). Per query row i of each batch*head, over
 * the Lk keys j:
 *   x_ij = (((float)S_ij * q_scale_i) * k_scale_j) * softmax_scale   (S as in
 *          bwta_attn_scores; the score before the factor is the fp32 value that
 *          bwta_attn_scores writes)
 *   p_ij = e_ij / Z_i, e_ij = exp(x_ij - max_j x) (fp32), Z_i = sum_j e_ij (fp64)
 *   kept iff p_ij > 0.5 * mean_j p_ij, where the mean of a softmax row is
 *   exactly 1/Lk, so kept iff p_ij > 1/(2 Lk); every p is positive, so a kept
 *   value is +1 and the sign plane is all zero; p_scale_i = mean of the kept p.
 * The Lq x Lk scores are never written to memory. The sums, the kept decision
 * (e_ij > Z_i / (2 Lk)) and the scale are taken in fp64, so they do not depend
 * on the order of the sums; exp is the fp32 library function, so a probability
 * within about 1e-6 (relative) of 1/(2 Lk) can fall either way.
 *  q_*, k_*, BH, Lq, Lk, D, ld_words   as bwta_attn_scores (ld_words <= 32)
 *  p_mask, p_sign  uint32 [BH*Lq][ldp_words] out (ldp_words >= ceil(Lk/32),
 *                  % 4 == 0; padding words written as zero)
 *  p_scale         fp32 [BH*Lq] out
 *  Limits: Lk * (32 * ceil(ld_words/4) + 36) bytes <= 200 KB (shared memory).
 *  Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA. */
int bwta_attn_softmax_ternarize(const uint32_t *q_mask, const uint32_t *q_sign,
                                const float *q_scale, const uint32_t *k_mask,
                                const uint32_t *k_sign, const float *k_scale, int64_t BH,
                                int64_t Lq, int64_t Lk, int64_t D, int64_t ld_words,
                                float softmax_scale, uint32_t *p_mask, uint32_t *p_sign,
                                int64_t ldp_words, float *p_scale, bwta_stream_t stream);

/* The A . V product of attention with ternary operands (BWTA abstract:
 * binary/ternary MatMul for the attention operators): the ternary
 * probabilities from bwta_attn_softmax_ternarize times V, ternarized per
 * output channel over the sequence (bwta_quantize_pack_acts on the rows of
 * V^T, so that each channel's scale factors out of the sum over keys):
 *   O_i32[h][i][d] = sum_j p_ij * v_dj   (p in {0, 1}, v in {-1, 0, 1})
 *   O_f32[h][i][d] = ((float)O_i32 * p_scale[h][i]) * v_scale[h][d]
 *  p_mask, p_sign, p_scale   [BH*Lq][ld_words], [BH*Lq]
 *  vt_mask, vt_sign, vt_scale [BH*D][ld_words], [BH*D]: row d of head h is
 *                  channel d of V over the Lk keys
 *  ld_words        >= ceil(Lk/32), % 4 == 0, the same for both sides
 *  O_i32, O_f32    [BH][Lq][D] out, either may be NULL (not both)
 *  Errors: INVALID_ARG, UNSUPPORTED (ld_words > 32), ALIGNMENT, CUDA. */
int bwta_attn_av(const uint32_t *p_mask, const uint32_t *p_sign, const float *p_scale,
                 const uint32_t *vt_mask, const uint32_t *vt_sign, const float *vt_scale,
                 int64_t BH, int64_t Lq, int64_t D, int64_t Lk, int64_t ld_words, int32_t *O_i32,
                 float *O_f32, bwta_stream_t stream);

/* BiLLM packed weights (BiLLM "Approach" and "Limitations"). Per block j of
 * `block` = 128 columns and row n:
 *  sign   uint32 [N][ldw_words]  1 = negative (b for non-salient, b1 for salient)
 *  gmap   uint32 [N][ldw_words]  1 = sparse group (0 at salient columns)
 *  res    uint8  [N][K/block]    bit i: 1 = b2 of salient column sal[j][i] negative
 *  sal    uint8  [K/block][n_sal] salient columns of block j, ascending
 *  bscale fp32   [N][K/block][4] (alpha_c, alpha_sp, alpha1, alpha2)
 * Dequantized weight: alpha_c*b (concentrated), alpha_sp*b (sparse),
 * alpha1*b1 + alpha2*b2 (salient). */
typedef struct billm_weights {
  const uint32_t *sign;
  const uint32_t *gmap;
  const uint8_t *res;
  const uint8_t *sal;
  const float *bscale;
  int64_t N, K, ldw_words, block, n_sal;
} billm_weights;

/* Build the BiLLM packed weights from latent fp32 weights on the GPU.
 *  Salient columns: per block, the n_sal columns with the largest sum_n w^2
 *  (fp64, rows ascending; the Hessian of the pages' metric taken as the
 *  identity, as no calibration data is used); ties go to the lower column.
 *  Salient weights: alpha1 = mean|w|, b1 = sign(w), r = w - alpha1*b1,
 *  alpha2 = mean|r|, b2 = sign(r). Other weights: a break-point p per row
 *  and block, the sparse group is |w| > p; split selects p:
 *    0  no split (every non-salient weight is concentrated)
 *    1  p = 0.5*max|w| over the row's non-salient weights in the block
 *    2  the searched break-point (BiLLM abstract: "optimal splitting search"):
 *       the non-salient magnitude of the row-block whose split minimizes the
 *       squared binarization error sum (|w| - alpha_group)^2 of both groups,
 *       evaluated in fp64 in ascending column order; ties go to the smaller p
 *  alpha = mean|w| per group (0 if empty). Every mean is an fp64 sum in
 *  ascending column order divided by the count and rounded once to fp32.
 *  W fp32 [N][ldW]; out: the buffers of `out` (cast away const; device memory).
 *  block must be 128; 0 <= n_sal <= 8; K % 128 == 0.
 *  Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA; NONFINITE flag. */
int billm_pack_weights(const float *W, int64_t ldW, int split, const billm_weights *out,
                       int32_t *d_status, bwta_stream_t stream);

/* BiLLM-format GEMM (BiLLM abstract and "Approach": salient columns with a
 * residual plane, non-salient weights in two groups with their own scales):
 * Y[m][n] = sum_k x[m][k] * what[n][k], the same real value as the per-block form
 *   alpha_c*sum_C b x + alpha_sp*sum_S b x + alpha1*sum_sal b1 x + alpha2*sum_sal b2 x.
 *  M <= 8: CUDA cores, one 128-column block at a time (fp32 sums per block,
 *  folded into Y per block). M > 8 with X 16-byte aligned and ldX % 8 == 0:
 *  tensor cores; each weight is rebuilt as what * 2^E (E per weight row)
 *  split into fp16 hi + lo, and X*hi + X*lo accumulates in fp32 over all of
 *  K. Other M > 8: CUDA cores as for M <= 8.
 *  Accuracy: fp32 sums, so the error is not bounded by a fixed fraction of
 *  sum_k |x_k what_k| in the worst case (about K * 2^-24 of it for the
 *  tensor-core path, 128 * 2^-24 per block for the CUDA-core paths); measured
 *  on the tested workloads (normal and Laplace data, K <= 8192) it stays below
 *  1e-5 * sum_k |x_k what_k|, which the tests require of every output.
 *  X   fp16 bits [M][ldX]
 *  W   host pointer to a billm_weights whose buffers are device memory
 *  Y   fp32 [M][ldY] out
 *  Errors: INVALID_ARG, UNSUPPORTED (K > 40960), ALIGNMENT, CUDA; NONFINITE and
 *  TIMEOUT flags. */
int billm_gemm(const uint16_t *X, int64_t M, int64_t ldX, const billm_weights *W, float *Y,
               int64_t ldY, int32_t *d_status, bwta_stream_t stream);

/* Failure-path self-test of the bounded waits. The paper has no counterpart:
 * this exercises the library's own error handling. It runs the tiled kernel of
 * bwta_gemm (arguments as there; M must be > 8) with one extra wait per CTA, on
 * a shared-memory barrier that nothing ever completes, bounded by
 * wait_limit_ns. Every CTA then takes the kernel's timeout path: it ORs
 * BWTA_STATUS_TIMEOUT into *d_status, lets the tile loads it issued land, and
 * returns. Y and dots are left unspecified. No fault is raised and the context
 * stays usable: later calls compute normally.
 *  wait_limit_ns  1 .. 2000000000
 *  d_status       required (device int32)
 *  Errors: as bwta_gemm; INVALID_ARG if M <= 8, d_status is NULL or the limit
 *  is out of range. */
int bwta_selftest_gemm_timeout(const uint32_t *a_mask, const uint32_t *a_sign,
                               const float *a_scale, int64_t M, int64_t lda_words,
                               const uint32_t *wbits, const float *wscale, int64_t N,
                               int64_t ldw_words, int64_t K, int64_t group, float *Y, int64_t ldY,
                               int32_t *dots, int64_t ldD, int64_t wait_limit_ns,
                               int32_t *d_status, bwta_stream_t stream);

/* Library version string, e.g. "bwta 0.1 sm_100a". */
const char *bwta_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BWTA_H */
