// abi.cu -- the extern "C" entry points of libbwta.so (declared in
// include/bwta.h): argument validation on the host, then one or two kernel
// launches on the caller's stream. Nothing here allocates memory.
#include <cuda_fp16.h>

#include "common.cuh"

using namespace bwta;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? BWTA_OK : BWTA_ERR_CUDA; }

int64_t words_for(int64_t K) { return (K + 31) / 32; }

int check_plane(const void *p, int64_t rows, int64_t ld, int64_t K) {
  if (rows > 0 && !p) return BWTA_ERR_INVALID_ARG;
  if (ld < words_for(K)) return BWTA_ERR_INVALID_ARG;
  if (ld % 4 != 0 || !aligned16(p)) return BWTA_ERR_ALIGNMENT;
  return BWTA_OK;
}

int check_group(int64_t group) {
  if (group < 0) return BWTA_ERR_INVALID_ARG;
  if (group != 0 && group % 128 != 0) return BWTA_ERR_UNSUPPORTED;
  return BWTA_OK;
}

}  // namespace

extern "C" {

const char *bwta_version(void) { return "bwta 0.1 sm_100a"; }

int bwta_pack_weights(const float *W, int64_t N, int64_t K, int64_t ldW, int64_t group,
                      uint32_t *wbits, int64_t ldw_words, float *wscale, int32_t *d_status,
                      bwta_stream_t stream) {
  if (N < 0 || K <= 0 || ldW < K) return BWTA_ERR_INVALID_ARG;
  if (int r = check_group(group)) return r;
  if (N > 0 && (!W || !wscale)) return BWTA_ERR_INVALID_ARG;
  if (int r = check_plane(wbits, N, ldw_words, K)) return r;
  return cuda_status(launch_pack_weights(W, N, K, ldW, group, wbits, ldw_words, wscale, d_status,
                                         (cudaStream_t)stream));
}

int bwta_quantize_pack_acts(const uint16_t *X, int64_t M, int64_t K, int64_t ldX, int mode,
                            float thresh_ratio, uint32_t *mask, uint32_t *sign,
                            int64_t lda_words, float *scale, int32_t *d_status,
                            bwta_stream_t stream) {
  if (M < 0 || K <= 0 || ldX < K) return BWTA_ERR_INVALID_ARG;
  if (mode != BWTA_TERNARY && mode != BWTA_BINARY) return BWTA_ERR_INVALID_ARG;
  if (thresh_ratio != 0.5f || K > BWTA_MAX_K) return BWTA_ERR_UNSUPPORTED;
  if (M > 0 && (!X || !scale)) return BWTA_ERR_INVALID_ARG;
  if (int r = check_plane(mask, M, lda_words, K)) return r;
  if (int r = check_plane(sign, M, lda_words, K)) return r;
  return cuda_status(launch_quantize_pack_acts(X, M, K, ldX, mode, mask, sign, lda_words, scale,
                                               nullptr, 0, d_status, (cudaStream_t)stream));
}

int bwta_quantize_pack_acts_ex(const uint16_t *X, int64_t M, int64_t K, int64_t ldX, int mode,
                               float thresh_ratio, uint32_t *mask, uint32_t *sign,
                               int64_t lda_words, uint8_t *a_e4m3, int64_t ld_e4m3, float *scale,
                               int32_t *d_status, bwta_stream_t stream) {
  if (M < 0 || K <= 0 || ldX < K) return BWTA_ERR_INVALID_ARG;
  if (mode != BWTA_TERNARY && mode != BWTA_BINARY) return BWTA_ERR_INVALID_ARG;
  if (thresh_ratio != 0.5f || K > BWTA_MAX_K) return BWTA_ERR_UNSUPPORTED;
  if (M > 0 && (!X || !scale)) return BWTA_ERR_INVALID_ARG;
  if ((mask == nullptr) != (sign == nullptr)) return BWTA_ERR_INVALID_ARG;
  if (!mask && !a_e4m3) return BWTA_ERR_INVALID_ARG;
  if (lda_words < words_for(K)) return BWTA_ERR_INVALID_ARG;
  if (lda_words % 4 != 0) return BWTA_ERR_ALIGNMENT;
  if (mask) {
    if (int r = check_plane(mask, M, lda_words, K)) return r;
    if (int r = check_plane(sign, M, lda_words, K)) return r;
  }
  if (a_e4m3) {
    if (ld_e4m3 < lda_words * 32) return BWTA_ERR_INVALID_ARG;
    if (ld_e4m3 % 16 != 0 || !aligned16(a_e4m3)) return BWTA_ERR_ALIGNMENT;
  }
  return cuda_status(launch_quantize_pack_acts(X, M, K, ldX, mode, mask, sign, lda_words, scale,
                                               a_e4m3, ld_e4m3, d_status, (cudaStream_t)stream));
}

int bwta_gemm_tc(const uint8_t *a_e4m3, int64_t ld_e4m3, const float *a_scale, int64_t M,
                 const uint32_t *wbits, const float *wscale, int64_t N, int64_t ldw_words, int64_t K,
                 int64_t group, float *Y, int64_t ldY, int32_t *dots, int64_t ldD,
                 int32_t *d_status, bwta_stream_t stream) {
  if (M < 0 || N < 0 || K <= 0) return BWTA_ERR_INVALID_ARG;
  if (K > BWTA_MAX_K) return BWTA_ERR_UNSUPPORTED;
  if (int r = check_group(group)) return r;
  if (!Y && !dots) return BWTA_ERR_INVALID_ARG;
  if (Y && ldY < N) return BWTA_ERR_INVALID_ARG;
  if (dots && ldD < N) return BWTA_ERR_INVALID_ARG;
  if (M > 0 && Y && !a_scale) return BWTA_ERR_INVALID_ARG;
  if (N > 0 && !wscale) return BWTA_ERR_INVALID_ARG;
  if (M > 0 && !a_e4m3) return BWTA_ERR_INVALID_ARG;
  if (ld_e4m3 < ((K + 127) / 128) * 128) return BWTA_ERR_INVALID_ARG;
  if (ld_e4m3 % 16 != 0 || !aligned16(a_e4m3)) return BWTA_ERR_ALIGNMENT;
  if (int r = check_plane(wbits, N, ldw_words, K)) return r;
  if (M == 0 || N == 0) return BWTA_OK;
  return cuda_status(launch_gemm_tc(a_e4m3, ld_e4m3, a_scale, M, wbits, wscale, N, ldw_words, K,
                                    group, Y, ldY, dots, ldD, d_status, (cudaStream_t)stream));
}

int bwta_gemm(const uint32_t *a_mask, const uint32_t *a_sign, const float *a_scale, int64_t M,
              int64_t lda_words, const uint32_t *wbits, const float *wscale, int64_t N,
              int64_t ldw_words, int64_t K, int64_t group, float *Y, int64_t ldY, int32_t *dots,
              int64_t ldD, int32_t *d_status, bwta_stream_t stream) {
  return bwta_gemm_ex(a_mask, a_sign, a_scale, M, lda_words, wbits, wscale, N, ldw_words, K, group,
                      Y, ldY, dots, ldD, 0u, d_status, stream);
}

int bwta_gemm_ex(const uint32_t *a_mask, const uint32_t *a_sign, const float *a_scale, int64_t M,
                 int64_t lda_words, const uint32_t *wbits, const float *wscale, int64_t N,
                 int64_t ldw_words, int64_t K, int64_t group, float *Y, int64_t ldY,
                 int32_t *dots, int64_t ldD, uint32_t flags, int32_t *d_status,
                 bwta_stream_t stream) {
  if (flags & ~BWTA_GEMM_WEIGHTS_READY) return BWTA_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K <= 0) return BWTA_ERR_INVALID_ARG;
  if (K > BWTA_MAX_K) return BWTA_ERR_UNSUPPORTED;
  if (int r = check_group(group)) return r;
  if (!Y && !dots) return BWTA_ERR_INVALID_ARG;
  if (Y && ldY < N) return BWTA_ERR_INVALID_ARG;
  if (dots && ldD < N) return BWTA_ERR_INVALID_ARG;
  if (M > 0 && !a_scale) return BWTA_ERR_INVALID_ARG;
  if (N > 0 && !wscale) return BWTA_ERR_INVALID_ARG;
  if (int r = check_plane(a_mask, M, lda_words, K)) return r;
  if (int r = check_plane(a_sign, M, lda_words, K)) return r;
  if (int r = check_plane(wbits, N, ldw_words, K)) return r;
  if (M == 0 || N == 0) return BWTA_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (decode_fits(M, K)) {
    DecodeSpec job = {};
    job.am = a_mask;
    job.as = a_sign;
    job.ascale = a_scale;
    job.lda = lda_words;
    job.M = M;
    job.K = K;
    job.wbits = wbits;
    job.wscale = wscale;
    job.N = N;
    job.ldw = ldw_words;
    job.group = group;
    job.Y = Y;
    job.ldY = ldY;
    job.dots = dots;
    job.ldD = ldD;
    return cuda_status(launch_decode(&job, 1, false, BWTA_TERNARY,
                                     (flags & BWTA_GEMM_WEIGHTS_READY) != 0, d_status, s));
  }
  return cuda_status(launch_gemm_tiled(a_mask, a_sign, a_scale, M, lda_words, wbits, wscale, N,
                                       ldw_words, K, group, Y, ldY, dots, ldD, d_status, 0, s));
}

int bwta_selftest_gemm_timeout(const uint32_t *a_mask, const uint32_t *a_sign,
                               const float *a_scale, int64_t M, int64_t lda_words,
                               const uint32_t *wbits, const float *wscale, int64_t N,
                               int64_t ldw_words, int64_t K, int64_t group, float *Y, int64_t ldY,
                               int32_t *dots, int64_t ldD, int64_t wait_limit_ns,
                               int32_t *d_status, bwta_stream_t stream) {
  if (!d_status || M <= 8 || wait_limit_ns < 1 || wait_limit_ns > 2000000000LL)
    return BWTA_ERR_INVALID_ARG;
  if (N < 0 || K <= 0) return BWTA_ERR_INVALID_ARG;
  if (K > BWTA_MAX_K) return BWTA_ERR_UNSUPPORTED;
  if (int r = check_group(group)) return r;
  if (!Y && !dots) return BWTA_ERR_INVALID_ARG;
  if (Y && ldY < N) return BWTA_ERR_INVALID_ARG;
  if (dots && ldD < N) return BWTA_ERR_INVALID_ARG;
  if (!a_scale || (N > 0 && !wscale)) return BWTA_ERR_INVALID_ARG;
  if (int r = check_plane(a_mask, M, lda_words, K)) return r;
  if (int r = check_plane(a_sign, M, lda_words, K)) return r;
  if (int r = check_plane(wbits, N, ldw_words, K)) return r;
  if (N == 0) return BWTA_OK;
  return cuda_status(launch_gemm_tiled(a_mask, a_sign, a_scale, M, lda_words, wbits, wscale, N,
                                       ldw_words, K, group, Y, ldY, dots, ldD, d_status,
                                       (uint64_t)wait_limit_ns, (cudaStream_t)stream));
}

// Validation shared by the single and the batched fused decode.
static int check_decode_job(const bwta_decode_job &J) {
  if (J.M < 0 || J.N < 0 || J.K <= 0 || J.ldX < J.K) return BWTA_ERR_INVALID_ARG;
  if (J.M > 8 || !decode_fits(J.M > 0 ? J.M : 1, J.K)) return BWTA_ERR_UNSUPPORTED;
  if (int r = check_group(J.group)) return r;
  if (J.M > 0 && J.N > 0 && !J.Y && !J.dots) return BWTA_ERR_INVALID_ARG;
  if (J.Y && J.ldY < J.N) return BWTA_ERR_INVALID_ARG;
  if (J.dots && J.ldD < J.N) return BWTA_ERR_INVALID_ARG;
  if (J.M > 0 && !J.X) return BWTA_ERR_INVALID_ARG;
  if (J.N > 0 && !J.wscale) return BWTA_ERR_INVALID_ARG;
  if (int r = check_plane(J.wbits, J.N, J.ldw_words, J.K)) return r;
  return BWTA_OK;
}

static DecodeSpec fused_spec(const bwta_decode_job &J) {
  DecodeSpec d = {};
  d.X = J.X;
  d.ldX = J.ldX;
  d.M = J.M;
  d.K = J.K;
  d.wbits = J.wbits;
  d.wscale = J.wscale;
  d.N = J.N;
  d.ldw = J.ldw_words;
  d.group = J.group;
  d.Y = J.Y;
  d.ldY = J.ldY;
  d.dots = J.dots;
  d.ldD = J.ldD;
  return d;
}

int bwta_linear_decode(const uint16_t *X, int64_t M, int64_t K, int64_t ldX, int mode,
                       float thresh_ratio, const uint32_t *wbits, const float *wscale, int64_t N,
                       int64_t ldw_words, int64_t group, float *Y, int64_t ldY, int32_t *dots,
                       int64_t ldD, uint32_t flags, int32_t *d_status, bwta_stream_t stream) {
  const bwta_decode_job J = {X, M, K, ldX, wbits, wscale, N, ldw_words, group, Y, ldY, dots, ldD};
  return bwta_linear_decode_batched(&J, 1, mode, thresh_ratio, flags, d_status, stream);
}

int bwta_linear_decode_batched(const bwta_decode_job *jobs, int64_t njobs, int mode,
                               float thresh_ratio, uint32_t flags, int32_t *d_status,
                               bwta_stream_t stream) {
  if (flags & ~BWTA_GEMM_WEIGHTS_READY) return BWTA_ERR_INVALID_ARG;
  if (njobs < 0 || (njobs > 0 && !jobs)) return BWTA_ERR_INVALID_ARG;
  if (njobs > decode_max_jobs()) return BWTA_ERR_UNSUPPORTED;
  if (mode != BWTA_TERNARY && mode != BWTA_BINARY) return BWTA_ERR_INVALID_ARG;
  if (thresh_ratio != 0.5f) return BWTA_ERR_UNSUPPORTED;
  DecodeSpec spec[8];
  size_t act = 0;
  int n = 0;
  for (int64_t i = 0; i < njobs; ++i) {
    if (int r = check_decode_job(jobs[i])) return r;
    if (jobs[i].M == 0 || jobs[i].N == 0) continue;
    act += decode_act_bytes(jobs[i].M, jobs[i].K);
    spec[n++] = fused_spec(jobs[i]);
  }
  if (act > decode_max_act_bytes()) return BWTA_ERR_UNSUPPORTED;
  if (n == 0) return BWTA_OK;
  return cuda_status(launch_decode(spec, n, true, mode, (flags & BWTA_GEMM_WEIGHTS_READY) != 0,
                                   d_status, (cudaStream_t)stream));
}

int bwta_attn_scores(const uint32_t *q_mask, const uint32_t *q_sign, const float *q_scale,
                     const uint32_t *k_mask, const uint32_t *k_sign, const float *k_scale,
                     int64_t BH, int64_t Lq, int64_t Lk, int64_t D, int64_t ld_words,
                     int32_t *S_i32, float *S_f32, bwta_stream_t stream) {
  if (BH < 0 || Lq < 0 || Lk < 0 || D <= 0) return BWTA_ERR_INVALID_ARG;
  if (!S_i32 && !S_f32) return BWTA_ERR_INVALID_ARG;
  if (ld_words > 32) return BWTA_ERR_UNSUPPORTED;
  if (int r = check_plane(q_mask, BH * Lq, ld_words, D)) return r;
  if (int r = check_plane(q_sign, BH * Lq, ld_words, D)) return r;
  if (int r = check_plane(k_mask, BH * Lk, ld_words, D)) return r;
  if (int r = check_plane(k_sign, BH * Lk, ld_words, D)) return r;
  if (S_f32 && BH * Lq > 0 && !q_scale) return BWTA_ERR_INVALID_ARG;
  if (S_f32 && BH * Lk > 0 && !k_scale) return BWTA_ERR_INVALID_ARG;
  if ((S_i32 && !aligned16(S_i32)) || (S_f32 && !aligned16(S_f32))) return BWTA_ERR_ALIGNMENT;
  return cuda_status(launch_attn_scores(q_mask, q_sign, q_scale, k_mask, k_sign, k_scale, BH, Lq,
                                        Lk, D, ld_words, S_i32, S_f32, (cudaStream_t)stream));
}

int bwta_attn_softmax_ternarize(const uint32_t *q_mask, const uint32_t *q_sign,
                                const float *q_scale, const uint32_t *k_mask,
                                const uint32_t *k_sign, const float *k_scale, int64_t BH,
                                int64_t Lq, int64_t Lk, int64_t D, int64_t ld_words,
                                float softmax_scale, uint32_t *p_mask, uint32_t *p_sign,
                                int64_t ldp_words, float *p_scale, bwta_stream_t stream) {
  if (BH < 0 || Lq < 0 || Lk <= 0 || D <= 0) return BWTA_ERR_INVALID_ARG;
  if (ld_words > 32 || !(softmax_scale == softmax_scale)) return BWTA_ERR_UNSUPPORTED;
  if (attn_softmax_smem(Lk, ld_words) > 200 * 1024) return BWTA_ERR_UNSUPPORTED;
  if (int r = check_plane(q_mask, BH * Lq, ld_words, D)) return r;
  if (int r = check_plane(q_sign, BH * Lq, ld_words, D)) return r;
  if (int r = check_plane(k_mask, BH * Lk, ld_words, D)) return r;
  if (int r = check_plane(k_sign, BH * Lk, ld_words, D)) return r;
  if (int r = check_plane(p_mask, BH * Lq, ldp_words, Lk)) return r;
  if (int r = check_plane(p_sign, BH * Lq, ldp_words, Lk)) return r;
  if (BH * Lq > 0 && (!q_scale || !p_scale)) return BWTA_ERR_INVALID_ARG;
  if (BH > 0 && !k_scale) return BWTA_ERR_INVALID_ARG;
  return cuda_status(launch_attn_softmax(q_mask, q_sign, q_scale, k_mask, k_sign, k_scale, BH, Lq,
                                         Lk, D, ld_words, softmax_scale, p_mask, p_sign, ldp_words,
                                         p_scale, (cudaStream_t)stream));
}

int bwta_attn_av(const uint32_t *p_mask, const uint32_t *p_sign, const float *p_scale,
                 const uint32_t *vt_mask, const uint32_t *vt_sign, const float *vt_scale,
                 int64_t BH, int64_t Lq, int64_t D, int64_t Lk, int64_t ld_words, int32_t *O_i32,
                 float *O_f32, bwta_stream_t stream) {
  // the ternary x ternary product of bwta_attn_scores with the probabilities
  // as the query side and the channels of V as the key side
  return bwta_attn_scores(p_mask, p_sign, p_scale, vt_mask, vt_sign, vt_scale, BH, Lq, D, Lk,
                          ld_words, O_i32, O_f32, stream);
}

static int check_billm(const billm_weights *W) {
  if (!W) return BWTA_ERR_INVALID_ARG;
  if (W->N < 0 || W->K <= 0) return BWTA_ERR_INVALID_ARG;
  if (W->block != 128 || W->K % 128 != 0 || W->n_sal < 0 || W->n_sal > 8)
    return BWTA_ERR_UNSUPPORTED;
  if (W->N > 0 && (!W->res || !W->bscale)) return BWTA_ERR_INVALID_ARG;
  if (W->n_sal > 0 && !W->sal) return BWTA_ERR_INVALID_ARG;
  if (int r = check_plane(W->sign, W->N, W->ldw_words, W->K)) return r;
  if (int r = check_plane(W->gmap, W->N, W->ldw_words, W->K)) return r;
  if (!aligned16(W->bscale)) return BWTA_ERR_ALIGNMENT;
  return BWTA_OK;
}

int billm_pack_weights(const float *W, int64_t ldW, int split, const billm_weights *out,
                       int32_t *d_status, bwta_stream_t stream) {
  if (int r = check_billm(out)) return r;
  if (ldW < out->K || (out->N > 0 && !W)) return BWTA_ERR_INVALID_ARG;
  if (split < 0 || split > 2) return BWTA_ERR_INVALID_ARG;
  if (out->N > 0 && (out->n_sal == 0 ? false : !out->sal)) return BWTA_ERR_INVALID_ARG;
  return cuda_status(launch_billm_pack(W, ldW, split, out, d_status, (cudaStream_t)stream));
}

int billm_gemm(const uint16_t *X, int64_t M, int64_t ldX, const billm_weights *W, float *Y,
               int64_t ldY, int32_t *d_status, bwta_stream_t stream) {
  if (int r = check_billm(W)) return r;
  if (M < 0 || ldX < W->K || ldY < W->N) return BWTA_ERR_INVALID_ARG;
  if (M > 0 && (!X || !Y)) return BWTA_ERR_INVALID_ARG;
  if (W->K > 40960) return BWTA_ERR_UNSUPPORTED;
  return cuda_status(launch_billm_gemm(X, M, ldX, W, Y, ldY, d_status, (cudaStream_t)stream));
}

}  // extern "C"
