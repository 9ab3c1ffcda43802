// common.cuh -- device helpers and internal launch declarations of libbwta.
// Everything here is private to the library; the public surface is include/bwta.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bwta.h"

namespace bwta {

constexpr unsigned FULL = 0xffffffffu;

// ----------------------------------------------------------------- status
__device__ __forceinline__ void flag_status(int32_t *d_status, int32_t flag) {
  if (d_status) atomicOr(d_status, flag);
}

// ------------------------------------------------------------ fp16 magnitudes
// |x| of a 15-bit fp16 magnitude pattern in units of 2^-24 (exact integer < 2^40).
__device__ __forceinline__ uint64_t mag_units(uint32_t hm) {
  uint32_t e = hm >> 10, f = hm & 1023u;
  return e ? ((uint64_t)(1024u | f) << (e - 1u)) : (uint64_t)f;
}

// Largest 15-bit magnitude pattern h with mag_units(h) <= T. Because
// mag_units is strictly increasing over finite patterns, v > T <=> h > result.
__device__ __forceinline__ uint32_t mag_threshold_pattern(uint64_t T) {
  if (T < 2048u) return (uint32_t)T;            // exponent field 0 or 1: v == h
  int p = 63 - __clzll((long long)T);           // floor(log2 T) >= 11
  int e = p - 9;                                // top bit of (1024|f) << (e-1) is e+9
  if (e >= 31) return 0x7BFFu;
  uint32_t f = (uint32_t)(T >> (e - 1)) - 1024u;
  return ((uint32_t)e << 10) | f;
}

// ------------------------------------------------------------ small helpers
__device__ __forceinline__ uint32_t lop3_and_xor(uint32_t m, uint32_t a, uint32_t b) {
  // m & (a ^ b) as a single LOP3: with the operand patterns m = 0xF0,
  // a = 0xCC, b = 0xAA the truth table is 0xF0 & (0xCC ^ 0xAA) = 0x60
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x60;" : "=r"(r) : "r"(m), "r"(a), "r"(b));
  return r;
}

// (float)d for |d| < 2^22 via the 1.5*2^23 bias trick: exact, and it keeps
// the conversion off the int->float conversion unit. `biased` = d + 0x4B400000.
__device__ __forceinline__ float biased_int_to_float(int32_t biased) {
  return __int_as_float(biased) - 12582912.0f;
}
constexpr int32_t INT_FLOAT_BIAS = 0x4B400000;

template <typename T>
__host__ __device__ __forceinline__ T ceil_div(T a, T b) {
  return (a + b - 1) / b;
}

// ------------------------------------------------------------ launchers
// Every launcher is called after host-side validation in abi.cu and returns
// the launch's cudaError_t.
cudaError_t launch_pack_weights(const float *W, int64_t N, int64_t K, int64_t ldW, int64_t group,
                                uint32_t *wbits, int64_t ldw, float *wscale, int32_t *d_status,
                                cudaStream_t s);
cudaError_t launch_quantize_pack_acts(const uint16_t *X, int64_t M, int64_t K, int64_t ldX,
                                      int mode, uint32_t *mask, uint32_t *sign, int64_t lda,
                                      float *scale, int32_t *d_status, cudaStream_t s);
cudaError_t launch_gemm_tiled(const uint32_t *am, const uint32_t *as, const float *ascale,
                              int64_t M, int64_t lda, const uint32_t *wb, const float *wscale,
                              int64_t N, int64_t ldw, int64_t K, int64_t group, float *Y,
                              int64_t ldY, int32_t *dots, int64_t ldD, int32_t *d_status,
                              cudaStream_t s);
cudaError_t launch_gemv(const uint32_t *am, const uint32_t *as, const float *ascale, int64_t M,
                        int64_t lda, const uint32_t *wb, const float *wscale, int64_t N,
                        int64_t ldw, int64_t K, int64_t group, float *Y, int64_t ldY,
                        int32_t *dots, int64_t ldD, cudaStream_t s);
bool gemv_fits(int64_t M, int64_t lda, int64_t K, int64_t group);
cudaError_t launch_attn_scores(const uint32_t *qm, const uint32_t *qs, const float *qscale,
                               const uint32_t *km, const uint32_t *ks, const float *kscale,
                               int64_t BH, int64_t Lq, int64_t Lk, int64_t ld, int32_t *Si,
                               float *Sf, cudaStream_t s);
cudaError_t launch_billm_pack(const float *W, int64_t ldW, int split, const billm_weights *out,
                              int32_t *d_status, cudaStream_t s);
cudaError_t launch_billm_gemm(const uint16_t *X, int64_t M, int64_t ldX, const billm_weights *W,
                              float *Y, int64_t ldY, int32_t *d_status, cudaStream_t s);

}  // namespace bwta
