// common.cuh -- device helpers and internal launch declarations of libbwta.
// Everything here is private to the library; the public surface is include/bwta.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#ifndef __CUDACC_RTC__
#include <atomic>
#endif

#include "../../include/bwta.h"

namespace bwta {

constexpr unsigned FULL = 0xffffffffu;

// Bound of the waits that let a CTA's own copies and MMAs finish after one of
// its barrier waits timed out (the normal waits are bounded at 2 s).
constexpr uint64_t DRAIN_NS = 1000000000ull;

#ifndef __CUDACC_RTC__
// The >48 KB dynamic shared-memory opt-in of one kernel, made once per device
// (the device current at the call). Only a success is remembered, so a call
// that failed is retried on the next launch. With max_carveout the kernel also
// asks for the largest shared-memory carveout, so that an SM running one of
// its CTAs keeps room for a CTA of the next kernel in the stream (left to
// itself the driver may size the carveout for this kernel's CTA alone).
class SmemOptIn {
 public:
  template <typename Kern>
  cudaError_t operator()(Kern *kern, int bytes, bool max_carveout = false) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cached = dev >= 0 && dev < kDevices;
    if (cached && set_[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && max_carveout)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess && cached) set_[dev].store(bytes, std::memory_order_release);
    return e;
  }

 private:
  static constexpr int kDevices = 64;
  std::atomic<int> set_[kDevices] = {};
};
#endif

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

// Full adder on 32 bit positions at once: per bit, a + b + c = sum + 2*carry.
__device__ __forceinline__ uint32_t xor3(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;  // 0xF0 ^ 0xCC ^ 0xAA = 0x96
  asm("lop3.b32 %0, %1, %2, %3, 0x96;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
__device__ __forceinline__ uint32_t maj3(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;  // majority of (0xF0, 0xCC, 0xAA) = 0xE8
  asm("lop3.b32 %0, %1, %2, %3, 0xE8;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// popc(t0) + popc(t1) + popc(t2) + popc(t3) with three POPCs: a carry-save
// full adder folds t0, t1, t2 into a sum plane (weight 1) and a carry plane
// (weight 2). Four words take at least three POPCs (0..4 per bit needs three
// bit planes); the two extra LOP3s run on the ALU pipe, which has 4x the
// POPC pipe's throughput.
__device__ __forceinline__ int popc4_csa(uint32_t t0, uint32_t t1, uint32_t t2, uint32_t t3) {
  return __popc(xor3(t0, t1, t2)) + __popc(t3) + 2 * __popc(maj3(t0, t1, t2));
}

// (float)d for |d| < 2^22 via the 1.5*2^23 bias trick: exact, and it keeps
// the conversion off the int->float conversion unit. `biased` = d + 0x4B400000.
__device__ __forceinline__ float biased_int_to_float(int32_t biased) {
  return __int_as_float(biased) - 12582912.0f;
}
constexpr int32_t INT_FLOAT_BIAS = 0x4B400000;

// Programmatic dependent launch. Every kernel lets the next kernel in the
// stream be scheduled as soon as all of its own blocks are running, and waits
// for the previous kernel's completion (and memory) before it reads any global
// input. Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

#ifndef __CUDACC_RTC__
// Launch `kern` on `s` with programmatic stream serialization allowed.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
#ifdef BWTA_NO_PDL
  cfg.numAttrs = 0;  // build-time option: plain stream-ordered launches
#else
  cfg.numAttrs = 1;
#endif
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}
#endif

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
                                      float *scale, uint8_t *a8, int64_t ld8, int32_t *d_status,
                                      cudaStream_t s);
cudaError_t launch_gemm_tc(const uint8_t *a8, int64_t ld8, const float *ascale, int64_t M,
                           const uint32_t *wb, const float *wscale, int64_t N, int64_t ldw,
                           int64_t K, int64_t group, float *Y, int64_t ldY, int32_t *dots,
                           int64_t ldD, int32_t *d_status, cudaStream_t s);
cudaError_t launch_gemm_tiled(const uint32_t *am, const uint32_t *as, const float *ascale,
                              int64_t M, int64_t lda, const uint32_t *wb, const float *wscale,
                              int64_t N, int64_t ldw, int64_t K, int64_t group, float *Y,
                              int64_t ldY, int32_t *dots, int64_t ldD, int32_t *d_status,
                              uint64_t stall_ns, cudaStream_t s);
// One decode projection (M <= 8 activation rows): fp16 rows X to ternarize in
// the kernel (fused) or packed planes am / as / ascale.
struct DecodeSpec {
  const uint16_t *X;
  int64_t ldX;
  const uint32_t *am, *as;
  const float *ascale;
  int64_t lda;
  int64_t M, K;
  const uint32_t *wbits;
  const float *wscale;
  int64_t N, ldw, group;
  float *Y;
  int64_t ldY;
  int32_t *dots;
  int64_t ldD;
};
bool decode_fits(int64_t M, int64_t K);
int decode_max_jobs();
size_t decode_act_bytes(int64_t M, int64_t K);
size_t decode_max_act_bytes();
cudaError_t launch_decode(const DecodeSpec *jobs, int njobs, bool fused, int mode, bool ready,
                          int32_t *d_status, cudaStream_t s);
cudaError_t launch_attn_scores(const uint32_t *qm, const uint32_t *qs, const float *qscale,
                               const uint32_t *km, const uint32_t *ks, const float *kscale,
                               int64_t BH, int64_t Lq, int64_t Lk, int64_t D, int64_t ld,
                               int32_t *Si, float *Sf, cudaStream_t s);
size_t attn_softmax_smem(int64_t Lk, int64_t ld);
cudaError_t launch_attn_softmax(const uint32_t *qm, const uint32_t *qs, const float *qscale,
                                const uint32_t *km, const uint32_t *ks, const float *kscale,
                                int64_t BH, int64_t Lq, int64_t Lk, int64_t D, int64_t ld, float c,
                                uint32_t *pm, uint32_t *ps, int64_t ldp, float *pscale,
                                cudaStream_t s);
cudaError_t launch_billm_pack(const float *W, int64_t ldW, int split, const billm_weights *out,
                              int32_t *d_status, cudaStream_t s);
cudaError_t launch_billm_gemm_tc(const uint16_t *X, int64_t M, int64_t ldX, const billm_weights *W,
                                 float *Y, int64_t ldY, int32_t *d_status, cudaStream_t s);
cudaError_t launch_billm_gemm(const uint16_t *X, int64_t M, int64_t ldX, const billm_weights *W,
                              float *Y, int64_t ldY, int32_t *d_status, cudaStream_t s);

}  // namespace bwta
