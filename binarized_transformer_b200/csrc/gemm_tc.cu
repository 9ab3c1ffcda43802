// gemm_tc.cu -- the binary x ternary GEMM on the 5th-generation tensor cores.
//
// BWTA: Accurate and Efficient Binarized Transformer by Algorithm-Hardware
// Co-design -- abstract: a bit-packed MatMul of binary weights with ternary
// activations. The product of a weight in {-1,+1} and an activation in
// {-1,0,+1} is exact in 8-bit floating point (E4M3 holds -1, 0, +1 exactly),
// and so is every partial sum in the fp32 accumulator (integers below 2^24).
// This kernel therefore runs the contraction as tcgen05.mma kind::f8f6f4 and
// gets the same integer dots as the popcount path, then applies the scales in
// the same order (acc = fma((float)d_g, alpha_g, acc) over the weight groups,
// times the activation scale), so its fp32 outputs match bit for bit.
//
// Layout (one CTA = 128 weight rows x 128 tokens, 1 CTA per SM):
//  * the weight rows are the MMA's M dimension and live in TMEM as operand A:
//    four "expand" warps read each row's sign bits (TMA-loaded, 16 bytes per
//    row per 128-column block), turn them into E4M3 +-1 bytes through a
//    16-entry table and store them with tcgen05.st (one lane per row);
//  * the activations are operand B: E4M3 bytes written by the activation
//    packer, TMA-loaded 128 tokens x 128 bytes with the 128-byte swizzle;
//  * the accumulator of one weight group is D (fp32, 128 lanes x 128
//    columns, three buffers); eight epilogue warps (two per TMEM lane
//    quarter, 64 token columns each) load a finished group with two
//    tcgen05.ld, release the buffer, and fold it into running fp32 sums held in
//    registers; the group scales are prefetched one group ahead;
//  * one warp issues the TMA loads and the MMAs (one elected thread).
// Every mbarrier wait is bounded (bwta::mbar_wait); on a timeout the CTA
// records BWTA_STATUS_TIMEOUT and drains.
#include <algorithm>

#include "common.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace bwta {

constexpr int TC_BM = 128;        // weight rows per CTA (TMEM lanes, MMA M)
constexpr int TC_BN = 128;        // tokens per CTA (MMA N)
constexpr int TC_KB = 128;        // K elements per block = one 128-byte swizzle row
constexpr int TC_STAGES = 7;  // > half the SM's shared memory: one CTA (one TMEM owner) per SM
constexpr int TC_THREADS = 416;   // warps 0-3 expand, 4-11 epilogue, 12 TMA + MMA
constexpr int TC_ISSUER = 12;
constexpr int TC_DBUF = 3;        // accumulator buffers: the MMAs may run two groups ahead
constexpr int TC_ABUF = 4;        // expanded-weight buffers: expansion may run three blocks ahead
constexpr int TC_X_BYTES = TC_BN * TC_KB;     // 16 KB of E4M3 activations per stage
constexpr int TC_W_BYTES = TC_BM * 16;        // 2 KB of weight sign bits per stage
constexpr int TC_STAGE_BYTES = TC_X_BYTES + TC_W_BYTES;
// TMEM columns: D0 0..127, D1 128..255, D2 256..383, A0..A3 384..511 (32 each)
constexpr uint32_t TC_TMEM_COLS = 512, TC_COL_A = 384;
constexpr size_t TC_SMEM = 1024 + (size_t)TC_STAGES * TC_STAGE_BYTES + 1024;

struct TcBarriers {
  uint64_t full[TC_STAGES];   // TMA landed (tx bytes)
  uint64_t empty[TC_STAGES];  // MMA done with the stage (commit) + 4 expand warps done
  uint64_t a_full[TC_ABUF];   // expanded weights in TMEM (4 expand warps)
  uint64_t a_empty[TC_ABUF];  // MMA done with the A buffer (commit)
  uint64_t d_full[TC_DBUF];   // group accumulated (commit)
  uint64_t d_empty[TC_DBUF];  // epilogue has read the D buffer (8 epilogue warps)
  uint32_t tmem_base;
  int32_t timeout;
};

__device__ __forceinline__ uint64_t *bar_of(TcBarriers *b, int which, int i) {
  switch (which) {
    case 0: return &b->full[i];
    case 1: return &b->empty[i];
    case 2: return &b->a_full[i];
    case 3: return &b->a_empty[i];
    case 4: return &b->d_full[i];
    default: return &b->d_empty[i];
  }
}

// Bounded wait that also records a timeout for the whole CTA.
__device__ __forceinline__ bool tc_wait(TcBarriers *b, uint64_t *bar, uint32_t parity) {
  if (b->timeout) return false;
  if (mbar_wait(bar, parity, 2000000000ull)) return true;
  b->timeout = 1;
  return false;
}

// E4M3 encodings: +1.0 = 0x38, -1.0 = 0xB8, 0 = 0x00. Table entry n holds the
// four bytes of four weights whose sign bits are the nibble n (bit i = weight i,
// 1 = negative).
__device__ __forceinline__ uint32_t e4m3_pm1_word(uint32_t nib) {
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) w |= (((nib >> i) & 1u) ? 0xB8u : 0x38u) << (8 * i);
  return w;
}

template <bool GROUPED, bool WANT_Y, bool WANT_DOTS>
__global__ void __launch_bounds__(TC_THREADS, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
          const float *__restrict__ ascale, const float *__restrict__ wscale, int64_t M, int64_t N,
          int KB, int seg_len, int64_t G, float *__restrict__ Y, int64_t ldY,
          int32_t *__restrict__ dots, int64_t ldD, int32_t *d_status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  TcBarriers *bars = reinterpret_cast<TcBarriers *>(smem + TC_STAGES * TC_STAGE_BYTES);
  uint32_t *lut = reinterpret_cast<uint32_t *>(bars + 1);
  float *sA = reinterpret_cast<float *>(lut + 16);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t n0 = (int64_t)blockIdx.x * TC_BM, m0 = (int64_t)blockIdx.y * TC_BN;
  const int nseg = (KB + seg_len - 1) / seg_len;

  pdl_trigger();
  if (threadIdx.x == 0) {
    prefetch_tensormap(&map_x);
    prefetch_tensormap(&map_w);
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1 + 4);
    }
    for (int i = 0; i < TC_ABUF; ++i) {
      mbar_init(&bars->a_full[i], 4);
      mbar_init(&bars->a_empty[i], 1);
    }
    for (int i = 0; i < TC_DBUF; ++i) {
      mbar_init(&bars->d_full[i], 1);
      mbar_init(&bars->d_empty[i], 8);
    }
    bars->timeout = 0;
    mbar_fence_init();
  }
  if (threadIdx.x < 16) lut[threadIdx.x] = e4m3_pm1_word(threadIdx.x);
  if (warp == TC_ISSUER) {
    tmem_alloc(&bars->tmem_base, TC_TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();
  if (threadIdx.x < TC_BN) sA[threadIdx.x] = (WANT_Y && m0 + threadIdx.x < M) ? __ldg(ascale + m0 + threadIdx.x) : 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == TC_ISSUER) {
    // ------------------------------------------------ TMA + MMA issuer
    if (lane == 0) {
      auto tma = [&](int kb) -> bool {
        const int s = kb % TC_STAGES;
        if (kb >= TC_STAGES && !tc_wait(bars, &bars->empty[s], ((kb / TC_STAGES) - 1) & 1))
          return false;
        uint8_t *st = stages + s * TC_STAGE_BYTES;
        mbar_arrive_expect_tx(&bars->full[s], TC_STAGE_BYTES);
        tma_load_2d(st, &map_x, kb * TC_KB, (int32_t)m0, &bars->full[s]);
        tma_load_2d(st + TC_X_BYTES, &map_w, kb * 4, (int32_t)n0, &bars->full[s]);
        return true;
      };
      constexpr int LOOK = TC_STAGES - 2;  // loads run LOOK blocks ahead of the MMAs
      bool ok = true;
      for (int kb = 0; kb < LOOK && kb < KB && ok; ++kb) ok = tma(kb);
      const uint32_t idesc = idesc_e4m3_f32(TC_BM, TC_BN);
      for (int kb = 0; kb < KB && ok; ++kb) {
        if (kb + LOOK < KB && !tma(kb + LOOK)) break;
        const int seg = kb / seg_len, d = seg % TC_DBUF, s = kb % TC_STAGES, b = kb % TC_ABUF;
        const bool first = (kb % seg_len) == 0;
        const bool last = (kb % seg_len) == seg_len - 1 || kb == KB - 1;
        if (first && seg >= TC_DBUF &&
            !tc_wait(bars, &bars->d_empty[d], ((seg / TC_DBUF) - 1) & 1))
          break;
        if (!tc_wait(bars, &bars->full[s], (kb / TC_STAGES) & 1)) break;
        if (!tc_wait(bars, &bars->a_full[b], (kb / TC_ABUF) & 1)) break;
        tc_fence_after();
        const uint32_t xs = smem_addr(stages + s * TC_STAGE_BYTES);
#pragma unroll
        for (int k4 = 0; k4 < TC_KB / 32; ++k4)
          mma_f8f6f4_ts(tmem + d * 128, tmem + TC_COL_A + b * 32 + k4 * 8,
                        smem_desc_k_sw128(xs + k4 * 32), idesc, (first && k4 == 0) ? 0u : 1u);
        tc_commit(&bars->empty[s]);
        tc_commit(&bars->a_empty[b]);
        if (last) tc_commit(&bars->d_full[d]);
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------ weight bits -> E4M3 in TMEM
    const int r = warp * 32 + lane;
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % TC_STAGES, b = kb % TC_ABUF;
      bool ok = tc_wait(bars, &bars->full[s], (kb / TC_STAGES) & 1);
      if (ok && kb >= TC_ABUF) ok = tc_wait(bars, &bars->a_empty[b], ((kb / TC_ABUF) - 1) & 1);
      if (!__all_sync(FULL, ok)) break;
      const uint4 bits = *reinterpret_cast<const uint4 *>(stages + s * TC_STAGE_BYTES + TC_X_BYTES + r * 16);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty[s]);
      const uint32_t wd[4] = {bits.x, bits.y, bits.z, bits.w};
      uint32_t v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = lut[(wd[j >> 3] >> (4 * (j & 7))) & 15u];
      tmem_st32(tmem_addr(tmem, warp * 32, TC_COL_A + b * 32), v);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->a_full[b]);
    }
  } else {
    // ------------------------------------------------ epilogue: fold groups, write Y
    const int h = (warp - 4) / 4, q = warp % 4, r = q * 32 + lane;
    const int64_t n = n0 + r;
    float y[64];
    uint32_t dv0[32], dv1[32];
    float alpha = (n < N) ? __ldg(wscale + (GROUPED ? n * G : n)) : 0.0f;
    for (int seg = 0; seg < nseg; ++seg) {
      const int d = seg % TC_DBUF;
      const float alpha_next =
          (GROUPED && seg + 1 < nseg && n < N) ? __ldg(wscale + n * G + seg + 1) : 0.0f;
      const bool ok = tc_wait(bars, &bars->d_full[d], (seg / TC_DBUF) & 1);
      if (!__all_sync(FULL, ok)) break;
      tc_fence_after();
      tmem_ld32(tmem_addr(tmem, q * 32, d * 128 + h * 64), dv0);
      tmem_ld32(tmem_addr(tmem, q * 32, d * 128 + h * 64 + 32), dv1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->d_empty[d]);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        y[i] = fmaf(__uint_as_float(dv0[i]), alpha, seg > 0 ? y[i] : 0.0f);
        y[32 + i] = fmaf(__uint_as_float(dv1[i]), alpha, seg > 0 ? y[32 + i] : 0.0f);
      }
      alpha = alpha_next;
    }
    if (n < N && !bars->timeout) {
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const int64_t m = m0 + h * 64 + i;
        if (m < M) {
          if (WANT_Y) Y[m * ldY + n] = y[i] * sA[h * 64 + i];
          if (WANT_DOTS)
            dots[m * ldD + n] = __float2int_rn(__uint_as_float(i < 32 ? dv0[i] : dv1[i - 32]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == TC_ISSUER) {
    tc_fence_after();
    tmem_dealloc(tmem, TC_TMEM_COLS);
  }
  if (threadIdx.x == 0 && bars->timeout) flag_status(d_status, BWTA_STATUS_TIMEOUT);
}

template <bool GROUPED, bool WANT_Y, bool WANT_DOTS>
static cudaError_t launch_tc_t(const CUtensorMap &mx, const CUtensorMap &mw, const float *ascale,
                               const float *wscale, int64_t M, int64_t N, int KB, int seg_len,
                               int64_t G, float *Y, int64_t ldY, int32_t *dots, int64_t ldD,
                               int32_t *d_status, cudaStream_t s) {
  auto kern = k_gemm_tc<GROUPED, WANT_Y, WANT_DOTS>;
  static cudaError_t attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TC_SMEM);
  if (attr != cudaSuccess) return attr;
  dim3 grid((unsigned)ceil_div<int64_t>(N, TC_BM), (unsigned)ceil_div<int64_t>(M, TC_BN));
  return launch_pdl(kern, grid, dim3(TC_THREADS), TC_SMEM, s, mx, mw, ascale, wscale, M, N, KB,
                    seg_len, G, Y, ldY, dots, ldD, d_status);
}

cudaError_t launch_gemm_tc(const uint8_t *a8, int64_t ld8, const float *ascale, int64_t M,
                           const uint32_t *wb, const float *wscale, int64_t N, int64_t ldw,
                           int64_t K, int64_t group, float *Y, int64_t ldY, int32_t *dots,
                           int64_t ldD, int32_t *d_status, cudaStream_t s) {
  if (M == 0 || N == 0) return cudaSuccess;
  CUtensorMap mx, mw;
  if (!make_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a8, M, ld8, TC_KB, TC_BN,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, wb, N, ldw, 4, TC_BM,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const int KB = (int)ceil_div<int64_t>(K, TC_KB);
  if (group == 0) {
    if (Y && dots)
      return launch_tc_t<false, true, true>(mx, mw, ascale, wscale, M, N, KB, KB, 1, Y, ldY, dots,
                                            ldD, d_status, s);
    if (Y)
      return launch_tc_t<false, true, false>(mx, mw, ascale, wscale, M, N, KB, KB, 1, Y, ldY, dots,
                                             ldD, d_status, s);
    return launch_tc_t<false, false, true>(mx, mw, ascale, wscale, M, N, KB, KB, 1, Y, ldY, dots,
                                           ldD, d_status, s);
  }
  const int seg_len = (int)(group / TC_KB);
  const int64_t G = ceil_div<int64_t>(K, group);
  cudaError_t e = cudaSuccess;
  if (Y)
    e = launch_tc_t<true, true, false>(mx, mw, ascale, wscale, M, N, KB, seg_len, G, Y, ldY,
                                       nullptr, ldD, d_status, s);
  if (e == cudaSuccess && dots)  // full-K integer dots: one segment over all of K
    e = launch_tc_t<false, false, true>(mx, mw, ascale, wscale, M, N, KB, KB, 1, nullptr, ldY,
                                        dots, ldD, d_status, s);
  return e;
}

}  // namespace bwta
