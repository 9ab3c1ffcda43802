// billm_tc.cu -- the BiLLM-format GEMM on the 5th-generation tensor cores.
//
// BiLLM: Pushing the Limit of Post-Training Quantization for LLMs -- abstract
// and "Approach": a weight is alpha_c*b or alpha_sp*b (non-salient, by its
// group bit) or alpha1*b1 + alpha2*b2 (salient column, residual plane), with
// the scales held per row and 128-column block; activations stay fp16.
//
// Y[m][n] = sum_k x[m][k] * w[n][k]. The kernel rebuilds w as fp32 from the
// bit planes and scales, multiplies it by a power of two 2^E per weight row
// (E chosen so that the row's largest |scale| lands in [2^14, 2^15)), and
// splits it into two fp16 numbers hi + lo (hi = fp16(v), lo = fp16(v - hi)).
// Two tcgen05.mma kind::f16 products, X*hi^T + X*lo^T, accumulate in fp32
// in TMEM over all of K; Y = D * 2^-E (exact). hi + lo carries w to about
// 2^-22 of its size (lo's own rounding), and x * (hi + lo) products are exact
// in fp32, so the error of Y is that of an fp32 sum of K terms: well inside
// 1e-5 of sum_k |x w|.
//
// Persistent kernel, one CTA per SM; tiles of 128 weight rows x BN tokens
// (BN = 64 or 256), k-blocks of 64 columns (one 128-byte fp16 swizzle row):
//  * warp 16 (one thread): TMA loads of the fp16 activations (BN rows x 128 B,
//    128-byte swizzle) into a ring of stages;
//  * warps 0-7: two threads per weight row, 32 columns each, read the row's
//    sign and group-map words (prefetched four k-blocks ahead), its block
//    scales, residual bits and the block's salient columns, and write the hi
//    and lo operand tiles (K-major, 128-byte swizzle) into the same stage;
//  * warp 17 (one thread): 8 MMAs per k-block (M=128, N=BN, K=16; hi and lo)
//    into one of two fp32 accumulators (one per tile in flight), one commit
//    per k-block;
//  * warps 8-15: read a finished accumulator (two warps per TMEM lane quarter),
//    scale by 2^-E and write Y.
// Every wait is bounded; on a timeout the CTA records BWTA_STATUS_TIMEOUT,
// drains and returns.
#include <algorithm>

#include <cuda_fp16.h>

#include "common.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace bwta {

constexpr int BT_BM = 128;                 // weight rows per tile (MMA M, TMEM lanes)
constexpr int BT_KB = 64;                  // K per k-block: 128 bytes of fp16
constexpr int BT_A_BYTES = BT_BM * 128;    // one 128 x 64 fp16 operand tile
constexpr int BT_EXPAND = 8, BT_EPI = 8;   // warps per role
constexpr int BT_PRODUCER = 16, BT_ISSUER = 17;
constexpr int BT_THREADS = 18 * 32;
constexpr int BT_DBUF = 2;
constexpr int BT_MAX_STAGES = 5;
constexpr int BT_MAX_SAL = 40960 / 128 * 8;  // salient-column table bytes (K <= 40960)

template <int BN>
struct BtShape {
  static constexpr int X_BYTES = BN * 128;
  static constexpr int STAGE = X_BYTES + 2 * BT_A_BYTES;
  static constexpr int STAGES = BN == 256 ? 3 : 5;
  static constexpr uint32_t TMEM_COLS = BN == 256 ? 512 : 128;  // BT_DBUF accumulators
};
static_assert(BtShape<256>::STAGE % 1024 == 0 && BtShape<64>::STAGE % 1024 == 0, "alignment");

struct BtSync {
  uint64_t xfull[BT_MAX_STAGES];  // activations landed (TMA transaction bytes)
  uint64_t afull[BT_MAX_STAGES];  // hi / lo tiles written (8 expand warps)
  uint64_t done[BT_MAX_STAGES];   // MMAs of the stage's k-block complete (commit)
  uint64_t d_full[BT_DBUF];       // tile accumulated (commit)
  uint64_t d_empty[BT_DBUF];      // accumulator read out (8 epilogue warps)
  uint64_t drain;
  uint32_t tmem_base;
  int32_t timeout;
  int32_t undrained;  // a post-timeout drain ran out of time
};

template <int BN>
constexpr size_t bt_smem() {
  return 1024 + (size_t)BtShape<BN>::STAGES * BtShape<BN>::STAGE + sizeof(BtSync) + 64 + BT_MAX_SAL + 64;
}

__device__ __forceinline__ bool bt_wait(BtSync *b, uint64_t *bar, uint32_t parity) {
  if (b->timeout) return false;
  if (mbar_wait(bar, parity, 2000000000ull)) return true;
  b->timeout = 1;
  return false;
}

// Power-of-two exponent E of a weight row: the row's largest |scale| (the
// salient pair counted as |alpha1| + |alpha2|) times 2^E lies in [2^14, 2^15).
// Computed the same way by the expand and the epilogue threads.
__device__ __forceinline__ int bt_row_exp(const float4 *bs_row, int nb) {
  float amax = 0.0f;
#pragma unroll 8
  for (int j = 0; j < nb; ++j) {
    const float4 a = __ldg(bs_row + j);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fabsf(a.z) + fabsf(a.w)));
  }
  if (!(amax > 0.0f) || !(amax < 3.0e38f)) return 0;
  int e;
  frexpf(amax, &e);  // amax in [2^(e-1), 2^e)
  return min(100, max(-100, 15 - e));
}

// fp16 bit patterns of v (hi) and of v - hi (lo).
__device__ __forceinline__ void bt_split(float v, uint32_t &hi, uint32_t &lo) {
  const __half h = __float2half_rn(v);
  const __half l = __float2half_rn(v - __half2float(h));
  hi = __half_as_ushort(h);
  lo = __half_as_ushort(l);
}

template <int BN>
__global__ void __launch_bounds__(BT_THREADS, 1)
k_billm_gemm_tc(const __grid_constant__ CUtensorMap map_x, const uint32_t *__restrict__ sign,
                const uint32_t *__restrict__ gmap, const uint8_t *__restrict__ res,
                const uint8_t *__restrict__ sal, const float *__restrict__ bscale, int64_t M,
                int64_t N, int64_t K, int64_t ldw, int n_sal, float *__restrict__ Y, int64_t ldY,
                int32_t *d_status) {
  using Sh = BtShape<BN>;
  constexpr int S = Sh::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *stages = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  BtSync *sy = reinterpret_cast<BtSync *>(stages + S * Sh::STAGE);
  uint32_t *sel_lut = reinterpret_cast<uint32_t *>(sy + 1);  // 16 PRMT selectors
  uint8_t *sal_s = reinterpret_cast<uint8_t *>(sel_lut + 16);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nb = (int)(K / 128), KB = (int)(K / BT_KB);
  const int64_t NT = ceil_div<int64_t>(M, BN);                 // token tiles
  const int64_t ntiles = ceil_div<int64_t>(N, BT_BM) * NT;     // row tile major

  pdl_trigger();
  if (threadIdx.x == 0) {
    prefetch_tensormap(&map_x);
    for (int s = 0; s < S; ++s) {
      mbar_init(&sy->xfull[s], 1);
      mbar_init(&sy->afull[s], BT_EXPAND);
      mbar_init(&sy->done[s], 1);
    }
    for (int i = 0; i < BT_DBUF; ++i) {
      mbar_init(&sy->d_full[i], 1);
      mbar_init(&sy->d_empty[i], BT_EPI);
    }
    mbar_init(&sy->drain, 1);
    sy->timeout = 0;
    sy->undrained = 0;
    mbar_fence_init();
  }
  if (warp == BT_ISSUER) {
    tmem_alloc(&sy->tmem_base, Sh::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();
  for (int i = threadIdx.x; i < nb * n_sal; i += BT_THREADS) sal_s[i] = sal[i];
  if (threadIdx.x < 16) {
    // code c = g0 | g1 << 1 | s0 << 2 | s1 << 3 of an element pair -> byte selector
    // picking pattern g + 2s (+alpha_c, +alpha_sp, -alpha_c, -alpha_sp) for each
    const uint32_t c = threadIdx.x;
    const uint32_t i0 = (c & 1u) + ((c >> 1) & 2u), i1 = ((c >> 1) & 1u) + ((c >> 2) & 2u);
    sel_lut[c] = (2 * i0) | ((2 * i0 + 1) << 4) | ((2 * i1) << 8) | ((2 * i1 + 1) << 12);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sy->tmem_base;

  if (warp == BT_PRODUCER) {
    // ------------------------------------------------ TMA loads of the activations
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int32_t m0 = (int32_t)((tile % NT) * BN);
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % S;
          if (g >= S && !bt_wait(sy, &sy->done[s], ((g / S) - 1) & 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sy->xfull[s], Sh::X_BYTES);
          tma_load_2d(stages + s * Sh::STAGE, &map_x, kb * BT_KB, m0, &sy->xfull[s]);
        }
      }
      // a stage is reloaded only after the MMAs that read it, which waited for
      // its load: the last S loads are the only ones that can be pending
      for (uint32_t j = g > (uint32_t)S ? g - S : 0; j < g; ++j)
        if (!mbar_wait(&sy->xfull[j % S], (j / S) & 1, DRAIN_NS)) sy->undrained = 1;
    }
    __syncwarp();
  } else if (warp == BT_ISSUER) {
    // ------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(BT_BM, BN);
      uint32_t g = 0, tl = 0;  // k-blocks, tiles of this CTA so far
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tl) {
        const int d = tl % BT_DBUF;
        if (tl >= BT_DBUF && !bt_wait(sy, &sy->d_empty[d], ((tl / BT_DBUF) - 1) & 1)) break;
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % S;
          if (!bt_wait(sy, &sy->xfull[s], (g / S) & 1) || !bt_wait(sy, &sy->afull[s], (g / S) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xs = smem_addr(stages + s * Sh::STAGE);
          const uint32_t ah = xs + Sh::X_BYTES, al = ah + BT_A_BYTES;
#pragma unroll
          for (int k16 = 0; k16 < BT_KB / 16; ++k16) {
            const uint64_t bd = smem_desc_k_sw128(xs + k16 * 32);
            mma_f16_ss(tmem + d * BN, smem_desc_k_sw128(ah + k16 * 32), bd, idesc,
                       (kb > 0 || k16 > 0) ? 1u : 0u);
            mma_f16_ss(tmem + d * BN, smem_desc_k_sw128(al + k16 * 32), bd, idesc, 1u);
          }
          tc_commit(&sy->done[s]);
          if (kb == KB - 1) tc_commit(&sy->d_full[d]);
        }
      }
      tc_commit(&sy->drain);
      if (!mbar_wait(&sy->drain, 0, DRAIN_NS)) sy->undrained = 1;
    }
    __syncwarp();
  } else if (warp < BT_EXPAND) {
    // ------------------------------------------------ bit planes + scales -> hi / lo tiles
    const int r = threadIdx.x & (BT_BM - 1), h = threadIdx.x / BT_BM;  // row, 32-column half
    uint32_t g = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const int64_t n0r = (tile / NT) * BT_BM + r;
      const int64_t n = n0r < N ? n0r : N - 1;  // rows past N: any valid row
      const uint32_t *srow = sign + n * ldw, *grow = gmap + n * ldw;
      const float4 *bs_row = reinterpret_cast<const float4 *>(bscale) + n * nb;
      const float pw = ldexpf(1.0f, bt_row_exp(bs_row, nb));
      // four k-blocks of sign / group words in flight ahead of use; two blocks of scales
      uint32_t s0 = __ldg(srow + h), g0 = __ldg(grow + h);
      uint32_t s1 = KB > 1 ? __ldg(srow + 2 + h) : 0u, g1 = KB > 1 ? __ldg(grow + 2 + h) : 0u;
      uint32_t s2 = KB > 2 ? __ldg(srow + 4 + h) : 0u, g2 = KB > 2 ? __ldg(grow + 4 + h) : 0u;
      uint32_t s3 = KB > 3 ? __ldg(srow + 6 + h) : 0u, g3 = KB > 3 ? __ldg(grow + 6 + h) : 0u;
      float4 sc_next = __ldg(bs_row), sc_next2 = nb > 1 ? __ldg(bs_row + 1) : make_float4(0, 0, 0, 0);
      uint32_t rb_next = res[n * nb], rb_next2 = nb > 1 ? res[n * nb + 1] : 0u;
      float4 sc = sc_next;
      uint32_t rb = rb_next;
      // byte pools of the four non-salient values (+alpha_c, +alpha_sp, -alpha_c,
      // -alpha_sp; x 2^E, fp16): hi parts in th0/th1, lo parts in tl0/tl1; and the
      // salient pair values alpha1 + alpha2, alpha1 - alpha2
      uint32_t th0 = 0, th1 = 0, tl0 = 0, tl1 = 0, ppp_h = 0, ppp_l = 0, ppm_h = 0, ppm_l = 0;
      for (int kb = 0; kb < KB; ++kb, ++g) {
        const int s = g % S, j = kb >> 1;
        if ((kb & 1) == 0) {  // a new 128-column block: its scales, the next block's in flight
          sc = sc_next;
          rb = rb_next;
          sc_next = sc_next2;
          rb_next = rb_next2;
          if (j + 2 < nb) {
            sc_next2 = __ldg(bs_row + j + 2);
            rb_next2 = res[n * nb + j + 2];
          }
          uint32_t pc_h, pc_l, psp_h, psp_l;
          bt_split(sc.x * pw, pc_h, pc_l);
          bt_split(sc.y * pw, psp_h, psp_l);
          bt_split((sc.z + sc.w) * pw, ppp_h, ppp_l);
          bt_split((sc.z - sc.w) * pw, ppm_h, ppm_l);
          th0 = pc_h | (psp_h << 16);
          th1 = th0 ^ 0x80008000u;
          tl0 = pc_l | (psp_l << 16);
          tl1 = tl0 ^ 0x80008000u;
        }
        const uint32_t S_w = s0, G_w = g0;
        s0 = s1;
        g0 = g1;
        s1 = s2;
        g1 = g2;
        s2 = s3;
        g2 = g3;
        if (kb + 4 < KB) {
          s3 = __ldg(srow + 2 * (kb + 4) + h);
          g3 = __ldg(grow + 2 * (kb + 4) + h);
        }
        const int cb = (kb & 1) * 64 + h * 32;  // this thread's 32 columns of block j
        uint32_t hw[16], lw[16];
#pragma unroll
        for (int p = 0; p < 16; ++p) {  // element pair 2p, 2p+1: one byte permute per plane
          const uint32_t code = ((G_w >> (2 * p)) & 3u) | (((S_w >> (2 * p)) & 3u) << 2);
          const uint32_t sel = sel_lut[code];
          hw[p] = __byte_perm(th0, th1, sel);
          lw[p] = __byte_perm(tl0, tl1, sel);
        }
        // the stage's previous k-block is done with its tiles
        bool fine = true;
        if (lane == 0 && g >= (uint32_t)S) fine = bt_wait(sy, &sy->done[s], ((g / S) - 1) & 1);
        fine = __shfl_sync(FULL, fine, 0);
        __syncwarp();
        if (!fine) {
          ok = false;
          break;
        }
        uint8_t *ahi = stages + s * Sh::STAGE + Sh::X_BYTES, *alo = ahi + BT_A_BYTES;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const uint32_t off = swz128(r, h * 4 + c4);
          *reinterpret_cast<uint4 *>(ahi + off) =
              make_uint4(hw[4 * c4], hw[4 * c4 + 1], hw[4 * c4 + 2], hw[4 * c4 + 3]);
          *reinterpret_cast<uint4 *>(alo + off) =
              make_uint4(lw[4 * c4], lw[4 * c4 + 1], lw[4 * c4 + 2], lw[4 * c4 + 3]);
        }
        // salient columns: b1 * (alpha1 + alpha2) when b1 == b2, b1 * (alpha1 - alpha2) otherwise
        for (int i = 0; i < n_sal; ++i) {
          const int c = (int)sal_s[j * n_sal + i] - cb;
          if (c >= 0 && c < 32) {
            const uint32_t b1 = (S_w >> c) & 1u, b2 = (rb >> i) & 1u;
            const uint32_t vh = (b1 == b2 ? ppp_h : ppm_h) ^ (b1 << 15);
            const uint32_t vl = (b1 == b2 ? ppp_l : ppm_l) ^ (b1 << 15);
            const uint32_t off = swz128(r, h * 4 + (c >> 3)) + 2 * (c & 7);
            *reinterpret_cast<uint16_t *>(ahi + off) = (uint16_t)vh;
            *reinterpret_cast<uint16_t *>(alo + off) = (uint16_t)vl;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&sy->afull[s]);
      }
    }
  } else if (warp < BT_EXPAND + BT_EPI) {
    // ------------------------------------------------ epilogue: D * 2^-E -> Y
    const int q = warp % 4, hh = (warp - BT_EXPAND) / 4, r = q * 32 + lane;
    uint32_t tl = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tl) {
      const int64_t n = (tile / NT) * BT_BM + r, m0 = (tile % NT) * BN + hh * (BN / 2);
      const int64_t nc = n < N ? n : N - 1;
      const float inv = ldexpf(1.0f, -bt_row_exp(reinterpret_cast<const float4 *>(bscale) + nc * nb, nb));
      const int d = tl % BT_DBUF;
      bool fine = true;
      if (lane == 0) fine = bt_wait(sy, &sy->d_full[d], (tl / BT_DBUF) & 1);
      fine = __shfl_sync(FULL, fine, 0);
      __syncwarp();
      if (!fine) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < BN / 2; c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem_addr(tmem, q * 32, d * BN + hh * (BN / 2) + c), v);
        tmem_wait_ld();
        if (n < N) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int64_t m = m0 + c + i;
            if (m < M) Y[m * ldY + n] = __uint_as_float(v[i]) * inv;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sy->d_empty[d]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == BT_ISSUER) {
    tc_fence_after();
    tmem_dealloc(tmem, Sh::TMEM_COLS);
  }
  // TMEM is released even after a drain ran out of time (a later CTA on this
  // SM would otherwise block in its allocation); the DRAIN flag reports it
  if (threadIdx.x == 0 && sy->timeout)
    flag_status(d_status, BWTA_STATUS_TIMEOUT | (sy->undrained ? BWTA_STATUS_DRAIN : 0));
}

template <int BN>
static cudaError_t launch_bt_t(const CUtensorMap &mx, const billm_weights *W, int64_t M, float *Y,
                               int64_t ldY, int32_t *d_status, cudaStream_t s) {
  auto kern = k_billm_gemm_tc<BN>;
  static SmemOptIn opt_in;
  if (cudaError_t e = opt_in(kern, (int)bt_smem<BN>())) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntiles = ceil_div<int64_t>(W->N, BT_BM) * ceil_div<int64_t>(M, BN);
  const unsigned grid = (unsigned)std::min<int64_t>(ntiles, std::max(sms, 1));
  return launch_pdl(kern, dim3(grid), dim3(BT_THREADS), bt_smem<BN>(), s, mx, W->sign, W->gmap,
                    W->res, W->sal, W->bscale, M, W->N, W->K, W->ldw_words, (int)W->n_sal, Y, ldY,
                    d_status);
}

// Tensor-core BiLLM GEMM. Needs X 16-byte aligned with ldX % 8 == 0 (TMA);
// returns cudaErrorNotSupported otherwise, and the caller takes the CUDA-core path.
cudaError_t launch_billm_gemm_tc(const uint16_t *X, int64_t M, int64_t ldX, const billm_weights *W,
                                 float *Y, int64_t ldY, int32_t *d_status, cudaStream_t s) {
  if (M == 0 || W->N == 0) return cudaSuccess;
  if ((reinterpret_cast<uintptr_t>(X) & 15u) || ldX % 8 || W->K % BT_KB || W->K > 40960)
    return cudaErrorNotSupported;
  const int BN = M > 64 ? 256 : 64;
  CUtensorMap mx;
  if (!make_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, X, M, ldX, BT_KB, (uint32_t)BN,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  return BN == 256 ? launch_bt_t<256>(mx, W, M, Y, ldY, d_status, s)
                   : launch_bt_t<64>(mx, W, M, Y, ldY, d_status, s);
}

}  // namespace bwta
