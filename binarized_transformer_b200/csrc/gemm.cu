// gemm.cu -- the bit-packed binary x ternary GEMM (prefill) and GEMV (decode).
//
// BWTA: Accurate and Efficient Binarized Transformer by Algorithm-Hardware
// Co-design -- abstract and "Core claim": a bit-packed MatMul of binary
// weights with ternary activations. Per 32-bit word of a row pair:
//     dot += popc(mask) - 2 * popc(mask & (a_sign ^ w_sign))
// since a nonzero activation and a weight agree in sign exactly where the
// sign bits are equal. popc(mask) does not depend on the weight row, so it is
// counted once per (activation row, 128-element chunk) and shared by a whole
// tile; per 4-word chunk of one output the inner loop is four LOP3s
// (mask & (a ^ w)), a carry-save full adder (two LOP3s) and three POPCs.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "quant.cuh"
#include "tma.cuh"

namespace bwta {

// ===================================================================== host
PFN_encodeTiled get_encode_tiled() {
  static PFN_encodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  });
  return fn;
}

bool make_plane_map(CUtensorMap *map, const uint32_t *base, int64_t rows, int64_t ld,
                    uint32_t box_w, uint32_t box_h) {
  PFN_encodeTiled enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)ld, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  cuuint32_t box[2] = {box_w, box_h};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map_2d(CUtensorMap *map, CUtensorMapDataType dtype, int elem_bytes, const void *base,
                 int64_t rows, int64_t ld, uint32_t box_w, uint32_t box_h,
                 CUtensorMapSwizzle swizzle) {
  PFN_encodeTiled enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)ld, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * (cuuint64_t)elem_bytes};
  cuuint32_t box[2] = {box_w, box_h};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ============================================================ tiled GEMM (K2)
// CTA tile 128 (activation rows) x 128 (weight rows), K staged 32 words
// (1024 elements) at a time by TMA into a 3-deep ring of 128-byte-swizzled
// tiles (mask, sign, weight: 16 KB each). 512 threads (16 warps: enough to
// cover the LOP3 -> POPC -> add latencies); thread (ty, tx) = (warp, lane) owns
// rows ty + 16*i (i < 8) and columns tx + 32*j (j < 4): 16-byte shared loads of
// four K-words, broadcast for the rows and conflict-free for the columns thanks
// to the swizzle. Per stage the CTA first
// counts popc(mask) per (row, 4-word chunk) and stages the weight scales of
// each chunk's group; at the end of every weight group each thread folds its
// 64 integer dots into fp32 with acc = fma((float)d_g, alpha_g, acc), in group
// order, and the epilogue multiplies by the activation scale.
constexpr int GM_BM = 128, GM_BN = 128, GM_BKW = 32, GM_STAGES = 3, GM_THREADS = 512;
constexpr int GM_TI = 8, GM_TJ = 4;  // outputs per thread: rows ty + 16*i, columns tx + 32*j
constexpr int GM_CHUNKS = GM_BKW / 4;
constexpr int GM_TILE_WORDS = GM_BM * GM_BKW;
constexpr int GM_TILE_BYTES = GM_TILE_WORDS * 4;
constexpr size_t GM_SMEM = 1024 + (size_t)GM_STAGES * 3 * GM_TILE_BYTES +
                           2 * GM_CHUNKS * GM_BM * 4 + GM_STAGES * 8;

template <bool GROUPED, bool WANT_Y, bool WANT_DOTS>
__global__ void __launch_bounds__(GM_THREADS, 1)
k_gemm_tiled(const __grid_constant__ CUtensorMap map_am, const __grid_constant__ CUtensorMap map_as,
             const __grid_constant__ CUtensorMap map_w, const float *__restrict__ ascale,
             const float *__restrict__ wscale, int64_t M, int64_t N, int nchunks, int gchunks,
             int64_t G, float *__restrict__ Y, int64_t ldY, int32_t *__restrict__ dots,
             int64_t ldD, int32_t *d_status) {
  static_assert(!(GROUPED && WANT_DOTS), "grouped dots come from the ungrouped pass");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *tiles = smem;
  uint32_t *Pst = reinterpret_cast<uint32_t *>(tiles + GM_STAGES * 3 * GM_TILE_BYTES);
  float *Ast = reinterpret_cast<float *>(Pst + GM_CHUNKS * GM_BM);
  uint64_t *full = reinterpret_cast<uint64_t *>(Ast + GM_CHUNKS * GM_BN);

  const int tid = threadIdx.x, ty = tid / 32, tx = tid % 32;
  const int64_t m0 = (int64_t)blockIdx.y * GM_BM, n0 = (int64_t)blockIdx.x * GM_BN;
  const int KT = (nchunks + GM_CHUNKS - 1) / GM_CHUNKS;

  auto tile = [&](int st, int which) { return tiles + (st * 3 + which) * GM_TILE_BYTES; };
  auto issue = [&](int kt, int st) {
    mbar_arrive_expect_tx(&full[st], 3 * GM_TILE_BYTES);
    tma_load_2d(tile(st, 0), &map_am, kt * GM_BKW, (int32_t)m0, &full[st]);
    tma_load_2d(tile(st, 1), &map_as, kt * GM_BKW, (int32_t)m0, &full[st]);
    tma_load_2d(tile(st, 2), &map_w, kt * GM_BKW, (int32_t)n0, &full[st]);
  };

  pdl_trigger();
  pdl_wait();
  if (tid == 0) {
    prefetch_tensormap(&map_am);
    prefetch_tensormap(&map_as);
    prefetch_tensormap(&map_w);
    for (int s = 0; s < GM_STAGES; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (tid == 0)
    for (int s = 0; s < GM_STAGES && s < KT; ++s) issue(s, s);

  int acc[GM_TI][GM_TJ];
  float y[GM_TI][GM_TJ];
  int prow[GM_TI];
#pragma unroll
  for (int i = 0; i < GM_TI; ++i) {
    prow[i] = 0;
#pragma unroll
    for (int j = 0; j < GM_TJ; ++j) {
      acc[i][j] = 0;
      y[i][j] = 0.0f;
    }
  }

  for (int kt = 0; kt < KT; ++kt) {
    const int st = kt % GM_STAGES;
    const bool ok = mbar_wait(&full[st], (kt / GM_STAGES) & 1);
    if (!__syncthreads_and(ok)) {
      if (tid == 0) {
        flag_status(d_status, BWTA_STATUS_TIMEOUT);
        // let the loads this CTA issued and has not consumed land before it exits
        for (int j = kt; j < KT && j < kt + GM_STAGES; ++j)
          mbar_wait(&full[j % GM_STAGES], (j / GM_STAGES) & 1, 100000000ull);
      }
      __syncthreads();
      return;
    }
    const uint8_t *Am = tile(st, 0), *As = tile(st, 1), *Wt = tile(st, 2);
    // per-chunk mask popcounts (shared by every weight row) and group scales
    for (int idx = tid; idx < GM_CHUNKS * GM_BM; idx += GM_THREADS) {
      const int c = idx >> 7, r = idx & 127;
      const uint4 v = *reinterpret_cast<const uint4 *>(Am + swz128(r, c));
      Pst[idx] = __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
      if (GROUPED) {
        const int gc = kt * GM_CHUNKS + c;
        const int64_t n = n0 + r;
        Ast[idx] = (gc < nchunks && n < N) ? __ldg(wscale + n * G + gc / gchunks) : 0.0f;
      }
    }
    __syncthreads();
    const int cmax = min(GM_CHUNKS, nchunks - kt * GM_CHUNKS);
    for (int c = 0; c < cmax; ++c) {
      uint4 wv[GM_TJ];
#pragma unroll
      for (int j = 0; j < GM_TJ; ++j)
        wv[j] = *reinterpret_cast<const uint4 *>(Wt + swz128(tx + 32 * j, c));
#pragma unroll
      for (int i = 0; i < GM_TI; ++i) {
        const int r = ty + 16 * i;
        const uint4 am = *reinterpret_cast<const uint4 *>(Am + swz128(r, c));
        const uint4 as = *reinterpret_cast<const uint4 *>(As + swz128(r, c));
        prow[i] += (int)Pst[c * GM_BM + r];
#pragma unroll
        for (int j = 0; j < GM_TJ; ++j) {
          acc[i][j] += popc4_csa(lop3_and_xor(am.x, as.x, wv[j].x), lop3_and_xor(am.y, as.y, wv[j].y),
                                 lop3_and_xor(am.z, as.z, wv[j].z), lop3_and_xor(am.w, as.w, wv[j].w));
        }
      }
      if (GROUPED) {
        const int gc = kt * GM_CHUNKS + c;
        if ((gc + 1) % gchunks == 0 || gc + 1 == nchunks) {
          float a[GM_TJ];
#pragma unroll
          for (int j = 0; j < GM_TJ; ++j) a[j] = Ast[c * GM_BN + tx + 32 * j];
#pragma unroll
          for (int i = 0; i < GM_TI; ++i) {
#pragma unroll
            for (int j = 0; j < GM_TJ; ++j) {
              const int d = prow[i] - 2 * acc[i][j];
              y[i][j] = fmaf(biased_int_to_float(d + INT_FLOAT_BIAS), a[j], y[i][j]);
              acc[i][j] = 0;
            }
            prow[i] = 0;
          }
        }
      }
    }
    __syncthreads();
    if (tid == 0 && kt + GM_STAGES < KT) issue(kt + GM_STAGES, st);
  }

  // epilogue: a warp stores 32 consecutive columns of one row per (i, j)
#pragma unroll
  for (int i = 0; i < GM_TI; ++i) {
    const int64_t row = m0 + ty + 16 * i;
    if (row >= M) continue;
    const float s = __ldg(ascale + row);
#pragma unroll
    for (int j = 0; j < GM_TJ; ++j) {
      const int64_t col = n0 + tx + 32 * j;
      if (col >= N) continue;
      if (GROUPED) {
        if (WANT_Y) Y[row * ldY + col] = y[i][j] * s;
      } else {
        const int d = prow[i] - 2 * acc[i][j];
        if (WANT_DOTS) dots[row * ldD + col] = d;
        if (WANT_Y) Y[row * ldY + col] = fmaf(__int2float_rn(d), __ldg(wscale + col), 0.0f) * s;
      }
    }
  }
}

template <bool GROUPED, bool WANT_Y, bool WANT_DOTS>
static cudaError_t launch_tiled_t(const CUtensorMap &mam, const CUtensorMap &mas,
                                  const CUtensorMap &mw, const float *ascale, const float *wscale,
                                  int64_t M, int64_t N, int nchunks, int gchunks, int64_t G,
                                  float *Y, int64_t ldY, int32_t *dots, int64_t ldD,
                                  int32_t *d_status, cudaStream_t s) {
  auto kern = k_gemm_tiled<GROUPED, WANT_Y, WANT_DOTS>;
  static cudaError_t attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)GM_SMEM);
  if (attr != cudaSuccess) return attr;
  dim3 grid((unsigned)ceil_div<int64_t>(N, GM_BN), (unsigned)ceil_div<int64_t>(M, GM_BM));
  return launch_pdl(kern, grid, dim3(GM_THREADS), GM_SMEM, s, mam, mas, mw, ascale, wscale, M, N,
                    nchunks, gchunks, G, Y, ldY, dots, ldD, d_status);
}

cudaError_t launch_gemm_tiled(const uint32_t *am, const uint32_t *as, const float *ascale,
                              int64_t M, int64_t lda, const uint32_t *wb, const float *wscale,
                              int64_t N, int64_t ldw, int64_t K, int64_t group, float *Y,
                              int64_t ldY, int32_t *dots, int64_t ldD, int32_t *d_status,
                              cudaStream_t s) {
  if (M == 0 || N == 0) return cudaSuccess;
  CUtensorMap mam, mas, mw;
  if (!make_plane_map(&mam, am, M, lda, GM_BKW, GM_BM) ||
      !make_plane_map(&mas, as, M, lda, GM_BKW, GM_BM) ||
      !make_plane_map(&mw, wb, N, ldw, GM_BKW, GM_BN))
    return cudaErrorInvalidValue;
  const int nchunks = (int)ceil_div<int64_t>(ceil_div<int64_t>(K, 32), 4);
  if (group == 0) {
    if (Y && dots)
      return launch_tiled_t<false, true, true>(mam, mas, mw, ascale, wscale, M, N, nchunks, nchunks,
                                               1, Y, ldY, dots, ldD, d_status, s);
    if (Y)
      return launch_tiled_t<false, true, false>(mam, mas, mw, ascale, wscale, M, N, nchunks,
                                                nchunks, 1, Y, ldY, dots, ldD, d_status, s);
    return launch_tiled_t<false, false, true>(mam, mas, mw, ascale, wscale, M, N, nchunks, nchunks,
                                              1, Y, ldY, dots, ldD, d_status, s);
  }
  const int gchunks = (int)(group / 128);
  const int64_t G = ceil_div<int64_t>(K, group);
  cudaError_t e = cudaSuccess;
  if (Y)
    e = launch_tiled_t<true, true, false>(mam, mas, mw, ascale, wscale, M, N, nchunks, gchunks, G,
                                          Y, ldY, nullptr, ldD, d_status, s);
  if (e == cudaSuccess && dots)  // full-K integer dots: the same kernel without groups
    e = launch_tiled_t<false, false, true>(mam, mas, mw, ascale, wscale, M, N, nchunks, nchunks, 1,
                                           nullptr, ldY, dots, ldD, d_status, s);
  return e;
}

// ================================================================ GEMV (K3)
// Decode: M <= 8 activation rows against all N weight rows. The activation
// planes and their per-chunk mask popcounts sit in shared memory. A warp owns
// GV_ROWS weight rows at a time and issues every 16-byte load of them (lane c
// reads chunk c, c + 32, ...: 512 contiguous bytes per warp-load) before it
// computes, so each lane keeps several loads in flight. Integer dots are
// reduced exactly with shuffles; grouped outputs accumulate
// alpha_g * d_chunk per lane in fp32 and reduce as a tree.
constexpr int GV_THREADS = 256, GV_WARPS = GV_THREADS / 32, GV_ROWS = 2;
constexpr int GV_MAX_CPL = 4;  // chunks per lane: K <= 32 * 4 * 128 = 16384
constexpr size_t GV_SMEM_MAX = 96 * 1024;

__device__ __forceinline__ uint4 ldg_stream(const uint32_t *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <int MR, int CPL, bool GROUPED, bool WANT_Y, bool WANT_DOTS>
__device__ __forceinline__ void gemv_load_rows(uint4 (&w)[GV_ROWS][CPL], float (&a)[GV_ROWS][CPL],
                                               const uint32_t *__restrict__ wb,
                                               const float *__restrict__ wscale, int64_t n0,
                                               int64_t N, int64_t ldw, int nchunks, int gchunks,
                                               int64_t G, int lane) {
#pragma unroll
  for (int r = 0; r < GV_ROWS; ++r)
#pragma unroll
    for (int q = 0; q < CPL; ++q) {
      const int c = lane + 32 * q;
      const int64_t n = n0 + r;
      const bool in = n < N && c < nchunks;
      w[r][q] = in ? ldg_stream(wb + n * ldw + 4 * c) : make_uint4(0, 0, 0, 0);
      a[r][q] = (GROUPED && in) ? __ldg(wscale + n * G + c / gchunks) : 0.0f;
    }
}

// Dots of GV_ROWS weight rows (already in registers) with the MR activation
// rows in shared memory; lane 0 writes the outputs.
template <int MR, int CPL, bool GROUPED>
__device__ __forceinline__ void gemv_rows(const uint4 (&w)[GV_ROWS][CPL], const float (&a)[GV_ROWS][CPL],
                                          const uint4 *sA, const uint4 *sS, const int *sP,
                                          const float *scale_m, int M, int64_t n0, int64_t N,
                                          int nchunks, int lane, const float *__restrict__ wscale,
                                          float *__restrict__ Y, int64_t ldY,
                                          int32_t *__restrict__ dots, int64_t ldD) {
#pragma unroll
  for (int r = 0; r < GV_ROWS; ++r) {
    const int64_t n = n0 + r;
    int dt[MR];
    float yp[MR];
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      dt[m] = 0;
      yp[m] = 0.0f;
    }
#pragma unroll
    for (int q = 0; q < CPL; ++q) {
      const int c = lane + 32 * q;
      if (c >= nchunks) break;
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        const uint4 A = sA[m * nchunks + c], S = sS[m * nchunks + c];
        const int cnt = popc4_csa(lop3_and_xor(A.x, S.x, w[r][q].x), lop3_and_xor(A.y, S.y, w[r][q].y),
                                  lop3_and_xor(A.z, S.z, w[r][q].z), lop3_and_xor(A.w, S.w, w[r][q].w));
        const int d = sP[m * nchunks + c] - 2 * cnt;
        dt[m] += d;
        if (GROUPED) yp[m] = fmaf(biased_int_to_float(d + INT_FLOAT_BIAS), a[r][q], yp[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < MR; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        dt[m] += __shfl_xor_sync(FULL, dt[m], o);
        if (GROUPED) yp[m] += __shfl_xor_sync(FULL, yp[m], o);
      }
    }
    if (lane == 0 && n < N) {
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        if (m >= M) break;
        if (dots) dots[m * ldD + n] = dt[m];
        if (Y)
          Y[m * ldY + n] = GROUPED ? yp[m] * scale_m[m]
                                   : fmaf(__int2float_rn(dt[m]), __ldg(wscale + n), 0.0f) * scale_m[m];
      }
    }
  }
}

// Stream this warp's row pairs n0, n0 + step, ... with a register double
// buffer: the next pair's loads are in flight while the current pair computes.
// wA holds the first pair on entry.
template <int MR, int CPL, bool GROUPED>
__device__ __forceinline__ void gemv_stream(uint4 (&wA)[GV_ROWS][CPL], float (&aA)[GV_ROWS][CPL],
                                            const uint4 *sA, const uint4 *sS, const int *sP,
                                            const float *scale_m, int M, int64_t n0, int64_t step,
                                            int64_t N, int64_t ldw, int nchunks, int gchunks,
                                            int64_t G, int lane, const uint32_t *__restrict__ wb,
                                            const float *__restrict__ wscale, float *__restrict__ Y,
                                            int64_t ldY, int32_t *__restrict__ dots, int64_t ldD) {
  uint4 wB[GV_ROWS][CPL];
  float aB[GV_ROWS][CPL];
  while (n0 < N) {
    const int64_t n1 = n0 + step;
    if (n1 < N) gemv_load_rows<MR, CPL, GROUPED, true, false>(wB, aB, wb, wscale, n1, N, ldw, nchunks, gchunks, G, lane);
    gemv_rows<MR, CPL, GROUPED>(wA, aA, sA, sS, sP, scale_m, M, n0, N, nchunks, lane, wscale, Y, ldY, dots, ldD);
    if (n1 >= N) break;
    const int64_t n2 = n1 + step;
    if (n2 < N) gemv_load_rows<MR, CPL, GROUPED, true, false>(wA, aA, wb, wscale, n2, N, ldw, nchunks, gchunks, G, lane);
    gemv_rows<MR, CPL, GROUPED>(wB, aB, sA, sS, sP, scale_m, M, n1, N, nchunks, lane, wscale, Y, ldY, dots, ldD);
    n0 = n2;
  }
}

// READY: the weights are complete before launch, so the first rows' weights
// are requested before waiting on the previous kernel (programmatic dependent
// launch); the activation planes are read only after the wait.
template <int MR, int CPL, bool GROUPED, bool WANT_Y, bool WANT_DOTS, bool READY>
__global__ void __launch_bounds__(GV_THREADS)
k_gemv(const uint32_t *__restrict__ am, const uint32_t *__restrict__ as,
       const float *__restrict__ ascale, int64_t lda, const uint32_t *__restrict__ wb,
       const float *__restrict__ wscale, int64_t N, int64_t ldw, int nchunks, int gchunks,
       int64_t G, float *__restrict__ Y, int64_t ldY, int32_t *__restrict__ dots, int64_t ldD) {
  extern __shared__ uint4 sm4[];
  uint4 *sA = sm4;
  uint4 *sS = sA + MR * nchunks;
  int *sP = reinterpret_cast<int *>(sS + MR * nchunks);
  float *ssc = reinterpret_cast<float *>(sP + MR * nchunks);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t step = (int64_t)gridDim.x * GV_WARPS * GV_ROWS;
  const int64_t n0 = ((int64_t)blockIdx.x * GV_WARPS + warp) * GV_ROWS;
  uint4 w[GV_ROWS][CPL];
  float a[GV_ROWS][CPL];
  pdl_trigger();
  if (READY) gemv_load_rows<MR, CPL, GROUPED, true, false>(w, a, wb, wscale, n0, N, ldw, nchunks, gchunks, G, lane);
  pdl_wait();
  if (!READY) gemv_load_rows<MR, CPL, GROUPED, true, false>(w, a, wb, wscale, n0, N, ldw, nchunks, gchunks, G, lane);
  for (int idx = threadIdx.x; idx < MR * nchunks; idx += GV_THREADS) {
    const int m = idx / nchunks, c = idx % nchunks;
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(am + m * lda) + c);
    sA[idx] = v;
    sS[idx] = __ldg(reinterpret_cast<const uint4 *>(as + m * lda) + c);
    sP[idx] = __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
  }
  for (int m = threadIdx.x; m < MR; m += GV_THREADS) ssc[m] = WANT_Y ? __ldg(ascale + m) : 0.0f;
  __syncthreads();
  gemv_stream<MR, CPL, GROUPED>(w, a, sA, sS, sP, ssc, MR, n0, step, N, ldw, nchunks, gchunks, G,
                                lane, wb, wscale, WANT_Y ? Y : nullptr, ldY,
                                WANT_DOTS ? dots : nullptr, ldD);
}

static size_t gemv_smem(int64_t M, int64_t K) {
  const int64_t nchunks = ceil_div<int64_t>(ceil_div<int64_t>(K, 32), 4);
  return (size_t)M * nchunks * (2 * 16 + 4) + M * 4;
}

// One resident wave: CTAs per SM from the occupancy calculator (per kernel
// and shared-memory size, cached), times the SM count.
template <typename Kern>
static int64_t resident_grid(Kern kern, size_t smem, int64_t want) {
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, GV_THREADS, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  return std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)per_sm * sms));
}

bool gemv_fits(int64_t M, int64_t lda, int64_t K, int64_t group) {
  (void)lda;
  (void)group;
  const int64_t nchunks = ceil_div<int64_t>(ceil_div<int64_t>(K, 32), 4);
  return M >= 1 && M <= 8 && nchunks <= 32 * GV_MAX_CPL && gemv_smem(M, K) <= GV_SMEM_MAX;
}

template <int MR, int CPL, bool GROUPED, bool WANT_Y, bool WANT_DOTS>
static cudaError_t launch_gemv_t(const uint32_t *am, const uint32_t *as, const float *ascale,
                                 int64_t lda, const uint32_t *wb, const float *wscale, int64_t N,
                                 int64_t ldw, int nchunks, int gchunks, int64_t G, float *Y,
                                 int64_t ldY, int32_t *dots, int64_t ldD, bool ready,
                                 cudaStream_t s) {
  auto kern = ready ? k_gemv<MR, CPL, GROUPED, WANT_Y, WANT_DOTS, true>
                    : k_gemv<MR, CPL, GROUPED, WANT_Y, WANT_DOTS, false>;
  static cudaError_t attr =
      cudaFuncSetAttribute(k_gemv<MR, CPL, GROUPED, WANT_Y, WANT_DOTS, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GV_SMEM_MAX);
  static cudaError_t attr2 =
      cudaFuncSetAttribute(k_gemv<MR, CPL, GROUPED, WANT_Y, WANT_DOTS, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GV_SMEM_MAX);
  if (attr != cudaSuccess) return attr;
  if (attr2 != cudaSuccess) return attr2;
  const size_t smem = (size_t)MR * nchunks * (2 * 16 + 4) + MR * 4;
  const int64_t blocks = resident_grid(kern, smem, ceil_div<int64_t>(N, GV_WARPS * GV_ROWS));
  return launch_pdl(kern, dim3((unsigned)blocks), dim3(GV_THREADS), smem, s, am, as, ascale, lda, wb,
                    wscale, N, ldw, nchunks, gchunks, G, Y, ldY, dots, ldD);
}

template <int MR, int CPL>
static cudaError_t launch_gemv_m(const uint32_t *am, const uint32_t *as, const float *ascale,
                                 int64_t lda, const uint32_t *wb, const float *wscale, int64_t N,
                                 int64_t ldw, int nchunks, int gchunks, int64_t G, bool grouped,
                                 float *Y, int64_t ldY, int32_t *dots, int64_t ldD, bool ready,
                                 cudaStream_t s) {
#define BWTA_GV(GR, WY, WD)                                                                      \
  return launch_gemv_t<MR, CPL, GR, WY, WD>(am, as, ascale, lda, wb, wscale, N, ldw, nchunks, gchunks, \
                                       G, Y, ldY, dots, ldD, ready, s)
  if (grouped) {
    if (Y && dots) BWTA_GV(true, true, true);
    if (Y) BWTA_GV(true, true, false);
    BWTA_GV(true, false, true);
  }
  if (Y && dots) BWTA_GV(false, true, true);
  if (Y) BWTA_GV(false, true, false);
  BWTA_GV(false, false, true);
#undef BWTA_GV
}

cudaError_t launch_gemv(const uint32_t *am, const uint32_t *as, const float *ascale, int64_t M,
                        int64_t lda, const uint32_t *wb, const float *wscale, int64_t N,
                        int64_t ldw, int64_t K, int64_t group, float *Y, int64_t ldY,
                        int32_t *dots, int64_t ldD, bool ready, cudaStream_t s) {
  if (N == 0 || M == 0) return cudaSuccess;
  // chunks holding data; padding words past K are never read
  const int nchunks = (int)ceil_div<int64_t>(ceil_div<int64_t>(K, 32), 4);
  const bool grouped = group != 0;
  const int gchunks = grouped ? (int)(group / 128) : nchunks;
  const int64_t G = grouped ? ceil_div<int64_t>(K, group) : 1;
  const int cpl = ceil_div(nchunks, 32);
  switch (M * 8 + cpl) {
#define BWTA_GVM(m)                                                                                  \
  case m * 8 + 1:                                                                                   \
    return launch_gemv_m<m, 1>(am, as, ascale, lda, wb, wscale, N, ldw, nchunks, gchunks, G, grouped, \
                               Y, ldY, dots, ldD, ready, s);                                               \
  case m * 8 + 2:                                                                                   \
    return launch_gemv_m<m, 2>(am, as, ascale, lda, wb, wscale, N, ldw, nchunks, gchunks, G, grouped, \
                               Y, ldY, dots, ldD, ready, s);                                               \
  case m * 8 + 3:                                                                                   \
    return launch_gemv_m<m, 3>(am, as, ascale, lda, wb, wscale, N, ldw, nchunks, gchunks, G, grouped, \
                               Y, ldY, dots, ldD, ready, s);                                               \
  case m * 8 + 4:                                                                                   \
    return launch_gemv_m<m, 4>(am, as, ascale, lda, wb, wscale, N, ldw, nchunks, gchunks, G, grouped, \
                               Y, ldY, dots, ldD, ready, s)
    BWTA_GVM(1);
    BWTA_GVM(2);
    BWTA_GVM(3);
    BWTA_GVM(4);
    BWTA_GVM(5);
    BWTA_GVM(6);
    BWTA_GVM(7);
    BWTA_GVM(8);
#undef BWTA_GVM
    default:
      return cudaErrorInvalidValue;
  }
}

// ===================================================== fused decode (K3')
// Decode with the activation packer folded in: every CTA ternarizes the M <= 8
// fp16 rows itself (the exact integer threshold of quant.cuh, so its planes
// and scales equal bwta_quantize_pack_acts' bit for bit) into shared memory,
// then streams its weight rows as k_gemv does. The redundant per-CTA
// ternarization reads the activation rows from L2; it replaces a separate,
// latency-bound launch and the round trip of the planes through memory. With
// READY the first weight rows are requested before the wait on the previous
// kernel, so their DRAM latency overlaps that kernel's tail.
template <int MR, int CPL, bool GROUPED, bool READY>
__global__ void __launch_bounds__(GV_THREADS)
k_linear_decode(const uint16_t *__restrict__ X, int M, int64_t K, int64_t ldX, int ternary, int vec,
                const uint32_t *__restrict__ wb, const float *__restrict__ wscale, int64_t N,
                int64_t ldw, int nchunks, int gchunks, int64_t G, float *__restrict__ Y,
                int64_t ldY, int32_t *__restrict__ dots, int64_t ldD, int32_t *d_status) {
  extern __shared__ uint4 sm4[];
  uint4 *sA = sm4;
  uint4 *sS = sA + MR * nchunks;
  int *sP = reinterpret_cast<int *>(sS + MR * nchunks);
  float *ssc = reinterpret_cast<float *>(sP + MR * nchunks);
  __shared__ uint64_t red[QA_THREADS / 32];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t step = (int64_t)gridDim.x * GV_WARPS * GV_ROWS;
  int64_t n0 = ((int64_t)blockIdx.x * GV_WARPS + warp) * GV_ROWS;
  uint4 w[GV_ROWS][CPL];
  float a[GV_ROWS][CPL];
  pdl_trigger();
  if (READY) gemv_load_rows<MR, CPL, GROUPED, true, false>(w, a, wb, wscale, n0, N, ldw, nchunks,
                                                           gchunks, G, lane);
  pdl_wait();
  if (!READY) gemv_load_rows<MR, CPL, GROUPED, true, false>(w, a, wb, wscale, n0, N, ldw, nchunks,
                                                            gchunks, G, lane);

  // ternarize (or binarize) the M rows: the whole CTA is one team of 256
  // threads, 16 chunks of 128 elements per step
  constexpr int CPS = QA_THREADS / 16;
  const int cg = threadIdx.x / 16, l16 = threadIdx.x % 16;
  const int steps = (nchunks + CPS - 1) / CPS;
  bool bad = false;
  for (int m = 0; m < MR; ++m) {
    uint32_t *mrow = reinterpret_cast<uint32_t *>(sA + m * nchunks);
    uint32_t *srow = reinterpret_cast<uint32_t *>(sS + m * nchunks);
    if (m >= M) {  // rows past M stay empty: zero planes give zero dots
      for (int idx = threadIdx.x; idx < nchunks; idx += GV_THREADS) {
        sA[m * nchunks + idx] = make_uint4(0, 0, 0, 0);
        sS[m * nchunks + idx] = make_uint4(0, 0, 0, 0);
      }
      if (threadIdx.x == 0) ssc[m] = 0.0f;
      continue;
    }
    const uint16_t *xr = X + m * ldX;
    uint4 regs[QA_NREG];
    uint64_t S = 0;
#pragma unroll
    for (int st = 0; st < QA_NREG; ++st) {
      if (st < steps) {
        const int64_t k0 = (int64_t)(st * CPS + cg) * 128 + l16 * 8;
        regs[st] = vec ? load_half8<true>(xr, k0, K, true) : load_half8<false>(xr, k0, K, true);
        S += sum_mag8(regs[st], bad);
      }
    }
    S = team_sum_u64<QA_THREADS>(S, red);
    const uint32_t hT = ternary ? mag_threshold_pattern(S / (uint64_t)(2 * K)) : 0u;
    uint64_t ks = 0, kn = 0;
#pragma unroll
    for (int st = 0; st < QA_NREG; ++st) {
      if (st < steps) {
        const int chunk = st * CPS + cg;
        const int64_t k0 = (int64_t)chunk * 128 + l16 * 8;
        uint32_t kb, sb;
        if (ternary) keep8<true>(regs[st], hT, k0, K, kb, sb, ks);
        else keep8<false>(regs[st], hT, k0, K, kb, sb, ks);
        kn += __popc(kb);
        store_chunk(kb, sb, mrow, srow, chunk, chunk < nchunks);
      }
    }
    if (ternary) {
      ks = team_sum_u64<QA_THREADS>(ks, red);
      kn = team_sum_u64<QA_THREADS>(kn, red);
      if (threadIdx.x == 0) ssc[m] = row_scale(ks, kn);
    } else if (threadIdx.x == 0) {
      ssc[m] = row_scale(S, (uint64_t)K);
    }
  }
  if (bad) flag_status(d_status, BWTA_STATUS_NONFINITE);
  __syncthreads();
  for (int idx = threadIdx.x; idx < MR * nchunks; idx += GV_THREADS) {
    const uint4 v = sA[idx];
    sP[idx] = __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
  }
  __syncthreads();

  gemv_stream<MR, CPL, GROUPED>(w, a, sA, sS, sP, ssc, M, n0, step, N, ldw, nchunks, gchunks, G,
                                lane, wb, wscale, Y, ldY, dots, ldD);
}

static size_t decode_smem(int MR, int nchunks) { return (size_t)MR * nchunks * (2 * 16 + 4) + MR * 4; }

bool linear_decode_fits(int64_t M, int64_t K) {
  const int64_t nchunks = ceil_div<int64_t>(ceil_div<int64_t>(K, 32), 4);
  return M >= 1 && M <= 8 && nchunks <= 32 * GV_MAX_CPL;
}

template <int MR, int CPL, bool GROUPED>
static cudaError_t launch_decode_t(const uint16_t *X, int M, int64_t K, int64_t ldX, int ternary,
                                   int vec, const uint32_t *wb, const float *wscale, int64_t N,
                                   int64_t ldw, int nchunks, int gchunks, int64_t G, float *Y,
                                   int64_t ldY, int32_t *dots, int64_t ldD, bool ready,
                                   int32_t *d_status, cudaStream_t s) {
  const size_t smem = decode_smem(MR, nchunks);
  const int64_t want = ceil_div<int64_t>(N, GV_WARPS * GV_ROWS);
  const int64_t blocks = ready ? resident_grid(k_linear_decode<MR, CPL, GROUPED, true>, smem, want)
                               : resident_grid(k_linear_decode<MR, CPL, GROUPED, false>, smem, want);
  if (ready)
    return launch_pdl(k_linear_decode<MR, CPL, GROUPED, true>, dim3((unsigned)blocks),
                      dim3(GV_THREADS), smem, s, X, M, K, ldX, ternary, vec, wb, wscale, N, ldw,
                      nchunks, gchunks, G, Y, ldY, dots, ldD, d_status);
  return launch_pdl(k_linear_decode<MR, CPL, GROUPED, false>, dim3((unsigned)blocks),
                    dim3(GV_THREADS), smem, s, X, M, K, ldX, ternary, vec, wb, wscale, N, ldw,
                    nchunks, gchunks, G, Y, ldY, dots, ldD, d_status);
}

template <int MR>
static cudaError_t launch_decode_m(const uint16_t *X, int M, int64_t K, int64_t ldX, int ternary,
                                   int vec, const uint32_t *wb, const float *wscale, int64_t N,
                                   int64_t ldw, int nchunks, int gchunks, int64_t G, bool grouped,
                                   float *Y, int64_t ldY, int32_t *dots, int64_t ldD, bool ready,
                                   int32_t *d_status, cudaStream_t s) {
  const int cpl = ceil_div(nchunks, 32);
#define BWTA_DC(C)                                                                                  \
  if (cpl == C)                                                                                     \
    return grouped ? launch_decode_t<MR, C, true>(X, M, K, ldX, ternary, vec, wb, wscale, N, ldw,   \
                                                  nchunks, gchunks, G, Y, ldY, dots, ldD, ready,    \
                                                  d_status, s)                                      \
                   : launch_decode_t<MR, C, false>(X, M, K, ldX, ternary, vec, wb, wscale, N, ldw,  \
                                                   nchunks, gchunks, G, Y, ldY, dots, ldD, ready,   \
                                                   d_status, s);
  BWTA_DC(1)
  BWTA_DC(2)
  BWTA_DC(3)
  BWTA_DC(4)
#undef BWTA_DC
  return cudaErrorInvalidValue;
}

cudaError_t launch_linear_decode(const uint16_t *X, int64_t M, int64_t K, int64_t ldX, int mode,
                                 const uint32_t *wb, const float *wscale, int64_t N, int64_t ldw,
                                 int64_t group, float *Y, int64_t ldY, int32_t *dots, int64_t ldD,
                                 bool ready, int32_t *d_status, cudaStream_t s) {
  if (N == 0 || M == 0) return cudaSuccess;
  const int nchunks = (int)ceil_div<int64_t>(ceil_div<int64_t>(K, 32), 4);
  const bool grouped = group != 0;
  const int gchunks = grouped ? (int)(group / 128) : nchunks;
  const int64_t G = grouped ? ceil_div<int64_t>(K, group) : 1;
  const int ternary = mode == BWTA_TERNARY;
  const int vec = (reinterpret_cast<uintptr_t>(X) & 15u) == 0 && ldX % 8 == 0;
  const int m = (int)M;
  if (M <= 1)
    return launch_decode_m<1>(X, m, K, ldX, ternary, vec, wb, wscale, N, ldw, nchunks, gchunks, G,
                              grouped, Y, ldY, dots, ldD, ready, d_status, s);
  if (M <= 2)
    return launch_decode_m<2>(X, m, K, ldX, ternary, vec, wb, wscale, N, ldw, nchunks, gchunks, G,
                              grouped, Y, ldY, dots, ldD, ready, d_status, s);
  if (M <= 4)
    return launch_decode_m<4>(X, m, K, ldX, ternary, vec, wb, wscale, N, ldw, nchunks, gchunks, G,
                              grouped, Y, ldY, dots, ldD, ready, d_status, s);
  return launch_decode_m<8>(X, m, K, ldX, ternary, vec, wb, wscale, N, ldw, nchunks, gchunks, G,
                            grouped, Y, ldY, dots, ldD, ready, d_status, s);
}

}  // namespace bwta
