// gemm.cu -- the bit-packed binary x ternary GEMM (prefill) and GEMV (decode).
//
// BWTA: Accurate and Efficient Binarized Transformer by Algorithm-Hardware
// Co-design -- abstract and "Core claim": a bit-packed MatMul of binary
// weights with ternary activations. Per 32-bit word of a row pair:
//     dot += popc(mask) - 2 * popc(mask & (a_sign ^ w_sign))
// since a nonzero activation and a weight agree in sign exactly where the
// sign bits are equal. popc(mask) does not depend on the weight row, so it is
// counted once per (activation row, 128-element chunk) and shared by a whole
// tile; the inner loop is one LOP3 (mask & (a ^ w)), one POPC and one add.
#include <algorithm>
#include <mutex>

#include "common.cuh"
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

// ============================================================ tiled GEMM (K2)
// CTA tile 128 (activation rows) x 128 (weight rows), K staged 32 words
// (1024 elements) at a time by TMA into a 3-deep ring of 128-byte-swizzled
// tiles (mask, sign, weight: 16 KB each). 256 threads; thread (ty, tx) owns
// rows ty + 16*i and columns tx + 16*j (i, j < 8): 16-byte shared loads of
// four K-words, conflict-free thanks to the swizzle. Per stage the CTA first
// counts popc(mask) per (row, 4-word chunk) and stages the weight scales of
// each chunk's group; at the end of every weight group each thread folds its
// 64 integer dots into fp32 with acc = fma((float)d_g, alpha_g, acc), in group
// order, and the epilogue multiplies by the activation scale.
constexpr int GM_BM = 128, GM_BN = 128, GM_BKW = 32, GM_STAGES = 3, GM_THREADS = 256;
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

  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int64_t m0 = (int64_t)blockIdx.y * GM_BM, n0 = (int64_t)blockIdx.x * GM_BN;
  const int KT = (nchunks + GM_CHUNKS - 1) / GM_CHUNKS;

  auto tile = [&](int st, int which) { return tiles + (st * 3 + which) * GM_TILE_BYTES; };
  auto issue = [&](int kt, int st) {
    mbar_arrive_expect_tx(&full[st], 3 * GM_TILE_BYTES);
    tma_load_2d(tile(st, 0), &map_am, kt * GM_BKW, (int32_t)m0, &full[st]);
    tma_load_2d(tile(st, 1), &map_as, kt * GM_BKW, (int32_t)m0, &full[st]);
    tma_load_2d(tile(st, 2), &map_w, kt * GM_BKW, (int32_t)n0, &full[st]);
  };

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

  int acc[8][8];
  float y[8][8];
  int prow[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    prow[i] = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      acc[i][j] = 0;
      y[i][j] = 0.0f;
    }
  }

  for (int kt = 0; kt < KT; ++kt) {
    const int st = kt % GM_STAGES;
    const bool ok = mbar_wait(&full[st], (kt / GM_STAGES) & 1);
    if (!__syncthreads_and(ok)) {
      if (tid == 0) flag_status(d_status, BWTA_STATUS_TIMEOUT);
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
      uint4 wv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) wv[j] = *reinterpret_cast<const uint4 *>(Wt + swz128(tx + 16 * j, c));
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = ty + 16 * i;
        const uint4 am = *reinterpret_cast<const uint4 *>(Am + swz128(r, c));
        const uint4 as = *reinterpret_cast<const uint4 *>(As + swz128(r, c));
        prow[i] += (int)Pst[c * GM_BM + r];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          acc[i][j] += __popc(lop3_and_xor(am.x, as.x, wv[j].x)) +
                       __popc(lop3_and_xor(am.y, as.y, wv[j].y)) +
                       __popc(lop3_and_xor(am.z, as.z, wv[j].z)) +
                       __popc(lop3_and_xor(am.w, as.w, wv[j].w));
        }
      }
      if (GROUPED) {
        const int gc = kt * GM_CHUNKS + c;
        if ((gc + 1) % gchunks == 0 || gc + 1 == nchunks) {
          float a[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) a[j] = Ast[c * GM_BN + tx + 16 * j];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
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

  // epilogue
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t row = m0 + ty + 16 * i;
    if (row >= M) continue;
    const float s = __ldg(ascale + row);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t col = n0 + tx + 16 * j;
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
  kern<<<grid, GM_THREADS, GM_SMEM, s>>>(mam, mas, mw, ascale, wscale, M, N, nchunks, gchunks, G,
                                         Y, ldY, dots, ldD, d_status);
  return cudaGetLastError();
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
// planes and their per-chunk mask popcounts sit in shared memory; one warp per
// weight row streams the row's bits with 16-byte loads (lane c reads chunk c,
// c + 32, ...), so a warp reads 512 contiguous bytes per step. Integer dots are
// reduced exactly with shuffles; grouped outputs accumulate
// alpha_g * d_chunk per lane in fp32 and reduce as a tree.
constexpr int GV_THREADS = 256, GV_WARPS = GV_THREADS / 32;
constexpr size_t GV_SMEM_MAX = 96 * 1024;

__device__ __forceinline__ uint4 ldg_stream(const uint32_t *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <int MR, bool GROUPED, bool WANT_Y, bool WANT_DOTS>
__global__ void __launch_bounds__(GV_THREADS)
k_gemv(const uint32_t *__restrict__ am, const uint32_t *__restrict__ as,
       const float *__restrict__ ascale, int64_t lda, const uint32_t *__restrict__ wb,
       const float *__restrict__ wscale, int64_t N, int64_t ldw, int nchunks, int gchunks,
       int64_t G, float *__restrict__ Y, int64_t ldY, int32_t *__restrict__ dots, int64_t ldD) {
  extern __shared__ uint4 sm4[];
  uint4 *sA = sm4;
  uint4 *sS = sA + MR * nchunks;
  int *sP = reinterpret_cast<int *>(sS + MR * nchunks);
  for (int idx = threadIdx.x; idx < MR * nchunks; idx += GV_THREADS) {
    const int m = idx / nchunks, c = idx % nchunks;
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(am + m * lda) + c);
    sA[idx] = v;
    sS[idx] = __ldg(reinterpret_cast<const uint4 *>(as + m * lda) + c);
    sP[idx] = __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
  }
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int64_t n = (int64_t)blockIdx.x * GV_WARPS + warp; n < N; n += (int64_t)gridDim.x * GV_WARPS) {
    int dt[MR];
    float yp[MR];
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      dt[m] = 0;
      yp[m] = 0.0f;
    }
    const uint32_t *wrow = wb + n * ldw;
    for (int c = lane; c < nchunks; c += 32) {
      const uint4 w = ldg_stream(wrow + 4 * c);
      const float a = GROUPED ? __ldg(wscale + n * G + c / gchunks) : 0.0f;
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        const uint4 A = sA[m * nchunks + c], S = sS[m * nchunks + c];
        const int cnt = __popc(lop3_and_xor(A.x, S.x, w.x)) + __popc(lop3_and_xor(A.y, S.y, w.y)) +
                        __popc(lop3_and_xor(A.z, S.z, w.z)) + __popc(lop3_and_xor(A.w, S.w, w.w));
        const int d = sP[m * nchunks + c] - 2 * cnt;
        dt[m] += d;
        if (GROUPED) yp[m] = fmaf(biased_int_to_float(d + INT_FLOAT_BIAS), a, yp[m]);
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
    if (lane == 0) {
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        if (WANT_DOTS) dots[m * ldD + n] = dt[m];
        if (WANT_Y) {
          const float s = __ldg(ascale + m);
          Y[m * ldY + n] = GROUPED ? yp[m] * s
                                   : fmaf(__int2float_rn(dt[m]), __ldg(wscale + n), 0.0f) * s;
        }
      }
    }
  }
}

static size_t gemv_smem(int64_t M, int64_t K) {
  const int64_t nchunks = ceil_div<int64_t>(ceil_div<int64_t>(K, 32), 4);
  return (size_t)M * nchunks * (2 * 16 + 4);
}

bool gemv_fits(int64_t M, int64_t lda, int64_t K, int64_t group) {
  (void)lda;
  (void)group;
  return M >= 1 && M <= 8 && gemv_smem(M, K) <= GV_SMEM_MAX;
}

template <int MR, bool GROUPED, bool WANT_Y, bool WANT_DOTS>
static cudaError_t launch_gemv_t(const uint32_t *am, const uint32_t *as, const float *ascale,
                                 int64_t lda, const uint32_t *wb, const float *wscale, int64_t N,
                                 int64_t ldw, int nchunks, int gchunks, int64_t G, float *Y,
                                 int64_t ldY, int32_t *dots, int64_t ldD, cudaStream_t s) {
  auto kern = k_gemv<MR, GROUPED, WANT_Y, WANT_DOTS>;
  static cudaError_t attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GV_SMEM_MAX);
  if (attr != cudaSuccess) return attr;
  const size_t smem = (size_t)MR * nchunks * (2 * 16 + 4);
  const int64_t blocks = std::min<int64_t>(ceil_div<int64_t>(N, GV_WARPS), 148 * 16);
  kern<<<(unsigned)blocks, GV_THREADS, smem, s>>>(am, as, ascale, lda, wb, wscale, N, ldw,
                                                  nchunks, gchunks, G, Y, ldY, dots, ldD);
  return cudaGetLastError();
}

template <int MR>
static cudaError_t launch_gemv_m(const uint32_t *am, const uint32_t *as, const float *ascale,
                                 int64_t lda, const uint32_t *wb, const float *wscale, int64_t N,
                                 int64_t ldw, int nchunks, int gchunks, int64_t G, bool grouped,
                                 float *Y, int64_t ldY, int32_t *dots, int64_t ldD,
                                 cudaStream_t s) {
#define BWTA_GV(GR, WY, WD)                                                                      \
  return launch_gemv_t<MR, GR, WY, WD>(am, as, ascale, lda, wb, wscale, N, ldw, nchunks, gchunks, \
                                       G, Y, ldY, dots, ldD, s)
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
                        int32_t *dots, int64_t ldD, cudaStream_t s) {
  if (N == 0 || M == 0) return cudaSuccess;
  // chunks holding data; padding words past K are never read
  const int nchunks = (int)ceil_div<int64_t>(ceil_div<int64_t>(K, 32), 4);
  const bool grouped = group != 0;
  const int gchunks = grouped ? (int)(group / 128) : nchunks;
  const int64_t G = grouped ? ceil_div<int64_t>(K, group) : 1;
  switch (M) {
#define BWTA_GVM(m) \
  case m:           \
    return launch_gemv_m<m>(am, as, ascale, lda, wb, wscale, N, ldw, nchunks, gchunks, G, grouped, Y, ldY, dots, ldD, s)
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

}  // namespace bwta
