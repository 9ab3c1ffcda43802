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
// each chunk's group (loaded into registers one k-tile ahead, so the staging
// does not wait on global memory); at the end of every weight group each
// thread folds its 32 integer dots into fp32 with acc = fma((float)d_g,
// alpha_g, acc), in group order, and the epilogue multiplies by the
// activation scale. With 128-column groups (G1: every chunk is a group) a
// chunk's dot goes straight into that fold, with no integer accumulator.
constexpr int GM_BM = 128, GM_BN = 128, GM_BKW = 32, GM_STAGES = 3, GM_THREADS = 512;
constexpr int GM_TI = 8, GM_TJ = 4;  // outputs per thread: rows ty + 16*i, columns tx + 32*j
constexpr int GM_CHUNKS = GM_BKW / 4;
constexpr int GM_TILE_WORDS = GM_BM * GM_BKW;
constexpr int GM_TILE_BYTES = GM_TILE_WORDS * 4;
constexpr size_t GM_SMEM = 1024 + (size_t)GM_STAGES * 3 * GM_TILE_BYTES +
                           2 * GM_CHUNKS * GM_BM * 4 + (GM_STAGES + 1) * 8;

template <bool GROUPED, bool WANT_Y, bool WANT_DOTS, bool G1>
__global__ void __launch_bounds__(GM_THREADS, 1)
k_gemm_tiled(const __grid_constant__ CUtensorMap map_am, const __grid_constant__ CUtensorMap map_as,
             const __grid_constant__ CUtensorMap map_w, const float *__restrict__ ascale,
             const float *__restrict__ wscale, int64_t M, int64_t N, int nchunks, int gchunks,
             int64_t G, float *__restrict__ Y, int64_t ldY, int32_t *__restrict__ dots,
             int64_t ldD, int32_t *d_status, uint64_t stall_ns) {
  static_assert(!(GROUPED && WANT_DOTS), "grouped dots come from the ungrouped pass");
  static_assert(!G1 || GROUPED, "G1 is the grouped kernel with one chunk per group");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *tiles = smem;
  uint32_t *Pst = reinterpret_cast<uint32_t *>(tiles + GM_STAGES * 3 * GM_TILE_BYTES);
  float *Ast = reinterpret_cast<float *>(Pst + GM_CHUNKS * GM_BM);
  uint64_t *full = reinterpret_cast<uint64_t *>(Ast + GM_CHUNKS * GM_BN);
  // A barrier nothing ever completes: with stall_ns != 0 (the failure-path
  // self-test) the first k-tile waits on it instead of on its load, so every
  // CTA runs into the timeout path below after stall_ns.
  uint64_t *stall = full + GM_STAGES;

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
    mbar_init(stall, 1);
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
  // this thread's weight scales of the next k-tile: entries idx = tid + 512 q
  // of the [chunk][weight row] staging table
  constexpr int AQ = GM_CHUNKS * GM_BN / GM_THREADS;
  float anext[AQ];
  auto load_scales = [&](int kt) {
#pragma unroll
    for (int q = 0; q < AQ; ++q) {
      const int idx = tid + GM_THREADS * q, c = idx >> 7, r = idx & 127;
      const int gc = kt * GM_CHUNKS + c;
      const int64_t n = n0 + r;
      anext[q] = (GROUPED && kt < KT && gc < nchunks && n < N) ? __ldg(wscale + n * G + gc / gchunks)
                                                               : 0.0f;
    }
  };
  if (GROUPED) load_scales(0);

  for (int kt = 0; kt < KT; ++kt) {
    const int st = kt % GM_STAGES;
    const bool ok = (stall_ns != 0 && kt == 0) ? mbar_wait(stall, 0, stall_ns)
                                               : mbar_wait(&full[st], (kt / GM_STAGES) & 1);
    if (!__syncthreads_and(ok)) {
      if (tid == 0) {
        // let the loads this CTA issued and has not consumed land before it
        // exits: k-tiles kt .. kt + GM_STAGES - 1 are the only ones in flight
        bool drained = true;
        for (int j = kt; j < KT && j < kt + GM_STAGES; ++j)
          drained &= mbar_wait(&full[j % GM_STAGES], (j / GM_STAGES) & 1, DRAIN_NS);
        flag_status(d_status, drained ? BWTA_STATUS_TIMEOUT : BWTA_STATUS_TIMEOUT | BWTA_STATUS_DRAIN);
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
    }
    if (GROUPED) {
#pragma unroll
      for (int q = 0; q < AQ; ++q) Ast[tid + GM_THREADS * q] = anext[q];
    }
    __syncthreads();
    if (GROUPED) load_scales(kt + 1);  // in flight while this k-tile is computed
    const int cmax = min(GM_CHUNKS, nchunks - kt * GM_CHUNKS);
    if (G1) {
      // every chunk is a weight group: its dot goes straight into the fold
      for (int c = 0; c < cmax; ++c) {
        uint4 wv[GM_TJ];
        float a[GM_TJ];
#pragma unroll
        for (int j = 0; j < GM_TJ; ++j) {
          wv[j] = *reinterpret_cast<const uint4 *>(Wt + swz128(tx + 32 * j, c));
          a[j] = Ast[c * GM_BN + tx + 32 * j];
        }
#pragma unroll
        for (int i = 0; i < GM_TI; ++i) {
          const int r = ty + 16 * i;
          const uint4 am = *reinterpret_cast<const uint4 *>(Am + swz128(r, c));
          const uint4 as = *reinterpret_cast<const uint4 *>(As + swz128(r, c));
          const int pb = (int)Pst[c * GM_BM + r] + INT_FLOAT_BIAS;
#pragma unroll
          for (int j = 0; j < GM_TJ; ++j) {
            const int cnt = popc4_csa(lop3_and_xor(am.x, as.x, wv[j].x), lop3_and_xor(am.y, as.y, wv[j].y),
                                      lop3_and_xor(am.z, as.z, wv[j].z), lop3_and_xor(am.w, as.w, wv[j].w));
            y[i][j] = fmaf(biased_int_to_float(pb - 2 * cnt), a[j], y[i][j]);
          }
        }
      }
      __syncthreads();
      if (tid == 0 && kt + GM_STAGES < KT) issue(kt + GM_STAGES, st);
      continue;
    }
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

template <bool GROUPED, bool WANT_Y, bool WANT_DOTS, bool G1 = false>
static cudaError_t launch_tiled_t(const CUtensorMap &mam, const CUtensorMap &mas,
                                  const CUtensorMap &mw, const float *ascale, const float *wscale,
                                  int64_t M, int64_t N, int nchunks, int gchunks, int64_t G,
                                  float *Y, int64_t ldY, int32_t *dots, int64_t ldD,
                                  int32_t *d_status, uint64_t stall_ns, cudaStream_t s) {
  auto kern = k_gemm_tiled<GROUPED, WANT_Y, WANT_DOTS, G1>;
  static SmemOptIn opt_in;
  if (cudaError_t e = opt_in(kern, (int)GM_SMEM)) return e;
  dim3 grid((unsigned)ceil_div<int64_t>(N, GM_BN), (unsigned)ceil_div<int64_t>(M, GM_BM));
  return launch_pdl(kern, grid, dim3(GM_THREADS), GM_SMEM, s, mam, mas, mw, ascale, wscale, M, N,
                    nchunks, gchunks, G, Y, ldY, dots, ldD, d_status, stall_ns);
}

cudaError_t launch_gemm_tiled(const uint32_t *am, const uint32_t *as, const float *ascale,
                              int64_t M, int64_t lda, const uint32_t *wb, const float *wscale,
                              int64_t N, int64_t ldw, int64_t K, int64_t group, float *Y,
                              int64_t ldY, int32_t *dots, int64_t ldD, int32_t *d_status,
                              uint64_t stall_ns, cudaStream_t s) {
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
                                               1, Y, ldY, dots, ldD, d_status, stall_ns, s);
    if (Y)
      return launch_tiled_t<false, true, false>(mam, mas, mw, ascale, wscale, M, N, nchunks,
                                                nchunks, 1, Y, ldY, dots, ldD, d_status, stall_ns, s);
    return launch_tiled_t<false, false, true>(mam, mas, mw, ascale, wscale, M, N, nchunks, nchunks,
                                              1, Y, ldY, dots, ldD, d_status, stall_ns, s);
  }
  const int gchunks = (int)(group / 128);
  const int64_t G = ceil_div<int64_t>(K, group);
  cudaError_t e = cudaSuccess;
  if (Y && gchunks == 1)
    e = launch_tiled_t<true, true, false, true>(mam, mas, mw, ascale, wscale, M, N, nchunks, gchunks,
                                                G, Y, ldY, nullptr, ldD, d_status, stall_ns, s);
  else if (Y)
    e = launch_tiled_t<true, true, false>(mam, mas, mw, ascale, wscale, M, N, nchunks, gchunks, G,
                                          Y, ldY, nullptr, ldD, d_status, stall_ns, s);
  if (e == cudaSuccess && dots)  // full-K integer dots: the same kernel without groups
    e = launch_tiled_t<false, false, true>(mam, mas, mw, ascale, wscale, M, N, nchunks, nchunks, 1,
                                           nullptr, ldY, dots, ldD, d_status, stall_ns, s);
  return e;
}

}  // namespace bwta
