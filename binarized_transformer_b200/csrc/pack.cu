// pack.cu -- weight binarize+pack (offline) and the fused activation
// ternarize+pack kernel that runs in front of every bit GEMM.
//
// BWTA: Accurate and Efficient Binarized Transformer by Algorithm-Hardware
// Co-design -- abstract: binary weights, activations ternarized by projecting
// tiny values to zero; Figure 6: 32 fp16 values packed into one 32-bit word.
#include "common.cuh"
#include "quant.cuh"

namespace bwta {

// ============================================================ weights (K0)
// One warp owns a strip of 32 rows and one scale group (grid y), and walks the
// group's columns in tiles of 32. Lane j
// loads column j of the 32 rows (32 coalesced 128-byte loads); a ballot per
// row yields that row's sign word. The scale needs sum|w| in ascending column
// order (fp64), so the tile is transposed through shared memory and lane r
// adds row r's 32 values one by one. Every row's scale therefore comes out of
// one fixed serial fp64 sum: it is reproducible bit for bit.
constexpr int PW_WARPS = 4;

__global__ void __launch_bounds__(PW_WARPS * 32)
k_pack_weights(const float *__restrict__ W, int64_t N, int64_t K, int64_t ldW, int64_t gs,
               int64_t G, uint32_t *__restrict__ wbits, int64_t ldw,
               float *__restrict__ wscale, int32_t *d_status) {
  __shared__ float tile[PW_WARPS][32][33];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row0 = ((int64_t)blockIdx.x * PW_WARPS + warp) * 32;
  if (row0 >= N) return;
  const int64_t my_row = row0 + lane;
  const bool my_valid = my_row < N;
  // blockIdx.y = the scale group this warp sums (its words only; the last
  // group also writes the zero padding words up to ldw). Group sizes are
  // multiples of 128 columns, so a group starts on a 4-word store boundary.
  double sum = 0.0;
  int64_t g = blockIdx.y, g_end = (g + 1) * gs < K ? (g + 1) * gs : K;  // group and its end column
  const int64_t w_stop = (g == G - 1) ? ldw : (g + 1) * gs / 32;
  uint32_t words[4];
  bool bad = false;
  for (int64_t w = g * gs / 32; w < w_stop; ++w) {
    const int64_t k = w * 32 + lane;
    uint32_t my_word = 0;
    if (w * 32 < K) {
      float v[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        const int64_t row = row0 + r;
        v[r] = (row < N && k < K) ? __ldg(W + row * ldW + k) : 0.0f;
      }
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        bad |= !isfinite(v[r]);
        const uint32_t word = __ballot_sync(FULL, v[r] < 0.0f);
        if (lane == r) my_word = word;
        tile[warp][r][lane] = v[r];
      }
      __syncwarp();
      const int64_t kmax = (w * 32 + 32 < K) ? 32 : (K - w * 32);
      for (int c = 0; c < kmax; ++c) {
        sum += fabs((double)tile[warp][lane][c]);
        const int64_t kk = w * 32 + c;
        if (kk + 1 == g_end) {  // group g complete
          if (my_valid) wscale[my_row * G + g] = (float)(sum / (double)(g_end - g * gs));
          sum = 0.0;
          ++g;
          g_end = (g + 1) * gs < K ? (g + 1) * gs : K;
        }
      }
      __syncwarp();
    }
    words[w & 3] = my_word;
    if ((w & 3) == 3 && my_valid) {
      *reinterpret_cast<uint4 *>(wbits + my_row * ldw + (w - 3)) =
          make_uint4(words[0], words[1], words[2], words[3]);
    }
  }
  if (bad) flag_status(d_status, BWTA_STATUS_NONFINITE);
}

cudaError_t launch_pack_weights(const float *W, int64_t N, int64_t K, int64_t ldW, int64_t group,
                                uint32_t *wbits, int64_t ldw, float *wscale, int32_t *d_status,
                                cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  const int64_t gs = group ? group : K;
  const int64_t G = ceil_div(K, gs);
  const int64_t warps = ceil_div<int64_t>(N, 32);
  const int64_t blocks = ceil_div<int64_t>(warps, PW_WARPS);
  return launch_pdl(k_pack_weights, dim3((unsigned)blocks, (unsigned)G), dim3(PW_WARPS * 32), 0, s, W, N, K, ldW,
                    gs, G, wbits, ldw, wscale, d_status);
}

// ======================================================== activations (K1)
// One "team" of T threads (a power of two, 16..256) owns one row. The row is
// cut into chunks of 128 elements = 4 words per plane; 16 lanes cover a chunk
// with one 16-byte load each (8 halves), so a team covers T/16 chunks per step.
//  pass 1: exact S = sum |x| in units of 2^-24 (uint64), team reduction;
//  pass 2: threshold T = floor(S / (2K)) turned into a 15-bit fp16 magnitude
//          pattern hT, so "keep" is one integer compare per element
//          (|x| > 0.5*mean|x|  <=>  2K*v > S  <=>  v > T  <=>  h > hT);
//          8-bit keep/sign patterns are merged across lanes with shuffles and
//          lane 0 of every 16 writes 4 words of each plane with one 128-bit store;
//  pass 3: exact sum of kept magnitudes and kept count -> fp32 scale, with
//          the same IEEE roundings as the definition (int64->fp64, fp64
//          divide, times 2^-24, fp64->fp32).
// The row stays in registers between the passes for rows up to 16 steps.
template <int T, bool TERNARY, bool VEC>
__global__ void __launch_bounds__(QA_THREADS)
k_quantize_pack_acts(const uint16_t *__restrict__ X, int64_t M, int64_t K, int64_t ldX,
                     uint32_t *__restrict__ mask, uint32_t *__restrict__ sign, int64_t lda,
                     float *__restrict__ scale, uint8_t *__restrict__ a8, int64_t ld8,
                     int32_t *d_status) {
  constexpr int TEAMS = QA_THREADS / T;
  constexpr int CPS = T / 16;  // chunks per step
  __shared__ uint64_t red[QA_THREADS / 32];
  pdl_trigger();
  pdl_wait();
  const int t = threadIdx.x % T;
  const int64_t row = (int64_t)blockIdx.x * TEAMS + threadIdx.x / T;
  const bool valid = row < M;
  const int C = (int)(lda / 4);
  const int steps = (C + CPS - 1) / CPS;
  const int cg = t / 16, l16 = t % 16;
  const uint16_t *xr = X + (valid ? row : 0) * ldX;

  // pass 1: exact sum of magnitudes
  uint4 regs[QA_NREG];
  uint64_t S = 0;
  bool bad = false;
#pragma unroll
  for (int s = 0; s < QA_NREG; ++s) {
    if (s < steps) {
      const int64_t k0 = (int64_t)(s * CPS + cg) * 128 + l16 * 8;
      regs[s] = load_half8<VEC>(xr, k0, K, valid);
      S += sum_mag8(regs[s], bad);
    }
  }
  for (int s = QA_NREG; s < steps; ++s) {
    const int64_t k0 = (int64_t)(s * CPS + cg) * 128 + l16 * 8;
    S += sum_mag8(load_half8<VEC>(xr, k0, K, valid), bad);
  }
  if (bad && valid) flag_status(d_status, BWTA_STATUS_NONFINITE);
  S = team_sum_u64<T>(S, red);

  // pass 2: threshold, bit planes, kept sums
  const uint32_t hT = TERNARY ? mag_threshold_pattern(S / (uint64_t)(2 * K)) : 0u;
  uint32_t *mrow = mask ? mask + (valid ? row : 0) * lda : nullptr;
  uint32_t *srow = sign ? sign + (valid ? row : 0) * lda : nullptr;
  uint64_t ks = 0, kn = 0;
#pragma unroll
  for (int s = 0; s < QA_NREG; ++s) {
    if (s < steps) {
      const int chunk = s * CPS + cg;
      const int64_t k0 = (int64_t)chunk * 128 + l16 * 8;
      uint32_t kb, sb;
      keep8<TERNARY>(regs[s], hT, k0, K, kb, sb, ks);
      kn += __popc(kb);
      store_chunk(kb, sb, mrow, srow, chunk, valid && chunk < C && mask,
                  (a8 && valid && chunk < C) ? a8 + row * ld8 + k0 : nullptr);
    }
  }
  for (int s = QA_NREG; s < steps; ++s) {
    const int chunk = s * CPS + cg;
    const int64_t k0 = (int64_t)chunk * 128 + l16 * 8;
    uint32_t kb, sb;
    keep8<TERNARY>(load_half8<VEC>(xr, k0, K, valid), hT, k0, K, kb, sb, ks);
    kn += __popc(kb);
    store_chunk(kb, sb, mrow, srow, chunk, valid && chunk < C && mask,
                (a8 && valid && chunk < C) ? a8 + row * ld8 + k0 : nullptr);
  }

  // pass 3: row scale
  if (TERNARY) {
    ks = team_sum_u64<T>(ks, red);
    kn = team_sum_u64<T>(kn, red);
    if (valid && t == 0) {
      float sc = 0.0f;
      if (kn) sc = __double2float_rn(__dmul_rn(__ddiv_rn(__ull2double_rn(ks), __ull2double_rn(kn)),
                                               0x1p-24));
      scale[row] = sc;
    }
  } else {
    if (valid && t == 0) {
      float sc = 0.0f;
      if (K) sc = __double2float_rn(__dmul_rn(__ddiv_rn(__ull2double_rn(S), __ll2double_rn(K)),
                                              0x1p-24));
      scale[row] = sc;
    }
  }
}

template <int T>
static cudaError_t launch_qa_t(const uint16_t *X, int64_t M, int64_t K, int64_t ldX, int mode,
                               uint32_t *mask, uint32_t *sign, int64_t lda, float *scale,
                               uint8_t *a8, int64_t ld8, int32_t *d_status, cudaStream_t s) {
  constexpr int TEAMS = QA_THREADS / T;
  const int64_t blocks = ceil_div<int64_t>(M, TEAMS);
  const bool vec = (reinterpret_cast<uintptr_t>(X) & 15u) == 0 && ldX % 8 == 0;
#define BWTA_QA(TER, V)                                                                          \
  return launch_pdl(k_quantize_pack_acts<T, TER, V>, dim3((unsigned)blocks), dim3(QA_THREADS), 0, s, \
                    X, M, K, ldX, mask, sign, lda, scale, a8, ld8, d_status)
  if (mode == BWTA_TERNARY) {
    if (vec) BWTA_QA(true, true);
    BWTA_QA(true, false);
  }
  if (vec) BWTA_QA(false, true);
  BWTA_QA(false, false);
#undef BWTA_QA
}

cudaError_t launch_quantize_pack_acts(const uint16_t *X, int64_t M, int64_t K, int64_t ldX,
                                      int mode, uint32_t *mask, uint32_t *sign, int64_t lda,
                                      float *scale, uint8_t *a8, int64_t ld8, int32_t *d_status,
                                      cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  const int64_t C = lda / 4;  // 128-element chunks per row
  // Threads per row. Few rows (decode): wide teams, for latency. Many rows
  // (prefill): the narrowest team that still holds its row in registers
  // (at most QA_NREG chunk steps per thread), so that more rows, and more
  // loads, are in flight per SM.
  int T;
  if (M < 1024) {
    T = C <= 1 ? 16 : C <= 2 ? 32 : C <= 4 ? 64 : C <= 8 ? 128 : 256;
  } else {
    T = 256;
    for (int t = 16; t < 256; t *= 2)
      if (ceil_div<int64_t>(C, t / 16) <= QA_NREG) {
        T = t;
        break;
      }
  }
  switch (T) {
    case 16: return launch_qa_t<16>(X, M, K, ldX, mode, mask, sign, lda, scale, a8, ld8, d_status, s);
    case 32: return launch_qa_t<32>(X, M, K, ldX, mode, mask, sign, lda, scale, a8, ld8, d_status, s);
    case 64: return launch_qa_t<64>(X, M, K, ldX, mode, mask, sign, lda, scale, a8, ld8, d_status, s);
    case 128: return launch_qa_t<128>(X, M, K, ldX, mode, mask, sign, lda, scale, a8, ld8, d_status, s);
    default: return launch_qa_t<256>(X, M, K, ldX, mode, mask, sign, lda, scale, a8, ld8, d_status, s);
  }
}

}  // namespace bwta
