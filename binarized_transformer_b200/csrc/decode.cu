// decode.cu -- the decode GEMV (M <= 8 activation rows): one launch for one
// projection or for a batch of independent projections, with the activations
// either already packed (bwta_gemm) or ternarized inside the kernel
// (bwta_linear_decode, bwta_linear_decode_batched).
//
// BWTA: Accurate and Efficient Binarized Transformer by Algorithm-Hardware
// Co-design -- abstract and "Core claim": the bit-packed MatMul of binary
// weights with ternary activations; at decode it streams the weight bits once,
// so it is bound by memory bandwidth. Per 32-bit word:
//     dot += popc(mask) - 2 * popc(mask & (a_sign ^ w_sign))
// and per weight group g of a row, in group order,
//     acc = fma((float)d_g, alpha_g, acc);  Y = acc * s_a
// -- the same fp32 operations, in the same order, as the tiled GEMM, so the
// outputs agree bit for bit.
//
// Work is cut into tiles of DC_T = 8 weight rows of one projection, handed out
// round-robin first across the CTAs, then across the warps of a CTA, so that
// every SM streams even when there are few tiles. A warp walks its tiles in
// slices of 32 chunks (128 elements = 4 words per plane) and banks of DC_P
// rows: lane c copies chunk c of each row of a bank (512 contiguous bytes per
// row and warp) and that chunk's weight scale into a per-warp shared-memory
// ring with cp.async, DC_RING banks ahead of the bank it computes. Each lane
// reads back only what it copied itself, so its own cp.async group wait is
// the only synchronisation, and no register is held by a load in flight.
// The integer dot of each (row, chunk) and the chunk's weight scale go to a
// per-warp shared-memory table [chunk][row]; when a slice is complete, lane r
// folds row r's chunks in order (sum a group's chunks, then one fma per
// group), so the serial fp32 order costs a few instructions per chunk rather
// than a shuffle per group.
#include <algorithm>

#include "common.cuh"
#include "quant.cuh"
#include "tma.cuh"

namespace bwta {

constexpr int DC_THREADS = 256, DC_WARPS = DC_THREADS / 32;
constexpr int DC_T = 8;  // weight rows per tile
constexpr int DC_P = 4;     // rows per bank
constexpr int DC_RING = 4;  // banks in flight per warp
static_assert(DC_T % DC_P == 0, "a bank never straddles a slice");
constexpr int DC_SLOT_BYTES = DC_P * 32 * (16 + 4);  // bits + scales of one bank
constexpr int DC_MAX_JOBS = 8;
constexpr int DC_MAX_CHUNKS = 128;  // K <= 16384 (fused ternarization keeps a row in registers)
constexpr size_t DC_MAX_ACT_SMEM = 48 * 1024;  // + rings (80 KB) + fold tables (<= 83 KB) <= 227 KB
constexpr int DC_STAGE_BYTES = 24 * 1024;  // fused: fp16 rows staged per round (at least one row)

struct DecodeJob {
  const uint16_t *X;            // fused: fp16 rows [M][ldX]
  int64_t ldX;
  const uint32_t *am, *as;      // planes: [M][lda] words
  const float *ascale;
  int64_t lda;
  const uint32_t *wb;           // [N][ldw] weight sign words
  const float *ws;              // [N][G] scales
  int64_t N, ldw, G, K;
  float *Y;
  int64_t ldY;
  int32_t *dots;
  int64_t ldD;
  int64_t tile0;                // first global tile of this job
  int M, nchunks, gchunks, nslices;
  int act_off;                  // byte offset of the job's planes in shared memory
  int vec;                      // X rows 16-byte aligned
};

struct DecodeBatch {
  DecodeJob job[DC_MAX_JOBS];
  int64_t ntiles;
  int njobs, fused, ternary, ready;
  int ring_off;                 // byte offset of the per-warp cp.async rings
  int fold_off;                 // byte offset of the per-warp fold tables
  int stage_off, stage_pieces;  // fused: fp16 staging area (16-byte pieces), over the fold tables
};

// Shared-memory planes of one job: sA [M][nchunks] uint4 (mask), sS (sign),
// sP [M][nchunks] int (popc of the mask chunk), ssc [M] fp32 (scale).
struct JobActs {
  const uint4 *sA, *sS;
  const int *sP;
  const float *ssc;
};
__device__ __forceinline__ JobActs job_acts(uint8_t *smem, const DecodeJob &J) {
  uint4 *a = reinterpret_cast<uint4 *>(smem + J.act_off);
  uint4 *s = a + J.M * J.nchunks;
  int *p = reinterpret_cast<int *>(s + J.M * J.nchunks);
  return {a, s, p, reinterpret_cast<float *>(p + J.M * J.nchunks)};
}

// Position of a warp in its stream of (tile, slice, row) items.
struct DcCursor {
  int64_t tile, n0;
  int j, q, r;
  int c, g;  // this lane's chunk in the slice (32q + lane) and its weight group

  __device__ void locate(const DecodeBatch &p, int lane) {
    j = 0;
    while (j + 1 < p.njobs && tile >= p.job[j + 1].tile0) ++j;
    n0 = (tile - p.job[j].tile0) * DC_T;
    set_chunk(p, lane);
  }
  __device__ void set_chunk(const DecodeBatch &p, int lane) {
    c = 32 * q + lane;
    g = c / p.job[j].gchunks;
  }
  __device__ void advance(const DecodeBatch &p, int64_t stride, int lane) {
    r += DC_P;
    if (r < DC_T) return;
    r = 0;
    if (++q < p.job[j].nslices) {
      set_chunk(p, lane);
      return;
    }
    q = 0;
    tile += stride;
    if (tile < p.ntiles) locate(p, lane);
  }
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
  // copies src_bytes (0..16) and fills the rest of the 16 bytes with zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_addr(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// One ring slot: bits [DC_P][32 lanes] uint4, then scales [DC_P][32] fp32.
struct DcSlot {
  uint4 *bits;
  float *alpha;
};
__device__ __forceinline__ DcSlot dc_slot(uint8_t *ring, int k, int lane) {
  uint8_t *b = ring + k * DC_SLOT_BYTES;
  return {reinterpret_cast<uint4 *>(b) + lane,
          reinterpret_cast<float *>(b + DC_P * 32 * 16) + lane};
}

// Copy this lane's chunk of the bank at `cur` (rows r .. r + DC_P - 1) into
// its ring slot and close one cp.async group (empty when there is no bank):
// rows past N and chunks past K arrive as zeros.
__device__ __forceinline__ void dc_issue(const DecodeBatch &p, const DcCursor &cur, DcSlot sl) {
  if (cur.tile < p.ntiles) {
    const DecodeJob &J = p.job[cur.j];
    const bool cin = cur.c < J.nchunks;
#pragma unroll
    for (int i = 0; i < DC_P; ++i) {
      const int64_t n = cur.n0 + cur.r + i;
      const bool in = cin && n < J.N;
      cp_async16(sl.bits + i * 32, in ? J.wb + n * J.ldw + 4 * cur.c : J.wb, in ? 16u : 0u);
      if (J.Y) cp_async4(sl.alpha + i * 32, in ? J.ws + n * J.G + cur.g : J.ws, in ? 4u : 0u);
    }
  }
  cp_async_commit();
}

// Per-warp fold table: dots [MR][32 chunks][DC_T + 1] int, then scales
// [32][DC_T + 1] fp32 (odd row stride: conflict-free by chunk and by row).
template <int MR>
__host__ __device__ constexpr int dc_fold_bytes() {
  return (MR + 1) * 32 * (DC_T + 1) * 4;
}

// Running fold of the rows of the current tile (lane r < DC_T owns row r).
template <int MR>
struct DcFold {
  float acc[MR];
  int gd[MR], dt[MR];
  int gleft;  // chunks left in the current weight group

  __device__ void reset(int gchunks) {
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      acc[m] = 0.0f;
      gd[m] = 0;
      dt[m] = 0;
    }
    gleft = gchunks;
  }
};

template <int MR>
__device__ __forceinline__ void dc_compute(const DecodeBatch &p, uint8_t *smem, int *fold_d,
                                           float *fold_a, const DcCursor &cur, DcSlot sl,
                                           DcFold<MR> &f, int lane) {
  const DecodeJob &J = p.job[cur.j];
  const JobActs acts = job_acts(smem, J);
  const bool cin = cur.c < J.nchunks;
  uint4 w[DC_P];
  float a[DC_P];
#pragma unroll
  for (int i = 0; i < DC_P; ++i) {
    w[i] = sl.bits[i * 32];
    a[i] = J.Y ? sl.alpha[i * 32] : 0.0f;
  }
  // integer dots of this bank's rows with every activation row
#pragma unroll
  for (int i = 0; i < DC_P; ++i) {
    const int r = cur.r + i;
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      int d = 0;
      if (cin && m < J.M) {
        const uint4 A = acts.sA[m * J.nchunks + cur.c], S = acts.sS[m * J.nchunks + cur.c];
        d = acts.sP[m * J.nchunks + cur.c] -
            2 * popc4_csa(lop3_and_xor(A.x, S.x, w[i].x), lop3_and_xor(A.y, S.y, w[i].y),
                          lop3_and_xor(A.z, S.z, w[i].z), lop3_and_xor(A.w, S.w, w[i].w));
      }
      fold_d[(m * 32 + lane) * (DC_T + 1) + r] = d;
    }
    fold_a[lane * (DC_T + 1) + r] = a[i];
  }
  if (cur.r + DC_P < DC_T) return;

  // the slice is complete: lane r folds row r's chunks in order
  __syncwarp();
  const int cnt = min(32, J.nchunks - 32 * cur.q);
  if (lane < DC_T) {
    // eight chunks at a time: their table loads are issued together
    for (int c8 = 0; c8 < cnt; c8 += 8) {
      int dv[8][MR];
      float av[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int cc = min(c8 + u, 31);
#pragma unroll
        for (int m = 0; m < MR; ++m) dv[u][m] = fold_d[(m * 32 + cc) * (DC_T + 1) + lane];
        av[u] = fold_a[cc * (DC_T + 1) + lane];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (c8 + u >= cnt) break;
#pragma unroll
        for (int m = 0; m < MR; ++m) f.gd[m] += dv[u][m];
        if (--f.gleft == 0 || 32 * cur.q + c8 + u + 1 == J.nchunks) {
#pragma unroll
          for (int m = 0; m < MR; ++m) {
            f.acc[m] = fmaf(biased_int_to_float(f.gd[m] + INT_FLOAT_BIAS), av[u], f.acc[m]);
            f.dt[m] += f.gd[m];
            f.gd[m] = 0;
          }
          f.gleft = J.gchunks;
        }
      }
    }
  }
  __syncwarp();
  if (cur.q + 1 < J.nslices) return;

  // the tile is complete: row n0 + lane
  const int64_t n = cur.n0 + lane;
  if (lane < DC_T && n < J.N) {
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      if (m >= J.M) break;
      if (J.Y) J.Y[m * J.ldY + n] = f.acc[m] * acts.ssc[m];
      if (J.dots) J.dots[m * J.ldD + n] = f.dt[m];
    }
  }
}

// Planes of every job into shared memory: copied (bit-plane input) or made
// here from the fp16 rows with the exact integer threshold of quant.cuh (the
// same planes and scales as bwta_quantize_pack_acts, bit for bit). For the
// latter the rows are first copied into a staging area with cp.async -- as
// many rows per round as fit, so that one memory latency covers them -- and
// the whole CTA is then one team of 256 threads per row: piece p (8 halves)
// of a row belongs to thread p % 256, and 16 consecutive threads cover one
// 128-element chunk.
template <bool FUSED>
__device__ __forceinline__ void dc_setup_acts(const DecodeBatch &p, uint8_t *smem, int32_t *d_status) {
  __shared__ uint64_t red[QA_THREADS / 32];
  if (!FUSED) {
    for (int j = 0; j < p.njobs; ++j) {
      const DecodeJob &J = p.job[j];
      uint4 *sA = reinterpret_cast<uint4 *>(smem + J.act_off);
      uint4 *sS = sA + J.M * J.nchunks;
      int *sP = reinterpret_cast<int *>(sS + J.M * J.nchunks);
      float *ssc = reinterpret_cast<float *>(sP + J.M * J.nchunks);
      const int nch = J.nchunks;
      for (int idx = threadIdx.x; idx < J.M * nch; idx += DC_THREADS) {
        const int m = idx / nch, c = idx % nch;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(J.am + m * J.lda) + c);
        sA[idx] = v;
        sS[idx] = __ldg(reinterpret_cast<const uint4 *>(J.as + m * J.lda) + c);
        sP[idx] = __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
      }
      for (int m = threadIdx.x; m < J.M; m += DC_THREADS) ssc[m] = J.ascale ? __ldg(J.ascale + m) : 0.0f;
    }
    return;
  }
  uint4 *stage = reinterpret_cast<uint4 *>(smem + p.stage_off);
  bool bad = false;
  int j = 0, m = 0;  // next row to stage
  while (j < p.njobs) {
    // one round: stage rows (j, m) ... while they fit
    const int j0 = j, m0 = m;
    int used = 0;  // pieces of 16 bytes
    while (j < p.njobs) {
      const DecodeJob &J = p.job[j];
      const int pieces = J.nchunks * 16;
      if (used > 0 && used + pieces > p.stage_pieces) break;
      const uint16_t *xr = J.X + m * J.ldX;
      const int64_t K = J.K;
      for (int q = threadIdx.x; q < pieces; q += DC_THREADS) {
        const int64_t k0 = (int64_t)q * 8;
        uint4 *dst = stage + used + q;
        if (k0 >= K) {
          *dst = make_uint4(0, 0, 0, 0);
        } else if (J.vec) {
          cp_async16(dst, xr + k0, (uint32_t)(K - k0 >= 8 ? 16 : (K - k0) * 2));
        } else {
          *dst = load_half8<false>(xr, k0, K, true);
        }
      }
      used += pieces;
      if (++m == J.M) {
        m = 0;
        ++j;
      }
    }
    cp_async_wait_all();
    __syncthreads();
    // ternarize the staged rows
    int off = 0;
    for (int jj = j0, mm = m0; off < used;) {
      const DecodeJob &J = p.job[jj];
      const int nch = J.nchunks, steps = (nch + 15) / 16;
      const int64_t K = J.K;
      uint4 *sA = reinterpret_cast<uint4 *>(smem + J.act_off);
      uint4 *sS = sA + J.M * nch;
      float *ssc = reinterpret_cast<float *>(reinterpret_cast<int *>(sS + J.M * nch) + J.M * nch);
      uint32_t *mrow = reinterpret_cast<uint32_t *>(sA + mm * nch);
      uint32_t *srow = reinterpret_cast<uint32_t *>(sS + mm * nch);
      const uint4 *row = stage + off;
      uint64_t S = 0;
      for (int st = 0; st < steps; ++st) {
        const int q = st * DC_THREADS + threadIdx.x;
        if (q < nch * 16) S += sum_mag8(row[q], bad);
      }
      S = team_sum_u64<QA_THREADS>(S, red);
      const uint32_t hT = p.ternary ? mag_threshold_pattern(S / (uint64_t)(2 * K)) : 0u;
      uint64_t ks = 0, kn = 0;
      for (int st = 0; st < steps; ++st) {  // uniform trip count: store_chunk shuffles
        const int q = st * DC_THREADS + threadIdx.x, chunk = q / 16;
        const uint4 v = q < nch * 16 ? row[q] : make_uint4(0, 0, 0, 0);
        const int64_t k0 = (int64_t)q * 8;
        uint32_t kb, sb;
        if (p.ternary) keep8<true>(v, hT, k0, K, kb, sb, ks);
        else keep8<false>(v, hT, k0, K, kb, sb, ks);
        kn += __popc(kb);
        store_chunk(kb, sb, mrow, srow, chunk, chunk < nch);
      }
      if (p.ternary) {
        ks = team_sum_u64<QA_THREADS>(ks, red);
        kn = team_sum_u64<QA_THREADS>(kn, red);
        if (threadIdx.x == 0) ssc[mm] = row_scale(ks, kn);
      } else if (threadIdx.x == 0) {
        ssc[mm] = row_scale(S, (uint64_t)K);
      }
      off += nch * 16;
      if (++mm == J.M) {
        mm = 0;
        ++jj;
      }
    }
    __syncthreads();  // the staging area is free again; the planes are written
  }
  // popcounts of the mask chunks
  for (int jj = 0; jj < p.njobs; ++jj) {
    const DecodeJob &J = p.job[jj];
    const uint4 *sA = reinterpret_cast<const uint4 *>(smem + J.act_off);
    int *sP = reinterpret_cast<int *>(const_cast<uint4 *>(sA) + 2 * J.M * J.nchunks);
    for (int idx = threadIdx.x; idx < J.M * J.nchunks; idx += DC_THREADS) {
      const uint4 v = sA[idx];
      sP[idx] = __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
    }
  }
  if (bad) flag_status(d_status, BWTA_STATUS_NONFINITE);
}

template <int MR, bool FUSED>
__global__ void __launch_bounds__(DC_THREADS, 2)
k_decode(const __grid_constant__ DecodeBatch p, int32_t *d_status) {
  extern __shared__ uint4 dc_smem4[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(dc_smem4);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int *fold_d = reinterpret_cast<int *>(smem + p.fold_off + warp * dc_fold_bytes<MR>());
  float *fold_a = reinterpret_cast<float *>(fold_d + MR * 32 * (DC_T + 1));
  uint8_t *ring = smem + p.ring_off + warp * (DC_RING * DC_SLOT_BYTES);
  // tiles go round-robin over the CTAs first, then over the warps of a CTA
  const int64_t stride = (int64_t)gridDim.x * DC_WARPS;

  DcCursor ld, cur;  // the bank being copied, the bank being computed
  ld.tile = (int64_t)warp * gridDim.x + blockIdx.x;
  ld.q = 0;
  ld.r = 0;
  if (ld.tile < p.ntiles) ld.locate(p, lane);
  cur = ld;

  pdl_trigger();
  // with the weights known to be complete, the first banks are requested
  // before waiting for the previous kernel in the stream (its CTAs may still
  // be running on this SM: one CTA per SM leaves room for the next kernel's)
  for (int pass = 0; pass < 2; ++pass) {
    if (pass == 1) pdl_wait();
    if ((pass == 0) != (p.ready != 0)) continue;
#pragma unroll 1
    for (int k = 0; k < DC_RING; ++k) {
      dc_issue(p, ld, dc_slot(ring, k, lane));
      if (ld.tile < p.ntiles) ld.advance(p, stride, lane);
    }
  }
  dc_setup_acts<FUSED>(p, smem, d_status);
  __syncthreads();

  // the fold restarts at the first bank of every tile (slice 0, row 0)
  DcFold<MR> f;
  for (int k = 0; cur.tile < p.ntiles; k = (k + 1 == DC_RING) ? 0 : k + 1) {
    if (cur.q == 0 && cur.r == 0) f.reset(p.job[cur.j].gchunks);
    cp_async_wait<DC_RING - 1>();  // this lane's copies of bank `cur` have landed
    const DcSlot sl = dc_slot(ring, k, lane);
    dc_compute<MR>(p, smem, fold_d, fold_a, cur, sl, f, lane);
    dc_issue(p, ld, sl);           // the slot is free again: the bank DC_RING ahead
    if (ld.tile < p.ntiles) ld.advance(p, stride, lane);
    cur.advance(p, stride, lane);
  }
  cp_async_wait<0>();
}

// ------------------------------------------------------------------ host
static size_t dc_act_bytes(int M, int nchunks) {
  return ((size_t)M * nchunks * 36 + (size_t)M * 4 + 15) / 16 * 16;
}

bool decode_fits(int64_t M, int64_t K) {
  const int64_t nchunks = ceil_div<int64_t>(ceil_div<int64_t>(K, 32), 4);
  return M >= 1 && M <= 8 && nchunks <= DC_MAX_CHUNKS &&
         dc_act_bytes((int)M, (int)nchunks) <= DC_MAX_ACT_SMEM;
}

template <int MR, bool FUSED>
static cudaError_t launch_decode_t(const DecodeBatch &p, size_t smem, int32_t *d_status,
                                   cudaStream_t s) {
  auto kern = k_decode<MR, FUSED>;
  static SmemOptIn opt_in;
  if (cudaError_t e = opt_in(kern, (int)smem)) return e;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, DC_THREADS, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  // One CTA per SM when the tiles do not fill two CTAs' warps on every SM:
  // the SM then keeps room for a CTA of the next kernel in the stream, which
  // starts its weight loads early. Long streams get two CTAs per SM (twice the
  // loads in flight). Tiles go to CTAs first, so every SM streams.
  const int64_t per = (p.ntiles > (int64_t)2 * sms * DC_WARPS && per_sm >= 2) ? 2 : 1;
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(p.ntiles, per * sms));
  return launch_pdl(kern, dim3((unsigned)blocks), dim3(DC_THREADS), smem, s, p, d_status);
}

cudaError_t launch_decode(const DecodeSpec *jobs, int njobs, bool fused, int mode, bool ready,
                          int32_t *d_status, cudaStream_t s) {
  DecodeBatch p = {};
  int MR = 1;
  size_t act = 0;
  int nj = 0;
  for (int i = 0; i < njobs; ++i) {
    const DecodeSpec &in = jobs[i];
    if (in.M == 0 || in.N == 0) continue;
    DecodeJob &J = p.job[nj];
    J.X = in.X;
    J.ldX = in.ldX;
    J.am = in.am;
    J.as = in.as;
    J.ascale = in.ascale;
    J.lda = in.lda;
    J.wb = in.wbits;
    J.ws = in.wscale;
    J.N = in.N;
    J.ldw = in.ldw;
    J.K = in.K;
    J.Y = in.Y;
    J.ldY = in.ldY;
    J.dots = in.dots;
    J.ldD = in.ldD;
    J.M = (int)in.M;
    J.nchunks = (int)ceil_div<int64_t>(ceil_div<int64_t>(in.K, 32), 4);
    J.gchunks = in.group ? (int)(in.group / 128) : J.nchunks;
    J.G = in.group ? ceil_div<int64_t>(in.K, in.group) : 1;
    J.nslices = ceil_div(J.nchunks, 32);
    J.vec = (reinterpret_cast<uintptr_t>(in.X) & 15u) == 0 && in.ldX % 8 == 0;
    J.act_off = (int)act;
    act += dc_act_bytes(J.M, J.nchunks);
    J.tile0 = p.ntiles;
    p.ntiles += ceil_div<int64_t>(in.N, DC_T);
    MR = std::max(MR, J.M);
    ++nj;
  }
  if (nj == 0) return cudaSuccess;
  if (act > DC_MAX_ACT_SMEM) return cudaErrorInvalidValue;
  p.njobs = nj;
  p.fused = fused;
  p.ternary = mode == BWTA_TERNARY;
  p.ready = ready;
  p.ring_off = (int)act;
  const size_t ring = (size_t)DC_WARPS * DC_RING * DC_SLOT_BYTES;
  p.fold_off = (int)(act + ring);
  const size_t fold = (size_t)DC_WARPS * (MR <= 1 ? dc_fold_bytes<1>() : MR <= 2 ? dc_fold_bytes<2>()
                                          : MR <= 4 ? dc_fold_bytes<4>() : dc_fold_bytes<8>());
  size_t stage = 0;
  if (fused) {  // every staged row fits; as many rows per round as DC_STAGE_BYTES holds
    size_t rows_bytes = 0, row_max = 0;
    for (int i = 0; i < nj; ++i) {
      const size_t rb = (size_t)p.job[i].nchunks * 256;
      rows_bytes += rb * p.job[i].M;
      row_max = std::max(row_max, rb);
    }
    stage = std::max(row_max, std::min(rows_bytes, (size_t)DC_STAGE_BYTES));
  }
  // the staging area is used only before the main loop: it shares the space
  // of the fold tables (not of the rings, whose first copies are in flight)
  p.stage_off = p.fold_off;
  p.stage_pieces = (int)(stage / 16);
  const size_t smem = act + ring + std::max(fold, stage);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
#define BWTA_DC(R)                                                                              \
  return fused ? launch_decode_t<R, true>(p, smem, d_status, s)                                 \
               : launch_decode_t<R, false>(p, smem, d_status, s)
  if (MR <= 1) BWTA_DC(1);
  if (MR <= 2) BWTA_DC(2);
  if (MR <= 4) BWTA_DC(4);
  BWTA_DC(8);
#undef BWTA_DC
}

int decode_max_jobs() { return DC_MAX_JOBS; }

size_t decode_act_bytes(int64_t M, int64_t K) {
  return dc_act_bytes((int)M, (int)ceil_div<int64_t>(ceil_div<int64_t>(K, 32), 4));
}

size_t decode_max_act_bytes() { return DC_MAX_ACT_SMEM; }

}  // namespace bwta
