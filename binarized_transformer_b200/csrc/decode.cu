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
// Work is cut into tiles of R weight rows of one projection (R = 32 when two
// such tiles fit the copy ring and at most two activation rows are batched,
// else 16); a CTA takes tiles blockIdx.x, blockIdx.x + gridDim.x, ... (all
// of a tile's K at once). Every wait and release below is per tile, so the
// taller tile halves their count per row. Warp roles:
//  * the copy warp (one thread) brings each tile into a ring of shared-memory
//    stages with two bulk copies -- the tile's rows of sign words are one
//    contiguous block (rows are ldw words apart), and so are its rows of
//    weight scales -- completing on the stage's mbarrier; with the weights
//    known to be complete it fills the ring before the kernel waits for the
//    previous kernel in the stream;
//  * eight dot warps compute the integer dots: warp w takes rows R/8 w ...
//    R/8 (w + 1) - 1 of the tile, lane c the 128-element chunks c, c + 32, ... (16
//    contiguous bytes per lane, conflict-free), and write each chunk's dot
//    (int16: |d| <= 128) and weight scale to a fold table [row][chunk] with an
//    odd row pitch, then release the stage;
//  * four fold warps take the tiles in turn (tile i: fold warp i mod 4):
//    lane r walks row r's chunks in order (integer group sums, one fma per
//    group) and writes Y -- reads at an odd pitch, so the R lanes hit R
//    banks. The fold is a serial chain per row; keeping it off the dot warps
//    lets them run ahead by as many tiles as there are fold tables.
// The activation planes of every job sit in shared memory for the whole
// launch: copied (bit-plane input) or made in the kernel from the fp16 rows
// with the exact integer threshold of quant.cuh.
// Every mbarrier wait is bounded; on a timeout the CTA records
// BWTA_STATUS_TIMEOUT, lets the copies it issued land and returns.
#include <algorithm>

#include "common.cuh"
#include "quant.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace bwta {

constexpr int DC_WARPS = 8;                      // dot warps
constexpr int DC_CTHREADS = DC_WARPS * 32;       // dot threads (named barrier 1)
constexpr int DC_FOLD_WARPS = 4;                 // fold warps
constexpr int DC_COPY_WARP = DC_WARPS + DC_FOLD_WARPS;
constexpr int DC_THREADS = (DC_COPY_WARP + 1) * 32;
constexpr int DC_MAX_STAGES = 16;
constexpr int DC_MAX_TABS = 8;
constexpr int DC_MAX_JOBS = 8;
constexpr int DC_MAX_CHUNKS = 128;               // K <= 16384
constexpr size_t DC_MAX_ACT_SMEM = 48 * 1024;
constexpr size_t DC_RING_BUDGET = 56 * 1024;     // bytes of weight tiles in flight per CTA
#ifndef DC_PF_BYTES
#define DC_PF_BYTES (128 * 1024)                  // bytes of weight tiles prefetched into L2 per CTA
#endif
constexpr size_t DC_TAB_BUDGET = 48 * 1024;      // fold tables (at least two)
constexpr int DC_STAGE_ROWS_BYTES = 48 * 1024;   // fused: fp16 rows staged per round
constexpr int DC_ROUND_ROWS = 32;                // fused: at most this many rows per round

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
  double inv2k;                 // fused: 1 / (2 K), the threshold's divisor as a reciprocal
  int64_t tile0;                // first global tile of this job
  int M, nchunks, gchunks;
  int act_off;                  // byte offset of the job's planes in shared memory
  int vec;                      // X rows 16-byte aligned
};

struct DecodeBatch {
  DecodeJob job[DC_MAX_JOBS];
  int64_t ntiles;
  int njobs, ternary, ready;
  int stages, stage_bits, stage_bytes;  // copy ring: depth, bytes of sign words / of a stage
  int pf_ahead;                         // tiles prefetched into L2 ahead of the ring
  int ring_off;
  int ntabs, nfold;                     // fold tables (a multiple of nfold), active fold warps
  int tab_off, tab_bytes, pitch;        // fold tables (pitch odd, in elements)
  int stage_off, stage_pieces;          // fused: fp16 staging area (over the fold tables)
  int red_off;                          // fused: per-row partial sums (after tables and staging)
};

struct DcBars {
  uint64_t full[DC_MAX_STAGES];   // copy of the stage landed (transaction bytes)
  uint64_t empty[DC_MAX_STAGES];  // the dot warps have read the stage (8 arrivals)
  uint64_t tfull[DC_MAX_TABS];    // the fold table is written (8 arrivals)
  uint64_t tempty[DC_MAX_TABS];   // the fold table is folded (1 arrival)
  int32_t timeout;
  int32_t last_j0, last_m0, last_nr;  // fused: the rows of the last setup round (first job, row; count)
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

// The dot warps' barrier (the fold and copy warps never take part).
__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, %0;" ::"n"(DC_CTHREADS) : "memory"); }

// L2 policy for data read once: evict it first, so the weight stream does not
// push the activations and outputs of neighbouring launches out of L2.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Bulk prefetch of global memory into L2 under the policy `pol` (no
// completion to track: a later copy of the same bytes finds them in L2).
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes, uint64_t pol) {
  asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;" ::"l"(src), "r"(bytes),
               "l"(pol)
               : "memory");
}

// The job a tile belongs to, with the fields the copy thread needs, kept in
// registers while tiles advance through the jobs in order.
struct DcCursor {
  int j = -1;
  int64_t tend = 0, t0 = 0, N = 0, ldw = 0, G = 0;
  const uint32_t *wb = nullptr;
  const float *ws = nullptr;
  bool Y = false;
  __device__ __forceinline__ void seek(const DecodeBatch &p, int64_t tile) {
    while (tile >= tend) {
      const DecodeJob &J = p.job[++j];
      t0 = J.tile0, N = J.N, ldw = J.ldw, G = J.G, wb = J.wb, ws = J.ws, Y = J.Y != nullptr;
      tend = j + 1 < p.njobs ? p.job[j + 1].tile0 : p.ntiles;
    }
  }
  // rows of the tile of R rows that starts at row n0 (the job's last tile may be short)
  __device__ __forceinline__ int64_t rows(int64_t n0, int R) const { return N - n0 < R ? N - n0 : R; }
};

// Bulk copy global -> this CTA's shared memory (no multicast), completing on
// `bar`, under the L2 policy `pol`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                          uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, "
      "[%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
  // copies src_bytes (0..16) and fills the rest of the 16 bytes with zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Bounded wait that also records a timeout for the whole CTA. A phase that
// has already completed (the usual case in the tile loops) is seen by one
// non-blocking test, without entering the suspending wait.
__device__ __forceinline__ bool dc_wait(DcBars &b, uint64_t *bar, uint32_t parity) {
  if (mbar_test(bar, parity)) return true;
  if (*(volatile int32_t *)&b.timeout) return false;
  if (mbar_wait(bar, parity, 2000000000ull)) return true;
  b.timeout = 1;
  return false;
}

// ------------------------------------------------------------- activations
// Warp sum of a uint64, modulo 2^64 like a plain sum (every lane gets the
// total): three 22-bit limbs summed by independent redux.sync instructions
// (32 limbs of 22 bits cannot overflow 32), in place of a chain of ten
// dependent 32-bit shuffles.
__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t v) {
  constexpr uint64_t L22 = (1u << 22) - 1;
  const uint64_t lo = __reduce_add_sync(FULL, (uint32_t)(v & L22));
  const uint64_t mid = __reduce_add_sync(FULL, (uint32_t)((v >> 22) & L22));
  const uint64_t hi = __reduce_add_sync(FULL, (uint32_t)(v >> 44));
  return lo + (mid << 22) + (hi << 44);
}

// The row scales of one setup round's nr rows (round row r = job jj, row mm,
// counted from (j0, m0)), from the round's per-warp partial sums; thread t of
// the calling group computes row t.
__device__ __forceinline__ void dc_row_scales(const DecodeBatch &p, uint8_t *smem, int j0, int m0,
                                              int nr, int t) {
  if (t >= nr) return;
  const uint64_t *red_s = reinterpret_cast<const uint64_t *>(smem + p.red_off);
  const uint64_t *red_k = red_s + DC_ROUND_ROWS * DC_WARPS;
  const uint64_t *red_n = red_k + DC_ROUND_ROWS * DC_WARPS;
  int jj = j0, mm = m0;
  for (int r = 0; r < t; ++r)
    if (++mm == p.job[jj].M) {
      mm = 0;
      ++jj;
    }
  const DecodeJob &J = p.job[jj];
  float *ssc = reinterpret_cast<float *>(smem + J.act_off + (size_t)J.M * J.nchunks * 36);
  uint64_t a = 0, b = 0;
  if (p.ternary) {
#pragma unroll
    for (int w = 0; w < DC_WARPS; ++w) {
      a += red_k[t * DC_WARPS + w];
      b += red_n[t * DC_WARPS + w];
    }
  } else {
#pragma unroll
    for (int w = 0; w < DC_WARPS; ++w) a += red_s[t * DC_WARPS + w];
    b = (uint64_t)J.K;
  }
  ssc[mm] = row_scale(a, b);
}

// Named barriers of the fused setup's hand-off to the fold warps: the dot
// warps arrive on DC_BAR_SETUP (without waiting) once the last round's
// partial sums are written; the fold warps wait on it, make that round's row
// scales, and meet on DC_BAR_FOLD before their first output.
constexpr int DC_BAR_SETUP = 2, DC_BAR_FOLD = 3;
__device__ __forceinline__ void bar_arrive_n(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void bar_sync_n(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// floor(S / d) for d = 2K: S is a sum of K magnitudes below 2^40 units, so the
// quotient is below 2^39 and the fp64 estimate S * (1/d) is within 2^-12 of
// it; one integer correction step in either direction makes it exact (a 64-bit
// integer division is a long dependent subroutine on the setup's critical
// path).
__device__ __forceinline__ uint64_t floor_div_2k(uint64_t S, int64_t d, double inv_d) {
  if (d <= 0) return 0;  // an empty row: no element to threshold
  uint64_t q = (uint64_t)__dmul_rz(__ull2double_rn(S), inv_d);
  const uint64_t ud = (uint64_t)d;
  if (q * ud > S) --q;
  else if (S - q * ud >= ud) ++q;
  return q;
}

// Planes of every job into shared memory: copied (bit-plane input) or made
// here from the fp16 rows with the exact integer threshold of quant.cuh (the
// same planes and scales as bwta_quantize_pack_acts, bit for bit). For the
// latter, rows are copied into a staging area with cp.async -- as many rows
// per round as fit, so that one memory latency covers them -- and the 256
// compute threads then make the planes of every staged row: pass 1 sums the
// magnitudes of all the round's rows (one partial per row and warp), pass 2
// derives each row's threshold from them and writes the row's bits and kept
// sums (and the popcount of each mask chunk), and the row scales follow --
// three barriers per round. Piece q (8
// halves) of a row belongs to thread q % 256; 16 consecutive threads cover
// one 128-element chunk.
template <bool FUSED>
__device__ __forceinline__ void dc_setup_acts(const DecodeBatch &p, uint8_t *smem, DcBars &bars,
                                              int32_t *d_status) {
  const int tid = threadIdx.x, wid = tid / 32, lane = tid % 32;
  if (!FUSED) {
    for (int j = 0; j < p.njobs; ++j) {
      const DecodeJob &J = p.job[j];
      uint4 *sA = reinterpret_cast<uint4 *>(smem + J.act_off);
      uint4 *sS = sA + J.M * J.nchunks;
      int *sP = reinterpret_cast<int *>(sS + J.M * J.nchunks);
      float *ssc = reinterpret_cast<float *>(sP + J.M * J.nchunks);
      const int nch = J.nchunks;
      for (int idx = tid; idx < J.M * nch; idx += DC_CTHREADS) {
        const int m = idx / nch, c = idx % nch;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(J.am + m * J.lda) + c);
        sA[idx] = v;
        sS[idx] = __ldg(reinterpret_cast<const uint4 *>(J.as + m * J.lda) + c);
        sP[idx] = __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
      }
      for (int m = tid; m < J.M; m += DC_CTHREADS) ssc[m] = J.ascale ? __ldg(J.ascale + m) : 0.0f;
    }
    cbar();
    return;
  }
  uint4 *stage = reinterpret_cast<uint4 *>(smem + p.stage_off);
  uint64_t *red_s = reinterpret_cast<uint64_t *>(smem + p.red_off);  // [row][warp]
  uint64_t *red_k = red_s + DC_ROUND_ROWS * DC_WARPS;
  uint64_t *red_n = red_k + DC_ROUND_ROWS * DC_WARPS;
  bool bad = false;
  int j = 0, m = 0;  // next row to stage
  while (j < p.njobs) {
    // one round: stage rows (j, m) ... while they fit
    const int j0 = j, m0 = m;
    int used = 0, nr = 0;  // pieces of 16 bytes, rows
    while (j < p.njobs && nr < DC_ROUND_ROWS) {
      const DecodeJob &J = p.job[j];
      const int pieces = J.nchunks * 16;
      if (used > 0 && used + pieces > p.stage_pieces) break;
      const uint16_t *xr = J.X + m * J.ldX;
      const int64_t K = J.K;
      for (int q = tid; q < pieces; q += DC_CTHREADS) {
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
      ++nr;
      if (++m == J.M) {
        m = 0;
        ++j;
      }
    }
    // Each thread reads back only the pieces it staged itself (piece q of
    // every row is staged and read by thread q % 256), so its own wait is
    // the only ordering pass 1 needs.
    cp_async_wait_all();
    // pass 1: magnitude sums of every staged row
    {
      int off = 0;
      for (int r = 0, jj = j0, mm = m0; r < nr; ++r) {
        const DecodeJob &J = p.job[jj];
        const int pieces = J.nchunks * 16;
        const uint4 *row = stage + off;
        uint64_t S = 0;
        for (int q = tid; q < pieces; q += DC_CTHREADS) S += sum_mag8(row[q], bad);
        S = warp_sum_u64(S);
        if (lane == 0) red_s[r * DC_WARPS + wid] = S;
        off += pieces;
        if (++mm == J.M) {
          mm = 0;
          ++jj;
        }
      }
    }
    cbar();
    // pass 2: threshold, bit planes, kept sums
    {
      int off = 0;
      for (int r = 0, jj = j0, mm = m0; r < nr; ++r) {
        const DecodeJob &J = p.job[jj];
        const int nch = J.nchunks, pieces = nch * 16;
        const int steps = (pieces + DC_CTHREADS - 1) / DC_CTHREADS;
        const int64_t K = J.K;
        uint64_t S = 0;
#pragma unroll
        for (int w = 0; w < DC_WARPS; ++w) S += red_s[r * DC_WARPS + w];
        const uint32_t hT = p.ternary ? mag_threshold_pattern(floor_div_2k(S, 2 * K, J.inv2k)) : 0u;
        uint4 *sA = reinterpret_cast<uint4 *>(smem + J.act_off);
        uint32_t *mrow = reinterpret_cast<uint32_t *>(sA + mm * nch);
        uint32_t *srow = reinterpret_cast<uint32_t *>(sA + J.M * nch + mm * nch);
        int *prow = reinterpret_cast<int *>(sA + 2 * J.M * nch) + mm * nch;
        const uint4 *row = stage + off;
        uint64_t ks = 0, kn = 0;
        for (int st = 0; st < steps; ++st) {  // uniform trip count: store_chunk shuffles
          const int q = st * DC_CTHREADS + tid, chunk = q / 16;
          const uint4 v = q < pieces ? row[q] : make_uint4(0, 0, 0, 0);
          const int64_t k0 = (int64_t)q * 8;
          uint32_t kb, sb;
          if (p.ternary) keep8<true>(v, hT, k0, K, kb, sb, ks);
          else keep8<false>(v, hT, k0, K, kb, sb, ks);
          kn += __popc(kb);
          store_chunk(kb, sb, mrow, srow, chunk, chunk < nch, nullptr, prow);
        }
        ks = warp_sum_u64(ks);
        kn = __reduce_add_sync(FULL, (uint32_t)kn);  // at most K kept elements
        if (lane == 0) {
          red_k[r * DC_WARPS + wid] = ks;
          red_n[r * DC_WARPS + wid] = kn;
        }
        off += pieces;
        if (++mm == J.M) {
          mm = 0;
          ++jj;
        }
      }
    }
    if (j < p.njobs) {
      // more rounds follow: this round's row scales now (one thread per row),
      // before the staging area and the partial sums are reused
      cbar();
      dc_row_scales(p, smem, j0, m0, nr, tid);
      cbar();
    } else {
      // the last round: its row scales are made by the fold warps (the only
      // readers of scales), off the dot warps' way to their first tile
      if (tid == 0) {
        bars.last_j0 = j0;
        bars.last_m0 = m0;
        bars.last_nr = nr;
      }
      bar_arrive_n(DC_BAR_SETUP, DC_CTHREADS + DC_FOLD_WARPS * 32);
      cbar();  // every plane of the round is written before any dot warp reads one
    }
  }
  if (bad) flag_status(d_status, BWTA_STATUS_NONFINITE);
}

// ------------------------------------------------------------------ kernel
// Fold table b: d [MR][R][pitch] int16, then alpha [R][pitch] fp32.
__host__ __device__ __forceinline__ size_t dc_tab_d_bytes(int mr, int R, int pitch) {
  return ((size_t)mr * R * pitch * 2 + 15) / 16 * 16;
}

// Two CTAs per SM by registers: an SM running a CTA of this launch keeps room
// for a CTA of the next kernel in the stream (416 threads x 80 registers, the
// allocation of 74, would not fit twice in 64 K registers).
template <int MR, bool FUSED, int R>
__global__ void __launch_bounds__(DC_THREADS, 2)
k_decode(const __grid_constant__ DecodeBatch pk, int32_t *d_status) {
  extern __shared__ uint4 dc_smem4[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(dc_smem4);
  __shared__ DcBars bars;
  // The launch parameters (1.4 KB) are copied to shared memory with one load
  // per thread: read in place, the job lookups below would be chains of
  // dependent constant-cache misses at the start of every launch.
  __shared__ DecodeBatch p_s;
  static_assert(sizeof(DecodeBatch) % 4 == 0, "copied as words");
  for (int w = threadIdx.x; w < (int)(sizeof(DecodeBatch) / 4); w += DC_THREADS)
    reinterpret_cast<uint32_t *>(&p_s)[w] = reinterpret_cast<const uint32_t *>(&pk)[w];
  __syncthreads();
  const DecodeBatch &p = p_s;
  static_assert((R == 16 || R == 32) && R % DC_WARPS == 0, "fold lanes 0..R-1, R/8 rows per dot warp");
  constexpr int RPW = R / DC_WARPS;  // rows per dot warp
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t stride = gridDim.x;
  uint8_t *ring = smem + p.ring_off;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], DC_WARPS);
    }
    for (int t = 0; t < p.ntabs; ++t) {
      mbar_init(&bars.tfull[t], DC_WARPS);
      mbar_init(&bars.tempty[t], 1);
    }
    bars.timeout = 0;
    mbar_fence_init();
  }
  __syncthreads();
  pdl_trigger();

  if (warp == DC_COPY_WARP) {
    // ------------------------------------------------ copy warp
    if (lane == 0) {
      if (!p.ready) pdl_wait();  // weights may still be written by the previous kernel
      const uint64_t pol = l2_evict_first();  // every weight byte is read once per launch
      // This single thread is the CTA's only source of copies: its loop keeps
      // the stage index and round in counters and the current job's fields
      // in registers (a CTA meets each job's tiles in one run). The ring holds
      // `stages` tiles; a second cursor keeps the next `pf_ahead` tiles on
      // their way into L2 (bulk prefetches, no shared memory), so that more
      // bytes per SM are in flight than the ring can hold and a refilled
      // stage finds its bytes in L2.
      int i = 0, s = 0;
      uint32_t round = 0;
      DcCursor c, pc;
      int64_t ptile = blockIdx.x + (int64_t)p.stages * stride;
      int pi = p.stages;
      for (int64_t tile = blockIdx.x; tile < p.ntiles; tile += stride, ++i) {
        if (i >= p.stages && !dc_wait(bars, &bars.empty[s], (round & 1) ^ 1)) break;
        c.seek(p, tile);
        const int64_t n0 = (tile - c.t0) * R;
        const int64_t rows = c.rows(n0, R);
        uint8_t *st = ring + (size_t)s * p.stage_bytes;
        const uint32_t bbytes = (uint32_t)(rows * c.ldw * 4);
        const uint32_t sbytes = c.Y ? (uint32_t)(rows * c.G * 4) : 0u, s16 = sbytes & ~15u;
        // a scale tail that is not a whole 16 bytes: plain loads (published by the arrive)
        float *sdst = reinterpret_cast<float *>(st + p.stage_bits);
        for (uint32_t q = s16 / 4; q < sbytes / 4; ++q) sdst[q] = __ldg(c.ws + n0 * c.G + q);
        mbar_arrive_expect_tx(&bars.full[s], bbytes + s16);
        bulk_load(st, c.wb + n0 * c.ldw, bbytes, &bars.full[s], pol);
        if (s16) bulk_load(sdst, c.ws + n0 * c.G, s16, &bars.full[s], pol);
        if (++s == p.stages) {
          s = 0;
          ++round;
        }
        // once the ring's first fill is out, keep tiles i+1 .. i+pf_ahead prefetched
        for (; i + 1 >= p.stages && pi <= i + p.pf_ahead && ptile < p.ntiles; ptile += stride, ++pi) {
          pc.seek(p, ptile);
          const int64_t m0 = (ptile - pc.t0) * R, prow = pc.rows(m0, R);
          bulk_prefetch_l2(pc.wb + m0 * pc.ldw, (uint32_t)(prow * pc.ldw * 4), pol);
          const uint32_t ps16 = pc.Y ? (uint32_t)(prow * pc.G * 4) & ~15u : 0u;
          if (ps16) bulk_prefetch_l2(pc.ws + m0 * pc.G, ps16, pol);
        }
      }
      // Copies still in flight (after a timeout) land before the CTA exits; a
      // stage is refilled only after its previous copy was consumed, so only
      // the last `stages` copies can be pending.
      bool drained = true;
      for (int q = i > p.stages ? i - p.stages : 0; q < i; ++q)
        drained &= mbar_wait(&bars.full[q % p.stages], (q / p.stages) & 1, DRAIN_NS);
      if (!drained) flag_status(d_status, BWTA_STATUS_DRAIN);
    }
    return;
  }

  if (warp >= DC_WARPS) {
    // ------------------------------------------------ fold warps
    pdl_wait();  // outputs follow the previous kernel in the stream
    if (FUSED) {
      // the last setup round's row scales (the earlier rounds' are made by
      // the dot warps), visible to every fold warp before its first output
      bar_sync_n(DC_BAR_SETUP, DC_CTHREADS + DC_FOLD_WARPS * 32);
      if (warp == DC_WARPS) dc_row_scales(p, smem, bars.last_j0, bars.last_m0, bars.last_nr, lane);
      bar_sync_n(DC_BAR_FOLD, DC_FOLD_WARPS * 32);
    }
    // Fold warp f takes tiles f, f + nfold, ...; with ntabs a multiple of
    // nfold, table b = i % ntabs is only ever folded by warp b % nfold, so
    // each table's barriers are waited on in order by one warp (a parity
    // wait never sees a phase two ahead).
    const int f = warp - DC_WARPS;
    int b = f, j = -1;
    uint32_t round = 0;
    int64_t tend = 0;
    for (int64_t tile = blockIdx.x + (int64_t)f * stride; f < p.nfold && tile < p.ntiles;
         tile += (int64_t)p.nfold * stride) {
      if (!__all_sync(FULL, dc_wait(bars, &bars.tfull[b], round & 1))) break;
      while (tile >= tend) {
        ++j;
        tend = j + 1 < p.njobs ? p.job[j + 1].tile0 : p.ntiles;
      }
      const DecodeJob &J = p.job[j];
      const JobActs acts = job_acts(smem, J);
      const uint8_t *tab = smem + p.tab_off + (size_t)b * p.tab_bytes;
      const int nch = J.nchunks, gc = J.gchunks;
      const int64_t n = (tile - J.tile0) * R + lane;
      if (lane < R) {
        // lane r walks row r's chunks in order
        const int16_t *dr = reinterpret_cast<const int16_t *>(tab) + lane * p.pitch;
        const float *ar = reinterpret_cast<const float *>(tab + dc_tab_d_bytes(MR, R, p.pitch)) + lane * p.pitch;
        const int dstride = R * p.pitch;
        float acc[MR];
        int dt[MR], gd[MR];
#pragma unroll
        for (int m = 0; m < MR; ++m) {
          acc[m] = 0.0f;
          dt[m] = 0;
          gd[m] = 0;
        }
        if (gc == 1) {  // one weight group per chunk (group 128): every chunk closes a group
          constexpr int U = MR <= 2 ? 16 : 4;  // chunks whose loads are issued together
          int c = 0;
          for (; c + U <= nch; c += U) {
            float av[U], dv[U][MR];
#pragma unroll
            for (int u = 0; u < U; ++u) {
              av[u] = ar[c + u];
#pragma unroll
              for (int m = 0; m < MR; ++m) {
                const int d = dr[m * dstride + c + u];
                dt[m] += d;
                dv[u][m] = biased_int_to_float(d + INT_FLOAT_BIAS);
              }
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
              for (int m = 0; m < MR; ++m) acc[m] = fmaf(dv[u][m], av[u], acc[m]);
          }
          for (; c < nch; ++c) {
            const float a = ar[c];
#pragma unroll
            for (int m = 0; m < MR; ++m) {
              const int d = dr[m * dstride + c];
              acc[m] = fmaf(biased_int_to_float(d + INT_FLOAT_BIAS), a, acc[m]);
              dt[m] += d;
            }
          }
        } else {
          int left = gc;
          for (int c = 0; c < nch; ++c) {
#pragma unroll
            for (int m = 0; m < MR; ++m) gd[m] += dr[m * dstride + c];
            if (--left == 0 || c + 1 == nch) {
              const float a = ar[c];
#pragma unroll
              for (int m = 0; m < MR; ++m) {
                acc[m] = fmaf(biased_int_to_float(gd[m] + INT_FLOAT_BIAS), a, acc[m]);
                dt[m] += gd[m];
                gd[m] = 0;
              }
              left = gc;
            }
          }
        }
        if (n < J.N) {
#pragma unroll
          for (int m = 0; m < MR; ++m) {
            if (m >= J.M) break;
            if (J.Y) J.Y[m * J.ldY + n] = acc[m] * acts.ssc[m];
            if (J.dots) J.dots[m * J.ldD + n] = dt[m];
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.tempty[b]);
      b += p.nfold;  // tables f, f + nfold, ... (ntabs is a multiple of nfold)
      if (b >= p.ntabs) {
        b -= p.ntabs;
        ++round;
      }
    }
    return;
  }

  // ------------------------------------------------ dot warps
  pdl_wait();  // activations follow the previous kernel in the stream
  dc_setup_acts<FUSED>(p, smem, bars, d_status);

  // stage and table indices and their rounds in counters; the current job's
  // fields in registers, reloaded when the tiles move into the next job
  int i = 0, s = 0, b = 0, j = -1;
  uint32_t sround = 0, bround = 0;
  int64_t tend = 0, jldw = 0, jG = 0;
  int nch = 0, gc = 1, jM = 0;
  bool jY = false;
  JobActs acts = {};
  for (int64_t tile = blockIdx.x; tile < p.ntiles; tile += stride, ++i) {
    while (tile >= tend) {
      const DecodeJob &J = p.job[++j];
      jldw = J.ldw, jG = J.G, nch = J.nchunks, gc = J.gchunks, jM = J.M, jY = J.Y != nullptr;
      acts = job_acts(smem, J);
      tend = j + 1 < p.njobs ? p.job[j + 1].tile0 : p.ntiles;
    }
    bool ok = dc_wait(bars, &bars.full[s], sround & 1);
    if (ok && i >= p.ntabs) ok = dc_wait(bars, &bars.tempty[b], (bround & 1) ^ 1);
    if (!__all_sync(FULL, ok)) break;  // warp-uniform: the loop below synchronizes the warp
    const uint8_t *st = ring + (size_t)s * p.stage_bytes;
    uint8_t *tab = smem + p.tab_off + (size_t)b * p.tab_bytes;
    int16_t *td = reinterpret_cast<int16_t *>(tab);
    float *ta = reinterpret_cast<float *>(tab + dc_tab_d_bytes(MR, R, p.pitch));
    // integer dots of this warp's RPW rows with every activation row. The
    // rows share each activation chunk's loads, and all of a chunk's loads are
    // issued before its stores (a store to the table may alias a later load,
    // so the compiler keeps them in program order).
    const int r0 = warp * RPW;
    const uint8_t *bits0 = st + (size_t)r0 * jldw * 4;
    const float *sc0 = reinterpret_cast<const float *>(st + p.stage_bits) + r0 * jG;
    for (int c = lane; c < nch; c += 32) {
      const int g = gc == 1 ? c : c / gc;
      uint4 w[RPW];
      float a[RPW];
#pragma unroll
      for (int q = 0; q < RPW; ++q) {
        w[q] = reinterpret_cast<const uint4 *>(bits0 + (size_t)q * jldw * 4)[c];
        a[q] = jY ? sc0[q * jG + g] : 0.0f;
      }
      int d[RPW][MR];
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        if (m < jM) {
          const uint4 A = acts.sA[m * nch + c], S = acts.sS[m * nch + c];
          const int P = acts.sP[m * nch + c];
#pragma unroll
          for (int q = 0; q < RPW; ++q)
            d[q][m] = P - 2 * popc4_csa(lop3_and_xor(A.x, S.x, w[q].x), lop3_and_xor(A.y, S.y, w[q].y),
                                        lop3_and_xor(A.z, S.z, w[q].z), lop3_and_xor(A.w, S.w, w[q].w));
        } else {
#pragma unroll
          for (int q = 0; q < RPW; ++q) d[q][m] = 0;
        }
      }
#pragma unroll
      for (int q = 0; q < RPW; ++q) ta[(r0 + q) * p.pitch + c] = a[q];
#pragma unroll
      for (int m = 0; m < MR; ++m)
#pragma unroll
        for (int q = 0; q < RPW; ++q) td[(m * R + r0 + q) * p.pitch + c] = (int16_t)d[q][m];
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&bars.empty[s]);
      mbar_arrive(&bars.tfull[b]);
    }
    if (++s == p.stages) {
      s = 0;
      ++sround;
    }
    if (++b == p.ntabs) {
      b = 0;
      ++bround;
    }
  }
  if (lane == 0 && warp == 0 && *(volatile int32_t *)&bars.timeout)
    flag_status(d_status, BWTA_STATUS_TIMEOUT);
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

template <int MR, bool FUSED, int R>
static cudaError_t launch_decode_t(const DecodeBatch &p, size_t smem, int32_t *d_status,
                                   cudaStream_t s) {
  auto kern = k_decode<MR, FUSED, R>;
  static SmemOptIn opt_in;
  if (cudaError_t e = opt_in(kern, (int)smem, true)) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // One CTA per SM (tiles go to CTAs round-robin, so every SM streams); an
  // SM keeps room for a CTA of the next kernel in the stream, which fills its
  // own ring while this one finishes.
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(p.ntiles, sms));
  return launch_pdl(kern, dim3((unsigned)blocks), dim3(DC_THREADS), smem, s, p, d_status);
}

cudaError_t launch_decode(const DecodeSpec *jobs, int njobs, bool fused, int mode, bool ready,
                          int32_t *d_status, cudaStream_t s) {
  DecodeBatch p = {};
  int MR = 1, nch_max = 1;
  int64_t ldw_max = 4, G_max = 1;
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
    J.inv2k = 1.0 / (2.0 * (double)in.K);
    J.M = (int)in.M;
    J.nchunks = (int)ceil_div<int64_t>(ceil_div<int64_t>(in.K, 32), 4);
    J.gchunks = in.group ? (int)(in.group / 128) : J.nchunks;
    J.G = in.group ? ceil_div<int64_t>(in.K, in.group) : 1;
    J.vec = (reinterpret_cast<uintptr_t>(in.X) & 15u) == 0 && in.ldX % 8 == 0;
    J.act_off = (int)act;
    act += dc_act_bytes(J.M, J.nchunks);
    MR = std::max(MR, J.M);
    nch_max = std::max(nch_max, J.nchunks);
    ldw_max = std::max(ldw_max, J.ldw);
    G_max = std::max(G_max, J.G);
    ++nj;
  }
  if (nj == 0) return cudaSuccess;
  if (act > DC_MAX_ACT_SMEM) return cudaErrorInvalidValue;
  p.njobs = nj;
  p.ternary = mode == BWTA_TERNARY;
  p.ready = ready;
  const int mr = MR <= 1 ? 1 : MR <= 2 ? 2 : MR <= 4 ? 4 : 8;
  // tile height: 32 rows where two such tiles of the widest job fit the copy
  // ring and the dot warps' registers hold 4 rows x MR dots
  auto stage_of = [&](int64_t R) { return (R * ldw_max * 4 + R * G_max * 4 + 15) / 16 * 16; };
  const int R = (mr <= 2 && 2 * (size_t)stage_of(32) <= DC_RING_BUDGET) ? 32 : 16;
  for (int i = 0; i < nj; ++i) {
    p.job[i].tile0 = p.ntiles;
    p.ntiles += ceil_div<int64_t>(p.job[i].N, R);
  }
  // copy ring: R rows of sign words and of scales of the widest job
  p.stage_bits = (int)(R * ldw_max * 4);
  p.stage_bytes = (int)stage_of(R);
  p.stages = (int)std::min<size_t>(DC_MAX_STAGES,
                                   std::max<size_t>(2, DC_RING_BUDGET / (size_t)p.stage_bytes));
  // L2 prefetch window: about DC_PF_BYTES of tiles per CTA beyond the ring
  p.pf_ahead = (int)(DC_PF_BYTES / (size_t)p.stage_bytes);
  p.ring_off = (int)act;
  const size_t ring = (size_t)p.stages * p.stage_bytes;
  // fold tables; fused: the staging area over them, then the partial sums
  // after both (read by the scale threads after the last barrier of the
  // setup, while other warps may already be writing fold tables)
  p.pitch = nch_max | 1;
  p.tab_bytes = (int)((dc_tab_d_bytes(mr, R, p.pitch) + (size_t)R * p.pitch * 4 + 15) / 16 * 16);
  p.tab_off = (int)(act + ring);
  size_t stage = 0, red = 0;
  if (fused) {  // every staged row fits; as many rows per round as the staging area holds
    size_t rows_bytes = 0, row_max = 0;
    for (int i = 0; i < nj; ++i) {
      const size_t rb = (size_t)p.job[i].nchunks * 256;
      rows_bytes += rb * p.job[i].M;
      row_max = std::max(row_max, rb);
    }
    stage = std::max(row_max, std::min(rows_bytes, (size_t)DC_STAGE_ROWS_BYTES));
    p.stage_off = p.tab_off;
    p.stage_pieces = (int)(stage / 16);
    red = (size_t)3 * DC_ROUND_ROWS * DC_WARPS * 8;
  }
  const size_t limit = 227 * 1024;
  auto total = [&](int nt) { return act + ring + std::max((size_t)nt * p.tab_bytes, stage) + red; };
  p.ntabs = (int)std::max<size_t>(2, std::min<size_t>(DC_MAX_TABS, DC_TAB_BUDGET / p.tab_bytes));
  while (p.ntabs > 2 && total(p.ntabs) > limit) --p.ntabs;
  p.nfold = std::min(p.ntabs, DC_FOLD_WARPS);
  p.ntabs -= p.ntabs % p.nfold;
  p.red_off = (int)(p.tab_off + std::max((size_t)p.ntabs * p.tab_bytes, stage));
  const size_t smem = total(p.ntabs);
  if (smem > limit) return cudaErrorInvalidValue;
#define BWTA_DC(MRV, RV)                                                                        \
  return fused ? launch_decode_t<MRV, true, RV>(p, smem, d_status, s)                           \
               : launch_decode_t<MRV, false, RV>(p, smem, d_status, s)
  if (mr == 1 && R == 32) BWTA_DC(1, 32);
  if (mr == 2 && R == 32) BWTA_DC(2, 32);
  if (mr == 1) BWTA_DC(1, 16);
  if (mr == 2) BWTA_DC(2, 16);
  if (mr == 4) BWTA_DC(4, 16);
  BWTA_DC(8, 16);
#undef BWTA_DC
}

int decode_max_jobs() { return DC_MAX_JOBS; }

size_t decode_act_bytes(int64_t M, int64_t K) {
  return dc_act_bytes((int)M, (int)ceil_div<int64_t>(ceil_div<int64_t>(K, 32), 4));
}

size_t decode_max_act_bytes() { return DC_MAX_ACT_SMEM; }

}  // namespace bwta
