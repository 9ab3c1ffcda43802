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
// Persistent kernel, one CTA per SM, tiles of 128 weight rows x 128 tokens
// handed out round-robin; every ring below runs on across tile boundaries, so
// the loads and MMAs of the next tile overlap the last groups and the stores
// of the current one. Warp roles:
//  * warp 0 (one thread) issues the TMA loads of each 128-column k-block:
//    128 tokens x 128 E4M3 bytes of activations (128-byte swizzle) and the
//    weight rows' sign bits (16 bytes per row), into an 8-stage ring;
//  * warps 2-5 expand the sign bits into E4M3 +-1 in TMEM (operand A, one TMEM
//    lane per weight row, 4 buffers). Weight k + 8j of a 32-column block goes
//    to byte j of word k, the order in which the activation packer writes its
//    E4M3 bytes, so a word costs one shift and one LOP3;
//  * warps 1 and 14 (one thread each) issue 4 MMAs (M=128, N=128, K=32) per
//    k-block into one of three fp32 accumulators in TMEM (one per weight
//    group in flight); with groups of one or two k-blocks issuer i takes the
//    groups with index = i (mod 2), so every MMA of a group comes from one
//    thread, in order; with longer groups warp 1 issues them all;
//  * warps 6-13 fold each finished group into running fp32 sums in registers
//    (two warps per TMEM lane quarter, 64 tokens each) and write Y at the end
//    of a tile.
// MMA issue blocks until the tensor pipe takes the instruction, and the pipe
// takes the next MMA only as the previous one finishes (64 cycles for
// M=128, N=128, K=32), so every gap in an issuing thread is idle pipe time.
// Two issuers on different SM sub-partitions keep the pipe fed through each
// other's gaps, and each does as little as possible between MMAs: one commit
// per k-block, into a
// ring of "k-block done" barriers that frees the smem stage, the A buffer and
// (for groups of at most two k-blocks) signals the finished accumulator all
// at once; the barriers of the next k-blocks are tested, without blocking,
// and two ready k-blocks are issued back to back, so the bookkeeping gap
// comes once per 8 MMAs.
// Every mbarrier wait is bounded (bwta::mbar_wait); on a timeout the CTA
// records BWTA_STATUS_TIMEOUT, lets its loads in flight land and its MMAs
// finish, frees TMEM and returns.
#include <algorithm>

#include "common.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace bwta {

constexpr int TC_BM = 128;      // weight rows per tile (TMEM lanes, MMA M)
constexpr int TC_BN = 128;      // tokens per tile (MMA N)
constexpr int TC_KB = 128;      // K elements per k-block = one 128-byte swizzle row
constexpr int TC_STAGES = 8;    // smem ring of (activations, weight bits) k-blocks
constexpr int TC_ABUF = 4;      // expanded-weight buffers in TMEM
constexpr int TC_DBUF = 3;      // fp32 accumulators in TMEM
constexpr int TC_BATCH = 2;     // ready k-blocks issued back to back (<= TC_DBUF)
// Warps: 0 TMA, 1 and 14 MMA issue, 2-5 expand, 6-13 epilogue. A warp reaches the
// TMEM lanes of quarter warp % 4 only, so the expand and epilogue warps cover
// the four quarters by their index mod 4. The MMA issuer shares its SM
// sub-partition with busy expand and epilogue warps; measured alone, its MMA
// rate drops 3.6x when high-ILP warps compete for the same issue slots, so it
// is the lowest-numbered warp there and the epilogue issues half as many FMA
// instructions (two fp32 FMAs per instruction).
constexpr int TC_PRODUCER = 0, TC_ISSUER = 1, TC_EXPAND0 = 2, TC_EPI0 = 6, TC_ISSUER2 = 14;
constexpr int TC_THREADS = 15 * 32;
constexpr int TC_X_BYTES = TC_BN * TC_KB;  // 16 KB of E4M3 activations per stage
constexpr int TC_W_BYTES = TC_BM * 16;     // 2 KB of weight sign bits per stage
constexpr int TC_STAGE_BYTES = TC_X_BYTES + TC_W_BYTES;
// TMEM columns: D0..D2 at 0, 128, 256; A0..A3 at 384 + 32 b.
constexpr uint32_t TC_TMEM_COLS = 512, TC_COL_A = TC_DBUF * TC_BN;
constexpr size_t TC_SMEM = 1024 + (size_t)TC_STAGES * TC_STAGE_BYTES + 1024;
static_assert(TC_COL_A + TC_ABUF * 32 <= TC_TMEM_COLS, "TMEM budget");
static_assert(TC_STAGE_BYTES % 1024 == 0, "stages must stay 1024-byte aligned");
// done[g % TC_STAGES] completes once per k-block g. A thread waiting there for
// k-block g must not find the phase of k-block g + TC_STAGES completed as well;
// that cannot happen when k-block g + TC_STAGES needs something the waiter
// provides after its wait: the producer's load (always), the expand warps'
// A buffer (TC_STAGES >= TC_ABUF) and the epilogue's accumulator release
// (groups of seg_len k-blocks with TC_STAGES >= TC_DBUF * seg_len; longer
// groups get their own commit on d_full). A commit tracks the MMAs of its own
// thread, and every wait names the k-block whose MMAs it needs.
// Two issuers: an issuer waits on full[] and a_full[] for its k-blocks only,
// skipping the other's. A parity wait for k-block g is sound when the slot's
// previous phase (k-block g - TC_STAGES, resp. g - TC_ABUF) has completed, and
// that holds when that k-block is the same issuer's (it waited for it). With
// groups of seg_len k-blocks handed out alternately, g - R is the same
// issuer's for every g exactly when R / seg_len is even: seg_len 1 or 2 for
// R = 4 and 8. Longer groups (up to a whole K) would let an issuer find a
// phase of the same parity from two rounds before, so they run on one issuer.
constexpr int TC_DUAL_MAX_GROUP = 2;
static_assert(TC_ABUF % (2 * TC_DUAL_MAX_GROUP) == 0 && TC_STAGES % (2 * TC_DUAL_MAX_GROUP) == 0,
              "two issuers need whole pairs of groups in every ring");
static_assert(TC_STAGES >= TC_ABUF && TC_STAGES >= 2 * TC_DBUF, "ring sizes");
constexpr int TC_SHORT_GROUP = TC_STAGES / TC_DBUF;  // longest group signalled through done[]

struct TcBarriers {
  uint64_t full[TC_STAGES];   // TMA landed (transaction bytes)
  uint64_t done[TC_STAGES];   // MMAs of k-block g (and all before) complete (commit)
  uint64_t a_full[TC_ABUF];   // expanded weights in TMEM (4 expand warps)
  uint64_t d_full[TC_DBUF];   // long group accumulated (commit)
  uint64_t d_empty[TC_DBUF];  // epilogue has read the accumulator (8 epilogue warps)
  uint64_t drain;             // all MMAs of the CTA complete (teardown)
  uint32_t tmem_base;
  int32_t timeout;
  int32_t undrained;          // a post-timeout drain ran out of time
};

// Bounded wait that also records a timeout for the whole CTA.
__device__ __forceinline__ bool tc_wait(TcBarriers *b, uint64_t *bar, uint32_t parity) {
  if (b->timeout) return false;
  if (mbar_wait(bar, parity, 2000000000ull)) return true;
  b->timeout = 1;
  return false;
}

// (y0, y1) = (fma(d0, a, y0), fma(d1, a, y1)) in one instruction: two IEEE
// fp32 fused multiply-adds, the same results as two fmaf calls.
__device__ __forceinline__ void fma2(float &y0, float &y1, float d0, float d1, float a) {
  uint64_t yy, dd, aa, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(yy) : "f"(y0), "f"(y1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(dd) : "f"(d0), "f"(d1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(aa) : "f"(a));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(dd), "l"(aa), "l"(yy));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(y0), "=f"(y1) : "l"(r));
}

// Four E4M3 weights +-1 from the sign-bit word w: byte j is weight 8j + k
// (sign bit 1 = -1 = 0xB8, 0 = +1 = 0x38).
template <int k>
__device__ __forceinline__ uint32_t e4m3_pm1_tc(uint32_t w) {
  return ((w << (7 - k)) & 0x80808080u) | 0x38383838u;
}

// Position of the MMA issuer in the (tile, k-block) sequence of its CTA.
struct TcCursor {
  int64_t tile;
  int kb, pos;       // k-block within the tile, within the current group
  uint32_t g, sg;    // k-blocks and groups before this one (all tiles)
  bool first, last;  // first / last k-block of its group

  __device__ void set_flags(int KB, int seg_len) {
    first = pos == 0;
    last = pos == seg_len - 1 || kb == KB - 1;
  }
  __device__ void advance(int KB, int seg_len, int64_t stride) {
    ++g;
    if (last) {
      ++sg;
      pos = 0;
    } else {
      ++pos;
    }
    if (++kb == KB) {
      kb = 0;
      tile += stride;
    }
    set_flags(KB, seg_len);
  }
};

template <bool GROUPED, bool WANT_Y, bool WANT_DOTS>
__global__ void __launch_bounds__(TC_THREADS, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
          const float *__restrict__ ascale, const float *__restrict__ wscale, int64_t M, int64_t N,
          int KB, int seg_len, int64_t G, float *__restrict__ Y, int64_t ldY,
          int32_t *__restrict__ dots, int64_t ldD, int32_t *d_status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *stages = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  TcBarriers *bars = reinterpret_cast<TcBarriers *>(stages + TC_STAGES * TC_STAGE_BYTES);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t NB = ceil_div<int64_t>(N, TC_BM);
  const int64_t ntiles = NB * ceil_div<int64_t>(M, TC_BN);
  const int nseg = (KB + seg_len - 1) / seg_len;
  const bool short_group = seg_len <= TC_SHORT_GROUP;  // accumulator signalled through done[]

  pdl_trigger();
  if (threadIdx.x == 0) {
    prefetch_tensormap(&map_x);
    prefetch_tensormap(&map_w);
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->done[s], 1);
    }
    for (int i = 0; i < TC_ABUF; ++i) mbar_init(&bars->a_full[i], 4);
    for (int i = 0; i < TC_DBUF; ++i) {
      mbar_init(&bars->d_full[i], 1);
      mbar_init(&bars->d_empty[i], 8);
    }
    mbar_init(&bars->drain, 2);  // one commit per issuer
    bars->timeout = 0;
    bars->undrained = 0;
    mbar_fence_init();
  }
  if (warp == TC_ISSUER) {
    tmem_alloc(&bars->tmem_base, TC_TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == TC_PRODUCER) {
    // ------------------------------------------------ TMA loads
    if (lane == 0) {
      uint32_t g = 0;  // k-blocks loaded so far (all tiles)
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int32_t n0 = (int32_t)((tile % NB) * TC_BM), m0 = (int32_t)((tile / NB) * TC_BN);
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % TC_STAGES;
          // the stage's previous k-block is done (its bits were read before its MMAs)
          if (g >= TC_STAGES && !tc_wait(bars, &bars->done[s], ((g / TC_STAGES) - 1) & 1)) {
            ok = false;
            break;
          }
          uint8_t *st = stages + s * TC_STAGE_BYTES;
          mbar_arrive_expect_tx(&bars->full[s], TC_STAGE_BYTES);
          tma_load_2d(st, &map_x, kb * TC_KB, m0, &bars->full[s]);
          tma_load_2d(st + TC_X_BYTES, &map_w, kb * 4, n0, &bars->full[s]);
        }
      }
      // Loads still in flight (after a timeout) land before the CTA exits; in
      // a normal run these phases are complete already. A stage is reloaded
      // only after the MMAs that read its previous load, which waited for that
      // load, so the last TC_STAGES loads are the only ones that can be pending.
      for (uint32_t j = g > TC_STAGES ? g - TC_STAGES : 0; j < g; ++j)
        if (!mbar_wait(&bars->full[j % TC_STAGES], (j / TC_STAGES) & 1, DRAIN_NS))
          bars->undrained = 1;
    }
    __syncwarp();
  } else if (warp == TC_ISSUER || warp == TC_ISSUER2) {
    // ------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t me = warp == TC_ISSUER ? 0u : 1u;  // this issuer's groups: sg % 2 == me
      const bool dual = seg_len <= TC_DUAL_MAX_GROUP;    // else warp 1 issues every group
      const uint32_t idesc = idesc_e4m3_f32(TC_BM, TC_BN);
      // Non-blocking test of everything k-block c needs.
      auto ready = [&](const TcCursor &c) -> bool {
        bool r = mbar_test(&bars->full[c.g % TC_STAGES], (c.g / TC_STAGES) & 1) &
                 mbar_test(&bars->a_full[c.g % TC_ABUF], (c.g / TC_ABUF) & 1);
        if (c.first && c.sg >= TC_DBUF)
          r &= mbar_test(&bars->d_empty[c.sg % TC_DBUF], ((c.sg / TC_DBUF) - 1) & 1);
        return r;
      };
      // Blocking (bounded) version of the same.
      auto wait_all = [&](const TcCursor &c) -> bool {
        if (c.first && c.sg >= TC_DBUF &&
            !tc_wait(bars, &bars->d_empty[c.sg % TC_DBUF], ((c.sg / TC_DBUF) - 1) & 1))
          return false;
        return tc_wait(bars, &bars->full[c.g % TC_STAGES], (c.g / TC_STAGES) & 1) &&
               tc_wait(bars, &bars->a_full[c.g % TC_ABUF], (c.g / TC_ABUF) & 1);
      };
      // The 4 MMAs and the commits of one k-block.
      auto issue = [&](const TcCursor &c) {
        const int d = c.sg % TC_DBUF, b = c.g % TC_ABUF;
        const uint32_t xs = smem_addr(stages + (c.g % TC_STAGES) * TC_STAGE_BYTES);
#pragma unroll
        for (int k4 = 0; k4 < TC_KB / 32; ++k4)
          mma_f8f6f4_ts(tmem + d * TC_BN, tmem + TC_COL_A + b * 32 + k4 * 8,
                        smem_desc_k_sw128(xs + k4 * 32), idesc, (c.first && k4 == 0) ? 0u : 1u);
        tc_commit(&bars->done[c.g % TC_STAGES]);
        if (c.last && !short_group) tc_commit(&bars->d_full[d]);
      };
      // Step c to this issuer's next k-block (or past the last tile).
      auto own = [&](TcCursor &c) {
        while (dual && c.tile < ntiles && (c.sg & 1u) != me) c.advance(KB, seg_len, gridDim.x);
      };
      TcCursor cur{(int64_t)blockIdx.x, 0, 0, 0u, 0u, true, true};
      cur.set_flags(KB, seg_len);
      if (!dual && me == 1) cur.tile = ntiles;  // nothing to issue
      own(cur);
      bool rdy = cur.tile < ntiles && ready(cur);
      while (cur.tile < ntiles) {
        if (!rdy && !wait_all(cur)) break;
        // The next k-block joins this batch when all it needs is ready now:
        // the MMAs of both then follow one another with no bookkeeping in
        // between, and the pipe runs 8 MMAs per gap of this thread instead of
        // 4 (measured: 90.5 -> 83.7 us at 4096x4096, M = 2048; batches of
        // three were slower again).
        TcCursor batch[TC_BATCH];
        batch[0] = cur;
        int nb = 1;
        TcCursor nxt = cur;
        nxt.advance(KB, seg_len, gridDim.x);
        own(nxt);
        while (nb < TC_BATCH && nxt.tile < ntiles && ready(nxt)) {
          batch[nb++] = nxt;
          nxt.advance(KB, seg_len, gridDim.x);
          own(nxt);
        }
        tc_fence_after();
#pragma unroll
        for (int i = 0; i < TC_BATCH; ++i)
          if (i < nb) issue(batch[i]);
        cur = nxt;
        rdy = cur.tile < ntiles && ready(cur);
      }
      // Every MMA issued (by both issuers) has completed before TMEM is released.
      tc_commit(&bars->drain);
      if (!mbar_wait(&bars->drain, 0, DRAIN_NS)) bars->undrained = 1;
    }
    __syncwarp();
  } else if (warp >= TC_EXPAND0 && warp < TC_EPI0) {
    // ------------------------------------------------ weight bits -> E4M3 in TMEM
    const int qx = warp % 4, r = qx * 32 + lane;
    uint32_t g = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb, ++g) {
        const int s = g % TC_STAGES, b = g % TC_ABUF;
        bool fine = tc_wait(bars, &bars->full[s], (g / TC_STAGES) & 1);
        if (fine && g >= TC_ABUF)  // the A buffer's previous k-block is done
          fine = tc_wait(bars, &bars->done[(g - TC_ABUF) % TC_STAGES],
                         ((g - TC_ABUF) / TC_STAGES) & 1);
        if (!__all_sync(FULL, fine)) {
          ok = false;
          break;
        }
        const uint4 bits =
            *reinterpret_cast<const uint4 *>(stages + s * TC_STAGE_BYTES + TC_X_BYTES + r * 16);
        uint32_t v[32];
        const uint32_t wd[4] = {bits.x, bits.y, bits.z, bits.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          v[8 * q + 0] = e4m3_pm1_tc<0>(wd[q]);
          v[8 * q + 1] = e4m3_pm1_tc<1>(wd[q]);
          v[8 * q + 2] = e4m3_pm1_tc<2>(wd[q]);
          v[8 * q + 3] = e4m3_pm1_tc<3>(wd[q]);
          v[8 * q + 4] = e4m3_pm1_tc<4>(wd[q]);
          v[8 * q + 5] = e4m3_pm1_tc<5>(wd[q]);
          v[8 * q + 6] = e4m3_pm1_tc<6>(wd[q]);
          v[8 * q + 7] = e4m3_pm1_tc<7>(wd[q]);
        }
        tmem_st32(tmem_addr(tmem, qx * 32, TC_COL_A + b * 32), v);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->a_full[b]);
      }
    }
  } else {
    // ------------------------------------------------ epilogue: fold groups, write Y
    const int h = (warp - TC_EPI0) / 4, q = warp % 4, r = q * 32 + lane;
    uint32_t sg = 0, g0 = 0;  // groups and k-blocks of the tiles before this one
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, g0 += KB) {
      const int64_t n = (tile % NB) * TC_BM + r, m0 = (tile / NB) * TC_BN + h * 64;
      float y[64];
      float alpha = (WANT_Y && n < N) ? __ldg(wscale + (GROUPED ? n * G : n)) : 0.0f;
      for (int seg = 0; seg < nseg; ++seg, ++sg) {
        const int d = sg % TC_DBUF;
        const float alpha_next =
            (WANT_Y && GROUPED && seg + 1 < nseg && n < N) ? __ldg(wscale + n * G + seg + 1) : 0.0f;
        bool fine;
        if (short_group) {  // wait for the group's last k-block
          const uint32_t ge = g0 + (uint32_t)min((seg + 1) * seg_len, KB) - 1;
          fine = tc_wait(bars, &bars->done[ge % TC_STAGES], (ge / TC_STAGES) & 1);
        } else {
          fine = tc_wait(bars, &bars->d_full[d], (sg / TC_DBUF) & 1);
        }
        if (!__all_sync(FULL, fine)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t dv[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tmem_ld32(tmem_addr(tmem, q * 32, d * TC_BN + h * 64 + c * 32), dv);
          tmem_wait_ld();
          if (c == 1) {  // the accumulator is in registers: hand it back to the MMAs
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->d_empty[d]);
          }
          if (seg == 0) {
#pragma unroll
            for (int i = 0; i < 32; ++i) y[c * 32 + i] = 0.0f;
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            fma2(y[c * 32 + i], y[c * 32 + i + 1], __uint_as_float(dv[i]), __uint_as_float(dv[i + 1]), alpha);
          if (WANT_DOTS && seg == nseg - 1 && n < N) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int64_t m = m0 + c * 32 + i;
              if (m < M) dots[m * ldD + n] = __float2int_rn(__uint_as_float(dv[i]));
            }
          }
        }
        alpha = alpha_next;
      }
      if (!ok) break;
      if (WANT_Y && n < N) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int64_t m = m0 + i;
          if (m < M) Y[m * ldY + n] = y[i] * __ldg(ascale + m);
        }
      }
    }
  }

  // TMEM is released even when a drain ran out of time: a later CTA on this SM
  // would otherwise block in its allocation for good. The DRAIN flag tells the
  // caller that the context is no longer to be trusted.
  tc_fence_before();
  __syncthreads();
  if (warp == TC_ISSUER) {
    tc_fence_after();
    tmem_dealloc(tmem, TC_TMEM_COLS);
  }
  if (threadIdx.x == 0 && bars->timeout)
    flag_status(d_status, BWTA_STATUS_TIMEOUT | (bars->undrained ? BWTA_STATUS_DRAIN : 0));
}

template <bool GROUPED, bool WANT_Y, bool WANT_DOTS>
static cudaError_t launch_tc_t(const CUtensorMap &mx, const CUtensorMap &mw, const float *ascale,
                               const float *wscale, int64_t M, int64_t N, int KB, int seg_len,
                               int64_t G, float *Y, int64_t ldY, int32_t *dots, int64_t ldD,
                               int32_t *d_status, cudaStream_t s) {
  auto kern = k_gemm_tc<GROUPED, WANT_Y, WANT_DOTS>;
  static SmemOptIn opt_in;
  if (cudaError_t e = opt_in(kern, (int)TC_SMEM)) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntiles = ceil_div<int64_t>(N, TC_BM) * ceil_div<int64_t>(M, TC_BN);
  const unsigned grid = (unsigned)std::min<int64_t>(ntiles, std::max(sms, 1));
  return launch_pdl(kern, dim3(grid), dim3(TC_THREADS), TC_SMEM, s, mx, mw, ascale, wscale, M, N,
                    KB, seg_len, G, Y, ldY, dots, ldD, d_status);
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
