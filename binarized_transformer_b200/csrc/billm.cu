// billm.cu -- BiLLM-format binary weights: the GPU builder of the packed
// format and the GEMM against fp16 activations.
//
// BiLLM: Pushing the Limit of Post-Training Quantization for LLMs --
// abstract and "Approach": salient weights are selected structurally, by
// column, and binarized with a residual approximation (w ~ a1*b1 + a2*b2);
// the bell-shaped non-salient weights are split at a break-point into a
// concentrated and a sparse group, each binarized with its own scale;
// "Limitations": one extra bit per weight identifies the group; block-size
// ablation: 128-column blocks. The pages give no kernel for this format.
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"

namespace bwta {

// ======================================================= builder: saliency
// One CTA per 128-column block, one thread per column: the column's metric
// sum_n w^2 is an fp64 sum over rows in ascending order (the Hessian of the
// saliency metric taken as the identity). Then thread 0 picks the n_sal
// largest (ties: lower column) and writes them in ascending order.
__global__ void __launch_bounds__(128)
k_billm_salient(const float *__restrict__ W, int64_t N, int64_t ldW, int n_sal,
                uint8_t *__restrict__ sal, int32_t *d_status) {
  __shared__ double metric[128];
  __shared__ unsigned char taken[128];
  pdl_trigger();
  pdl_wait();
  const int c = threadIdx.x;
  const int64_t col = (int64_t)blockIdx.x * 128 + c;
  double acc = 0.0;
  bool bad = false;
  int64_t n = 0;
  for (; n + 8 <= N; n += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(W + (n + u) * ldW + col);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      bad |= !isfinite(v[u]);
      const double wd = (double)v[u];
      acc = __dadd_rn(acc, __dmul_rn(wd, wd));
    }
  }
  for (; n < N; ++n) {
    const float v = __ldg(W + n * ldW + col);
    bad |= !isfinite(v);
    const double wd = (double)v;
    acc = __dadd_rn(acc, __dmul_rn(wd, wd));
  }
  if (bad) flag_status(d_status, BWTA_STATUS_NONFINITE);
  metric[c] = acc;
  taken[c] = 0;
  __syncthreads();
  if (c == 0) {
    for (int s = 0; s < n_sal; ++s) {
      int best = -1;
      for (int k = 0; k < 128; ++k)
        if (!taken[k] && (best < 0 || metric[k] > metric[best])) best = k;
      taken[best] = 1;
    }
    int i = 0;
    for (int k = 0; k < 128; ++k)
      if (taken[k]) sal[(int64_t)blockIdx.x * n_sal + i++] = (uint8_t)k;
  }
}

// ================================================ builder: per row-block
// One thread per (row, block): every statistic is a serial fp64 sum over the
// block's columns in ascending order, divided by the count and rounded once
// to fp32, so the scales are reproducible bit for bit.
//
// Break-point of the non-salient weights: split == 1 takes p = 0.5 * max|w|;
// split == 2 searches it (BiLLM abstract: "optimal splitting search"): every
// non-salient magnitude of the row-block is a candidate, and the one whose
// split has the smallest squared binarization error
//   E(p) = sum_{|w| <= p} (|w| - a_c)^2 + sum_{|w| > p} (|w| - a_s)^2
// (a = the group's mean magnitude, its L2-optimal scale) wins; ties go to the
// smaller p. E is evaluated in fp64 in ascending column order with explicit
// round-to-nearest operations (no fused multiply-add), so the decision is the
// same on every run; eight candidates share each pass over the columns.
// E(p) of eight candidate break-points at once: eight independent fp64
// chains per pass over the columns (the same operations, in the same column
// order, as one candidate at a time). Salient columns and candidates past the
// last one (cand[u] < 0) contribute nothing.
__device__ __forceinline__ void billm_split_errors8(const float *__restrict__ wr, const uint32_t (&salmask)[4],
                                    const double (&p)[8], double (&e)[8]) {
  double sc[8], ss[8];
  int nc[8], ns[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    sc[u] = ss[u] = 0.0;
    nc[u] = ns[u] = 0;
  }
  for (int c = 0; c < 128; ++c) {
    if ((salmask[c >> 5] >> (c & 31)) & 1u) continue;  // the same for all eight
    const double aw = fabs((double)__ldg(wr + c));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (aw <= p[u]) {
        sc[u] = __dadd_rn(sc[u], aw);
        ++nc[u];
      } else {
        ss[u] = __dadd_rn(ss[u], aw);
        ++ns[u];
      }
    }
  }
  double ac[8], as[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    ac[u] = nc[u] ? __ddiv_rn(sc[u], (double)nc[u]) : 0.0;
    as[u] = ns[u] ? __ddiv_rn(ss[u], (double)ns[u]) : 0.0;
    e[u] = 0.0;
  }
  for (int c = 0; c < 128; ++c) {
    if ((salmask[c >> 5] >> (c & 31)) & 1u) continue;
    const double aw = fabs((double)__ldg(wr + c));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const double d = __dsub_rn(aw, aw <= p[u] ? ac[u] : as[u]);
      e[u] = __dadd_rn(e[u], __dmul_rn(d, d));
    }
  }
}

__global__ void __launch_bounds__(256)
k_billm_quantize(const float *__restrict__ W, int64_t N, int64_t K, int64_t ldW, int n_sal,
                 int split, const uint8_t *__restrict__ sal, uint32_t *__restrict__ sign,
                 uint32_t *__restrict__ gmap, int64_t ldw, uint8_t *__restrict__ res,
                 float *__restrict__ bscale) {
  pdl_trigger();
  pdl_wait();
  const int64_t nb = K / 128;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= N * nb) return;
  const int64_t n = t / nb, j = t % nb;
  const float *wr = W + n * ldW + j * 128;
  uint32_t salmask[4] = {0, 0, 0, 0};
  uint8_t sidx[8];
  for (int i = 0; i < n_sal; ++i) {
    sidx[i] = sal[j * n_sal + i];
    salmask[sidx[i] >> 5] |= 1u << (sidx[i] & 31);
  }
  // salient columns: residual binarization
  float a1 = 0.0f, a2 = 0.0f;
  uint32_t rbits = 0;
  if (n_sal > 0) {
    double s1 = 0.0;
    for (int i = 0; i < n_sal; ++i) s1 = __dadd_rn(s1, fabs((double)__ldg(wr + sidx[i])));
    a1 = __double2float_rn(__ddiv_rn(s1, (double)n_sal));
    double s2 = 0.0;
    for (int i = 0; i < n_sal; ++i) {
      const float w = __ldg(wr + sidx[i]);
      const double r = __dsub_rn((double)w, (w < 0.0f) ? -(double)a1 : (double)a1);
      s2 = __dadd_rn(s2, fabs(r));
      if (r < 0.0) rbits |= 1u << i;
    }
    a2 = __double2float_rn(__ddiv_rn(s2, (double)n_sal));
  }
  // non-salient columns: break-point split
  double maxabs = 0.0;
  for (int c = 0; c < 128; ++c)
    if (!((salmask[c >> 5] >> (c & 31)) & 1u)) maxabs = fmax(maxabs, fabs((double)__ldg(wr + c)));
  double pbest = maxabs;
  if (split == 2) {
    // candidates: the non-salient magnitudes, eight per pass over the columns
    double ebest = __longlong_as_double(0x7ff0000000000000LL);  // +inf
    int c0 = 0;
    while (c0 < 128) {
      double p[8], e[8];
      bool v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // the next eight non-salient columns
        while (c0 < 128 && ((salmask[c0 >> 5] >> (c0 & 31)) & 1u)) ++c0;
        v[u] = c0 < 128;
        p[u] = v[u] ? fabs((double)__ldg(wr + c0)) : 0.0;
        if (v[u]) ++c0;
      }
      if (!v[0]) break;
#pragma unroll
      for (int u = 1; u < 8; ++u)
        if (!v[u]) p[u] = p[0];  // padding: repeats a candidate
      billm_split_errors8(wr, salmask, p, e);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (v[u] && (e[u] < ebest || (e[u] == ebest && p[u] < pbest))) {
          ebest = e[u];
          pbest = p[u];
        }
    }
  }
  double sc = 0.0, ss = 0.0;
  int nc = 0, ns = 0;
  uint32_t sw[4] = {0, 0, 0, 0}, gw[4] = {0, 0, 0, 0};
  for (int c = 0; c < 128; ++c) {
    const float w = __ldg(wr + c);
    if (w < 0.0f) sw[c >> 5] |= 1u << (c & 31);
    if ((salmask[c >> 5] >> (c & 31)) & 1u) continue;
    const double aw = fabs((double)w);
    if (split == 2 ? aw > pbest : (split && 2.0 * aw > maxabs)) {
      gw[c >> 5] |= 1u << (c & 31);
      ss = __dadd_rn(ss, aw);
      ++ns;
    } else {
      sc = __dadd_rn(sc, aw);
      ++nc;
    }
  }
  const float ac = nc ? __double2float_rn(__ddiv_rn(sc, (double)nc)) : 0.0f;
  const float as = ns ? __double2float_rn(__ddiv_rn(ss, (double)ns)) : 0.0f;
  *reinterpret_cast<uint4 *>(sign + n * ldw + 4 * j) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
  *reinterpret_cast<uint4 *>(gmap + n * ldw + 4 * j) = make_uint4(gw[0], gw[1], gw[2], gw[3]);
  res[n * nb + j] = (uint8_t)rbits;
  *reinterpret_cast<float4 *>(bscale + (n * nb + j) * 4) = make_float4(ac, as, a1, a2);
  if (j == nb - 1)  // zero the padding words of the row
    for (int64_t w = 4 * nb; w < ldw; ++w) {
      sign[n * ldw + w] = 0;
      gmap[n * ldw + w] = 0;
    }
}

cudaError_t launch_billm_pack(const float *W, int64_t ldW, int split, const billm_weights *o,
                              int32_t *d_status, cudaStream_t s) {
  const int64_t N = o->N, K = o->K, nb = K / 128;
  if (N == 0) return cudaSuccess;
  uint8_t *sal = const_cast<uint8_t *>(o->sal);
  cudaError_t e = launch_pdl(k_billm_salient, dim3((unsigned)nb), dim3(128), 0, s, W, N, ldW,
                             (int)o->n_sal, sal, d_status);
  if (e != cudaSuccess) return e;
  const int64_t total = N * nb;
  return launch_pdl(k_billm_quantize, dim3((unsigned)ceil_div<int64_t>(total, 256)), dim3(256), 0, s,
                    W, N, K, ldW, (int)o->n_sal, split, (const uint8_t *)sal,
                    const_cast<uint32_t *>(o->sign), const_cast<uint32_t *>(o->gmap), o->ldw_words,
                    const_cast<uint8_t *>(o->res), const_cast<float *>(o->bscale));
}

// ================================================================= GEMM
// CUDA-core path, M <= 16 activation rows per pass (larger M with unaligned X
// loops over groups of 16). Four threads own one weight row (lanes 4r .. 4r+3
// of a warp; thread p takes the row's 128-column blocks j = p, p + 4, ...), so
// a warp-load covers 64 contiguous bytes of each of eight rows, and each
// thread keeps its row's MP output partial sums in registers for all of K.
// The activations are staged in shared memory as fp32, [block][column][MP]
// (one 16-byte load gives four rows of one column; blocks 128 * MP + 4 floats
// apart, so the four threads of a row, on four different blocks, read four
// different bank groups), a slice of K at a time, with the block sums
// X_j[m] = sum_c x[m][c] of every 128-column block.
// Per block of a row (BiLLM "Approach"; the sign plane carries b for
// non-salient columns and b1 for salient ones):
//   y += alpha_c * (X_j - 2 * sum_{sign bit 1} x)          every column as +-alpha_c
//      + sum_{sparse}  (alpha_sp - alpha_c) * b  * x        sparse columns
//      + sum_{salient} ((alpha1 - alpha_c) * b1 + alpha2 * b2) * x
// which is the same real value as the pages' four-sum form: one predicated
// add per weight and row of X, plus a few multiply-adds for the ~10% of
// columns that are sparse or salient. Partial sums are per 128-column block
// (fp32 error ~128 * 2^-24 of the block's magnitude), folded into y per block.
constexpr int BR_SPLIT = 4;  // threads per weight row
// 256 threads (64 rows) per CTA for MP <= 4; 512 (128 rows) for larger MP,
// whose inner loop is latency-bound at 8 warps per SM.
template <int MP>
constexpr int br_threads() { return MP <= 4 ? 256 : 512; }
constexpr size_t BR_SMEM_BUDGET = 160 * 1024;
constexpr int BR_MAX_NB = 40960 / 128;

template <int MP, int BR_THREADS = br_threads<MP>(), int BR_ROWS = BR_THREADS / BR_SPLIT>
__global__ void __launch_bounds__(BR_THREADS)
k_billm_rows(const uint16_t *__restrict__ X, int64_t M, int64_t ldX, const uint32_t *__restrict__ sign,
             const uint32_t *__restrict__ gmap, const uint8_t *__restrict__ res,
             const uint8_t *__restrict__ sal, const float *__restrict__ bscale, int64_t N,
             int64_t K, int64_t ldw, int n_sal, float *__restrict__ Y, int64_t ldY, int slice,
             int32_t *d_status) {
  constexpr int BS = 128 * MP + 4;  // floats per staged block
  extern __shared__ float4 br_smem4[];
  float *xs = reinterpret_cast<float *>(br_smem4);     // [slice / 128][BS]
  float *xsum = xs + (size_t)(slice / 128) * BS;        // [slice / 128][MP]
  uint8_t *ssal = reinterpret_cast<uint8_t *>(xsum + (slice / 128) * MP);  // [nb][n_sal]
  pdl_trigger();
  pdl_wait();
  const int nb = (int)(K / 128);
  for (int i = threadIdx.x; i < nb * n_sal; i += BR_THREADS) ssal[i] = sal[i];
  const int lane = threadIdx.x % 32, part = lane % BR_SPLIT;
  const int slot = (threadIdx.x / 32) * (32 / BR_SPLIT) + lane / BR_SPLIT;
  const int64_t groups = ceil_div<int64_t>(N, BR_ROWS);
  bool bad = false;

  for (int64_t mt0 = 0; mt0 < M; mt0 += MP) {
    for (int64_t rg = blockIdx.x; rg < groups; rg += gridDim.x) {
      const int64_t n = rg * BR_ROWS + slot;
      const bool live = n < N;
      const int64_t nr = live ? n : N - 1;  // rows past N compute a valid row, store nothing
      float y[MP];
#pragma unroll
      for (int m = 0; m < MP; ++m) y[m] = 0.0f;
      for (int64_t k0 = 0; k0 < K; k0 += slice) {
        const int cols = (int)(K - k0 < slice ? K - k0 : (int64_t)slice), jb0 = (int)(k0 / 128);
        // this thread's first block of the slice: its words are requested
        // before the staging below, which does not need them
        const int jend = jb0 + cols / 128;
        int j = jb0 + part;
        uint4 sw = make_uint4(0, 0, 0, 0), gw = sw;
        float4 sc = make_float4(0, 0, 0, 0);
        uint32_t rb = 0;
        if (j < jend) {
          sw = __ldg(reinterpret_cast<const uint4 *>(sign + nr * ldw) + j);
          gw = __ldg(reinterpret_cast<const uint4 *>(gmap + nr * ldw) + j);
          sc = __ldg(reinterpret_cast<const float4 *>(bscale) + nr * nb + j);
          rb = res[nr * nb + j];
        }
        // stage rows mt0 .. mt0 + MP - 1 of X over this slice (consecutive
        // threads: consecutive rows of one column, so the stores are
        // conflict-free and each thread's loads stay in a few L1 sectors),
        // then the block sums in a fixed order
        __syncthreads();
        for (int idx = threadIdx.x; idx < cols * MP; idx += BR_THREADS) {
          const int m = idx % MP, c = idx / MP;
          float v = 0.0f;
          if (mt0 + m < M) {
            const __half_raw hr = {__ldg(X + (mt0 + m) * ldX + k0 + c)};
            bad |= (hr.x & 0x7C00u) == 0x7C00u;
            v = __half2float(__half(hr));
          }
          xs[(c >> 7) * BS + (c & 127) * MP + m] = v;
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < (cols / 128) * MP; idx += BR_THREADS) {
          const int jl = idx / MP, m = idx % MP;
          float acc = 0.0f;
          for (int c = 0; c < 128; ++c) acc += xs[jl * BS + c * MP + m];
          xsum[jl * MP + m] = acc;
        }
        __syncthreads();
        for (; j < jend; j += BR_SPLIT) {
          uint4 nsw = make_uint4(0, 0, 0, 0), ngw = nsw;
          float4 nsc = make_float4(0, 0, 0, 0);
          uint32_t nrb = 0;
          if (j + BR_SPLIT < jend) {
            nsw = __ldg(reinterpret_cast<const uint4 *>(sign + nr * ldw) + j + BR_SPLIT);
            ngw = __ldg(reinterpret_cast<const uint4 *>(gmap + nr * ldw) + j + BR_SPLIT);
            nsc = __ldg(reinterpret_cast<const float4 *>(bscale) + nr * nb + j + BR_SPLIT);
            nrb = res[nr * nb + j + BR_SPLIT];
          }
          const float *xj = xs + (size_t)(j - jb0) * BS;
          const uint32_t swa[4] = {sw.x, sw.y, sw.z, sw.w}, gwa[4] = {gw.x, gw.y, gw.z, gw.w};
          float neg[MP];
#pragma unroll
          for (int m = 0; m < MP; ++m) neg[m] = 0.0f;
          // sum of x over the columns whose sign bit is 1
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t w = swa[q];
            if (MP == 1) {
#pragma unroll
              for (int b4 = 0; b4 < 8; ++b4) {
                const float4 x4 = *reinterpret_cast<const float4 *>(xj + q * 32 + b4 * 4);
                if (w & (1u << (4 * b4 + 0))) neg[0] += x4.x;
                if (w & (1u << (4 * b4 + 1))) neg[0] += x4.y;
                if (w & (1u << (4 * b4 + 2))) neg[0] += x4.z;
                if (w & (1u << (4 * b4 + 3))) neg[0] += x4.w;
              }
            } else {
#pragma unroll 8
              for (int b = 0; b < 32; ++b) {
                if (w & (1u << b)) {
                  const float *xc = xj + (q * 32 + b) * MP;
                  if (MP >= 4) {
#pragma unroll
                    for (int m4 = 0; m4 < MP; m4 += 4) {
                      const float4 v = *reinterpret_cast<const float4 *>(xc + m4);
                      neg[m4] += v.x;
                      neg[m4 + 1] += v.y;
                      neg[m4 + 2] += v.z;
                      neg[m4 + 3] += v.w;
                    }
                  } else {
#pragma unroll
                    for (int m = 0; m < MP; ++m) neg[m] += xc[m];
                  }
                }
              }
            }
          }
          const float *xsj = xsum + (j - jb0) * MP;
#pragma unroll
          for (int m = 0; m < MP; ++m) y[m] = fmaf(sc.x, fmaf(-2.0f, neg[m], xsj[m]), y[m]);
          // sparse columns: (alpha_sp - alpha_c) * b * x
          const float dsp = sc.y - sc.x;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t g = gwa[q];
            while (g) {
              const int b = __ffs(g) - 1;
              g &= g - 1;
              const float cf = ((swa[q] >> b) & 1u) ? -dsp : dsp;
              const float *xc = xj + (q * 32 + b) * MP;
#pragma unroll
              for (int m = 0; m < MP; ++m) y[m] = fmaf(cf, xc[m], y[m]);
            }
          }
          // salient columns: (alpha1 - alpha_c) * b1 + alpha2 * b2
          const float d1 = sc.z - sc.x;
          for (int i = 0; i < n_sal; ++i) {
            const int c = ssal[j * n_sal + i];
            const uint32_t wc = c < 64 ? (c < 32 ? sw.x : sw.y) : (c < 96 ? sw.z : sw.w);
            const float cf = (((wc >> (c & 31)) & 1u) ? -d1 : d1) +
                             (((rb >> i) & 1u) ? -sc.w : sc.w);
            const float *xc = xj + c * MP;
#pragma unroll
            for (int m = 0; m < MP; ++m) y[m] = fmaf(cf, xc[m], y[m]);
          }
          sw = nsw;
          gw = ngw;
          sc = nsc;
          rb = nrb;
        }
      }
      // the row's four partial sums (blocks of all four residues)
#pragma unroll
      for (int m = 0; m < MP; ++m) {
        y[m] += __shfl_xor_sync(FULL, y[m], 1);
        y[m] += __shfl_xor_sync(FULL, y[m], 2);
      }
      if (live && part == 0) {
#pragma unroll
        for (int m = 0; m < MP; ++m)
          if (mt0 + m < M) Y[(mt0 + m) * ldY + n] = y[m];
      }
    }
  }
  if (bad) flag_status(d_status, BWTA_STATUS_NONFINITE);
}

// Columns of K staged per pass: all of K when it fits, else a multiple of 512
// (every thread then has blocks in each slice).
static int br_slice(int mp, int64_t K) {
  // per 128 columns: the staged block (128 * mp + 4 floats) and its mp sums
  const int64_t per_block = ((int64_t)128 * mp + 4 + mp) * 4;
  const int64_t fit = (int64_t)(BR_SMEM_BUDGET - BR_MAX_NB * 8) / per_block * 128;
  if (fit >= K) return (int)K;
  return (int)std::max<int64_t>(512, fit / 512 * 512);
}

template <int MP>
static cudaError_t launch_br_t(const uint16_t *X, int64_t M, int64_t ldX, const billm_weights *W,
                               float *Y, int64_t ldY, int32_t *d_status, cudaStream_t s) {
  auto kern = k_billm_rows<MP>;
  constexpr int BR_THREADS = br_threads<MP>(), BR_ROWS = BR_THREADS / BR_SPLIT;
  const int slice = br_slice(MP, W->K);
  const size_t smem = (size_t)(slice / 128) * (128 * MP + 4 + MP) * 4 +
                      (size_t)(W->K / 128) * W->n_sal;
  static SmemOptIn opt_in;
  if (cudaError_t e = opt_in(kern, (int)smem)) return e;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, BR_THREADS, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t blocks =
      std::min<int64_t>(ceil_div<int64_t>(W->N, BR_ROWS), (int64_t)sms * per_sm);
  return launch_pdl(kern, dim3((unsigned)blocks), dim3(BR_THREADS), smem, s, X, M, ldX, W->sign,
                    W->gmap, W->res, W->sal, W->bscale, W->N, W->K, W->ldw_words, (int)W->n_sal, Y,
                    ldY, slice, d_status);
}

cudaError_t launch_billm_gemm(const uint16_t *X, int64_t M, int64_t ldX, const billm_weights *W,
                              float *Y, int64_t ldY, int32_t *d_status, cudaStream_t s) {
  if (M == 0 || W->N == 0) return cudaSuccess;
  // M <= 8 on CUDA cores (the weight rebuild of the tensor-core kernel costs
  // as much at M = 2 as at M = 512: measured 648 us at M = 2..16 against 155,
  // 355 and 425 us here for M = 2, 4, 8); larger M on tensor cores, when X
  // satisfies the TMA alignment rules.
  if (M > 8) {
    const cudaError_t e = launch_billm_gemm_tc(X, M, ldX, W, Y, ldY, d_status, s);
    if (e != cudaErrorNotSupported) return e;
  }
  if (M == 1) return launch_br_t<1>(X, M, ldX, W, Y, ldY, d_status, s);
  if (M == 2) return launch_br_t<2>(X, M, ldX, W, Y, ldY, d_status, s);
  if (M <= 4) return launch_br_t<4>(X, M, ldX, W, Y, ldY, d_status, s);
  if (M <= 8) return launch_br_t<8>(X, M, ldX, W, Y, ldY, d_status, s);
  return launch_br_t<16>(X, M, ldX, W, Y, ldY, d_status, s);
}

}  // namespace bwta
