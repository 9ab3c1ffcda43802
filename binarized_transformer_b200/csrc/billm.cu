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
  double sc = 0.0, ss = 0.0;
  int nc = 0, ns = 0;
  uint32_t sw[4] = {0, 0, 0, 0}, gw[4] = {0, 0, 0, 0};
  for (int c = 0; c < 128; ++c) {
    const float w = __ldg(wr + c);
    if (w < 0.0f) sw[c >> 5] |= 1u << (c & 31);
    if ((salmask[c >> 5] >> (c & 31)) & 1u) continue;
    const double aw = fabs((double)w);
    if (split && 2.0 * aw > maxabs) {
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
// CUDA-core path. A warp owns one weight row; lane l owns blocks l, l+32, ...
// The CTA keeps up to MT activation rows in shared memory as fp32, laid out
// [m][column-in-block][block] so that the 32 lanes (32 blocks) read 32
// consecutive words. Per block a lane accumulates, per activation row,
//   T  = sum over all 128 columns of (+-x)   (b, or b1 at salient columns)
//   Ts = sum over the sparse group of (+-x)
//   T1 = sum over salient columns of b1*x,  T2 = the same with b2
// and adds alpha_c*(T - Ts - T1) + alpha_sp*Ts + alpha1*T1 + alpha2*T2.
// The sign flip is an XOR of the fp32 sign bit, so +-x costs one LOP3. T is
// kept as four partial sums (one per 32-column word) so that the adds of a
// lane form four independent chains. With one activation row the tile is
// 4*K bytes and several CTAs share an SM.
constexpr int BG_THREADS = 256, BG_WARPS = BG_THREADS / 32, BG_MT = 4;
constexpr size_t BG_SMEM_MAX = 160 * 1024;
template <int MT> constexpr int bg_ctas_per_sm() { return MT == 1 ? 4 : 1; }

template <int MT>
__global__ void __launch_bounds__(BG_THREADS, bg_ctas_per_sm<MT>())
k_billm_gemm(const uint16_t *__restrict__ X, int64_t M, int64_t ldX, const uint32_t *__restrict__ sign,
             const uint32_t *__restrict__ gmap, const uint8_t *__restrict__ res,
             const uint8_t *__restrict__ sal, const float *__restrict__ bscale, int64_t N,
             int64_t K, int64_t ldw, int n_sal, float *__restrict__ Y, int64_t ldY,
             int32_t *d_status) {
  extern __shared__ float xs[];  // [MT][128][nb]
  pdl_trigger();
  pdl_wait();
  const int nb = (int)(K / 128);
  uint8_t *ssal = reinterpret_cast<uint8_t *>(xs + (size_t)MT * K);
  for (int i = threadIdx.x; i < nb * n_sal; i += BG_THREADS) ssal[i] = sal[i];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  bool bad = false;
  for (int64_t mt0 = 0; mt0 < M; mt0 += MT) {
    __syncthreads();
    for (int64_t idx = threadIdx.x; idx < (int64_t)MT * K; idx += BG_THREADS) {
      const int m = (int)(idx / K);
      const int64_t k = idx % K;
      float v = 0.0f;
      if (mt0 + m < M) {
        const __half_raw hr = {X[(mt0 + m) * ldX + k]};
        if ((hr.x & 0x7C00u) == 0x7C00u) bad = true;
        v = __half2float(__half(hr));
      }
      xs[((size_t)m * 128 + (k & 127)) * nb + (k >> 7)] = v;
    }
    __syncthreads();
    for (int64_t n = (int64_t)blockIdx.x * BG_WARPS + warp; n < N; n += (int64_t)gridDim.x * BG_WARPS) {
      float y[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) y[m] = 0.0f;
      for (int j = lane; j < nb; j += 32) {
        const uint4 sw = __ldg(reinterpret_cast<const uint4 *>(sign + n * ldw) + j);
        const uint4 gw = __ldg(reinterpret_cast<const uint4 *>(gmap + n * ldw) + j);
        const float4 sc = __ldg(reinterpret_cast<const float4 *>(bscale) + n * nb + j);
        const uint32_t rb = res[n * nb + j];
        float T[MT], Ts[MT], T1[MT], T2[MT], Tq[4][MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          T[m] = Ts[m] = T1[m] = T2[m] = 0.0f;
#pragma unroll
          for (int q = 0; q < 4; ++q) Tq[q][m] = 0.0f;
        }
        const uint32_t swa[4] = {sw.x, sw.y, sw.z, sw.w}, gwa[4] = {gw.x, gw.y, gw.z, gw.w};
#pragma unroll 8
        for (int b = 0; b < 32; ++b) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t flip = (swa[q] << (31 - b)) & 0x80000000u;
            const int c = q * 32 + b;
#pragma unroll
            for (int m = 0; m < MT; ++m)
              Tq[q][m] += __uint_as_float(__float_as_uint(xs[((size_t)m * 128 + c) * nb + j]) ^ flip);
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) T[m] = (Tq[0][m] + Tq[1][m]) + (Tq[2][m] + Tq[3][m]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t s = swa[q];
          uint32_t g = gwa[q];
          while (g) {
            const int b = __ffs(g) - 1;
            g &= g - 1;
            const uint32_t flip = ((s >> b) & 1u) << 31;
            const int c = q * 32 + b;
#pragma unroll
            for (int m = 0; m < MT; ++m)
              Ts[m] += __uint_as_float(__float_as_uint(xs[((size_t)m * 128 + c) * nb + j]) ^ flip);
          }
        }
        for (int i = 0; i < n_sal; ++i) {
          const int c = ssal[j * n_sal + i];
          const uint32_t f1 = ((swa[c >> 5] >> (c & 31)) & 1u) << 31;
          const uint32_t f2 = ((rb >> i) & 1u) << 31;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const uint32_t xb = __float_as_uint(xs[((size_t)m * 128 + c) * nb + j]);
            T1[m] += __uint_as_float(xb ^ f1);
            T2[m] += __uint_as_float(xb ^ f2);
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m)
          y[m] += sc.x * (T[m] - Ts[m] - T1[m]) + sc.y * Ts[m] + sc.z * T1[m] + sc.w * T2[m];
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) y[m] += __shfl_xor_sync(FULL, y[m], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (mt0 + m < M) Y[(mt0 + m) * ldY + n] = y[m];
      }
    }
  }
  if (bad) flag_status(d_status, BWTA_STATUS_NONFINITE);
}

// ------------------------------------------------------------ M = 1 (decode)
// One activation row: it is staged once per CTA in shared memory as fp32,
// block-major with a row stride of 132 floats (16-byte aligned, and lanes j
// reading x[j][c..c+3] hit distinct bank quads), together with the block sums
// X_j = sum_c x[j][c]. A warp owns a weight row, lane l the blocks l, l+32, ...
// For a block, sum_c (+-x) = X_j - 2 * sum_{sign bit 1} x: one predicated add
// per weight, x read four at a time. The sparse group and the salient columns
// are added as before. The next row's planes and scales are loaded while the
// current row is summed.
constexpr int BV_STRIDE = 132;

__global__ void __launch_bounds__(BG_THREADS)
k_billm_gemv(const uint16_t *__restrict__ X, const uint32_t *__restrict__ sign,
             const uint32_t *__restrict__ gmap, const uint8_t *__restrict__ res,
             const uint8_t *__restrict__ sal, const float *__restrict__ bscale, int64_t N,
             int64_t K, int64_t ldw, int n_sal, float *__restrict__ Y, int32_t *d_status) {
  extern __shared__ float xs[];  // [nb][BV_STRIDE], then X_j [nb], then salient table
  pdl_trigger();
  pdl_wait();
  const int nb = (int)(K / 128);
  float *xsum = xs + (size_t)nb * BV_STRIDE;
  uint8_t *ssal = reinterpret_cast<uint8_t *>(xsum + nb);
  for (int i = threadIdx.x; i < nb * n_sal; i += BG_THREADS) ssal[i] = sal[i];
  bool bad = false;
  for (int64_t k = threadIdx.x; k < K; k += BG_THREADS) {
    const __half_raw hr = {X[k]};
    if ((hr.x & 0x7C00u) == 0x7C00u) bad = true;
    xs[(k >> 7) * BV_STRIDE + (k & 127)] = __half2float(__half(hr));
  }
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int j = warp; j < nb; j += BG_WARPS) {  // block sums, fp32, fixed order
    float v = xs[j * BV_STRIDE + lane] + xs[j * BV_STRIDE + lane + 32] +
              xs[j * BV_STRIDE + lane + 64] + xs[j * BV_STRIDE + lane + 96];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    if (lane == 0) xsum[j] = v;
  }
  __syncthreads();
  if (bad) flag_status(d_status, BWTA_STATUS_NONFINITE);

  const int64_t stride = (int64_t)gridDim.x * BG_WARPS;
  int64_t n = (int64_t)blockIdx.x * BG_WARPS + warp;
  // planes and scales of the first block pair of the first row
  auto load = [&](int64_t row, int j, uint4 &sw, uint4 &gw, float4 &sc, uint32_t &rb) {
    if (row < N && j < nb) {
      sw = __ldg(reinterpret_cast<const uint4 *>(sign + row * ldw) + j);
      gw = __ldg(reinterpret_cast<const uint4 *>(gmap + row * ldw) + j);
      sc = __ldg(reinterpret_cast<const float4 *>(bscale) + row * nb + j);
      rb = res[row * nb + j];
    } else {
      sw = gw = make_uint4(0, 0, 0, 0);
      sc = make_float4(0, 0, 0, 0);
      rb = 0;
    }
  };
  uint4 sw0, gw0, sw1, gw1;
  float4 sc0, sc1;
  uint32_t rb0, rb1;
  load(n, lane, sw0, gw0, sc0, rb0);
  load(n, lane + 32, sw1, gw1, sc1, rb1);
  for (; n < N; n += stride) {
    // next row in flight
    uint4 nsw0, ngw0, nsw1, ngw1;
    float4 nsc0, nsc1;
    uint32_t nrb0, nrb1;
    load(n + stride, lane, nsw0, ngw0, nsc0, nrb0);
    load(n + stride, lane + 32, nsw1, ngw1, nsc1, nrb1);
    float y = 0.0f;
    for (int jj = 0; jj < nb; jj += 64) {  // this lane's blocks lane + jj, lane + jj + 32
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int j = lane + jj + half * 32;
        if (j >= nb) continue;
        uint4 sw = half ? sw1 : sw0, gw = half ? gw1 : gw0;
        float4 sc = half ? sc1 : sc0;
        uint32_t rb = half ? rb1 : rb0;
        if (jj > 0) load(n, j, sw, gw, sc, rb);  // K > 8192: blocks past the first 64
        const float *xj = xs + j * BV_STRIDE;
        const uint32_t swa[4] = {sw.x, sw.y, sw.z, sw.w}, gwa[4] = {gw.x, gw.y, gw.z, gw.w};
        float neg[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int b4 = 0; b4 < 8; ++b4) {
            const float4 x4 = *reinterpret_cast<const float4 *>(xj + q * 32 + b4 * 4);
            const uint32_t s = swa[q] >> (b4 * 4);
            if (s & 1u) neg[q] += x4.x;
            if (s & 2u) neg[q] += x4.y;
            if (s & 4u) neg[q] += x4.z;
            if (s & 8u) neg[q] += x4.w;
          }
        }
        const float T = xsum[j] - 2.0f * ((neg[0] + neg[1]) + (neg[2] + neg[3]));
        float Ts = 0.0f, T1 = 0.0f, T2 = 0.0f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t g = gwa[q];
          while (g) {
            const int b = __ffs(g) - 1;
            g &= g - 1;
            const uint32_t flip = ((swa[q] >> b) & 1u) << 31;
            Ts += __uint_as_float(__float_as_uint(xj[q * 32 + b]) ^ flip);
          }
        }
        for (int i = 0; i < n_sal; ++i) {
          const int c = ssal[j * n_sal + i];
          const uint32_t xb = __float_as_uint(xj[c]);
          T1 += __uint_as_float(xb ^ (((swa[c >> 5] >> (c & 31)) & 1u) << 31));
          T2 += __uint_as_float(xb ^ (((rb >> i) & 1u) << 31));
        }
        y += sc.x * (T - Ts - T1) + sc.y * Ts + sc.z * T1 + sc.w * T2;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) y += __shfl_xor_sync(FULL, y, o);
    if (lane == 0) Y[n] = y;
    sw0 = nsw0; gw0 = ngw0; sc0 = nsc0; rb0 = nrb0;
    sw1 = nsw1; gw1 = ngw1; sc1 = nsc1; rb1 = nrb1;
  }
}

static cudaError_t launch_billm_gemv(const uint16_t *X, const billm_weights *W, float *Y,
                                     int32_t *d_status, cudaStream_t s) {
  const size_t smem = (size_t)(W->K / 128) * (BV_STRIDE + 1) * 4 + 8 * (W->K / 128);
  static cudaError_t attr = cudaFuncSetAttribute(
      k_billm_gemv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BG_SMEM_MAX);
  if (attr != cudaSuccess) return attr;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_billm_gemv, BG_THREADS, smem) !=
          cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t blocks =
      std::min<int64_t>(ceil_div<int64_t>(W->N, BG_WARPS), (int64_t)sms * per_sm);
  return launch_pdl(k_billm_gemv, dim3((unsigned)blocks), dim3(BG_THREADS), smem, s, X, W->sign,
                    W->gmap, W->res, W->sal, W->bscale, W->N, W->K, W->ldw_words, (int)W->n_sal,
                    Y, d_status);
}

int billm_gemm_mt(int64_t K) {
  const int64_t per = K * 4;
  int mt = BG_MT;
  while (mt > 1 && (size_t)(mt * per) + 8 * (K / 128) > BG_SMEM_MAX) mt /= 2;
  return ((size_t)(mt * per) + 8 * (K / 128) > BG_SMEM_MAX) ? 0 : mt;
}

template <int MT>
static cudaError_t launch_bg_t(const uint16_t *X, int64_t M, int64_t ldX, const billm_weights *W,
                               float *Y, int64_t ldY, int32_t *d_status, cudaStream_t s) {
  auto kern = k_billm_gemm<MT>;
  static cudaError_t attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BG_SMEM_MAX);
  if (attr != cudaSuccess) return attr;
  const size_t smem = (size_t)MT * W->K * 4 + 8 * (W->K / 128);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, BG_THREADS, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t blocks =
      std::min<int64_t>(ceil_div<int64_t>(W->N, BG_WARPS), (int64_t)sms * per_sm);
  return launch_pdl(kern, dim3((unsigned)blocks), dim3(BG_THREADS), smem, s, X, M, ldX, W->sign,
                    W->gmap, W->res, W->sal, W->bscale, W->N, W->K, W->ldw_words, (int)W->n_sal, Y,
                    ldY, d_status);
}

cudaError_t launch_billm_gemm(const uint16_t *X, int64_t M, int64_t ldX, const billm_weights *W,
                              float *Y, int64_t ldY, int32_t *d_status, cudaStream_t s) {
  if (M == 0 || W->N == 0) return cudaSuccess;
  if (M >= 2) {  // tensor cores, when X satisfies the TMA alignment rules
    const cudaError_t e = launch_billm_gemm_tc(X, M, ldX, W, Y, ldY, d_status, s);
    if (e != cudaErrorNotSupported) return e;
  }
  if (M == 1 && (size_t)(W->K / 128) * (BV_STRIDE + 1) * 4 + 8 * (W->K / 128) <= BG_SMEM_MAX)
    return launch_billm_gemv(X, W, Y, d_status, s);
  const int mt = billm_gemm_mt(W->K);
  if (mt >= 4 && M >= 4) return launch_bg_t<4>(X, M, ldX, W, Y, ldY, d_status, s);
  if (mt >= 2 && M >= 2) return launch_bg_t<2>(X, M, ldX, W, Y, ldY, d_status, s);
  return launch_bg_t<1>(X, M, ldX, W, Y, ldY, d_status, s);
}

}  // namespace bwta
