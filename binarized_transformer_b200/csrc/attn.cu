// attn.cu -- ternary x ternary attention scores Q . K^T.
//
// BWTA: Accurate and Efficient Binarized Transformer by Algorithm-Hardware
// Co-design -- abstract: the binary/ternary MatMul also serves the attention
// operators. With both operands ternary, a position contributes only where
// both masks are set:
//     S = popc(mq & mk) - 2 * popc(mq & mk & (sq ^ sk))
// The output (B*H*L*L scores) is far larger than the input (two planes of
// D/32 words per row), so the kernel is bound by its output stream: each warp
// writes 512 contiguous bytes per row with 16-byte streaming stores, and the
// small per-thread state keeps several CTAs (many stores in flight) per SM.
#include "common.cuh"

namespace bwta {

constexpr int AT_TQ = 128, AT_TK = 128, AT_THREADS = 256;

__device__ __forceinline__ void st_cs(int32_t *p, int4 v) { __stcs(reinterpret_cast<int4 *>(p), v); }
__device__ __forceinline__ void st_cs(float *p, float4 v) { __stcs(reinterpret_cast<float4 *>(p), v); }

// Per word, with m = mq & mk and x = m & (sq ^ sk):
//   popc(m) - 2*popc(x) = popc(m & ~x) - popc(x) = popc(agree) + popc(~x) - 32,
// so a row pair's score is a plain sum of popcounts over 2*NW words minus 32*NW,
// which carry-save adders fold into fewer POPCs (3 for NW = 2, 4 for NW = 4).
__device__ __forceinline__ uint32_t agree_w(uint32_t m, uint32_t a, uint32_t b) {
  uint32_t r;  // m & ~(a ^ b): 0xF0 & ~(0xCC ^ 0xAA) = 0x90
  asm("lop3.b32 %0, %1, %2, %3, 0x90;" : "=r"(r) : "r"(m), "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t ndis_w(uint32_t m, uint32_t a, uint32_t b) {
  uint32_t r;  // ~(m & (a ^ b)): ~0x60 = 0x9F
  asm("lop3.b32 %0, %1, %2, %3, 0x9F;" : "=r"(r) : "r"(m), "r"(a), "r"(b));
  return r;
}

template <int NW>
__device__ __forceinline__ int tern_dot(const uint4 &qm, const uint4 &qs, const uint4 &km, const uint4 &ks) {
  const uint32_t m0 = qm.x & km.x;
  if (NW == 1) return __popc(agree_w(m0, qs.x, ks.x)) - __popc(lop3_and_xor(m0, qs.x, ks.x));
  const uint32_t m1 = qm.y & km.y;
  if (NW == 2)
    return popc4_csa(agree_w(m0, qs.x, ks.x), agree_w(m1, qs.y, ks.y), ndis_w(m0, qs.x, ks.x),
                     ndis_w(m1, qs.y, ks.y)) - 64;
  const uint32_t m2 = qm.z & km.z, m3 = qm.w & km.w;
  const uint32_t a0 = agree_w(m0, qs.x, ks.x), a1 = agree_w(m1, qs.y, ks.y),
                 a2 = agree_w(m2, qs.z, ks.z), a3 = agree_w(m3, qs.w, ks.w);
  const uint32_t n0 = ndis_w(m0, qs.x, ks.x), n1 = ndis_w(m1, qs.y, ks.y),
                 n2 = ndis_w(m2, qs.z, ks.z), n3 = ndis_w(m3, qs.w, ks.w);
  // eight words -> ones (s3, n3), twos (s4), fours (c4)
  const uint32_t s1 = xor3(a0, a1, a2), c1 = maj3(a0, a1, a2);
  const uint32_t s2 = xor3(a3, n0, n1), c2 = maj3(a3, n0, n1);
  const uint32_t s3 = xor3(s1, s2, n2), c3 = maj3(s1, s2, n2);
  const uint32_t s4 = xor3(c1, c2, c3), c4 = maj3(c1, c2, c3);
  return __popc(s3) + __popc(n3) + 2 * __popc(s4) + 4 * __popc(c4) - 128;
}

// CTA tile: 128 query rows x 128 key rows of one (batch, head). Lane l holds
// the planes of key rows 4l .. 4l+3 in registers for the whole tile; warp w
// walks query rows w, w + 8, ... (16 of them), and for each computes its 4
// scores and stores them at once (16 bytes; 512 contiguous bytes per warp), so
// no scores are held in registers and many CTAs stay resident per SM. NW =
// data words per row (1 or 2 in one chunk; 4 = any D in 4-word chunks).
template <int NW, bool WI, bool WF, bool VEC>
__global__ void __launch_bounds__(AT_THREADS, 4)
k_attn_scores(const uint32_t *__restrict__ qm, const uint32_t *__restrict__ qs,
              const float *__restrict__ qscale, const uint32_t *__restrict__ km,
              const uint32_t *__restrict__ ks, const float *__restrict__ kscale, int64_t Lq,
              int64_t Lk, int ld, int32_t *__restrict__ Si, float *__restrict__ Sf) {
  extern __shared__ uint4 at_sm[];
  const int nc = NW == 4 ? ld / 4 : 1;  // 4-word chunks per row
  uint4 *sQm = at_sm;
  uint4 *sQs = sQm + AT_TQ * nc;
  uint4 *sKm = sQs + AT_TQ * nc;
  uint4 *sKs = sKm + AT_TK * nc;
  float *sq = reinterpret_cast<float *>(sKs + AT_TK * nc);
  float *sk = sq + AT_TQ;
  pdl_trigger();
  pdl_wait();
  const int64_t bh = blockIdx.z;
  const int64_t i0 = (int64_t)blockIdx.y * AT_TQ, j0 = (int64_t)blockIdx.x * AT_TK;
  const uint4 z4 = make_uint4(0, 0, 0, 0);
  for (int idx = threadIdx.x; idx < AT_TQ * nc; idx += AT_THREADS) {
    const int r = idx / nc, c = idx % nc;
    const int64_t i = i0 + r;
    const bool in = i < Lq;
    const int64_t off = (bh * Lq + i) * ld;
    sQm[idx] = in ? __ldg(reinterpret_cast<const uint4 *>(qm + off) + c) : z4;
    sQs[idx] = in ? __ldg(reinterpret_cast<const uint4 *>(qs + off) + c) : z4;
  }
  // K tile: [key][chunk] for one-chunk rows; chunk-major [chunk][key] for the
  // general path, so that lanes reading consecutive keys hit consecutive
  // 16-byte slots (no bank conflicts)
  for (int idx = threadIdx.x; idx < AT_TK * nc; idx += AT_THREADS) {
    const int r = idx / nc, c = idx % nc;
    const int64_t j = j0 + r;
    const bool in = j < Lk;
    const int64_t off = (bh * Lk + j) * ld;
    const int dst = NW == 4 ? c * AT_TK + r : idx;
    sKm[dst] = in ? __ldg(reinterpret_cast<const uint4 *>(km + off) + c) : z4;
    sKs[dst] = in ? __ldg(reinterpret_cast<const uint4 *>(ks + off) + c) : z4;
  }
  if (WF) {
    for (int idx = threadIdx.x; idx < AT_TQ; idx += AT_THREADS)
      sq[idx] = (i0 + idx < Lq) ? __ldg(qscale + bh * Lq + i0 + idx) : 0.0f;
    for (int idx = threadIdx.x; idx < AT_TK; idx += AT_THREADS)
      sk[idx] = (j0 + idx < Lk) ? __ldg(kscale + bh * Lk + j0 + idx) : 0.0f;
  }
  __syncthreads();

  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  // this lane's keys: 4l .. 4l+3 (one-chunk rows, one 16-byte store per row)
  // or l, l+32, l+64, l+96 (general path, four coalesced 4-byte stores)
  auto key = [&](int t) { return NW == 4 ? l + 32 * t : 4 * l + t; };
  const int64_t jb = j0 + 4 * l;
  float skv[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) skv[t] = WF ? sk[key(t)] : 0.0f;
  uint4 kmv[4], ksv[4];
  if (NW != 4) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      kmv[t] = sKm[4 * l + t];
      ksv[t] = sKs[4 * l + t];
    }
  }
  for (int r = w; r < AT_TQ; r += AT_THREADS / 32) {
    const int64_t i = i0 + r;
    if (i >= Lq) break;
    int d[4] = {0, 0, 0, 0};
    if (NW != 4) {
      const uint4 a = sQm[r], b = sQs[r];
#pragma unroll
      for (int t = 0; t < 4; ++t) d[t] = tern_dot<NW>(a, b, kmv[t], ksv[t]);
    } else {
      for (int c = 0; c < nc; ++c) {
        const uint4 a = sQm[r * nc + c], b = sQs[r * nc + c];
#pragma unroll
        for (int t = 0; t < 4; ++t)
          d[t] += tern_dot<4>(a, b, sKm[c * AT_TK + key(t)], sKs[c * AT_TK + key(t)]);
      }
    }
    float f[4];
    if (WF) {
      const float sqi = sq[r];
#pragma unroll
      for (int t = 0; t < 4; ++t) f[t] = (__int2float_rn(d[t]) * sqi) * skv[t];
    }
    if (NW == 4) {
      const int64_t orow = (bh * Lq + i) * Lk + j0;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (j0 + key(t) >= Lk) break;
        if (WI) __stcs(Si + orow + key(t), d[t]);
        if (WF) __stcs(Sf + orow + key(t), f[t]);
      }
      continue;
    }
    const int64_t o = (bh * Lq + i) * Lk + jb;
    if (VEC && jb + 3 < Lk) {
      if (WI) st_cs(Si + o, make_int4(d[0], d[1], d[2], d[3]));
      if (WF) st_cs(Sf + o, make_float4(f[0], f[1], f[2], f[3]));
    } else {
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (jb + t >= Lk) break;
        if (WI) Si[o + t] = d[t];
        if (WF) Sf[o + t] = f[t];
      }
    }
  }
}

template <int NW, bool WI, bool WF, bool VEC>
static cudaError_t launch_attn_t(const uint32_t *qm, const uint32_t *qs, const float *qscale,
                                 const uint32_t *km, const uint32_t *ks, const float *kscale,
                                 int64_t BH, int64_t Lq, int64_t Lk, int64_t ld, int32_t *Si,
                                 float *Sf, cudaStream_t s) {
  const int nc = NW == 4 ? (int)(ld / 4) : 1;
  const size_t smem = (size_t)(AT_TQ + AT_TK) * nc * 2 * 16 + (AT_TQ + AT_TK) * 4;
  auto kern = k_attn_scores<NW, WI, WF, VEC>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((unsigned)ceil_div<int64_t>(Lk, AT_TK), (unsigned)ceil_div<int64_t>(Lq, AT_TQ),
            (unsigned)BH);
  return launch_pdl(kern, grid, dim3(AT_THREADS), smem, s, qm, qs, qscale, km, ks, kscale, Lq, Lk,
                    (int)ld, Si, Sf);
}

template <int NW>
static cudaError_t launch_attn_nw(const uint32_t *qm, const uint32_t *qs, const float *qscale,
                                  const uint32_t *km, const uint32_t *ks, const float *kscale,
                                  int64_t BH, int64_t Lq, int64_t Lk, int64_t ld, int32_t *Si,
                                  float *Sf, cudaStream_t s) {
  const bool vec = (Lk % 4) == 0;
#define BWTA_AT(WI, WF)                                                                         \
  return vec ? launch_attn_t<NW, WI, WF, true>(qm, qs, qscale, km, ks, kscale, BH, Lq, Lk, ld, Si, \
                                               Sf, s)                                            \
             : launch_attn_t<NW, WI, WF, false>(qm, qs, qscale, km, ks, kscale, BH, Lq, Lk, ld, Si, \
                                                Sf, s)
  if (Si && Sf) BWTA_AT(true, true);
  if (Si) BWTA_AT(true, false);
  BWTA_AT(false, true);
#undef BWTA_AT
}

// ============================================ softmax -> ternary probabilities
// The attention probabilities are the activations of the A . V product, so
// they are ternarized like any activation (BWTA abstract: binary/ternary
// MatMul for the attention operators): keep p iff p > 0.5 * mean(p) over the
// row. A softmax row sums to one, so that threshold is 1/(2 Lk); every p is
// positive, so the kept values are +1 (the sign plane is all zero) and the row
// scale is the mean of the kept p. This kernel goes from the ternary Q and K
// planes straight to those planes: the Lq x Lk scores are never written to
// memory. One CTA per (batch*head, 64 query rows) holds the head's K planes in
// shared memory; a warp owns a query row: per key, the ternary dot, the fp32
// score ((float)S * s_q) * s_k (the same value bwta_attn_scores writes) times
// the softmax factor (fp32); the row max; e = exp(x - max) in fp32 (the CUDA
// expf, a few ulp); then in fp64 the sum Z, the keep decision e > Z / (2 Lk)
// (that is p = e / Z > 1/(2 Lk), without a divide per key; one ballot per 32
// keys is one mask word) and the kept sum. The fp64 sums make the decision and
// the scale independent of the summation order; what remains is expf's
// rounding, so a probability within ~1e-6 (relative) of the threshold can
// fall either way.
constexpr int AS_ROWS = 64, AS_THREADS = 256, AS_WARPS = AS_THREADS / 32;

template <int NW>
__global__ void __launch_bounds__(AS_THREADS)
k_attn_softmax_pack(const uint32_t *__restrict__ qm, const uint32_t *__restrict__ qs,
                    const float *__restrict__ qscale, const uint32_t *__restrict__ km,
                    const uint32_t *__restrict__ ks, const float *__restrict__ kscale, int64_t Lq,
                    int64_t Lk, int ld, float c, uint32_t *__restrict__ pm, uint32_t *__restrict__ ps,
                    int ldp, float *__restrict__ pscale) {
  extern __shared__ uint4 as_sm[];
  const int nc = NW == 4 ? ld / 4 : 1;
  uint4 *sKm = as_sm;
  uint4 *sKs = sKm + Lk * nc;
  float *sk = reinterpret_cast<float *>(sKs + Lk * nc);
  float *xw = sk + Lk + (threadIdx.x / 32) * Lk;  // this warp's row of scores, then of exp
  pdl_trigger();
  pdl_wait();
  const int64_t bh = blockIdx.y;
  for (int idx = threadIdx.x; idx < Lk * nc; idx += AS_THREADS) {
    const int64_t off = (bh * Lk + idx / nc) * ld;
    sKm[idx] = __ldg(reinterpret_cast<const uint4 *>(km + off) + idx % nc);
    sKs[idx] = __ldg(reinterpret_cast<const uint4 *>(ks + off) + idx % nc);
  }
  for (int idx = threadIdx.x; idx < Lk; idx += AS_THREADS) sk[idx] = __ldg(kscale + bh * Lk + idx);
  __syncthreads();

  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  const double thr = 0.5 / (double)Lk;  // the keep test e > Z * thr
  for (int r = w; r < AS_ROWS; r += AS_WARPS) {
    const int64_t i = (int64_t)blockIdx.x * AS_ROWS + r;
    if (i >= Lq) break;
    const int64_t qrow = (bh * Lq + i) * ld;
    const float sqi = __ldg(qscale + bh * Lq + i);
    uint4 qa[NW == 4 ? 8 : 1], qb[NW == 4 ? 8 : 1];
#pragma unroll
    for (int cc = 0; cc < (NW == 4 ? 8 : 1); ++cc) {
      if (cc < nc) {
        qa[cc] = __ldg(reinterpret_cast<const uint4 *>(qm + qrow) + cc);
        qb[cc] = __ldg(reinterpret_cast<const uint4 *>(qs + qrow) + cc);
      }
    }
    // scores times the softmax factor, and the row max
    float mx = -INFINITY;
    const int lk = (int)Lk;
    for (int j = l; j < lk; j += 32) {
      int d = 0;
      if (NW != 4) {
        d = tern_dot<NW>(qa[0], qb[0], sKm[j], sKs[j]);
      } else {
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          if (cc < nc) d += tern_dot<4>(qa[cc], qb[cc], sKm[j * nc + cc], sKs[j * nc + cc]);
      }
      const float x = ((__int2float_rn(d) * sqi) * sk[j]) * c;
      xw[j] = x;
      mx = fmaxf(mx, x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
    double z = 0.0;
    for (int j = l; j < lk; j += 32) {
      const float e = expf(xw[j] - mx);
      xw[j] = e;
      z += (double)e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(FULL, z, o);
    const double cut = z * thr;
    // For an fp32 value e, e > cut exactly when e > cut rounded down to fp32
    // (the largest fp32 not above cut): the keep test runs in fp32.
    const float cut32 = __double2float_rd(cut);
    // keep bits: key j = 32t + l is bit l of mask word t
    double ksum = 0.0;
    int kn = 0;
    uint32_t *mrow = pm + (bh * Lq + i) * ldp, *srow = ps + (bh * Lq + i) * ldp;
    uint32_t myword = 0;  // lane l keeps mask word l (of each group of 32 words)
    const int nt = (lk + 31) / 32;
    for (int t = 0; t < nt; ++t) {
      const int j = t * 32 + l;
      const float e = j < lk ? xw[j] : 0.0f;
      const bool keep = e > cut32;
      const uint32_t word = __ballot_sync(FULL, keep);
      if (keep) ksum += (double)e;
      kn += keep;
      if (l == (t & 31)) myword = word;
      if ((t & 31) == 31 || t + 1 == nt) {  // one coalesced store per 32 words
        const int t0 = t & ~31;
        if (t0 + l <= t) {
          mrow[t0 + l] = myword;
          srow[t0 + l] = 0u;
        }
      }
    }
    for (int t = nt + l; t < ldp; t += 32) {  // padding words
      mrow[t] = 0u;
      srow[t] = 0u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ksum += __shfl_xor_sync(FULL, ksum, o);
      kn += __shfl_xor_sync(FULL, kn, o);
    }
    // scale = mean of the kept p = (sum of the kept e / Z) / count
    if (l == 0) pscale[bh * Lq + i] = kn ? __double2float_rn(__ddiv_rn(__ddiv_rn(ksum, z), (double)kn)) : 0.0f;
  }
}

size_t attn_softmax_smem(int64_t Lk, int64_t ld) {
  const int64_t nc = ld / 4 > 1 ? ld / 4 : 1;
  return (size_t)Lk * nc * 32 + (size_t)Lk * 4 + (size_t)AS_WARPS * Lk * 4;
}

template <int NW>
static cudaError_t launch_softmax_t(const uint32_t *qm, const uint32_t *qs, const float *qscale,
                                    const uint32_t *km, const uint32_t *ks, const float *kscale,
                                    int64_t BH, int64_t Lq, int64_t Lk, int64_t ld, float c,
                                    uint32_t *pm, uint32_t *ps, int64_t ldp, float *pscale,
                                    cudaStream_t s) {
  auto kern = k_attn_softmax_pack<NW>;
  const size_t smem = attn_softmax_smem(Lk, NW == 4 ? ld : 4);
  static SmemOptIn opt_in;
  if (cudaError_t e = opt_in(kern, (int)smem)) return e;
  dim3 grid((unsigned)ceil_div<int64_t>(Lq, AS_ROWS), (unsigned)BH);
  return launch_pdl(kern, grid, dim3(AS_THREADS), smem, s, qm, qs, qscale, km, ks, kscale, Lq, Lk,
                    (int)ld, c, pm, ps, (int)ldp, pscale);
}

cudaError_t launch_attn_softmax(const uint32_t *qm, const uint32_t *qs, const float *qscale,
                                const uint32_t *km, const uint32_t *ks, const float *kscale,
                                int64_t BH, int64_t Lq, int64_t Lk, int64_t D, int64_t ld, float c,
                                uint32_t *pm, uint32_t *ps, int64_t ldp, float *pscale,
                                cudaStream_t s) {
  if (BH == 0 || Lq == 0) return cudaSuccess;
  const int64_t nw = ceil_div<int64_t>(D, 32);
  if (nw == 1)
    return launch_softmax_t<1>(qm, qs, qscale, km, ks, kscale, BH, Lq, Lk, ld, c, pm, ps, ldp, pscale, s);
  if (nw == 2)
    return launch_softmax_t<2>(qm, qs, qscale, km, ks, kscale, BH, Lq, Lk, ld, c, pm, ps, ldp, pscale, s);
  return launch_softmax_t<4>(qm, qs, qscale, km, ks, kscale, BH, Lq, Lk, ld, c, pm, ps, ldp, pscale, s);
}

cudaError_t launch_attn_scores(const uint32_t *qm, const uint32_t *qs, const float *qscale,
                               const uint32_t *km, const uint32_t *ks, const float *kscale,
                               int64_t BH, int64_t Lq, int64_t Lk, int64_t D, int64_t ld,
                               int32_t *Si, float *Sf, cudaStream_t s) {
  if (BH == 0 || Lq == 0 || Lk == 0) return cudaSuccess;
  const int64_t nw = ceil_div<int64_t>(D, 32);  // data words per row
  if (nw == 1) return launch_attn_nw<1>(qm, qs, qscale, km, ks, kscale, BH, Lq, Lk, ld, Si, Sf, s);
  if (nw == 2) return launch_attn_nw<2>(qm, qs, qscale, km, ks, kscale, BH, Lq, Lk, ld, Si, Sf, s);
  return launch_attn_nw<4>(qm, qs, qscale, km, ks, kscale, BH, Lq, Lk, ld, Si, Sf, s);
}

}  // namespace bwta
