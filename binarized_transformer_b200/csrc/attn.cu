// attn.cu -- ternary x ternary attention scores Q . K^T.
//
// BWTA: Accurate and Efficient Binarized Transformer by Algorithm-Hardware
// Co-design -- abstract: the binary/ternary MatMul also serves the attention
// operators. With both operands ternary, a position contributes only where
// both masks are set:
//     S = popc(mq & mk) - 2 * popc(mq & mk & (sq ^ sk))
// The output (B*H*L*L scores) is far larger than the input (two planes of
// D/32 words per row), so the kernel is bound by its output stream: each warp
// writes 512 contiguous bytes per row with 16-byte streaming stores.
#include "common.cuh"

namespace bwta {

constexpr int AT_TQ = 64, AT_TK = 128, AT_THREADS = 256;

__device__ __forceinline__ void st_cs(int32_t *p, int4 v) { __stcs(reinterpret_cast<int4 *>(p), v); }
__device__ __forceinline__ void st_cs(float *p, float4 v) { __stcs(reinterpret_cast<float4 *>(p), v); }

// CTA tile: 64 query rows x 128 key rows of one (batch, head). Warp w owns
// query rows w + 8*r (r < 8); lane l owns key rows 4l .. 4l+3, so a warp's
// stores for one query row are 128 consecutive scores.
template <bool WI, bool WF, bool VEC>
__global__ void __launch_bounds__(AT_THREADS)
k_attn_scores(const uint32_t *__restrict__ qm, const uint32_t *__restrict__ qs,
              const float *__restrict__ qscale, const uint32_t *__restrict__ km,
              const uint32_t *__restrict__ ks, const float *__restrict__ kscale, int64_t Lq,
              int64_t Lk, int ld, int32_t *__restrict__ Si, float *__restrict__ Sf) {
  extern __shared__ uint4 at_sm[];
  const int nc = ld / 4;  // 4-word chunks per row
  uint4 *sQm = at_sm;
  uint4 *sQs = sQm + AT_TQ * nc;
  uint4 *sKm = sQs + AT_TQ * nc;
  uint4 *sKs = sKm + AT_TK * nc;
  float *sq = reinterpret_cast<float *>(sKs + AT_TK * nc);
  float *sk = sq + AT_TQ;

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
  for (int idx = threadIdx.x; idx < AT_TK * nc; idx += AT_THREADS) {
    const int r = idx / nc, c = idx % nc;
    const int64_t j = j0 + r;
    const bool in = j < Lk;
    const int64_t off = (bh * Lk + j) * ld;
    sKm[idx] = in ? __ldg(reinterpret_cast<const uint4 *>(km + off) + c) : z4;
    sKs[idx] = in ? __ldg(reinterpret_cast<const uint4 *>(ks + off) + c) : z4;
  }
  if (WF) {
    for (int idx = threadIdx.x; idx < AT_TQ; idx += AT_THREADS)
      sq[idx] = (i0 + idx < Lq) ? __ldg(qscale + bh * Lq + i0 + idx) : 0.0f;
    for (int idx = threadIdx.x; idx < AT_TK; idx += AT_THREADS)
      sk[idx] = (j0 + idx < Lk) ? __ldg(kscale + bh * Lk + j0 + idx) : 0.0f;
  }
  __syncthreads();

  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  int P[8][4], X[8][4];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int t = 0; t < 4; ++t) P[r][t] = X[r][t] = 0;

  for (int c = 0; c < nc; ++c) {
    uint4 kmv[4], ksv[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      kmv[t] = sKm[(4 * l + t) * nc + c];
      ksv[t] = sKs[(4 * l + t) * nc + c];
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const uint4 a = sQm[(w + 8 * r) * nc + c], b = sQs[(w + 8 * r) * nc + c];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t m0 = a.x & kmv[t].x, m1 = a.y & kmv[t].y, m2 = a.z & kmv[t].z,
                       m3 = a.w & kmv[t].w;
        P[r][t] += __popc(m0) + __popc(m1) + __popc(m2) + __popc(m3);
        X[r][t] += __popc(lop3_and_xor(m0, b.x, ksv[t].x)) + __popc(lop3_and_xor(m1, b.y, ksv[t].y)) +
                   __popc(lop3_and_xor(m2, b.z, ksv[t].z)) + __popc(lop3_and_xor(m3, b.w, ksv[t].w));
      }
    }
  }

#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int64_t i = i0 + w + 8 * r;
    if (i >= Lq) continue;
    const int64_t jb = j0 + 4 * l;
    const int64_t o = (bh * Lq + i) * Lk + jb;
    int d[4];
    float f[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      d[t] = P[r][t] - 2 * X[r][t];
      if (WF) f[t] = (__int2float_rn(d[t]) * sq[w + 8 * r]) * sk[4 * l + t];
    }
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

template <bool WI, bool WF, bool VEC>
static cudaError_t launch_attn_t(const uint32_t *qm, const uint32_t *qs, const float *qscale,
                                 const uint32_t *km, const uint32_t *ks, const float *kscale,
                                 int64_t BH, int64_t Lq, int64_t Lk, int64_t ld, int32_t *Si,
                                 float *Sf, cudaStream_t s) {
  const int nc = (int)(ld / 4);
  const size_t smem = (size_t)(AT_TQ + AT_TK) * nc * 2 * 16 + (AT_TQ + AT_TK) * 4;
  auto kern = k_attn_scores<WI, WF, VEC>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((unsigned)ceil_div<int64_t>(Lk, AT_TK), (unsigned)ceil_div<int64_t>(Lq, AT_TQ),
            (unsigned)BH);
  kern<<<grid, AT_THREADS, smem, s>>>(qm, qs, qscale, km, ks, kscale, Lq, Lk, (int)ld, Si, Sf);
  return cudaGetLastError();
}

cudaError_t launch_attn_scores(const uint32_t *qm, const uint32_t *qs, const float *qscale,
                               const uint32_t *km, const uint32_t *ks, const float *kscale,
                               int64_t BH, int64_t Lq, int64_t Lk, int64_t ld, int32_t *Si,
                               float *Sf, cudaStream_t s) {
  if (BH == 0 || Lq == 0 || Lk == 0) return cudaSuccess;
  const bool vec = (Lk % 4) == 0;
#define BWTA_AT(WI, WF)                                                                           \
  return vec ? launch_attn_t<WI, WF, true>(qm, qs, qscale, km, ks, kscale, BH, Lq, Lk, ld, Si, Sf, s) \
             : launch_attn_t<WI, WF, false>(qm, qs, qscale, km, ks, kscale, BH, Lq, Lk, ld, Si, Sf, s)
  if (Si && Sf) BWTA_AT(true, true);
  if (Si) BWTA_AT(true, false);
  BWTA_AT(false, true);
#undef BWTA_AT
}

}  // namespace bwta
