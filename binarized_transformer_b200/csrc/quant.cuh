// quant.cuh -- device helpers of the exact activation ternarizer, shared by
// the standalone packer (pack.cu) and the fused decode kernel (gemm.cu).
//
// BWTA: Accurate and Efficient Binarized Transformer by Algorithm-Hardware
// Co-design -- abstract: activations are ternarized by projecting tiny values
// to zero; Figure 6: 32 fp16 values packed into one 32-bit word. Keep x iff
// |x| > 0.5*mean|x|, decided exactly on integer magnitudes (units of 2^-24).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace bwta {

constexpr int QA_THREADS = 256;
constexpr int QA_NREG = 8;

template <int T>
__device__ __forceinline__ uint64_t team_sum_u64(uint64_t v, uint64_t *red) {
  if constexpr (T <= 32) {
#pragma unroll
    for (int o = T / 2; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    const int warp = threadIdx.x / 32;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[warp] = v;
    __syncthreads();
    const int w0 = (threadIdx.x / T) * (T / 32);
    uint64_t r = 0;
#pragma unroll
    for (int i = 0; i < T / 32; ++i) r += red[w0 + i];
    return r;
  }
}

// 8 halves starting at k0 (zeros past K). VEC: the row start is 16-byte
// aligned (X aligned, ldX % 8 == 0), so full groups use one 16-byte load.
template <bool VEC>
__device__ __forceinline__ uint4 load_half8(const uint16_t *row, int64_t k0, int64_t K, bool valid) {
  if (!valid || k0 >= K) return make_uint4(0, 0, 0, 0);
  if (VEC && k0 + 8 <= K) return __ldg(reinterpret_cast<const uint4 *>(row + k0));
  uint32_t w[4] = {0, 0, 0, 0};
  for (int i = 0; i < 8; ++i)
    if (k0 + i < K) w[i >> 1] |= (uint32_t)__ldg(row + k0 + i) << (16 * (i & 1));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Exact sum of 8 fp16 magnitudes in units of 2^-24. Every finite fp16 value
// is a multiple of 2^-24 below 2^16, so a sum of 8 needs at most 19 + 24 = 43
// significant bits: its fp64 sum is exact in any order, and so is its product
// with 2^24 and the conversion to an integer (the same value as the sum of
// mag_units of the 8 patterns).
__device__ __forceinline__ uint64_t units_of(double d) { return (uint64_t)(d * 16777216.0); }

// Both halves of a word as fp64 (exact): one conversion per element.
__device__ __forceinline__ void f16x2_to_f64(uint32_t w, double &lo, double &hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f64.f16 %0, l;\n\tcvt.f64.f16 %1, h;\n\t}"
      : "=d"(lo), "=d"(hi)
      : "r"(w));
}
// Sum of the 8 halves of four words of magnitude patterns (sign bits clear),
// in a balanced tree. A non-finite pattern makes the sum non-finite.
__device__ __forceinline__ double f64_sum8(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  double a0, a1, b0, b1, c0, c1, d0, d1;
  f16x2_to_f64(a, a0, a1);
  f16x2_to_f64(b, b0, b1);
  f16x2_to_f64(c, c0, c1);
  f16x2_to_f64(d, d0, d1);
  return ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
}
__device__ __forceinline__ bool finite_f64(double d) { return fabs(d) < __longlong_as_double(0x7FF0000000000000ll); }

constexpr uint32_t MAG2 = 0x7FFF7FFFu;  // the magnitude bits of two halves

// The same sum one element at a time, leaving out (and reporting) the
// non-finite ones; taken only when the fast sum is not finite.
__device__ __forceinline__ uint64_t sum_mag8_nonfinite(uint4 v, bool &bad) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t f[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t r = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t hm = (w[j] >> (16 * h)) & 0x7FFFu;
      bad |= hm >= 0x7C00u;
      r |= (hm < 0x7C00u ? hm : 0u) << (16 * h);
    }
    f[j] = r;
  }
  return units_of(f64_sum8(f[0], f[1], f[2], f[3]));
}

__device__ __forceinline__ uint64_t sum_mag8(const uint4 &v, bool &bad) {
  const double d = f64_sum8(v.x & MAG2, v.y & MAG2, v.z & MAG2, v.w & MAG2);
  if (finite_f64(d)) return units_of(d);
  return sum_mag8_nonfinite(v, bad);
}

// Bit i of the result = bit 15 + 16*(i&1) of word i>>1, for 8 halves held in
// four words whose other bits are clear.
__device__ __forceinline__ uint32_t gather_bit15(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  const uint32_t t = (a >> 15) | (b >> 13) | (c >> 11) | (d >> 9);  // bits 2j and 2j + 16
  return (t | (t >> 15)) & 0xFFu;
}

// keep / sign bit patterns of 8 halves, plus the sum of the kept magnitudes.
// Ternary: keep iff the magnitude pattern exceeds hT, two halves per integer
// subtract: per half, (0x8000 | hT) - hm has bit 15 clear exactly when
// hm > hT, and never borrows from the half above. A kept half has hm >= 1,
// so its sign bit alone decides "negative". Non-finite kept halves are kept
// but left out of the sum (as in the element-wise form, taken for them).
template <bool TERNARY>
__device__ __forceinline__ void keep8(const uint4 &v, uint32_t hT, int64_t k0, int64_t K,
                                      uint32_t &kb, uint32_t &sb, uint64_t &ks) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if (TERNARY) {
    const uint32_t tc = (hT | 0x8000u) * 0x00010001u;
    uint32_t kw[4], nw[4], kv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t hm2 = w[j] & MAG2;
      kw[j] = ~(tc - hm2) & 0x80008000u;
      nw[j] = w[j] & kw[j];
      kv[j] = hm2 & ((kw[j] >> 15) * 0x7FFFu);
    }
    kb = gather_bit15(kw[0], kw[1], kw[2], kw[3]);
    sb = gather_bit15(nw[0], nw[1], nw[2], nw[3]);
    const double kd = f64_sum8(kv[0], kv[1], kv[2], kv[3]);
    if (finite_f64(kd)) {
      ks += units_of(kd);
    } else {
      bool unused = false;
      ks += sum_mag8_nonfinite(make_uint4(kv[0], kv[1], kv[2], kv[3]), unused);
    }
  } else {
    kb = 0;
    sb = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t h = (w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
      const uint32_t keep = (k0 + i) < K;
      kb |= keep << i;
      sb |= (keep & (h >> 15) & ((h & 0x7FFFu) != 0u)) << i;
    }
  }
}

// E4M3 word k (k = 0..7) of a 32-element block in the tensor-core order: its
// byte j (j = 0..3) is element 8j + k of the block, +1 = 0x38, -1 = 0xB8,
// 0 = 0x00. mw / sw are the block's keep / sign words (bit i = element i).
// Gathering elements k, k+8, k+16, k+24 into one word is a shift and a mask,
// which is what lets the GEMM expand weight bits into the same order cheaply.
__device__ __forceinline__ uint32_t e4m3_tc_word(uint32_t mw, uint32_t sw, int k) {
  return ((mw >> k) & 0x01010101u) * 0x38u | (((sw >> k) << 7) & 0x80808080u);
}

// Merge the 8-bit patterns of a 16-lane chunk group into 4 words; lane 0 of
// the group stores them (one 128-bit store per plane). With e4m3_dst set, every
// lane also writes its 8 bytes of the block's E4M3 words in the tensor-core
// order (lane j of a 4-lane quad: words 2j and 2j+1, which start at the same
// byte offset as its 8 elements).
__device__ __forceinline__ void store_chunk(uint32_t kb, uint32_t sb, uint32_t *mrow,
                                            uint32_t *srow, int chunk, bool do_store,
                                            uint8_t *e4m3_dst = nullptr, int *popc_dst = nullptr) {
  const int l16 = threadIdx.x & 15;
  uint32_t mw = kb << (8 * (l16 & 3)), sw = sb << (8 * (l16 & 3));
  mw |= __shfl_xor_sync(FULL, mw, 1);
  sw |= __shfl_xor_sync(FULL, sw, 1);
  mw |= __shfl_xor_sync(FULL, mw, 2);
  sw |= __shfl_xor_sync(FULL, sw, 2);
  if (e4m3_dst) {
    const int j = l16 & 3;
    *reinterpret_cast<uint2 *>(e4m3_dst) =
        make_uint2(e4m3_tc_word(mw, sw, 2 * j), e4m3_tc_word(mw, sw, 2 * j + 1));
  }
  const uint32_t m1 = __shfl_down_sync(FULL, mw, 4), m2 = __shfl_down_sync(FULL, mw, 8),
                 m3 = __shfl_down_sync(FULL, mw, 12);
  const uint32_t s1 = __shfl_down_sync(FULL, sw, 4), s2 = __shfl_down_sync(FULL, sw, 8),
                 s3 = __shfl_down_sync(FULL, sw, 12);
  if (do_store && l16 == 0) {
    *reinterpret_cast<uint4 *>(mrow + 4 * chunk) = make_uint4(mw, m1, m2, m3);
    *reinterpret_cast<uint4 *>(srow + 4 * chunk) = make_uint4(sw, s1, s2, s3);
    if (popc_dst) popc_dst[chunk] = __popc(mw) + __popc(m1) + __popc(m2) + __popc(m3);
  }
}

// Row scale from the exact kept sum / count (ternary) or the row sum (binary),
// with the roundings of the definition: int64 -> fp64, fp64 divide, times
// 2^-24, fp64 -> fp32.
__device__ __forceinline__ float row_scale(uint64_t num, uint64_t den) {
  if (!den) return 0.0f;
  return __double2float_rn(__dmul_rn(__ddiv_rn(__ull2double_rn(num), __ull2double_rn(den)), 0x1p-24));
}

}  // namespace bwta
