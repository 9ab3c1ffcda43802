// microbench.cu -- ceilings for the roofline of each kernel, measured on the
// GPU the library runs on:
//  * the LOP3+POPC+IADD "word-op" rate: the inner loop of the bit GEMM
//    (one 32-element word of one output per op), and its parts (LOP3, IADD3,
//    IMAD) on their own;
//  * legacy warp-level MMA rates: b1 AND+POPC (m16n8k256), s8 (m16n8k32) and
//    f16 (m16n8k16), for comparison with the CUDA-core path;
//  * HBM streaming read and write bandwidth.
//  * the bit GEMM's inner mix per 4-word chunk (4 LOP3 m & (a ^ w), a
//    carry-save adder of 2 LOP3s, 3 POPCs, adds): the ceiling of that kernel;
// Each kernel keeps independent dependency chains per thread so that issue
// throughput, not latency, bounds it; results feed a sink so nothing is
// optimized away. The caller times the launches with CUDA events.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int CH = 16;  // independent chains per thread

__device__ __forceinline__ uint32_t lop3_and_xor(uint32_t m, uint32_t a, uint32_t b) {
  uint32_t r;
  asm volatile("lop3.b32 %0, %1, %2, %3, 0x60;" : "=r"(r) : "r"(m), "r"(a), "r"(b));
  return r;
}

// one "word-op" = acc += popc(m & (a ^ acc)): LOP3 + POPC + IADD
__global__ void mb_wordop(uint32_t *sink, int iters, uint32_t seed) {
  uint32_t m[CH], acc[CH];
  const uint32_t a = seed * 0x9E3779B9u + threadIdx.x;
#pragma unroll
  for (int i = 0; i < CH; ++i) {
    m[i] = seed ^ (0x85EBCA6Bu * (i + 1) + threadIdx.x);
    acc[i] = i;
  }
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < CH; ++i) acc[i] += __popc(lop3_and_xor(m[i], a, acc[i]));
  }
  uint32_t r = 0;
#pragma unroll
  for (int i = 0; i < CH; ++i) r ^= acc[i];
  if (r == 0x12345678u) sink[0] = r;
}

// The bit GEMM's own inner mix for one output and one 4-word chunk: four
// m & (a ^ w) LOP3s, a carry-save full adder over three of them (two LOP3s),
// three POPCs and the adds that weight them, acc += popc(s) + popc(t3) +
// 2 * popc(c). The accumulator stands in for the weight words so that every
// iteration depends on the last; 4 word-ops per chain and iteration.
__global__ void mb_popc4(uint32_t *sink, int iters, uint32_t seed) {
  constexpr int C4 = 8;
  uint32_t m[4], a[4], acc[C4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = seed ^ (0x85EBCA6Bu * (i + 1) + threadIdx.x);
    a[i] = seed * 0x9E3779B9u + 0x27D4EB2Fu * i + threadIdx.x;
  }
#pragma unroll
  for (int c = 0; c < C4; ++c) acc[c] = c * 0x61C88647u;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int c = 0; c < C4; ++c) {
      const uint32_t t0 = lop3_and_xor(m[0], a[0], acc[c]), t1 = lop3_and_xor(m[1], a[1], acc[c]);
      const uint32_t t2 = lop3_and_xor(m[2], a[2], acc[c]), t3 = lop3_and_xor(m[3], a[3], acc[c]);
      uint32_t s, cy;
      asm volatile("lop3.b32 %0, %1, %2, %3, 0x96;" : "=r"(s) : "r"(t0), "r"(t1), "r"(t2));
      asm volatile("lop3.b32 %0, %1, %2, %3, 0xE8;" : "=r"(cy) : "r"(t0), "r"(t1), "r"(t2));
      acc[c] += __popc(s) + __popc(t3) + 2 * __popc(cy);
    }
  }
  uint32_t r = 0;
#pragma unroll
  for (int c = 0; c < C4; ++c) r ^= acc[c];
  if (r == 0x12345678u) sink[0] = r;
}

// LOP3 alone: x = lop3(x, y, z)
__global__ void mb_lop3(uint32_t *sink, int iters, uint32_t seed) {
  uint32_t x[CH];
  const uint32_t y = seed * 3u + threadIdx.x, z = seed ^ 0xA5A5A5A5u;
#pragma unroll
  for (int i = 0; i < CH; ++i) x[i] = seed + i * 7919u + threadIdx.x;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < CH; ++i) x[i] = lop3_and_xor(x[i], y, z) ^ x[i];
  }
  uint32_t r = 0;
#pragma unroll
  for (int i = 0; i < CH; ++i) r ^= x[i];
  if (r == 0x12345678u) sink[0] = r;
}

// POPC with the smallest companion: acc += popc(acc) -> POPC + IADD
__global__ void mb_popc(uint32_t *sink, int iters, uint32_t seed) {
  uint32_t acc[CH];
#pragma unroll
  for (int i = 0; i < CH; ++i) acc[i] = seed * (i + 3) + threadIdx.x;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < CH; ++i) acc[i] += __popc(acc[i]);
  }
  uint32_t r = 0;
#pragma unroll
  for (int i = 0; i < CH; ++i) r ^= acc[i];
  if (r == 0x12345678u) sink[0] = r;
}

// IMAD alone: x = x * k + y
__global__ void mb_imad(uint32_t *sink, int iters, uint32_t seed) {
  uint32_t x[CH];
  const uint32_t k = seed | 1u, y = threadIdx.x;
#pragma unroll
  for (int i = 0; i < CH; ++i) x[i] = seed + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      uint32_t r;
      asm volatile("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(x[i]), "r"(k), "r"(y));
      x[i] = r;
    }
  }
  uint32_t r = 0;
#pragma unroll
  for (int i = 0; i < CH; ++i) r ^= x[i];
  if (r == 0x12345678u) sink[0] = r;
}

// b1 MMA with AND+POPC: 16 x 8 x 256 bit products per instruction
__global__ void mb_mma_b1(uint32_t *sink, int iters, uint32_t seed) {
  constexpr int ACC = 4;
  uint32_t a[4], b[2];
  int d[ACC][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = seed * (i + 1) + threadIdx.x;
  b[0] = seed ^ threadIdx.x;
  b[1] = ~seed;
#pragma unroll
  for (int q = 0; q < ACC; ++q)
#pragma unroll
    for (int i = 0; i < 4; ++i) d[q][i] = q + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int q = 0; q < ACC; ++q) {
      asm volatile(
          "mma.sync.aligned.m16n8k256.row.col.s32.b1.b1.s32.and.popc "
          "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
          : "+r"(d[q][0]), "+r"(d[q][1]), "+r"(d[q][2]), "+r"(d[q][3])
          : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
    }
  }
  int r = 0;
#pragma unroll
  for (int q = 0; q < ACC; ++q)
#pragma unroll
    for (int i = 0; i < 4; ++i) r ^= d[q][i];
  if (r == 0x12345678) sink[0] = r;
}

// s8 MMA: 16 x 8 x 32 per instruction
__global__ void mb_mma_s8(uint32_t *sink, int iters, uint32_t seed) {
  constexpr int ACC = 4;
  uint32_t a[4], b[2];
  int d[ACC][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = seed * (i + 1) + threadIdx.x;
  b[0] = seed ^ threadIdx.x;
  b[1] = ~seed;
#pragma unroll
  for (int q = 0; q < ACC; ++q)
#pragma unroll
    for (int i = 0; i < 4; ++i) d[q][i] = q + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int q = 0; q < ACC; ++q) {
      asm volatile(
          "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
          "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
          : "+r"(d[q][0]), "+r"(d[q][1]), "+r"(d[q][2]), "+r"(d[q][3])
          : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
    }
  }
  int r = 0;
#pragma unroll
  for (int q = 0; q < ACC; ++q)
#pragma unroll
    for (int i = 0; i < 4; ++i) r ^= d[q][i];
  if (r == 0x12345678) sink[0] = r;
}

// f16 MMA with fp32 accumulation: 16 x 8 x 16 per instruction
__global__ void mb_mma_f16(uint32_t *sink, int iters, uint32_t seed) {
  constexpr int ACC = 4;
  uint32_t a[4], b[2];
  float d[ACC][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = 0x3C003C00u;  // (1.0, 1.0)
  b[0] = b[1] = 0x00010001u * (seed & 1u);
#pragma unroll
  for (int q = 0; q < ACC; ++q)
#pragma unroll
    for (int i = 0; i < 4; ++i) d[q][i] = 0.0f;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int q = 0; q < ACC; ++q) {
      asm volatile(
          "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
          "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
          : "+f"(d[q][0]), "+f"(d[q][1]), "+f"(d[q][2]), "+f"(d[q][3])
          : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
    }
  }
  float r = 0.0f;
#pragma unroll
  for (int q = 0; q < ACC; ++q)
#pragma unroll
    for (int i = 0; i < 4; ++i) r += d[q][i];
  if (r == 1234.5f) sink[0] = 1;
}

__global__ void mb_read(const uint4 *__restrict__ p, size_t n, uint32_t *sink) {
  uint32_t x = 0;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p + i));
    x ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  if (x == 0x12345678u) sink[0] = x;
}

__global__ void mb_write(uint4 *__restrict__ p, size_t n, uint32_t v) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    __stcs(p + i, make_uint4(v, v, v, v));
}

}  // namespace

extern "C" {

// Ops counted per thread per iteration (the caller multiplies by threads*iters):
//   wordop/lop3/popc/imad: 16; popc4: 32 word-ops; mma_*: 4 instructions per thread-iteration,
//   i.e. 4/32 per thread of the warp-wide instruction.
int bwta_mb_launch(int kind, int blocks, int threads, int iters, uint32_t *sink, void *stream) {
  cudaStream_t s = (cudaStream_t)stream;
  switch (kind) {
    case 0: mb_wordop<<<blocks, threads, 0, s>>>(sink, iters, 1u); break;
    case 1: mb_lop3<<<blocks, threads, 0, s>>>(sink, iters, 1u); break;
    case 2: mb_popc<<<blocks, threads, 0, s>>>(sink, iters, 1u); break;
    case 3: mb_imad<<<blocks, threads, 0, s>>>(sink, iters, 1u); break;
    case 4: mb_mma_b1<<<blocks, threads, 0, s>>>(sink, iters, 1u); break;
    case 5: mb_mma_s8<<<blocks, threads, 0, s>>>(sink, iters, 1u); break;
    case 6: mb_mma_f16<<<blocks, threads, 0, s>>>(sink, iters, 1u); break;
    case 7: mb_popc4<<<blocks, threads, 0, s>>>(sink, iters, 1u); break;
    default: return -1;
  }
  return (int)cudaGetLastError();
}

int bwta_mb_read(const void *p, size_t bytes, int blocks, uint32_t *sink, void *stream) {
  mb_read<<<blocks, 512, 0, (cudaStream_t)stream>>>((const uint4 *)p, bytes / 16, sink);
  return (int)cudaGetLastError();
}

int bwta_mb_write(void *p, size_t bytes, int blocks, void *stream) {
  mb_write<<<blocks, 512, 0, (cudaStream_t)stream>>>((uint4 *)p, bytes / 16, 0x01020304u);
  return (int)cudaGetLastError();
}

}  // extern "C"
