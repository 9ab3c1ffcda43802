// tma.cuh -- TMA tensor maps (host) and mbarrier / bulk-tensor primitives
// (device) written as inline PTX for sm_100a. No cluster multicast is used
// anywhere: every TMA load brings a tile of this GPU's own memory into the
// issuing CTA's shared memory.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bwta {

// ------------------------------------------------------------------ host
// cuTensorMapEncodeTiled, fetched through the runtime so that the library does
// not link libcuda directly.
typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                    const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                    const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

PFN_encodeTiled get_encode_tiled();

// A 2-D map over a row-major uint32 matrix [rows][ld], box = box_w words x
// box_h rows, 128-byte swizzle (box_w * 4 must be 128). Out-of-range rows and
// columns read as zero. Returns false if the driver rejects the map.
bool make_plane_map(CUtensorMap *map, const uint32_t *base, int64_t rows, int64_t ld,
                    uint32_t box_w, uint32_t box_h);

// A 2-D map over a row-major matrix [rows][ld] of `elem_bytes`-byte elements
// (dtype UINT8 or UINT32), box = box_w x box_h elements, the given swizzle.
bool make_map_2d(CUtensorMap *map, CUtensorMapDataType dtype, int elem_bytes, const void *base,
                 int64_t rows, int64_t ld, uint32_t box_w, uint32_t box_h,
                 CUtensorMapSwizzle swizzle);

// ---------------------------------------------------------------- device
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of the barrier to complete. Each try_wait carries a
// suspend-time hint, so a waiting thread sleeps until the phase completes (or
// about a millisecond passes) instead of polling shared memory, where its
// polls would compete with the tensor cores and TMA for bandwidth. Bounded:
// gives up after about `limit_ns` nanoseconds of waiting and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint64_t limit_ns = 2000000000ull) {
  const uint32_t a = smem_addr(bar);
  uint32_t done = 0;
  uint64_t t0 = 0;
  for (;;) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(a), "r"(parity), "r"(1000000u)
        : "memory");
    if (done) return true;
    const uint64_t t = global_ns();
    if (t0 == 0) t0 = t;
    else if (t - t0 > limit_ns) return false;
  }
}

// Non-blocking test: has phase `parity` of the barrier completed?
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// 2-D tiled bulk tensor load global -> shared, completion signalled on `bar`.
// x (innermost coordinate, in elements) must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int32_t x,
                                            int32_t y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 16-byte chunk c (0..7) of row r in a [rows][128 B] tile written by TMA with
// 128-byte swizzle (tile base 1024-byte aligned).
__device__ __forceinline__ uint32_t swz128(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

}  // namespace bwta
