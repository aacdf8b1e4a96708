// tma.cuh -- tensor-memory-accelerator (TMA) tile loads for sm_100a.
//
// A tensor map (CUtensorMap, 128 bytes) describes a tensor in global memory: its element type,
// up to five dimensions with byte strides, the box one copy moves and the shared-memory swizzle.
// It is encoded once on the host (tma_encode, tma_host.cu) and passed to kernels as a
// __grid_constant__ parameter.  One thread issues cp.async.bulk.tensor; the copy signals its
// bytes on an mbarrier that the consumers wait on (phase parity), after the issuing thread has
// announced the byte count with expect_tx.
//
// Every load here reads this GPU's own memory and none uses cluster multicast.  The innermost
// box coordinate is always 0 or a multiple of 64 fp16 elements (a multiple of 16 bytes).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace rtp {

__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}

// Make mbarrier initialisation visible to the async proxy (the TMA unit) before first use.
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      :
      : "r"(dst), "l"(map), "r"(x), "r"(y), "r"(mbar)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                            uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];"
      :
      : "r"(dst), "l"(map), "r"(x), "r"(y), "r"(z), "r"(mbar)
      : "memory");
}

// Host: encode a tiled tensor map (no interleave, zero fill out of bounds).  dims/strides as
// cuTensorMapEncodeTiled takes them: dims[0] innermost, strides[i] (bytes) for dims[i + 1].
// Returns false (and leaves *map unspecified) if the driver refuses the description.
bool tma_encode(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* base, const uint64_t* dims,
                const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle swizzle);

}  // namespace rtp
