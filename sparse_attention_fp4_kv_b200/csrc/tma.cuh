// Host-side creation of TMA tensor maps and the device-side copy helpers
// shared by the kernels that stage tiles with the Tensor Memory Accelerator.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace csa2 {

// 2D row-major tensor [rows][inner] of `dtype`, rows `row_bytes` apart, copied
// in boxes of [box_rows][box_inner] with 128-byte swizzle. Uses
// cuTensorMapEncodeTiled through the runtime's driver entry point. Returns
// false if the driver call is unavailable or rejects the arguments.
bool make_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *ptr, uint64_t inner,
                  uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows);

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

}  // namespace csa2
