// tma.h -- tensor-memory-accelerator (TMA) helpers: host-side tensor-map encoding (through the
// driver entry point, no link against libcuda) and the device-side tiled load into shared memory.
//
// Every tiled load used here starts at an innermost element offset that is a multiple of 64 bf16
// (128 bytes), so the 16-byte rule for the innermost coordinate always holds, and each load fills
// only the issuing CTA's own shared memory.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace csa {

// 2-D tiled load of one box at (x = inner element offset, y = row) into this CTA's shared memory at
// `dst`, completing its bytes of transaction count on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// A 2-D bf16 tensor map over `rows` rows of `inner` elements (row pitch `pitch_bytes`), box of
// box_inner x box_rows elements, with the 128-byte swizzle (swizzle128) or none; cached per
// (base, inner, rows, pitch, box, swizzle).  Returns cudaSuccess, or an error when the driver entry
// point is missing or the encoding is rejected.
cudaError_t tensor_map_2d_bf16(CUtensorMap* out, const void* base, uint64_t inner, uint64_t rows,
                               uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows, bool swizzle128 = true);

}  // namespace csa
