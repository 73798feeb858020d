// tma.h -- host creation of TMA tensor maps (cuTensorMapEncodeTiled through the
// runtime's driver entry point, so libdcp needs no link against libcuda) and
// the device-side tiled TMA load.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dcp {

// 2-D tensor map over a row-major matrix [outer][inner] of `elem_bytes`
// elements with rows `row_bytes` apart; box = [box_outer][box_inner].
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

// 4-D tensor map: dims[0] is contiguous (elements), dims[1..3] are `strides_bytes`
// apart (any order of strides, as long as the view does not overlap itself);
// box = box[0] x box[1] x box[2] x box[3], laid out in shared memory with
// dimension 0 fastest.
bool make_tmap_4d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, const uint64_t dims[4],
                  const uint64_t strides_bytes[3], const uint32_t box[4], CUtensorMapSwizzle swizzle);

#if defined(__CUDACC__)
// 2-D tiled load into this CTA's shared memory, completion on `bar`.
// x (innermost coordinate) times the element size must be a multiple of 16 B.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
        "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar))), "l"(policy)
        : "memory");
}

// 4-D tiled load; x (innermost coordinate) times the element size must be a
// multiple of 16 B.
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, int32_t x, int32_t y, int32_t z,
                                            int32_t w, uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w),
        "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar))), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
#endif

}  // namespace dcp
