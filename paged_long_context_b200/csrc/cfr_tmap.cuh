// cfr_tmap.cuh -- 2-D TMA tensor maps over a page pool (host side) and the
// tiled TMA load (device side, no multicast).
//
// A pool of format f is viewed as a 2-D tensor of rows = slots * Hkv * P rows
// of head_dim elements; the (slot, kv head) sub-page of page slot `id` starts at
// row (id * Hkv + g) * P.  Boxes are 128 bytes wide (the 128-byte swizzle
// span) and `box_rows` rows high; the shared-memory image of a box is the
// 128-byte-swizzled layout (16-byte chunk c of row r stored at chunk c ^ (r % 8)
// within each 1024-byte group of 8 rows).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "cfr_common.cuh"

namespace cfr {

// Encodes a row-major [rows][cols] tensor of `elem_bytes` elements (cols *
// elem_bytes a multiple of 16) with 128-byte-wide, box_rows-high boxes and the
// 128-byte swizzle.  Returns false when the driver entry point is missing or
// the encode fails.
bool encode_pool_map(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                     long long rows, int cols, int box_rows);

// ---- device side ----------------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_map(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// byte offset of 16-byte chunk c (0..7) of row r inside a 128-byte-swizzled box image
__device__ __forceinline__ int sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

}  // namespace cfr
