// tensor_maps.h — TMA tensor maps over a paged cache (host side).
#pragma once
#include <cuda.h>

#include "internal.h"

namespace pkv {

// 5-D view of one 16-bit cache [num_blocks, block_size, num_kv_heads,
// head_dim] with block_stride elements between blocks: (64 dims, KV head,
// slot in block, 64-dim half, block).  One box of 64 x 1 x 16 x
// (head_dim / 64) x 1 lands in shared memory as head_dim / 64 sub-tiles of
// 16 rows x 128 bytes, 128-byte swizzled: 16 slots of one block, all dims.
// With box_halves = 1 a box is one 64-dim half (coordinate 3 picks it).
int encode_paged_map_16bit(CUtensorMap* map, const void* cache, pkv_dtype dtype, int head_dim,
                           int num_kv_heads, int block_size, int num_blocks,
                           int64_t block_stride, int box_halves = 0);

}  // namespace pkv
