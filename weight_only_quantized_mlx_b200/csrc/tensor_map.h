// TMA tensor maps (CUtensorMap) for the kernels: the CUDA driver's encoder is
// reached through the CUDA runtime (no libcuda link), and the maps of a
// weight's three buffers are cached per (buffers, shape, box) so repeated
// calls on the same weight do not re-encode them.
#pragma once

#include <cuda.h>

#include "kernels.h"

namespace mlxq {

struct TensorMaps3 {
    CUtensorMap packed;  // uint8 view [N, K] of the packed words
    CUtensorMap scales;  // bf16 [N, G]
    CUtensorMap biases;  // bf16 [N, G]
};

bool tensor_maps_available();

// 2-D tiled map: `inner` x `outer` elements, rows `row_bytes` apart, box
// `box_inner` x `box_outer`, zero fill out of bounds.
bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);

// 3-D tiled map over a row-major [outer, inner] array viewed as
// {chunk, outer, inner / chunk} (strides row_bytes and chunk * elem bytes),
// so that one box {chunk, box_outer, box_chunks} brings box_chunks
// consecutive chunks of box_outer rows, chunk-major in shared memory
// ([box_chunks][box_outer][chunk]); 128-byte swizzle, zero fill out of bounds.
bool encode_3d_chunks(CUtensorMap* map, CUtensorMapDataType dt, uint32_t elem_bytes, const void* base, uint64_t inner,
                      uint64_t outer, uint64_t row_bytes, uint32_t chunk, uint32_t box_outer, uint32_t box_chunks);

// Maps of a weight: packed box {box_k_bytes, box_rows} with swizzle
// `packed_sw`; scale/bias boxes {box_groups, box_rows} (box_groups == 0: no
// scale/bias maps).  Returns false if encoding failed.
bool weight_tensor_maps(const WeightView& w, int box_rows, int box_k_bytes, CUtensorMapSwizzle packed_sw,
                        int box_groups, TensorMaps3* out);

}  // namespace mlxq
