// tma_host.h -- host-side TMA tensor-map creation.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace s3r {

// Tensor map over a [rows, H, 64] bf16 tensor for boxes of one head's [box_rows, 64] tile,
// 128-byte swizzled, zero fill out of bounds. False if the driver entry point is unavailable or
// the arguments are rejected (base must be 16-byte aligned).
bool make_tmap_head_rows(CUtensorMap* map, const void* base, int64_t rows, int H, int box_rows);

// Tensor map over a [rows, 64] bf16 tensor (rows of 128 contiguous bytes, e.g. a head-major
// [H, Lp, 64] copy viewed as H*Lp rows) for [box_rows, 64] boxes, 128-byte swizzled.
bool make_tmap_rows64(CUtensorMap* map, const void* base, int64_t rows, int box_rows);

}  // namespace s3r
