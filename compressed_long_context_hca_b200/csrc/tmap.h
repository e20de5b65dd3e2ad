// tmap.h -- TMA tensor-map encoding through the driver entry point (no -lcuda needed).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hca {

// 2-D bf16 map over a row-major [rows, cols] array, 128-byte swizzle, box
// [box_rows, box_cols] (box_cols * 2 bytes must be 128). Loads that fall outside the
// array are zero-filled by the hardware.
cudaError_t encode_bf16_rows(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                             uint32_t box_cols, uint32_t box_rows);

// 3-D bf16 map over a row-major [rows, 512] array seen as {64 elements, rows, 8 chunks}
// (row stride 1024 B, chunk stride 128 B), 128-byte swizzle. One box = box_rows rows x
// box_chunks consecutive 64-element chunks, landing in shared memory chunk-major:
// [box_chunks][box_rows][64], each chunk a stack of 128-byte swizzled rows.
cudaError_t encode_bf16_chunks(CUtensorMap* map, const void* base, uint64_t rows,
                               uint32_t box_rows, uint32_t box_chunks);

// 2-D bf16 map over a row-major [rows, cols] array with a row stride of ld elements
// (ld * 2 a multiple of 16), 128-byte swizzle, box [box_rows, box_cols] (box_cols * 2 must
// be 128). Loads that fall outside the array are zero-filled.
cudaError_t encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint64_t ld, uint32_t box_cols, uint32_t box_rows);

// 3-D map over a row-major [rows, 512] array of bytes (e4m3 codes) seen as
// {128 bytes, rows, 4 chunks} (row stride 512 B, chunk stride 128 B), 128-byte swizzle.
// One box = box_rows rows x box_chunks consecutive 128-byte chunks, chunk-major in shared
// memory like encode_bf16_chunks.
cudaError_t encode_u8_chunks(CUtensorMap* map, const void* base, uint64_t rows,
                             uint32_t box_rows, uint32_t box_chunks);

}  // namespace hca
