// Tiles of Q and K rows for the tcgen05 hash kernels (hash_tc.cu and
// hash_tc_stream.cu): 128 rows of bf16 values, read by cp.async into the
// 128-byte-swizzled K-major layout the MMA descriptors expect.
#pragma once
#include "tc_common.cuh"

namespace elsaa {
namespace hash {

constexpr int kTile = 128;
constexpr int kPass = 128;            // TMEM columns per pass
constexpr int kSmemLimit = 227 * 1024;

// Rows tile * 128 .. + 127 of [Q rows; K rows] (rows_per_tensor each) into
// dst; rows past the end read as zeros.  NT threads share the copies.
template <int D, int NT>
ELSAA_DEV void load_tile(uint32_t dst, const __nv_bfloat16* q, const __nv_bfloat16* k,
                         int64_t rows_per_tensor, int64_t tile) {
  constexpr int kChunks = D / 8;
  const int64_t total = 2 * rows_per_tensor;
  for (int i = threadIdx.x; i < kTile * kChunks; i += NT) {
    const int row = i / kChunks, ch = i % kChunks;
    const int64_t grow = tile * kTile + row;
    const bool valid = grow < total;
    const int64_t g = valid ? grow : 0;
    const __nv_bfloat16* src =
        (g < rows_per_tensor ? q + g * D : k + (g - rows_per_tensor) * D) + ch * 8;
    tc::cp_async16(dst + (ch >> 3) * (kTile * 128) + tc::sw128_off(row, ch & 7), src,
                   valid ? 16 : 0);
  }
}

}  // namespace hash
}  // namespace elsaa
