// Device helpers shared by the libelsaa kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#define ELSAA_DEV __device__ __forceinline__

namespace elsaa {

// Error word bits written by kernels into the workspace (see elsaa_check).
enum : uint32_t { ERR_TIMEOUT = 1u, ERR_CHECK = 2u };

ELSAA_DEV float to_f32(float x) { return x; }
ELSAA_DEV float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> ELSAA_DEV T from_f32(float x);
template <> ELSAA_DEV float from_f32<float>(float x) { return x; }
template <> ELSAA_DEV __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Round a float through the storage type (what a later read would see).
template <typename T> ELSAA_DEV float round_through(float x) { return to_f32(from_f32<T>(x)); }

ELSAA_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
ELSAA_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
ELSAA_DEV double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

ELSAA_DEV float sigmoidf_(float x) { return 1.0f / (1.0f + __expf(-x)); }

ELSAA_DEV void raise_error(uint32_t* err, uint32_t bit) {
  if (err) atomicOr(err, bit);
}

}  // namespace elsaa
