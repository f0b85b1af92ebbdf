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

// ---- cache-policy hints for 16-byte accesses --------------------------------

// An L2 policy that keeps the lines it touches in preference to others: used
// for small tables that every row gathers from many times.
ELSAA_DEV uint64_t l2_keep_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
ELSAA_DEV uint4 ld16_keep(const void* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}
// Streaming (read once) load and store: evict-first in both caches.
ELSAA_DEV uint4 ld16_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
ELSAA_DEV void st16_stream(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

ELSAA_DEV void raise_error(uint32_t* err, uint32_t bit) {
  if (err) atomicOr(err, bit);
}

}  // namespace elsaa
