// Backward of the denominator-aware fusion and the token-wise gates.
//
// Forward ("Two Efficient Attentions, One Denominator Problem", section "Two
// efficient branches can still be mis-scaled", and the ELSAA overview's learned
// or fixed gates with an optional learnable lambda):
//   g_s = sigmoid(w_s . q + b_s), g_r = sigmoid(w_r . q + b_r)
//   m = Z_sp / (Z_sp + lambda Z_race) = sigmoid(lse - log(lambda Z_race))
//   y = g_s m O_sp + g_r O_race
// Given dy, per query:
//   dm = g_s (dy . O_sp)            dlse = dm m (1 - m)
//   dlambda += -dm m^2 Z_race / Z_sp   (m = 1 and this still holds at lambda = 0)
//   da_s = m (dy . O_sp) g_s (1 - g_s),  da_r = (dy . O_race) g_r (1 - g_r)
//   dq_gate = da_s w_s + da_r w_r,  dw += da q,  db += da
//   dO_sp = g_s m dy,  D' = dO_sp . O_sp - dlse  (the sparse backward's row term)
//   dO_race / Ctot = g_r dy / Ctot  (scattered into the RACE table gradient)
// One warp per query; per-block partial sums of (dw_s, dw_r, db_s, db_r,
// dlambda) go to a fixed number of slots and are reduced in a fixed order, so
// the parameter gradients are deterministic.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace elsaa {
namespace {

template <typename T, int VEC>
__global__ void __launch_bounds__(256)
fuse_bwd_kernel(const T* __restrict__ q, const T* __restrict__ dy, const T* __restrict__ o_sp,
                const T* __restrict__ o_race, const float* __restrict__ lse,
                const int32_t* __restrict__ ctot, const float* __restrict__ gate_w,
                const float* __restrict__ gate_b, int gate_fixed, float gs_fixed, float gr_fixed,
                const float* __restrict__ lam, int64_t rows, int L, int d, T* __restrict__ d_o,
                float* __restrict__ dprime, float* __restrict__ dq_acc, float* __restrict__ dor,
                float* __restrict__ partials) {
  __shared__ float red[8][2 * 128 + 3];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const float lam_v = *lam;
  float pws[VEC], pwr[VEC], pbs = 0.f, pbr = 0.f, plam = 0.f;
#pragma unroll
  for (int i = 0; i < VEC; ++i) pws[i] = pwr[i] = 0.f;
  float ws_[VEC], wr_[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) ws_[i] = wr_[i] = 0.f;
  float bs = 0.f, br = 0.f;
  if (!gate_fixed) {
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      ws_[i] = gate_w[lane * VEC + i];
      wr_[i] = gate_w[d + lane * VEC + i];
    }
    bs = gate_b[0];
    br = gate_b[1];
  }
  for (int64_t r = (int64_t)blockIdx.x * nw + w; r < rows; r += (int64_t)gridDim.x * nw) {
    const size_t base = (size_t)r * d + lane * VEC;
    float qv[VEC], g[VEC], os[VEC], orc[VEC];
    float dyo = 0.f, dyr = 0.f, as = 0.f, ar = 0.f;
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      qv[i] = to_f32(q[base + i]);
      g[i] = to_f32(dy[base + i]);
      os[i] = to_f32(o_sp[base + i]);
      orc[i] = to_f32(o_race[base + i]);
      dyo += g[i] * os[i];
      dyr += g[i] * orc[i];
      if (!gate_fixed) {
        as += qv[i] * ws_[i];
        ar += qv[i] * wr_[i];
      }
    }
    dyo = warp_sum(dyo);
    dyr = warp_sum(dyr);
    float gs = gs_fixed, gr = gr_fixed;
    if (!gate_fixed) {
      gs = 1.0f / (1.0f + expf(-(warp_sum(as) + bs)));
      gr = 1.0f / (1.0f + expf(-(warp_sum(ar) + br)));
    }
    const int c = ctot[r];
    const float zr = (float)c / (float)L;
    const float l = lse[r];
    const float lz = lam_v * zr;
    const float m = lz > 0.f ? 1.0f / (1.0f + expf(logf(lz) - l)) : 1.0f;
    const float dm = gs * dyo;
    const float dlse = dm * m * (1.0f - m);
    const float dlam = zr > 0.f ? -dm * m * m * expf(logf(zr) - l) : 0.f;
    float da_s = 0.f, da_r = 0.f;
    if (!gate_fixed) {
      da_s = m * dyo * gs * (1.0f - gs);
      da_r = dyr * gr * (1.0f - gr);
    }
    const float inv_c = c > 0 ? 1.0f / (float)c : 0.f;
    float dd = 0.f;
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      const T dov = from_f32<T>(gs * m * g[i]);
      d_o[base + i] = dov;
      dd += to_f32(dov) * os[i];
      dq_acc[base + i] = gate_fixed ? 0.f : da_s * ws_[i] + da_r * wr_[i];
      dor[base + i] = gr * g[i] * inv_c;
      if (!gate_fixed) {
        pws[i] += da_s * qv[i];
        pwr[i] += da_r * qv[i];
      }
    }
    dd = warp_sum(dd);
    if (lane == 0) {
      dprime[r] = dd - dlse;
      pbs += da_s;
      pbr += da_r;
      plam += dlam;
    }
  }
  // block reduction of the partial parameter gradients
  const int P = 2 * d + 3;
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    red[w][lane * VEC + i] = pws[i];
    red[w][d + lane * VEC + i] = pwr[i];
  }
  if (lane == 0) {
    red[w][2 * d] = pbs;
    red[w][2 * d + 1] = pbr;
    red[w][2 * d + 2] = plam;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < P; e += blockDim.x) {
    float s = 0.f;
    for (int ww = 0; ww < nw; ++ww) s += red[ww][e];
    partials[(size_t)blockIdx.x * P + e] = s;
  }
}

__global__ void param_reduce_kernel(const float* __restrict__ partials, int blocks, int d,
                                    float* __restrict__ dgate_w, float* __restrict__ dgate_b,
                                    float* __restrict__ dlambda) {
  const int P = 2 * d + 3;
  for (int e = threadIdx.x; e < P; e += blockDim.x) {
    double s = 0.0;
    for (int b = 0; b < blocks; ++b) s += (double)partials[(size_t)b * P + e];
    if (e < 2 * d) {
      if (dgate_w) dgate_w[e] = (float)s;
    } else if (e < 2 * d + 2) {
      if (dgate_b) dgate_b[e - 2 * d] = (float)s;
    } else {
      *dlambda = (float)s;
    }
  }
}

template <typename T>
__global__ void cast_out_kernel(const float* __restrict__ src, T* __restrict__ dst, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = from_f32<T>(src[i]);
}

template <typename T>
cudaError_t fuse_bwd(const Geometry& g, const void* q, const void* dy, const void* o_sp,
                     const void* o_race, const float* lse, const int32_t* ctot,
                     const float* gate_w, const float* gate_b, const float* lam, void* d_o,
                     float* dprime, float* dq_acc, float* dor, float* partials, cudaStream_t s) {
  const int64_t rows = (int64_t)g.BH * g.N;
#define ELSAA_FB(VEC)                                                                          \
  fuse_bwd_kernel<T, VEC><<<kParamBlocks, 256, 0, s>>>(                                        \
      static_cast<const T*>(q), static_cast<const T*>(dy), static_cast<const T*>(o_sp),        \
      static_cast<const T*>(o_race), lse, ctot, gate_w, gate_b, g.gate_fixed, g.gate_s,        \
      g.gate_r, lam, rows, g.L, g.d, static_cast<T*>(d_o), dprime, dq_acc, dor, partials)
  switch (g.d / 32) {
    case 1: ELSAA_FB(1); break;
    case 2: ELSAA_FB(2); break;
    default: ELSAA_FB(4); break;
  }
#undef ELSAA_FB
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fuse_bwd(const Geometry& g, const void* q, const void* dy, const void* o_sp,
                            const void* o_race, const float* lse, const int32_t* ctot,
                            const float* gate_w, const float* gate_b, const float* lam,
                            void* d_o, float* dprime, float* dq_acc, float* dor,
                            float* partials, cudaStream_t s) {
  return g.bf16 ? fuse_bwd<__nv_bfloat16>(g, q, dy, o_sp, o_race, lse, ctot, gate_w, gate_b, lam,
                                          d_o, dprime, dq_acc, dor, partials, s)
                : fuse_bwd<float>(g, q, dy, o_sp, o_race, lse, ctot, gate_w, gate_b, lam, d_o,
                                  dprime, dq_acc, dor, partials, s);
}

cudaError_t launch_param_reduce(const Geometry& g, const float* partials, float* dgate_w,
                                float* dgate_b, float* dlambda, cudaStream_t s) {
  param_reduce_kernel<<<1, 256, 0, s>>>(partials, kParamBlocks, g.d, dgate_w, dgate_b, dlambda);
  return cudaGetLastError();
}

cudaError_t launch_cast_out(const Geometry& g, const float* src, void* dst, cudaStream_t s) {
  const int64_t n = (int64_t)g.BH * g.N * g.d;
  const int grid = 148 * 8;
  if (g.bf16)
    cast_out_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(src, static_cast<__nv_bfloat16*>(dst), n);
  else
    cast_out_kernel<float><<<grid, 256, 0, s>>>(src, static_cast<float*>(dst), n);
  return cudaGetLastError();
}

}  // namespace elsaa
