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
// dq_gate goes out either as fp32 rows (dq_acc) or as the pair (da_s, da_r)
// per row (da_out) for a consumer that forms da_s w_s + da_r w_r itself.
// A query takes d / 4 lanes (four values each), so a warp serves 128 / d
// queries per step; per-block partial sums of (dw_s, dw_r, db_s, db_r,
// dlambda) go to a fixed number of slots and are reduced in a fixed order, so
// the parameter gradients are deterministic.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace elsaa {
namespace {

template <typename T>
ELSAA_DEV void ld4(const T* p, float* v);
template <>
ELSAA_DEV void ld4<float>(const float* p, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <>
ELSAA_DEV void ld4<__nv_bfloat16>(const __nv_bfloat16* p, float* v) {
  const uint2 raw = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
// Rounds 4 values to T, stores them, and returns the rounded values in v.
template <typename T>
ELSAA_DEV void st4_round(T* p, float* v);
template <>
ELSAA_DEV void st4_round<float>(float* p, float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
ELSAA_DEV void st4_round<__nv_bfloat16>(__nv_bfloat16* p, float* v) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
  const __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
  uint2 raw;
  raw.x = *reinterpret_cast<const uint32_t*>(&a);
  raw.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = raw;
  const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  v[0] = fa.x; v[1] = fa.y; v[2] = fb.x; v[3] = fb.y;
}

template <int QL>
ELSAA_DEV float gsum(float v) {
#pragma unroll
  for (int o = QL / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// QL = d / 4 lanes per query (4 consecutive values each: 8-byte accesses for
// bf16, 16-byte for fp32), 32 / QL queries per warp.
template <typename T, int QL>
__global__ void __launch_bounds__(256, 4)
fuse_bwd_kernel(const T* __restrict__ q, const T* __restrict__ dy, const T* __restrict__ o_sp,
                const T* __restrict__ o_race, const float* __restrict__ lse,
                const int32_t* __restrict__ ctot, const float* __restrict__ gate_w,
                const float* __restrict__ gate_b, int gate_fixed, float gs_fixed, float gr_fixed,
                const float* __restrict__ lam, int64_t rows, int N, int L, int d,
                T* __restrict__ d_o, float* __restrict__ dprime, float* __restrict__ dq_acc,
                float2* __restrict__ da_out, T* __restrict__ dor, float* __restrict__ absmax,
                float* __restrict__ partials) {
  constexpr int QW = 32 / QL;
  constexpr int CB = 4 * (int)sizeof(T);   // bytes of one lane's 4 values
  __shared__ float red[8][2 * 128 + 3];
  // per warp, two rows in flight: each lane copies its own chunks of q, dy,
  // O_sp, O_race (and its row's lse, Ctot) for the next row by cp.async and
  // reads them back when that row comes up
  __shared__ __align__(16) uint8_t s_stage[8][2][4][32 * CB];
  __shared__ __align__(16) uint32_t s_scal[8][2][2][32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int ql = lane % QL, sub = lane / QL;
  const float lam_v = *lam;
  // gate weights (w_s then w_r) in shared memory, zero for fixed gates; the
  // row chunks are read from the staging ring where they are used, so few
  // values stay live across the row
  __shared__ __align__(16) float s_w[2 * 128];
  for (int i = threadIdx.x; i < 2 * d; i += blockDim.x) s_w[i] = gate_fixed ? 0.f : gate_w[i];
  const float* ws4 = s_w + ql * 4;
  const float* wr4 = s_w + d + ql * 4;
  float pws[4] = {0.f, 0.f, 0.f, 0.f}, pwr[4] = {0.f, 0.f, 0.f, 0.f};
  float pbs = 0.f, pbr = 0.f, plam = 0.f;
  const float bs = gate_fixed ? 0.f : gate_b[0], br = gate_fixed ? 0.f : gate_b[1];
  int64_t cur_bh = -1;   // unit whose largest |g_r dy / Ctot| this lane holds (lanes ql == 0)
  float cur_max = 0.f;
  const int64_t first = ((int64_t)blockIdx.x * nw + w) * QW;
  const int64_t stride = (int64_t)gridDim.x * nw * QW;
  auto stage = [&](int64_t r0, int buf) {
    const int64_t rr = min(r0 + sub, rows - 1);
    const size_t base = (size_t)rr * d + ql * 4;
    const T* src[4] = {q + base, dy + base, o_sp + base, o_race + base};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&s_stage[w][buf][t][lane * CB]));
      if (CB == 8)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src[t]) : "memory");
      else
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src[t]) : "memory");
    }
    const uint32_t d0 = static_cast<uint32_t>(__cvta_generic_to_shared(&s_scal[w][buf][0][lane]));
    const uint32_t d1 = static_cast<uint32_t>(__cvta_generic_to_shared(&s_scal[w][buf][1][lane]));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d0), "l"(lse + rr) : "memory");
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d1), "l"(ctot + rr) : "memory");
  };
  if (first < rows) stage(first, 0);
  asm volatile("cp.async.commit_group;" ::: "memory");
  __syncthreads();   // s_w
  int buf = 0;
  for (int64_t r0 = first; r0 < rows; r0 += stride, buf ^= 1) {
    const int64_t r = r0 + sub;
    const bool valid = r < rows;
    const int64_t rr = valid ? r : rows - 1;
    const size_t base = (size_t)rr * d + ql * 4;
    if (r0 + stride < rows) stage(r0 + stride, buf ^ 1);
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 1;" ::: "memory");   // this row's chunks are in
    const T* st_q = reinterpret_cast<const T*>(&s_stage[w][buf][0][lane * CB]);
    const T* st_g = reinterpret_cast<const T*>(&s_stage[w][buf][1][lane * CB]);
    const T* st_os = reinterpret_cast<const T*>(&s_stage[w][buf][2][lane * CB]);
    const T* st_or = reinterpret_cast<const T*>(&s_stage[w][buf][3][lane * CB]);
    const float l = __uint_as_float(s_scal[w][buf][0][lane]);
    const int c = (int)s_scal[w][buf][1][lane];
    float dyo = 0.f, dyr = 0.f, as = 0.f, ar = 0.f;
    {
      float g[4], os[4], orc[4];
      ld4<T>(st_g, g);
      ld4<T>(st_os, os);
      ld4<T>(st_or, orc);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dyo += g[i] * os[i];
        dyr += g[i] * orc[i];
      }
    }
    if (!gate_fixed) {
      float qv[4], w4s[4], w4r[4];
      ld4<T>(st_q, qv);
      ld4<float>(ws4, w4s);
      ld4<float>(wr4, w4r);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        as += qv[i] * w4s[i];
        ar += qv[i] * w4r[i];
      }
    }
    dyo = gsum<QL>(dyo);
    dyr = gsum<QL>(dyr);
    float gs = gs_fixed, gr = gr_fixed;
    if (!gate_fixed) {
      gs = 1.0f / (1.0f + expf(-(gsum<QL>(as) + bs)));
      gr = 1.0f / (1.0f + expf(-(gsum<QL>(ar) + br)));
    }
    const float zr = (float)c / (float)L;
    const float lz = lam_v * zr;
    const float m = lz > 0.f ? 1.0f / (1.0f + expf(logf(lz) - l)) : 1.0f;
    const float dm = gs * dyo;
    const float dlse = dm * m * (1.0f - m);
    // a causal window without keys (lse = -inf) has Z_sp = 0: m is 0 or 1 and
    // carries no lambda gradient
    const float dlam = (zr > 0.f && l > -INFINITY) ? -dm * m * m * expf(logf(zr) - l) : 0.f;
    float da_s = 0.f, da_r = 0.f;
    if (!gate_fixed) {
      da_s = m * dyo * gs * (1.0f - gs);
      da_r = dyr * gr * (1.0f - gr);
    }
    const float inv_c = c > 0 ? 1.0f / (float)c : 0.f;
    float dov[4], drv[4];
    float vmax = 0.f;
    {
      float g[4];
      ld4<T>(st_g, g);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dov[i] = gs * m * g[i];
        drv[i] = gr * g[i] * inv_c;
        vmax = fmaxf(vmax, fabsf(drv[i]));
      }
    }
    vmax = fmaxf(vmax, 0.f);
#pragma unroll
    for (int o = QL / 2; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    float dd = 0.f;
    if (valid) {
      st4_round<T>(d_o + base, dov);   // dov now holds the stored (rounded) values
      if (dq_acc) {
        float w4s[4], w4r[4];
        ld4<float>(ws4, w4s);
        ld4<float>(wr4, w4r);
        *reinterpret_cast<float4*>(dq_acc + base) =
            make_float4(da_s * w4s[0] + da_r * w4r[0], da_s * w4s[1] + da_r * w4r[1],
                        da_s * w4s[2] + da_r * w4r[2], da_s * w4s[3] + da_r * w4r[3]);
      }
      st4_round<T>(dor + base, drv);
      float os[4];
      ld4<T>(st_os, os);
#pragma unroll
      for (int i = 0; i < 4; ++i) dd += dov[i] * os[i];
      if (!gate_fixed) {
        float qv[4];
        ld4<T>(st_q, qv);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          pws[i] += da_s * qv[i];
          pwr[i] += da_r * qv[i];
        }
      }
    }
    dd = gsum<QL>(dd);
    if (valid && ql == 0) {
      dprime[rr] = dd - dlse;
      if (da_out) da_out[rr] = make_float2(da_s, da_r);
      pbs += da_s;
      pbr += da_r;
      plam += dlam;
      const int64_t bh = rr / N;
      if (bh != cur_bh) {
        if (cur_bh >= 0) atomicMax(reinterpret_cast<int*>(absmax) + cur_bh, __float_as_int(cur_max));
        cur_bh = bh;
        cur_max = 0.f;
      }
      cur_max = fmaxf(cur_max, vmax);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  if (ql == 0 && cur_bh >= 0)
    atomicMax(reinterpret_cast<int*>(absmax) + cur_bh, __float_as_int(cur_max));
  // block reduction of the partial parameter gradients: first across the row
  // groups of a warp, then across warps
#pragma unroll
  for (int o = QL; o < 32; o <<= 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      pws[i] += __shfl_xor_sync(0xffffffffu, pws[i], o);
      pwr[i] += __shfl_xor_sync(0xffffffffu, pwr[i], o);
    }
    pbs += __shfl_xor_sync(0xffffffffu, pbs, o);
    pbr += __shfl_xor_sync(0xffffffffu, pbr, o);
    plam += __shfl_xor_sync(0xffffffffu, plam, o);
  }
  const int P = 2 * d + 3;
  if (sub == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      red[w][ql * 4 + i] = pws[i];
      red[w][d + ql * 4 + i] = pwr[i];
    }
    if (ql == 0) {
      red[w][2 * d] = pbs;
      red[w][2 * d + 1] = pbr;
      red[w][2 * d + 2] = plam;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < P; e += blockDim.x) {
    float s = 0.f;
    for (int ww = 0; ww < nw; ++ww) s += red[ww][e];
    partials[(size_t)blockIdx.x * P + e] = s;
  }
}

// One warp per parameter: lane l sums partial blocks l, l + 32, ... in fp64,
// then the lanes combine in a fixed butterfly order (deterministic).
__global__ void param_reduce_kernel(const float* __restrict__ partials, int blocks, int d,
                                    float* __restrict__ dgate_w, float* __restrict__ dgate_b,
                                    float* __restrict__ dlambda) {
  const int P = 2 * d + 3;
  const int e = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (e >= P) return;
  double s = 0.0;
  for (int b = lane; b < blocks; b += 32) s += (double)partials[(size_t)b * P + e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane != 0) return;
  if (e < 2 * d) {
    if (dgate_w) dgate_w[e] = (float)s;
  } else if (e < 2 * d + 2) {
    if (dgate_b) dgate_b[e - 2 * d] = (float)s;
  } else {
    *dlambda = (float)s;
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
                     float* dprime, float* dq_acc, float2* da_out, void* dor, float* absmax,
                     float* partials, cudaStream_t s) {
  const int64_t rows = (int64_t)g.BH * g.N;
  cudaError_t e = cudaMemsetAsync(absmax, 0, (size_t)g.BH * sizeof(float), s);
  if (e != cudaSuccess) return e;
#define ELSAA_FB(VEC)                                                                          \
  fuse_bwd_kernel<T, VEC><<<kParamBlocks, 256, 0, s>>>(                                        \
      static_cast<const T*>(q), static_cast<const T*>(dy), static_cast<const T*>(o_sp),        \
      static_cast<const T*>(o_race), lse, ctot, gate_w, gate_b, g.gate_fixed, g.gate_s,        \
      g.gate_r, lam, rows, g.N, g.L, g.d, static_cast<T*>(d_o), dprime, dq_acc, da_out,       \
      static_cast<T*>(dor), absmax,                                                            \
      partials)
  switch (g.d) {
    case 32: ELSAA_FB(8); break;
    case 64: ELSAA_FB(16); break;
    default: ELSAA_FB(32); break;
  }
#undef ELSAA_FB
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fuse_bwd(const Geometry& g, const void* q, const void* dy, const void* o_sp,
                            const void* o_race, const float* lse, const int32_t* ctot,
                            const float* gate_w, const float* gate_b, const float* lam,
                            void* d_o, float* dprime, float* dq_acc, float2* da_out, void* dor,
                            float* absmax, float* partials, cudaStream_t s) {
  return g.bf16 ? fuse_bwd<__nv_bfloat16>(g, q, dy, o_sp, o_race, lse, ctot, gate_w, gate_b, lam,
                                          d_o, dprime, dq_acc, da_out, dor, absmax, partials, s)
                : fuse_bwd<float>(g, q, dy, o_sp, o_race, lse, ctot, gate_w, gate_b, lam, d_o,
                                  dprime, dq_acc, da_out, dor, absmax, partials, s);
}

cudaError_t launch_param_reduce(const Geometry& g, const float* partials, float* dgate_w,
                                float* dgate_b, float* dlambda, cudaStream_t s) {
  const int P = 2 * g.d + 3;
  param_reduce_kernel<<<(P * 32 + 255) / 256, 256, 0, s>>>(partials, kParamBlocks, g.d, dgate_w,
                                                           dgate_b, dlambda);
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
