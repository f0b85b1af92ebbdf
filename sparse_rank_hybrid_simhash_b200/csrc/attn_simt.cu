// Exact sparse branch on CUDA cores (fp32 data and shapes the tcgen05
// kernels do not tile).
//
// "Two Efficient Attentions, One Denominator Problem" (section "Two efficient
// branches can still be mis-scaled"): the sparse branch computes only the
// selected query-key interactions, exactly, and keeps their mass.  The query at
// sorted rank r (chunk j = r / chunk) attends the keys at sorted ranks
// [max(0, (j-lb) chunk), (j+1) chunk), lb = 1 on the pages (other lookbacks are
// an extension this kernel serves): O_sp = softmax(s) V, lse = log sum exp(s),
// s = scale q . k.  One warp per query: lanes over keys for the scores, lanes
// over d for the output; results land at the query's token index.  Causal
// (an extension): keys whose token index exceeds the query's are left out; a
// query left with no key gets O_sp = 0 and lse = -inf.
//
// Backward (one warp per query, keys' gradients by fp32 atomics):
//   p = exp(s - lse), dP = dO . v, dS = p (dP - D'),  D' = dO . O - dlse,
//   dq = scale sum dS k,  dk += scale dS q,  dv += p dO.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace elsaa {
namespace {

template <typename T>
__global__ void __launch_bounds__(128)
attn_fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const int32_t* __restrict__ perm_q, const int32_t* __restrict__ perm_k,
                     int64_t rows, int N, int d, int chunk, int lookback, int causal,
                     float scale, T* __restrict__ o_sp, float* __restrict__ lse) {
  extern __shared__ float sm[];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  float* qs = sm + (size_t)w * (d + (lookback + 1) * chunk);
  float* ps = qs + d;
  for (int64_t row = (int64_t)blockIdx.x * nw + w; row < rows; row += (int64_t)gridDim.x * nw) {
    const int64_t bh = row / N;
    const int r = (int)(row % N);
    const int i = perm_q[bh * N + r];
    const T* qi = q + (bh * N + i) * d;
    for (int e = lane; e < d; e += 32) qs[e] = to_f32(qi[e]);
    __syncwarp();
    const int j = r / chunk;
    const int lo = max(0, (j - lookback) * chunk), nk = (j + 1) * chunk - lo;
    const int32_t* pk = perm_k + bh * N + lo;
    float mx = -INFINITY;
    for (int t = lane; t < nk; t += 32) {
      float s = -INFINITY;
      if (!causal || pk[t] <= i) {
        const T* kr = k + (bh * N + pk[t]) * d;
        s = 0.f;
        for (int e = 0; e < d; ++e) s += qs[e] * to_f32(kr[e]);
        s *= scale;
      }
      ps[t] = s;
      mx = fmaxf(mx, s);
    }
    mx = warp_max(mx);
    const bool any = mx > -INFINITY;   // false only for a causal window without keys
    float sum = 0.f;
    for (int t = lane; t < nk; t += 32) {
      const float p = any ? expf(ps[t] - mx) : 0.f;
      ps[t] = p;
      sum += p;
    }
    sum = warp_sum(sum);
    __syncwarp();
    const float inv = any ? 1.0f / sum : 0.f;
    for (int e = lane; e < d; e += 32) {
      float o = 0.f;
      for (int t = 0; t < nk; ++t) o += ps[t] * to_f32(v[(bh * N + pk[t]) * d + e]);
      o_sp[(bh * N + i) * d + e] = from_f32<T>(o * inv);
    }
    if (lane == 0) lse[bh * N + i] = any ? mx + logf(sum) : -INFINITY;
    __syncwarp();
  }
}

template <typename T>
__global__ void __launch_bounds__(128)
attn_bwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const int32_t* __restrict__ perm_q, const int32_t* __restrict__ perm_k,
                     const T* __restrict__ d_o, const float* __restrict__ lse,
                     const float* __restrict__ dprime, int64_t rows, int N, int d, int chunk,
                     int lookback, int causal, float scale, float* __restrict__ dq_acc,
                     float* __restrict__ dk_acc, float* __restrict__ dv_acc) {
  extern __shared__ float sm[];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int win = (lookback + 1) * chunk;
  float* qs = sm + (size_t)w * (2 * d + 2 * win);
  float* dos = qs + d;
  float* ps = dos + d;
  float* dss = ps + win;
  for (int64_t row = (int64_t)blockIdx.x * nw + w; row < rows; row += (int64_t)gridDim.x * nw) {
    const int64_t bh = row / N;
    const int r = (int)(row % N);
    const int i = perm_q[bh * N + r];
    for (int e = lane; e < d; e += 32) {
      qs[e] = to_f32(q[(bh * N + i) * d + e]);
      dos[e] = to_f32(d_o[(bh * N + i) * d + e]);
    }
    __syncwarp();
    const float l = lse[bh * N + i], dp_i = dprime[bh * N + i];
    const int j = r / chunk;
    const int lo = max(0, (j - lookback) * chunk), nk = (j + 1) * chunk - lo;
    const int32_t* pk = perm_k + bh * N + lo;
    for (int t = lane; t < nk; t += 32) {
      const T* kr = k + (bh * N + pk[t]) * d;
      const T* vr = v + (bh * N + pk[t]) * d;
      float s = 0.f, dp = 0.f;
      for (int e = 0; e < d; ++e) {
        s += qs[e] * to_f32(kr[e]);
        dp += dos[e] * to_f32(vr[e]);
      }
      const float p = (!causal || pk[t] <= i) ? expf(s * scale - l) : 0.f;
      ps[t] = p;
      dss[t] = p * (dp - dp_i);
    }
    __syncwarp();
    for (int e = lane; e < d; e += 32) {
      float dq = 0.f;
      for (int t = 0; t < nk; ++t) {
        const int64_t kr = (bh * N + pk[t]) * d + e;
        dq += dss[t] * to_f32(k[kr]);
        atomicAdd(dk_acc + kr, scale * dss[t] * qs[e]);
        atomicAdd(dv_acc + kr, ps[t] * dos[e]);
      }
      dq_acc[(bh * N + i) * d + e] += scale * dq;
    }
    __syncwarp();
  }
}

int rows_grid(int64_t rows, int warps) {
  const int64_t b = (rows + warps - 1) / warps;
  return (int)(b < 148 * 64 ? b : 148 * 64);
}

template <typename T>
cudaError_t fwd(const Geometry& g, const void* q, const void* k, const void* v,
                const int32_t* perm_q, const int32_t* perm_k, void* o_sp, float* lse,
                cudaStream_t s) {
  const size_t smem = 4 * (size_t)(g.d + (g.lookback + 1) * g.chunk) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t rows = (int64_t)g.BH * g.N;
  attn_fwd_simt_kernel<T><<<rows_grid(rows, 4), 128, smem, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), perm_q,
      perm_k, rows, g.N, g.d, g.chunk, g.lookback, g.causal, g.scale, static_cast<T*>(o_sp), lse);
  return cudaGetLastError();
}

template <typename T>
cudaError_t bwd(const Geometry& g, const void* q, const void* k, const void* v,
                const int32_t* perm_q, const int32_t* perm_k, const void* d_o, const float* lse,
                const float* dprime, float* dq_acc, float* dk_acc, float* dv_acc,
                cudaStream_t s) {
  const size_t smem = 4 * (size_t)(2 * g.d + 2 * (g.lookback + 1) * g.chunk) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t rows = (int64_t)g.BH * g.N;
  attn_bwd_simt_kernel<T><<<rows_grid(rows, 4), 128, smem, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), perm_q,
      perm_k, static_cast<const T*>(d_o), lse, dprime, rows, g.N, g.d, g.chunk, g.lookback,
      g.causal, g.scale, dq_acc, dk_acc, dv_acc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_simt(const Geometry& g, const void* q, const void* k, const void* v,
                                 const int32_t* perm_q, const int32_t* perm_k, void* o_sp,
                                 float* lse, cudaStream_t s) {
  return g.bf16 ? fwd<__nv_bfloat16>(g, q, k, v, perm_q, perm_k, o_sp, lse, s)
                : fwd<float>(g, q, k, v, perm_q, perm_k, o_sp, lse, s);
}

cudaError_t launch_attn_bwd_simt(const Geometry& g, const void* q, const void* k, const void* v,
                                 const int32_t* perm_q, const int32_t* perm_k, const void* d_o,
                                 const float* lse, const float* dprime, float* dq_acc,
                                 float* dk_acc, float* dv_acc, cudaStream_t s) {
  return g.bf16 ? bwd<__nv_bfloat16>(g, q, k, v, perm_q, perm_k, d_o, lse, dprime, dq_acc,
                                     dk_acc, dv_acc, s)
                : bwd<float>(g, q, k, v, perm_q, perm_k, d_o, lse, dprime, dq_acc, dk_acc,
                             dv_acc, s);
}

}  // namespace elsaa
