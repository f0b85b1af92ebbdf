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
// Several hash rounds (an extension): every round has its own order of Q and
// K; the query attends the union of its rounds' windows, each key once.
//
// Backward (one warp per query, keys' gradients by fp32 atomics):
//   p = exp(s - lse), dP = dO . v, dS = p (dP - D'),  D' = dO . O - dlse,
//   dq = scale sum dS k,  dk += scale dS q,  dv += p dO.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace elsaa {
namespace {

// Several hash rounds (an extension): round t's permutations sit t * rstride
// after round 0's, and rank_* hold their inverses.  The query's window in
// round t is [lo_t, hi_t) of that round's sorted keys; a key of round t's
// window that an earlier round's window already holds is left out, so every
// key of the union counts once.  win: slots per round in the score buffer.
ELSAA_DEV void query_windows(const int32_t* __restrict__ rank_q, int64_t rstride, int64_t qi,
                             int r0, int N, int chunk, int lookback, int rounds, int* lo,
                             int* hi) {
  for (int t = 0; t < rounds; ++t) {
    const int r = t == 0 ? r0 : rank_q[t * rstride + qi];
    const int j = r / chunk;
    lo[t] = max(0, (j - lookback) * chunk);
    hi[t] = min(N, (j + 1) * chunk);
  }
}

// true if the key at row kidx lies in an earlier round's window of this query
ELSAA_DEV bool seen_before(const int32_t* __restrict__ rank_k, int64_t rstride, int64_t kidx,
                           int t, const int* lo, const int* hi) {
  for (int u = 0; u < t; ++u) {
    const int rk = rank_k[u * rstride + kidx];
    if (rk >= lo[u] && rk < hi[u]) return true;
  }
  return false;
}

template <typename T>
__global__ void __launch_bounds__(128)
attn_fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const int32_t* __restrict__ perm_q, const int32_t* __restrict__ perm_k,
                     const int32_t* __restrict__ rank, int64_t rows, int N, int d, int chunk,
                     int lookback, int causal, int rounds, float scale, T* __restrict__ o_sp,
                     float* __restrict__ lse) {
  extern __shared__ float sm[];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int win = (lookback + 1) * chunk;
  const int64_t rstride = 2 * rows;   // one round's permutations: queries then keys
  float* qs = sm + (size_t)w * (d + rounds * win + 2 * kMaxRounds);
  float* ps = qs + d;
  int* wlo = reinterpret_cast<int*>(ps + rounds * win);
  int* whi = wlo + kMaxRounds;
  const int32_t* rank_q = rank;
  const int32_t* rank_k = rank + rows;
  for (int64_t row = (int64_t)blockIdx.x * nw + w; row < rows; row += (int64_t)gridDim.x * nw) {
    const int64_t bh = row / N;
    const int r = (int)(row % N);
    const int i = perm_q[bh * N + r];
    const T* qi = q + (bh * N + i) * d;
    for (int e = lane; e < d; e += 32) qs[e] = to_f32(qi[e]);
    if (lane == 0)
      query_windows(rank_q, rstride, bh * N + i, r, N, chunk, lookback, rounds, wlo, whi);
    __syncwarp();
    float mx = -INFINITY;
    for (int t = 0; t < rounds; ++t) {
      const int lo = wlo[t], nk = whi[t] - lo;
      const int32_t* pk = perm_k + t * rstride + bh * N + lo;
      for (int x = lane; x < nk; x += 32) {
        float s = -INFINITY;
        const int key = pk[x];
        if ((!causal || key <= i) &&
            (t == 0 || !seen_before(rank_k, rstride, bh * N + key, t, wlo, whi))) {
          const T* kr = k + (bh * N + key) * d;
          s = 0.f;
          for (int e = 0; e < d; ++e) s += qs[e] * to_f32(kr[e]);
          s *= scale;
        }
        ps[t * win + x] = s;
        mx = fmaxf(mx, s);
      }
    }
    mx = warp_max(mx);
    const bool any = mx > -INFINITY;   // false only for a causal window without keys
    float sum = 0.f;
    for (int t = 0; t < rounds; ++t) {
      const int nk = whi[t] - wlo[t];
      for (int x = lane; x < nk; x += 32) {
        const float p = any ? expf(ps[t * win + x] - mx) : 0.f;
        ps[t * win + x] = p;
        sum += p;
      }
    }
    sum = warp_sum(sum);
    __syncwarp();
    const float inv = any ? 1.0f / sum : 0.f;
    for (int e = lane; e < d; e += 32) {
      float o = 0.f;
      for (int t = 0; t < rounds; ++t) {
        const int lo = wlo[t], nk = whi[t] - lo;
        const int32_t* pk = perm_k + t * rstride + bh * N + lo;
        for (int x = 0; x < nk; ++x) {
          const float p = ps[t * win + x];
          if (p != 0.f) o += p * to_f32(v[(bh * N + pk[x]) * d + e]);   // warp-uniform
        }
      }
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
                     const int32_t* __restrict__ rank, const T* __restrict__ d_o,
                     const float* __restrict__ lse, const float* __restrict__ dprime,
                     int64_t rows, int N, int d, int chunk, int lookback, int causal, int rounds,
                     float scale, float* __restrict__ dq_acc, float* __restrict__ dk_acc,
                     float* __restrict__ dv_acc) {
  extern __shared__ float sm[];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int win = (lookback + 1) * chunk;
  const int64_t rstride = 2 * rows;
  float* qs = sm + (size_t)w * (2 * d + 2 * rounds * win + 2 * kMaxRounds);
  float* dos = qs + d;
  float* ps = dos + d;
  float* dss = ps + rounds * win;
  int* wlo = reinterpret_cast<int*>(dss + rounds * win);
  int* whi = wlo + kMaxRounds;
  const int32_t* rank_q = rank;
  const int32_t* rank_k = rank + rows;
  for (int64_t row = (int64_t)blockIdx.x * nw + w; row < rows; row += (int64_t)gridDim.x * nw) {
    const int64_t bh = row / N;
    const int r = (int)(row % N);
    const int i = perm_q[bh * N + r];
    for (int e = lane; e < d; e += 32) {
      qs[e] = to_f32(q[(bh * N + i) * d + e]);
      dos[e] = to_f32(d_o[(bh * N + i) * d + e]);
    }
    if (lane == 0)
      query_windows(rank_q, rstride, bh * N + i, r, N, chunk, lookback, rounds, wlo, whi);
    __syncwarp();
    const float l = lse[bh * N + i], dp_i = dprime[bh * N + i];
    for (int t = 0; t < rounds; ++t) {
      const int lo = wlo[t], nk = whi[t] - lo;
      const int32_t* pk = perm_k + t * rstride + bh * N + lo;
      for (int x = lane; x < nk; x += 32) {
        const int key = pk[x];
        float p = 0.f, ds = 0.f;
        if ((!causal || key <= i) &&
            (t == 0 || !seen_before(rank_k, rstride, bh * N + key, t, wlo, whi))) {
          const T* kr = k + (bh * N + key) * d;
          const T* vr = v + (bh * N + key) * d;
          float s = 0.f, dp = 0.f;
          for (int e = 0; e < d; ++e) {
            s += qs[e] * to_f32(kr[e]);
            dp += dos[e] * to_f32(vr[e]);
          }
          p = expf(s * scale - l);
          ds = p * (dp - dp_i);
        }
        ps[t * win + x] = p;
        dss[t * win + x] = ds;
      }
    }
    __syncwarp();
    for (int e = lane; e < d; e += 32) {
      float dq = 0.f;
      for (int t = 0; t < rounds; ++t) {
        const int lo = wlo[t], nk = whi[t] - lo;
        const int32_t* pk = perm_k + t * rstride + bh * N + lo;
        for (int x = 0; x < nk; ++x) {
          const float p = ps[t * win + x], ds = dss[t * win + x];
          if (p == 0.f && ds == 0.f) continue;   // masked or already counted (warp-uniform)
          const int64_t kr = (bh * N + pk[x]) * d + e;
          dq += ds * to_f32(k[kr]);
          atomicAdd(dk_acc + kr, scale * ds * qs[e]);
          atomicAdd(dv_acc + kr, p * dos[e]);
        }
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
                const int32_t* perm_q, const int32_t* perm_k, const int32_t* rank, void* o_sp,
                float* lse, cudaStream_t s) {
  const size_t smem =
      4 * (size_t)(g.d + g.rounds * (g.lookback + 1) * g.chunk + 2 * kMaxRounds) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t rows = (int64_t)g.BH * g.N;
  attn_fwd_simt_kernel<T><<<rows_grid(rows, 4), 128, smem, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), perm_q,
      perm_k, rank, rows, g.N, g.d, g.chunk, g.lookback, g.causal, g.rounds, g.scale,
      static_cast<T*>(o_sp), lse);
  return cudaGetLastError();
}

template <typename T>
cudaError_t bwd(const Geometry& g, const void* q, const void* k, const void* v,
                const int32_t* perm_q, const int32_t* perm_k, const int32_t* rank,
                const void* d_o, const float* lse, const float* dprime, float* dq_acc,
                float* dk_acc, float* dv_acc, cudaStream_t s) {
  const size_t smem =
      4 * (size_t)(2 * g.d + 2 * g.rounds * (g.lookback + 1) * g.chunk + 2 * kMaxRounds) *
      sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t rows = (int64_t)g.BH * g.N;
  attn_bwd_simt_kernel<T><<<rows_grid(rows, 4), 128, smem, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), perm_q,
      perm_k, rank, static_cast<const T*>(d_o), lse, dprime, rows, g.N, g.d, g.chunk,
      g.lookback, g.causal, g.rounds, g.scale, dq_acc, dk_acc, dv_acc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_simt(const Geometry& g, const void* q, const void* k, const void* v,
                                 const int32_t* perm_q, const int32_t* perm_k,
                                 const int32_t* rank, void* o_sp, float* lse, cudaStream_t s) {
  if (g.rounds > kMaxRounds || (g.rounds > 1 && rank == nullptr)) return cudaErrorInvalidValue;
  return g.bf16 ? fwd<__nv_bfloat16>(g, q, k, v, perm_q, perm_k, rank, o_sp, lse, s)
                : fwd<float>(g, q, k, v, perm_q, perm_k, rank, o_sp, lse, s);
}

cudaError_t launch_attn_bwd_simt(const Geometry& g, const void* q, const void* k, const void* v,
                                 const int32_t* perm_q, const int32_t* perm_k,
                                 const int32_t* rank, const void* d_o, const float* lse,
                                 const float* dprime, float* dq_acc, float* dk_acc,
                                 float* dv_acc, cudaStream_t s) {
  if (g.rounds > kMaxRounds || (g.rounds > 1 && rank == nullptr)) return cudaErrorInvalidValue;
  return g.bf16 ? bwd<__nv_bfloat16>(g, q, k, v, perm_q, perm_k, rank, d_o, lse, dprime, dq_acc,
                                     dk_acc, dv_acc, s)
                : bwd<float>(g, q, k, v, perm_q, perm_k, rank, d_o, lse, dprime, dq_acc, dk_acc,
                             dv_acc, s);
}

}  // namespace elsaa
