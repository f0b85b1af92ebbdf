// Causal ELSAA: the RACE branch restricted to keys j <= i, and the fusion
// that consumes it.
//
// The pages leave causal use open ("Two Efficient Attentions, One Denominator
// Problem": causal ELSAA was not evaluated).  This extension keeps, for query
// i, only keys with token index j <= i in both branches.  The RACE read-out of
// query i is then a prefix of the tables:
//   Ctot_i = sum_l #{j <= i : h_l(k_j) = h_l(q_i)},
//   O_race_i = sum_l sum_{j <= i, h_l(k_j) = h_l(q_i)} v_j / Ctot_i,
// and its value gradient runs the same prefix backwards:
//   dv_j = sum_l sum_{i >= j, h_l(q_i) = h_l(k_j)} (g_r dy / Ctot)_i.
//
// One CTA per (unit, table) walks the unit's tokens in order with the table
// (fp32 sums and counts) in shared memory: token i adds key i to its bucket,
// then reads query i's bucket and adds that row into the query's accumulator
// (fp32 atomics over the L tables).  Thread c owns column c of every bucket,
// so a token's update and read need no barrier; thread 0 also owns the
// counts.  The backward walk runs from the last token down.  These kernels
// trade speed for simplicity: one token at a time per table.
#include "common.cuh"
#include "internal.h"

namespace elsaa {
namespace {

template <typename TV, typename CodeT>
__global__ void race_causal_fwd_kernel(const CodeT* __restrict__ rcode_q,
                                       const CodeT* __restrict__ rcode_k,
                                       const TV* __restrict__ v, int N, int L, int NB, int d,
                                       float* __restrict__ num, int32_t* __restrict__ ctot,
                                       float* __restrict__ sums, int32_t* __restrict__ counts) {
  extern __shared__ float tab[];                        // [NB][d] sums, then [NB] counts
  int32_t* cnt = reinterpret_cast<int32_t*>(tab + (size_t)NB * d);
  const int l = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  for (int b = 0; b < NB; ++b) tab[(size_t)b * d + c] = 0.f;
  if (c == 0)
    for (int b = 0; b < NB; ++b) cnt[b] = 0;
  const size_t u = (size_t)bh * N;
  for (int i = 0; i < N; ++i) {
    const size_t row = u + i;
    const int kb = (int)rcode_k[row * L + l];
    const int qb = (int)rcode_q[row * L + l];
    if (kb >= NB || qb >= NB) continue;   // codes have race_bits bits; never taken
    tab[(size_t)kb * d + c] += to_f32(v[row * d + c]);   // key i joins its bucket first (j <= i)
    atomicAdd(num + row * d + c, tab[(size_t)qb * d + c]);
    if (c == 0) {
      cnt[kb] += 1;
      atomicAdd(ctot + row, cnt[qb]);
    }
  }
  // the full tables (every key), the saved state of the forward
  const size_t t0 = ((size_t)bh * L + l) * NB;
  for (int b = 0; b < NB; ++b) sums[(t0 + b) * d + c] = tab[(size_t)b * d + c];
  if (c == 0)
    for (int b = 0; b < NB; ++b) counts[t0 + b] = cnt[b];
}

template <typename T, typename CodeT>
__global__ void race_causal_bwd_kernel(const CodeT* __restrict__ rcode_q,
                                       const CodeT* __restrict__ rcode_k,
                                       const T* __restrict__ dor, int N, int L, int NB, int d,
                                       float* __restrict__ dv_acc) {
  extern __shared__ float tab[];                        // [NB][d] table gradient
  const int l = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  for (int b = 0; b < NB; ++b) tab[(size_t)b * d + c] = 0.f;
  const size_t u = (size_t)bh * N;
  for (int i = N - 1; i >= 0; --i) {
    const size_t row = u + i;
    const int qb = (int)rcode_q[row * L + l];
    const int kb = (int)rcode_k[row * L + l];
    if (kb >= NB || qb >= NB) continue;   // codes have race_bits bits; never taken
    tab[(size_t)qb * d + c] += to_f32(dor[row * d + c]);   // query i reads key i too (i >= j)
    atomicAdd(dv_acc + row * d + c, tab[(size_t)kb * d + c]);
  }
}

// y = g_s m O_sp + g_r O_race with the causal read-out: O_race = num / Ctot
// (0 when Ctot = 0), m = 1 / (1 + exp(log(lambda Ctot / L) - lse)); a window
// without keys has lse = -inf and gives m = 0 (m = 1 when lambda Ctot = 0).
// One warp per row, lanes over d.
template <typename T>
__global__ void __launch_bounds__(256)
fuse_causal_kernel(const T* __restrict__ q, const T* __restrict__ o_sp,
                   const float* __restrict__ lse, const float* __restrict__ num,
                   const int32_t* __restrict__ ctot, const float* __restrict__ gate_w,
                   const float* __restrict__ gate_b, int gate_fixed, float gs_fixed,
                   float gr_fixed, const float* __restrict__ lam, int64_t rows, int L, int d,
                   T* __restrict__ y, T* __restrict__ o_race) {
  const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const float lam_v = *lam;
  for (int64_t r = (int64_t)blockIdx.x * nw + (threadIdx.x >> 5); r < rows;
       r += (int64_t)gridDim.x * nw) {
    float gs = gs_fixed, gr = gr_fixed;
    if (!gate_fixed) {
      float as = 0.f, ar = 0.f;
      for (int e = lane; e < d; e += 32) {
        const float x = to_f32(q[r * d + e]);
        as += x * gate_w[e];
        ar += x * gate_w[d + e];
      }
      as = warp_sum(as) + gate_b[0];
      ar = warp_sum(ar) + gate_b[1];
      gs = 1.0f / (1.0f + expf(-as));
      gr = 1.0f / (1.0f + expf(-ar));
    }
    const int c = ctot[r];
    const float inv = c > 0 ? 1.0f / (float)c : 0.f;
    const float l = lse[r];
    const float lz = lam_v * (float)c / (float)L;
    const float m = lz > 0.f ? 1.0f / (1.0f + expf(logf(lz) - l)) : 1.0f;
    for (int e = lane; e < d; e += 32) {
      const float orc = num[r * d + e] * inv;
      y[r * d + e] = from_f32<T>(gs * m * to_f32(o_sp[r * d + e]) + gr * orc);
      if (o_race) o_race[r * d + e] = from_f32<T>(orc);
    }
  }
}

template <typename TV, typename CodeT>
cudaError_t fwd_scan(const Geometry& g, const void* rcode_q, const void* rcode_k, const void* v,
                     float* num, int32_t* ctot, float* sums, int32_t* counts, cudaStream_t s) {
  const size_t smem = (size_t)g.NB * (g.d + 1) * 4;
  cudaError_t e = cudaFuncSetAttribute(race_causal_fwd_kernel<TV, CodeT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  race_causal_fwd_kernel<TV, CodeT><<<dim3(g.L, g.BH), g.d, smem, s>>>(
      static_cast<const CodeT*>(rcode_q), static_cast<const CodeT*>(rcode_k),
      static_cast<const TV*>(v), g.N, g.L, g.NB, g.d, num, ctot, sums, counts);
  return cudaGetLastError();
}

template <typename T, typename CodeT>
cudaError_t bwd_scan(const Geometry& g, const void* rcode_q, const void* rcode_k,
                     const void* dor, float* dv_acc, cudaStream_t s) {
  const size_t smem = (size_t)g.NB * g.d * 4;
  cudaError_t e = cudaFuncSetAttribute(race_causal_bwd_kernel<T, CodeT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  race_causal_bwd_kernel<T, CodeT><<<dim3(g.L, g.BH), g.d, smem, s>>>(
      static_cast<const CodeT*>(rcode_q), static_cast<const CodeT*>(rcode_k),
      static_cast<const T*>(dor), g.N, g.L, g.NB, g.d, dv_acc);
  return cudaGetLastError();
}

}  // namespace

bool race_causal_supported(const Geometry& g) {
  return (size_t)g.NB * (g.d + 1) * 4 <= 200u * 1024u;
}

cudaError_t launch_race_causal_fwd(const Geometry& g, const void* rcode_q, const void* rcode_k,
                                   const void* v, float* num, int32_t* ctot, float* sums,
                                   int32_t* counts, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(num, 0, (size_t)g.BH * g.N * g.d * 4, s);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(ctot, 0, (size_t)g.BH * g.N * 4, s);
  if (e != cudaSuccess) return e;
  if (g.bf16)
    return g.rcode_bytes == 1
               ? fwd_scan<__nv_bfloat16, uint8_t>(g, rcode_q, rcode_k, v, num, ctot, sums, counts, s)
               : fwd_scan<__nv_bfloat16, uint16_t>(g, rcode_q, rcode_k, v, num, ctot, sums, counts, s);
  return g.rcode_bytes == 1
             ? fwd_scan<float, uint8_t>(g, rcode_q, rcode_k, v, num, ctot, sums, counts, s)
             : fwd_scan<float, uint16_t>(g, rcode_q, rcode_k, v, num, ctot, sums, counts, s);
}

cudaError_t launch_race_causal_bwd(const Geometry& g, const void* rcode_q, const void* rcode_k,
                                   const void* dor, float* dv_acc, cudaStream_t s) {
  if (g.bf16)
    return g.rcode_bytes == 1 ? bwd_scan<__nv_bfloat16, uint8_t>(g, rcode_q, rcode_k, dor, dv_acc, s)
                              : bwd_scan<__nv_bfloat16, uint16_t>(g, rcode_q, rcode_k, dor, dv_acc, s);
  return g.rcode_bytes == 1 ? bwd_scan<float, uint8_t>(g, rcode_q, rcode_k, dor, dv_acc, s)
                            : bwd_scan<float, uint16_t>(g, rcode_q, rcode_k, dor, dv_acc, s);
}

cudaError_t launch_fuse_causal(const Geometry& g, const void* q, const void* o_sp,
                               const float* lse, const float* num, const int32_t* ctot,
                               const float* gate_w, const float* gate_b, const float* lam,
                               void* y, void* o_race, cudaStream_t s) {
  const int64_t rows = (int64_t)g.BH * g.N;
  const int64_t want = (rows + 7) / 8;
  const int grid = (int)(want < 148 * 16 ? want : 148 * 16);
  if (g.bf16)
    fuse_causal_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(o_sp), lse, num,
        ctot, gate_w, gate_b, g.gate_fixed, g.gate_s, g.gate_r, lam, rows, g.L, g.d,
        static_cast<__nv_bfloat16*>(y), static_cast<__nv_bfloat16*>(o_race));
  else
    fuse_causal_kernel<float><<<grid, 256, 0, s>>>(
        static_cast<const float*>(q), static_cast<const float*>(o_sp), lse, num, ctot, gate_w,
        gate_b, g.gate_fixed, g.gate_s, g.gate_r, lam, rows, g.L, g.d, static_cast<float*>(y),
        static_cast<float*>(o_race));
  return cudaGetLastError();
}

}  // namespace elsaa
