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
// The walk: one warp takes 32 / L columns of all L tables of a unit (L
// dividing 32), lane = (column, table); the warp's slab of the tables sits in
// shared memory as [bucket][lane], so every lane always reads and writes its
// own bank.  Token by token (in order; the backward from the last token
// down) each lane adds the token's value column to its table's key bucket and
// reads its table's query bucket; a shuffle tree sums the L tables and one
// lane writes the row's column, so every output element has one writer and
// no atomics.  Ctot and the counts come from one more warp per unit that
// walks the bucket counts the same way.  Shapes whose tables do not fit
// (L > 32 or too many buckets) take the per-table scans: one CTA per (unit,
// table), one token at a time, thread c owning column c, fp32 atomics
// summing the tables.
#include "common.cuh"
#include "internal.h"

namespace elsaa {
namespace {

constexpr int kWalkWarps = 2;   // column groups per CTA
constexpr int kGroup = 32;      // tokens per prefetched group

// Code of token position p (0 .. 31) of a group whose codes of one table were
// loaded as consecutive 16-byte words.
template <typename CodeT>
ELSAA_DEV int code_at(const uint4* c, int p) {
  constexpr int per_word = 4 / (int)sizeof(CodeT);
  const int wi = p / per_word;
  const uint4 q = c[wi >> 2];
  const uint32_t w = (wi & 3) == 0 ? q.x : (wi & 3) == 1 ? q.y : (wi & 3) == 2 ? q.z : q.w;
  return (int)((w >> ((p % per_word) * 8 * (int)sizeof(CodeT))) &
               (sizeof(CodeT) == 1 ? 0xFFu : 0xFFFFu));
}

// MODE 0: forward (x = v; out = the numerators; at the end every warp writes
// its slab of the full tables, and one more block per unit walks the counts
// for Ctot and the count tables); MODE 1: backward (x = g_r dy / Ctot by
// query code; out = the RACE value gradient).  L = 2^LOGL tables; lane =
// (sub, l), sub picking one of the warp's 32 / L columns.  Codes come
// table-major ([BH][L][N]); tokens go in groups of 32, loaded two groups
// ahead: a lane's 32 codes of its table in 16-byte words, and one x value
// per lane that the shuffles hand to the lanes that need it.  After a
// group's shared-memory steps each lane holds 32 partial sums (its table's
// bucket rows); a reduce-scatter over the L lanes (31 shuffles for L = 32)
// leaves lane l the L-table sums of tokens 32 / L l .. + 32 / L - 1, which it
// stores.
template <int MODE, typename TX, typename CodeT, int LOGL>
__global__ void __launch_bounds__(kWalkWarps * 32)
race_causal_walk_kernel(const CodeT* __restrict__ rtq, const CodeT* __restrict__ rtk,
                        const TX* __restrict__ x, int N, int NB, int d, float* __restrict__ out,
                        int32_t* __restrict__ ctot, float* __restrict__ sums,
                        int32_t* __restrict__ counts) {
  constexpr int L = 1 << LOGL, CPW = 32 / L, G = kGroup, PER = G / L;
  constexpr int W16 = G * (int)sizeof(CodeT) / 16;   // 16-byte words per 32 codes
  extern __shared__ float slab[];   // [kWalkWarps][NB][32]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int l = lane & (L - 1), sub = lane >> LOGL;
  const int bh = blockIdx.y;
  const size_t u = (size_t)bh * N;
  const int nblk = d / CPW / kWalkWarps;
  const bool count_walk = MODE == 0 && (int)blockIdx.x == nblk;
  if (count_walk && warp != 0) return;
  float* tab = slab + (size_t)warp * NB * 32;
  int32_t* cnt = reinterpret_cast<int32_t*>(tab);
  for (int b = 0; b < NB; ++b) tab[b * 32 + lane] = 0.f;   // (as int: 0)
  __syncwarp();
  const int col = count_walk ? 0 : (blockIdx.x * kWalkWarps + warp) * CPW + sub;
  const uint4* tk = reinterpret_cast<const uint4*>(rtk + ((size_t)bh * L + l) * N);
  const uint4* tq = reinterpret_cast<const uint4*>(rtq + ((size_t)bh * L + l) * N);
  const int ngroups = N / G;
  struct In {
    uint4 kc[W16], qc[W16];
    float xv[PER];
  };
  // group g covers token positions base .. base + 31 (walked upwards in the
  // forward, downwards in the backward)
  auto base_of = [&](int g) { return MODE == 0 ? g * G : N - G - g * G; };
  auto fetch = [&](int g, In& in) {
    const int base = base_of(g);
#pragma unroll
    for (int w = 0; w < W16; ++w) {
      in.kc[w] = __ldg(tk + base / (16 / (int)sizeof(CodeT)) + w);
      in.qc[w] = __ldg(tq + base / (16 / (int)sizeof(CodeT)) + w);
    }
#pragma unroll
    for (int k = 0; k < PER; ++k)
      in.xv[k] = count_walk ? 0.f : to_f32(x[(u + base + l + L * k) * d + col]);
  };
  // two groups in flight ahead of the one being walked
  In cur, nxt, nxt2;
  fetch(0, nxt);
  if (ngroups > 1) fetch(1, nxt2);
  for (int g = 0; g < ngroups; ++g) {
    cur = nxt;
    nxt = nxt2;
    if (g + 2 < ngroups) fetch(g + 2, nxt2);
    const int base = base_of(g);
    if (count_walk) {
      int c[G];
#pragma unroll
      for (int e = 0; e < G; ++e) {
        const int p = e;   // the forward walks upwards
        cnt[code_at<CodeT>(cur.kc, p) * 32 + lane] += 1;   // key i joins its bucket first
        c[p] = cnt[code_at<CodeT>(cur.qc, p) * 32 + lane];
      }
#pragma unroll
      for (int lev = 0; lev < LOGL; ++lev) {
        const int o = L >> (lev + 1), C = G >> lev;
        const bool up = (l & o) != 0;
#pragma unroll
        for (int j = 0; j < C / 2; ++j) {
          const int send = up ? c[j] : c[j + C / 2];
          const int keep = up ? c[j + C / 2] : c[j];
          c[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      if (sub == 0)
#pragma unroll
        for (int j = 0; j < PER; ++j) ctot[u + base + l * PER + j] = c[j];
      continue;
    }
    float r[G];
#pragma unroll
    for (int e = 0; e < G; ++e) {
      const int p = MODE == 0 ? e : G - 1 - e;   // position in the group
      const float xe = __shfl_sync(0xffffffffu, cur.xv[p >> LOGL], (sub << LOGL) | (p & (L - 1)));
      const int kb = code_at<CodeT>(cur.kc, p), qb = code_at<CodeT>(cur.qc, p);
      // forward: key i joins its bucket, then query i reads (j <= i); backward:
      // query i joins its bucket, then key i reads (i >= j).  A lane only ever
      // touches its own bank column of the slab.
      tab[(MODE == 0 ? kb : qb) * 32 + lane] += xe;
      r[p] = tab[(MODE == 0 ? qb : kb) * 32 + lane];
    }
#pragma unroll
    for (int lev = 0; lev < LOGL; ++lev) {
      const int o = L >> (lev + 1), C = G >> lev;
      const bool up = (l & o) != 0;
#pragma unroll
      for (int j = 0; j < C / 2; ++j) {
        const float send = up ? r[j] : r[j + C / 2];
        const float keep = up ? r[j + C / 2] : r[j];
        r[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
#pragma unroll
    for (int j = 0; j < PER; ++j) out[(u + base + l * PER + j) * d + col] = r[j];
  }
  if (MODE == 0) {
    if (count_walk) {
      if (sub == 0)
        for (int b = 0; b < NB; ++b) counts[((size_t)bh * L + l) * NB + b] = cnt[b * 32 + lane];
    } else {
      for (int b = 0; b < NB; ++b)
        sums[(((size_t)bh * L + l) * NB + b) * d + col] = tab[b * 32 + lane];
    }
  }
}

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

// The warp walk applies for 4 to 32 tables (a power of two), whole 32-token
// groups, column groups that fill whole blocks, and slabs that fit shared
// memory.
bool walk_ok(const Geometry& g) {
  if (g.L != 4 && g.L != 8 && g.L != 16 && g.L != 32) return false;
  if (g.N % kGroup != 0) return false;
  const int cpw = 32 / g.L;
  if (g.d % cpw != 0 || (g.d / cpw) % kWalkWarps != 0) return false;
  return (size_t)kWalkWarps * g.NB * 32 * 4 <= 200u * 1024u;
}

template <int MODE, typename TX, typename CodeT, int LOGL>
cudaError_t walk_l(const Geometry& g, const void* rtq, const void* rtk, const void* x, float* out,
                   int32_t* ctot, float* sums, int32_t* counts, cudaStream_t s) {
  auto* kern = race_causal_walk_kernel<MODE, TX, CodeT, LOGL>;
  const size_t smem = (size_t)kWalkWarps * g.NB * 32 * 4;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int nblk = g.d / (32 / g.L) / kWalkWarps;
  kern<<<dim3(nblk + (MODE == 0 ? 1 : 0), g.BH), kWalkWarps * 32, smem, s>>>(
      static_cast<const CodeT*>(rtq), static_cast<const CodeT*>(rtk), static_cast<const TX*>(x),
      g.N, g.NB, g.d, out, ctot, sums, counts);
  return cudaGetLastError();
}

template <int MODE, typename TX, typename CodeT>
cudaError_t walk(const Geometry& g, const void* rtq, const void* rtk, const void* x, float* out,
                 int32_t* ctot, float* sums, int32_t* counts, cudaStream_t s) {
  switch (g.L) {
    case 4: return walk_l<MODE, TX, CodeT, 2>(g, rtq, rtk, x, out, ctot, sums, counts, s);
    case 8: return walk_l<MODE, TX, CodeT, 3>(g, rtq, rtk, x, out, ctot, sums, counts, s);
    case 16: return walk_l<MODE, TX, CodeT, 4>(g, rtq, rtk, x, out, ctot, sums, counts, s);
    default: return walk_l<MODE, TX, CodeT, 5>(g, rtq, rtk, x, out, ctot, sums, counts, s);
  }
}

}  // namespace

bool race_causal_supported(const Geometry& g) {
  return walk_ok(g) || (size_t)g.NB * (g.d + 1) * 4 <= 200u * 1024u;
}


namespace {
// Calls f(value-type tag, code-type tag) for the geometry's data dtype and
// RACE code width.
template <typename F>
cudaError_t by_types(const Geometry& g, F&& f) {
  if (g.bf16)
    return g.rcode_bytes == 1 ? f(__nv_bfloat16{}, uint8_t{}) : f(__nv_bfloat16{}, uint16_t{});
  return g.rcode_bytes == 1 ? f(float{}, uint8_t{}) : f(float{}, uint16_t{});
}
}  // namespace

cudaError_t launch_race_causal_fwd(const Geometry& g, const void* rcode_q, const void* rcode_k,
                                   const void* rcode_tq, const void* rcode_tk, const void* v,
                                   float* num, int32_t* ctot, float* sums, int32_t* counts,
                                   cudaStream_t s) {
  if (walk_ok(g))
    return by_types(g, [&](auto tv, auto tc) {
      return walk<0, decltype(tv), decltype(tc)>(g, rcode_tq, rcode_tk, v, num, ctot, sums,
                                                 counts, s);
    });
  cudaError_t e = cudaMemsetAsync(num, 0, (size_t)g.BH * g.N * g.d * 4, s);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(ctot, 0, (size_t)g.BH * g.N * 4, s);
  if (e != cudaSuccess) return e;
  return by_types(g, [&](auto tv, auto tc) {
    return fwd_scan<decltype(tv), decltype(tc)>(g, rcode_q, rcode_k, v, num, ctot, sums, counts,
                                                s);
  });
}

cudaError_t launch_race_causal_bwd(const Geometry& g, const void* rcode_q, const void* rcode_k,
                                   const void* rcode_tq, const void* rcode_tk, const void* dor,
                                   float* dv_acc, cudaStream_t s) {
  if (walk_ok(g))
    return by_types(g, [&](auto tv, auto tc) {
      return walk<1, decltype(tv), decltype(tc)>(g, rcode_tq, rcode_tk, dor, dv_acc, nullptr,
                                                 nullptr, nullptr, s);
    });
  return by_types(g, [&](auto tv, auto tc) {
    return bwd_scan<decltype(tv), decltype(tc)>(g, rcode_q, rcode_k, dor, dv_acc, s);
  });
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
