// The low-rank RACE branch: table build (scatter-add) and query gather.
//
// "Two Efficient Attentions, One Denominator Problem" (section "Two efficient
// branches can still be mis-scaled"): the RACE branch compresses broad
// interaction structure into hash-bucket summaries and gives every query
// global context.  Per (batch, head) unit and table l of 2^K_r buckets:
//   T[l][b] = sum of v_j over keys with h_l(k_j) = b,  C[l][b] = their count;
// a query reads its bucket in every table:
//   Ctot = sum_l C[l][h_l(q)],  O_race = sum_l T[l][h_l(q)] / Ctot  (0 if Ctot = 0),
//   Z_race = Ctot / L.
//
// Build: one block owns a slab of tables x a slice of d in shared memory and
// streams every key of its unit through it (shared-memory fp32 atomics; the
// slab is written once, so global memory sees no atomics).  Tables too large
// for shared memory take a global-atomic variant.
// Gather: one warp per query, lanes across d, codes broadcast by shuffle.
// The forward gather is fused with the gates, the multiplier and the output.
#include "common.cuh"
#include "internal.h"

namespace elsaa {
namespace {

constexpr int kBuildSmemBudget = 200 * 1024;

template <typename TV, typename CodeT>
__global__ void __launch_bounds__(512)
race_build_smem_kernel(const CodeT* __restrict__ codes, const TV* __restrict__ vals, int N,
                       int L, int NB, int d, int tabs, int dsl, float* __restrict__ sums,
                       int32_t* __restrict__ counts) {
  extern __shared__ float tab[];
  const int bh = blockIdx.y;
  const int nds = d / dsl;
  const int tgroup = blockIdx.x / nds, dpart = blockIdx.x % nds;
  const int l0 = tgroup * tabs, nt = min(L, l0 + tabs) - l0;
  const int d0 = dpart * dsl;
  const bool do_counts = counts != nullptr && dpart == 0;
  int* cnt = reinterpret_cast<int*>(tab + (size_t)tabs * NB * dsl);
  for (int i = threadIdx.x; i < nt * NB * dsl; i += blockDim.x) tab[i] = 0.f;
  for (int i = threadIdx.x; i < nt * NB; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const CodeT* cb = codes + (size_t)bh * N * L;
  const TV* vb = vals + (size_t)bh * N * d;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int per_lane = dsl >> 5;   // 1..4
  for (int j = w; j < N; j += nw) {
    float x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      x[i] = i < per_lane ? to_f32(vb[(size_t)j * d + d0 + lane + 32 * i]) : 0.f;
    for (int t = 0; t < nt; ++t) {
      const int b = (int)cb[(size_t)j * L + l0 + t];
      float* row = tab + ((size_t)t * NB + b) * dsl;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (i < per_lane) atomicAdd(row + lane + 32 * i, x[i]);
      if (do_counts && lane == 0) atomicAdd(cnt + t * NB + b, 1);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nt * NB * dsl; i += blockDim.x) {
    const int t = i / (NB * dsl), rem = i % (NB * dsl), b = rem / dsl, e = rem % dsl;
    sums[(((size_t)bh * L + l0 + t) * NB + b) * d + d0 + e] = tab[i];
  }
  if (do_counts)
    for (int i = threadIdx.x; i < nt * NB; i += blockDim.x)
      counts[((size_t)bh * L + l0) * NB + i] = cnt[i];
}

// Large tables: fp32 atomics straight into zeroed global tables.
template <typename TV, typename CodeT>
__global__ void __launch_bounds__(256)
race_build_global_kernel(const CodeT* __restrict__ codes, const TV* __restrict__ vals,
                         int64_t rows, int N, int L, int NB, int d, float* __restrict__ sums,
                         int32_t* __restrict__ counts) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int64_t r = (int64_t)blockIdx.x * nw + w; r < rows; r += (int64_t)gridDim.x * nw) {
    const int64_t bh = r / N;
    for (int t = 0; t < L; ++t) {
      const int b = (int)codes[r * L + t];
      float* row = sums + ((bh * L + t) * NB + b) * d;
      for (int e = lane; e < d; e += 32) atomicAdd(row + e, to_f32(vals[r * d + e]));
      if (counts && lane == 0) atomicAdd(counts + (bh * L + t) * NB + b, 1);
    }
  }
}

template <typename CodeT, int VEC>
__global__ void __launch_bounds__(256)
race_gather_sum_kernel(const CodeT* __restrict__ codes, const float* __restrict__ tables,
                       int64_t rows, int N, int L, int NB, int d, float* __restrict__ out) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int64_t r = (int64_t)blockIdx.x * nw + w; r < rows; r += (int64_t)gridDim.x * nw) {
    const int64_t bh = r / N;
    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
    for (int t0 = 0; t0 < L; t0 += 32) {
      const int mycode = t0 + lane < L ? (int)codes[r * L + t0 + lane] : 0;
      const int nt = min(32, L - t0);
      for (int t = 0; t < nt; ++t) {
        const int b = __shfl_sync(0xffffffffu, mycode, t);
        const float* row = tables + ((bh * L + t0 + t) * NB + b) * d + lane * VEC;
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[i] += row[i];
      }
    }
    float* o = out + r * d + lane * VEC;
#pragma unroll
    for (int i = 0; i < VEC; ++i) o[i] = acc[i];
  }
}

template <typename T, typename CodeT, int VEC>
__global__ void __launch_bounds__(256)
race_fuse_fwd_kernel(const T* __restrict__ q, const CodeT* __restrict__ rcode_q,
                     const float* __restrict__ sums, const int32_t* __restrict__ counts,
                     const T* __restrict__ o_sp, const float* __restrict__ lse,
                     const float* __restrict__ gate_w, const float* __restrict__ gate_b,
                     int gate_fixed, float gs_fixed, float gr_fixed,
                     const float* __restrict__ lam, int64_t rows, int N, int L, int NB, int d,
                     T* __restrict__ y, T* __restrict__ o_race, int32_t* __restrict__ ctot_out) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const float lam_v = *lam;
  for (int64_t r = (int64_t)blockIdx.x * nw + w; r < rows; r += (int64_t)gridDim.x * nw) {
    const int64_t bh = r / N;
    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
    int ctot = 0;
    for (int t0 = 0; t0 < L; t0 += 32) {
      const int mycode = t0 + lane < L ? (int)rcode_q[r * L + t0 + lane] : 0;
      if (t0 + lane < L) ctot += counts[(bh * L + t0 + lane) * NB + mycode];
      const int nt = min(32, L - t0);
      for (int t = 0; t < nt; ++t) {
        const int b = __shfl_sync(0xffffffffu, mycode, t);
        const float* row = sums + ((bh * L + t0 + t) * NB + b) * d + lane * VEC;
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[i] += row[i];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ctot += __shfl_xor_sync(0xffffffffu, ctot, o);
    const float inv = ctot > 0 ? 1.0f / (float)ctot : 0.f;
    float qv[VEC], os[VEC], orc[VEC];
    const size_t base = (size_t)r * d + lane * VEC;
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      qv[i] = to_f32(q[base + i]);
      os[i] = to_f32(o_sp[base + i]);
      orc[i] = acc[i] * inv;
    }
    float gs = gs_fixed, gr = gr_fixed;
    if (!gate_fixed) {
      float as = 0.f, ar = 0.f;
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        as += qv[i] * gate_w[lane * VEC + i];
        ar += qv[i] * gate_w[d + lane * VEC + i];
      }
      as = warp_sum(as) + gate_b[0];
      ar = warp_sum(ar) + gate_b[1];
      gs = 1.0f / (1.0f + expf(-as));
      gr = 1.0f / (1.0f + expf(-ar));
    }
    // m = Z_sp / (Z_sp + lambda Z_race) = 1 / (1 + exp(log(lambda Z_race) - lse))
    const float lz = lam_v * (float)ctot / (float)L;
    const float m = lz > 0.f ? 1.0f / (1.0f + expf(logf(lz) - lse[r])) : 1.0f;
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      y[base + i] = from_f32<T>(gs * m * os[i] + gr * orc[i]);
      if (o_race) o_race[base + i] = from_f32<T>(orc[i]);
    }
    if (ctot_out && lane == 0) ctot_out[r] = ctot;
  }
}

int grid_for_rows(int64_t rows, int warps_per_block) {
  const int64_t b = (rows + warps_per_block - 1) / warps_per_block;
  return (int)(b < 148 * 32 ? b : 148 * 32);
}

template <typename TV, typename CodeT>
cudaError_t build(const Geometry& g, const void* codes, const void* vals, float* sums,
                  int32_t* counts, cudaStream_t s) {
  // slab: `tabs` tables x a d-slice of `dsl` (a multiple of 32) in shared memory
  int dsl = g.d;
  while (dsl > 32 && (size_t)g.NB * (dsl + 1) * 4 > (size_t)kBuildSmemBudget) dsl >>= 1;
  const size_t per_table = (size_t)g.NB * (dsl + 1) * 4;
  if (per_table > (size_t)kBuildSmemBudget) {
    cudaError_t e = cudaMemsetAsync(sums, 0, (size_t)g.BH * g.L * g.NB * g.d * 4, s);
    if (e != cudaSuccess) return e;
    if (counts) {
      e = cudaMemsetAsync(counts, 0, (size_t)g.BH * g.L * g.NB * 4, s);
      if (e != cudaSuccess) return e;
    }
    const int64_t rows = (int64_t)g.BH * g.N;
    race_build_global_kernel<TV, CodeT><<<grid_for_rows(rows, 8), 256, 0, s>>>(
        static_cast<const CodeT*>(codes), static_cast<const TV*>(vals), rows, g.N, g.L, g.NB,
        g.d, sums, counts);
    return cudaGetLastError();
  }
  int tabs = (int)(kBuildSmemBudget / per_table);
  if (tabs > g.L) tabs = g.L;
  const int groups = (g.L + tabs - 1) / tabs;
  const size_t smem = (size_t)tabs * g.NB * dsl * 4 + (size_t)tabs * g.NB * 4;
  cudaError_t e = cudaFuncSetAttribute(race_build_smem_kernel<TV, CodeT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(groups * (g.d / dsl), g.BH);
  race_build_smem_kernel<TV, CodeT><<<grid, 512, smem, s>>>(
      static_cast<const CodeT*>(codes), static_cast<const TV*>(vals), g.N, g.L, g.NB, g.d, tabs,
      dsl, sums, counts);
  return cudaGetLastError();
}

template <typename CodeT>
cudaError_t gather_sum(const Geometry& g, const void* codes, const float* tables, float* out,
                       cudaStream_t s) {
  const int64_t rows = (int64_t)g.BH * g.N;
  const int grid = grid_for_rows(rows, 8);
  const CodeT* c = static_cast<const CodeT*>(codes);
  switch (g.d / 32) {
    case 1: race_gather_sum_kernel<CodeT, 1><<<grid, 256, 0, s>>>(c, tables, rows, g.N, g.L, g.NB, g.d, out); break;
    case 2: race_gather_sum_kernel<CodeT, 2><<<grid, 256, 0, s>>>(c, tables, rows, g.N, g.L, g.NB, g.d, out); break;
    default: race_gather_sum_kernel<CodeT, 4><<<grid, 256, 0, s>>>(c, tables, rows, g.N, g.L, g.NB, g.d, out); break;
  }
  return cudaGetLastError();
}

template <typename T, typename CodeT>
cudaError_t fuse_fwd(const Geometry& g, const void* q, const void* rcode_q, const float* sums,
                     const int32_t* counts, const void* o_sp, const float* lse,
                     const float* gate_w, const float* gate_b, const float* lam, void* y,
                     void* o_race, int32_t* ctot, cudaStream_t s, int gate_fixed, float gs,
                     float gr) {
  const int64_t rows = (int64_t)g.BH * g.N;
  const int grid = grid_for_rows(rows, 8);
#define ELSAA_FUSE(VEC)                                                                        \
  race_fuse_fwd_kernel<T, CodeT, VEC><<<grid, 256, 0, s>>>(                                    \
      static_cast<const T*>(q), static_cast<const CodeT*>(rcode_q), sums, counts,              \
      static_cast<const T*>(o_sp), lse, gate_w, gate_b, gate_fixed, gs, gr, lam, rows, g.N,    \
      g.L, g.NB, g.d, static_cast<T*>(y), static_cast<T*>(o_race), ctot)
  switch (g.d / 32) {
    case 1: ELSAA_FUSE(1); break;
    case 2: ELSAA_FUSE(2); break;
    default: ELSAA_FUSE(4); break;
  }
#undef ELSAA_FUSE
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_race_build(const Geometry& g, const void* codes, const void* vals,
                              bool vals_f32, float* sums, int32_t* counts, cudaStream_t s) {
  if (vals_f32 || !g.bf16)
    return g.rcode_bytes == 1 ? build<float, uint8_t>(g, codes, vals, sums, counts, s)
                              : build<float, uint16_t>(g, codes, vals, sums, counts, s);
  return g.rcode_bytes == 1 ? build<__nv_bfloat16, uint8_t>(g, codes, vals, sums, counts, s)
                            : build<__nv_bfloat16, uint16_t>(g, codes, vals, sums, counts, s);
}

cudaError_t launch_race_gather_sum(const Geometry& g, const void* codes, const float* tables,
                                   float* out, cudaStream_t s) {
  return g.rcode_bytes == 1 ? gather_sum<uint8_t>(g, codes, tables, out, s)
                            : gather_sum<uint16_t>(g, codes, tables, out, s);
}

cudaError_t launch_race_fuse_fwd(const Geometry& g, const void* q, const void* rcode_q,
                                 const float* sums, const int32_t* counts, const void* o_sp,
                                 const float* lse, const float* gate_w, const float* gate_b,
                                 const float* lam, void* y, void* o_race, int32_t* ctot,
                                 cudaStream_t s) {
  const float gs = g.gate_s, gr = g.gate_r;
  const int fixed = g.gate_fixed;
  if (g.bf16)
    return g.rcode_bytes == 1
               ? fuse_fwd<__nv_bfloat16, uint8_t>(g, q, rcode_q, sums, counts, o_sp, lse, gate_w,
                                                  gate_b, lam, y, o_race, ctot, s, fixed, gs, gr)
               : fuse_fwd<__nv_bfloat16, uint16_t>(g, q, rcode_q, sums, counts, o_sp, lse,
                                                   gate_w, gate_b, lam, y, o_race, ctot, s, fixed,
                                                   gs, gr);
  return g.rcode_bytes == 1
             ? fuse_fwd<float, uint8_t>(g, q, rcode_q, sums, counts, o_sp, lse, gate_w, gate_b,
                                        lam, y, o_race, ctot, s, fixed, gs, gr)
             : fuse_fwd<float, uint16_t>(g, q, rcode_q, sums, counts, o_sp, lse, gate_w, gate_b,
                                         lam, y, o_race, ctot, s, fixed, gs, gr);
}

}  // namespace elsaa
