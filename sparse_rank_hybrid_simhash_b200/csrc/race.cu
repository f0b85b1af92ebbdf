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
// Build (race_build_sorted_kernel, described where it is defined): one CTA
// per (unit, table) bucket-sorts the table's keys in shared memory and sums
// each bucket's value rows as one run, into a fixed-point table (exact,
// order-independent).  Shapes it does not fit take a slab build (a block owns
// tables x a 32-wide slice of d in shared memory and streams every key of its
// unit through it with shared-memory atomics) or, for tables too large for
// shared memory, a global-atomic build.
// Gather (race_gather_rows_kernel, race_fuse_rows_kernel): a row per group of
// d / 8 lanes with 16-byte table lines, the row's codes as whole words and
// the next row's codes prefetched; the forward gather is fused with the gates,
// the multiplier and the output.  Other code widths take a warp-per-query
// gather with codes broadcast by shuffle.
#include "common.cuh"
#include "internal.h"

namespace elsaa {
namespace {
ELSAA_DEV uint32_t smem_addr32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
}  // namespace
}  // namespace elsaa

namespace elsaa {
namespace {

constexpr int kBuildSmemBudget = 226 * 1024;

// One CTA owns tables [l0, l0 + nt) restricted to a 32-wide slice of d and
// streams every key of its unit through them in tiles of kBuildKT keys (loaded
// into registers one tile ahead, staged in shared memory).
//
// Sums accumulate in 32-bit fixed point: on B200 a warp-wide 32-bit integer
// shared-memory reduction runs about 4x faster than an fp32 (or 64-bit) one.
// A first pass counts the keys of every bucket (C); with C_max the largest
// count and vmax the unit's largest |value|, the scale 2^S is the largest power
// of two with C_max * (vmax 2^S + 1/2) < 2^31, so no partial sum can overflow.
// Each value is rounded once to a multiple of 2^-S; integer sums are exact and
// order-independent, so every table entry is within count * 2^-(S+1) of the
// exact sum of its values, and the result does not depend on thread timing.
constexpr int kBuildThreads = 1024;
constexpr int kBuildKT = 256;
constexpr int kDsl = 32;
constexpr int kValsPerThread = kBuildKT * kDsl / kBuildThreads;   // 8
constexpr int kCodesPerThreadMax = 8;                             // nt <= 32 over 4 threads per key

struct BuildShape {
  int nt, groups, nds, ntp;
  size_t smem;
};

template <typename TV>
ELSAA_DEV void load_vals8(const TV* src, float* dst);
template <>
ELSAA_DEV void load_vals8<__nv_bfloat16>(const __nv_bfloat16* src, float* dst) {
  const uint4 raw = *reinterpret_cast<const uint4*>(src);   // 8 bf16
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    dst[2 * i] = f.x;
    dst[2 * i + 1] = f.y;
  }
}
template <>
ELSAA_DEV void load_vals8<float>(const float* src, float* dst) {
  const float4 a = *reinterpret_cast<const float4*>(src);
  const float4 b = *reinterpret_cast<const float4*>(src + 4);
  dst[0] = a.x; dst[1] = a.y; dst[2] = a.z; dst[3] = a.w;
  dst[4] = b.x; dst[5] = b.y; dst[6] = b.z; dst[7] = b.w;
}

ELSAA_DEV void red_shared_add_u32(uint32_t addr, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

template <typename TV, typename CodeT>
__global__ void __launch_bounds__(kBuildThreads)
race_build_tiled_kernel(const CodeT* __restrict__ codes, const TV* __restrict__ vals, int N,
                        int L, int NB, int d, int nt_max, int ntp,
                        const float* __restrict__ absmax, float* __restrict__ sums,
                        __nv_bfloat16* __restrict__ gtab, int32_t* __restrict__ counts,
                        uint32_t* __restrict__ err) {
  extern __shared__ int32_t smi[];
  __shared__ int s_cmax;
  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int nds = d / kDsl;
  const int tg = blockIdx.x / nds, dsl = blockIdx.x % nds;
  const int l0 = tg * nt_max, nt = min(L, l0 + nt_max) - l0;
  const int d0 = dsl * kDsl;
  int32_t* tab = smi;                                              // [nt_max][NB][32]
  int32_t* cnt = tab + (size_t)nt_max * NB * kDsl;                 // [nt_max][NB]
  float* vst = reinterpret_cast<float*>(cnt + (((size_t)nt_max * NB + 3) & ~(size_t)3));
  uint16_t* cst = reinterpret_cast<uint16_t*>(vst + kBuildKT * kDsl);   // [KT][ntp]
  for (int i = tid; i < nt * NB * kDsl; i += kBuildThreads) tab[i] = 0;
  for (int i = tid; i < nt * NB; i += kBuildThreads) cnt[i] = 0;
  if (tid == 0) s_cmax = 0;
  __syncthreads();
  const CodeT* cb = codes + (size_t)bh * N * L + l0;
  const TV* vb = vals + (size_t)bh * N * d + d0;

  // pass 1: bucket counts of this CTA's tables (one thread per key)
  for (int key = tid; key < N; key += kBuildThreads) {
    const CodeT* kc = cb + (size_t)key * L;
    for (int t = 0; t < nt; ++t) atomicAdd(cnt + t * NB + (int)kc[t], 1);
  }
  __syncthreads();
  int cm = 0;
  for (int i = tid; i < nt * NB; i += kBuildThreads) cm = max(cm, cnt[i]);
  atomicMax(&s_cmax, cm);
  __syncthreads();
  const float vmax = absmax[bh];
  if (!(vmax < 3.0e38f)) {   // inf or nan among the values
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  int S = 100;
  if (s_cmax > 0 && vmax > 0.f) {
    S = (int)floorf(log2f(2147483000.0f / ((float)s_cmax * vmax))) - 1;
    S = max(-100, min(100, S));
  }
  const float scale = ldexpf(1.0f, S), inv_scale = ldexpf(1.0f, -S);

  // pass 2: fixed-point sums.  Thread tid stages key tid / 4: values [voff, voff + 8)
  // of the d-slice and codes [cq, cq + ncode) of its tables.
  const int vkey = tid >> 2, voff = (tid & 3) * 8;
  const int nq4 = (nt + 3) >> 2, cq = (tid & 3) * nq4;
  const int ncode = max(0, min(nq4, nt - cq));
  float pv[kValsPerThread];
  uint16_t pc[kCodesPerThreadMax];
  auto prefetch = [&](int tile) {
    const int j = tile * kBuildKT + vkey;
    if (j < N) {
      load_vals8<TV>(vb + (size_t)j * d + voff, pv);
      const CodeT* kc = cb + (size_t)j * L + cq;
#pragma unroll
      for (int c = 0; c < kCodesPerThreadMax; ++c)
        if (c < ncode) pc[c] = (uint16_t)kc[c];
    }
  };
  const int ntiles = (N + kBuildKT - 1) / kBuildKT;
  prefetch(0);
  const int w = tid >> 5, lane = tid & 31;
  const uint32_t tab_lane = smem_addr32(tab) + lane * 4;   // this lane's column
  const uint32_t table_bytes = (uint32_t)NB * kDsl * 4;
  for (int tile = 0; tile < ntiles; ++tile) {
    const int kcount = min(kBuildKT, N - tile * kBuildKT);
    __syncthreads();   // the previous tile is fully consumed
#pragma unroll
    for (int i = 0; i < kValsPerThread; i += 4)
      *reinterpret_cast<float4*>(vst + vkey * kDsl + voff + i) =
          make_float4(pv[i], pv[i + 1], pv[i + 2], pv[i + 3]);
#pragma unroll
    for (int c = 0; c < kCodesPerThreadMax; ++c)
      if (c < ncode) cst[vkey * ntp + cq + c] = pc[c];
    __syncthreads();
    if (tile + 1 < ntiles) prefetch(tile + 1);
    // warp w: keys [w * 8, w * 8 + 8) of the tile, two at a time, one row per reduction
    constexpr int kPerWarp = kBuildKT / (kBuildThreads / 32);
    const int kbeg = w * kPerWarp, kend = min(kbeg + kPerWarp, kcount);
    for (int key = kbeg; key < kend; key += 2) {
      const bool two_keys = key + 1 < kend;
      const uint32_t xa = (uint32_t)__float2int_rn(vst[key * kDsl + lane] * scale);
      const uint32_t xb =
          two_keys ? (uint32_t)__float2int_rn(vst[(key + 1) * kDsl + lane] * scale) : 0u;
      const uint16_t* ka = cst + key * ntp;
      const uint16_t* kb2 = cst + (two_keys ? key + 1 : key) * ntp;
      uint32_t tbase = tab_lane;
      for (int t = 0; t < nt; ++t, tbase += table_bytes) {
        const uint32_t ca = ka[t], cbk = kb2[t];
        red_shared_add_u32(tbase + ca * (kDsl * 4), xa);
        if (two_keys) red_shared_add_u32(tbase + cbk * (kDsl * 4), xb);
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < nt * NB * kDsl; i += kBuildThreads) {
    const int tb = i / kDsl, e = i % kDsl;
    const size_t o = ((size_t)bh * L + l0) * NB * d + (size_t)tb * d + d0 + e;
    const float val = (float)tab[i] * inv_scale;
    if (sums) sums[o] = val;
    if (gtab) gtab[o] = __float2bfloat16_rn(val);
  }
  if (counts != nullptr && dsl == 0)
    for (int i = tid; i < nt * NB; i += kBuildThreads)
      counts[((size_t)bh * L + l0) * NB + i] = cnt[i];
}

// The same build with the key stream as a 4-stage cp.async pipeline: tiles of
// kPipeKT keys (raw values of the CTA's d-slice and the codes of its tables)
// land in a ring of shared-memory stages while earlier tiles are reduced, with
// one barrier per tile.  Keys past N are zero-filled and add nothing.  Needs
// the codes of a CTA's tables to be 4-byte aligned per key.
constexpr int kPipeKT = 128;
constexpr int kPipeStages = 4;

ELSAA_DEV void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
ELSAA_DEV void cp_async16b(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// NT > 0 fixes the tables per CTA at compile time (unrolled, table bases hoisted).
template <typename TV, typename CodeT, int NT>
__global__ void __launch_bounds__(kBuildThreads)
race_build_pipe_kernel(const CodeT* __restrict__ codes, const TV* __restrict__ vals, int N,
                       int L, int NB, int d, int nt_max, const float* __restrict__ absmax,
                       float* __restrict__ sums, __nv_bfloat16* __restrict__ gtab,
                       int32_t* __restrict__ counts, uint32_t* __restrict__ err) {
  constexpr int VB = kDsl * (int)sizeof(TV);   // value bytes of one key's d-slice
  extern __shared__ int32_t smi[];
  __shared__ int s_cmax;
  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int nds = d / kDsl;
  const int tg = blockIdx.x / nds, dsl = blockIdx.x % nds;
  const int l0 = tg * nt_max, nt = min(L, l0 + nt_max) - l0;
  const int d0 = dsl * kDsl;
  const int CB = nt_max * (int)sizeof(CodeT);    // code bytes of one key (multiple of 4)
  int32_t* tab = smi;                                              // [nt_max][NB][32]
  int32_t* cnt = tab + (size_t)nt_max * NB * kDsl;                 // [nt_max][NB]
  uint8_t* stages = reinterpret_cast<uint8_t*>(cnt + (((size_t)nt_max * NB + 3) & ~(size_t)3));
  const int stage_bytes = kPipeKT * (VB + CB);
  for (int i = tid; i < nt * NB * kDsl; i += kBuildThreads) tab[i] = 0;
  for (int i = tid; i < nt * NB; i += kBuildThreads) cnt[i] = 0;
  if (tid == 0) s_cmax = 0;
  __syncthreads();
  const CodeT* cb = codes + (size_t)bh * N * L + l0;
  const TV* vb = vals + (size_t)bh * N * d + d0;

  // pass 1: bucket counts of this CTA's tables (one thread per key)
  for (int key = tid; key < N; key += kBuildThreads) {
    const CodeT* kc = cb + (size_t)key * L;
    for (int t = 0; t < nt; ++t) atomicAdd(cnt + t * NB + (int)kc[t], 1);
  }
  __syncthreads();
  int cm = 0;
  for (int i = tid; i < nt * NB; i += kBuildThreads) cm = max(cm, cnt[i]);
  atomicMax(&s_cmax, cm);
  __syncthreads();
  const float vmax = absmax[bh];
  if (!(vmax < 3.0e38f)) {
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  int S = 100;
  if (s_cmax > 0 && vmax > 0.f) {
    S = (int)floorf(log2f(2147483000.0f / ((float)s_cmax * vmax))) - 1;
    S = max(-100, min(100, S));
  }
  const float scale = ldexpf(1.0f, S), inv_scale = ldexpf(1.0f, -S);

  // pass 2: fixed-point sums over a cp.async ring of key tiles
  const uint32_t st0 = smem_addr32(stages);
  const int ntiles = (N + kPipeKT - 1) / kPipeKT;
  auto issue = [&](int tile, int slot) {
    const int k0 = tile * kPipeKT;
    const uint32_t sv = st0 + slot * stage_bytes;
    for (int c = tid; c < kPipeKT * (VB / 16); c += kBuildThreads) {
      const int key = c / (VB / 16), part = c % (VB / 16);
      const int j = k0 + key;
      const bool in = j < N;
      cp_async16b(sv + key * VB + part * 16,
                  vb + (size_t)(in ? j : 0) * d + part * (16 / (int)sizeof(TV)), in ? 16 : 0);
    }
    for (int c = tid; c < kPipeKT * (CB / 4); c += kBuildThreads) {
      const int key = c / (CB / 4), part = c % (CB / 4);
      const int j = k0 + key;
      const bool in = j < N;
      cp_async4(sv + kPipeKT * VB + key * CB + part * 4,
                reinterpret_cast<const uint8_t*>(cb + (size_t)(in ? j : 0) * L) + part * 4,
                in ? 4 : 0);
    }
  };
  for (int t = 0; t < kPipeStages - 1; ++t) {
    if (t < ntiles) issue(t, t);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  const int w = tid >> 5, lane = tid & 31;
  const uint32_t tab_lane = smem_addr32(tab) + lane * 4;
  const uint32_t table_bytes = (uint32_t)NB * kDsl * 4;
  for (int t = 0; t < ntiles; ++t) {
    asm volatile("cp.async.wait_group %0;" ::"n"(kPipeStages - 2) : "memory");
    __syncthreads();   // tile t is in; every thread is done with tile t - 1
    {
      const int tn = t + kPipeStages - 1;
      if (tn < ntiles) issue(tn, tn % kPipeStages);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    const uint8_t* sv = stages + (t % kPipeStages) * stage_bytes;
    // warp w: keys w and w + 32 of each 64-key half, two keys in flight
    for (int key = w; key < kPipeKT; key += 2 * (kBuildThreads / 32)) {
      const int key2 = key + kBuildThreads / 32;
      const float xa = to_f32(reinterpret_cast<const TV*>(sv + key * VB)[lane]);
      const float xb = to_f32(reinterpret_cast<const TV*>(sv + key2 * VB)[lane]);
      const uint32_t qa = (uint32_t)__float2int_rn(xa * scale);
      const uint32_t qb = (uint32_t)__float2int_rn(xb * scale);
      // codes in 32-bit words: 4 u8 codes or 2 u16 codes per load; a code is
      // pulled out with one byte permute and scaled into an address with one
      // multiply-add
      constexpr int PER = 4 / (int)sizeof(CodeT);
      const uint32_t* ka = reinterpret_cast<const uint32_t*>(sv + kPipeKT * VB + key * CB);
      const uint32_t* kb2 = reinterpret_cast<const uint32_t*>(sv + kPipeKT * VB + key2 * CB);
      if constexpr (NT > 0) {
#pragma unroll
        for (int tw = 0; tw < NT; tw += PER) {
          const uint32_t wa = ka[tw / PER], wb = kb2[tw / PER];
#pragma unroll
          for (int e = 0; e < PER; ++e) {
            const uint32_t sel = sizeof(CodeT) == 1 ? (0x4440u | e) : (e ? 0x4432u : 0x4410u);
            const uint32_t tb = tab_lane + (uint32_t)(tw + e) * table_bytes;
            red_shared_add_u32(tb + __byte_perm(wa, 0, sel) * (kDsl * 4), qa);
            red_shared_add_u32(tb + __byte_perm(wb, 0, sel) * (kDsl * 4), qb);
          }
        }
      } else {
        uint32_t tbase = tab_lane;
        for (int tw = 0; tw < nt; tw += PER) {   // nt is a multiple of PER
          const uint32_t wa = ka[tw / PER], wb = kb2[tw / PER];
#pragma unroll
          for (int e = 0; e < PER; ++e, tbase += table_bytes) {
            const uint32_t sel = sizeof(CodeT) == 1 ? (0x4440u | e) : (e ? 0x4432u : 0x4410u);
            red_shared_add_u32(tbase + __byte_perm(wa, 0, sel) * (kDsl * 4), qa);
            red_shared_add_u32(tbase + __byte_perm(wb, 0, sel) * (kDsl * 4), qb);
          }
        }
      }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  for (int i = tid; i < nt * NB * kDsl; i += kBuildThreads) {
    const int tb = i / kDsl, e = i % kDsl;
    const size_t o = ((size_t)bh * L + l0) * NB * d + (size_t)tb * d + d0 + e;
    const float val = (float)tab[i] * inv_scale;
    if (sums) sums[o] = val;
    if (gtab) gtab[o] = __float2bfloat16_rn(val);
  }
  if (counts != nullptr && dsl == 0)
    for (int i = tid; i < nt * NB; i += kBuildThreads)
      counts[((size_t)bh * L + l0) * NB + i] = cnt[i];
}

// Largest |value| of every unit (an upper bound for the fixed-point scale):
// absmax must be zeroed; non-negative floats order like their bit patterns.
template <typename TV>
__global__ void __launch_bounds__(256)
unit_absmax_kernel(const TV* __restrict__ vals, int64_t per_unit, float* __restrict__ absmax) {
  const int bh = blockIdx.y;
  const TV* v = vals + (size_t)bh * per_unit;
  float m = 0.f;
  const int64_t step = (int64_t)gridDim.x * blockDim.x * 8;
  int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  // four independent 8-value loads in flight per thread
  for (; i + 3 * step < per_unit; i += 4 * step) {
    float x[4][8];
#pragma unroll
    for (int u = 0; u < 4; ++u) load_vals8<TV>(v + i + u * step, x[u]);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(x[u][e]));
  }
  for (; i < per_unit; i += step) {
    float x[8];
    load_vals8<TV>(v + i, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(x[e]));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<int*>(absmax) + bh, __float_as_int(m));
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

// Gathers read bf16 copies of the tables: QL = d / 8 lanes per query (each
// lane owns 8 consecutive values and loads 16 bytes per table row), 32 / QL
// queries per warp.  The query's codes are loaded QL at a time, one per lane,
// and broadcast inside the lane group.
template <int QL>
ELSAA_DEV float group_sum(float v) {
#pragma unroll
  for (int o = QL / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
template <int QL>
ELSAA_DEV int group_sum_i(int v) {
#pragma unroll
  for (int o = QL / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 16 bytes as 8 bf16 or 4 fp32 values, and back.
ELSAA_DEV void unpack16(uint4 raw, float* v, const __nv_bfloat16*) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
ELSAA_DEV void unpack16(uint4 raw, float* v, const float*) {
  v[0] = __uint_as_float(raw.x); v[1] = __uint_as_float(raw.y);
  v[2] = __uint_as_float(raw.z); v[3] = __uint_as_float(raw.w);
}
ELSAA_DEV uint4 pack16(const float* v, const __nv_bfloat16*) {
  uint4 raw;
  uint32_t* w = reinterpret_cast<uint32_t*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return raw;
}
ELSAA_DEV uint4 pack16(const float* v, const float*) {
  return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                    __float_as_uint(v[3]));
}

// Adds the 16 bytes at `row` (8 bf16 or 4 fp32 values) to acc; the table line
// is read with the keep-in-L2 policy `pol`.
template <typename TT>
ELSAA_DEV void acc_row(float* acc, const TT* row, uint64_t pol) {
  constexpr int EL = 16 / sizeof(TT);
  float f[EL];
  unpack16(ld16_keep(row, pol), f, row);
#pragma unroll
  for (int i = 0; i < EL; ++i) acc[i] += f[i];
}

// Streaming 16-byte load / store of EL = 16 / sizeof(T) values.
template <typename T>
ELSAA_DEV void load16_stream(const T* p, float* v) { unpack16(ld16_stream(p), v, p); }
template <typename T>
ELSAA_DEV void store16_stream(T* p, const float* v) { st16_stream(p, pack16(v, p)); }

template <typename TT, typename CodeT, int QL>
__global__ void __launch_bounds__(256, 4)
race_gather_sum_kernel(const CodeT* __restrict__ codes, const TT* __restrict__ tables,
                       int64_t rows, int N, int L, int NB, int d, float* __restrict__ out) {
  constexpr int QW = 32 / QL, EL = 16 / sizeof(TT);
  const int lane = threadIdx.x & 31, ql = lane % QL, gbase = lane - ql;
  const uint64_t pol = l2_keep_policy();
  const int64_t first = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * QW;
  const int64_t stride = (int64_t)gridDim.x * (blockDim.x >> 5) * QW;
  for (int64_t r0 = first; r0 < rows; r0 += stride) {
    const int64_t r = r0 + lane / QL;
    const bool valid = r < rows;
    const int64_t rr = valid ? r : rows - 1;
    const int64_t bh = rr / N;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int t0 = 0; t0 < L; t0 += QL) {
      const int mycode = t0 + ql < L ? (int)codes[rr * L + t0 + ql] : 0;
      const int nt = min(QL, L - t0);
#pragma unroll 16
      for (int t = 0; t < nt; ++t) {
        const int b = __shfl_sync(0xffffffffu, mycode, gbase + t);
        acc_row(acc, tables + ((bh * L + t0 + t) * NB + b) * d + ql * EL, pol);
      }
    }
    if (valid) {
      float* o = out + rr * d + ql * EL;
#pragma unroll
      for (int i = 0; i < EL; i += 4) store16_stream(o + i, acc + i);
    }
  }
}

template <typename T>
ELSAA_DEV void load8(const T* p, float* v);
template <>
ELSAA_DEV void load8<float>(const float* p, float* v) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
ELSAA_DEV void load8<__nv_bfloat16>(const __nv_bfloat16* p, float* v) {
  const uint4 raw = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

template <typename T, int EL>
ELSAA_DEV void load_el(const T* p, float* v) {
#pragma unroll
  for (int i = 0; i < EL; ++i) v[i] = to_f32(p[i]);
}
template <>
ELSAA_DEV void load_el<__nv_bfloat16, 8>(const __nv_bfloat16* p, float* v) {
  load8<__nv_bfloat16>(p, v);
}
template <>
ELSAA_DEV void load_el<float, 8>(const float* p, float* v) {
  load8<float>(p, v);
}
template <>
ELSAA_DEV void load_el<float, 4>(const float* p, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}

// T: data type; the tables have the data type too (bf16 copy or fp32 sums).
template <typename T, typename CodeT, int QL>
__global__ void __launch_bounds__(256, 4)
race_fuse_fwd_kernel(const T* __restrict__ q, const CodeT* __restrict__ rcode_q,
                     const T* __restrict__ tables, const int32_t* __restrict__ counts,
                     const T* __restrict__ o_sp, const float* __restrict__ lse,
                     const float* __restrict__ gate_w, const float* __restrict__ gate_b,
                     int gate_fixed, float gs_fixed, float gr_fixed,
                     const float* __restrict__ lam, int64_t rows, int N, int L, int NB, int d,
                     T* __restrict__ y, T* __restrict__ o_race, int32_t* __restrict__ ctot_out) {
  constexpr int QW = 32 / QL, EL = 16 / sizeof(T);
  const int lane = threadIdx.x & 31, ql = lane % QL, gbase = lane - ql;
  const uint64_t pol = l2_keep_policy();
  const float lam_v = *lam;
  float ws8[EL], wr8[EL];
#pragma unroll
  for (int i = 0; i < EL; ++i) ws8[i] = wr8[i] = 0.f;
  float bs = 0.f, br = 0.f;
  if (!gate_fixed) {
    load_el<float, EL>(gate_w + ql * EL, ws8);
    load_el<float, EL>(gate_w + d + ql * EL, wr8);
    bs = gate_b[0];
    br = gate_b[1];
  }
  const int64_t first = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * QW;
  const int64_t stride = (int64_t)gridDim.x * (blockDim.x >> 5) * QW;
  for (int64_t r0 = first; r0 < rows; r0 += stride) {
    const int64_t r = r0 + lane / QL;
    const bool valid = r < rows;
    const int64_t rr = valid ? r : rows - 1;
    const int64_t bh = rr / N;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int ctot = 0;
    for (int t0 = 0; t0 < L; t0 += QL) {
      const int mycode = t0 + ql < L ? (int)rcode_q[rr * L + t0 + ql] : 0;
      if (t0 + ql < L) ctot += counts[(bh * L + t0 + ql) * NB + mycode];
      const int nt = min(QL, L - t0);
#pragma unroll 16
      for (int t = 0; t < nt; ++t) {
        const int b = __shfl_sync(0xffffffffu, mycode, gbase + t);
        acc_row(acc, tables + ((bh * L + t0 + t) * NB + b) * d + ql * EL, pol);
      }
    }
    ctot = group_sum_i<QL>(ctot);
    const float inv = ctot > 0 ? 1.0f / (float)ctot : 0.f;
    const size_t base = (size_t)rr * d + ql * EL;
    float qv[EL], os[EL], orc[EL];
    load16_stream(q + base, qv);
    load16_stream(o_sp + base, os);
#pragma unroll
    for (int i = 0; i < EL; ++i) orc[i] = acc[i] * inv;
    float gs = gs_fixed, gr = gr_fixed;
    if (!gate_fixed) {
      float as = 0.f, ar = 0.f;
#pragma unroll
      for (int i = 0; i < EL; ++i) {
        as += qv[i] * ws8[i];
        ar += qv[i] * wr8[i];
      }
      as = group_sum<QL>(as) + bs;
      ar = group_sum<QL>(ar) + br;
      gs = 1.0f / (1.0f + expf(-as));
      gr = 1.0f / (1.0f + expf(-ar));
    }
    // m = Z_sp / (Z_sp + lambda Z_race) = 1 / (1 + exp(log(lambda Z_race) - lse))
    const float lz = lam_v * (float)ctot / (float)L;
    const float m = lz > 0.f ? 1.0f / (1.0f + expf(logf(lz) - lse[rr])) : 1.0f;
    if (valid) {
      float yv[EL];
#pragma unroll
      for (int i = 0; i < EL; ++i) yv[i] = gs * m * os[i] + gr * orc[i];
      store16_stream(y + base, yv);
      if (o_race) store16_stream(o_race + base, orc);
      if (ctot_out && ql == 0) ctot_out[rr] = ctot;
    }
  }
}

// ---- bucket-sorted build --------------------------------------------------------
//
// One CTA per (unit, table).  A counting sort lists the table's keys bucket
// by bucket: each warp counts its contiguous share of the keys, a scan gives
// every (warp, bucket) its slot range, and the warp scatters its keys through
// its own cursors.  Lane groups then walk equal shares of the list, gather
// each key's value row from global memory (L2-resident for the unit) and add
// it in fp32 until the bucket changes, when the run total goes to the shared
// table as one fixed-point integer per column.
//
// Determinism: a cursor is shared only by the lanes of one warp instruction,
// whose conflicting shared-memory atomics the SM applies in a fixed order, so
// the list is the same on every run and so is every run's fp32 total; run
// totals are rounded once to the grid 2^-S (C_max vmax 2^S <= 2^30, so every
// total fits in int32) and summed as integers, whose order does not matter.

constexpr int kSortedThreads = 1024;
constexpr int kSortedWarps = kSortedThreads / 32;

struct SortedSmem {
  size_t tab, list, codes, whist, bend, misc, total;   // whist: u32 [warps][NB]
};
__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }
__host__ __device__ inline SortedSmem sorted_smem(int N, int NB, int d, int code_bytes) {
  SortedSmem m;
  m.tab = 0;
  m.list = align16(m.tab + (size_t)NB * d * 4);
  m.codes = align16(m.list + (size_t)N * 2);
  m.whist = align16(m.codes + (size_t)N * code_bytes);
  m.bend = align16(m.whist + (size_t)kSortedWarps * NB * 4);
  m.misc = align16(m.bend + (size_t)NB * 4);
  m.total = m.misc + 256;   // [0] C_max, [1] bad code, [16..48) warp sums of the scan
  return m;
}

// a += b on two fp32 lanes at once
ELSAA_DEV void add_f32x2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 x, y;\n\t"
      "mov.b64 x, {%0, %1};\n\t"
      "mov.b64 y, {%2, %3};\n\t"
      "add.rn.f32x2 x, x, y;\n\t"
      "mov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}
// acc += a row's 8 bf16 values by mixed-precision adds (bf16 operand, fp32
// accumulator: the sums of converting first, in fewer instructions)
ELSAA_DEV void add_row(float* acc, uint4 raw, const __nv_bfloat16*) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %0;\n\t"
        "add.rn.f32.bf16 %1, hi, %1;\n\t}"
        : "+f"(acc[2 * i]), "+f"(acc[2 * i + 1])
        : "r"(w[i]));
}
ELSAA_DEV void add_row(float* acc, uint4 raw, const float*) {
  add_f32x2(acc[0], acc[1], __uint_as_float(raw.x), __uint_as_float(raw.y));
  add_f32x2(acc[2], acc[3], __uint_as_float(raw.z), __uint_as_float(raw.w));
}

// codes_t: table-major codes [BH][L][N]; grid (L, BH); NB buckets.
template <typename TV, typename CodeT>
__global__ void __launch_bounds__(kSortedThreads, 1)
race_build_sorted_kernel(const CodeT* __restrict__ codes_t, const TV* __restrict__ vals, int N,
                         int L, int NB, int d, const float* __restrict__ absmax,
                         float* __restrict__ sums, __nv_bfloat16* __restrict__ gtab,
                         int32_t* __restrict__ counts, uint32_t* __restrict__ err) {
  constexpr int EL = 16 / (int)sizeof(TV);
  extern __shared__ __align__(16) uint8_t sm[];
  const SortedSmem lay = sorted_smem(N, NB, d, (int)sizeof(CodeT));
  int32_t* tab = reinterpret_cast<int32_t*>(sm + lay.tab);          // [NB][d] fixed point
  uint16_t* list = reinterpret_cast<uint16_t*>(sm + lay.list);      // keys, bucket by bucket
  CodeT* csm = reinterpret_cast<CodeT*>(sm + lay.codes);            // [N] this table's codes
  uint32_t* whist = reinterpret_cast<uint32_t*>(sm + lay.whist);    // [warps][NB]
  int32_t* bend = reinterpret_cast<int32_t*>(sm + lay.bend);        // [NB] end of each bucket
  int32_t* misc = reinterpret_cast<int32_t*>(sm + lay.misc);        // [0] C_max, [1] bad code
  int32_t* wsum = misc + 16;                                        // [32] scan warp sums
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = blockIdx.x, bh = blockIdx.y;
  const CodeT* ct = codes_t + ((size_t)bh * L + t) * N;
  // warp w owns keys [k0, k1)
  const int k0 = (int)((int64_t)N * warp / kSortedWarps);
  const int k1 = (int)((int64_t)N * (warp + 1) / kSortedWarps);
  uint32_t* wh = whist + (size_t)warp * NB;

  // the table's codes to shared memory (16-byte copies when aligned)
  {
    const size_t bytes = (size_t)N * sizeof(CodeT);
    if (((reinterpret_cast<uintptr_t>(ct) | bytes) & 15u) == 0) {
      const uint4* src = reinterpret_cast<const uint4*>(ct);
      uint4* dst = reinterpret_cast<uint4*>(csm);
      for (int i = tid; i < (int)(bytes / 16); i += kSortedThreads) dst[i] = __ldcs(src + i);
    } else {
      for (int i = tid; i < N; i += kSortedThreads) csm[i] = ct[i];
    }
  }
  for (int i = tid; i < NB * d; i += kSortedThreads) tab[i] = 0;
  for (int i = tid; i < kSortedWarps * NB; i += kSortedThreads) whist[i] = 0;
  if (tid < 2) misc[tid] = 0;
  __syncthreads();

  // per-warp bucket counts (warp-private counters)
  for (int j = k0 + lane; j < k1; j += 32) {
    const int c = (int)csm[j];
    if (c < NB) atomicAdd(wh + c, 1u);
    else misc[1] = 1;
  }
  __syncthreads();

  // bucket totals, their exclusive scan, and each warp's starting slot
  {
    int c = 0;
    if (tid < NB)
      for (int w = 0; w < kSortedWarps; ++w) c += (int)whist[w * NB + tid];
    int x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    int cm = c;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cm = max(cm, __shfl_xor_sync(0xffffffffu, cm, o));
    if (lane == 0) atomicMax(misc, cm);
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    if (tid < NB) {
      uint32_t run = (uint32_t)(before + x - c);
      bend[tid] = before + x;
      for (int w = 0; w < kSortedWarps; ++w) {
        const uint32_t h = whist[w * NB + tid];
        whist[w * NB + tid] = run;
        run += h;
      }
      if (counts) counts[((size_t)bh * L + t) * NB + tid] = c;
    }
  }
  __syncthreads();
  if (misc[1] != 0) {
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  // scatter through the warp-private cursors: only lanes of one warp
  // instruction share a cursor
  for (int j = k0 + lane; j < k1; j += 32) list[atomicAdd(wh + (int)csm[j], 1u)] = (uint16_t)j;
  const float vmax = absmax[bh];
  if (!(vmax < 3.0e38f)) {
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  __syncthreads();
  const int cmax = misc[0];
  int S = 0;
  if (cmax > 0 && vmax > 0.f)
    S = max(-100, min(100, (int)floorf(log2f(1073741824.0f / ((float)cmax * vmax)))));
  const float scale = ldexpf(1.0f, S), inv_scale = ldexpf(1.0f, -S);

  // lane groups of QL lanes walk equal shares [p0, p1) of the list
  const int QL = d / EL;
  const int groups = kSortedThreads / QL;
  const int g = tid / QL, ql = tid % QL;
  const int p0 = (int)((int64_t)N * g / groups), p1 = (int)((int64_t)N * (g + 1) / groups);
  const TV* vb = vals + (size_t)bh * N * d + ql * EL;
  float acc[EL];
#pragma unroll
  for (int e = 0; e < EL; ++e) acc[e] = 0.f;
  // the bucket holding position p0: the first b with bend[b] > p0
  int b = 0;
  if (p0 < p1) {
    int lo = 0, hi = NB - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (bend[mid] > p0) hi = mid;
      else lo = mid + 1;
    }
    b = lo;
  }
  int b_end = p0 < p1 ? bend[b] : 0;
  bool any = false;
  auto flush = [&]() {
    if (any) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(tab + (size_t)b * d + ql * EL);
#pragma unroll
      for (int e = 0; e < EL; ++e) {
        atomicAdd(dst + e, (uint32_t)__float2int_rn(acc[e] * scale));
        acc[e] = 0.f;
      }
    }
    any = false;
  };
  auto step = [&](int pos, uint4 raw) {
    if (pos >= b_end) {
      flush();
      do b_end = bend[++b]; while (pos >= b_end);
    }
    add_row(acc, raw, vb);
    any = true;
  };
  auto row = [&](int key) { return __ldg(reinterpret_cast<const uint4*>(vb + (size_t)key * d)); };
  int p = p0;
  for (; p < p1 && (p & 3) != 0; ++p) step(p, row(list[p]));
  for (; p + 4 <= p1; p += 4) {
    const uint2 k4 = *reinterpret_cast<const uint2*>(list + p);   // four u16 keys
    const uint4 r0 = row((int)(k4.x & 0xFFFFu)), r1 = row((int)(k4.x >> 16));
    const uint4 r2 = row((int)(k4.y & 0xFFFFu)), r3 = row((int)(k4.y >> 16));
    step(p, r0);
    step(p + 1, r1);
    step(p + 2, r2);
    step(p + 3, r3);
  }
  for (; p < p1; ++p) step(p, row(list[p]));
  flush();
  __syncthreads();

  const size_t o0 = ((size_t)bh * L + t) * NB * d;
  for (int i = tid * 4; i < NB * d; i += kSortedThreads * 4) {
    const int4 v4 = *reinterpret_cast<const int4*>(tab + i);
    const float f0 = (float)v4.x * inv_scale, f1 = (float)v4.y * inv_scale;
    const float f2 = (float)v4.z * inv_scale, f3 = (float)v4.w * inv_scale;
    if (sums) *reinterpret_cast<float4*>(sums + o0 + i) = make_float4(f0, f1, f2, f3);
    if (gtab) {
      const __nv_bfloat162 h0 = __floats2bfloat162_rn(f0, f1), h1 = __floats2bfloat162_rn(f2, f3);
      uint2 w2;
      w2.x = *reinterpret_cast<const uint32_t*>(&h0);
      w2.y = *reinterpret_cast<const uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(gtab + o0 + i) = w2;
    }
  }
}

// ---- segmented bucket-sorted build (long sequences, large tables) ------------
//
// For shapes whose table or key list does not fit one CTA's shared memory
// (needle-256k: N = 262144 keys, 1024 buckets x 128 values): one CTA per
// (unit, table, segment of kSegKeys keys) bucket-sorts its segment's keys the
// same way (warp-private counters and cursors, so the list is the same on
// every run), sums each bucket's run of value rows in fp32 registers, rounds
// the run total to the grid 2^-S and adds it, as an integer, into a zeroed
// int32 table in global memory (the fp32 table's bytes).  S is chosen from the
// table's largest bucket count (from a counting pass) and the unit's largest
// |value| as in the single-CTA build (C_max vmax 2^S <= 2^30): integer sums
// are exact and order-independent, so the table is the same on every run.  A
// last pass turns each table into fp32 (and the bf16 copy) in place.

constexpr int kSegThreads = 1024;
constexpr int kSegWarps = kSegThreads / 32;
constexpr int kSegKeys = 32768;

// whist: [warps][NB] 16-bit counts, then cursors, two to a 32-bit word (a
// warp counts at most seg / warps keys of a bucket and a cursor is at most
// seg <= 32768, so neither half ever carries into the other); after the
// scatter the same bytes hold the lane groups' run totals (stg: d ints per
// group).  The codes are read from global memory where they are counted and
// scattered.
struct SegSmem {
  size_t list, whist, stg, bend, misc, total;
};
__host__ __device__ inline SegSmem seg_smem(int seg, int NB, int /*code_bytes*/) {
  SegSmem m;
  m.list = 0;
  m.whist = align16((size_t)seg * 2);
  m.stg = m.whist;
  const size_t hist = (size_t)kSegWarps * NB * 2, runs = (size_t)kSegThreads * 8 * 4;
  m.bend = align16(m.whist + (hist > runs ? hist : runs));
  m.misc = align16(m.bend + (size_t)NB * 4);
  m.total = m.misc + 256;   // misc: [0] C_max, [1] bad code, [16..48) warp sums of the scan
  return m;
}

// counts[bh][t][b] += the segment's keys in bucket b (counts zeroed first)
template <typename CodeT>
__global__ void __launch_bounds__(256)
race_seg_hist_kernel(const CodeT* __restrict__ codes_t, int N, int L, int NB, int seg,
                     int32_t* __restrict__ counts, uint32_t* __restrict__ err) {
  extern __shared__ int32_t hist[];
  const int t = blockIdx.y, bh = blockIdx.z;
  const int j0 = blockIdx.x * seg, j1 = min(N, j0 + seg);
  const CodeT* ct = codes_t + ((size_t)bh * L + t) * N;
  for (int b = threadIdx.x; b < NB; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  bool bad = false;
  for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
    const int c = (int)ct[j];
    if (c < NB) atomicAdd(hist + c, 1);
    else bad = true;
  }
  if (bad) raise_error(err, ERR_CHECK);
  __syncthreads();
  int32_t* dst = counts + ((size_t)bh * L + t) * NB;
  for (int b = threadIdx.x; b < NB; b += blockDim.x)
    if (hist[b]) atomicAdd(dst + b, hist[b]);
}

// Grid exponent S of one table: C_max vmax 2^S <= 2^30 (every integer total fits int32).
ELSAA_DEV int seg_grid(int cmax, float vmax) {
  if (cmax > 0 && vmax > 0.f)
    return max(-100, min(100, (int)floorf(log2f(1073741824.0f / ((float)cmax * vmax)))));
  return 0;
}

template <typename TV, typename CodeT>
__global__ void __launch_bounds__(kSegThreads, 1)
race_build_seg_kernel(const CodeT* __restrict__ codes_t, const TV* __restrict__ vals, int N,
                      int L, int NB, int d, int seg, const float* __restrict__ absmax,
                      const int32_t* __restrict__ counts, float* __restrict__ sums,
                      uint32_t* __restrict__ err) {
  constexpr int EL = 16 / (int)sizeof(TV);
  extern __shared__ __align__(16) uint8_t sm[];
  const SegSmem lay = seg_smem(seg, NB, (int)sizeof(CodeT));
  uint16_t* list = reinterpret_cast<uint16_t*>(sm + lay.list);      // segment keys, by bucket
  uint16_t* wh16 = reinterpret_cast<uint16_t*>(sm + lay.whist);     // [warps][NB] counts, cursors
  uint32_t* wh32 = reinterpret_cast<uint32_t*>(sm + lay.whist);     // the same, two to a word
  int32_t* bend = reinterpret_cast<int32_t*>(sm + lay.bend);        // [NB] end of each bucket
  int32_t* misc = reinterpret_cast<int32_t*>(sm + lay.misc);        // [0] C_max, [1] bad code
  int32_t* wsum = misc + 16;                                        // [kSegWarps] scan sums
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // grid (table, segment, unit): the CTAs that run together share a few
  // segments of the unit's value rows, which stay in L2 for all tables
  const int t = blockIdx.x, bh = blockIdx.z;
  const int j0 = blockIdx.y * seg, n = min(N, j0 + seg) - j0;   // keys [j0, j0 + n)
  const CodeT* ct = codes_t + ((size_t)bh * L + t) * N + j0;
  // warp w owns segment keys [k0, k1)
  const int k0 = (int)((int64_t)n * warp / kSegWarps);
  const int k1 = (int)((int64_t)n * (warp + 1) / kSegWarps);
  const int fw = warp * NB;   // this warp's counters: flat 16-bit index fw + bucket
  for (int i = tid; i < (kSegWarps * NB + 1) / 2; i += kSegThreads) wh32[i] = 0;
  if (tid < 2) misc[tid] = 0;
  __syncthreads();
  // the table's largest bucket count (all segments), for the grid 2^-S
  {
    const int32_t* cnt = counts + ((size_t)bh * L + t) * NB;
    int cm = 0;
    for (int b = tid; b < NB; b += kSegThreads) cm = max(cm, cnt[b]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cm = max(cm, __shfl_xor_sync(0xffffffffu, cm, o));
    if (lane == 0) atomicMax(misc, cm);
  }
  for (int j = k0 + lane; j < k1; j += 32) {
    const int c = (int)ct[j];
    if (c < NB) {
      const int f = fw + c;
      atomicAdd(wh32 + (f >> 1), 1u << (16 * (f & 1)));
    } else {
      misc[1] = 1;
    }
  }
  __syncthreads();
  if (misc[1] != 0) {
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  // bucket totals of the segment, their exclusive scan (blocks of 32 buckets
  // per warp, kSegWarps warps per pass), and each warp's starting slot
  int carry = 0;
  for (int b0 = 0; b0 < NB; b0 += kSegThreads) {
    const int b = b0 + tid;
    int c = 0;
    if (b < NB)
      for (int w = 0; w < kSegWarps; ++w) c += (int)wh16[w * NB + b];
    int x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int before = carry;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    int total = 0;
    for (int w = 0; w < kSegWarps; ++w) total += wsum[w];
    if (b < NB) {
      uint32_t run = (uint32_t)(before + x - c);
      bend[b] = before + x;
      for (int w = 0; w < kSegWarps; ++w) {
        const uint32_t h = wh16[w * NB + b];
        wh16[w * NB + b] = (uint16_t)run;
        run += h;
      }
    }
    carry += total;
    __syncthreads();
  }
  // scatter through the warp-private cursors
  for (int j = k0 + lane; j < k1; j += 32) {
    const int f = fw + (int)ct[j];
    const uint32_t sh = 16u * (uint32_t)(f & 1);
    list[(atomicAdd(wh32 + (f >> 1), 1u << sh) >> sh) & 0xFFFFu] = (uint16_t)j;
  }
  const float vmax = absmax[bh];
  if (!(vmax < 3.0e38f)) {
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  __syncthreads();
  const float scale = ldexpf(1.0f, seg_grid(misc[0], vmax));

  // lane groups of QL lanes walk equal shares [p0, p1) of the list
  const int QL = d / EL;
  const int groups = kSegThreads / QL;
  const int gi = tid / QL, ql = tid % QL;
  const int p0 = (int)((int64_t)n * gi / groups), p1 = (int)((int64_t)n * (gi + 1) / groups);
  const TV* vb = vals + ((size_t)bh * N + j0) * d + ql * EL;
  // the fp32 table's bytes hold the int32 sums until the finishing pass
  uint32_t* tb = reinterpret_cast<uint32_t*>(sums + ((size_t)bh * L + t) * NB * d);
  // a run total goes through the group's staging row, so that lane ql adds
  // columns ql, ql + QL, ...: each add instruction of the group covers QL
  // consecutive columns (two 32-byte sectors at QL = 16, not QL sectors)
  int32_t* stg = reinterpret_cast<int32_t*>(sm + lay.stg) + gi * d;
  const unsigned gmask = QL == 32 ? 0xffffffffu : ((1u << QL) - 1u) << (lane & ~(QL - 1));
  float acc[EL];
#pragma unroll
  for (int e = 0; e < EL; ++e) acc[e] = 0.f;
  int b = 0;
  if (p0 < p1) {
    int lo = 0, hi = NB - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (bend[mid] > p0) hi = mid;
      else lo = mid + 1;
    }
    b = lo;
  }
  int b_end = p0 < p1 ? bend[b] : 0;
  bool any = false;
  auto flush = [&]() {
    if (any) {
#pragma unroll
      for (int e = 0; e < EL; ++e) {
        stg[ql * EL + e] = __float2int_rn(acc[e] * scale);
        acc[e] = 0.f;
      }
      __syncwarp(gmask);
      uint32_t* dst = tb + (size_t)b * d + ql;
#pragma unroll
      for (int e = 0; e < EL; ++e) atomicAdd(dst + e * QL, (uint32_t)stg[e * QL + ql]);
      __syncwarp(gmask);   // the row is read before the group's next flush writes it
    }
    any = false;
  };
  auto step = [&](int pos, uint4 raw) {
    if (pos >= b_end) {
      flush();
      do b_end = bend[++b]; while (pos >= b_end);
    }
    add_row(acc, raw, vb);
    any = true;
  };
  auto row = [&](int key) { return __ldg(reinterpret_cast<const uint4*>(vb + (size_t)key * d)); };
  int p = p0;
  for (; p < p1 && (p & 3) != 0; ++p) step(p, row(list[p]));
  for (; p + 4 <= p1; p += 4) {
    const uint2 k4 = *reinterpret_cast<const uint2*>(list + p);
    const uint4 r0 = row((int)(k4.x & 0xFFFFu)), r1 = row((int)(k4.x >> 16));
    const uint4 r2 = row((int)(k4.y & 0xFFFFu)), r3 = row((int)(k4.y >> 16));
    step(p, r0);
    step(p + 1, r1);
    step(p + 2, r2);
    step(p + 3, r3);
  }
  for (; p < p1; ++p) step(p, row(list[p]));
  flush();
}

// One block per (unit, table): the int32 sums become fp32 (scaled by 2^-S of
// that table) in place, and the bf16 copy is written if gtab is non-null.
__global__ void __launch_bounds__(256)
race_seg_finish_kernel(float* __restrict__ sums, __nv_bfloat16* __restrict__ gtab,
                       const int32_t* __restrict__ counts, const float* __restrict__ absmax,
                       int L, int NB, int d) {
  __shared__ int s_cmax;
  const int t = blockIdx.x, bh = blockIdx.y;
  if (threadIdx.x == 0) s_cmax = 0;
  __syncthreads();
  const int32_t* cnt = counts + ((size_t)bh * L + t) * NB;
  int cm = 0;
  for (int b = threadIdx.x; b < NB; b += blockDim.x) cm = max(cm, cnt[b]);
  cm = __reduce_max_sync(0xffffffffu, cm);
  if ((threadIdx.x & 31) == 0) atomicMax(&s_cmax, cm);
  __syncthreads();
  const float inv_scale = ldexpf(1.0f, -seg_grid(s_cmax, absmax[bh]));
  const size_t o0 = ((size_t)bh * L + t) * NB * d;
  for (int i = threadIdx.x * 4; i < NB * d; i += blockDim.x * 4) {
    const int4 v = *reinterpret_cast<const int4*>(sums + o0 + i);
    const float f0 = (float)v.x * inv_scale, f1 = (float)v.y * inv_scale;
    const float f2 = (float)v.z * inv_scale, f3 = (float)v.w * inv_scale;
    *reinterpret_cast<float4*>(sums + o0 + i) = make_float4(f0, f1, f2, f3);
    if (gtab) {
      const __nv_bfloat162 a = __floats2bfloat162_rn(f0, f1), b = __floats2bfloat162_rn(f2, f3);
      uint2 w;
      w.x = *reinterpret_cast<const uint32_t*>(&a);
      w.y = *reinterpret_cast<const uint32_t*>(&b);
      *reinterpret_cast<uint2*>(gtab + o0 + i) = w;
    }
  }
}

// ---- row-pipelined gathers ---------------------------------------------------
//
// Used when a row's codes are whole 32-bit words (L * code bytes % 4 == 0).
// A row is served by QL lanes; lane ql of the group holds the row's code
// words ql, ql + QL, ... (WPL at most), loaded with one access each, and the
// next row's words are fetched while this row's table lines are gathered, so
// every gather of a row is independent of any load issued in the same pass.

template <typename CodeT, int QL, int WPL>
ELSAA_DEV void load_row_codes(const CodeT* row, int W, int ql, uint32_t (&w)[WPL]) {
  const uint32_t* p = reinterpret_cast<const uint32_t*>(row);
#pragma unroll
  for (int i = 0; i < WPL; ++i) {
    const int wi = ql + i * QL;
    w[i] = wi < W ? __ldcs(p + wi) : 0u;
  }
}

template <typename CodeT>
ELSAA_DEV int code_of(uint32_t word, int e) {
  return sizeof(CodeT) == 1 ? (int)((word >> (8 * e)) & 0xFFu) : (int)((word >> (16 * e)) & 0xFFFFu);
}

// acc += sum over tables t of tab[t][code_t][ql * EL ...], tab = this unit's
// tables offset by the lane's column slice.  Offsets are 32-bit (a unit's
// tables are far below 4 GB): table t starts t * table_bytes in, and a
// bucket's row is code << row_shift further.
ELSAA_DEV void add_lines(float* acc, uint4 raw, const __nv_bfloat16*) {
  const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    add_f32x2(acc[2 * i], acc[2 * i + 1], __uint_as_float(w4[i] << 16),
              __uint_as_float(w4[i] & 0xFFFF0000u));
}
ELSAA_DEV void add_lines(float* acc, uint4 raw, const float*) {
  add_f32x2(acc[0], acc[1], __uint_as_float(raw.x), __uint_as_float(raw.y));
  add_f32x2(acc[2], acc[3], __uint_as_float(raw.z), __uint_as_float(raw.w));
}

template <typename TT, typename CodeT, int QL, int WPL>
ELSAA_DEV void gather_row(const TT* tab, const uint32_t (&w)[WPL], int L, uint32_t table_bytes,
                          int row_shift, int gbase, uint64_t pol, float* acc) {
  constexpr int PER = 4 / (int)sizeof(CodeT);
  const char* base = reinterpret_cast<const char*>(tab);
  uint32_t toff = 0;
#pragma unroll
  for (int i = 0; i < WPL; ++i) {
#pragma unroll
    for (int sl = 0; sl < QL; ++sl) {
      const int t0 = (i * QL + sl) * PER;
      if (t0 < L) {
        const uint32_t word = __shfl_sync(0xffffffffu, w[i], gbase + sl);
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          const uint32_t code =
              sizeof(CodeT) == 1 ? __byte_perm(word, 0, 0x4440u | (uint32_t)e)
                                 : __byte_perm(word, 0, e ? 0x4432u : 0x4410u);
          add_lines(acc, ld16_keep(base + toff + (code << row_shift), pol), tab);
          toff += table_bytes;
        }
      }
    }
  }
}

template <typename TT, typename CodeT, int QL, int WPL>
__global__ void __launch_bounds__(256, 4)
race_gather_rows_kernel(const CodeT* __restrict__ codes, const TT* __restrict__ tables,
                        int64_t rows, int N, int L, int NB, int d, float* __restrict__ out,
                        TT* __restrict__ add_out) {
  constexpr int QW = 32 / QL, EL = 16 / sizeof(TT);
  const int lane = threadIdx.x & 31, ql = lane % QL, gbase = lane - ql;
  const uint64_t pol = l2_keep_policy();
  const int W = L * (int)sizeof(CodeT) / 4;
  const uint32_t table_bytes = (uint32_t)NB * (uint32_t)d * (uint32_t)sizeof(TT);
  const int row_shift = 31 - __clz(d * (int)sizeof(TT));   // d * sizeof is a power of two
  const int64_t first = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * QW;
  const int64_t stride = (int64_t)gridDim.x * (blockDim.x >> 5) * QW;
  uint32_t w[WPL];
  {
    const int64_t r = min(first + lane / QL, rows - 1);
    load_row_codes<CodeT, QL, WPL>(codes + r * L, W, ql, w);
  }
  for (int64_t r0 = first; r0 < rows; r0 += stride) {
    const int64_t r = r0 + lane / QL;
    const bool valid = r < rows;
    const int64_t rr = valid ? r : rows - 1;
    const int64_t bh = rr / N;
    uint32_t wn[WPL];
    load_row_codes<CodeT, QL, WPL>(codes + min(r + stride, rows - 1) * L, W, ql, wn);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    gather_row<TT, CodeT, QL, WPL>(tables + (size_t)bh * L * NB * d + ql * EL, w, L, table_bytes,
                                   row_shift, gbase, pol, acc);
    if (valid) {
      if (add_out) {   // add_out[row] += sum, in the data dtype
        TT* o = add_out + rr * d + ql * EL;
        float cur[EL];
        unpack16(*reinterpret_cast<const uint4*>(o), cur, o);
#pragma unroll
        for (int i = 0; i < EL; ++i) cur[i] += acc[i];
        *reinterpret_cast<uint4*>(o) = pack16(cur, o);
      } else {
        float* o = out + rr * d + ql * EL;
#pragma unroll
        for (int i = 0; i < EL; i += 4) store16_stream(o + i, acc + i);
      }
    }
#pragma unroll
    for (int i = 0; i < WPL; ++i) w[i] = wn[i];
  }
}

template <typename T, typename CodeT, int QL, int WPL>
__global__ void __launch_bounds__(256, 4)
race_fuse_rows_kernel(const T* __restrict__ q, const CodeT* __restrict__ rcode_q,
                      const T* __restrict__ tables, const int32_t* __restrict__ counts,
                      const T* __restrict__ o_sp, const float* __restrict__ lse,
                      const float* __restrict__ gate_w, const float* __restrict__ gate_b,
                      int gate_fixed, float gs_fixed, float gr_fixed,
                      const float* __restrict__ lam, int64_t rows, int N, int L, int NB, int d,
                      T* __restrict__ y, T* __restrict__ o_race, int32_t* __restrict__ ctot_out) {
  constexpr int QW = 32 / QL, EL = 16 / sizeof(T);
  constexpr int PER = 4 / (int)sizeof(CodeT);
  // gate weights, and a two-row staging ring per warp for the q and O_sp
  // chunks (each lane copies its own 16-byte chunks and reads them back), so
  // neither sits in registers while the table lines are in flight
  __shared__ float s_w[2 * 128];
  __shared__ __align__(16) uint4 s_stage[8][2][2][32];
  const int lane = threadIdx.x & 31, ql = lane % QL, gbase = lane - ql, wi = threadIdx.x >> 5;
  const uint64_t pol = l2_keep_policy();
  const int W = L * (int)sizeof(CodeT) / 4;
  const uint32_t table_bytes = (uint32_t)NB * (uint32_t)d * (uint32_t)sizeof(T);
  const int row_shift = 31 - __clz(d * (int)sizeof(T));   // d * sizeof is a power of two
  const float lam_v = *lam;
  const float inv_L = 1.0f / (float)L;
  for (int i = threadIdx.x; i < 2 * d; i += blockDim.x) s_w[i] = gate_fixed ? 0.f : gate_w[i];
  const float bs = gate_fixed ? 0.f : gate_b[0], br = gate_fixed ? 0.f : gate_b[1];
  __syncthreads();
  const int64_t first = ((int64_t)blockIdx.x * (blockDim.x >> 5) + wi) * QW;
  const int64_t stride = (int64_t)gridDim.x * (blockDim.x >> 5) * QW;
  auto stage = [&](int64_t r0, int buf) {
    const int64_t rr = min(r0 + lane / QL, rows - 1);
    const size_t base = (size_t)rr * d + ql * EL;
    cp_async16b(smem_addr32(&s_stage[wi][buf][0][lane]), q + base, 16);
    cp_async16b(smem_addr32(&s_stage[wi][buf][1][lane]), o_sp + base, 16);
  };
  uint32_t w[WPL];
  {
    const int64_t r = min(first + lane / QL, rows - 1);
    load_row_codes<CodeT, QL, WPL>(rcode_q + r * L, W, ql, w);
  }
  if (first < rows) stage(first, 0);
  asm volatile("cp.async.commit_group;" ::: "memory");
  int buf = 0;
  for (int64_t r0 = first; r0 < rows; r0 += stride, buf ^= 1) {
    const int64_t r = r0 + lane / QL;
    const bool valid = r < rows;
    const int64_t rr = valid ? r : rows - 1;
    const int64_t bh = rr / N;
    const size_t base = (size_t)rr * d + ql * EL;
    // the next row's q / O_sp chunks and codes go out before this row's gathers
    if (r0 + stride < rows) stage(r0 + stride, buf ^ 1);
    asm volatile("cp.async.commit_group;" ::: "memory");
    const float lse_r = lse[rr];
    uint32_t wn[WPL];
    load_row_codes<CodeT, QL, WPL>(rcode_q + min(r + stride, rows - 1) * L, W, ql, wn);
    // Ctot: this lane's words' bucket counts
    int ctot = 0;
    const int32_t* cnt = counts + (size_t)bh * L * NB;
#pragma unroll
    for (int i = 0; i < WPL; ++i) {
      const int wd = ql + i * QL;
      if (wd < W) {
#pragma unroll
        for (int e = 0; e < PER; ++e) ctot += cnt[(size_t)(wd * PER + e) * NB + code_of<CodeT>(w[i], e)];
      }
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    gather_row<T, CodeT, QL, WPL>(tables + (size_t)bh * L * NB * d + ql * EL, w, L, table_bytes,
                                  row_shift, gbase, pol, acc);
    ctot = group_sum_i<QL>(ctot);
    const float inv = ctot > 0 ? __fdividef(1.0f, (float)ctot) : 0.f;
    asm volatile("cp.async.wait_group 1;" ::: "memory");   // this row's chunks are in
    float qv[EL], os[EL], orc[EL];
    unpack16(s_stage[wi][buf][0][lane], qv, q);
    unpack16(s_stage[wi][buf][1][lane], os, o_sp);
#pragma unroll
    for (int i = 0; i < EL; ++i) orc[i] = acc[i] * inv;
    float gs = gs_fixed, gr = gr_fixed;
    if (!gate_fixed) {
      float as = 0.f, ar = 0.f;
#pragma unroll
      for (int i = 0; i < EL; ++i) {
        as += qv[i] * s_w[ql * EL + i];
        ar += qv[i] * s_w[d + ql * EL + i];
      }
      as = group_sum<QL>(as) + bs;
      ar = group_sum<QL>(ar) + br;
      gs = __fdividef(1.0f, 1.0f + __expf(-as));
      gr = __fdividef(1.0f, 1.0f + __expf(-ar));
    }
    // m = Z_sp / (Z_sp + lambda Z_race) = 1 / (1 + exp(log(lambda Z_race) - lse))
    const float lz = lam_v * (float)ctot * inv_L;
    const float m = lz > 0.f ? __fdividef(1.0f, 1.0f + __expf(__logf(lz) - lse_r)) : 1.0f;
    if (valid) {
      float yv[EL];
#pragma unroll
      for (int i = 0; i < EL; ++i) yv[i] = gs * m * os[i] + gr * orc[i];
      store16_stream(y + base, yv);
      if (o_race) store16_stream(o_race + base, orc);
      if (ctot_out && ql == 0) ctot_out[rr] = ctot;
    }
#pragma unroll
    for (int i = 0; i < WPL; ++i) w[i] = wn[i];
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

__global__ void to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                               int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

int grid_for_rows(int64_t rows, int warps_per_block) {
  const int64_t b = (rows + warps_per_block - 1) / warps_per_block;
  return (int)(b < 148 * 32 ? b : 148 * 32);
}

BuildShape build_shape(const Geometry& g) {
  BuildShape b;
  const size_t stage = (size_t)kBuildKT * kDsl * 4;
  const size_t per_table = (size_t)g.NB * (kDsl + 1) * 4 + (size_t)kBuildKT * 2;
  const size_t budget = (size_t)kBuildSmemBudget - stage - 64;
  int nt_max = (int)(budget / per_table);
  if (nt_max > g.L) nt_max = g.L;
  if (nt_max > 4 * kCodesPerThreadMax) nt_max = 4 * kCodesPerThreadMax;   // codes per thread bound
  b.nds = g.d / kDsl;
  // Choose the tables per CTA: every CTA streams all N keys, paying about one
  // pass over its values plus two cycles per table reduction per key; CTAs run
  // one per SM in waves of 148, so minimise waves x (2 nt + 1).
  int best = nt_max;
  long long best_cost = -1;
  for (int nt = nt_max; nt >= 1; --nt) {
    const long long ctas = (long long)((g.L + nt - 1) / nt) * b.nds * g.BH;
    const long long waves = (ctas + 147) / 148;
    const long long cost = waves * (2 * nt + 1);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = nt;
    }
  }
  const int nt = nt_max >= 1 ? best : 0;
  b.nt = nt;
  b.groups = nt > 0 ? (g.L + nt - 1) / nt : 0;
  b.ntp = (nt + 1) & ~1;
  b.smem = (size_t)nt * g.NB * kDsl * 4 + (((size_t)nt * g.NB + 3) & ~(size_t)3) * 4 + stage +
           (size_t)kBuildKT * b.ntp * 2 + 16;
  return b;
}

template <typename TV, typename CodeT>
cudaError_t build(const Geometry& g, const void* codes, const void* codes_t, const void* vals,
                  const float* absmax,
                  float* sums, bool keep_sums, __nv_bfloat16* gtab, int32_t* counts,
                  int32_t* count_scratch, uint32_t* err, cudaStream_t s) {
  {
    // bucket-sorted build: key indices fit u16, one bucket per thread in the
    // scan, and the whole table plus the key list fit in shared memory
    const SortedSmem m = sorted_smem(g.N, g.NB, g.d, (int)sizeof(CodeT));
    if (g.N <= 65536 && g.NB <= kSortedThreads && m.total <= (size_t)kBuildSmemBudget &&
        g.d % (16 / (int)sizeof(TV)) == 0) {
      auto kernel = race_build_sorted_kernel<TV, CodeT>;
      cudaError_t e =
          cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)m.total);
      if (e != cudaSuccess) return e;
      kernel<<<dim3(g.L, g.BH), kSortedThreads, m.total, s>>>(
          static_cast<const CodeT*>(codes_t), static_cast<const TV*>(vals), g.N, g.L, g.NB, g.d,
          absmax, keep_sums ? sums : nullptr, gtab, counts, err);
      return cudaGetLastError();
    }
  }
  {
    // segmented bucket-sorted build: counts by a counting pass, then one CTA
    // per (unit, table, segment) adding exact run totals into the zeroed table
    const int seg = g.N < kSegKeys ? g.N : kSegKeys;
    const SegSmem m = seg_smem(seg, g.NB, (int)sizeof(CodeT));
    if (g.NB <= 1024 && m.total <= (size_t)kBuildSmemBudget &&
        g.d % (16 / (int)sizeof(TV)) == 0 && (g.d / (16 / (int)sizeof(TV))) <= 32 &&
        sums != nullptr) {
      const size_t tab = (size_t)g.BH * g.L * g.NB;
      // the table's counts (the caller's output, or scratch where it has none)
      int32_t* cnt = counts != nullptr ? counts : count_scratch;
      if (cnt == nullptr) return cudaErrorInvalidValue;
      cudaError_t e = cudaMemsetAsync(cnt, 0, tab * 4, s);
      if (e != cudaSuccess) return e;
      e = cudaMemsetAsync(sums, 0, tab * g.d * 4, s);
      if (e != cudaSuccess) return e;
      const dim3 grid((g.N + seg - 1) / seg, g.L, g.BH);
      race_seg_hist_kernel<CodeT><<<grid, 256, g.NB * 4, s>>>(
          static_cast<const CodeT*>(codes_t), g.N, g.L, g.NB, seg, cnt, err);
      auto kernel = race_build_seg_kernel<TV, CodeT>;
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)m.total);
      if (e != cudaSuccess) return e;
      const dim3 bgrid(g.L, (g.N + seg - 1) / seg, g.BH);
      kernel<<<bgrid, kSegThreads, m.total, s>>>(static_cast<const CodeT*>(codes_t),
                                                static_cast<const TV*>(vals), g.N, g.L, g.NB, g.d,
                                                seg, absmax, cnt, sums, err);
      race_seg_finish_kernel<<<dim3(g.L, g.BH), 256, 0, s>>>(sums, gtab, cnt, absmax, g.L, g.NB,
                                                              g.d);
      return cudaGetLastError();
    }
  }
  const BuildShape b = build_shape(g);
  if (b.nt < 1) {
    // tables too large for shared memory even one at a time: global fp32
    // atomics into `sums`, then the bf16 copy
    const size_t n = (size_t)g.BH * g.L * g.NB * g.d;
    cudaError_t e = cudaMemsetAsync(sums, 0, n * 4, s);
    if (e != cudaSuccess) return e;
    if (counts) {
      e = cudaMemsetAsync(counts, 0, (size_t)g.BH * g.L * g.NB * 4, s);
      if (e != cudaSuccess) return e;
    }
    const int64_t rows = (int64_t)g.BH * g.N;
    race_build_global_kernel<TV, CodeT><<<grid_for_rows(rows, 8), 256, 0, s>>>(
        static_cast<const CodeT*>(codes), static_cast<const TV*>(vals), rows, g.N, g.L, g.NB,
        g.d, sums, counts);
    if (gtab) to_bf16_kernel<<<148 * 8, 256, 0, s>>>(sums, gtab, (int64_t)n);
    return cudaGetLastError();
  }
  // pipelined variant: tables per CTA dividing L, codes 4-byte aligned per key
  if ((g.L * (int)sizeof(CodeT)) % 4 == 0) {
    const int esz_v = (int)sizeof(TV), rb = (int)sizeof(CodeT), step = 4 / rb;
    auto smem_for = [&](int nt) {
      return (size_t)nt * g.NB * kDsl * 4 + (((size_t)nt * g.NB + 3) & ~(size_t)3) * 4 +
             (size_t)kPipeStages * kPipeKT * (kDsl * esz_v + nt * rb) + 16;
    };
    int best = 0;
    long long best_cost = -1;
    for (int nt = step; nt <= g.L && smem_for(nt) <= (size_t)kBuildSmemBudget; nt += step) {
      if (g.L % nt != 0) continue;
      const long long ctas = (long long)(g.L / nt) * b.nds * g.BH;
      const long long cost = (ctas + 147) / 148 * (2 * nt + 1);
      if (best_cost < 0 || cost <= best_cost) {
        best_cost = cost;
        best = nt;
      }
    }
    if (best > 0) {
      const size_t smem = smem_for(best);
      const dim3 grid(g.L / best * b.nds, g.BH);
      auto go = [&](auto kernel) -> cudaError_t {
        cudaError_t e =
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kernel<<<grid, kBuildThreads, smem, s>>>(
            static_cast<const CodeT*>(codes), static_cast<const TV*>(vals), g.N, g.L, g.NB, g.d,
            best, absmax, keep_sums ? sums : nullptr, gtab, counts, err);
        return cudaGetLastError();
      };
      if (best == 4) return go(race_build_pipe_kernel<TV, CodeT, 4>);
      if (best == 8) return go(race_build_pipe_kernel<TV, CodeT, 8>);
      return go(race_build_pipe_kernel<TV, CodeT, 0>);
    }
  }
  cudaError_t e = cudaFuncSetAttribute(race_build_tiled_kernel<TV, CodeT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)b.smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(b.groups * b.nds, g.BH);
  race_build_tiled_kernel<TV, CodeT><<<grid, kBuildThreads, b.smem, s>>>(
      static_cast<const CodeT*>(codes), static_cast<const TV*>(vals), g.N, g.L, g.NB, g.d, b.nt,
      b.ntp, absmax, keep_sums ? sums : nullptr, gtab, counts, err);
  return cudaGetLastError();
}

// Words per lane of the row-pipelined gathers (0: not applicable).
int row_wpl(const Geometry& g, int QL) {
  if ((g.L * g.rcode_bytes) % 4 != 0) return 0;
  const int W = g.L * g.rcode_bytes / 4;
  const int wpl = (W + QL - 1) / QL;
  return wpl <= 1 ? 1 : wpl <= 2 ? 2 : wpl <= 4 ? 4 : 0;
}

int rows_grid(int64_t rows, int QL) {
  const int64_t warps = (rows * QL + 31) / 32;
  const int64_t b = (warps + 7) / 8;
  return (int)(b < 148 * 4 ? b : 148 * 4);
}

template <typename TT, typename CodeT>
cudaError_t gather_sum(const Geometry& g, const void* codes, const TT* tables, float* out,
                       TT* add_out, cudaStream_t s) {
  constexpr int EL = 16 / sizeof(TT);
  const int64_t rows = (int64_t)g.BH * g.N;
  const int QLr = g.d / EL;
  const CodeT* c = static_cast<const CodeT*>(codes);
  const int wpl = row_wpl(g, QLr);
  if (wpl > 0) {
    const int grid = rows_grid(rows, QLr);
#define ELSAA_GROWS(QL, WPL)                                                                   \
  race_gather_rows_kernel<TT, CodeT, QL, WPL><<<grid, 256, 0, s>>>(c, tables, rows, g.N, g.L,  \
                                                                    g.NB, g.d, out, add_out)
#define ELSAA_GROWS_W(QL)                                                                      \
  switch (wpl) {                                                                               \
    case 1: ELSAA_GROWS(QL, 1); break;                                                         \
    case 2: ELSAA_GROWS(QL, 2); break;                                                         \
    default: ELSAA_GROWS(QL, 4); break;                                                        \
  }
    switch (g.d) {   // QL = d / EL for d in {32, 64, 128}
      case 32: ELSAA_GROWS_W(32 / EL); break;
      case 64: ELSAA_GROWS_W(64 / EL); break;
      default: ELSAA_GROWS_W(128 / EL); break;
    }
#undef ELSAA_GROWS_W
#undef ELSAA_GROWS
    return cudaGetLastError();
  }
  if (add_out) return cudaErrorNotSupported;   // callers check race_gather_add_supported
  const int grid = grid_for_rows((rows * g.d / EL + 31) / 32, 8);
  switch (g.d) {
    case 32: race_gather_sum_kernel<TT, CodeT, 32 / EL><<<grid, 256, 0, s>>>(c, tables, rows, g.N, g.L, g.NB, g.d, out); break;
    case 64: race_gather_sum_kernel<TT, CodeT, 64 / EL><<<grid, 256, 0, s>>>(c, tables, rows, g.N, g.L, g.NB, g.d, out); break;
    default: race_gather_sum_kernel<TT, CodeT, 128 / EL><<<grid, 256, 0, s>>>(c, tables, rows, g.N, g.L, g.NB, g.d, out); break;
  }
  return cudaGetLastError();
}

template <typename T, typename CodeT>
cudaError_t fuse_fwd(const Geometry& g, const void* q, const void* rcode_q,
                     const void* tables, const int32_t* counts, const void* o_sp,
                     const float* lse, const float* gate_w, const float* gate_b, const float* lam,
                     void* y, void* o_race, int32_t* ctot, cudaStream_t s, int gate_fixed, float gs,
                     float gr) {
  constexpr int EL = 16 / sizeof(T);
  const int64_t rows = (int64_t)g.BH * g.N;
  const int QLr = g.d / EL;
  const int wpl = row_wpl(g, QLr);
  if (wpl > 0) {
    const int grid = rows_grid(rows, QLr);
#define ELSAA_FROWS(QL, WPL)                                                                   \
  race_fuse_rows_kernel<T, CodeT, QL, WPL><<<grid, 256, 0, s>>>(                               \
      static_cast<const T*>(q), static_cast<const CodeT*>(rcode_q),                            \
      static_cast<const T*>(tables), counts, static_cast<const T*>(o_sp), lse, gate_w, gate_b, \
      gate_fixed, gs, gr, lam, rows, g.N, g.L, g.NB, g.d, static_cast<T*>(y),                  \
      static_cast<T*>(o_race), ctot)
#define ELSAA_FROWS_W(QL)                                                                      \
  switch (wpl) {                                                                               \
    case 1: ELSAA_FROWS(QL, 1); break;                                                         \
    case 2: ELSAA_FROWS(QL, 2); break;                                                         \
    default: ELSAA_FROWS(QL, 4); break;                                                        \
  }
    switch (g.d) {   // QL = d / EL for d in {32, 64, 128}
      case 32: ELSAA_FROWS_W(32 / EL); break;
      case 64: ELSAA_FROWS_W(64 / EL); break;
      default: ELSAA_FROWS_W(128 / EL); break;
    }
#undef ELSAA_FROWS_W
#undef ELSAA_FROWS
    return cudaGetLastError();
  }
  const int grid = grid_for_rows((rows * g.d / EL + 31) / 32, 8);
#define ELSAA_FUSE(QL)                                                                         \
  race_fuse_fwd_kernel<T, CodeT, QL><<<grid, 256, 0, s>>>(                                     \
      static_cast<const T*>(q), static_cast<const CodeT*>(rcode_q),                            \
      static_cast<const T*>(tables), counts,                                                    \
      static_cast<const T*>(o_sp), lse, gate_w, gate_b, gate_fixed, gs, gr, lam, rows, g.N,    \
      g.L, g.NB, g.d, static_cast<T*>(y), static_cast<T*>(o_race), ctot)
  switch (g.d) {
    case 32: ELSAA_FUSE(32 / EL); break;
    case 64: ELSAA_FUSE(64 / EL); break;
    default: ELSAA_FUSE(128 / EL); break;
  }
#undef ELSAA_FUSE
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_unit_absmax(const Geometry& g, const void* vals, bool vals_f32, float* absmax,
                               cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(absmax, 0, (size_t)g.BH * sizeof(float), s);
  if (e != cudaSuccess) return e;
  const int64_t per_unit = (int64_t)g.N * g.d;
  const int64_t want = (per_unit / 8 + 255) / 256;
  const dim3 grid((unsigned)(want < 64 ? want : 64), g.BH);
  if (vals_f32 || !g.bf16)
    unit_absmax_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(vals), per_unit,
                                                    absmax);
  else
    unit_absmax_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(vals), per_unit, absmax);
  return cudaGetLastError();
}

int race_build_kernels(const Geometry& g, bool vals_f32, bool gtab) {
  const int esz = (vals_f32 || !g.bf16) ? 4 : 2;
  const int cb = g.rcode_bytes;
  const SortedSmem m = sorted_smem(g.N, g.NB, g.d, cb);
  if (g.N <= 65536 && g.NB <= kSortedThreads && m.total <= (size_t)kBuildSmemBudget &&
      g.d % (16 / esz) == 0)
    return 1;
  const int seg = g.N < kSegKeys ? g.N : kSegKeys;
  if (g.NB <= 1024 && seg_smem(seg, g.NB, cb).total <= (size_t)kBuildSmemBudget &&
      g.d % (16 / esz) == 0 && g.d / (16 / esz) <= 32)
    return 3;   // counting pass, build, finishing pass
  const BuildShape b = build_shape(g);
  if (b.nt < 1) return 1 + (gtab ? 1 : 0);   // global atomics, bf16 copy
  return 1;
}

cudaError_t launch_race_build(const Geometry& g, const void* codes, const void* codes_t,
                              const void* vals,
                              bool vals_f32, const float* absmax, float* sums, bool keep_sums,
                              __nv_bfloat16* gtab, int32_t* counts, int32_t* count_scratch,
                              uint32_t* err, cudaStream_t s) {
  if (vals_f32 || !g.bf16)
    return g.rcode_bytes == 1
               ? build<float, uint8_t>(g, codes, codes_t, vals, absmax, sums, keep_sums, gtab,
                                       counts, count_scratch, err, s)
               : build<float, uint16_t>(g, codes, codes_t, vals, absmax, sums, keep_sums, gtab,
                                        counts, count_scratch, err, s);
  return g.rcode_bytes == 1
             ? build<__nv_bfloat16, uint8_t>(g, codes, codes_t, vals, absmax, sums, keep_sums,
                                             gtab, counts, count_scratch, err, s)
             : build<__nv_bfloat16, uint16_t>(g, codes, codes_t, vals, absmax, sums, keep_sums,
                                              gtab, counts, count_scratch, err, s);
}

cudaError_t launch_tables_to_bf16(const Geometry& g, const float* sums, __nv_bfloat16* gtab,
                                  cudaStream_t s) {
  const int64_t n = (int64_t)g.BH * g.L * g.NB * g.d;
  to_bf16_kernel<<<148 * 8, 256, 0, s>>>(sums, gtab, n);
  return cudaGetLastError();
}

cudaError_t launch_race_gather_sum(const Geometry& g, const void* codes, const void* tables,
                                   float* out, cudaStream_t s) {
  if (g.bf16) {
    const __nv_bfloat16* t = static_cast<const __nv_bfloat16*>(tables);
    return g.rcode_bytes == 1 ? gather_sum<__nv_bfloat16, uint8_t>(g, codes, t, out, nullptr, s)
                              : gather_sum<__nv_bfloat16, uint16_t>(g, codes, t, out, nullptr, s);
  }
  const float* t = static_cast<const float*>(tables);
  return g.rcode_bytes == 1 ? gather_sum<float, uint8_t>(g, codes, t, out, nullptr, s)
                            : gather_sum<float, uint16_t>(g, codes, t, out, nullptr, s);
}

bool race_gather_add_supported(const Geometry& g) {
  return row_wpl(g, g.d / (g.bf16 ? 8 : 4)) > 0;
}

cudaError_t launch_race_gather_add(const Geometry& g, const void* codes, const void* tables,
                                   void* dst, cudaStream_t s) {
  if (g.bf16) {
    const __nv_bfloat16* t = static_cast<const __nv_bfloat16*>(tables);
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(dst);
    return g.rcode_bytes == 1 ? gather_sum<__nv_bfloat16, uint8_t>(g, codes, t, nullptr, o, s)
                              : gather_sum<__nv_bfloat16, uint16_t>(g, codes, t, nullptr, o, s);
  }
  const float* t = static_cast<const float*>(tables);
  float* o = static_cast<float*>(dst);
  return g.rcode_bytes == 1 ? gather_sum<float, uint8_t>(g, codes, t, nullptr, o, s)
                            : gather_sum<float, uint16_t>(g, codes, t, nullptr, o, s);
}

cudaError_t launch_race_fuse_fwd(const Geometry& g, const void* q, const void* rcode_q,
                                 const void* tables, const int32_t* counts,
                                 const void* o_sp, const float* lse, const float* gate_w,
                                 const float* gate_b, const float* lam, void* y, void* o_race,
                                 int32_t* ctot, cudaStream_t s) {
  const float gs = g.gate_s, gr = g.gate_r;
  const int fixed = g.gate_fixed;
  if (g.bf16)
    return g.rcode_bytes == 1
               ? fuse_fwd<__nv_bfloat16, uint8_t>(g, q, rcode_q, tables, counts, o_sp, lse, gate_w,
                                                  gate_b, lam, y, o_race, ctot, s, fixed, gs, gr)
               : fuse_fwd<__nv_bfloat16, uint16_t>(g, q, rcode_q, tables, counts, o_sp, lse,
                                                   gate_w, gate_b, lam, y, o_race, ctot, s, fixed,
                                                   gs, gr);
  return g.rcode_bytes == 1
             ? fuse_fwd<float, uint8_t>(g, q, rcode_q, tables, counts, o_sp, lse, gate_w, gate_b,
                                        lam, y, o_race, ctot, s, fixed, gs, gr)
             : fuse_fwd<float, uint16_t>(g, q, rcode_q, tables, counts, o_sp, lse, gate_w, gate_b,
                                         lam, y, o_race, ctot, s, fixed, gs, gr);
}

}  // namespace elsaa
