// Exact sparse branch, forward, as a persistent warp-specialized tcgen05
// pipeline (bf16, d = 64, chunk c <= 128 with 128 % c == 0).
//
// The sparse branch ("Two Efficient Attentions, One Denominator Problem",
// section "Two efficient branches can still be mis-scaled") is exact softmax
// attention over each query's Sort-LSH window: the query at sorted rank r
// (chunk j = r / c) sees the keys at sorted ranks [max(0,(j-1)c), (j+1)c).
// A tile of 128 sorted queries starting at r0 sees the keys [r0 - c, r0 + 128)
// (r0 = 0: [0, 128)), at most 256, so its scores fit in 256 TMEM columns and
// the softmax is exact in one pass (row max first, then exp).
//
// Roles (320 threads, one CTA per SM, tiles strided over the grid):
//   warp 0      producer: stages the tile's token indices, then gathers the Q,
//               K and V rows with cp.async into a two-stage ring of
//               128B-swizzled tiles; completion arrives on full[stage]
//   warp 1      MMA issuer (one thread) and TMEM owner:
//                 S = Q K^T            -> TMEM [0, 256)
//                 O = P V              -> TMEM [256, 320) or [320, 384)
//   warps 2..9  softmax and epilogue: warp w reaches TMEM lanes (query rows)
//               32 (w % 4) .. +31 and takes half of the key columns (warps 2..5
//               the first half, 6..9 the second); row max and row sum are
//               combined through shared memory; p = exp2(scale log2e s - m)
//               (masked to the row's own window when c < 128), P (bf16) to
//               shared memory, then O / l and the log-mass to the query's
//               token index
// Barriers: full/empty per stage, s_full, p_full, o_full/o_free per O buffer.
// Every wait is bounded; a timeout records ERR_TIMEOUT and every role leaves
// its loop, frees TMEM and returns.
#include <math.h>

#include "internal.h"
#include "tc_common.cuh"

namespace elsaa {
namespace {

using namespace tc;

constexpr int D = 64;
constexpr int kTile = 128;
constexpr int kMaxKeys = 256;
constexpr int kThreads = 320;
constexpr int kSoftmaxThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTS = 0, kTO = 256;   // S: 256 columns, O: 2 x 64 columns

struct PipeLayout {
  static constexpr uint32_t kQ = 128 * 128;           // one stage: Q 128 rows
  static constexpr uint32_t kKV = kMaxKeys * 128;     // K or V: 256 rows
  static constexpr uint32_t kStage = kQ + 2 * kKV;    // 80 KB
  static constexpr uint32_t kP = 2 * kStage;          // P: 128 x 256 bf16, 4 sub-tiles of 64 keys
  static constexpr uint32_t kRed = kP + 4 * 128 * 128;   // row max and sum: [2 halves][128 rows] x2
  static constexpr uint32_t kBar = kRed + 2 * 2 * 128 * 4;
  static constexpr uint32_t kDyn = kBar + 128;
};

struct Bars {
  uint64_t full[2], empty[2], s_full, p_full, o_full[2], o_free[2];
  uint32_t tmem;
};

ELSAA_DEV void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 2^x on the special-function unit (approximate, flushes denormals).
ELSAA_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Barrier among the softmax warps only.
ELSAA_DEV void softmax_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory"); }

ELSAA_DEV void tile_of(int64_t t, int tiles_per_unit, int* bh, int* r0) {
  *bh = (int)(t / tiles_per_unit);
  *r0 = (int)(t % tiles_per_unit) * kTile;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_pipe_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                     const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ perm_q,
                     const int32_t* __restrict__ perm_k, int BH, int N, int chunk,
                     float scale_log2, __nv_bfloat16* __restrict__ o_sp, float* __restrict__ lse,
                     uint32_t* __restrict__ err) {
  using Lay = PipeLayout;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  Bars* bars = reinterpret_cast<Bars*>(smem + Lay::kBar);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((sbase & 1023u) != 0) {
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  const int tiles_per_unit = N / kTile;
  const int64_t ntiles = (int64_t)BH * tiles_per_unit;
  // tiles handled by this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int64_t my_count =
      ntiles > blockIdx.x ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->full[s], 32);
      mbar_init(&bars->empty[s], 1);
      mbar_init(&bars->o_full[s], 1);
      mbar_init(&bars->o_free[s], kSoftmaxThreads);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, kSoftmaxThreads);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem, kTmemCols);
    tmem_relinquish();
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = bars->tmem;
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // Token indices stay in registers (lane j holds rows j, j + 32, ...) and
    // are broadcast with shuffles while the cp.async gathers are issued.
    for (int64_t i = 0; i < my_count && ok; ++i) {
      const int s = (int)(i & 1);
      if (i >= 2) ok = mbar_wait(&bars->empty[s], (uint32_t)(((i >> 1) - 1) & 1), err);
      if (!ok) break;
      int bh, r0;
      tile_of(blockIdx.x + i * gridDim.x, tiles_per_unit, &bh, &r0);
      const size_t unit = (size_t)bh * N;
      const int kbase = max(0, r0 - chunk);
      const int nk = r0 + kTile - kbase;
      int qr[kTile / 32], kr[kMaxKeys / 32];
#pragma unroll
      for (int j = 0; j < kTile / 32; ++j) qr[j] = perm_q[unit + r0 + lane + 32 * j];
#pragma unroll
      for (int j = 0; j < kMaxKeys / 32; ++j)
        kr[j] = lane + 32 * j < nk ? perm_k[unit + kbase + lane + 32 * j] : 0;
      const uint32_t st = sbase + s * Lay::kStage;
      const __nv_bfloat16* qb = q + unit * D;
      const __nv_bfloat16* kb = k + unit * D;
      const __nv_bfloat16* vb = v + unit * D;
      const int ch = lane & 7;
      // 4 rows per iteration (8 lanes per row, one 16-byte chunk each)
#pragma unroll
      for (int it = 0; it < kTile / 4; ++it) {
        const int row = 4 * it + (lane >> 3);
        const int tok = __shfl_sync(0xffffffffu, qr[it >> 3], row & 31);
        cp_async16(st + sw128_off(row, ch), qb + (size_t)tok * D + ch * 8, 16);
      }
#pragma unroll
      for (int it = 0; it < kMaxKeys / 4; ++it) {
        if (4 * it < nk) {   // nk is a multiple of 16: whole iterations only
          const int row = 4 * it + (lane >> 3);
          const int tok = __shfl_sync(0xffffffffu, kr[it >> 3], row & 31);
          const size_t src = (size_t)tok * D + ch * 8;
          cp_async16(st + Lay::kQ + sw128_off(row, ch), kb + src, 16);
          cp_async16(st + Lay::kQ + Lay::kKV + sw128_off(row, ch), vb + src, 16);
        }
      }
      cp_async_arrive(&bars->full[s]);
    }
    cp_async_wait_all();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_pv = idesc_bf16(128, D, false, true);
      auto issue_pv = [&](int64_t j) -> bool {
        // O[j % 2] = P V_j ; needs P (p_full) and a free O buffer
        const int o = (int)(j & 1);
        if (j >= 2 && !mbar_wait(&bars->o_free[o], (uint32_t)(((j >> 1) - 1) & 1), err))
          return false;
        fence_after();
        int bh, r0;
        tile_of(blockIdx.x + j * gridDim.x, tiles_per_unit, &bh, &r0);
        const int nk = r0 + kTile - max(0, r0 - chunk);
        const uint32_t vst = sbase + (uint32_t)(j & 1) * Lay::kStage + Lay::kQ + Lay::kKV;
        for (int s = 0; s < nk / 16; ++s) {
          const uint32_t poff = (s >> 2) * (128 * 128) + (s & 3) * 32;
          mma_bf16_ss(tmem + kTO + o * D, sw128_desc(sbase + Lay::kP + poff, 16, 1024),
                      sw128_desc(vst + s * 2048, 128 * 128, 1024), id_pv, s > 0 ? 1u : 0u);
        }
        mma_commit(&bars->o_full[o]);
        mma_commit(&bars->empty[j & 1]);
        return true;
      };
      for (int64_t i = 0; i < my_count && ok; ++i) {
        const int s = (int)(i & 1);
        ok = mbar_wait(&bars->full[s], (uint32_t)((i >> 1) & 1), err);
        if (!ok) break;
        fence_async_smem();   // cp.async data -> tensor core
        if (i >= 1) {
          ok = mbar_wait(&bars->p_full, (uint32_t)((i - 1) & 1), err);
          if (!ok) break;
          ok = issue_pv(i - 1);
          if (!ok) break;
        }
        int bh, r0;
        tile_of(blockIdx.x + i * gridDim.x, tiles_per_unit, &bh, &r0);
        const int nk = r0 + kTile - max(0, r0 - chunk);
        const uint32_t st = sbase + s * Lay::kStage;
        const uint32_t id_s = idesc_bf16(128, nk, false, false);
        fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tmem + kTS, sw128_desc(st + kk * 32, 16, 1024),
                      sw128_desc(st + Lay::kQ + kk * 32, 16, 1024), id_s, kk > 0 ? 1u : 0u);
        mma_commit(&bars->s_full);
      }
      if (ok && my_count > 0) {
        ok = mbar_wait(&bars->p_full, (uint32_t)((my_count - 1) & 1), err);
        if (ok) ok = issue_pv(my_count - 1);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int quarter = warp & 3, half = (warp - 2) >> 2;
    const int row = 32 * quarter + lane;               // TMEM lane = query row of the tile
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    float* red_m = reinterpret_cast<float*>(smem + Lay::kRed);   // [2][128]
    float* red_l = red_m + 2 * 128;                              // [2][128]
    const bool masked = chunk < kTile;
    for (int64_t i = 0; i < my_count; ++i) {
      int bh, r0;
      tile_of(blockIdx.x + i * gridDim.x, tiles_per_unit, &bh, &r0);
      const size_t unit = (size_t)bh * N;
      const int token = perm_q[unit + r0 + row];
      const int kbase = max(0, r0 - chunk);
      const int nk = r0 + kTile - kbase;
      const int cw = nk >> 1, cbeg = half * cw;          // this warp's key columns
      const int jr = (r0 + row) / chunk;
      const int lo = max(0, (jr - 1) * chunk) - kbase, hi = (jr + 1) * chunk - kbase;
      ok = mbar_wait(&bars->s_full, (uint32_t)(i & 1), err);
      if (!ok) break;
      fence_after();
      float m = -INFINITY;
      for (int c0 = cbeg; c0 < cbeg + cw; c0 += 32) {
        float sv[32];
        tmem_ld32(tmem + kTS + lane_off + c0, sv);
        tmem_ld_wait();
        if (masked) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c0 + e >= lo && c0 + e < hi) m = fmaxf(m, sv[e]);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) m = fmaxf(m, sv[e]);
        }
      }
      red_m[half * 128 + row] = m;
      softmax_sync();
      m = fmaxf(m, red_m[(half ^ 1) * 128 + row]) * scale_log2;   // scale > 0
      float l = 0.f;
      for (int c0 = cbeg; c0 < cbeg + cw; c0 += 32) {
        float sv[32];
        tmem_ld32(tmem + kTS + lane_off + c0, sv);
        tmem_ld_wait();
        uint32_t packed[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float p0 = ex2(fmaf(sv[e], scale_log2, -m));
          float p1 = ex2(fmaf(sv[e + 1], scale_log2, -m));
          if (masked) {
            p0 = (c0 + e >= lo && c0 + e < hi) ? p0 : 0.f;
            p1 = (c0 + e + 1 >= lo && c0 + e + 1 < hi) ? p1 : 0.f;
          }
          l += p0 + p1;
          const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
          packed[e >> 1] = *reinterpret_cast<const uint32_t*>(&h);
        }
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const int key = c0 + q8 * 8;
          uint8_t* dst = smem + Lay::kP + (key >> 6) * (128 * 128) + sw128_off(row, (key & 63) >> 3);
          *reinterpret_cast<uint4*>(dst) =
              make_uint4(packed[q8 * 4], packed[q8 * 4 + 1], packed[q8 * 4 + 2], packed[q8 * 4 + 3]);
        }
      }
      red_l[half * 128 + row] = l;
      fence_async_smem();
      fence_before();
      mbar_arrive(&bars->p_full);
      softmax_sync();
      l += red_l[(half ^ 1) * 128 + row];
      // epilogue: O of this tile; each warp of the pair writes 32 of the 64 columns
      const int o = (int)(i & 1);
      ok = mbar_wait(&bars->o_full[o], (uint32_t)((i >> 1) & 1), err);
      if (!ok) break;
      fence_after();
      const float inv = 1.0f / l;
      __nv_bfloat16* orow = o_sp + (unit + token) * D;
      {
        const int c0 = half * 32;
        float ov[32];
        tmem_ld32(tmem + kTO + o * D + lane_off + c0, ov);
        tmem_ld_wait();
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 h =
                __floats2bfloat162_rn(ov[q8 * 8 + 2 * e] * inv, ov[q8 * 8 + 2 * e + 1] * inv);
            w4[e] = *reinterpret_cast<const uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(orow + c0 + q8 * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      if (half == 0) lse[unit + token] = (m + log2f(l)) * 0.69314718055994531f;
      fence_before();
      mbar_arrive(&bars->o_free[o]);
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool attn_pipe_supported(const Geometry& g) {
  return g.bf16 && g.d == 64 && g.N % kTile == 0 && g.chunk % 16 == 0 && g.chunk <= kTile &&
         kTile % g.chunk == 0;
}

cudaError_t launch_attn_fwd_pipe(const Geometry& g, const void* q, const void* k, const void* v,
                                 const int32_t* perm_q, const int32_t* perm_k, void* o_sp,
                                 float* lse, uint32_t* err, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_pipe_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)PipeLayout::kDyn);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntiles = (int64_t)g.BH * (g.N / kTile);
  const int grid_x = (int)(ntiles < sms ? ntiles : sms);
  attn_fwd_pipe_kernel<<<grid_x, kThreads, PipeLayout::kDyn, s>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), perm_q, perm_k, g.BH, g.N, g.chunk,
      g.scale * 1.4426950408889634f, static_cast<__nv_bfloat16*>(o_sp), lse, err);
  return cudaGetLastError();
}

}  // namespace elsaa
