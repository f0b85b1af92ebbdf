// Exact sparse branch, forward, as a persistent warp-specialized tcgen05
// pipeline (bf16, d = 64, chunk c <= 128 with 128 % c == 0).
//
// The sparse branch ("Two Efficient Attentions, One Denominator Problem",
// section "Two efficient branches can still be mis-scaled") is exact softmax
// attention over each query's Sort-LSH window: the query at sorted rank r
// (chunk j = r / c) sees the keys at sorted ranks [max(0,(j-1)c), (j+1)c).
//
// Work unit: a tile of 128 sorted queries (rank r0 = 128 tb).  Its keys lie in
// two 128-key blocks of the sorted order: block tb - 1 (only its last c keys
// are seen; none when tb = 0) and block tb.  Each CTA takes a contiguous run
// of tiles, so consecutive tiles share a key block: every block is gathered
// once (plus one extra at the start of the run) and kept in a four-slot ring.
// Scores fit in 256 TMEM columns (block tb - 1 in [0, 128), block tb in
// [128, 256)); the softmax is exact in one pass (row max first, then exp).
//
// Roles (416 threads, one CTA per SM):
//   warps 0..3  producers: token indices (prefetched one tile ahead), TMA row
//               gathers (four rows per instruction) of Q tiles (two-slot
//               ring) and K/V blocks (four-slot ring) into 128B-swizzled
//               tiles; completion counted in bytes on full_q / full_kv.  A
//               warp issues its gathers one after another at a few tens of
//               nanoseconds each, so each 128-row tile is split over four
//               warps (one per SM sub-partition, 32 rows each)
//   warp 12     MMA issuer (one thread) and TMEM owner:
//                 O(j-1) = P V        as soon as P of tile j-1 is written,
//                                     P read from TMEM as the A operand
//                 S(j)   = Q K^T      -> TMEM [0, 256)
//               and releases Q and K/V slots through tcgen05.commit
//   warps 4..11 softmax and epilogue: warp w reaches TMEM lanes (query rows)
//               32 (w % 4) .. +31 and takes one of two column ranges; row max
//               and row sum are combined through shared memory;
//               p = exp2(scale log2e s - m) masked to the row's own window,
//               P (bf16 pairs) to TMEM [384, 512), then O / l and the
//               log-mass to the query's token index
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
constexpr int kThreads = 416;
constexpr int kProducers = 4;            // warps 0..3
constexpr int kSoftmaxWarp0 = 4;         // warps 4..11
constexpr int kMmaWarp = 12;
constexpr int kSoftmaxThreads = 256;
constexpr int kKvSlots = 4;
constexpr int kQSlots = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTS = 0, kTO = 256;   // S: 256 columns, O: 2 x 64 columns
constexpr uint32_t kTP = 384;            // P: 128 columns, two bf16 per column

struct PipeLayout {
  static constexpr uint32_t kTileBytes = 128 * 128;              // 128 rows x 64 bf16
  static constexpr uint32_t kKv = 0;                             // [4][K | V]
  static constexpr uint32_t kKvSlot = 2 * kTileBytes;
  static constexpr uint32_t kQ = kKv + kKvSlots * kKvSlot;       // [2][Q]
  static constexpr uint32_t kRed = kQ + kQSlots * kTileBytes;    // row max and sum [2][2][128]
  static constexpr uint32_t kBar = kRed + 2 * 2 * 128 * 4;
  static constexpr uint32_t kDyn = kBar + 256;
};

// TMA maps of Q, K and V as [B H N, 64] row matrices.
struct FwdMaps {
  CUtensorMap q, k, v;
};

struct Bars {
  uint64_t full_q[kQSlots], empty_q[kQSlots], full_kv[kKvSlots], empty_kv[kKvSlots];
  uint64_t s_full, p_full, o_full[2], o_free[2];
  uint32_t tmem;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// Geometry of tile j of this CTA's run.
struct TileInfo {
  int bh, tb;          // unit and tile within the unit (r0 = 128 tb)
  bool has_prev;       // block tb - 1 is part of the window
  int64_t own, prev;   // ring sequence numbers of blocks tb and tb - 1
  bool own_last;       // block tb is not used by the next tile
};

struct Run {
  int64_t begin, count;
  int tiles_per_unit;
  int extra;           // 1 if the run starts with the previous block of its first tile
  ELSAA_DEV TileInfo tile(int64_t j) const {
    TileInfo ti;
    const int64_t t = begin + j;
    ti.bh = (int)(t / tiles_per_unit);
    ti.tb = (int)(t % tiles_per_unit);
    ti.has_prev = ti.tb > 0;
    ti.own = j + extra;
    ti.prev = ti.own - 1;
    ti.own_last = (j + 1 == count) || (ti.tb + 1 == tiles_per_unit);
    return ti;
  }
};

// 2^x on the special-function unit (approximate, flushes denormals).
ELSAA_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Barrier among the softmax warps only.
ELSAA_DEV void softmax_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory"); }

// Barrier among the softmax warps that also ANDs a flag over them, so that a
// bounded wait that gave up in one thread makes all of them leave together.
ELSAA_DEV bool softmax_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kSoftmaxThreads)
      : "memory");
  return r != 0;
}

// Column ranges of a tile's scores: live columns [col_lo, ncols); the two
// softmax halves take [col_lo & ~31, mid) and [mid, ncols).
struct Cols {
  int col0;            // sorted rank of column 0
  int col_lo, ncols, mid;
};
ELSAA_DEV Cols tile_cols(const TileInfo& ti, int chunk) {
  Cols c;
  const int r0 = ti.tb * kTile;
  c.col0 = ti.has_prev ? r0 - kTile : r0;
  c.col_lo = ti.has_prev ? kTile - chunk : 0;
  c.ncols = ti.has_prev ? 2 * kTile : kTile;
  const int lo32 = c.col_lo & ~31;
  c.mid = ((lo32 + c.ncols) >> 1) & ~31;
  return c;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_pipe_kernel(const __grid_constant__ FwdMaps maps, const int32_t* __restrict__ perm_q,
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
  Run run;
  run.tiles_per_unit = N / kTile;
  {
    const int64_t ntiles = (int64_t)BH * run.tiles_per_unit;
    run.begin = ntiles * blockIdx.x / gridDim.x;
    run.count = ntiles * (blockIdx.x + 1) / gridDim.x - run.begin;
    run.extra = (run.count > 0 && run.begin % run.tiles_per_unit != 0) ? 1 : 0;
  }

  if (tid == 0) {
    for (int s = 0; s < kQSlots; ++s) {
      mbar_init(&bars->full_q[s], kProducers);   // each producer warp's byte-count arrival
      mbar_init(&bars->empty_q[s], 1);
    }
    for (int s = 0; s < kKvSlots; ++s) {
      mbar_init(&bars->full_kv[s], kProducers);
      mbar_init(&bars->empty_kv[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->o_full[s], 1);
      mbar_init(&bars->o_free[s], kSoftmaxThreads);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, kSoftmaxThreads);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem, kTmemCols);
    tmem_relinquish();
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = bars->tmem;
  bool ok = true;

  if (warp < kProducers) {
    // ---------------------------------------------------------------- producers
    // Producer warp pw loads rows 32 pw .. 32 pw + 31 of each Q tile and K/V
    // block: lane l < 8 takes rows 32 pw + 4 l .. + 3, whose four token
    // indices arrive in one 16-byte load (prefetched one tile ahead) and each
    // matrix's four rows in one TMA gather; lane 0 first arms the slot's
    // barrier with this warp's share of the bytes.
    const bool gl = lane < 8;
    const int rbase = 32 * warp + 4 * lane;   // first row of this lane
    auto load_idx = [&](const int32_t* perm, size_t base) {
      return gl ? *reinterpret_cast<const int4*>(perm + base + rbase) : make_int4(0, 0, 0, 0);
    };
    auto issue_kv = [&](int64_t n, size_t unit, int4 t4) -> bool {
      const int s = (int)(n % kKvSlots);
      if (n >= kKvSlots &&
          !__all_sync(0xffffffffu,
                      mbar_wait(&bars->empty_kv[s], (uint32_t)(((n / kKvSlots) - 1) & 1), err)))
        return false;
      if (lane == 0) mbar_arrive_expect_tx(&bars->full_kv[s], 2u * kTile * 128u / kProducers);
      __syncwarp();
      const uint32_t kst = sbase + Lay::kKv + s * Lay::kKvSlot + (uint32_t)rbase * 128;
      const int u = (int)unit;
      if (gl) {
        tma_gather4(kst, &maps.k, u + t4.x, u + t4.y, u + t4.z, u + t4.w, &bars->full_kv[s]);
        tma_gather4(kst + Lay::kTileBytes, &maps.v, u + t4.x, u + t4.y, u + t4.z, u + t4.w,
                    &bars->full_kv[s]);
      }
      return true;
    };
    auto issue_q = [&](int64_t j, size_t unit, int4 t4) -> bool {
      const int s = (int)(j % kQSlots);
      if (j >= kQSlots &&
          !__all_sync(0xffffffffu,
                      mbar_wait(&bars->empty_q[s], (uint32_t)(((j / kQSlots) - 1) & 1), err)))
        return false;
      if (lane == 0) mbar_arrive_expect_tx(&bars->full_q[s], kTile * 128u / kProducers);
      __syncwarp();
      const uint32_t qst = sbase + Lay::kQ + s * Lay::kTileBytes + (uint32_t)rbase * 128;
      const int u = (int)unit;
      if (gl) tma_gather4(qst, &maps.q, u + t4.x, u + t4.y, u + t4.z, u + t4.w, &bars->full_q[s]);
      return true;
    };
    int4 qi = make_int4(0, 0, 0, 0), ki = make_int4(0, 0, 0, 0);
    if (run.count > 0) {
      const TileInfo t0 = run.tile(0);
      const size_t unit = (size_t)t0.bh * N;
      if (run.extra) ok = issue_kv(0, unit, load_idx(perm_k, unit + (size_t)(t0.tb - 1) * kTile));
      qi = load_idx(perm_q, unit + (size_t)t0.tb * kTile);
      ki = load_idx(perm_k, unit + (size_t)t0.tb * kTile);
    }
    for (int64_t j = 0; j < run.count && ok; ++j) {
      const TileInfo ti = run.tile(j);
      const size_t unit = (size_t)ti.bh * N;
      ok = issue_q(j, unit, qi) && issue_kv(ti.own, unit, ki);
      if (!ok) break;
      if (j + 1 < run.count) {   // prefetch the next tile's indices
        const TileInfo tn = run.tile(j + 1);
        const size_t un = (size_t)tn.bh * N;
        qi = load_idx(perm_q, un + (size_t)tn.tb * kTile);
        ki = load_idx(perm_k, un + (size_t)tn.tb * kTile);
      }
    }

  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_pv = idesc_bf16(128, D, false, true);
      const uint32_t id_s = idesc_bf16(128, kTile, false, false);
      auto kv_slot = [&](int64_t n) -> uint32_t {
        return sbase + Lay::kKv + (uint32_t)(n % kKvSlots) * Lay::kKvSlot;
      };
      // descriptors of every slot's tile, built once: K-major (K step +32
      // bytes) for Q and K, MN-major (16-row K step +2048 bytes) for V, and
      // the K-major P tile
      const uint64_t q_d0 = sw128_desc(sbase + Lay::kQ, 16, 1024);
      const uint64_t k_d0 = sw128_desc(kv_slot(0), 16, 1024);
      const uint64_t v_n0 = sw128_desc(kv_slot(0) + Lay::kTileBytes, Lay::kTileBytes, 1024);
      auto qk = [&](int64_t j) { return desc_add(q_d0, (uint32_t)(j % kQSlots) * Lay::kTileBytes); };
      auto kk_d = [&](int64_t n) { return desc_add(k_d0, (uint32_t)(n % kKvSlots) * Lay::kKvSlot); };
      auto vn = [&](int64_t n) { return desc_add(v_n0, (uint32_t)(n % kKvSlots) * Lay::kKvSlot); };
      auto issue_pv = [&](int64_t j) -> bool {
        // O[j % 2] = P V over the live key columns; needs a free O buffer
        const int o = (int)(j & 1);
        if (j >= 2 && !mbar_wait(&bars->o_free[o], (uint32_t)(((j >> 1) - 1) & 1), err))
          return false;
        fence_after();
        const TileInfo ti = run.tile(j);
        const Cols cc = tile_cols(ti, chunk);
        for (int x = cc.col_lo; x < cc.ncols; x += 16) {
          const bool in_prev = ti.has_prev && x < kTile;
          const uint64_t vd = vn(in_prev ? ti.prev : ti.own);
          const int row = in_prev ? x : (ti.has_prev ? x - kTile : x);
          mma_bf16_ts(tmem + kTO + o * D, tmem + kTP + (uint32_t)(x >> 1),
                      desc_add(vd, (row >> 4) * 2048), id_pv, x > cc.col_lo ? 1u : 0u);
        }
        mma_commit(&bars->o_full[o]);
        if (ti.has_prev) mma_commit(&bars->empty_kv[ti.prev % kKvSlots]);
        if (ti.own_last) mma_commit(&bars->empty_kv[ti.own % kKvSlots]);
        return true;
      };
      int64_t kv_ready = 0;   // blocks whose arrival this thread has seen
      for (int64_t j = 0; j < run.count && ok; ++j) {
        if (j >= 1) {
          ok = mbar_wait(&bars->p_full, (uint32_t)((j - 1) & 1), err);
          if (!ok) break;
          ok = issue_pv(j - 1);
          if (!ok) break;
        }
        const TileInfo ti = run.tile(j);
        ok = mbar_wait(&bars->full_q[j % kQSlots], (uint32_t)((j / kQSlots) & 1), err);
        for (; ok && kv_ready <= ti.own; ++kv_ready)
          ok = mbar_wait(&bars->full_kv[kv_ready % kKvSlots],
                         (uint32_t)((kv_ready / kKvSlots) & 1), err);
        if (!ok) break;
        fence_after();
        const uint64_t qd = qk(j);
        if (ti.has_prev) {
          const uint64_t kd = kk_d(ti.prev);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(tmem + kTS, desc_add(qd, kk * 32), desc_add(kd, kk * 32), id_s,
                        kk > 0 ? 1u : 0u);
        }
        const uint32_t own_col = ti.has_prev ? (uint32_t)kTile : 0u;
        const uint64_t kd = kk_d(ti.own);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tmem + kTS + own_col, desc_add(qd, kk * 32), desc_add(kd, kk * 32), id_s,
                      kk > 0 ? 1u : 0u);
        mma_commit(&bars->s_full);
        mma_commit(&bars->empty_q[j % kQSlots]);
      }
      if (ok && run.count > 0) {
        ok = mbar_wait(&bars->p_full, (uint32_t)((run.count - 1) & 1), err);
        if (ok) ok = issue_pv(run.count - 1);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int quarter = warp & 3, half = (warp - kSoftmaxWarp0) >> 2;
    const int row = 32 * quarter + lane;               // TMEM lane = query row of the tile
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    float* red_m = reinterpret_cast<float*>(smem + Lay::kRed);   // [2][128]
    float* red_l = red_m + 2 * 128;                              // [2][128]
    const bool masked = chunk < kTile;
    for (int64_t j = 0; j < run.count; ++j) {
      const TileInfo ti = run.tile(j);
      const size_t unit = (size_t)ti.bh * N;
      const int r0 = ti.tb * kTile;
      const int token = perm_q[unit + r0 + row];
      const Cols cc = tile_cols(ti, chunk);
      const int cbeg = half ? cc.mid : (cc.col_lo & ~31);
      const int cend = half ? cc.ncols : cc.mid;
      const int jr = (r0 + row) / chunk;
      const int lo = max(0, (jr - 1) * chunk) - cc.col0, hi = (jr + 1) * chunk - cc.col0;
      ok = softmax_all(mbar_wait(&bars->s_full, (uint32_t)(j & 1), err));
      if (!ok) break;
      fence_after();
      float m = -INFINITY;
      for (int c0 = cbeg; c0 < cend; c0 += 32) {
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
      for (int c0 = cbeg; c0 < cend; c0 += 32) {
        float sv[32];
        tmem_ld32(tmem + kTS + lane_off + c0, sv);
        tmem_ld_wait();
        uint32_t packed[16];
        float l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float a0 = sv[e], a1 = sv[e + 1];
          fma2(a0, a1, scale_log2, scale_log2, -m, -m);
          float p0 = ex2(a0), p1 = ex2(a1);
          if (masked) {
            p0 = (c0 + e >= lo && c0 + e < hi) ? p0 : 0.f;
            p1 = (c0 + e + 1 >= lo && c0 + e + 1 < hi) ? p1 : 0.f;
          }
          add2(l0, l1, p0, p1);
          const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
          packed[e >> 1] = *reinterpret_cast<const uint32_t*>(&h);
        }
        l += l0 + l1;
        // the row's P values of keys c0 .. c0 + 31 into TMEM columns c0 / 2 ..
        tmem_st16(tmem + kTP + lane_off + (uint32_t)(c0 >> 1), packed);
      }
      tmem_st_wait();
      red_l[half * 128 + row] = l;
      fence_before();
      mbar_arrive(&bars->p_full);
      softmax_sync();
      l += red_l[(half ^ 1) * 128 + row];
      // epilogue: O of this tile; each warp of the pair writes 32 of the 64 columns
      const int o = (int)(j & 1);
      ok = softmax_all(mbar_wait(&bars->o_full[o], (uint32_t)((j >> 1) & 1), err));
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
  if (warp == kMmaWarp) {
    fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool attn_pipe_supported(const Geometry& g) {
  // TMA row coordinates are 32-bit
  return g.bf16 && g.lookback == 1 && !g.causal && g.rounds == 1 && g.d == 64 && g.N % kTile == 0 &&
         g.chunk % 16 == 0 && g.chunk <= kTile &&
         kTile % g.chunk == 0 && (int64_t)g.BH * g.N < (int64_t)1 << 31;
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
  FwdMaps maps;
  const uint64_t rows = (uint64_t)g.BH * g.N;
  if ((e = make_row_map(&maps.q, q, rows)) != cudaSuccess) return e;
  if ((e = make_row_map(&maps.k, k, rows)) != cudaSuccess) return e;
  if ((e = make_row_map(&maps.v, v, rows)) != cudaSuccess) return e;
  attn_fwd_pipe_kernel<<<grid_x, kThreads, PipeLayout::kDyn, s>>>(
      maps, perm_q, perm_k, g.BH, g.N, g.chunk,
      g.scale * 1.4426950408889634f, static_cast<__nv_bfloat16*>(o_sp), lse, err);
  return cudaGetLastError();
}

}  // namespace elsaa
