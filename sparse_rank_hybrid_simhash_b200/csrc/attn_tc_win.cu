// Exact sparse branch, forward, for any Sort-LSH window: a persistent
// warp-specialized tcgen05 pipeline that streams the window in 128-key blocks
// (bf16, d = 64 or 128, any chunk c with c % 16 == 0, any lookback).
//
// The sparse branch ("Two Efficient Attentions, One Denominator Problem",
// section "Two efficient branches can still be mis-scaled") is exact softmax
// attention over each query's Sort-LSH window.  The query at sorted rank r
// (chunk j = r / c) sees the keys at sorted ranks [max(0, (j - lb) c),
// (j + 1) c): its own chunk and lb earlier ones (lb = 1 in the pages).
//
// Work unit: a tile of 128 sorted queries.  The union of its rows' windows
// covers the 128-key blocks kb_lo .. kb_lo + nb - 1 of the sorted keys; the
// rows' own windows are applied as a mask (none is needed when c is a multiple
// of 128: every row of the tile then has the same, block-aligned window).
// With the causal mask (an extension; the pages did not evaluate causal use)
// a row also drops the keys whose token index exceeds its own; a row left
// without keys gets O_sp = 0 and lse = -inf.  With several hash rounds (an
// extension: a query attends the union of its rounds' windows, each key once)
// the kernel runs once per round t on that round's orders, drops the keys
// that lie in the query's window of an earlier round (by the keys' and the
// query's ranks in that round; the keys' earlier ranks come laid out in round
// t's key order, from round_key_ranks_kernel), and writes the round's partial
// softmax (O_t normalized by its own mass, in fp32, and lse_t) for
// round_combine_kernel.
// A window may exceed what TMEM holds next to O, so each tile takes two
// passes over its blocks: pass 1 computes S = Q K^T block by block for the
// exact row maximum; pass 2 computes S again, P = exp(scale s - m) (bf16, in
// TMEM) and O += P V.  The softmax is therefore the same as a one-pass
// softmax over the whole window: P <= 1, no rescaling of O.
//
// Roles (416 threads, one CTA per SM):
//   warps 0..3  producers: TMA row gathers (four rows per instruction; two
//               64-column halves per row when d = 128) of Q tiles (two-slot
//               ring), K blocks (a ring for both passes) and V blocks (pass 2).
//               A warp issues its gathers one after another at a few tens of
//               nanoseconds each, so every 128-row load is split over four
//               warps (one per SM sub-partition, 32 rows each) that arm the
//               slot's barrier with their own byte counts
//   warp 12     MMA issuer (one thread) and TMEM owner: S into two 128-column
//               TMEM buffers, one block ahead of the softmax; O += P V with P
//               read from TMEM as the A operand (two 64-column P buffers)
//   warps 4..11 softmax and epilogue: warp w reaches TMEM lanes (query rows)
//               32 (w % 4) .. +31 and one of the two 64-column halves of a
//               block; row maximum and row sum are combined through shared
//               memory; then O / l and the log-mass to the query's token
// TMEM: S [0, 256), P [256, 384), O [384, 512) (two 64-column buffers for
// alternating tiles when d = 64, one 128-column buffer when d = 128).
// Every wait is bounded; a timeout records ERR_TIMEOUT and every role leaves
// its loop; the MMA issuer waits for its last MMAs and the producer for its
// last copies before TMEM is freed.
#include <math.h>

#include "internal.h"
#include "tc_common.cuh"

namespace elsaa {
namespace {

using namespace tc;

constexpr int kTile = 128;
constexpr int kThreads = 416;
constexpr int kProducers = 4;            // warps 0..3
constexpr int kSoftmaxWarp0 = 4;         // warps 4..11
constexpr int kMmaWarp = 12;
constexpr int kSoftmaxThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTS = 0, kTP = 256, kTO = 384;
constexpr uint32_t kAtom = 128 * 128;   // 128 rows x 64 bf16

template <int D>
struct WinLayout {
  static constexpr uint32_t kTileBytes = kAtom * (D / 64);   // 128 rows x D bf16
  static constexpr int kQSlots = 2;
  static constexpr int kKSlots = D == 64 ? 4 : 3;
  static constexpr int kVSlots = D == 64 ? 4 : 2;
  static constexpr int kOBufs = D == 64 ? 2 : 1;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kQSlots * kTileBytes;
  static constexpr uint32_t kV = kK + kKSlots * kTileBytes;
  static constexpr uint32_t kRed = kV + kVSlots * kTileBytes;   // row max and sum [2][2][128]
  static constexpr uint32_t kBar = kRed + 2 * 2 * 128 * 4;
  static constexpr uint32_t kDyn = kBar + 512;
};
static_assert(WinLayout<128>::kDyn <= 232448, "shared memory of the d = 128 pipeline");

struct WinMaps {
  CUtensorMap q, k, v;
};

struct WinBars {
  uint64_t full_q[2], empty_q[2];
  uint64_t full_k[4], empty_k[4], full_v[4], empty_v[4];
  uint64_t s_full[2], s_free[2], p_full[2], p_free[2];
  uint64_t o_full[2], o_free[2];
  uint64_t drain;
  uint32_t tmem;
};
static_assert(sizeof(WinBars) <= 512, "barrier block");

// The blocks of tile t (of the whole grid's tile order).
struct WinTile {
  int bh, tb;
  int kb_lo, nb;
};
ELSAA_DEV WinTile win_tile(int64_t t, int tiles_per_unit, int N, int chunk, int lb) {
  WinTile w;
  w.bh = (int)(t / tiles_per_unit);
  w.tb = (int)(t % tiles_per_unit);
  const int r0 = w.tb * kTile;
  const int jf = r0 / chunk, jl = (r0 + kTile - 1) / chunk;
  const int lo = max(0, (jf - lb) * chunk);
  const int hi = min(N, (jl + 1) * chunk);
  w.kb_lo = lo / kTile;
  w.nb = (hi + kTile - 1) / kTile - w.kb_lo;
  return w;
}

// 2^x on the special-function unit (approximate, flushes denormals).
ELSAA_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

ELSAA_DEV void softmax_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory"); }

// Barrier among the softmax warps that also ANDs a flag over them.
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

// Parity to wait for before the n-th use (n >= slots) of a ring slot: the
// release of its previous use.
ELSAA_DEV uint32_t reuse_parity(int64_t n, int slots) { return (uint32_t)(((n / slots) - 1) & 1); }
ELSAA_DEV uint32_t use_parity(int64_t n, int slots) { return (uint32_t)((n / slots) & 1); }

// MR: the largest hash-round count the instance handles (1, or kMaxRounds
// for the several-round passes; the one-round instance keeps no per-round
// state in registers).
template <int D, int MR>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_win_kernel(const __grid_constant__ WinMaps maps, const int32_t* __restrict__ perm_q,
                    const int32_t* __restrict__ perm_k, int BH, int N, int chunk, int lookback,
                    int causal, float scale_log2, __nv_bfloat16* __restrict__ o_sp,
                    float* __restrict__ lse, const int32_t* __restrict__ rank, int round,
                    int64_t rank_len, const int32_t* __restrict__ kranks,
                    float* __restrict__ o_part, float* __restrict__ lse_part,
                    uint32_t* __restrict__ err) {
  using Lay = WinLayout<D>;
  constexpr int KS = Lay::kKSlots, VS = Lay::kVSlots, OB = Lay::kOBufs;
  constexpr uint32_t kTileBytes = Lay::kTileBytes;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  WinBars* bars = reinterpret_cast<WinBars*>(smem + Lay::kBar);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((sbase & 1023u) != 0) {
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  const int T = N / kTile;
  int64_t begin, count;
  {
    const int64_t ntiles = (int64_t)BH * T;
    begin = ntiles * blockIdx.x / gridDim.x;
    count = ntiles * (blockIdx.x + 1) / gridDim.x - begin;
  }
  auto tile = [&](int64_t j) { return win_tile(begin + j, T, N, chunk, lookback); };

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->full_q[s], kProducers);   // each producer warp's byte-count arrival
      mbar_init(&bars->empty_q[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->s_free[s], kSoftmaxThreads);
      mbar_init(&bars->p_full[s], kSoftmaxThreads);
      mbar_init(&bars->p_free[s], 1);
      mbar_init(&bars->o_full[s], 1);
      mbar_init(&bars->o_free[s], kSoftmaxThreads);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bars->full_k[s], kProducers);
      mbar_init(&bars->empty_k[s], 1);
      mbar_init(&bars->full_v[s], kProducers);
      mbar_init(&bars->empty_v[s], 1);
    }
    mbar_init(&bars->drain, 1);
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
    // Producer warp pw loads rows 32 pw .. 32 pw + 31 of every tile or block:
    // lane l < 8 takes rows 32 pw + 4 l .. + 3 (its four token indices in one
    // 16-byte load, prefetched one load ahead); lane 0 first arms the slot's
    // barrier with this warp's share of the bytes.
    const int pw = warp;
    const bool gl = lane < 8;
    const int rbase = 32 * pw + 4 * lane;   // first row of this lane
    // The load sequence: Q(0); then per tile j the pass-1 K blocks, Q(j + 1),
    // and the pass-2 blocks (K and V of a block share one index set).
    struct Item {
      int64_t j;   // tile (for a Q item: the tile whose Q it loads)
      int kind;    // 0 Q, 1 K of pass 1, 2 K and V of pass 2
      int b;       // block of the tile's window
    };
    auto next_item = [&](const Item& it) -> Item {
      if (it.kind == 0) return it.j == 0 ? Item{0, 1, 0} : Item{it.j - 1, 2, 0};
      if (it.b + 1 < tile(it.j).nb) return Item{it.j, it.kind, it.b + 1};
      if (it.kind == 1) return it.j + 1 < count ? Item{it.j + 1, 0, 0} : Item{it.j, 2, 0};
      return Item{it.j + 1, 1, 0};
    };
    auto item_rows = [&](const Item& it) -> int4 {
      const WinTile w = tile(it.j);
      const size_t unit = (size_t)w.bh * N;
      const size_t at = it.kind == 0 ? unit + (size_t)w.tb * kTile
                                     : unit + (size_t)(w.kb_lo + it.b) * kTile;
      const int32_t* perm = it.kind == 0 ? perm_q : perm_k;
      return gl ? *reinterpret_cast<const int4*>(perm + at + rbase) : make_int4(0, 0, 0, 0);
    };
    auto gather = [&](uint32_t dst, const CUtensorMap* map, int u, int4 t4, uint64_t* bar) {
      if (gl) {
#pragma unroll
        for (int a = 0; a < D / 64; ++a)
          tma_gather4_x(dst + a * kAtom + (uint32_t)rbase * 128, map, 64 * a, u + t4.x, u + t4.y,
                        u + t4.z, u + t4.w, bar);
      }
    };
    auto load = [&](uint64_t* full, uint64_t* empty, int slots, uint32_t region, int64_t n,
                    const CUtensorMap* map, int u, int4 t4) -> bool {
      const int s = (int)(n % slots);
      if (n >= slots &&
          !__all_sync(0xffffffffu, mbar_wait(&empty[s], reuse_parity(n, slots), err)))
        return false;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], kTileBytes / kProducers);
      __syncwarp();
      gather(sbase + region + (uint32_t)s * kTileBytes, map, u, t4, &full[s]);
      return true;
    };
    int64_t nk = 0, nv = 0;
    if (count > 0) {
      Item it{0, 0, 0};
      int4 t4 = item_rows(it);
      for (;;) {
        const bool last = it.kind == 2 && it.j + 1 == count && it.b + 1 == tile(it.j).nb;
        const Item nx = last ? it : next_item(it);
        const int4 n4 = last ? t4 : item_rows(nx);   // the next item's indices, in flight
        const int u = (int)((size_t)tile(it.j).bh * N);
        if (it.kind == 0) {
          ok = load(bars->full_q, bars->empty_q, 2, Lay::kQ, it.j, &maps.q, u, t4);
        } else if (it.kind == 1) {
          ok = load(bars->full_k, bars->empty_k, KS, Lay::kK, nk++, &maps.k, u, t4);
        } else {
          ok = load(bars->full_k, bars->empty_k, KS, Lay::kK, nk++, &maps.k, u, t4) &&
               load(bars->full_v, bars->empty_v, VS, Lay::kV, nv++, &maps.v, u, t4);
        }
        if (!ok || last) break;
        it = nx;
        t4 = n4;
      }
    }
    // every copy this warp started has landed before the CTA may exit (on the
    // normal path the consumers have already waited for all of them)
    if (lane == 0) {
      for (int64_t n = nk - 1; n >= 0 && n >= nk - KS; --n)
        mbar_wait(&bars->full_k[n % KS], use_parity(n, KS), err);
      for (int64_t n = nv - 1; n >= 0 && n >= nv - VS; --n)
        mbar_wait(&bars->full_v[n % VS], use_parity(n, VS), err);
    }
    __syncwarp();

  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(128, kTile, false, false);
      const uint32_t id_pv = idesc_bf16(128, D, false, true);
      const uint64_t q_d0 = sw128_desc(sbase + Lay::kQ, 16, 1024);
      const uint64_t k_d0 = sw128_desc(sbase + Lay::kK, 16, 1024);
      const uint64_t v_d0 = sw128_desc(sbase + Lay::kV, kAtom, 1024);
      int64_t ns = 0, np = 0;
      // S job ns: S[ns % 2] = Q K^T of the K load ns
      auto issue_s = [&](int64_t j) -> bool {
        const int sb = (int)(ns & 1);
        if (ns >= 2 && !mbar_wait(&bars->s_free[sb], reuse_parity(ns, 2), err)) return false;
        if (!mbar_wait(&bars->full_k[ns % KS], use_parity(ns, KS), err)) return false;
        fence_after();
        const uint64_t qd = desc_add(q_d0, (uint32_t)(j & 1) * kTileBytes);
        const uint64_t kd = desc_add(k_d0, (uint32_t)(ns % KS) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kAtom + (uint32_t)(kk & 3) * 32;
          mma_bf16_ss(tmem + kTS + sb * kTile, desc_add(qd, off), desc_add(kd, off), id_s,
                      kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[sb]);
        mma_commit(&bars->empty_k[ns % KS]);
        ++ns;
        return true;
      };
      // PV job np: O[o] (+)= P[np % 2] V of the V load np
      auto issue_pv = [&](int64_t j, bool first) -> bool {
        const int pb = (int)(np & 1), o = (int)(j % OB);
        if (!mbar_wait(&bars->p_full[pb], use_parity(np, 2), err)) return false;
        if (!mbar_wait(&bars->full_v[np % VS], use_parity(np, VS), err)) return false;
        if (first && j >= OB && !mbar_wait(&bars->o_free[o], reuse_parity(j, OB), err))
          return false;
        fence_after();
        const uint64_t vd = desc_add(v_d0, (uint32_t)(np % VS) * kTileBytes);
#pragma unroll
        for (int x = 0; x < kTile; x += 16)
          mma_bf16_ts(tmem + kTO + (uint32_t)(o * D), tmem + kTP + (uint32_t)(pb * 64 + (x >> 1)),
                      desc_add(vd, (uint32_t)(x >> 4) * 2048), id_pv, (!first || x > 0) ? 1u : 0u);
        mma_commit(&bars->p_free[pb]);
        mma_commit(&bars->empty_v[np % VS]);
        ++np;
        return true;
      };
      for (int64_t j = 0; j < count && ok; ++j) {
        const WinTile w = tile(j);
        ok = mbar_wait(&bars->full_q[j & 1], use_parity(j, 2), err);
        for (int b = 0; b < w.nb && ok; ++b) ok = issue_s(j);   // pass 1
        for (int b = 0; b < w.nb && ok; ++b) {                  // pass 2, S one block ahead
          ok = issue_s(j);
          if (ok && b + 1 == w.nb) mma_commit(&bars->empty_q[j & 1]);
          if (ok && b > 0) ok = issue_pv(j, b == 1);
        }
        if (ok) ok = issue_pv(j, w.nb == 1);
        if (ok) mma_commit(&bars->o_full[j % OB]);
      }
      // the MMAs issued so far have completed before TMEM is freed
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, err);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int quarter = warp & 3, half = (warp - kSoftmaxWarp0) >> 2;
    const int row = 32 * quarter + lane;   // TMEM lane = query row of the tile
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    float* red_m = reinterpret_cast<float*>(smem + Lay::kRed);   // [2][128]
    float* red_l = red_m + 2 * 128;                              // [2][128]
    const bool masked = causal || round > 0 || chunk % kTile != 0;
    const int64_t rows = (int64_t)BH * N, rstride = 2 * rows;   // rank: [R][2][BH][N]
    int64_t ns = 0, np = 0;
    for (int64_t j = 0; j < count; ++j) {
      const WinTile w = tile(j);
      const size_t unit = (size_t)w.bh * N;
      const int r = w.tb * kTile + row;
      const int token = perm_q[unit + r];
      const int jr = r / chunk;
      // the row's window in columns of the tile's first block
      const int lo = max(0, (jr - lookback) * chunk) - w.kb_lo * kTile;
      const int hi = (jr + 1) * chunk - w.kb_lo * kTile;
      const int cb = half * 64;   // this thread's 64 columns of every block
      // the query's windows in the earlier rounds (several hash rounds)
      int wlo[MR], whi[MR];
#pragma unroll
      for (int u = 0; u < MR; ++u) {
        wlo[u] = whi[u] = 0;
        if (u < round) {
          const int64_t at = u * rstride + (int64_t)unit + token;
          if (at < 0 || at >= rank_len || token < 0 || token >= N) {   // checked: never taken
            raise_error(err, ERR_CHECK);
            continue;
          }
          const int ju = rank[at] / chunk;
          wlo[u] = max(0, (ju - lookback) * chunk);
          whi[u] = min(N, (ju + 1) * chunk);
        }
      }
      // bit e: column cb + e of block b is a key of the row (its window; with
      // the causal mask, a token index at most the query's; with several
      // rounds, not in an earlier round's window of the query)
      auto allow_bits = [&](int b) -> uint64_t {
        const int c0 = b * kTile + cb;
        const int a = max(0, lo - c0), z = min(64, hi - c0);
        if (a >= z) return 0ull;
        uint64_t bits = (z == 64 ? ~0ull : (1ull << z) - 1ull) & ~((1ull << a) - 1ull);
        const size_t pos = unit + (size_t)(w.kb_lo + b) * kTile + cb;   // sorted key position
        if (causal) {
          const int4* kt = reinterpret_cast<const int4*>(perm_k + pos);
          uint64_t c = 0;
#pragma unroll 2
          for (int e4 = 0; e4 < 16; ++e4) {
            const int4 t = __ldg(kt + e4);
            c |= ((uint64_t)(t.x <= token) | (uint64_t)(t.y <= token) << 1 |
                  (uint64_t)(t.z <= token) << 2 | (uint64_t)(t.w <= token) << 3)
                 << (4 * e4);
          }
          bits &= c;
        }
#pragma unroll
        for (int u = 0; u < MR; ++u) {
          if (u >= round) break;
          const int4* kr = reinterpret_cast<const int4*>(kranks + u * rows + pos);
          const int lo_u = wlo[u], hi_u = whi[u];
          auto in = [&](int x) { return (uint64_t)(x >= lo_u && x < hi_u); };
          uint64_t sb = 0;
#pragma unroll 2
          for (int e4 = 0; e4 < 16; ++e4) {
            const int4 t = __ldg(kr + e4);
            sb |= (in(t.x) | in(t.y) << 1 | in(t.z) << 2 | in(t.w) << 3) << (4 * e4);
          }
          bits &= ~sb;
        }
        return bits;
      };
      // pass 1: row maximum
      float m = -INFINITY;
      for (int b = 0; b < w.nb; ++b) {
        const int sb = (int)(ns & 1);
        ok = softmax_all(mbar_wait(&bars->s_full[sb], use_parity(ns, 2), err));
        if (!ok) break;
        fence_after();
        float sv[64];
        tmem_ld32(tmem + kTS + sb * kTile + lane_off + cb, sv);
        tmem_ld32(tmem + kTS + sb * kTile + lane_off + cb + 32, sv + 32);
        tmem_ld_wait();
        fence_before();
        mbar_arrive(&bars->s_free[sb]);
        ++ns;
        if (masked) {
          const uint64_t al = allow_bits(b);
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if ((al >> e) & 1ull) m = fmaxf(m, sv[e]);
        } else {
#pragma unroll
          for (int e = 0; e < 64; ++e) m = fmaxf(m, sv[e]);
        }
      }
      if (!ok) break;
      red_m[half * 128 + row] = m;
      softmax_sync();
      m = fmaxf(m, red_m[(half ^ 1) * 128 + row]) * scale_log2;   // scale > 0
      // pass 2: P = exp2(scale log2e s - m) into TMEM, row sum
      float l = 0.f;
      for (int b = 0; b < w.nb; ++b) {
        const int sb = (int)(ns & 1), pb = (int)(np & 1);
        ok = softmax_all(mbar_wait(&bars->s_full[sb], use_parity(ns, 2), err) &&
                         (np < 2 || mbar_wait(&bars->p_free[pb], reuse_parity(np, 2), err)));
        if (!ok) break;
        fence_after();
        const uint64_t al = masked ? allow_bits(b) : ~0ull;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float sv[32];
          tmem_ld32(tmem + kTS + sb * kTile + lane_off + cb + 32 * h, sv);
          tmem_ld_wait();
          uint32_t packed[16];
          float l0 = 0.f, l1 = 0.f;
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float a0 = sv[e], a1 = sv[e + 1];
            fma2(a0, a1, scale_log2, scale_log2, -m, -m);
            float p0 = ex2(a0), p1 = ex2(a1);
            if (masked) {
              p0 = ((al >> (32 * h + e)) & 1ull) ? p0 : 0.f;
              p1 = ((al >> (32 * h + e + 1)) & 1ull) ? p1 : 0.f;
            }
            add2(l0, l1, p0, p1);
            const __nv_bfloat162 hv = __floats2bfloat162_rn(p0, p1);
            packed[e >> 1] = *reinterpret_cast<const uint32_t*>(&hv);
          }
          l += l0 + l1;
          // keys cb + 32 h .. +31 of the block: P columns (cb + 32 h) / 2 ..
          tmem_st16(tmem + kTP + (uint32_t)(pb * 64 + ((cb + 32 * h) >> 1)) + lane_off, packed);
        }
        tmem_st_wait();
        fence_before();
        mbar_arrive(&bars->s_free[sb]);
        mbar_arrive(&bars->p_full[pb]);
        ++ns;
        ++np;
      }
      if (!ok) break;
      red_l[half * 128 + row] = l;
      softmax_sync();
      l += red_l[(half ^ 1) * 128 + row];
      // epilogue: each half writes D / 2 columns of the row
      const int o = (int)(j % OB);
      ok = softmax_all(mbar_wait(&bars->o_full[o], use_parity(j, OB), err));
      if (!ok) break;
      fence_after();
      const float inv = l > 0.f ? 1.0f / l : 0.f;   // l = 0: a row without keys
      __nv_bfloat16* orow = o_sp + (unit + token) * D;
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        const int c0 = half * (D / 2) + 32 * h;
        float ov[32];
        tmem_ld32(tmem + kTO + (uint32_t)(o * D + c0) + lane_off, ov);
        tmem_ld_wait();
        if (o_part != nullptr) {   // a round's partial, fp32
          float* prow = o_part + (unit + token) * D + c0;
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            *reinterpret_cast<float4*>(prow + 4 * q4) =
                make_float4(ov[4 * q4] * inv, ov[4 * q4 + 1] * inv, ov[4 * q4 + 2] * inv,
                            ov[4 * q4 + 3] * inv);
          continue;
        }
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 hv =
                __floats2bfloat162_rn(ov[q8 * 8 + 2 * e] * inv, ov[q8 * 8 + 2 * e + 1] * inv);
            w4[e] = *reinterpret_cast<const uint32_t*>(&hv);
          }
          *reinterpret_cast<uint4*>(orow + c0 + q8 * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      if (half == 0)
        (o_part != nullptr ? lse_part : lse)[unit + token] =
            l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
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

template <int D, int MR>
cudaError_t launch(const Geometry& g, const void* q, const void* k, const void* v,
                   const int32_t* perm_q, const int32_t* perm_k, void* o_sp, float* lse,
                   const int32_t* rank, int round, const int32_t* kranks, float* o_part,
                   float* lse_part, uint32_t* err, cudaStream_t s) {
  using Lay = WinLayout<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_win_kernel<D, MR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Lay::kDyn);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntiles = (int64_t)g.BH * (g.N / kTile);
  const int grid_x = (int)(ntiles < sms ? ntiles : sms);
  WinMaps maps;
  const uint64_t rows = (uint64_t)g.BH * g.N;
  if ((e = make_row_map(&maps.q, q, rows, D)) != cudaSuccess) return e;
  if ((e = make_row_map(&maps.k, k, rows, D)) != cudaSuccess) return e;
  if ((e = make_row_map(&maps.v, v, rows, D)) != cudaSuccess) return e;
  attn_fwd_win_kernel<D, MR><<<grid_x, kThreads, Lay::kDyn, s>>>(
      maps, perm_q, perm_k, g.BH, g.N, g.chunk, g.lookback, g.causal ? 1 : 0,
      g.scale * 1.4426950408889634f, static_cast<__nv_bfloat16*>(o_sp), lse, rank, round,
      (int64_t)g.rounds * 2 * g.BH * g.N, kranks, o_part, lse_part, err);
  return cudaGetLastError();
}

// O_sp and lse of the union of the rounds' windows from the rounds' partials:
// lse = log sum_t exp(lse_t), O = sum_t exp(lse_t - lse) O_t (rows without keys
// in every round: O = 0, lse = -inf).  One warp per row, lanes over d.
__global__ void __launch_bounds__(256)
round_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                     int R, int64_t rows, int d, __nv_bfloat16* __restrict__ o_sp,
                     float* __restrict__ lse) {
  const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int64_t r = (int64_t)blockIdx.x * nw + (threadIdx.x >> 5); r < rows;
       r += (int64_t)gridDim.x * nw) {
    float m = -INFINITY;
    for (int t = 0; t < R; ++t) m = fmaxf(m, lse_part[t * rows + r]);
    if (m == -INFINITY) {
      for (int e = lane; e < d; e += 32) o_sp[r * d + e] = __float2bfloat16_rn(0.f);
      if (lane == 0) lse[r] = -INFINITY;
      continue;
    }
    float z = 0.f;
    for (int t = 0; t < R; ++t) z += expf(lse_part[t * rows + r] - m);
    const float lz = m + logf(z);
    for (int e = lane; e < d; e += 32) {
      float acc = 0.f;
      for (int t = 0; t < R; ++t) {
        const float wt = expf(lse_part[t * rows + r] - lz);
        acc += wt * o_part[(t * rows + r) * d + e];
      }
      o_sp[r * d + e] = __float2bfloat16_rn(acc);
    }
    if (lane == 0) lse[r] = lz;
  }
}

// For round pairs u < t: the rank in round u of round t's sorted key pos,
// kranks[(t (t - 1) / 2 + u) rows + unit + pos] = rank_k[u][unit + perm_k[t][unit + pos]]
// (perm and rank: [R][2][BH][N], token indices within the unit).
__global__ void __launch_bounds__(256)
round_key_ranks_kernel(const int32_t* __restrict__ perm, const int32_t* __restrict__ rank,
                       int R, int64_t rows, int N, int32_t* __restrict__ kranks) {
  const int64_t total = (int64_t)R * (R - 1) / 2 * rows;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t pair = i / rows, x = i - pair * rows;
    int t = 1;
    while ((int64_t)t * (t + 1) / 2 <= pair) ++t;   // pairs t (t - 1) / 2 .. t (t + 1) / 2 - 1
    const int u = (int)(pair - (int64_t)t * (t - 1) / 2);
    const int64_t unit = x / N * N;
    const int key = perm[(int64_t)t * 2 * rows + rows + x];
    kranks[i] = rank[(int64_t)u * 2 * rows + rows + unit + key];
  }
}

}  // namespace

bool attn_win_supported(const Geometry& g) {
  // TMA row coordinates are 32-bit
  return g.bf16 && (g.d == 64 || g.d == 128) && g.N % kTile == 0 && g.chunk % 16 == 0 &&
         g.N % g.chunk == 0 && g.lookback >= 0 && g.rounds >= 1 && g.rounds <= kMaxRounds &&
         (int64_t)g.BH * g.N < (int64_t)1 << 31;
}

cudaError_t launch_attn_fwd_win(const Geometry& g, const void* q, const void* k, const void* v,
                                const int32_t* perm_q, const int32_t* perm_k, void* o_sp,
                                float* lse, uint32_t* err, cudaStream_t s) {
  return g.d == 64 ? launch<64, 1>(g, q, k, v, perm_q, perm_k, o_sp, lse, nullptr, 0, nullptr,
                                   nullptr, nullptr, err, s)
                   : launch<128, 1>(g, q, k, v, perm_q, perm_k, o_sp, lse, nullptr, 0, nullptr,
                                    nullptr, nullptr, err, s);
}

cudaError_t launch_attn_fwd_win_rounds(const Geometry& g, const void* q, const void* k,
                                       const void* v, const int32_t* perm, const int32_t* rank,
                                       int32_t* kranks, float* o_part, float* lse_part,
                                       void* o_sp, float* lse, uint32_t* err, cudaStream_t s) {
  const int64_t rows = (int64_t)g.BH * g.N;
  const int64_t total = (int64_t)g.rounds * (g.rounds - 1) / 2 * rows;
  const int64_t want = (total + 255) / 256;
  round_key_ranks_kernel<<<(int)(want < 148 * 32 ? want : 148 * 32), 256, 0, s>>>(
      perm, rank, g.rounds, rows, g.N, kranks);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  for (int t = 0; t < g.rounds; ++t) {
    const int32_t* pq = perm + (size_t)t * 2 * rows;
    const int32_t* kr = kranks + (size_t)t * (t - 1) / 2 * rows;
    float* op = o_part + (size_t)t * rows * g.d;
    float* lp = lse_part + (size_t)t * rows;
    e = g.d == 64 ? launch<64, kMaxRounds>(g, q, k, v, pq, pq + rows, o_sp, lse, rank, t, kr, op,
                                           lp, err, s)
                  : launch<128, kMaxRounds>(g, q, k, v, pq, pq + rows, o_sp, lse, rank, t, kr, op,
                                            lp, err, s);
    if (e != cudaSuccess) return e;
  }
  const int64_t wc = (rows + 7) / 8;
  const int grid = (int)(wc < 148 * 16 ? wc : 148 * 16);
  round_combine_kernel<<<grid, 256, 0, s>>>(o_part, lse_part, g.rounds, rows, g.d,
                                            static_cast<__nv_bfloat16*>(o_sp), lse);
  return cudaGetLastError();
}

}  // namespace elsaa
