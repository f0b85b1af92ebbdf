// RACE query-side read-out from tables resident in shared memory.
//
// "Two Efficient Attentions, One Denominator Problem" (section "Two efficient
// branches can still be mis-scaled"): every query reads its bucket in each of
// the L RACE tables; the bucket sums give it global context, O_race =
// sum_l T[l][h_l(q)] / Ctot with Ctot = sum_l C[l][h_l(q)], and its RACE mass
// Z_race = Ctot / L enters the denominator-aware fusion
//   m = Z_sp / (Z_sp + lambda Z_race),   y = g_s m O_sp + g_r O_race.
// The same gather, by key codes over the table gradient, is the value
// gradient of the RACE branch: dv_j += sum_l dT[l][h_l(k_j)].
//
// A unit's bf16 tables (L x 2^K_r rows of d values) do not fit in one SM's
// shared memory, but a slab of 8 columns of every table does (32 x 256 x 16 B
// = 128 KB at L = 32, K_r = 8).  A CTA holds the slab of NSUB 8-column groups
// of one unit (NSUB = d / 8 where the whole table fits) and reads it for every
// query of a block: one thread per query, 16 bytes per table.
//
// Bank conflicts: a 16-byte shared load is served 8 lanes at a time, and 8
// lanes reading random buckets of one table would collide on banks.  The slab
// interleaves 16 tables per bucket (16-byte slot ((t / 16) NB + b) 16 + t % 16,
// so a bucket row is 256 bytes and the slot's bank group is t % 8), and lane r
// of each group of 8 walks the tables of an octet starting at table r: the 8
// lanes of a phase always read 8 different tables, hence 8 different bank
// groups, whatever their buckets.  Lanes 8g .. 8g + 7 also start at octet g,
// so a warp's 32 lanes read 32 different tables in every step, and the bucket
// counts (laid out [b][64], bank = table) are conflict-free too.  The rotation
// is applied once per query to its code bytes (a selection of octets and a
// funnel shift); one byte permute per step then yields the bucket row offset.
//
// Row pieces (one CTA per column group): every warp moves its 32 rows' 16-byte
// pieces of O_sp, y and O_race (or of dv) through its own TMA boxes, loaded
// under the gather and stored from shared memory, with its own mbarriers.
//
// Work: persistent CTAs (one per SM) in teams of G, one CTA per column group;
// a team walks a contiguous run of (unit, block of 1024 queries) items, so a
// CTA reloads its slab only when its run enters another unit, and the G CTAs
// that write the column groups of one row do so at about the same time (each
// writes 16 bytes of a 128-byte row: the row's sectors fill up in L2 before
// they are written back).
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace elsaa {
namespace {

constexpr int kSlabThreads = 1024;
constexpr int kSlabSmemMax = 200 * 1024;     // slab and counts
constexpr int kSlabSmemLimit = 227 * 1024;   // with the row tiles

// Shared memory of one CTA: the slab, the bucket counts (fuse), the row tiles
// (one column group per CTA: three tiles to fuse, two to add) and two
// mbarriers; the offsets are computed here once and passed to the kernel.
struct SlabShape {
  int oct, nsub, groups, qblocks;
  uint32_t cnt_off, tiles_off, bars_off;
  size_t smem;
};

// FUSE: forward read-out fused with the gates, the multiplier and the output.
// ADD: dst[j] += the gathered sums (the value gradient of the RACE branch).
enum SlabMode { kFuse = 0, kAdd = 1 };

ELSAA_DEV uint4 pack_bf16x8(const float* v) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

ELSAA_DEV void unpack_bf16x8(uint4 raw, float* v) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Codes of one row (OCT octets of 8 one-byte codes) rotated for this lane:
// byte e of oc[u] is the code of table 8 ((u + g) % OCT) + ((e + r) % 8).
template <int OCT>
ELSAA_DEV void rotate_codes(const uint32_t* w, int g, int r, uint32_t (&lo)[OCT],
                            uint32_t (&hi)[OCT]) {
#pragma unroll
  for (int u = 0; u < OCT; ++u) {
    lo[u] = w[2 * u];
    hi[u] = w[2 * u + 1];
  }
  if constexpr (OCT == 4) {
    const bool s2 = (g & 2) != 0, s1 = (g & 1) != 0;
    uint32_t l2[4], h2[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      l2[u] = s2 ? lo[(u + 2) & 3] : lo[u];
      h2[u] = s2 ? hi[(u + 2) & 3] : hi[u];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      lo[u] = s1 ? l2[(u + 1) & 3] : l2[u];
      hi[u] = s1 ? h2[(u + 1) & 3] : h2[u];
    }
  } else if constexpr (OCT == 2) {
    const bool s1 = (g & 1) != 0;
    const uint32_t l0 = lo[0], h0 = hi[0];
    lo[0] = s1 ? lo[1] : lo[0];
    hi[0] = s1 ? hi[1] : hi[0];
    lo[1] = s1 ? l0 : lo[1];
    hi[1] = s1 ? h0 : hi[1];
  }
  // rotate each octet right by r bytes
  const bool sw = (r & 4) != 0;
  const uint32_t sh = 8u * (uint32_t)(r & 3);
#pragma unroll
  for (int u = 0; u < OCT; ++u) {
    const uint32_t a = sw ? hi[u] : lo[u], b = sw ? lo[u] : hi[u];
    lo[u] = __funnelshift_r(a, b, sh);
    hi[u] = __funnelshift_r(b, a, sh);
  }
}

// acc[0..8) += the 8 bf16 values of a 16-byte line, by mixed-precision adds
// (bf16 operand, fp32 accumulator: the same rounded sums as converting to fp32
// first, in fewer instructions)
ELSAA_DEV void add_line_mixed(float* acc, uint4 raw) {
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

// One row's OCT octets of one-byte codes as 2 OCT words.
template <int OCT>
ELSAA_DEV void load_codes(const uint8_t* __restrict__ codes, size_t row, uint32_t* w) {
  const uint4* cp = reinterpret_cast<const uint4*>(codes + row * (8 * OCT));
#pragma unroll
  for (int v4 = 0; v4 < OCT / 2; ++v4) {
    const uint4 c4 = cp[v4];
    w[4 * v4] = c4.x;
    w[4 * v4 + 1] = c4.y;
    w[4 * v4 + 2] = c4.z;
    w[4 * v4 + 3] = c4.w;
  }
}

template <int MODE, int OCT, int NSUB>
__global__ void __launch_bounds__(kSlabThreads, 1)
race_slab_kernel(const uint8_t* __restrict__ codes, const __nv_bfloat16* __restrict__ tables,
                 const int32_t* __restrict__ counts, int BH, int N, int d, int NB, int groups,
                 int qblocks, uint32_t cnt_off, uint32_t tiles_off, uint32_t bars_off,
                 const __grid_constant__ CUtensorMap map_a,
                 const __grid_constant__ CUtensorMap map_y,
                 const __grid_constant__ CUtensorMap map_r, int has_orace,
                 const __nv_bfloat16* __restrict__ o_sp, const float* __restrict__ lse,
                 const float2* __restrict__ gl, const float* __restrict__ gate_b, int gate_fixed,
                 float gs_fixed, float gr_fixed, const float* __restrict__ lam,
                 __nv_bfloat16* __restrict__ y, __nv_bfloat16* __restrict__ o_race,
                 int32_t* __restrict__ ctot_out, __nv_bfloat16* __restrict__ dst,
                 uint32_t* __restrict__ err) {
  static_assert(OCT == 2 || OCT == 4, "16 or 32 tables");
  constexpr int L = 8 * OCT;
  // one 8-column group per CTA: each warp moves its 32 rows' pieces through
  // its own TMA boxes (512 bytes), so no barrier couples the warps
  constexpr bool kTiles = NSUB == 1;
  constexpr uint32_t kSlot = 32 * 16;                    // one warp's rows x 16 bytes
  constexpr uint32_t kSlots = kSlabThreads / 32 * kSlot;  // one tile: every warp's slot
  extern __shared__ __align__(128) uint8_t sm[];
  const uint32_t sub_bytes = (uint32_t)L * NB * 16;
  uint8_t* tab = sm;                                                  // [NSUB][L/16][NB][16][16 B]
  int32_t* cnt = reinterpret_cast<int32_t*>(sm + cnt_off);            // [NB][32] (fuse)
  // fuse: O_sp in, y out, O_race out; add: two buffers of dst rows
  uint8_t* tiles = sm + tiles_off;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + bars_off);        // [2][warps]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = (lane >> 3) % OCT, r = lane & 7;
  const uint32_t tab_s = tc::smem_u32(tab);
  const uint32_t cnt_s = tc::smem_u32(cnt);
  const uint32_t tiles_s = tc::smem_u32(tiles);
  // lane constants: where octet (u + g) % OCT starts in a bucket row of the
  // slab (and in a row of counts, at half that stride), and the slot of step
  // e, (e + r) % 8
  uint32_t abase[OCT], cbase[OCT], roff[8];
#pragma unroll
  for (int u = 0; u < OCT; ++u) {
    const int ou = (u + g) % OCT;
    abase[u] = tab_s + (uint32_t)(ou >> 1) * NB * 256u + (uint32_t)(ou & 1) * 128u;
    cbase[u] = cnt_s + (uint32_t)ou * 32u;   // 4 bytes x 8 tables per octet
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) roff[e] = 16u * (uint32_t)((e + r) & 7);
  float lam_v = 0.f, bs = 0.f, br = 0.f;
  if (MODE == kFuse) {
    lam_v = *lam;
    if (!gate_fixed) {
      bs = gate_b[0];
      br = gate_b[1];
    }
  }
  const float inv_L = 1.0f / (float)L;
  if (kTiles && lane == 0) {
    tc::mbar_init(&bars[warp], 1);
    tc::mbar_init(&bars[kSlabThreads / 32 + warp], 1);
    tc::fence_mbar_init();
  }
  __syncthreads();

  // team blockIdx.x / groups, column group blockIdx.x % groups
  const int grp = (int)(blockIdx.x % groups);
  const int teams = (int)(gridDim.x / groups), team = (int)(blockIdx.x / groups);
  const int64_t items = (int64_t)BH * qblocks;
  const int64_t beg = items * team / teams;
  const int64_t end = items * (team + 1) / teams;
  const int c0 = grp * NSUB * 8;   // first column of the group
  int loaded = -1;
  // blocks in which this warp had rows (and so moved a TMA box): picks the
  // buffer (add) and the mbarrier phase
  uint32_t n = 0;
  // the row this thread reads in item `it` (row 0 of its unit past the end)
  auto row_of = [&](int64_t it) -> size_t {
    const int unit = (int)(it / qblocks);
    const int i = (int)(it - (int64_t)unit * qblocks) * kSlabThreads + tid;
    return (size_t)unit * N + (i < N ? i : 0);
  };
  uint32_t wnext[2 * OCT];
  if (beg < end) load_codes<OCT>(codes, row_of(beg), wnext);
  for (int64_t it = beg; it < end; ++it) {
    const int unit = (int)(it / qblocks);
    const int qb = (int)(it - (int64_t)unit * qblocks);
    if (unit != loaded) {
      __syncthreads();   // every thread is done with the previous slab
      // slab: sub-group s, table t, bucket b -> slot ((t / 16) NB + b) 16 + t % 16,
      // visited in slot order (conflict-free stores)
      const int lines = NSUB * L * NB;
      for (int x = tid; x < lines; x += kSlabThreads) {
        const int sg = x / (L * NB), rem = x - sg * (L * NB);
        const int h = rem / (16 * NB), rem2 = rem - h * (16 * NB);
        const int b = rem2 >> 4, t = h * 16 + (rem2 & 15);
        const uint4 v = *reinterpret_cast<const uint4*>(
            tables + (((size_t)unit * L + t) * NB + b) * d + c0 + sg * 8);
        *reinterpret_cast<uint4*>(tab + (size_t)x * 16) = v;
      }
      if (MODE == kFuse)
        for (int x = tid; x < NB * 32; x += kSlabThreads) {
          const int b = x >> 5, t = x & 31;
          if (t < L) cnt[x] = counts[((size_t)unit * L + t) * NB + b];
        }
      __syncthreads();
      loaded = unit;
    }
    const int i0 = qb * kSlabThreads + warp * 32, i = i0 + lane;   // i0: the warp's first row
    const bool valid = i < N;
    const size_t row = (size_t)unit * N + (valid ? i : 0);
    const uint32_t buf = MODE == kAdd ? (n & 1u) : 0u;
    uint64_t* bar = &bars[buf * (kSlabThreads / 32) + warp];
    const uint32_t slot_in = tiles_s + buf * kSlots + (uint32_t)warp * kSlot;
    if (kTiles && lane == 0 && i0 < N) {
      // the warp's rows of O_sp (fuse) or dst (add), under the gather
      if (MODE == kAdd) tc::bulk_wait_read<1>();   // the store two boxes back has read the slot
      tc::mbar_arrive_expect_tx(bar, kSlot);
      tc::tma_load_3d(slot_in, &map_a, c0, i0, unit, bar);
    }
    // this row's codes (loaded one block ahead), rotated for the lane; the
    // next block's row codes go out now, under this block's gather
    uint32_t clo[OCT], chi[OCT];
    rotate_codes<OCT>(wnext, g, r, clo, chi);
    if (it + 1 < end) load_codes<OCT>(codes, row_of(it + 1), wnext);
    // per-row scalars of the read-out, also ahead of the gather
    float lse_r = 0.f;
    float2 gl_r = make_float2(0.f, 0.f);
    if (MODE == kFuse && valid) {
      lse_r = lse[row];
      if (!gate_fixed) gl_r = gl[row];
    }
    int ctot = 0;
    float inv = 0.f, gs = gs_fixed, gr = gr_fixed, m = 1.f;
#pragma unroll 1
    for (int s = 0; s < NSUB; ++s) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const uint32_t soff = (uint32_t)s * sub_bytes;
#pragma unroll
      for (int u = 0; u < OCT; ++u) {
        const uint32_t base = abase[u] + soff;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          // bucket b of this step's table, as the row offset b * 256
          const uint32_t brow =
              __byte_perm(e < 4 ? clo[u] : chi[u], 0, 0x4404u | ((uint32_t)(e & 3) << 4));
          uint4 v;
          asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(base + brow + roff[e]));
          add_line_mixed(acc, v);
          if (MODE == kFuse && s == 0) {
            int c;
            asm volatile("ld.shared.b32 %0, [%1];"
                         : "=r"(c)
                         : "r"(cbase[u] + (brow >> 1) + (roff[e] >> 2)));
            ctot += c;
          }
        }
      }
      if (MODE == kFuse && s == 0 && valid) {
        inv = ctot > 0 ? __fdividef(1.0f, (float)ctot) : 0.f;
        if (!gate_fixed) {
          gs = __fdividef(1.0f, 1.0f + __expf(-(gl_r.x + bs)));
          gr = __fdividef(1.0f, 1.0f + __expf(-(gl_r.y + br)));
        }
        // m = Z_sp / (Z_sp + lambda Z_race) = 1 / (1 + exp(log(lambda Z_race) - lse))
        const float lz = lam_v * (float)ctot * inv_L;
        m = lz > 0.f ? __fdividef(1.0f, 1.0f + __expf(__logf(lz) - lse_r)) : 1.0f;
        if (ctot_out != nullptr && grp == 0) ctot_out[row] = ctot;
      }
      if constexpr (kTiles) {
        if (i0 < N) {   // warp-uniform: a warp entirely past N has nothing to move
          if (MODE == kFuse) {
            if (lane == 0) tc::bulk_wait_read<0>();   // the last block's stores read y / O_race
            __syncwarp();
          }
          // a wait that runs out leaves the error word set (the rows are then garbage)
          tc::mbar_wait(bar, (MODE == kAdd ? (n >> 1) : n) & 1u, err);
          uint4* slot = reinterpret_cast<uint4*>(tiles + buf * kSlots + warp * kSlot) + lane;
          const uint32_t slot_y = tiles_s + kSlots + (uint32_t)warp * kSlot;
          const uint32_t slot_r = tiles_s + 2 * kSlots + (uint32_t)warp * kSlot;
          if (MODE == kFuse) {
            float os[8], yv[8], orc[8];
            unpack_bf16x8(*slot, os);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              orc[e] = acc[e] * inv;
              yv[e] = gs * m * os[e] + gr * orc[e];
            }
            reinterpret_cast<uint4*>(tiles + kSlots + warp * kSlot)[lane] = pack_bf16x8(yv);
            reinterpret_cast<uint4*>(tiles + 2 * kSlots + warp * kSlot)[lane] = pack_bf16x8(orc);
          } else {
            float cur[8];
            unpack_bf16x8(*slot, cur);
#pragma unroll
            for (int e = 0; e < 8; ++e) cur[e] += acc[e];
            *slot = pack_bf16x8(cur);
          }
          tc::fence_async_smem();   // the slots' generic writes, before the async-proxy stores
          __syncwarp();
          if (lane == 0) {
            if (MODE == kFuse) {
              tc::tma_store_3d(&map_y, c0, i0, unit, slot_y);
              if (has_orace) tc::tma_store_3d(&map_r, c0, i0, unit, slot_r);
            } else {
              tc::tma_store_3d(&map_a, c0, i0, unit, slot_in);
            }
            tc::bulk_commit();
          }
          ++n;
        }
      } else if (valid) {
        const size_t off = row * d + (size_t)(c0 + s * 8);
        if (MODE == kFuse) {
          float os[8], yv[8], orc[8];
          unpack_bf16x8(*reinterpret_cast<const uint4*>(o_sp + off), os);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            orc[e] = acc[e] * inv;
            yv[e] = gs * m * os[e] + gr * orc[e];
          }
          *reinterpret_cast<uint4*>(y + off) = pack_bf16x8(yv);
          if (o_race != nullptr) *reinterpret_cast<uint4*>(o_race + off) = pack_bf16x8(orc);
        } else {
          float cur[8];
          uint4* p = reinterpret_cast<uint4*>(dst + off);
          unpack_bf16x8(*p, cur);
#pragma unroll
          for (int e = 0; e < 8; ++e) cur[e] += acc[e];
          *p = pack_bf16x8(cur);
        }
      }
    }
  }
  if (kTiles && lane == 0) tc::bulk_wait<0>();   // every store has completed
}

SlabShape slab_shape(const Geometry& g, int mode) {
  SlabShape s{};
  s.oct = g.L / 8;
  const size_t sub = (size_t)g.L * g.NB * 16;
  const size_t cnt = mode == kFuse ? (size_t)g.NB * 32 * 4 : 0;
  const int ngroups8 = g.d / 8;
  s.nsub = 0;
  for (int n = ngroups8; n >= 1; n >>= 1)
    if (ngroups8 % n == 0 && n * sub + cnt <= (size_t)kSlabSmemMax) {
      s.nsub = n;
      break;
    }
  if (s.nsub == 0) return s;
  s.groups = ngroups8 / s.nsub;
  s.qblocks = (g.N + kSlabThreads - 1) / kSlabThreads;
  const size_t tiles = s.nsub == 1 ? (size_t)(mode == kFuse ? 3 : 2) * kSlabThreads * 16 : 0;
  s.cnt_off = (uint32_t)(s.nsub * sub);
  s.tiles_off = (uint32_t)(s.cnt_off + cnt);
  s.bars_off = (uint32_t)(s.tiles_off + tiles);
  s.smem = (size_t)s.bars_off + 2 * (kSlabThreads / 32) * sizeof(uint64_t);
  if (s.smem > (size_t)kSlabSmemLimit) s.nsub = 0;
  return s;
}

template <int MODE, int OCT, int NSUB>
cudaError_t launch(const Geometry& g, const SlabShape& sh, const void* codes, const void* tables,
                   const int32_t* counts, const void* o_sp, const float* lse, const float2* gl,
                   const float* gate_b, const float* lam, void* y, void* o_race, int32_t* ctot,
                   void* dst, uint32_t* err, cudaStream_t s) {
  auto kernel = race_slab_kernel<MODE, OCT, NSUB>;
  CUtensorMap map_a{}, map_y{}, map_r{};
  if (NSUB == 1) {
    const void* a = MODE == kFuse ? o_sp : dst;
    cudaError_t e = make_slab_map(&map_a, a, g.BH, g.N, g.d, 32);
    if (e == cudaSuccess && MODE == kFuse) e = make_slab_map(&map_y, y, g.BH, g.N, g.d, 32);
    if (e == cudaSuccess && MODE == kFuse && o_race != nullptr)
      e = make_slab_map(&map_r, o_race, g.BH, g.N, g.d, 32);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sh.smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // whole teams of sh.groups CTAs, at most one team per work item
  const int64_t items = (int64_t)g.BH * sh.qblocks;
  int64_t teams = sms / sh.groups;
  if (teams < 1) teams = 1;
  if (teams > items) teams = items;
  const int grid = (int)(teams * sh.groups);
  kernel<<<grid, kSlabThreads, sh.smem, s>>>(
      static_cast<const uint8_t*>(codes), static_cast<const __nv_bfloat16*>(tables), counts,
      g.BH, g.N, g.d, g.NB, sh.groups, sh.qblocks, sh.cnt_off, sh.tiles_off, sh.bars_off, map_a,
      map_y, map_r, o_race != nullptr ? 1 : 0,
      static_cast<const __nv_bfloat16*>(o_sp), lse, gl, gate_b, g.gate_fixed, g.gate_s, g.gate_r,
      lam, static_cast<__nv_bfloat16*>(y), static_cast<__nv_bfloat16*>(o_race), ctot,
      static_cast<__nv_bfloat16*>(dst), err);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t dispatch(const Geometry& g, const void* codes, const void* tables,
                     const int32_t* counts, const void* o_sp, const float* lse, const float2* gl,
                     const float* gate_b, const float* lam, void* y, void* o_race, int32_t* ctot,
                     void* dst, uint32_t* err, cudaStream_t s) {
  const SlabShape sh = slab_shape(g, MODE);
#define ELSAA_SLAB(OCT, NSUB)                                                                \
  if (sh.oct == OCT && sh.nsub == NSUB)                                                       \
    return launch<MODE, OCT, NSUB>(g, sh, codes, tables, counts, o_sp, lse, gl, gate_b,       \
                                         lam, y, o_race, ctot, dst, err, s);
#define ELSAA_SLAB_N(OCT) \
  ELSAA_SLAB(OCT, 1) ELSAA_SLAB(OCT, 2) ELSAA_SLAB(OCT, 4) ELSAA_SLAB(OCT, 8) ELSAA_SLAB(OCT, 16)
  ELSAA_SLAB_N(2)
  ELSAA_SLAB_N(4)
#undef ELSAA_SLAB_N
#undef ELSAA_SLAB
  return cudaErrorNotSupported;
}

}  // namespace

bool race_slab_supported(const Geometry& g, bool fuse) {
  if (!g.bf16 || g.rcode_bytes != 1 || g.causal) return false;
  if ((g.L != 16 && g.L != 32) || g.d % 8 != 0) return false;
  return slab_shape(g, fuse ? kFuse : kAdd).nsub > 0;
}

cudaError_t launch_race_slab_fuse(const Geometry& g, const void* rcode_q, const void* tables,
                                  const int32_t* counts, const void* o_sp, const float* lse,
                                  const float2* gl, const float* gate_b, const float* lam,
                                  void* y, void* o_race, int32_t* ctot, uint32_t* err,
                                  cudaStream_t s) {
  if (!g.gate_fixed && gl == nullptr) return cudaErrorInvalidValue;
  return dispatch<kFuse>(g, rcode_q, tables, counts, o_sp, lse, gl, gate_b, lam, y, o_race, ctot,
                         nullptr, err, s);
}

cudaError_t launch_race_slab_add(const Geometry& g, const void* codes, const void* tables,
                                 void* dst, uint32_t* err, cudaStream_t s) {
  return dispatch<kAdd>(g, codes, tables, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                        nullptr, nullptr, nullptr, dst, err, s);
}

}  // namespace elsaa
