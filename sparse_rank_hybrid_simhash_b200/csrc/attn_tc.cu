// Exact sparse branch on tcgen05 tensor cores (bf16 data, d in {64, 128}).
//
// "Two Efficient Attentions, One Denominator Problem" (section "Two efficient
// branches can still be mis-scaled"): the sparse branch evaluates only the
// selected query-key interactions, exactly, and keeps their attention mass.
// With Sort-LSH the selection of the query at sorted rank r (chunk j = r / c)
// is the keys at sorted ranks [max(0, (j-1) c), (j+1) c).
//
// One CTA takes 128 consecutive sorted queries (the MMA's M).  The union of
// their windows is walked in blocks of up to 128 keys:
//   S   = Q K_b^T                     tcgen05 (SS), fp32 in TMEM columns [0, 128)
//   p   = exp(scale s - m), masked to each row's own window, online max m
//   O  += P V_b                       tcgen05 (SS), fp32 in TMEM columns [128, 128 + d)
// Q, K and V rows are gathered by the sort permutations with cp.async into
// 128-byte-swizzled shared-memory tiles; P goes to shared memory as bf16.
// 128 threads: thread t owns TMEM lane t = query row t for the softmax and the
// epilogue, thread 0 issues the MMAs.  The output row and its log-mass
// lse = log sum exp(scale s) land at the query's token index.
#include <math.h>

#include "internal.h"
#include "tc_common.cuh"

namespace elsaa {
namespace {

using namespace tc;

constexpr int kTile = 128;   // query rows per CTA (MMA M)
constexpr int kKB = 128;     // keys per block
constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 256;

template <int D>
struct FwdLayout {
  static constexpr int kSub = D / 64;                       // 64-element sub-tiles along d
  static constexpr uint32_t kSubBytes = 128 * 128;          // one sub-tile of 128 rows
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK0 = kQ + kSub * kSubBytes;    // two key-block slots
  static constexpr uint32_t kV0 = kK0 + 2 * kSub * kSubBytes;
  static constexpr uint32_t kP = kV0 + 2 * kSub * kSubBytes;
  static constexpr uint32_t kBar = kP + 2 * kSubBytes;      // P: 128 x 128 bf16 in 2 sub-tiles
  static constexpr uint32_t kDyn = kBar + 64;
  // Token indices of the rows being gathered live in the P buffer, which is
  // idle whenever a gather is issued.
  static constexpr uint32_t kIdx = kP;
};

// Gathers `rows` rows of a [*, D] bf16 matrix into a swizzled tile; the token
// index of each row comes from shared memory (staged by one coalesced load).
template <int D>
ELSAA_DEV void gather_rows(uint32_t dst, const __nv_bfloat16* src_base, const int32_t* idx,
                           int rows) {
  constexpr int kChunks = D / 8;   // 16-byte chunks per row
  for (int i = threadIdx.x; i < rows * kChunks; i += kThreads) {
    const int row = i / kChunks, ch = i % kChunks;
    const int sub = ch >> 3, c8 = ch & 7;
    const __nv_bfloat16* src = src_base + (size_t)idx[row] * D + ch * 8;
    cp_async16(dst + sub * (128 * 128) + sw128_off(row, c8), src, 16);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads)
attn_fwd_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                   const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ perm_q,
                   const int32_t* __restrict__ perm_k, int N, int chunk, float scale_log2,
                   __nv_bfloat16* __restrict__ o_sp, float* __restrict__ lse,
                   uint32_t* __restrict__ err) {
  using Lay = FwdLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
  uint64_t* bar_o = bar_s + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s + 2);
  int32_t* qidx = reinterpret_cast<int32_t*>(smem + Lay::kIdx);   // [128], prologue only
  int32_t* kidx = qidx + 128;                                     // [2][128]

  const int tid = threadIdx.x, warp = tid >> 5;
  if ((sbase & 1023u) != 0) {   // the swizzled tiles need a 1024-byte aligned base
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  const int bh = blockIdx.y;
  const int r0 = blockIdx.x * kTile;
  const size_t unit = (size_t)bh * N;
  const int32_t* pq = perm_q + unit;
  const int32_t* pk = perm_k + unit;
  const __nv_bfloat16* qb = q + unit * D;
  const __nv_bfloat16* kb = k + unit * D;
  const __nv_bfloat16* vb = v + unit * D;

  // the tile's key range: union of its rows' windows
  const int kbase = max(0, (r0 / chunk - 1) * chunk);
  const int kend = ((r0 + kTile - 1) / chunk + 1) * chunk;
  const int nkb = (kend - kbase + kKB - 1) / kKB;
  // this thread's row window
  const int r = r0 + tid;
  const int jr = r / chunk;
  const int lo = max(0, (jr - 1) * chunk) - kbase, hi = (jr + 1) * chunk - kbase;

  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // prologue loads: token indices, then the Q tile and the first two key blocks
  const int my_token = pq[r0 + tid];   // this thread's query row, kept for the epilogue
  qidx[tid] = my_token;
  for (int b = 0; b < nkb && b < 2; ++b)
    if (tid < kend - kbase - b * kKB) kidx[b * 128 + tid] = pk[kbase + b * kKB + tid];
  __syncthreads();
  gather_rows<D>(sbase + Lay::kQ, qb, qidx, kTile);
  for (int b = 0; b < nkb && b < 2; ++b) {
    const int nb = min(kKB, kend - kbase - b * kKB);
    gather_rows<D>(sbase + Lay::kK0 + b * Lay::kSub * Lay::kSubBytes, kb, kidx + b * 128, nb);
    gather_rows<D>(sbase + Lay::kV0 + b * Lay::kSub * Lay::kSubBytes, vb, kidx + b * 128, nb);
  }
  cp_async_commit();
  cp_async_wait_all();
  fence_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s = tmem, t_o = tmem + 128;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  float m_run = -INFINITY, l_run = 0.f;
  bool ok = true;
  for (int b = 0; b < nkb; ++b) {
    const int nb = min(kKB, kend - kbase - b * kKB);
    const uint32_t slot = (b & 1) * Lay::kSub * Lay::kSubBytes;
    if (b >= 1) {
      ok = mbar_wait(bar_o, (b - 1) & 1, err);
      if (__syncthreads_or(!ok)) {  // every thread leaves with ok false
        ok = false;
        break;
      }
      fence_after();
    }
    if (b >= 2) {
      int32_t* ki = kidx + (b & 1) * 128;
      if (tid < nb) ki[tid] = pk[kbase + b * kKB + tid];
      __syncthreads();
      gather_rows<D>(sbase + Lay::kK0 + slot, kb, ki, nb);
      gather_rows<D>(sbase + Lay::kV0 + slot, vb, ki, nb);
      cp_async_commit();
      cp_async_wait_all();
      fence_async_smem();
      __syncthreads();
    }
    // S = Q K_b^T
    if (tid == 0) {
      fence_after();
      const uint32_t idesc = idesc_bf16(128, nb, false, false);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const uint32_t koff = (s >> 2) * Lay::kSubBytes + (s & 3) * 32;
        mma_bf16_ss(t_s, sw128_desc(sbase + Lay::kQ + koff, 16, 1024),
                    sw128_desc(sbase + Lay::kK0 + slot + koff, 16, 1024), idesc, s > 0);
      }
      mma_commit(bar_s);
    }
    ok = mbar_wait(bar_s, b & 1, err);
    if (__syncthreads_or(!ok)) {  // every thread leaves with ok false
      ok = false;
      break;
    }
    fence_after();
    // online softmax over this block, row t of TMEM lane t
    const int c_lo = lo - b * kKB, c_hi = min(hi - b * kKB, nb);
    float mb = -INFINITY;
    for (int c0 = 0; c0 < nb; c0 += 32) {
      float sv[32];
      tmem_ld32(t_s + lane_off + c0, sv);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (c0 + i >= c_lo && c0 + i < c_hi) mb = fmaxf(mb, sv[i] * scale_log2);
    }
    const float m_new = fmaxf(m_run, mb);
    const float alpha = (m_run == -INFINITY) ? 0.f : exp2f(m_run - m_new);
    if (b >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
      // rescale this warp's O rows (PV of the previous block has completed)
      for (int c0 = 0; c0 < D; c0 += 32) {
        float ov[32];
        tmem_ld32(t_o + lane_off + c0, ov);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] *= alpha;
        tmem_st32(t_o + lane_off + c0, ov);
      }
      tmem_st_wait();
    }
    float lsum = 0.f;
    uint8_t* prow = smem + Lay::kP;
    for (int c0 = 0; c0 < nb; c0 += 32) {
      float sv[32];
      tmem_ld32(t_s + lane_off + c0, sv);
      tmem_ld_wait();
      uint32_t packed[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float p0 = 0.f, p1 = 0.f;
        if (m_new != -INFINITY) {
          if (c0 + i >= c_lo && c0 + i < c_hi) p0 = exp2f(sv[i] * scale_log2 - m_new);
          if (c0 + i + 1 >= c_lo && c0 + i + 1 < c_hi) p1 = exp2f(sv[i + 1] * scale_log2 - m_new);
        }
        lsum += p0 + p1;
        const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
        packed[i >> 1] = *reinterpret_cast<const uint32_t*>(&h);
      }
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        const int key = c0 + q8 * 8;   // first key of this 16-byte chunk
        if (key < nb) {
          uint8_t* dst = prow + (key >> 6) * Lay::kSubBytes + sw128_off(tid, (key & 63) >> 3);
          *reinterpret_cast<uint4*>(dst) =
              make_uint4(packed[q8 * 4], packed[q8 * 4 + 1], packed[q8 * 4 + 2], packed[q8 * 4 + 3]);
        }
      }
    }
    l_run = l_run * alpha + lsum;
    m_run = m_new;
    fence_async_smem();
    fence_before();
    __syncthreads();
    // O += P V_b
    if (tid == 0) {
      fence_after();
      const uint32_t idesc = idesc_bf16(128, D, false, true);
      for (int s = 0; s < nb / 16; ++s) {
        const uint32_t poff = (s >> 2) * Lay::kSubBytes + (s & 3) * 32;
        mma_bf16_ss(t_o, sw128_desc(sbase + Lay::kP + poff, 16, 1024),
                    sw128_desc(sbase + Lay::kV0 + slot + s * 2048, Lay::kSubBytes, 1024), idesc,
                    (b > 0 || s > 0) ? 1u : 0u);
      }
      mma_commit(bar_o);
    }
  }
  if (ok) {
    ok = mbar_wait(bar_o, (nkb - 1) & 1, err);
    ok = !__syncthreads_or(!ok);
  }
  if (ok) {
    fence_after();
    const int i = my_token;
    const float inv = 1.0f / l_run;
    __nv_bfloat16* orow = o_sp + (unit + i) * D;
    for (int c0 = 0; c0 < D; c0 += 32) {
      float ov[32];
      tmem_ld32(t_o + lane_off + c0, ov);
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
    lse[unit + i] = (m_run + log2f(l_run)) * 0.69314718055994531f;
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t fwd(const Geometry& g, const void* q, const void* k, const void* v,
                const int32_t* perm_q, const int32_t* perm_k, void* o_sp, float* lse,
                uint32_t* err, cudaStream_t s) {
  using Lay = FwdLayout<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kDyn);
  if (e != cudaSuccess) return e;
  const dim3 grid(g.N / kTile, g.BH);
  attn_fwd_tc_kernel<D><<<grid, kThreads, Lay::kDyn, s>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), perm_q, perm_k, g.N, g.chunk,
      g.scale * 1.4426950408889634f, static_cast<__nv_bfloat16*>(o_sp), lse, err);
  return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(const Geometry& g) {
  if (!g.bf16 || (g.d != 64 && g.d != 128)) return false;
  if (g.lookback != 1) return false;   // the tiles hold the own and the previous chunk
  if (g.causal) return false;
  if (g.N % kTile != 0 || g.chunk % 16 != 0) return false;
  return (kTile % g.chunk == 0) || (g.chunk % kTile == 0);
}

cudaError_t launch_attn_fwd_tc(const Geometry& g, const void* q, const void* k, const void* v,
                               const int32_t* perm_q, const int32_t* perm_k, void* o_sp,
                               float* lse, uint32_t* err, cudaStream_t s) {
  return g.d == 64 ? fwd<64>(g, q, k, v, perm_q, perm_k, o_sp, lse, err, s)
                   : fwd<128>(g, q, k, v, perm_q, perm_k, o_sp, lse, err, s);
}

}  // namespace elsaa
