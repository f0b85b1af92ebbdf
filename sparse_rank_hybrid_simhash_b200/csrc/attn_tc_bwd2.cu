// Backward of the exact sparse branch, overlapped variant (bf16, d = 64,
// chunk c in {64, 128}).
//
// Same mathematics as attn_tc_bwd.cu ("Two Efficient Attentions, One
// Denominator Problem", section "Two efficient branches can still be
// mis-scaled": the sparse branch is exact attention over each query's window,
// and its log-mass feeds the fusion):
//   P = exp(scale s - lse), dS = P (dO V^T - D'),
//   dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
// One CTA owns 128 sorted keys [k0, k0 + 128) and the sorted queries
// [k0, k0 + 128 + c) that see them, in blocks of <= 128.  Changes against the
// plain variant, all aimed at keeping the tensor cores fed:
//   * 8 warps: warp w reaches TMEM lanes 32 (w % 4) .. +31 and takes half of
//     the columns of each elementwise pass;
//   * TMEM: S^T [0,128), dP^T [128,256), dV [256,320), dK [320,384),
//     dQ [384,448) — dQ has its own columns, so the next block's S^T and dP^T
//     MMAs are issued right behind this block's dV, dK and dQ MMAs;
//   * Q and dO of block b + 2 are gathered (cp.async) into the buffer block b
//     used while block b + 1 is processed;
//   * the dQ rows are staged in shared memory and added to the fp32
//     accumulator with 16-byte vector reductions while the tensor cores run
//     the next block's S^T and dP^T.
#include <math.h>

#include "internal.h"
#include "tc_common.cuh"

namespace elsaa {
namespace {

using namespace tc;

constexpr int D = 64;
constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTS = 0, kTdP = 128, kTdV = 256, kTdK = 320, kTdQ = 384;

struct Bwd2Layout {
  static constexpr uint32_t kSub = 128 * 128;               // 128 rows x 128 bytes
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kSub;
  static constexpr uint32_t kQ = kV + kSub;                  // [2] buffers
  static constexpr uint32_t kDO = kQ + 2 * kSub;             // [2] buffers
  static constexpr uint32_t kPT = kDO + 2 * kSub;            // 128 keys x 128 queries bf16
  static constexpr uint32_t kDST = kPT + 2 * kSub;
  static constexpr uint32_t kDQ = kDST + 2 * kSub;           // fp32 128 x 64 staging
  static constexpr uint32_t kLse = kDQ + 128 * 64 * 4;       // [2][128]
  static constexpr uint32_t kDpr = kLse + 2 * 128 * 4;       // [2][128]
  static constexpr uint32_t kIdx = kDpr + 2 * 128 * 4;       // keys [128], queries [2][128]
  static constexpr uint32_t kBar = kIdx + 3 * 128 * 4;
  static constexpr uint32_t kDyn = kBar + 64;
};

ELSAA_DEV uint32_t pack2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

ELSAA_DEV void red_v4(float* addr, float4 v) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}

ELSAA_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// rows of a [*, 64] bf16 matrix, token indices from shared memory, into a swizzled tile
ELSAA_DEV void gather64(uint32_t dst, const __nv_bfloat16* src, const int32_t* idx, int rows) {
  for (int i = threadIdx.x; i < rows * 8; i += kThreads) {
    const int row = i >> 3, ch = i & 7;
    cp_async16(dst + sw128_off(row, ch), src + (size_t)idx[row] * D + ch * 8, 16);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd2_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                 const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ perm_q,
                 const int32_t* __restrict__ perm_k, const __nv_bfloat16* __restrict__ d_o,
                 const float* __restrict__ lse, const float* __restrict__ dprime,
                 const float* __restrict__ dv_race, int N, int chunk, float scale,
                 float scale_log2, float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dk,
                 __nv_bfloat16* __restrict__ dv, uint32_t* __restrict__ err) {
  using Lay = Bwd2Layout;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(smem + Lay::kBar);   // S^T, dP^T done
  uint64_t* bar_g = bar_s + 1;                                        // dV, dK, dQ done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s + 2);
  float* s_lse = reinterpret_cast<float*>(smem + Lay::kLse);
  float* s_dpr = reinterpret_cast<float*>(smem + Lay::kDpr);
  int32_t* kidx = reinterpret_cast<int32_t*>(smem + Lay::kIdx);
  int32_t* qidx = kidx + 128;                                         // [2][128]
  float* s_dq = reinterpret_cast<float*>(smem + Lay::kDQ);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, half = warp >> 2;
  const int row = 32 * quarter + lane;                                // TMEM lane
  const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
  if ((sbase & 1023u) != 0) {
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  const int bh = blockIdx.y;
  const int k0 = blockIdx.x * kTile;
  const size_t unit = (size_t)bh * N;
  const int32_t* pq = perm_q + unit;
  const int32_t* pk = perm_k + unit;
  const __nv_bfloat16* qb = q + unit * D;
  const __nv_bfloat16* ob = d_o + unit * D;
  const int qend = min(N, k0 + kTile + chunk);   // c divides 128: queries [k0, k0 + 128 + c)
  const int nqb = (qend - k0 + kTile - 1) / kTile;
  const int key_chunk = (k0 + row) / chunk;

  auto stage_block = [&](int b) {   // indices, lse, D' and the Q / dO gathers of block b
    const int qb0 = k0 + b * kTile, nq = min(kTile, qend - qb0), buf = b & 1;
    int32_t* qi = qidx + buf * 128;
    if (tid < nq) {
      const int i = pq[qb0 + tid];
      qi[tid] = i;
      s_lse[buf * 128 + tid] = lse[unit + i] * 1.4426950408889634f;
      s_dpr[buf * 128 + tid] = dprime[unit + i];
    }
    __syncthreads();
    gather64(sbase + Lay::kQ + buf * Lay::kSub, qb, qi, nq);
    gather64(sbase + Lay::kDO + buf * Lay::kSub, ob, qi, nq);
    cp_async_commit();
  };
  auto issue_sdp = [&](int b) {   // S^T = K Q_b^T, dP^T = V dO_b^T
    const int nq = min(kTile, qend - (k0 + b * kTile)), buf = b & 1;
    const uint32_t idesc = idesc_bf16(128, nq, false, false);
#pragma unroll
    for (int s = 0; s < D / 16; ++s)
      mma_bf16_ss(tmem_slot[0] + kTS, sw128_desc(sbase + Lay::kK + s * 32, 16, 1024),
                  sw128_desc(sbase + Lay::kQ + buf * Lay::kSub + s * 32, 16, 1024), idesc, s > 0);
#pragma unroll
    for (int s = 0; s < D / 16; ++s)
      mma_bf16_ss(tmem_slot[0] + kTdP, sw128_desc(sbase + Lay::kV + s * 32, 16, 1024),
                  sw128_desc(sbase + Lay::kDO + buf * Lay::kSub + s * 32, 16, 1024), idesc, s > 0);
    mma_commit(bar_s);
  };

  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_g, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid < kTile) kidx[tid] = pk[k0 + tid];
  __syncthreads();
  gather64(sbase + Lay::kK, k + unit * D, kidx, kTile);
  gather64(sbase + Lay::kV, v + unit * D, kidx, kTile);
  cp_async_commit();
  stage_block(0);
  cp_async_wait_all();
  fence_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = tmem_slot[0];
  if (tid == 0) {
    fence_after();
    issue_sdp(0);
  }
  if (nqb > 1) stage_block(1);
  bool ok = true;

  for (int b = 0; b < nqb; ++b) {
    const int qb0 = k0 + b * kTile, nq = min(kTile, qend - qb0), buf = b & 1;
    ok = mbar_wait(bar_s, b & 1, err);
    if (__syncthreads_or(!ok)) {  // every thread leaves with ok false
      ok = false;
      break;
    }
    fence_after();
    // P^T and dS^T: this thread's key row, half of the query columns
    {
      const int cw = nq >> 1, cbeg = half * cw;
      const float* ls = s_lse + buf * 128;
      const float* dps = s_dpr + buf * 128;
      for (int c0 = cbeg; c0 < cbeg + cw; c0 += 32) {
        float sv[32], dp[32];
        tmem_ld32(tmem + kTS + lane_off + c0, sv);
        tmem_ld32(tmem + kTdP + lane_off + c0, dp);
        tmem_ld_wait();
        uint32_t pp[16], dd[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float p[2], ds[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int col = c0 + i + e;
            const int dj = (qb0 + col) / chunk - key_chunk;
            const float pe = ex2(fmaf(sv[i + e], scale_log2, -ls[col]));
            const bool in = dj == 0 || dj == 1;
            p[e] = in ? pe : 0.f;
            ds[e] = in ? scale * pe * (dp[i + e] - dps[col]) : 0.f;
          }
          pp[i >> 1] = pack2(p[0], p[1]);
          dd[i >> 1] = pack2(ds[0], ds[1]);
        }
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const int col = c0 + q8 * 8;
          const uint32_t off = (col >> 6) * Lay::kSub + sw128_off(row, (col & 63) >> 3);
          *reinterpret_cast<uint4*>(smem + Lay::kPT + off) =
              make_uint4(pp[q8 * 4], pp[q8 * 4 + 1], pp[q8 * 4 + 2], pp[q8 * 4 + 3]);
          *reinterpret_cast<uint4*>(smem + Lay::kDST + off) =
              make_uint4(dd[q8 * 4], dd[q8 * 4 + 1], dd[q8 * 4 + 2], dd[q8 * 4 + 3]);
        }
      }
    }
    cp_async_wait_all();   // Q / dO of block b + 1 (issued one block ago)
    fence_async_smem();
    fence_before();
    __syncthreads();
    if (tid == 0) {
      fence_after();
      const uint32_t id_kv = idesc_bf16(128, D, false, true);
      for (int s = 0; s < nq / 16; ++s) {
        const uint32_t aoff = (s >> 2) * Lay::kSub + (s & 3) * 32;
        const uint32_t acc = (b > 0 || s > 0) ? 1u : 0u;
        mma_bf16_ss(tmem + kTdV, sw128_desc(sbase + Lay::kPT + aoff, 16, 1024),
                    sw128_desc(sbase + Lay::kDO + buf * Lay::kSub + s * 2048, Lay::kSub, 1024),
                    id_kv, acc);
        mma_bf16_ss(tmem + kTdK, sw128_desc(sbase + Lay::kDST + aoff, 16, 1024),
                    sw128_desc(sbase + Lay::kQ + buf * Lay::kSub + s * 2048, Lay::kSub, 1024),
                    id_kv, acc);
      }
      const uint32_t id_q = idesc_bf16(128, D, true, true);
#pragma unroll
      for (int s = 0; s < kTile / 16; ++s)
        mma_bf16_ss(tmem + kTdQ, sw128_desc(sbase + Lay::kDST + s * 2048, Lay::kSub, 1024),
                    sw128_desc(sbase + Lay::kK + s * 2048, Lay::kSub, 1024), id_q, s > 0);
      mma_commit(bar_g);
      if (b + 1 < nqb) issue_sdp(b + 1);
    }
    ok = mbar_wait(bar_g, b & 1, err);
    if (__syncthreads_or(!ok)) {  // every thread leaves with ok false
      ok = false;
      break;
    }
    fence_after();
    // dQ of block b: TMEM lane = query row, this warp's 32 columns; staged with
    // chunk c of row r at position (c + r) mod 16 so neither pass conflicts
    {
      float g[32];
      tmem_ld32(tmem + kTdQ + lane_off + half * 32, g);
      tmem_ld_wait();
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const int chunk16 = (half * 8 + q4 + row) & 15;
        *reinterpret_cast<float4*>(s_dq + row * D + chunk16 * 4) =
            make_float4(g[q4 * 4], g[q4 * 4 + 1], g[q4 * 4 + 2], g[q4 * 4 + 3]);
      }
    }
    __syncthreads();
    {
      const int c = tid & 15;
      const int32_t* qi = qidx + buf * 128;
      for (int r = tid >> 4; r < nq; r += kThreads / 16) {
        const float4 val = *reinterpret_cast<const float4*>(s_dq + r * D + ((c + r) & 15) * 4);
        red_v4(dq_acc + (unit + qi[r]) * D + c * 4, val);
      }
    }
    __syncthreads();   // staging and qidx[buf] are free again
    if (b + 2 < nqb) stage_block(b + 2);
  }
  if (ok) {
    // dV (half 0) and dK (half 1) of this thread's key row, written once in bf16
    const int i = kidx[row];
    float gv[32], gw[32];
    const uint32_t col = half == 0 ? kTdV : kTdK;
    __nv_bfloat16* out = (half == 0 ? dv : dk) + (unit + i) * D;
    const float* add = dv_race + (unit + i) * D;
    for (int c0 = 0; c0 < D; c0 += 32) {
      tmem_ld32(tmem + col + lane_off + c0, gv);
      tmem_ld_wait();
      if (half == 0) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 a = *reinterpret_cast<const float4*>(add + c0 + e);
          gw[e] = gv[e] + a.x; gw[e + 1] = gv[e + 1] + a.y;
          gw[e + 2] = gv[e + 2] + a.z; gw[e + 3] = gv[e + 3] + a.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) gw[e] = gv[e];
      }
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8)
        *reinterpret_cast<uint4*>(out + c0 + q8 * 8) =
            make_uint4(pack2(gw[q8 * 8], gw[q8 * 8 + 1]), pack2(gw[q8 * 8 + 2], gw[q8 * 8 + 3]),
                       pack2(gw[q8 * 8 + 4], gw[q8 * 8 + 5]), pack2(gw[q8 * 8 + 6], gw[q8 * 8 + 7]));
    }
  }
  cp_async_wait_all();
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool attn_bwd2_supported(const Geometry& g) {
  return g.bf16 && g.lookback == 1 && !g.causal && g.rounds == 1 && g.d == D && g.N % kTile == 0 &&
         (g.chunk == 64 || g.chunk == 128);
}

cudaError_t launch_attn_bwd2(const Geometry& g, const void* q, const void* k, const void* v,
                             const int32_t* perm_q, const int32_t* perm_k, const void* d_o,
                             const float* lse, const float* dprime, const float* dv_race,
                             float* dq_acc, void* dk, void* dv, uint32_t* err, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(attn_bwd2_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Bwd2Layout::kDyn);
  if (e != cudaSuccess) return e;
  const dim3 grid(g.N / kTile, g.BH);
  attn_bwd2_kernel<<<grid, kThreads, Bwd2Layout::kDyn, s>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), perm_q, perm_k,
      static_cast<const __nv_bfloat16*>(d_o), lse, dprime, dv_race, g.N, g.chunk, g.scale,
      g.scale * 1.4426950408889634f, dq_acc, static_cast<__nv_bfloat16*>(dk),
      static_cast<__nv_bfloat16*>(dv), err);
  return cudaGetLastError();
}

}  // namespace elsaa
