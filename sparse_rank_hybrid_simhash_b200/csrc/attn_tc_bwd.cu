// Backward of the exact sparse branch on tcgen05 tensor cores (bf16, d in {64, 128}).
//
// The sparse branch ("Two Efficient Attentions, One Denominator Problem",
// section "Two efficient branches can still be mis-scaled") is softmax
// attention over each query's Sort-LSH window; its row mass also feeds the
// fusion multiplier, so its log-mass lse carries a gradient of its own.  With
// P = exp(scale s - lse), dP = dO V^T and D' = rowsum(dO * O) - dlse:
//   dS = P (dP - D'),  dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
//
// Key-major CTAs: one CTA owns 128 consecutive sorted keys (the MMA's M) and
// walks, in blocks of up to 128, the sorted queries whose window holds them
// (query chunk j sees key chunks j - lb .. j, so key chunk i is seen by query
// chunks i .. i + lb; lb = 1 in the pages), for any chunk c with c % 16 == 0,
// optionally with the causal mask (key token index at most the query's):
//   S^T  = K Q_b^T,  dP^T = V dO_b^T          tcgen05 (SS) -> TMEM
//   P^T, dS^T (bf16)                           thread t = key row t -> shared memory
//   dV += P^T dO_b,  dK += dS^T Q_b            tcgen05, accumulated in TMEM
//   dQ_b = dS K                                tcgen05 with dS^T read as an
//                                              MN-major operand; added to the
//                                              fp32 dq accumulator with atomics
// dK and dV (plus the RACE branch's dv) are written once, in bf16, at the
// keys' token indices.  With several hash rounds (an extension: the union of
// the rounds' windows, each key once) the kernel runs once per round t on that
// round's orders with the final lse, masks the (key, query) pairs whose key an
// earlier round's window of the query already holds, and adds dK and dV into
// fp32 accumulators instead.  Every wait is bounded.
#include <math.h>

#include "internal.h"
#include "tc_common.cuh"

namespace elsaa {
namespace {

using namespace tc;

constexpr int kTile = 128;
constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 512;

template <int D>
struct BwdLayout {
  static constexpr int kSub = D / 64;
  static constexpr uint32_t kSubBytes = 128 * 128;
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kSub * kSubBytes;
  static constexpr uint32_t kQ = kV + kSub * kSubBytes;
  static constexpr uint32_t kDO = kQ + kSub * kSubBytes;
  static constexpr uint32_t kPT = kDO + kSub * kSubBytes;    // 128 keys x 128 queries bf16
  static constexpr uint32_t kDST = kPT + 2 * kSubBytes;
  static constexpr uint32_t kLse = kDST + 2 * kSubBytes;     // 128 floats
  static constexpr uint32_t kDpr = kLse + 128 * 4;           // 128 floats
  static constexpr uint32_t kIdx = kDpr + 128 * 4;           // token indices: keys, queries
  static constexpr uint32_t kWin = kIdx + 2 * 128 * 4;       // earlier rounds' query windows
  static constexpr uint32_t kBar = kWin + 2 * (kMaxRounds - 1) * 128 * 4;
  static constexpr uint32_t kDQ = kPT;   // dQ staging (fp32, 128 x D) reuses P^T and dS^T
  static constexpr uint32_t kDyn = kBar + 64;
  // TMEM columns
  static constexpr uint32_t kTS = 0, kTdP = 128, kTdV = 256, kTdK = 256 + D, kTdQ = 0;
};

// Gathers `rows` rows of a [*, D] bf16 matrix into a swizzled tile; the token
// index of each row comes from shared memory.
template <int D>
ELSAA_DEV void gather_rows(uint32_t dst, const __nv_bfloat16* src_base, const int32_t* idx,
                           int rows) {
  constexpr int kChunks = D / 8;
  for (int i = threadIdx.x; i < rows * kChunks; i += kThreads) {
    const int row = i / kChunks, ch = i % kChunks;
    const __nv_bfloat16* src = src_base + (size_t)idx[row] * D + ch * 8;
    cp_async16(dst + (ch >> 3) * (128 * 128) + sw128_off(row, ch & 7), src, 16);
  }
}

ELSAA_DEV void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

ELSAA_DEV uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// MR: the largest hash-round count the instance handles (1, or kMaxRounds
// for the several-round passes); CAUSAL: the causal mask (compile-time, so the
// element loop of the other instances carries no test for it).
template <int D, int MR, bool CAUSAL>
__global__ void __launch_bounds__(kThreads)
attn_bwd_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                   const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ perm_q,
                   const int32_t* __restrict__ perm_k, const __nv_bfloat16* __restrict__ d_o,
                   const float* __restrict__ lse, const float* __restrict__ dprime,
                   const float* __restrict__ dv_race, int N, int chunk, int lookback,
                   const int32_t* __restrict__ rank, int round, float* __restrict__ dk_acc,
                   float* __restrict__ dv_acc, float scale,
                   float scale_log2, float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dk,
                   __nv_bfloat16* __restrict__ dv, uint32_t* __restrict__ err) {
  using Lay = BwdLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bar_a = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
  uint64_t* bar_b = bar_a + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_a + 2);
  float* s_lse = reinterpret_cast<float*>(smem + Lay::kLse);
  float* s_dpr = reinterpret_cast<float*>(smem + Lay::kDpr);
  int32_t* kidx = reinterpret_cast<int32_t*>(smem + Lay::kIdx);   // [128] keys of the tile
  int32_t* qidx = kidx + 128;                                      // [128] queries of the block
  float* s_dq = reinterpret_cast<float*>(smem + Lay::kDQ);         // [128][D], chunk-rotated
  const int tid = threadIdx.x, warp = tid >> 5;
  if ((sbase & 1023u) != 0) {
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  const int bh = blockIdx.y;
  const int k0 = blockIdx.x * kTile;
  const size_t unit = (size_t)bh * N;
  const int32_t* pq = perm_q + unit;
  const int32_t* pk = perm_k + unit;
  // queries whose window holds a key of this tile: chunks chunk(k0) .. chunk(k0+127)+lb
  const int qbase = (k0 / chunk) * chunk;
  const int qend = min(N, ((k0 + kTile - 1) / chunk + 1 + lookback) * chunk);
  const int nqb = (qend - qbase + kTile - 1) / kTile;
  const int key_chunk = (k0 + tid) / chunk;
  const int my_tok = pk[k0 + tid];
  // several rounds: this key's chunk in each earlier round, and per query
  // column the query's chunk there (a key is in a query's window of round u
  // when 0 <= query chunk - key chunk <= lookback); s_qc: the columns' chunks
  // in this round
  const int64_t rows = (int64_t)gridDim.y * N, rstride = 2 * rows;   // rank: [R][2][BH][N]
  int my_chunk[MR];
#pragma unroll
  for (int u = 0; u < MR; ++u)
    my_chunk[u] = u < round ? rank[u * rstride + rows + unit + my_tok] / chunk : 0;
  int32_t* s_qj = reinterpret_cast<int32_t*>(smem + Lay::kWin);   // [kMaxRounds - 1][128]
  int32_t* s_qc = s_qj + (kMaxRounds - 1) * 128;                  // [128]

  if (tid == 0) {
    mbar_init(bar_a, 1);
    mbar_init(bar_b, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  kidx[tid] = pk[k0 + tid];
  __syncthreads();
  gather_rows<D>(sbase + Lay::kK, k + unit * D, kidx, kTile);
  gather_rows<D>(sbase + Lay::kV, v + unit * D, kidx, kTile);
  cp_async_commit();
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  bool ok = true;

  for (int b = 0; b < nqb; ++b) {
    const int qb0 = qbase + b * kTile;
    const int nq = min(kTile, qend - qb0);
    if (tid < nq) {
      qidx[tid] = pq[qb0 + tid];
      s_qc[tid] = (qb0 + tid) / chunk;
      for (int u = 0; u < round; ++u)
        s_qj[u * 128 + tid] = rank[u * rstride + unit + qidx[tid]] / chunk;
    }
    __syncthreads();
    gather_rows<D>(sbase + Lay::kQ, q + unit * D, qidx, nq);
    gather_rows<D>(sbase + Lay::kDO, d_o + unit * D, qidx, nq);
    cp_async_commit();
    if (tid < nq) {
      const int i = qidx[tid];
      s_lse[tid] = lse[unit + i] * 1.4426950408889634f;
      s_dpr[tid] = dprime[unit + i];
    }
    cp_async_wait_all();
    fence_async_smem();
    fence_before();
    __syncthreads();
    // S^T = K Q_b^T and dP^T = V dO_b^T
    if (tid == 0) {
      fence_after();
      const uint32_t idesc = idesc_bf16(128, nq, false, false);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const uint32_t off = (s >> 2) * Lay::kSubBytes + (s & 3) * 32;
        mma_bf16_ss(tmem + Lay::kTS, sw128_desc(sbase + Lay::kK + off, 16, 1024),
                    sw128_desc(sbase + Lay::kQ + off, 16, 1024), idesc, s > 0);
      }
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const uint32_t off = (s >> 2) * Lay::kSubBytes + (s & 3) * 32;
        mma_bf16_ss(tmem + Lay::kTdP, sw128_desc(sbase + Lay::kV + off, 16, 1024),
                    sw128_desc(sbase + Lay::kDO + off, 16, 1024), idesc, s > 0);
      }
      mma_commit(bar_a);
    }
    ok = mbar_wait(bar_a, b & 1, err);
    if (__syncthreads_or(!ok)) {  // every thread leaves with ok false
      ok = false;
      break;
    }
    fence_after();
    // P^T and dS^T rows of this thread's key; a query in chunk jq sees this key
    // iff 0 <= jq - key_chunk <= lb (and, causal, the key's token index is at
    // most the query's)
    for (int c0 = 0; c0 < nq; c0 += 32) {
      float sv[32], dp[32];
      tmem_ld32(tmem + Lay::kTS + lane_off + c0, sv);
      tmem_ld32(tmem + Lay::kTdP + lane_off + c0, dp);
      tmem_ld_wait();
      // bit i: column c0 + i is a query of this key (in this round's window,
      // causal if asked, not in an earlier round's window); the one-round
      // instance tests each element in place instead
      uint32_t okb = 0;
      if constexpr (MR > 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int col = c0 + i;
          const bool in = col < nq && (uint32_t)(s_qc[col] - key_chunk) <= (uint32_t)lookback &&
                          (!CAUSAL || my_tok <= qidx[col]);
          okb |= (uint32_t)in << i;
        }
#pragma unroll
        for (int u = 0; u < MR; ++u) {
          if (u >= round) break;
          uint32_t sb = 0;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            sb |= (uint32_t)((uint32_t)(s_qj[u * 128 + c0 + i] - my_chunk[u]) <=
                             (uint32_t)lookback)
                  << i;
          okb &= ~sb;
        }
      }
      uint32_t pp[16], dd[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float p[2], ds[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int col = c0 + i + e;
          p[e] = 0.f;
          ds[e] = 0.f;
          bool ok;
          if constexpr (MR > 1) {
            ok = (okb >> (i + e)) & 1u;
          } else {
            const int dj = (qb0 + col) / chunk - key_chunk;
            ok = col < nq && dj >= 0 && dj <= lookback;
            if constexpr (CAUSAL) ok = ok && my_tok <= qidx[col];
          }
          if (ok) {
            p[e] = exp2f(sv[i + e] * scale_log2 - s_lse[col]);
            ds[e] = scale * p[e] * (dp[i + e] - s_dpr[col]);
          }
        }
        pp[i >> 1] = pack_bf16(p[0], p[1]);
        dd[i >> 1] = pack_bf16(ds[0], ds[1]);
      }
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        const int col = c0 + q8 * 8;
        if (col < nq) {
          const uint32_t off = (col >> 6) * Lay::kSubBytes + sw128_off(tid, (col & 63) >> 3);
          *reinterpret_cast<uint4*>(smem + Lay::kPT + off) =
              make_uint4(pp[q8 * 4], pp[q8 * 4 + 1], pp[q8 * 4 + 2], pp[q8 * 4 + 3]);
          *reinterpret_cast<uint4*>(smem + Lay::kDST + off) =
              make_uint4(dd[q8 * 4], dd[q8 * 4 + 1], dd[q8 * 4 + 2], dd[q8 * 4 + 3]);
        }
      }
    }
    fence_async_smem();
    fence_before();
    __syncthreads();
    // dV += P^T dO_b, dK += dS^T Q_b, dQ_b = dS K
    if (tid == 0) {
      fence_after();
      const uint32_t id_kv = idesc_bf16(128, D, false, true);
      for (int s = 0; s < nq / 16; ++s) {
        const uint32_t aoff = (s >> 2) * Lay::kSubBytes + (s & 3) * 32;
        const uint32_t acc = (b > 0 || s > 0) ? 1u : 0u;
        mma_bf16_ss(tmem + Lay::kTdV, sw128_desc(sbase + Lay::kPT + aoff, 16, 1024),
                    sw128_desc(sbase + Lay::kDO + s * 2048, Lay::kSubBytes, 1024), id_kv, acc);
        mma_bf16_ss(tmem + Lay::kTdK, sw128_desc(sbase + Lay::kDST + aoff, 16, 1024),
                    sw128_desc(sbase + Lay::kQ + s * 2048, Lay::kSubBytes, 1024), id_kv, acc);
      }
      const uint32_t id_q = idesc_bf16(128, D, true, true);
#pragma unroll
      for (int s = 0; s < kTile / 16; ++s) {
        mma_bf16_ss(tmem + Lay::kTdQ,
                    sw128_desc(sbase + Lay::kDST + s * 2048, Lay::kSubBytes, 1024),
                    sw128_desc(sbase + Lay::kK + s * 2048, Lay::kSubBytes, 1024), id_q, s > 0);
      }
      mma_commit(bar_b);
    }
    ok = mbar_wait(bar_b, b & 1, err);
    if (__syncthreads_or(!ok)) {  // every thread leaves with ok false
      ok = false;
      break;
    }
    fence_after();
    // dQ rows of this block: TMEM lane t = query qb0 + t.  Stage them in shared
    // memory (16-byte chunk c of row t at chunk position (c + t) mod D/4, so
    // neither the column writes nor the row reads conflict), then add whole
    // rows to the fp32 accumulator with 16-byte vector reductions.
    for (int c0 = 0; c0 < D; c0 += 32) {
      float g[32];
      tmem_ld32(tmem + Lay::kTdQ + lane_off + c0, g);
      tmem_ld_wait();
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const int chunk = (c0 / 4 + q4 + tid) % (D / 4);
        *reinterpret_cast<float4*>(s_dq + tid * D + chunk * 4) =
            make_float4(g[q4 * 4], g[q4 * 4 + 1], g[q4 * 4 + 2], g[q4 * 4 + 3]);
      }
    }
    __syncthreads();
    {
      constexpr int kRowLanes = D / 4;               // lanes per row
      constexpr int kRowsPerIter = kThreads / kRowLanes;
      const int c = tid % kRowLanes;
      for (int row = tid / kRowLanes; row < nq; row += kRowsPerIter) {
        const float4 val =
            *reinterpret_cast<const float4*>(s_dq + row * D + ((c + row) % kRowLanes) * 4);
        red_add_v4(dq_acc + (unit + qidx[row]) * D + c * 4, val.x, val.y, val.z, val.w);
      }
    }
    fence_before();
    __syncthreads();
  }
  if (ok) {
    fence_after();
    const int i = kidx[tid];
    const float* dvr = dv_race + (unit + i) * D;
    __nv_bfloat16* dvo = dv + (unit + i) * D;
    __nv_bfloat16* dko = dk + (unit + i) * D;
    for (int c0 = 0; c0 < D; c0 += 32) {
      float gv[32], gk[32];
      tmem_ld32(tmem + Lay::kTdV + lane_off + c0, gv);
      tmem_ld32(tmem + Lay::kTdK + lane_off + c0, gk);
      tmem_ld_wait();
      if (dk_acc != nullptr) {   // several rounds: one writer per key row and round
        float* ka = dk_acc + (unit + i) * D + c0;
        float* va = dv_acc + (unit + i) * D + c0;
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          float4 a = *reinterpret_cast<float4*>(ka + 4 * c4);
          float4 b = *reinterpret_cast<float4*>(va + 4 * c4);
          a.x += gk[4 * c4]; a.y += gk[4 * c4 + 1]; a.z += gk[4 * c4 + 2]; a.w += gk[4 * c4 + 3];
          b.x += gv[4 * c4]; b.y += gv[4 * c4 + 1]; b.z += gv[4 * c4 + 2]; b.w += gv[4 * c4 + 3];
          *reinterpret_cast<float4*>(ka + 4 * c4) = a;
          *reinterpret_cast<float4*>(va + 4 * c4) = b;
        }
        continue;
      }
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        uint32_t wv[4], wk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = q8 * 8 + 2 * e;
          wv[e] = pack_bf16(gv[c] + dvr[c0 + c], gv[c + 1] + dvr[c0 + c + 1]);
          wk[e] = pack_bf16(gk[c], gk[c + 1]);
        }
        *reinterpret_cast<uint4*>(dvo + c0 + q8 * 8) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        *reinterpret_cast<uint4*>(dko + c0 + q8 * 8) = make_uint4(wk[0], wk[1], wk[2], wk[3]);
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int MR, bool CAUSAL>
cudaError_t bwd1(const Geometry& g, const void* q, const void* k, const void* v,
                const int32_t* perm_q, const int32_t* perm_k, const void* d_o, const float* lse,
                const float* dprime, const float* dv_race, float* dq_acc, void* dk, void* dv,
                const int32_t* rank, int round, float* dk_acc, float* dv_acc, uint32_t* err,
                cudaStream_t s) {
  using Lay = BwdLayout<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_tc_kernel<D, MR, CAUSAL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kDyn);
  if (e != cudaSuccess) return e;
  const dim3 grid(g.N / kTile, g.BH);
  attn_bwd_tc_kernel<D, MR, CAUSAL><<<grid, kThreads, Lay::kDyn, s>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), perm_q, perm_k,
      static_cast<const __nv_bfloat16*>(d_o), lse, dprime, dv_race, g.N, g.chunk, g.lookback,
      rank, round, dk_acc, dv_acc, g.scale,
      g.scale * 1.4426950408889634f, dq_acc, static_cast<__nv_bfloat16*>(dk),
      static_cast<__nv_bfloat16*>(dv), err);
  return cudaGetLastError();
}

template <int D, int MR>
cudaError_t bwd(const Geometry& g, const void* q, const void* k, const void* v,
                const int32_t* perm_q, const int32_t* perm_k, const void* d_o, const float* lse,
                const float* dprime, const float* dv_race, float* dq_acc, void* dk, void* dv,
                const int32_t* rank, int round, float* dk_acc, float* dv_acc, uint32_t* err,
                cudaStream_t s) {
  return g.causal ? bwd1<D, MR, true>(g, q, k, v, perm_q, perm_k, d_o, lse, dprime, dv_race,
                                      dq_acc, dk, dv, rank, round, dk_acc, dv_acc, err, s)
                  : bwd1<D, MR, false>(g, q, k, v, perm_q, perm_k, d_o, lse, dprime, dv_race,
                                       dq_acc, dk, dv, rank, round, dk_acc, dv_acc, err, s);
}

}  // namespace

bool attn_tc_supported(const Geometry& g) {
  // the forward of this domain is the streamed-window kernel; TMA row
  // coordinates are 32-bit
  return g.bf16 && (g.d == 64 || g.d == 128) && g.N % kTile == 0 &&
         g.chunk % 16 == 0 && g.lookback >= 0 && (int64_t)g.BH * g.N < (int64_t)1 << 31;
}

cudaError_t launch_attn_bwd_tc(const Geometry& g, const void* q, const void* k, const void* v,
                               const int32_t* perm_q, const int32_t* perm_k, const void* d_o,
                               const float* lse, const float* dprime, const float* dv_race,
                               float* dq_acc, void* dk, void* dv, uint32_t* err, cudaStream_t s) {
  return g.d == 64 ? bwd<64, 1>(g, q, k, v, perm_q, perm_k, d_o, lse, dprime, dv_race, dq_acc,
                                dk, dv, nullptr, 0, nullptr, nullptr, err, s)
                   : bwd<128, 1>(g, q, k, v, perm_q, perm_k, d_o, lse, dprime, dv_race, dq_acc,
                                 dk, dv, nullptr, 0, nullptr, nullptr, err, s);
}

cudaError_t launch_attn_bwd_tc_rounds(const Geometry& g, const void* q, const void* k,
                                      const void* v, const int32_t* perm, const int32_t* rank,
                                      const void* d_o, const float* lse, const float* dprime,
                                      float* dq_acc, float* dk_acc, float* dv_acc, uint32_t* err,
                                      cudaStream_t s) {
  const int64_t rows = (int64_t)g.BH * g.N;
  for (int t = 0; t < g.rounds; ++t) {
    const int32_t* pq = perm + (size_t)t * 2 * rows;
    const cudaError_t e =
        g.d == 64 ? bwd<64, kMaxRounds - 1>(g, q, k, v, pq, pq + rows, d_o, lse, dprime, nullptr,
                                            dq_acc, nullptr, nullptr, rank, t, dk_acc, dv_acc,
                                            err, s)
                  : bwd<128, kMaxRounds - 1>(g, q, k, v, pq, pq + rows, d_o, lse, dprime,
                                             nullptr, dq_acc, nullptr, nullptr, rank, t, dk_acc,
                                             dv_acc, err, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace elsaa
