// Backward of the exact sparse branch as a persistent warp-specialized tcgen05
// pipeline (bf16, d = 64, chunk c <= 128 with 128 % c == 0).
//
// Mathematics ("Two Efficient Attentions, One Denominator Problem", section
// "Two efficient branches can still be mis-scaled": the sparse branch is exact
// attention over each query's Sort-LSH window, and its log-mass feeds the
// fusion):
//   P = exp(scale s - lse), dS = P (dO V^T - D'),
//   dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
//
// Work: key tiles of 128 sorted keys, key tile kb covering keys [128 kb,
// 128 kb + 128).  The keys of tile kb are seen by the queries of query block
// kb ("own") and by the first c queries of block kb + 1 ("next").  Each CTA
// takes a contiguous run of key tiles, so consecutive tiles share a query
// block.  The dQ of block qb has two contributions, from tiles qb - 1 and
// qb; both are accumulated in TMEM by the CTA that owns tile qb and written
// once, in bf16, together with the gate part of dQ, da_s w_s + da_r w_r (the
// per-row pair (da_s, da_r) comes from the fusion backward).  For
// the first tile of a run the contribution of tile qb - 1 belongs to another
// CTA; this CTA recomputes it (a "pre" pair: dQ only), and the CTA owning
// tile qb - 1 skips the dQ of its last "next" pair.  No atomics, and every
// output element is written by exactly one thread.  dv holds the sparse part
// only; the RACE branch's part is added afterwards.
//
// Roles (448 threads, one CTA per SM):
//   warp 0      producer: TMA row gathers (four rows per instruction, into
//               128B-swizzled tiles) of K/V key tiles (two-slot ring) and Q/dO
//               query blocks (two-slot ring), with the blocks' lse, D' and
//               (da_s, da_r) by cp.async
//   warp 1      MMA issuer (one thread) and TMEM owner; for pair p it issues
//               S^T/dP^T of pair p + 1 as soon as the elementwise warps have
//               read S^T/dP^T of pair p out of TMEM (s_free), then, once P^T
//               and dS^T of pair p are in shared memory (p_full), dV of pair p
//               (its completion frees P^T: pt_free) and dK, dQ (pd_free)
//   warps 2..9  elementwise: warp w reaches TMEM lanes 32 (w % 4) .. +31 and
//               takes half of the query columns, read in 16-column chunks with
//               the next chunk's load in flight; P^T (bf16) goes to shared
//               memory chunk by chunk after pt_free of the previous pair, dS^T
//               is held in registers and stored after its pd_free; they also
//               stage the token indices (and gate pairs) the epilogue needs
//   warps 10-13 epilogue: a finished query block's dQ (+ gate part) and a
//               finished key tile's dV and dK from TMEM to bf16 rows; TMEM is
//               released as soon as it has been read, before the stores
// TMEM: S^T [0,128), dP^T [128,256), dV [256,320), dK [320,384),
//       dQ [384,448) and [448,512) for alternating query blocks.
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
constexpr int kThreads = 448;
constexpr int kEwThreads = 256;
constexpr int kEpThreads = 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTS = 0, kTdP = 128, kTdV = 256, kTdK = 320, kTdQ = 384;

struct Lay3 {
  static constexpr uint32_t kSub = 128 * 128;               // 128 rows x 64 bf16
  static constexpr uint32_t kKv = 0;                        // [2][K | V]
  static constexpr uint32_t kKvSlot = 2 * kSub;
  static constexpr uint32_t kQ = kKv + 2 * kKvSlot;         // [2][Q | dO]
  static constexpr uint32_t kQSlot = 2 * kSub;
  static constexpr uint32_t kPT = kQ + 2 * kQSlot;          // P^T  [128 keys][128 queries]
  static constexpr uint32_t kDST = kPT + 2 * kSub;          // dS^T [128 keys][128 queries]
  static constexpr uint32_t kKidx = kDST + 2 * kSub;        // [2][128] key tokens
  static constexpr uint32_t kQidx = kKidx + 2 * 128 * 4;    // [2][128] query tokens
  static constexpr uint32_t kLse = kQidx + 2 * 128 * 4;     // [2][128] lse (-log2 units once used)
  static constexpr uint32_t kDpr = kLse + 2 * 128 * 4;      // [2][128] D' (negated once used)
  static constexpr uint32_t kDa = kDpr + 2 * 128 * 4;       // [2][128] (da_s, da_r)
  static constexpr uint32_t kW = kDa + 2 * 128 * 8;         // [2][64] w_s, w_r
  static constexpr uint32_t kFtok = kW + 2 * 64 * 4;        // [2][128] flush: query tokens
  static constexpr uint32_t kFda = kFtok + 2 * 128 * 4;     // [2][128] flush: (da_s, da_r)
  static constexpr uint32_t kKtok = kFda + 2 * 128 * 8;     // [2][128] write-out: key tokens
  static constexpr uint32_t kBar = kKtok + 2 * 128 * 4;
  static constexpr uint32_t kDyn = kBar + 256;
};

// TMA maps of Q, K, V and dO as [B H N, 64] row matrices.
struct RowMaps {
  CUtensorMap q, k, v, o;
};

struct Bars3 {
  uint64_t full_kv[2], empty_kv[2], full_q[2], empty_q[2];
  uint64_t s_full, s_free, p_full, pt_free, pd_free, kvacc_full, dq_full[2];
  uint64_t dq_free[2], kvacc_free[2], fl_ready[2], key_ready[2];
  uint32_t tmem;
};
static_assert(sizeof(Bars3) <= 256, "barrier block");

// One (key tile, query block) pair of the run.
struct Pair {
  int bh, kb, qb;
  int64_t kvs, qs;       // ring sequence numbers of the key tile and the query block
  int64_t tile;          // tile index in the run (-1: pre pair)
  int nq;                // query columns that can see the tile
  bool kv, dq, dq_acc;   // adds to dV/dK; adds to dQ; dQ adds to an earlier contribution
  bool flush;            // the query block's dQ is complete after this pair
  bool first_of_tile, last_of_tile, release_kv, release_q, q_first;
};

struct Run3 {
  int64_t begin, count;
  int T, chunk;
  int extra;   // 1: the run starts with a pre pair
  ELSAA_DEV int bh_of(int64_t j) const { return (int)((begin + j) / T); }
  ELSAA_DEV int kb_of(int64_t j) const { return (int)((begin + j) % T); }
  ELSAA_DEV bool has_next(int64_t j) const { return kb_of(j) + 1 < T; }
};

// Enumerates the run's pairs: [pre], then per tile own and (if any) next.
struct PairIter {
  const Run3* r;
  int64_t j;
  int kind;   // 0 pre, 1 own, 2 next
  ELSAA_DEV void init(const Run3* run) {
    r = run;
    j = 0;
    kind = run->extra ? 0 : 1;
  }
  ELSAA_DEV bool done() const { return j >= r->count; }
  ELSAA_DEV void advance() {
    if (kind == 0) kind = 1;
    else if (kind == 1 && r->has_next(j)) kind = 2;
    else { ++j; kind = 1; }
  }
  ELSAA_DEV Pair get() const {
    Pair p;
    p.bh = r->bh_of(j);
    const int kb = r->kb_of(j);
    if (kind == 0) {
      p.kb = kb - 1; p.qb = kb; p.kvs = 0; p.qs = 0; p.tile = -1; p.nq = r->chunk;
      p.kv = false; p.dq = true; p.dq_acc = false; p.flush = false;
      p.first_of_tile = true; p.last_of_tile = true; p.release_kv = true; p.release_q = false;
      p.q_first = true;
    } else if (kind == 1) {
      p.kb = kb; p.qb = kb; p.kvs = j + r->extra; p.qs = j; p.tile = j; p.nq = kTile;
      p.kv = true; p.dq = true;
      p.dq_acc = j == 0 ? r->extra != 0 : r->has_next(j - 1);
      p.flush = true;
      p.first_of_tile = true; p.last_of_tile = !r->has_next(j);
      p.release_kv = p.last_of_tile; p.release_q = true;
      p.q_first = j == 0 ? r->extra == 0 : !r->has_next(j - 1);
    } else {
      p.kb = kb; p.qb = kb + 1; p.kvs = j + r->extra; p.qs = j + 1; p.tile = j; p.nq = r->chunk;
      p.kv = true; p.dq = j + 1 < r->count; p.dq_acc = false; p.flush = false;
      p.first_of_tile = false; p.last_of_tile = true; p.release_kv = true;
      p.release_q = j + 1 == r->count; p.q_first = true;
    }
    return p;
  }
};

// Waits for this thread's TMEM loads, with the 32 destination registers of
// the two 16-column loads tied to the wait so that no use of them is
// scheduled above it.
ELSAA_DEV void tmem_wait_hold(float* a, float* b) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+f"(a[0]), "+f"(a[1]), "+f"(a[2]), "+f"(a[3]), "+f"(a[4]), "+f"(a[5]),
                 "+f"(a[6]), "+f"(a[7]), "+f"(a[8]), "+f"(a[9]), "+f"(a[10]), "+f"(a[11]),
                 "+f"(a[12]), "+f"(a[13]), "+f"(a[14]), "+f"(a[15]), "+f"(b[0]), "+f"(b[1]),
                 "+f"(b[2]), "+f"(b[3]), "+f"(b[4]), "+f"(b[5]), "+f"(b[6]), "+f"(b[7]),
                 "+f"(b[8]), "+f"(b[9]), "+f"(b[10]), "+f"(b[11]), "+f"(b[12]), "+f"(b[13]),
                 "+f"(b[14]), "+f"(b[15])
               :
               : "memory");
}

ELSAA_DEV uint32_t pack2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

ELSAA_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

ELSAA_DEV void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
ELSAA_DEV void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}

ELSAA_DEV void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

ELSAA_DEV void ew_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kEwThreads) : "memory"); }

// Barrier among the elementwise warps that ANDs a flag over them.
ELSAA_DEV bool ew_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kEwThreads)
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd3_kernel(const __grid_constant__ RowMaps maps, const int32_t* __restrict__ perm_q,
                 const int32_t* __restrict__ perm_k, const float* __restrict__ lse, const float* __restrict__ dprime,
                 const float2* __restrict__ da, const float* __restrict__ gate_w, int BH,
                 int N, int chunk, float scale, float scale_log2, __nv_bfloat16* __restrict__ dq,
                 __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                 uint32_t* __restrict__ err) {
  using Lay = Lay3;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  Bars3* bars = reinterpret_cast<Bars3*>(smem + Lay::kBar);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((sbase & 1023u) != 0) {
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  Run3 run;
  run.T = N / kTile;
  run.chunk = chunk;
  {
    const int64_t ntiles = (int64_t)BH * run.T;
    run.begin = ntiles * blockIdx.x / gridDim.x;
    run.count = ntiles * (blockIdx.x + 1) / gridDim.x - run.begin;
    run.extra = (run.count > 0 && run.begin % run.T != 0) ? 1 : 0;
  }
  int32_t* s_kidx = reinterpret_cast<int32_t*>(smem + Lay::kKidx);
  int32_t* s_qidx = reinterpret_cast<int32_t*>(smem + Lay::kQidx);
  float* s_lse = reinterpret_cast<float*>(smem + Lay::kLse);
  float* s_dpr = reinterpret_cast<float*>(smem + Lay::kDpr);
  float2* s_da = reinterpret_cast<float2*>(smem + Lay::kDa);
  float* s_w = reinterpret_cast<float*>(smem + Lay::kW);
  for (int i = tid; i < 2 * D; i += kThreads) s_w[i] = gate_w ? gate_w[i] : 0.f;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      // full: the producer's byte-count arrival, 32 plain arrivals (token
      // indices) and, for query blocks, 32 cp.async arrivals (lse, D', da)
      mbar_init(&bars->full_kv[s], 1 + 32);
      mbar_init(&bars->empty_kv[s], 1);
      mbar_init(&bars->full_q[s], 1 + 32 + 32);
      mbar_init(&bars->empty_q[s], 1);
      mbar_init(&bars->dq_full[s], 1);
      mbar_init(&bars->dq_free[s], kEpThreads);
      mbar_init(&bars->kvacc_free[s], kEpThreads);
      mbar_init(&bars->fl_ready[s], 128);   // elementwise threads of half 0
      mbar_init(&bars->key_ready[s], 128);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, kEwThreads);
    mbar_init(&bars->p_full, kEwThreads);
    mbar_init(&bars->pt_free, 1);
    mbar_init(&bars->pd_free, 1);
    mbar_init(&bars->kvacc_full, 1);
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
    // Lane l handles rows 4 l .. 4 l + 3 of a tile or block: one 16-byte load
    // of their token indices, one TMA gather of the four rows per matrix.
    auto load_kv = [&](int64_t n, int bh, int kb) -> bool {
      const size_t unit = (size_t)bh * N;
      const int4 t4 = *reinterpret_cast<const int4*>(perm_k + unit + (size_t)kb * kTile + 4 * lane);
      const int s = (int)(n & 1);
      if (n >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bars->empty_kv[s],
                                                      (uint32_t)(((n >> 1) - 1) & 1), err)))
        return false;
      if (lane == 0) mbar_arrive_expect_tx(&bars->full_kv[s], 2u * kTile * 128u);
      __syncwarp();
      const uint32_t kst = sbase + Lay::kKv + s * Lay::kKvSlot + lane * 512;
      const int u = (int)unit;
      tma_gather4(kst, &maps.k, u + t4.x, u + t4.y, u + t4.z, u + t4.w, &bars->full_kv[s]);
      tma_gather4(kst + Lay::kSub, &maps.v, u + t4.x, u + t4.y, u + t4.z, u + t4.w,
                  &bars->full_kv[s]);
      *reinterpret_cast<int4*>(s_kidx + s * 128 + 4 * lane) = t4;
      mbar_arrive(&bars->full_kv[s]);
      return true;
    };
    auto load_q = [&](int64_t n, int bh, int qb) -> bool {
      const size_t unit = (size_t)bh * N;
      const int4 t4 = *reinterpret_cast<const int4*>(perm_q + unit + (size_t)qb * kTile + 4 * lane);
      const int s = (int)(n & 1);
      if (n >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bars->empty_q[s],
                                                      (uint32_t)(((n >> 1) - 1) & 1), err)))
        return false;
      if (lane == 0) mbar_arrive_expect_tx(&bars->full_q[s], 2u * kTile * 128u);
      __syncwarp();
      const uint32_t qst = sbase + Lay::kQ + s * Lay::kQSlot + lane * 512;
      const int u = (int)unit;
      tma_gather4(qst, &maps.q, u + t4.x, u + t4.y, u + t4.z, u + t4.w, &bars->full_q[s]);
      tma_gather4(qst + Lay::kSub, &maps.o, u + t4.x, u + t4.y, u + t4.z, u + t4.w,
                  &bars->full_q[s]);
      const int tk[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = 4 * lane + j;
        cp_async4(smem_u32(s_lse + s * 128 + r), lse + unit + tk[j]);
        cp_async4(smem_u32(s_dpr + s * 128 + r), dprime + unit + tk[j]);
        cp_async8(smem_u32(s_da + s * 128 + r), da + unit + tk[j]);
      }
      *reinterpret_cast<int4*>(s_qidx + s * 128 + 4 * lane) = t4;
      cp_async_arrive(&bars->full_q[s]);
      mbar_arrive(&bars->full_q[s]);
      return true;
    };
    if (run.count > 0) {
      const int bh0 = run.bh_of(0), kb0 = run.kb_of(0);
      if (run.extra) ok = load_kv(0, bh0, kb0 - 1);
      if (ok) ok = load_q(0, bh0, kb0);
      const int64_t nq_blocks = run.count + (run.has_next(run.count - 1) ? 1 : 0);
      for (int64_t j = 0; j < run.count && ok; ++j) {
        ok = load_kv(j + run.extra, run.bh_of(j), run.kb_of(j));
        if (!ok) break;
        if (j + 1 < nq_blocks) {
          // query block j + 1: the own block of tile j + 1, or the next block of the last tile
          const bool last = j + 1 == run.count;
          ok = load_q(j + 1, last ? run.bh_of(j) : run.bh_of(j + 1),
                      last ? run.kb_of(j) + 1 : run.kb_of(j + 1));
        }
      }
    }
    cp_async_wait_all();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && run.count > 0) {
      int64_t kv_seen = 0, q_seen = 0;
      auto wait_data = [&](const Pair& p) -> bool {
        for (; kv_seen <= p.kvs; ++kv_seen)
          if (!mbar_wait(&bars->full_kv[kv_seen & 1], (uint32_t)((kv_seen >> 1) & 1), err))
            return false;
        for (; q_seen <= p.qs; ++q_seen)
          if (!mbar_wait(&bars->full_q[q_seen & 1], (uint32_t)((q_seen >> 1) & 1), err))
            return false;
        fence_async_smem();   // cp.async data -> tensor core
        fence_after();
        return true;
      };
      auto kv_slot = [&](int64_t n) { return sbase + Lay::kKv + (uint32_t)(n & 1) * Lay::kKvSlot; };
      auto q_slot = [&](int64_t n) { return sbase + Lay::kQ + (uint32_t)(n & 1) * Lay::kQSlot; };
      // descriptors of slot 0's tiles, K-major (a K step adds 32 bytes) and
      // MN-major (LBO = one tile; a 16-row K step adds 2048 bytes); slot 1 is
      // one slot size further on
      const uint64_t kd0 = sw128_desc(kv_slot(0), 16, 1024), qd0 = sw128_desc(q_slot(0), 16, 1024);
      const uint64_t kn0 = sw128_desc(kv_slot(0), Lay::kSub, 1024);
      const uint64_t qn0 = sw128_desc(q_slot(0), Lay::kSub, 1024);
      const uint64_t pt_d = sw128_desc(sbase + Lay::kPT, 16, 1024);
      const uint64_t ds_d = sw128_desc(sbase + Lay::kDST, 16, 1024);
      const uint64_t ds_n = sw128_desc(sbase + Lay::kDST, Lay::kSub, 1024);
      auto issue_s = [&](const Pair& p) {   // S^T = K Q^T, dP^T = V dO^T
        const uint32_t idesc = idesc_bf16(128, p.nq, false, false);
        const uint64_t kd = desc_add(kd0, (uint32_t)(p.kvs & 1) * Lay::kKvSlot);
        const uint64_t qd = desc_add(qd0, (uint32_t)(p.qs & 1) * Lay::kQSlot);
#pragma unroll
        for (int s = 0; s < D / 16; ++s)
          mma_bf16_ss(tmem + kTS, desc_add(kd, s * 32), desc_add(qd, s * 32), idesc, s > 0);
#pragma unroll
        for (int s = 0; s < D / 16; ++s)
          mma_bf16_ss(tmem + kTdP, desc_add(kd, Lay::kSub + s * 32),
                      desc_add(qd, Lay::kSub + s * 32), idesc, s > 0);
        mma_commit(&bars->s_full);
      };
      PairIter it;
      it.init(&run);
      Pair cur = it.get();
      // per dQ buffer b (bit b): has it been flushed yet; parity of its flush count
      uint32_t fl_any = 0u, fl_par = 0u;
      ok = wait_data(cur);
      if (ok) issue_s(cur);
      for (int64_t pi = 0; ok; ++pi) {
        // the next pair's S and dP go out as soon as every elementwise thread
        // has read this pair's S and dP from TMEM; its gradients once P^T and
        // dS^T are in shared memory
        ok = mbar_wait(&bars->s_free, (uint32_t)(pi & 1), err);
        if (!ok) break;
        fence_after();
        PairIter nx = it;
        nx.advance();
        const bool more = !nx.done();
        Pair nxt;
        if (more) {
          nxt = nx.get();
          ok = wait_data(nxt);
          if (!ok) break;
          issue_s(nxt);
        }
        ok = mbar_wait(&bars->p_full, (uint32_t)(pi & 1), err);
        if (!ok) break;
        fence_after();
        const uint64_t kn = desc_add(kn0, (uint32_t)(cur.kvs & 1) * Lay::kKvSlot);
        const uint64_t qn = desc_add(qn0, (uint32_t)(cur.qs & 1) * Lay::kQSlot);
        if (cur.kv && cur.first_of_tile && cur.tile >= 1) {
          // the epilogue has read the previous tile's dV / dK
          ok = mbar_wait(&bars->kvacc_free[(cur.tile - 1) & 1],
                         (uint32_t)(((cur.tile - 1) >> 1) & 1), err);
          if (!ok) break;
        }
        if (cur.dq && !cur.dq_acc && ((fl_any >> (cur.qs & 1)) & 1u)) {
          // the epilogue has read this dQ buffer's previous block
          const int b = (int)(cur.qs & 1);
          ok = mbar_wait(&bars->dq_free[b], ((fl_par >> b) & 1u) ^ 1u, err);
          if (!ok) break;
        }
        fence_after();
        // dV first: its completion frees P^T for the next pair's stores
        const uint32_t id_kv = idesc_bf16(128, D, false, true);
        if (cur.kv) {
          for (int s = 0; s < cur.nq / 16; ++s) {
            const uint32_t aoff = (s >> 2) * Lay::kSub + (s & 3) * 32;
            const uint32_t acc = (!cur.first_of_tile || s > 0) ? 1u : 0u;
            mma_bf16_ss(tmem + kTdV, desc_add(pt_d, aoff), desc_add(qn, Lay::kSub + s * 2048),
                        id_kv, acc);
          }
        }
        mma_commit(&bars->pt_free);
        if (cur.kv) {
          for (int s = 0; s < cur.nq / 16; ++s) {
            const uint32_t aoff = (s >> 2) * Lay::kSub + (s & 3) * 32;
            const uint32_t acc = (!cur.first_of_tile || s > 0) ? 1u : 0u;
            mma_bf16_ss(tmem + kTdK, desc_add(ds_d, aoff), desc_add(qn, s * 2048), id_kv, acc);
          }
        }
        if (cur.dq) {
          const uint32_t id_q = idesc_bf16(128, D, true, true);
          const uint32_t dqc = kTdQ + (uint32_t)(cur.qs & 1) * D;
#pragma unroll
          for (int s = 0; s < kTile / 16; ++s)
            mma_bf16_ss(tmem + dqc, desc_add(ds_n, s * 2048), desc_add(kn, s * 2048), id_q,
                        (cur.dq_acc || s > 0) ? 1u : 0u);
        }
        mma_commit(&bars->pd_free);
        if (cur.release_kv) mma_commit(&bars->empty_kv[cur.kvs & 1]);
        if (cur.release_q) mma_commit(&bars->empty_q[cur.qs & 1]);
        if (cur.kv && cur.last_of_tile) mma_commit(&bars->kvacc_full);
        if (cur.flush) {
          mma_commit(&bars->dq_full[cur.qs & 1]);
          fl_any |= 1u << (cur.qs & 1);
          fl_par ^= 1u << (cur.qs & 1);
        }
        if (!more) break;
        it = nx;
        cur = nxt;
      }
    }
    __syncwarp();
  } else if (warp < 10) {
    // ---------------------------------------------------------------- elementwise
    const int ew = tid - 64;                           // 0 .. 255
    const int quarter = warp & 3, half = (warp - 2) >> 2;
    const int row = 32 * quarter + lane;               // TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const bool masked = chunk < kTile;
    int lc = 0;
    while ((1 << lc) < chunk) ++lc;
    uint32_t fl_any = 0u, fl_par = 0u;   // per dQ buffer b (bit b): staged yet; parity of count
    int32_t* s_ftok = reinterpret_cast<int32_t*>(smem + Lay::kFtok);
    float2* s_fda = reinterpret_cast<float2*>(smem + Lay::kFda);
    int32_t* s_ktok = reinterpret_cast<int32_t*>(smem + Lay::kKtok);
    PairIter it;
    it.init(&run);
    for (int64_t pi = 0; run.count > 0 && !it.done(); ++pi, it.advance()) {
      const Pair p = it.get();
      const int qslot = (int)(p.qs & 1), kslot = (int)(p.kvs & 1);
      ok = ew_all(mbar_wait(&bars->s_full, (uint32_t)(pi & 1), err) &&
                  mbar_wait(&bars->full_q[qslot], (uint32_t)((p.qs >> 1) & 1), err) &&
                  mbar_wait(&bars->full_kv[kslot], (uint32_t)((p.kvs >> 1) & 1), err));
      if (!ok) break;
      fence_after();
      float* ls = s_lse + qslot * 128;
      float* dps = s_dpr + qslot * 128;
      if (p.q_first) {   // once per block: -lse in log2 units and -D'
        if (ew < 128) {
          ls[ew] *= -1.4426950408889634f;
          dps[ew] = -dps[ew];
        }
        ew_sync();
      }
      // stage the epilogue's inputs (key tokens of a new tile; query tokens
      // and gate pairs of a block whose dQ completes with this pair), once
      // the epilogue is done with the buffer's previous contents
      if (p.kv && p.first_of_tile) {
        const int par = (int)(p.tile & 1);
        if (p.tile >= 2) {
          ok = ew_all(mbar_wait(&bars->kvacc_free[par], (uint32_t)(((p.tile >> 1) - 1) & 1), err));
          if (!ok) break;
        }
        if (half == 0) {
          s_ktok[par * 128 + row] = s_kidx[kslot * 128 + row];
          mbar_arrive(&bars->key_ready[par]);
        }
      }
      if (p.flush) {
        const int b = qslot;
        if ((fl_any >> b) & 1u) {
          ok = ew_all(mbar_wait(&bars->dq_free[b], ((fl_par >> b) & 1u) ^ 1u, err));
          if (!ok) break;
        }
        fl_any |= 1u << b;
        fl_par ^= 1u << b;
        if (half == 0) {
          s_ftok[b * 128 + row] = s_qidx[qslot * 128 + row];
          s_fda[b * 128 + row] = s_da[qslot * 128 + row];
          mbar_arrive(&bars->fl_ready[b]);
        }
      }
      // visible query columns of this key row: ranks [i c, (i + 2) c)
      const int key_chunk = (p.kb * kTile + row) >> lc;
      const int lo = (key_chunk << lc) - p.qb * kTile, hi = lo + 2 * chunk;
      const int cend = min(hi, p.nq);
      // four 16-column chunks of S and dP per thread; the next chunk's TMEM
      // loads are in flight while this one is computed. P^T goes out chunk by
      // chunk once the previous pair's dV has read it; dS^T is held and goes
      // out once the previous pair's dK and dQ have read theirs.
      const int cbase = half * 64;
      const bool edge = masked || p.nq < kTile;
      float sv0[16], dp0[16], sv1[16], dp1[16];
      uint32_t dw[4][8];
      tmem_ld16(tmem + kTS + lane_off + cbase, sv0);
      tmem_ld16(tmem + kTdP + lane_off + cbase, dp0);
#pragma unroll
      for (int jc = 0; jc < 4; ++jc) {
        float* sv = (jc & 1) ? sv1 : sv0;
        float* dp = (jc & 1) ? dp1 : dp0;
        tmem_wait_hold(sv, dp);
        if (jc == 3) {   // this pair's S and dP are read: TMEM may take the next pair's
          fence_before();
          mbar_arrive(&bars->s_free);
        }
        if (jc + 1 < 4) {
          tmem_ld16(tmem + kTS + lane_off + cbase + (jc + 1) * 16, (jc & 1) ? sv0 : sv1);
          tmem_ld16(tmem + kTdP + lane_off + cbase + (jc + 1) * 16, (jc & 1) ? dp0 : dp1);
        }
        const int c0 = cbase + jc * 16;
        uint32_t pw[8];
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const float4 nl = *reinterpret_cast<const float4*>(ls + c0 + i);    // -lse log2 e
          const float4 nd = *reinterpret_cast<const float4*>(dps + c0 + i);   // -D'
          float a0 = sv[i], a1 = sv[i + 1], a2 = sv[i + 2], a3 = sv[i + 3];
          fma2(a0, a1, scale_log2, scale_log2, nl.x, nl.y);
          fma2(a2, a3, scale_log2, scale_log2, nl.z, nl.w);
          float p0 = ex2(a0), p1 = ex2(a1), p2 = ex2(a2), p3 = ex2(a3);
          if (edge) {
            const int col = c0 + i;
            p0 = (col >= lo && col < cend) ? p0 : 0.f;
            p1 = (col + 1 >= lo && col + 1 < cend) ? p1 : 0.f;
            p2 = (col + 2 >= lo && col + 2 < cend) ? p2 : 0.f;
            p3 = (col + 3 >= lo && col + 3 < cend) ? p3 : 0.f;
          }
          float g0 = dp[i], g1 = dp[i + 1], g2 = dp[i + 2], g3 = dp[i + 3];
          add2(g0, g1, nd.x, nd.y);
          add2(g2, g3, nd.z, nd.w);
          mul2(g0, g1, p0, p1);
          mul2(g2, g3, p2, p3);
          pw[i >> 1] = pack2(p0, p1);
          pw[(i >> 1) + 1] = pack2(p2, p3);
          dw[jc][i >> 1] = pack2(g0, g1);
          dw[jc][(i >> 1) + 1] = pack2(g2, g3);
        }
        if (jc == 0 && pi >= 1) {   // the previous pair's dV is done with P^T
          ok = ew_all(mbar_wait(&bars->pt_free, (uint32_t)((pi - 1) & 1), err));
          if (!ok) {
            tmem_ld_wait();
            break;
          }
        }
        if (p.kv) {
#pragma unroll
          for (int q8 = 0; q8 < 2; ++q8) {
            const int col = c0 + q8 * 8;
            const uint32_t off = (col >> 6) * Lay::kSub + sw128_off(row, (col & 63) >> 3);
            *reinterpret_cast<uint4*>(smem + Lay::kPT + off) =
                make_uint4(pw[q8 * 4], pw[q8 * 4 + 1], pw[q8 * 4 + 2], pw[q8 * 4 + 3]);
          }
        }
      }
      if (!ok) break;
      if (pi >= 1) {   // the previous pair's dK and dQ are done with dS^T
        ok = ew_all(mbar_wait(&bars->pd_free, (uint32_t)((pi - 1) & 1), err));
        if (!ok) break;
      }
#pragma unroll
      for (int jc = 0; jc < 4; ++jc) {
#pragma unroll
        for (int q8 = 0; q8 < 2; ++q8) {
          const int col = cbase + jc * 16 + q8 * 8;
          const uint32_t off = (col >> 6) * Lay::kSub + sw128_off(row, (col & 63) >> 3);
          *reinterpret_cast<uint4*>(smem + Lay::kDST + off) =
              make_uint4(dw[jc][q8 * 4], dw[jc][q8 * 4 + 1], dw[jc][q8 * 4 + 2], dw[jc][q8 * 4 + 3]);
        }
      }
      if (!ok) break;
      fence_async_smem();
      fence_before();
      mbar_arrive(&bars->p_full);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // warp w reaches TMEM lanes 32 (w % 4) .. +31: row = query row of a dQ
    // buffer or key row of dV / dK
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int32_t* s_ftok = reinterpret_cast<const int32_t*>(smem + Lay::kFtok);
    const float2* s_fda = reinterpret_cast<const float2*>(smem + Lay::kFda);
    const int32_t* s_ktok = reinterpret_cast<const int32_t*>(smem + Lay::kKtok);
    uint32_t fl_par = 0u;   // bit b: parity of the next flush of dQ buffer b
    int64_t ntile = 0;
    PairIter it;
    it.init(&run);
    for (; run.count > 0 && !it.done() && ok; it.advance()) {
      const Pair p = it.get();
      const size_t unit = (size_t)p.bh * N;
      if (p.flush) {
        const int b = (int)(p.qs & 1);
        const uint32_t par = (fl_par >> b) & 1u;
        ok = mbar_wait(&bars->fl_ready[b], par, err) && mbar_wait(&bars->dq_full[b], par, err);
        if (!ok) break;
        fl_par ^= 1u << b;
        fence_after();
        float g[64];
        tmem_ld32(tmem + kTdQ + b * D + lane_off, g);
        tmem_ld32(tmem + kTdQ + b * D + lane_off + 32, g + 32);
        tmem_ld_wait();
        const int tok = s_ftok[b * 128 + row];
        const float2 da2 = s_fda[b * 128 + row];
        fence_before();
        mbar_arrive(&bars->dq_free[b]);
        __nv_bfloat16* out = dq + (unit + tok) * D;
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = q8 * 8 + e;
            x[e] = fmaf(da2.x, s_w[c], fmaf(da2.y, s_w[D + c], scale * g[c]));
          }
          *reinterpret_cast<uint4*>(out + q8 * 8) =
              make_uint4(pack2(x[0], x[1]), pack2(x[2], x[3]), pack2(x[4], x[5]), pack2(x[6], x[7]));
        }
      }
      if (p.kv && p.last_of_tile) {
        const int par = (int)(ntile & 1);
        ok = mbar_wait(&bars->key_ready[par], (uint32_t)((ntile >> 1) & 1), err) &&
             mbar_wait(&bars->kvacc_full, (uint32_t)(ntile & 1), err);
        if (!ok) break;
        fence_after();
        uint32_t vw[32], kw[32];
        for (int c0 = 0; c0 < D; c0 += 32) {
          float gv[32], gk[32];
          tmem_ld32(tmem + kTdV + lane_off + c0, gv);
          tmem_ld32(tmem + kTdK + lane_off + c0, gk);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            vw[(c0 + e) >> 1] = pack2(gv[e], gv[e + 1]);
            kw[(c0 + e) >> 1] = pack2(scale * gk[e], scale * gk[e + 1]);
          }
        }
        const int tok = s_ktok[par * 128 + row];
        fence_before();
        mbar_arrive(&bars->kvacc_free[par]);
        ++ntile;
        __nv_bfloat16* ov = dv + (unit + tok) * D;
        __nv_bfloat16* ok_ = dk + (unit + tok) * D;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          *reinterpret_cast<uint4*>(ov + q * 8) =
              make_uint4(vw[4 * q], vw[4 * q + 1], vw[4 * q + 2], vw[4 * q + 3]);
          *reinterpret_cast<uint4*>(ok_ + q * 8) =
              make_uint4(kw[4 * q], kw[4 * q + 1], kw[4 * q + 2], kw[4 * q + 3]);
        }
      }
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

bool attn_bwd3_supported(const Geometry& g) {
  // TMA row coordinates are 32-bit
  return g.bf16 && g.lookback == 1 && !g.causal && g.rounds == 1 && g.d == D && g.N % kTile == 0 &&
         g.chunk >= 16 && g.chunk <= kTile &&
         kTile % g.chunk == 0 && (int64_t)g.BH * g.N < (int64_t)1 << 31;
}

cudaError_t launch_attn_bwd3(const Geometry& g, const void* q, const void* k, const void* v,
                             const int32_t* perm_q, const int32_t* perm_k, const void* d_o,
                             const float* lse, const float* dprime, const float2* da,
                             const float* gate_w, void* dq, void* dk, void* dv, uint32_t* err,
                             cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(attn_bwd3_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Lay3::kDyn);
  if (e != cudaSuccess) return e;
  RowMaps maps;
  const uint64_t rows = (uint64_t)g.BH * g.N;
  if ((e = make_row_map(&maps.q, q, rows)) != cudaSuccess) return e;
  if ((e = make_row_map(&maps.k, k, rows)) != cudaSuccess) return e;
  if ((e = make_row_map(&maps.v, v, rows)) != cudaSuccess) return e;
  if ((e = make_row_map(&maps.o, d_o, rows)) != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntiles = (int64_t)g.BH * (g.N / kTile);
  const int grid = (int)(ntiles < sms ? ntiles : sms);
  attn_bwd3_kernel<<<grid, kThreads, Lay3::kDyn, s>>>(
      maps, perm_q, perm_k, lse, dprime, da, gate_w, g.BH, g.N, g.chunk,
      g.scale, g.scale * 1.4426950408889634f, static_cast<__nv_bfloat16*>(dq),
      static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), err);
  return cudaGetLastError();
}

}  // namespace elsaa
