// The C ABI of libelsaa: validation, saved-state and workspace layout, and the
// launch sequences of the forward and backward (see include/elsaa.h).
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace elsaa {

bool make_geometry(const elsaa_params* p, Geometry* g, elsaa_status* why) {
  *why = ELSAA_ERR_INVALID_ARG;
  if (!p) return false;
  if (p->B <= 0 || p->H <= 0 || p->N <= 0 || p->d <= 0) return false;
  if (p->dtype != ELSAA_BF16 && p->dtype != ELSAA_F32) return false;
  if (p->chunk <= 0 || p->N % p->chunk != 0) return false;
  if (p->sort_bits < 0 || p->sort_bits > 16) return false;
  if (p->sort_order != ELSAA_SORT_BINARY && p->sort_order != ELSAA_SORT_GRAY &&
      p->sort_order != ELSAA_SORT_LOCAL)
    return false;
  if (p->lookback < 0 || p->lookback > 64) return false;
  if (p->causal != 0 && p->causal != 1) return false;
  if (p->hash_rounds < 0 || p->hash_rounds > kMaxRounds) return false;
  if (p->race_tables < 1 || p->race_tables > 4096) return false;
  if (p->race_bits < 0 || p->race_bits > 16) return false;
  if ((int64_t)p->B * p->H * p->N * (p->d > p->race_tables ? p->d : p->race_tables) >
      ((int64_t)1 << 40))
    return false;
  *why = ELSAA_ERR_UNSUPPORTED;
  if (p->d != 32 && p->d != 64 && p->d != 128) return false;
  // the CUDA-core attention keeps a query's windows of scores in shared memory
  const int rounds = p->hash_rounds > 1 ? p->hash_rounds : 1;
  if ((int64_t)rounds * (p->lookback + 1) * p->chunk > 6144) return false;
  // extra rounds' sort codes: (rounds - 1) * sort_bits projections per row
  if ((rounds - 1) * p->sort_bits > 128) return false;
  g->B = p->B;
  g->H = p->H;
  g->N = p->N;
  g->d = p->d;
  g->BH = p->B * p->H;
  g->bf16 = p->dtype == ELSAA_BF16;
  g->esz = g->bf16 ? 2 : 4;
  g->sort_bits = p->sort_bits;
  g->chunk = p->chunk;
  g->L = p->race_tables;
  g->kr = p->race_bits;
  g->NB = 1 << p->race_bits;
  g->rcode_bytes = p->race_bits <= 8 ? 1 : 2;
  g->scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
  g->gate_fixed = p->gate_fixed ? 1 : 0;
  g->gate_s = p->gate_s;
  g->gate_r = p->gate_r;
  g->sort_order = p->sort_order;
  g->lookback = p->lookback;
  g->causal = p->causal;
  g->rounds = rounds;
  g->sort_passes = p->sort_bits <= 8 ? 1 : 2;
  g->sort_digit_bits = (p->sort_bits + g->sort_passes - 1) / g->sort_passes;
  g->sort_bins = 1 << g->sort_digit_bits;
  g->sort_tiles = (p->N + kSortTile - 1) / kSortTile;
  g->tc_hash = hash_tc_supported(*g);
  g->tc_attn = attn_tc_supported(*g);
  if (g->causal && !race_causal_supported(*g)) return false;
  *why = ELSAA_OK;
  return true;
}

SavedLayout saved_layout(const Geometry& g) {
  SavedLayout s;
  const size_t bhn = (size_t)g.BH * g.N;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes); return o; };
  s.code = take((size_t)g.rounds * 2 * bhn * 2);
  s.perm = take((size_t)g.rounds * 2 * bhn * 4);
  s.rcode = take(2 * bhn * g.L * g.rcode_bytes);
  s.rcode_t = take(2 * bhn * g.L * g.rcode_bytes);
  s.race_count = take((size_t)g.BH * g.L * g.NB * 4);
  s.race_sum = take((size_t)g.BH * g.L * g.NB * g.d * 4);
  s.lse = take(bhn * 4);
  s.o_sp = take(bhn * g.d * g.esz);
  s.o_race = take(bhn * g.d * g.esz);
  s.ctot = take(bhn * 4);
  s.rank = take(g.rounds > 1 ? (size_t)g.rounds * 2 * bhn * 4 : 0);
  s.total = off;
  return s;
}

WorkLayout work_layout(const Geometry& g) {
  WorkLayout w;
  const size_t bhn = (size_t)g.BH * g.N;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes); return o; };
  w.err = take(256);
  w.sort_hist = take((size_t)2 * g.BH * g.sort_bins * g.sort_tiles * 4);
  w.sort_tmp = take(2 * bhn * 4);
  w.absmax = take((size_t)2 * g.BH * 4);
  w.gtab = take((size_t)g.BH * g.L * g.NB * g.d * 2);
  w.gl = take(bhn * sizeof(float2));
  w.count_scratch = take((size_t)g.BH * g.L * g.NB * 4);
  w.causal_num = take(g.causal ? bhn * g.d * 4 : 0);
  const size_t shared_base = off;
  // forward without a saved buffer: the saved layout lives here
  w.saved = take(saved_layout(g).total);
  // several hash rounds on the tcgen05 forward: each round's partial softmax
  const bool parts = g.rounds > 1 && g.tc_attn;
  w.round_o = take(parts ? (size_t)g.rounds * bhn * g.d * 4 : 0);
  w.round_lse = take(parts ? (size_t)g.rounds * bhn * 4 : 0);
  w.round_kr = take(parts ? (size_t)g.rounds * (g.rounds - 1) / 2 * bhn * 4 : 0);
  const size_t fwd_end = off;
  // backward temporaries reuse the same bytes (a backward always has a saved buffer)
  off = shared_base;
  w.d_o = take(bhn * g.d * g.esz);
  w.dprime = take(bhn * 4);
  w.dq_acc = take(bhn * g.d * 4);
  w.dk_acc = take(bhn * g.d * 4);
  w.dv_acc = take(bhn * g.d * 4);
  w.dor = take(bhn * g.d * g.esz);
  w.d_t = take((size_t)g.BH * g.L * g.NB * g.d * 4);
  w.partials = take((size_t)kParamBlocks * (2 * g.d + 3) * 4);
  w.total = off > fwd_end ? off : fwd_end;
  return w;
}

}  // namespace elsaa

using namespace elsaa;

namespace {

inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

inline cudaError_t mark(void* const* events, int i, cudaStream_t s) {
  if (!events || !events[i]) return cudaSuccess;
  return cudaEventRecord((cudaEvent_t)events[i], s);
}

// The RACE read-out runs from shared-memory table slabs where they fit; it
// takes the learned gates' logits from the hash GEMM.
bool slab_fwd(const Geometry& g) {
  return g.tc_hash && !g.causal && race_slab_supported(g, true) &&
         (g.gate_fixed || hash_tc_gate_logits_supported(g));
}
// The sparse forward streams the window in 128-key blocks where the
// lookback-1 pipeline does not apply (d = 128, chunks above 128, other
// lookbacks).
bool win_fwd(const Geometry& g) {
  return !(g.tc_attn && attn_pipe_supported(g)) && attn_win_supported(g);
}
// The persistent sparse backward writes dq, dk and dv itself; the RACE
// branch's dv is then added in place by a key-code gather.
bool direct_bwd(const Geometry& g) {
  return g.tc_attn && attn_bwd3_supported(g) && race_gather_add_supported(g);
}
bool slab_bwd(const Geometry& g) { return direct_bwd(g) && race_slab_supported(g, false); }
// The streamed-window sparse forward: one pass, or one per hash round and the
// combine of their partial softmaxes.
cudaError_t sparse_win(const Geometry& g, const void* q, const void* k, const void* v,
                       const int32_t* perm, const int32_t* rank, char* w, const WorkLayout& wl,
                       void* o_sp, float* lse, uint32_t* err, cudaStream_t s) {
  const size_t bhn = (size_t)g.BH * g.N;
  if (g.rounds == 1) return launch_attn_fwd_win(g, q, k, v, perm, perm + bhn, o_sp, lse, err, s);
  return launch_attn_fwd_win_rounds(g, q, k, v, perm, rank, (int32_t*)(w + wl.round_kr),
                                    (float*)(w + wl.round_o), (float*)(w + wl.round_lse), o_sp,
                                    lse, err, s);
}
// Several hash rounds: the tcgen05 hash GEMM gives every round's sort codes.
bool rounds_in_hash(const Geometry& g) {
  return g.rounds > 1 && g.tc_hash && hash_tc_rounds_supported(g, slab_fwd(g) && !g.gate_fixed);
}
// the shared-memory value-gradient gather on its own (any attention path)
bool slab_bwd_add(const Geometry& g) { return race_slab_supported(g, false); }

#define ELSAA_TRY(expr)                               \
  do {                                                \
    if ((expr) != cudaSuccess) return ELSAA_ERR_CUDA; \
  } while (0)

}  // namespace

extern "C" {

elsaa_status elsaa_validate(const elsaa_params* p) {
  Geometry g;
  elsaa_status why;
  make_geometry(p, &g, &why);
  return why;
}

size_t elsaa_workspace_bytes(const elsaa_params* p) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return 0;
  return work_layout(g).total;
}

size_t elsaa_saved_bytes(const elsaa_params* p) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return 0;
  return saved_layout(g).total;
}

int32_t elsaa_uses_tensor_cores(const elsaa_params* p) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return 0;
  return (g.tc_hash && g.tc_attn) ? 1 : 0;
}

elsaa_status elsaa_saved_views(const elsaa_params* p, const void* saved, elsaa_views* out) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return why;
  if (!saved || !out) return ELSAA_ERR_INVALID_ARG;
  const SavedLayout s = saved_layout(g);
  char* b = (char*)saved;
  const size_t bhn = (size_t)g.BH * g.N;
  out->code_q = (uint16_t*)(b + s.code);
  out->code_k = out->code_q + bhn;
  out->perm_q = (int32_t*)(b + s.perm);
  out->perm_k = out->perm_q + bhn;
  out->rcode_q = b + s.rcode;
  out->rcode_k = b + s.rcode + bhn * g.L * g.rcode_bytes;
  out->rcode_bytes = g.rcode_bytes;
  out->race_count = (int32_t*)(b + s.race_count);
  out->race_sum = (float*)(b + s.race_sum);
  out->lse_sp = (float*)(b + s.lse);
  out->o_sp = b + s.o_sp;
  out->o_race = b + s.o_race;
  out->ctot = (int32_t*)(b + s.ctot);
  out->round_code = (uint16_t*)(b + s.code);
  out->round_perm = (int32_t*)(b + s.perm);
  out->hash_rounds = g.rounds;
  return ELSAA_OK;
}

}  // extern "C"

namespace {

// RACE tables given by the caller instead of built from this call's keys (a
// sequence shard: the tables are sums over every shard's keys).
struct ExtTables {
  const float* sums;       // [BH][L][NB][d] fp32
  const int32_t* counts;   // [BH][L][NB]
};

elsaa_status forward_impl(const elsaa_params* p, const void* q, const void* k, const void* v,
                          const void* r_sort, const void* r_race, const float* gate_w,
                          const float* gate_b, const float* lambda, void* y, void* saved,
                          void* ws, size_t ws_bytes, void* stream, void* const* events,
                          const ExtTables* ext) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return why;
  if (ext && (g.causal || !ext->sums || !ext->counts)) return ELSAA_ERR_INVALID_ARG;
  if (!q || !k || !v || !lambda || !y || !ws) return ELSAA_ERR_INVALID_ARG;
  if ((g.sort_bits > 0 && !r_sort) || (g.kr > 0 && !r_race)) return ELSAA_ERR_INVALID_ARG;
  if (!g.gate_fixed && (!gate_w || !gate_b)) return ELSAA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, y, r_sort, r_race, gate_w, gate_b, saved};
  for (const void* x : ptrs)
    if (x && !aligned(x, 16)) return ELSAA_ERR_INVALID_ARG;
  if (!aligned(ws, 256) || (saved && !aligned(saved, 256))) return ELSAA_ERR_INVALID_ARG;
  const WorkLayout wl = work_layout(g);
  if (ws_bytes < wl.total) return ELSAA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* w = (char*)ws;
  char* sv = saved ? (char*)saved : w + wl.saved;
  const SavedLayout sl = saved_layout(g);
  const size_t bhn = (size_t)g.BH * g.N;
  uint16_t* code = (uint16_t*)(sv + sl.code);
  int32_t* perm = (int32_t*)(sv + sl.perm);
  char* rcode = sv + sl.rcode;
  char* rcode_k = rcode + bhn * g.L * g.rcode_bytes;
  char* rcode_t = sv + sl.rcode_t;   // table-major: queries, then keys
  char* rcode_tk = rcode_t + bhn * g.L * g.rcode_bytes;
  int32_t* counts = (int32_t*)(sv + sl.race_count);
  float* sums = (float*)(sv + sl.race_sum);
  float* lse = (float*)(sv + sl.lse);
  void* o_sp = sv + sl.o_sp;
  uint32_t* err = (uint32_t*)(w + wl.err);
  ELSAA_TRY(cudaMemsetAsync(err, 0, sizeof(uint32_t), s));
  ELSAA_TRY(mark(events, 0, s));

  const bool slab = slab_fwd(g);
  float2* gl = (slab && !g.gate_fixed) ? (float2*)(w + wl.gl) : nullptr;
  // 1. SimHash codes of Q and K (and the gate logits)
  if (g.tc_hash)
    ELSAA_TRY(launch_hash_tc(g, q, k, r_sort, r_race, code, rcode, rcode_t, gate_w, gl,
                             rounds_in_hash(g) ? g.rounds : 1, err, s));
  else
    ELSAA_TRY(launch_hash_simt(g, q, k, r_sort, r_race, code, rcode, rcode_t, s));
  // several hash rounds: the other rounds' sort codes
  if (g.rounds > 1 && !rounds_in_hash(g))
    ELSAA_TRY(launch_hash_sort_rounds(g, q, k, r_sort, code, s));
  ELSAA_TRY(mark(events, 1, s));
  // 2. Sort-LSH order of Q and K (every round), and with several rounds the
  // inverse orders the attention uses to count each key once
  for (int t = 0; t < g.rounds; ++t)
    ELSAA_TRY(launch_sort(g, code + (size_t)t * 2 * bhn, perm + (size_t)t * 2 * bhn,
                          (int32_t*)(w + wl.sort_hist), (int32_t*)(w + wl.sort_tmp), s));
  int32_t* rank = g.rounds > 1 ? (int32_t*)(sv + sl.rank) : nullptr;
  if (rank) ELSAA_TRY(launch_ranks(g, perm, rank, (int64_t)g.rounds * 2 * g.BH, s));
  ELSAA_TRY(mark(events, 2, s));
  if (g.causal) {
    // causal: the RACE read-out of query i takes keys j <= i only (a token
    // scan per table), the sparse window likewise
    float* num = (float*)(w + wl.causal_num);
    int32_t* ct = (int32_t*)(sv + sl.ctot);
    ELSAA_TRY(mark(events, 3, s));   // (no separate build stage)
    ELSAA_TRY(launch_race_causal_fwd(g, rcode, rcode_k, rcode_t, rcode_tk, v, num, ct, sums,
                                     counts, s));
    if (win_fwd(g))
      ELSAA_TRY(sparse_win(g, q, k, v, perm, rank, w, wl, o_sp, lse, err, s));
    else
      ELSAA_TRY(launch_attn_fwd_simt(g, q, k, v, perm, perm + bhn, rank, o_sp, lse, s));
    ELSAA_TRY(mark(events, 4, s));
    ELSAA_TRY(launch_fuse_causal(g, q, o_sp, lse, num, ct, gate_w, gate_b, lambda, y,
                                 sv + sl.o_race, s));
    ELSAA_TRY(mark(events, 5, s));
    return ELSAA_OK;
  }
  // 3. RACE tables from the keys (or the caller's tables)
  float* absmax = (float*)(w + wl.absmax);
  // gathers read tables in the data dtype: a bf16 copy, or the fp32 sums themselves
  __nv_bfloat16* gtab = g.bf16 ? (__nv_bfloat16*)(w + wl.gtab) : nullptr;
  const void* gather_tables = g.bf16 ? (const void*)gtab : (const void*)sums;
  if (ext) {
    const size_t tab = (size_t)g.BH * g.L * g.NB;
    ELSAA_TRY(cudaMemcpyAsync(sums, ext->sums, tab * g.d * 4, cudaMemcpyDeviceToDevice, s));
    ELSAA_TRY(cudaMemcpyAsync(counts, ext->counts, tab * 4, cudaMemcpyDeviceToDevice, s));
    if (gtab) ELSAA_TRY(launch_tables_to_bf16(g, sums, gtab, s));
  } else {
    ELSAA_TRY(launch_unit_absmax(g, v, false, absmax, s));
    ELSAA_TRY(launch_race_build(g, rcode_k, rcode_tk, v, false, absmax, sums, true, gtab, counts,
                                (int32_t*)(w + wl.count_scratch), err, s));
  }
  ELSAA_TRY(mark(events, 3, s));
  // 4. exact sparse branch
  if (g.tc_attn && attn_pipe_supported(g))
    ELSAA_TRY(launch_attn_fwd_pipe(g, q, k, v, perm, perm + bhn, o_sp, lse, err, s));
  else if (win_fwd(g))
    ELSAA_TRY(sparse_win(g, q, k, v, perm, rank, w, wl, o_sp, lse, err, s));
  else
    ELSAA_TRY(launch_attn_fwd_simt(g, q, k, v, perm, perm + bhn, rank, o_sp, lse, s));
  ELSAA_TRY(mark(events, 4, s));
  // 5. RACE gather, gates, multiplier and output
  if (slab)
    ELSAA_TRY(launch_race_slab_fuse(g, rcode, gather_tables, counts, o_sp, lse, gl, gate_b,
                                    lambda, y, saved ? sv + sl.o_race : nullptr,
                                    saved ? (int32_t*)(sv + sl.ctot) : nullptr, err, s));
  else
    ELSAA_TRY(launch_race_fuse_fwd(g, q, rcode, gather_tables, counts, o_sp, lse, gate_w, gate_b,
                                   lambda, y,
                                   saved ? sv + sl.o_race : nullptr,
                                   saved ? (int32_t*)(sv + sl.ctot) : nullptr, s));
  ELSAA_TRY(mark(events, 5, s));
  return ELSAA_OK;
}

elsaa_status backward_impl(const elsaa_params* p, const void* q, const void* k, const void* v,
                           const float* gate_w, const float* gate_b, const float* lambda,
                           const void* saved, const void* dy, void* dq, void* dk, void* dv,
                           float* dgate_w, float* dgate_b, float* dlambda, void* ws,
                           size_t ws_bytes, void* stream, void* const* events, float* d_tables) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return why;
  if (d_tables && g.causal) return ELSAA_ERR_INVALID_ARG;
  if (!q || !k || !v || !lambda || !saved || !dy || !dq || !dk || !dv || !dlambda || !ws)
    return ELSAA_ERR_INVALID_ARG;
  if (!g.gate_fixed && (!gate_w || !gate_b)) return ELSAA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, dy, dq, dk, dv};
  for (const void* x : ptrs)
    if (!aligned(x, 16)) return ELSAA_ERR_INVALID_ARG;
  if (!aligned(ws, 256) || !aligned(saved, 256)) return ELSAA_ERR_INVALID_ARG;
  const WorkLayout wl = work_layout(g);
  if (ws_bytes < wl.total) return ELSAA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* w = (char*)ws;
  const char* sv = (const char*)saved;
  const SavedLayout sl = saved_layout(g);
  const size_t bhn = (size_t)g.BH * g.N;
  const int32_t* perm = (const int32_t*)(sv + sl.perm);
  const int32_t* rank = g.rounds > 1 ? (const int32_t*)(sv + sl.rank) : nullptr;
  const char* rcode = sv + sl.rcode;
  const char* rcode_k = rcode + bhn * g.L * g.rcode_bytes;
  const char* rcode_t = sv + sl.rcode_t;   // table-major query codes
  const float* lse = (const float*)(sv + sl.lse);
  const void* o_sp = sv + sl.o_sp;
  const void* o_race = sv + sl.o_race;
  const int32_t* ctot = (const int32_t*)(sv + sl.ctot);
  void* d_o = w + wl.d_o;
  float* dprime = (float*)(w + wl.dprime);
  float* dq_acc = (float*)(w + wl.dq_acc);
  float* dk_acc = (float*)(w + wl.dk_acc);
  float* dv_acc = (float*)(w + wl.dv_acc);
  void* dor = w + wl.dor;
  float* d_t = (float*)(w + wl.d_t);
  float* partials = (float*)(w + wl.partials);
  ELSAA_TRY(cudaMemsetAsync(w + wl.err, 0, sizeof(uint32_t), s));
  ELSAA_TRY(mark(events, 0, s));

  // The persistent sparse backward writes dq, dk and dv itself; the RACE
  // branch's dv is then added in place by the key-code gather.
  const bool direct = direct_bwd(g);
  __nv_bfloat16* gtab = g.bf16 ? (__nv_bfloat16*)(w + wl.gtab) : nullptr;
  const void* race_grad = g.bf16 ? (const void*)gtab : (const void*)d_t;
  // 1. fusion and gate backward: dO_sp, D', the gate part of dq, g_r dy / Ctot
  float* absmax = (float*)(w + wl.absmax) + g.BH;
  float2* da = reinterpret_cast<float2*>(dq_acc);   // direct path: (da_s, da_r) per row
  ELSAA_TRY(launch_fuse_bwd(g, q, dy, o_sp, o_race, lse, ctot, gate_w, gate_b, lambda, d_o,
                            dprime, direct ? nullptr : dq_acc, direct ? da : nullptr, dor,
                            absmax, partials, s));
  ELSAA_TRY(mark(events, 1, s));
  // 2. RACE backward: scatter into the table gradient by query code (and, off
  // the direct path, gather by key code into dv_acc); causal: one reverse
  // token scan per table straight into dv_acc
  if (g.causal) {
    ELSAA_TRY(cudaMemsetAsync(dv_acc, 0, bhn * g.d * 4, s));
    ELSAA_TRY(launch_race_causal_bwd(g, rcode, rcode_k, rcode_t,
                                     rcode_t + bhn * g.L * g.rcode_bytes, dor, dv_acc, s));
  } else if (d_tables) {
    // the caller's table gradient (fp32); the value gradient of the RACE
    // branch is left to the caller (elsaa_race_value_grad once dT is summed)
    ELSAA_TRY(launch_race_build(g, rcode, rcode_t, dor, false, absmax, d_tables, true, nullptr,
                                nullptr, (int32_t*)(w + wl.count_scratch),
                                (uint32_t*)(w + wl.err), s));
    if (!direct) ELSAA_TRY(cudaMemsetAsync(dv_acc, 0, bhn * g.d * 4, s));
  } else {
    ELSAA_TRY(launch_race_build(g, rcode, rcode_t, dor, false, absmax, d_t, !g.bf16, gtab,
                                nullptr, (int32_t*)(w + wl.count_scratch),
                                (uint32_t*)(w + wl.err), s));
    if (!direct) ELSAA_TRY(launch_race_gather_sum(g, rcode_k, race_grad, dv_acc, s));
  }
  ELSAA_TRY(mark(events, 2, s));
  // 3. sparse branch backward, 4. outputs
  if (direct) {
    ELSAA_TRY(launch_attn_bwd3(g, q, k, v, perm, perm + bhn, d_o, lse, dprime, da,
                               g.gate_fixed ? nullptr : gate_w, dq, dk, dv,
                               (uint32_t*)(w + wl.err), s));
    ELSAA_TRY(mark(events, 3, s));
    if (d_tables) {
      // (the caller adds the RACE value gradient)
    } else if (slab_bwd(g)) {
      ELSAA_TRY(launch_race_slab_add(g, rcode_k, race_grad, dv, (uint32_t*)(w + wl.err), s));
    } else {
      ELSAA_TRY(launch_race_gather_add(g, rcode_k, race_grad, dv, s));
    }
  } else if (g.tc_attn && attn_bwd2_supported(g)) {
    ELSAA_TRY(launch_attn_bwd2(g, q, k, v, perm, perm + bhn, d_o, lse, dprime, dv_acc, dq_acc,
                               dk, dv, (uint32_t*)(w + wl.err), s));
    ELSAA_TRY(mark(events, 3, s));
    ELSAA_TRY(launch_cast_out(g, dq_acc, dq, s));
  } else if (g.tc_attn && g.rounds > 1) {
    // one key-major pass per hash round, dk and dv accumulated in fp32 (dv_acc
    // holds the RACE part)
    ELSAA_TRY(cudaMemsetAsync(dk_acc, 0, bhn * g.d * 4, s));
    ELSAA_TRY(launch_attn_bwd_tc_rounds(g, q, k, v, perm, rank, d_o, lse, dprime, dq_acc, dk_acc,
                                        dv_acc, (uint32_t*)(w + wl.err), s));
    ELSAA_TRY(mark(events, 3, s));
    ELSAA_TRY(launch_cast_out(g, dq_acc, dq, s));
    ELSAA_TRY(launch_cast_out(g, dk_acc, dk, s));
    ELSAA_TRY(launch_cast_out(g, dv_acc, dv, s));
  } else if (g.tc_attn) {
    ELSAA_TRY(launch_attn_bwd_tc(g, q, k, v, perm, perm + bhn, d_o, lse, dprime, dv_acc, dq_acc,
                                 dk, dv, (uint32_t*)(w + wl.err), s));
    ELSAA_TRY(mark(events, 3, s));
    ELSAA_TRY(launch_cast_out(g, dq_acc, dq, s));
  } else {
    ELSAA_TRY(cudaMemsetAsync(dk_acc, 0, bhn * g.d * 4, s));
    ELSAA_TRY(launch_attn_bwd_simt(g, q, k, v, perm, perm + bhn, rank, d_o, lse, dprime,
                                   dq_acc, dk_acc, dv_acc, s));
    ELSAA_TRY(mark(events, 3, s));
    ELSAA_TRY(launch_cast_out(g, dq_acc, dq, s));
    ELSAA_TRY(launch_cast_out(g, dk_acc, dk, s));
    ELSAA_TRY(launch_cast_out(g, dv_acc, dv, s));
  }
  ELSAA_TRY(launch_param_reduce(g, partials, dgate_w, dgate_b, dlambda, s));
  ELSAA_TRY(mark(events, 4, s));
  return ELSAA_OK;
}

}  // namespace

extern "C" {

elsaa_status elsaa_forward_staged(const elsaa_params* p, const void* q, const void* k,
                                  const void* v, const void* r_sort, const void* r_race,
                                  const float* gate_w, const float* gate_b, const float* lambda,
                                  void* y, void* saved, void* ws, size_t ws_bytes, void* stream,
                                  void* const* events) {
  return forward_impl(p, q, k, v, r_sort, r_race, gate_w, gate_b, lambda, y, saved, ws, ws_bytes,
                      stream, events, nullptr);
}

elsaa_status elsaa_forward(const elsaa_params* p, const void* q, const void* k, const void* v,
                           const void* r_sort, const void* r_race, const float* gate_w,
                           const float* gate_b, const float* lambda, void* y, void* saved,
                           void* ws, size_t ws_bytes, void* stream) {
  return forward_impl(p, q, k, v, r_sort, r_race, gate_w, gate_b, lambda, y, saved, ws, ws_bytes,
                      stream, nullptr, nullptr);
}

elsaa_status elsaa_forward_tables(const elsaa_params* p, const void* q, const void* k,
                                  const void* v, const void* r_sort, const void* r_race,
                                  const float* gate_w, const float* gate_b, const float* lambda,
                                  const float* race_sum, const int32_t* race_count, void* y,
                                  void* saved, void* ws, size_t ws_bytes, void* stream) {
  const ExtTables ext{race_sum, race_count};
  return forward_impl(p, q, k, v, r_sort, r_race, gate_w, gate_b, lambda, y, saved, ws, ws_bytes,
                      stream, nullptr, &ext);
}

elsaa_status elsaa_backward_staged(const elsaa_params* p, const void* q, const void* k,
                                   const void* v, const void* r_sort, const void* r_race,
                                   const float* gate_w, const float* gate_b, const float* lambda,
                                   const void* saved, const void* dy, void* dq, void* dk, void* dv,
                                   float* dgate_w, float* dgate_b, float* dlambda, void* ws,
                                   size_t ws_bytes, void* stream, void* const* events) {
  (void)r_sort;
  (void)r_race;
  return backward_impl(p, q, k, v, gate_w, gate_b, lambda, saved, dy, dq, dk, dv, dgate_w,
                       dgate_b, dlambda, ws, ws_bytes, stream, events, nullptr);
}

elsaa_status elsaa_backward(const elsaa_params* p, const void* q, const void* k, const void* v,
                            const void* r_sort, const void* r_race, const float* gate_w,
                            const float* gate_b, const float* lambda, const void* saved,
                            const void* dy, void* dq, void* dk, void* dv, float* dgate_w,
                            float* dgate_b, float* dlambda, void* ws, size_t ws_bytes,
                            void* stream) {
  (void)r_sort;
  (void)r_race;
  return backward_impl(p, q, k, v, gate_w, gate_b, lambda, saved, dy, dq, dk, dv, dgate_w,
                       dgate_b, dlambda, ws, ws_bytes, stream, nullptr, nullptr);
}

elsaa_status elsaa_backward_tables(const elsaa_params* p, const void* q, const void* k,
                                   const void* v, const void* r_sort, const void* r_race,
                                   const float* gate_w, const float* gate_b, const float* lambda,
                                   const void* saved, const void* dy, void* dq, void* dk, void* dv,
                                   float* dgate_w, float* dgate_b, float* dlambda,
                                   float* d_race_sum, void* ws, size_t ws_bytes, void* stream) {
  (void)r_sort;
  (void)r_race;
  if (!d_race_sum) return ELSAA_ERR_INVALID_ARG;
  return backward_impl(p, q, k, v, gate_w, gate_b, lambda, saved, dy, dq, dk, dv, dgate_w,
                       dgate_b, dlambda, ws, ws_bytes, stream, nullptr, d_race_sum);
}

elsaa_status elsaa_kernel_launches(const elsaa_params* p, int32_t* fwd, int32_t* bwd) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return why;
  if (!fwd || !bwd) return ELSAA_ERR_INVALID_ARG;
  // hash 1, sort 3 per pass, |V| max 1 + RACE build 1, sparse 1, RACE gather + fusion 1
  // (local order: one kernel writes token order instead of the radix passes;
  // causal: one RACE token scan, then the sparse branch and the fusion)
  // (several hash rounds: one more hash kernel, one sort per round and the
  // inverse orders; zero-bit extra codes are a memset)
  const int sort1 = g.sort_order == ELSAA_SORT_LOCAL ? 1 : 3 * g.sort_passes;
  const int sort = g.rounds * sort1 +
                   (g.rounds > 1 ? 1 + (g.sort_bits > 0 && !rounds_in_hash(g) ? 1 : 0) : 0);
  const int build = race_build_kernels(g, false, g.bf16);
  // (several rounds on tcgen05: the key ranks, one window pass per round and
  // the combine)
  const int sparse_fwd = g.rounds > 1 && win_fwd(g) ? 1 + g.rounds + 1 : 1;
  *fwd = g.causal ? 1 + sort + 1 + sparse_fwd + 1 : 1 + sort + 1 + build + sparse_fwd + 1;
  // fusion backward 1, RACE build 1 + gather 1, sparse 1 (+ casts), reduction 1
  // (direct path: the sparse kernel writes dq itself and the gather adds into dv)
  const bool direct = direct_bwd(g);
  // (several rounds on tcgen05: one key-major pass per round + 3 casts)
  const int sparse = direct ? 1 : g.tc_attn ? (g.rounds > 1 ? g.rounds + 3 : 1 + 1) : 1 + 3;
  // (the RACE backward: the table-gradient build, then, off the direct path, a gather)
  const int race_bwd = g.causal ? 1 : race_build_kernels(g, false, g.bf16) + (direct ? 0 : 1);
  *bwd = 1 + race_bwd + sparse + (direct ? 1 : 0) + 1;
  return ELSAA_OK;
}

// ---- pieces of the operator for a sequence split across devices ------------

elsaa_status elsaa_sort_codes_of(const elsaa_params* p, const void* q, const void* k,
                                 const void* r_sort, const void* r_race, uint16_t* code,
                                 void* ws, size_t ws_bytes, void* stream) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return why;
  if (!q || !k || !code || !ws || (g.sort_bits > 0 && !r_sort) || (g.kr > 0 && !r_race))
    return ELSAA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(code, 16) || !aligned(ws, 256))
    return ELSAA_ERR_INVALID_ARG;
  const WorkLayout wl = work_layout(g);
  if (ws_bytes < wl.total) return ELSAA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* w = (char*)ws;
  char* sv = w + wl.saved;   // the hash writes into the workspace's saved-state area
  const SavedLayout sl = saved_layout(g);
  const size_t bhn = (size_t)g.BH * g.N;
  uint16_t* c = (uint16_t*)(sv + sl.code);
  char* rcode = sv + sl.rcode;
  char* rcode_t = sv + sl.rcode_t;
  uint32_t* err = (uint32_t*)(w + wl.err);
  ELSAA_TRY(cudaMemsetAsync(err, 0, sizeof(uint32_t), s));
  if (g.tc_hash)
    ELSAA_TRY(
        launch_hash_tc(g, q, k, r_sort, r_race, c, rcode, rcode_t, nullptr, nullptr, 1, err, s));
  else
    ELSAA_TRY(launch_hash_simt(g, q, k, r_sort, r_race, c, rcode, rcode_t, s));
  ELSAA_TRY(cudaMemcpyAsync(code, c, 2 * bhn * 2, cudaMemcpyDeviceToDevice, s));
  return ELSAA_OK;
}

elsaa_status elsaa_sort_codes(const elsaa_params* p, const uint16_t* code, int32_t* perm,
                              void* ws, size_t ws_bytes, void* stream) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return why;
  if (!code || !perm || !ws) return ELSAA_ERR_INVALID_ARG;
  if (!aligned(code, 16) || !aligned(perm, 16) || !aligned(ws, 256)) return ELSAA_ERR_INVALID_ARG;
  const WorkLayout wl = work_layout(g);
  if (ws_bytes < wl.total) return ELSAA_ERR_WORKSPACE;
  char* w = (char*)ws;
  ELSAA_TRY(launch_sort(g, code, perm, (int32_t*)(w + wl.sort_hist), (int32_t*)(w + wl.sort_tmp),
                        (cudaStream_t)stream));
  return ELSAA_OK;
}

elsaa_status elsaa_race_tables(const elsaa_params* p, const void* k, const void* v,
                               const void* r_race, float* race_sum, int32_t* race_count,
                               void* ws, size_t ws_bytes, void* stream) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return why;
  if (!k || !v || !race_sum || !race_count || !ws || (g.kr > 0 && !r_race))
    return ELSAA_ERR_INVALID_ARG;
  const void* ptrs[] = {k, v, race_sum, race_count};
  for (const void* x : ptrs)
    if (!aligned(x, 16)) return ELSAA_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return ELSAA_ERR_INVALID_ARG;
  const WorkLayout wl = work_layout(g);
  if (ws_bytes < wl.total) return ELSAA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* w = (char*)ws;
  char* sv = w + wl.saved;
  const SavedLayout sl = saved_layout(g);
  const size_t bhn = (size_t)g.BH * g.N;
  uint16_t* c = (uint16_t*)(sv + sl.code);
  char* rcode = sv + sl.rcode;
  char* rcode_t = sv + sl.rcode_t;
  uint32_t* err = (uint32_t*)(w + wl.err);
  ELSAA_TRY(cudaMemsetAsync(err, 0, sizeof(uint32_t), s));
  // the keys' RACE codes (the hash also codes its first operand: the keys
  // again); no sort hyperplanes are read
  Geometry gk = g;
  gk.sort_bits = 0;
  if (gk.tc_hash)
    ELSAA_TRY(
        launch_hash_tc(gk, k, k, nullptr, r_race, c, rcode, rcode_t, nullptr, nullptr, 1, err, s));
  else
    ELSAA_TRY(launch_hash_simt(gk, k, k, nullptr, r_race, c, rcode, rcode_t, s));
  float* absmax = (float*)(w + wl.absmax);
  ELSAA_TRY(launch_unit_absmax(g, v, false, absmax, s));
  ELSAA_TRY(launch_race_build(g, rcode + bhn * g.L * g.rcode_bytes,
                              rcode_t + bhn * g.L * g.rcode_bytes, v, false, absmax, race_sum,
                              true, nullptr, race_count, (int32_t*)(w + wl.count_scratch), err,
                              s));
  return ELSAA_OK;
}

elsaa_status elsaa_race_value_grad(const elsaa_params* p, const void* k, const void* r_race,
                                   const float* d_race_sum, void* dv, void* ws, size_t ws_bytes,
                                   void* stream) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return why;
  if (!k || !d_race_sum || !dv || !ws || (g.kr > 0 && !r_race)) return ELSAA_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(d_race_sum, 16) || !aligned(dv, 16) || !aligned(ws, 256))
    return ELSAA_ERR_INVALID_ARG;
  if (!race_gather_add_supported(g)) return ELSAA_ERR_UNSUPPORTED;
  const WorkLayout wl = work_layout(g);
  if (ws_bytes < wl.total) return ELSAA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* w = (char*)ws;
  char* sv = w + wl.saved;
  const SavedLayout sl = saved_layout(g);
  const size_t bhn = (size_t)g.BH * g.N;
  uint16_t* c = (uint16_t*)(sv + sl.code);
  char* rcode = sv + sl.rcode;
  char* rcode_t = sv + sl.rcode_t;
  uint32_t* err = (uint32_t*)(w + wl.err);
  ELSAA_TRY(cudaMemsetAsync(err, 0, sizeof(uint32_t), s));
  Geometry gk = g;   // RACE codes of the keys only: no sort hyperplanes
  gk.sort_bits = 0;
  if (gk.tc_hash)
    ELSAA_TRY(
        launch_hash_tc(gk, k, k, nullptr, r_race, c, rcode, rcode_t, nullptr, nullptr, 1, err, s));
  else
    ELSAA_TRY(launch_hash_simt(gk, k, k, nullptr, r_race, c, rcode, rcode_t, s));
  const char* rcode_k = rcode + bhn * g.L * g.rcode_bytes;
  const void* tables = d_race_sum;
  if (g.bf16) {
    __nv_bfloat16* gtab = (__nv_bfloat16*)(w + wl.gtab);
    ELSAA_TRY(launch_tables_to_bf16(g, d_race_sum, gtab, s));
    tables = gtab;
  }
  if (slab_bwd_add(g))
    ELSAA_TRY(launch_race_slab_add(g, rcode_k, tables, dv, err, s));
  else
    ELSAA_TRY(launch_race_gather_add(g, rcode_k, tables, dv, s));
  return ELSAA_OK;
}

int32_t elsaa_path_flags(const elsaa_params* p) {
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return 0;
  return (g.tc_hash ? ELSAA_PATH_TC_HASH : 0) | (g.tc_attn ? ELSAA_PATH_TC_ATTN : 0) |
         (slab_fwd(g) ? ELSAA_PATH_SLAB_FWD : 0) | (slab_bwd(g) ? ELSAA_PATH_SLAB_BWD : 0) |
         (win_fwd(g) ? ELSAA_PATH_TC_WIN : 0);
}

elsaa_status elsaa_check(void* ws, void* stream) {
  if (!ws) return ELSAA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ELSAA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ELSAA_ERR_CUDA;
  if (word == 0) return ELSAA_OK;
  if (cudaMemset(ws, 0, sizeof(word)) != cudaSuccess) return ELSAA_ERR_CUDA;
  return (word & ERR_TIMEOUT) ? ELSAA_ERR_DEVICE_TIMEOUT : ELSAA_ERR_DEVICE_CHECK;
}

const char* elsaa_status_str(elsaa_status st) {
  switch (st) {
    case ELSAA_OK: return "ok";
    case ELSAA_ERR_INVALID_ARG: return "invalid argument";
    case ELSAA_ERR_UNSUPPORTED: return "unsupported problem";
    case ELSAA_ERR_WORKSPACE: return "workspace too small";
    case ELSAA_ERR_CUDA: return "CUDA error";
    case ELSAA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case ELSAA_ERR_DEVICE_CHECK: return "device index check failed";
  }
  return "unknown status";
}

}  // extern "C"
