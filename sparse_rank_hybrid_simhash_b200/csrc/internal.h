// Host-side layout of the saved state and workspace, and the kernel
// launchers each .cu file provides.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/elsaa.h"

namespace elsaa {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

// Sort-LSH radix pass geometry: digit of at most 8 bits, tiles of kSortTile keys.
constexpr int kSortTile = 2048;
constexpr int kSortThreads = 256;
// Sort-LSH hash rounds the library serves.
constexpr int kMaxRounds = 8;

struct Geometry {
  int B, H, N, d, BH;
  bool bf16;
  int esz;            // bytes per element of q/k/v
  int sort_bits, chunk, L, kr, NB;   // NB = 2^kr buckets
  int rcode_bytes;    // 1 or 2
  float scale;
  int gate_fixed;      // nonzero: constant gates gate_s, gate_r
  float gate_s, gate_r;
  int sort_order;      // elsaa_sort_order
  int lookback;        // previous chunks a query chunk attends (1: own and previous)
  int causal;          // keys j <= i only (sparse window and RACE read-out)
  int rounds;          // Sort-LSH hash rounds R >= 1
  int sort_passes, sort_digit_bits, sort_bins, sort_tiles;
  bool tc_hash;       // tcgen05 kernel for the SimHash codes
  bool tc_attn;       // tcgen05 kernels for the sparse branch
};

// Byte offsets inside the saved buffer.
struct SavedLayout {
  size_t code, perm, rcode, rcode_t, race_count, race_sum, lse, o_sp, o_race, ctot, rank, total;
  // code = [R][2][BH][N] u16 (per hash round: queries then keys); perm =
  // [R][2][BH][N] i32; rcode = [2][BH][N][L] (u8 or u16); rcode_t = the same
  // codes table-major, [2][BH][L][N]; rank = the inverse permutations
  // [R][2][BH][N] i32 (0 bytes for one round)
};

// Byte offsets inside the workspace.
struct WorkLayout {
  size_t err;                // 256 bytes: uint32 error word and spare
  size_t sort_hist;          // [2][BH][bins][tiles] i32
  size_t sort_tmp;           // [2][BH][N] i32 (intermediate order of a 2-pass sort)
  size_t absmax;             // [2][BH] f32: largest |value| per unit (forward V, backward g_r dy / Ctot)
  size_t gtab;               // [BH][L][NB][d] bf16: the table copy the RACE gathers read
  size_t gl;                 // [BH][N] float2: gate logits from the hash (shared-memory gathers)
  size_t count_scratch;      // [BH][L][NB] i32: bucket counts of a build that has no counts output
  size_t causal_num;         // [BH][N][d] f32: causal RACE numerators (0 bytes unless causal)
  size_t saved;              // a SavedLayout used when the forward has no saved buffer
  size_t round_o, round_lse; // [R][BH][N][d] / [R][BH][N] f32: per-round partial softmax
  size_t round_kr;           // [R (R - 1) / 2][BH][N] i32: keys' earlier-round ranks
                             // (several hash rounds on the tcgen05 forward; else 0 bytes)
  size_t d_o;                // [BH][N][d] dtype: dO_sp
  size_t dprime;             // [BH][N] f32: D' = dO_sp . O_sp - dlse
  size_t dq_acc, dk_acc, dv_acc;   // [BH][N][d] f32
  size_t dor;                // [BH][N][d] dtype: g_r dy / Ctot
  size_t d_t;                // [BH][L][NB][d] f32: RACE table gradient
  size_t partials;           // [kParamBlocks][2d+3] f32
  size_t total;
};

constexpr int kParamBlocks = 592;   // one wave of 4 x 148 SMs; fixed so the reduction order is fixed

bool make_geometry(const elsaa_params* p, Geometry* g, elsaa_status* why);
SavedLayout saved_layout(const Geometry& g);
WorkLayout work_layout(const Geometry& g);

// ---- launchers (each returns cudaGetLastError() after enqueueing) ----------

// SimHash codes of Q and K on CUDA cores (fp64 accumulation of exact products).
// Codes go out twice: row-major (rcode) and table-major (rcode_t).
cudaError_t launch_hash_simt(const Geometry& g, const void* q, const void* k, const void* r_sort,
                             const void* r_race, uint16_t* code, void* rcode, void* rcode_t,
                             cudaStream_t s);
// SimHash codes on tcgen05 tensor cores (bf16 products, fp32 accumulation).
// With gl non-null (learned gates) the same GEMM also writes the gate logits
// gl[row] = (w_s . q_row, w_r . q_row) of every query row, w = gate_w [2][d]
// fp32 (hash_tc_gate_logits_supported).
cudaError_t launch_hash_tc(const Geometry& g, const void* q, const void* k, const void* r_sort,
                           const void* r_race, uint16_t* code, void* rcode, void* rcode_t,
                           const float* gate_w, float2* gl, int rounds, uint32_t* err,
                           cudaStream_t s);
// The GEMM also gives the sort codes of hash rounds 1 .. R - 1 (rounds = R in
// launch_hash_tc; code then holds [R][2][BH][N]).
bool hash_tc_rounds_supported(const Geometry& g, bool gates);
// The bit-stream variant of the tcgen05 hash (hash_tc_stream.cu) for shapes
// whose codes do not fill whole words or whose word-aligned hyperplanes do not
// fit shared memory; launch_hash_tc chooses it.
bool hash_tc_stream_fits(const Geometry& g, bool gates);
cudaError_t launch_hash_tc_stream(const Geometry& g, const void* q, const void* k,
                                  const void* r_sort, const void* r_race, uint16_t* code,
                                  void* rcode, void* rcode_t, const float* gate_w, float2* gl,
                                  uint32_t* err, cudaStream_t s);
bool hash_tc_supported(const Geometry& g);
bool hash_tc_gate_logits_supported(const Geometry& g);

// Sort codes of hash rounds 1 .. R-1 (round 0 comes with the main hash):
// code[t][2][BH][N] from r_sort[t] ([R][sort_bits][d]), on CUDA cores.
cudaError_t launch_hash_sort_rounds(const Geometry& g, const void* q, const void* k,
                                    const void* r_sort, uint16_t* code, cudaStream_t s);
// rank[seg][perm[seg][x]] = x over `segs` segments of N.
cudaError_t launch_ranks(const Geometry& g, const int32_t* perm, int32_t* rank, int64_t segs,
                         cudaStream_t s);

// Stable Sort-LSH order of the 2*BH code segments.
cudaError_t launch_sort(const Geometry& g, const uint16_t* code, int32_t* perm, int32_t* hist,
                        int32_t* tmp, cudaStream_t s);

// Largest |value| of every unit (zeroes absmax first); the fixed-point scale
// of the RACE build is derived from it.
cudaError_t launch_unit_absmax(const Geometry& g, const void* vals, bool vals_f32, float* absmax,
                               cudaStream_t s);
// RACE tables: sums[bh][l][b][:] = sum of vals rows whose code in table l is b,
// counts (optional) likewise, and (gtab non-null) a bf16 copy for the gathers.
// vals_f32 selects fp32 values instead of dtype; absmax[bh] must bound |vals|
// of unit bh; keep_sums = false leaves `sums` as scratch only.
// codes: [BH][N][L] row-major; codes_t: the same codes [BH][L][N] table-major.
// count_scratch: [BH][L][NB] int32 the segmented build counts into when
// `counts` is null (long sequences need the counts to size the fixed-point grid).
// bf16 copy of fp32 tables [BH][L][NB][d] (what the gathers read).
cudaError_t launch_tables_to_bf16(const Geometry& g, const float* sums, __nv_bfloat16* gtab,
                                  cudaStream_t s);
// Kernels one launch_race_build enqueues (memsets excluded).
int race_build_kernels(const Geometry& g, bool vals_f32, bool gtab);
cudaError_t launch_race_build(const Geometry& g, const void* codes, const void* codes_t,
                              const void* vals,
                              bool vals_f32, const float* absmax, float* sums, bool keep_sums,
                              __nv_bfloat16* gtab, int32_t* counts, int32_t* count_scratch,
                              uint32_t* err, cudaStream_t s);
// out[bh][i][:] = sum_l tables[bh][l][codes[bh][i][l]][:]  (f32, overwritten);
// tables in the data dtype (bf16 copy, or the fp32 sums for fp32 data).
// dst[bh][i][:] += sum_l tables[bh][l][codes[bh][i][l]][:], dst in the data dtype
// (row-pipelined gather only: race_gather_add_supported).
bool race_gather_add_supported(const Geometry& g);
cudaError_t launch_race_gather_add(const Geometry& g, const void* codes, const void* tables,
                                   void* dst, cudaStream_t s);
cudaError_t launch_race_gather_sum(const Geometry& g, const void* codes, const void* tables,
                                   float* out, cudaStream_t s);
// RACE read-out from tables resident in shared memory (race_slab.cu): bf16
// data, one-byte codes, 16 or 32 tables.  Forward: gathers by query codes
// fused with the gates (gl from the hash when learned), the multiplier and the
// output; add: dst[row] += the gathered table rows (the RACE value gradient).
bool race_slab_supported(const Geometry& g, bool fuse);
cudaError_t launch_race_slab_fuse(const Geometry& g, const void* rcode_q, const void* tables,
                                  const int32_t* counts, const void* o_sp, const float* lse,
                                  const float2* gl, const float* gate_b, const float* lam,
                                  void* y, void* o_race, int32_t* ctot, uint32_t* err,
                                  cudaStream_t s);
cudaError_t launch_race_slab_add(const Geometry& g, const void* codes, const void* tables,
                                 void* dst, uint32_t* err, cudaStream_t s);
// Forward RACE gather fused with the gates, the multiplier and the output.
cudaError_t launch_race_fuse_fwd(const Geometry& g, const void* q, const void* rcode_q,
                                 const void* tables, const int32_t* counts,
                                 const void* o_sp, const float* lse, const float* gate_w,
                                 const float* gate_b, const float* lam, void* y, void* o_race,
                                 int32_t* ctot, cudaStream_t s);

// Sparse branch, CUDA-core kernels.  perm_q / perm_k are round 0's; with
// g.rounds > 1 round t's permutations sit t * 2 BH N further, and `rank`
// holds every round's inverse permutations ([R][2][BH][N]; unused for one round).
cudaError_t launch_attn_fwd_simt(const Geometry& g, const void* q, const void* k, const void* v,
                                 const int32_t* perm_q, const int32_t* perm_k,
                                 const int32_t* rank, void* o_sp, float* lse, cudaStream_t s);
cudaError_t launch_attn_bwd_simt(const Geometry& g, const void* q, const void* k, const void* v,
                                 const int32_t* perm_q, const int32_t* perm_k,
                                 const int32_t* rank, const void* d_o, const float* lse,
                                 const float* dprime, float* dq_acc, float* dk_acc,
                                 float* dv_acc, cudaStream_t s);
// Sparse branch, tcgen05 kernels.  attn_tc_supported: the shapes whose
// forward and backward both run on them (bf16, d = 64 or 128, N % 128 == 0,
// any chunk c % 16 == 0 and any lookback, with or without the causal mask).
bool attn_tc_supported(const Geometry& g);
// Overlapped backward (d = 64, chunk 64 or 128).
// Persistent backward (d = 64, bf16, chunk dividing 128): writes dq (the gate
// part da_s w_s + da_r w_r from the per-row pair da, plus the sparse part),
// dk, and dv (sparse part only) directly.  gate_w may be NULL (fixed gates).
bool attn_bwd3_supported(const Geometry& g);
cudaError_t launch_attn_bwd3(const Geometry& g, const void* q, const void* k, const void* v,
                             const int32_t* perm_q, const int32_t* perm_k, const void* d_o,
                             const float* lse, const float* dprime, const float2* da,
                             const float* gate_w, void* dq, void* dk, void* dv, uint32_t* err,
                             cudaStream_t s);
bool attn_bwd2_supported(const Geometry& g);
cudaError_t launch_attn_bwd2(const Geometry& g, const void* q, const void* k, const void* v,
                             const int32_t* perm_q, const int32_t* perm_k, const void* d_o,
                             const float* lse, const float* dprime, const float* dv_race,
                             float* dq_acc, void* dk, void* dv, uint32_t* err, cudaStream_t s);
// Persistent warp-specialized forward (d = 64, chunk <= 128 dividing 128,
// lookback 1).
bool attn_pipe_supported(const Geometry& g);
cudaError_t launch_attn_fwd_pipe(const Geometry& g, const void* q, const void* k, const void* v,
                                 const int32_t* perm_q, const int32_t* perm_k, void* o_sp,
                                 float* lse, uint32_t* err, cudaStream_t s);
// Persistent forward over any Sort-LSH window, streamed in 128-key blocks
// (bf16, d = 64 or 128, one hash round, optionally causal).
bool attn_win_supported(const Geometry& g);
cudaError_t launch_attn_fwd_win(const Geometry& g, const void* q, const void* k, const void* v,
                                const int32_t* perm_q, const int32_t* perm_k, void* o_sp,
                                float* lse, uint32_t* err, cudaStream_t s);
// Several hash rounds: the keys' earlier-round ranks in each round's key order
// (kranks, [R (R - 1) / 2][BH][N] i32), one streamed-window pass per round
// (perm and rank [R][2][BH][N]), each writing its partial softmax to o_part /
// lse_part, then their combine into o_sp and lse.
cudaError_t launch_attn_fwd_win_rounds(const Geometry& g, const void* q, const void* k,
                                       const void* v, const int32_t* perm, const int32_t* rank,
                                       int32_t* kranks, float* o_part, float* lse_part,
                                       void* o_sp, float* lse, uint32_t* err, cudaStream_t s);
// tcgen05 backward for any window (key-major, one CTA per 128 sorted keys):
// dq_acc += dQ (fp32 atomics); dk, dv written (dv adds dv_race).
cudaError_t launch_attn_bwd_tc(const Geometry& g, const void* q, const void* k, const void* v,
                               const int32_t* perm_q, const int32_t* perm_k, const void* d_o,
                               const float* lse, const float* dprime, const float* dv_race,
                               float* dq_acc, void* dk, void* dv, uint32_t* err, cudaStream_t s);
// Several hash rounds: one key-major pass per round with the final lse,
// masking keys an earlier round's window of the query holds; dq_acc += dQ,
// dk_acc += dK, dv_acc += dV (fp32).
cudaError_t launch_attn_bwd_tc_rounds(const Geometry& g, const void* q, const void* k,
                                      const void* v, const int32_t* perm, const int32_t* rank,
                                      const void* d_o, const float* lse, const float* dprime,
                                      float* dq_acc, float* dk_acc, float* dv_acc, uint32_t* err,
                                      cudaStream_t s);

// Backward of the fusion and gates (per query), then the parameter reduction
// and the final casts.
// absmax[bh] (zeroed by the launcher) receives the largest |g_r dy / Ctot| of unit bh.
cudaError_t launch_fuse_bwd(const Geometry& g, const void* q, const void* dy, const void* o_sp,
                            const void* o_race, const float* lse, const int32_t* ctot,
                            const float* gate_w, const float* gate_b, const float* lam,
                            void* d_o, float* dprime, float* dq_acc, float2* da_out, void* dor,
                            float* absmax, float* partials, cudaStream_t s);
cudaError_t launch_param_reduce(const Geometry& g, const float* partials, float* dgate_w,
                                float* dgate_b, float* dlambda, cudaStream_t s);
cudaError_t launch_cast_out(const Geometry& g, const float* src, void* dst, cudaStream_t s);

// Causal RACE (race_causal.cu): token walks over the tables and the fusion on
// their read-out.  Codes row-major (rcode_*) and table-major (rcode_t*).
// num [BH][N][d] fp32 and ctot [BH][N] receive the prefix read-out, sums /
// counts the full tables; the backward writes the RACE value gradient into
// dv_acc (which must be zero on entry).
bool race_causal_supported(const Geometry& g);
cudaError_t launch_race_causal_fwd(const Geometry& g, const void* rcode_q, const void* rcode_k,
                                   const void* rcode_tq, const void* rcode_tk, const void* v,
                                   float* num, int32_t* ctot, float* sums, int32_t* counts,
                                   cudaStream_t s);
cudaError_t launch_race_causal_bwd(const Geometry& g, const void* rcode_q, const void* rcode_k,
                                   const void* rcode_tq, const void* rcode_tk, const void* dor,
                                   float* dv_acc, cudaStream_t s);
cudaError_t launch_fuse_causal(const Geometry& g, const void* q, const void* o_sp,
                               const float* lse, const float* num, const int32_t* ctot,
                               const float* gate_w, const float* gate_b, const float* lam,
                               void* y, void* o_race, cudaStream_t s);

// 2-D TMA map over a [rows, width] bf16 matrix (width 64 or 128): a box is 64
// columns of one row (128 bytes), 128-byte swizzle; the row gathers of the
// tcgen05 attention kernels use it.
cudaError_t make_row_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t width = 64);
// 3-D TMA map over a [units, n, d] bf16 tensor (d contiguous), no swizzle, box
// of 8 columns x box_rows rows x 1 unit: the RACE slab kernels' row tiles.
cudaError_t make_slab_map(CUtensorMap* map, const void* base, uint64_t units, uint64_t n,
                          uint64_t d, uint32_t box_rows);

}  // namespace elsaa
