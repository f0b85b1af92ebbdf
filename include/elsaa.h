/*
 * libelsaa: the ELSAA attention operator (forward and backward) on NVIDIA B200.
 *
 * ELSAA ("ELSAA: Efficient Low-Rank and Sparse Attention Approximation for
 * Training Transformers", overview) is the attention applied after the dense
 * Q/K/V projections (non-causal on the pages; elsaa_params.causal adds a
 * causal variant).  Per (batch, head) unit, with Q, K, V in R^{N x d}:
 *
 *   1. SimHash codes: bit j of a row x is [x . r_j > 0].  A sort code of
 *      sort_bits bits from r_sort, and one code of race_bits bits per RACE
 *      table l from r_race[l] (bit j has weight 2^j).
 *   2. Sort-LSH: Q and K are each ordered by their sort code, ties by token
 *      index (stable).  Sorted query chunk j (chunk rows) attends sorted key
 *      chunks j-1 and j (chunk 0 only its own), no wrap-around.
 *      (elsaa_params.sort_order, lookback and hash_rounds select other
 *      orders, window widths and several hash rounds.)
 *   3. Exact sparse branch: O_sp = softmax(scale * q k^T) V over that window
 *      and its unshifted mass Z_sp = exp(lse_sp) ("Two Efficient Attentions,
 *      One Denominator Problem", section "Two efficient branches can still be
 *      mis-scaled": the sparse branch evaluates only the selected
 *      interactions, exactly).
 *   4. Low-rank RACE branch: L tables of 2^race_bits buckets; C[l][b] counts
 *      the keys with h_l(k) = b and T[l][b] sums their values.  A query reads
 *      its bucket in every table: Ctot = sum_l C[l][h_l(q)],
 *      O_race = sum_l T[l][h_l(q)] / Ctot (0 if Ctot = 0), Z_race = Ctot / L.
 *   5. Denominator-aware fusion (same page and section; the formula itself is
 *      lost from the text, this library takes the mass ratio)
 *      m = Z_sp / (Z_sp + lambda * Z_race), m = 1 when lambda * Z_race = 0.
 *   6. Independent token-wise gates (ELSAA overview: "learned or fixed
 *      gates"): g_s = sigmoid(w_s . q_i + b_s), g_r = sigmoid(w_r . q_i + b_r)
 *      or fixed constants, and y = g_s * m * O_sp + g_r * O_race.
 *
 * Conventions for every entry point:
 *   - Every pointer named "device" is CUDA device memory owned by the caller.
 *     The library never allocates or frees device or pinned memory.  Apart
 *     from elsaa_sort_codes_noalloc (one fixed device array shared by all of
 *     its calls, and a cache of that array's address per CUDA context; see
 *     its comment) it keeps no mutable global state: calls on different
 *     streams with different workspaces may run concurrently.
 *   - All work is enqueued on `stream` (a cudaStream_t passed as void*; NULL
 *     is the legacy default stream).  Calls return without synchronising;
 *     device-side failures (a bounded wait that ran out) are recorded in the
 *     workspace's error word and read back by elsaa_check().
 *   - Layouts are dense and row-major: q, k, v, y, dy, dq, dk, dv are
 *     [B, H, N, d] with d contiguous, in params->dtype.
 *   - On an error status the contents of every output are undefined.  Host
 *     validation errors are returned before anything is enqueued.
 */
#ifndef ELSAA_H
#define ELSAA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ELSAA_OK = 0,
  ELSAA_ERR_INVALID_ARG = 1,     /* a null pointer, a bad size or misaligned buffer */
  ELSAA_ERR_UNSUPPORTED = 2,     /* a valid request this library does not implement */
  ELSAA_ERR_WORKSPACE = 3,       /* ws_bytes smaller than elsaa_workspace_bytes() */
  ELSAA_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed */
  ELSAA_ERR_DEVICE_TIMEOUT = 5,  /* a kernel's bounded wait ran out (elsaa_check) */
  ELSAA_ERR_DEVICE_CHECK = 6     /* a kernel's own index check failed (elsaa_check) */
} elsaa_status;

typedef enum { ELSAA_BF16 = 0, ELSAA_F32 = 1 } elsaa_dtype;

/* Order of the Sort-LSH chunks ("Two Efficient Attentions, One Denominator
 * Problem", section "The ablation isolates the actual contribution": tokens
 * sorted by hash code, consecutive chunks attend).  BINARY sorts by the code
 * value (the pages' Sort-LSH); GRAY sorts by the code's position in the
 * reflected binary Gray sequence, so neighbouring buckets differ in one
 * hyperplane (an extension); LOCAL keeps token order, i.e. local windows of
 * consecutive tokens (the ELSAA overview lists local windows among the sparse
 * patterns).  Every order is stable: equal keys keep token order. */
typedef enum { ELSAA_SORT_BINARY = 0, ELSAA_SORT_GRAY = 1, ELSAA_SORT_LOCAL = 2 } elsaa_sort_order;

typedef struct {
  int32_t B, H, N, d;     /* batch, heads, tokens per unit, head dim d in {32, 64, 128} */
  int32_t dtype;          /* elsaa_dtype of q, k, v, r_sort, r_race, y, dy, dq, dk, dv */
  int32_t sort_bits;      /* Sort-LSH code bits, 0..16 */
  int32_t chunk;          /* Sort-LSH chunk length; N % chunk == 0 */
  int32_t race_tables;    /* L >= 1 */
  int32_t race_bits;      /* bits per RACE code, 0..16 (2^race_bits buckets per table) */
  float scale;            /* score scale; <= 0 selects 1/sqrt(d) */
  int32_t gate_fixed;     /* nonzero: gates are the constants gate_s, gate_r */
  float gate_s, gate_r;
  int32_t sort_order;     /* elsaa_sort_order of the Sort-LSH chunks */
  int32_t lookback;       /* previous sorted chunks a query chunk attends besides its own,
                           * 0..64 with (lookback + 1) * chunk <= 6144: 1 is the pages'
                           * Sort-LSH (own and previous chunk); other values are an
                           * extension (bf16: the streamed-window tcgen05 forward and
                           * the key-major tcgen05 backward) */
  int32_t causal;         /* nonzero: query i sees only keys j <= i (token index), in the
                           * sparse window and in the RACE read-out (an extension: the
                           * pages did not evaluate causal use); a window left without
                           * keys has Z_sp = 0 (O_sp = 0, lse = -inf).  bf16 runs on
                           * the tcgen05 window forward and key-major backward with a
                           * token mask; the RACE read-out walks the tables token by
                           * token (L in {4, 8, 16, 32} and N % 32 == 0 with
                           * 2 * 2^race_bits * 128 <= 200 KB, else per-table scans that
                           * need 2^race_bits * (d + 1) * 4 <= 200 KB) */
  int32_t hash_rounds;    /* Sort-LSH hash rounds, 0..8 (0 and 1 both mean one round, the
                           * pages' setting).  With R > 1 rounds every round t sorts Q
                           * and K by its own sort hyperplanes r_sort[t], and a query
                           * attends the union of its R windows, each key once, with
                           * exact softmax (an extension; bf16: every round's codes from
                           * the hash GEMM, one tcgen05 window pass per round and a
                           * combine, one backward pass per round; needs R * (lookback
                           * + 1) * chunk <= 6144) */
} elsaa_params;

/* Device views into a forward's saved state (see elsaa_saved_views). */
typedef struct {
  uint16_t* code_q;       /* [B,H,N] sort codes of the queries */
  uint16_t* code_k;       /* [B,H,N] sort codes of the keys */
  int32_t* perm_q;        /* [B,H,N] token index at each sorted rank */
  int32_t* perm_k;        /* [B,H,N] */
  void* rcode_q;          /* [B,H,N,L] RACE codes, uint8 if race_bits <= 8 else uint16 */
  void* rcode_k;          /* [B,H,N,L] */
  int32_t rcode_bytes;    /* 1 or 2 */
  int32_t* race_count;    /* [B,H,L,2^race_bits] C */
  float* race_sum;        /* [B,H,L,2^race_bits,d] T */
  float* lse_sp;          /* [B,H,N] natural-log mass of the sparse window, token order */
  void* o_sp;             /* [B,H,N,d] sparse-branch output (dtype), token order */
  void* o_race;           /* [B,H,N,d] RACE-branch output (dtype), token order */
  int32_t* ctot;          /* [B,H,N] Ctot */
  uint16_t* round_code;   /* [R][2][B,H,N] sort codes of every hash round (queries then keys
                           * per round); round 0 is code_q / code_k */
  int32_t* round_perm;    /* [R][2][B,H,N] permutations of every round; round 0 is
                           * perm_q / perm_k */
  int32_t hash_rounds;    /* R */
} elsaa_views;

/* Returns ELSAA_OK if `p` describes a supported problem, else the reason. */
elsaa_status elsaa_validate(const elsaa_params* p);

/* Bytes of device workspace one forward or backward needs (the same figure
 * serves both); 0 if `p` is invalid.  Workspace contents need not be
 * initialised and are not preserved between calls except its error word. */
size_t elsaa_workspace_bytes(const elsaa_params* p);

/* Bytes of the saved state a training forward writes and the matching
 * backward reads; 0 if `p` is invalid. */
size_t elsaa_saved_bytes(const elsaa_params* p);

/* Forward.  q, k, v: device [B,H,N,d]; r_sort: device [R, sort_bits, d] with
 * R = hash_rounds (may be NULL when sort_bits = 0); r_race: device [L, race_bits, d] (may be NULL
 * when race_bits = 0); hyperplanes are shared by Q and K and by every unit
 * and have the data dtype.  gate_w: device fp32 [2,d] (row 0 sparse, row 1 RACE),
 * gate_b: device fp32 [2]; both ignored (may be NULL) if gate_fixed.
 * lambda: device fp32 scalar.  y: device [B,H,N,d] output.  saved: device
 * buffer of elsaa_saved_bytes() or NULL for inference.  ws: device buffer of
 * at least elsaa_workspace_bytes(), 256-byte aligned; its first 4 bytes are
 * the error word elsaa_check() reads.  All device pointers
 * must be 16-byte aligned. */
elsaa_status elsaa_forward(const elsaa_params* p, const void* q, const void* k, const void* v,
                           const void* r_sort, const void* r_race, const float* gate_w,
                           const float* gate_b, const float* lambda, void* y, void* saved,
                           void* ws, size_t ws_bytes, void* stream);

/* Backward of sum(y * dy) with the hash codes held constant (they are
 * piecewise constant).  Inputs as for elsaa_forward plus `saved` written by
 * a forward with the same inputs and dy: device [B,H,N,d].  Outputs (all
 * overwritten, never accumulated): dq, dk, dv device [B,H,N,d] (dtype);
 * dgate_w device fp32 [2,d] and dgate_b device fp32 [2] (written as zeros
 * when gate_fixed; may be NULL then); dlambda device fp32 scalar.  The gate
 * weights and lambda are shared by every unit, so their gradients are sums
 * over B, H and N. */
elsaa_status elsaa_backward(const elsaa_params* p, const void* q, const void* k, const void* v,
                            const void* r_sort, const void* r_race, const float* gate_w,
                            const float* gate_b, const float* lambda, const void* saved,
                            const void* dy, void* dq, void* dk, void* dv, float* dgate_w,
                            float* dgate_b, float* dlambda, void* ws, size_t ws_bytes,
                            void* stream);

/* Stages of one call, for per-kernel timing: elsaa_forward_staged and
 * elsaa_backward_staged take `events`, an array of ELSAA_*_STAGES + 1
 * cudaEvent_t handles (passed as void*; any entry may be NULL) created by the
 * caller; events[0] is recorded on `stream` before the first stage and
 * events[i + 1] after stage i.  Forward stages: SimHash codes, Sort-LSH
 * order, RACE build, sparse branch, RACE gather + fusion (causal: the RACE
 * token scan runs in the sparse-branch stage and the build stage is empty).  Backward stages:
 * fusion/gate backward, RACE backward, sparse backward, final casts and the
 * parameter-gradient reduction.  Otherwise identical to elsaa_forward and
 * elsaa_backward (which are these calls with events = NULL). */
#define ELSAA_FWD_STAGES 5
#define ELSAA_BWD_STAGES 4
elsaa_status elsaa_forward_staged(const elsaa_params* p, const void* q, const void* k,
                                  const void* v, const void* r_sort, const void* r_race,
                                  const float* gate_w, const float* gate_b, const float* lambda,
                                  void* y, void* saved, void* ws, size_t ws_bytes, void* stream,
                                  void* const* events);
elsaa_status elsaa_backward_staged(const elsaa_params* p, const void* q, const void* k,
                                   const void* v, const void* r_sort, const void* r_race,
                                   const float* gate_w, const float* gate_b, const float* lambda,
                                   const void* saved, const void* dy, void* dq, void* dk, void* dv,
                                   float* dgate_w, float* dgate_b, float* dlambda, void* ws,
                                   size_t ws_bytes, void* stream, void* const* events);

/* Number of kernels one elsaa_forward (fwd) and one elsaa_backward (bwd)
 * enqueue for `p` (memsets excluded). */
elsaa_status elsaa_kernel_launches(const elsaa_params* p, int32_t* fwd, int32_t* bwd);

/* Sort-LSH order of given sort codes, using no memory the caller or the
 * library allocates.  The paper has no counterpart: this exists for callers
 * that cannot provide scratch memory, such as a serving process whose pool
 * already holds all device memory, or a framework that forbids cudaMalloc and
 * cudaFree (which synchronise the device) during a step.
 * code: device [2][B,H,N] uint16, the sort codes of the queries followed by
 * those of the keys (elsaa_views.code_q is the start of both); perm: device
 * [2][B,H,N] int32 output, the token index at each sorted rank, equal to the
 * permutations elsaa_forward saves (for one hash round: hash_rounds is not
 * read).  Both 16-byte aligned.  Only p->B, H, N, sort_bits and sort_order
 * matter, but p must validate.
 * The radix sort's scratch sits in one fixed device array of
 * ELSAA_NOALLOC_SCRATCH_BYTES that every device loading the library keeps
 * until exit.  The first call in a CUDA context looks up that array's device
 * address in the current context, so make it before any stream capture; a
 * context created later (after cudaDeviceReset, or another context made
 * current) repeats the lookup on its first call.
 * Returns ELSAA_ERR_WORKSPACE if the problem needs more scratch than that
 * (2 B H 2^digit_bits ceil(N/2048) ints, plus 2 B H N ints when sort_bits > 8).
 * All calls share the array: calls that may overlap on the GPU (other
 * streams, other host threads on the same device) race and must be ordered
 * by the caller.  No part of the array needs to start cleared. */
#define ELSAA_NOALLOC_SCRATCH_BYTES (4u << 20)
elsaa_status elsaa_sort_codes_noalloc(const elsaa_params* p, const uint16_t* code, int32_t* perm,
                                      void* stream);

/* Fills `out` with device pointers into `saved` (no device access). */
elsaa_status elsaa_saved_views(const elsaa_params* p, const void* saved, elsaa_views* out);

/* Synchronises `stream`, reads and clears the workspace error word (which
 * every forward and backward clears when it starts), and
 * returns ELSAA_OK, ELSAA_ERR_DEVICE_TIMEOUT or ELSAA_ERR_DEVICE_CHECK. */
elsaa_status elsaa_check(void* ws, void* stream);

/* Static text for a status code. */
const char* elsaa_status_str(elsaa_status s);

/* Which kernel family the sparse branch and the hash take for `p`:
 * 1 = tcgen05 tensor-core kernels, 0 = CUDA-core kernels (fp32 data, head
 * dims other than 64/128, N not a multiple of 128, or chunks that are not
 * a multiple of 16). */
int32_t elsaa_uses_tensor_cores(const elsaa_params* p);

/* ---- Pieces of the operator for a sequence split across devices ---------
 *
 * A sequence can be split into token shards on several devices (the
 * package's sharding module): every shard's sort codes are gathered, every
 * device computes the same global Sort-LSH orders, the rows of each device's
 * range of sorted chunks (and one chunk before it) are exchanged to it, and
 * the RACE tables are summed over the shards.  These calls are the device
 * steps of that scheme; p describes the problem each call runs on (the shard,
 * or a device's sorted range).  All pointers are device memory; ws is a
 * workspace of elsaa_workspace_bytes(p).  Sharded problems need one hash
 * round and no causal mask (p is rejected otherwise where it matters). */

/* Sort codes of q and k ([B,H,N,d]): code [2][B,H,N] uint16 (queries then
 * keys), as elsaa_forward computes them. */
elsaa_status elsaa_sort_codes_of(const elsaa_params* p, const void* q, const void* k,
                                 const void* r_sort, const void* r_race, uint16_t* code,
                                 void* ws, size_t ws_bytes, void* stream);

/* Stable Sort-LSH order (p->sort_order) of given codes [2][B,H,N] uint16:
 * perm [2][B,H,N] int32, the token index at each sorted rank. */
elsaa_status elsaa_sort_codes(const elsaa_params* p, const uint16_t* code, int32_t* perm,
                              void* ws, size_t ws_bytes, void* stream);

/* RACE tables of the keys k and values v ([B,H,N,d]): race_sum [B,H,L,2^K_r,d]
 * fp32 and race_count [B,H,L,2^K_r] int32 (overwritten).  Tables of several
 * shards of one sequence add up to the tables of the whole sequence. */
elsaa_status elsaa_race_tables(const elsaa_params* p, const void* k, const void* v,
                               const void* r_race, float* race_sum, int32_t* race_count,
                               void* ws, size_t ws_bytes, void* stream);

/* elsaa_forward with the RACE tables given (race_sum / race_count as above,
 * e.g. summed over every shard of the sequence) instead of built from k and v.
 * The tables are copied into the saved state. */
elsaa_status elsaa_forward_tables(const elsaa_params* p, const void* q, const void* k,
                                  const void* v, const void* r_sort, const void* r_race,
                                  const float* gate_w, const float* gate_b, const float* lambda,
                                  const float* race_sum, const int32_t* race_count, void* y,
                                  void* saved, void* ws, size_t ws_bytes, void* stream);

/* elsaa_backward of a forward made by elsaa_forward_tables: writes the RACE
 * table gradient dT = d sum(y dy) / d race_sum of this call's queries into
 * d_race_sum ([B,H,L,2^K_r,d] fp32, overwritten) and leaves the RACE branch's
 * value gradient out of dv (dv holds the sparse branch's part only; see
 * elsaa_race_value_grad). */
elsaa_status elsaa_backward_tables(const elsaa_params* p, const void* q, const void* k,
                                   const void* v, const void* r_sort, const void* r_race,
                                   const float* gate_w, const float* gate_b, const float* lambda,
                                   const void* saved, const void* dy, void* dq, void* dk, void* dv,
                                   float* dgate_w, float* dgate_b, float* dlambda,
                                   float* d_race_sum, void* ws, size_t ws_bytes, void* stream);

/* The RACE branch's value gradient of keys k: dv[j] += sum_l dT[l][h_l(k_j)]
 * (dv in the data dtype, [B,H,N,d]; d_race_sum as written by
 * elsaa_backward_tables, summed over the shards). */
elsaa_status elsaa_race_value_grad(const elsaa_params* p, const void* k, const void* r_race,
                                   const float* d_race_sum, void* dv, void* ws, size_t ws_bytes,
                                   void* stream);

/* Bit mask of the kernel families elsaa_forward / elsaa_backward take for
 * `p` (0 if p is invalid): ELSAA_PATH_TC_HASH the tcgen05 SimHash GEMM;
 * ELSAA_PATH_TC_ATTN the tcgen05 sparse branch; ELSAA_PATH_SLAB_FWD the RACE
 * read-out from shared-memory table slabs (gate logits from the hash GEMM);
 * ELSAA_PATH_SLAB_BWD the RACE value gradient from shared-memory slabs;
 * ELSAA_PATH_TC_WIN the sparse forward on the tcgen05 kernel that streams
 * the window in 128-key blocks (d = 128, chunks above or not dividing 128,
 * lookback other than 1, causal, several hash rounds; their backward takes
 * the key-major tcgen05 kernel). */
#define ELSAA_PATH_TC_HASH 1
#define ELSAA_PATH_TC_ATTN 2
#define ELSAA_PATH_SLAB_FWD 4
#define ELSAA_PATH_SLAB_BWD 8
#define ELSAA_PATH_TC_WIN 16
int32_t elsaa_path_flags(const elsaa_params* p);

#ifdef __cplusplus
}
#endif

#endif /* ELSAA_H */
