// SimHash codes on tcgen05 tensor cores (bf16 data, d in {64, 128}).
//
// "ELSAA: Efficient Low-Rank and Sparse Attention Approximation for Training
// Transformers" (overview) selects the sparse branch by LSH; the RACE branch
// ("Two Efficient Attentions, One Denominator Problem") buckets tokens by hash.
// Bit j of a row x is [x . r_j > 0] with weight 2^j inside its code.  For one
// row that is a product with every hyperplane: a GEMM of (2 B H N) x d by d x P.
//
// Products of bf16 values are exact in fp32, so a code can differ from an
// exact evaluation only where a projection lies within fp32 accumulation
// error of zero.
//
// Column layout: RACE code t takes the cw columns [t cw, (t + 1) cw), cw = 8
// for byte codes and 16 for 16-bit codes, its bit b in column t cw + b (zero
// hyperplanes pad bits b >= race_bits, and a zero projection gives bit 0); the
// sort code takes the 16 columns after them.  Every 32 columns are then one
// 32-bit word of finished codes: the sign mask of 32 projections is stored as
// is, with no bit stream to assemble.
//
// Learned gates (ELSAA overview: token-wise gates g = sigmoid(w . q_i + b))
// need w_s . q_i and w_r . q_i for every query row; they ride along as four
// more columns after the sort code: w_s and w_r each split into a bf16 high
// part and the bf16 remainder (w - hi), so the two columns' fp32 sum carries
// w to about 16 significant bits and the products stay exact in fp32.  The
// read-out writes (w_s . q_i, w_r . q_i) for the query rows.
//
// Several Sort-LSH hash rounds (an extension): rounds 1 .. R - 1's sort codes
// take 16 more columns each after that word (two rounds per 32-bit word), so
// the one GEMM gives every round's codes.
//
// Persistent CTAs of 128 threads.  The hyperplanes stay resident in shared
// memory; 128-row tiles of Q then K stream in by cp.async (double-buffered
// where that costs no CTA per SM: at text-32k sizes four single-buffered CTAs
// per SM beat three double-buffered ones).  Per tile the columns go through TMEM in passes
// of 128: thread t reads the 32 projections of row t per tcgen05.ld and keeps
// the sign mask.  The tile's codes leave as one contiguous row-major block and,
// through a 4 x 4 (or 2 x 2) byte transpose across lanes, as 4-byte runs of
// each table's table-major codes.  Shapes this word-aligned layout does not
// fit take the bit-stream variant (hash_tc_stream.cu).
#include "hash_tile.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace elsaa {
namespace {

using namespace tc;
using hash::kTile;
using hash::kPass;
using hash::kSmemLimit;
using hash::load_tile;

constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 128;

struct HashShape {
  int P16;       // columns: 32 Wr RACE columns, 16 sort columns (+ 16 with gate columns)
  int cw, Wr;    // bits per RACE code; 32-bit words of RACE codes per row
  int S;         // staging stride in words (odd: conflict-free)
  int nbuf;
  uint32_t r_bytes, a_bytes, code_bytes, dyn;
};

HashShape hash_shape(const Geometry& g, bool gates, int rounds) {
  HashShape h;
  h.cw = 8 * g.rcode_bytes;
  h.Wr = g.L * h.cw / 32;
  h.P16 = 32 * h.Wr + (gates ? 32 : 16);
  if (rounds > 1) h.P16 = 32 * h.Wr + 32 + 16 * (rounds - 1);
  h.S = h.Wr | 1;
  h.r_bytes = (uint32_t)h.P16 * g.d * 2;
  h.a_bytes = (uint32_t)kTile * g.d * 2;
  // per-tile staging: 128 rows of RACE code words, then 128 sort codes (u16)
  h.code_bytes = (uint32_t)((kTile * h.S * 4 + kTile * 2 + 15) / 16 * 16);
  // two A buffers overlap a tile's load with the previous tile's passes; one
  // buffer wins where it lets one more CTA onto each SM (measured: 4 CTAs with
  // one buffer beat 3 with two at text-32k sizes)
  const uint32_t dyn1 = h.r_bytes + h.a_bytes + h.code_bytes + 64;
  const uint32_t dyn2 = dyn1 + h.a_bytes;
  auto per_sm = [](uint32_t dyn) {
    const int n = (int)((228u * 1024u) / (dyn + 1024u));
    return n > 4 ? 4 : n;
  };
  h.nbuf = (dyn2 <= (uint32_t)kSmemLimit && per_sm(dyn2) >= per_sm(dyn1)) ? 2 : 1;
  h.dyn = h.nbuf == 2 ? dyn2 : dyn1;
  return h;
}

template <int D, typename CodeT>
__global__ void __launch_bounds__(kThreads)
hash_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
               const __nv_bfloat16* __restrict__ r_sort, const __nv_bfloat16* __restrict__ r_race,
               int64_t rows_per_tensor, int N, int sort_bits, int L, int kr, int cw, int Wr, int S,
               int P16, int nbuf, int rounds, uint16_t* __restrict__ code,
               CodeT* __restrict__ rcode,
               CodeT* __restrict__ rcode_t, const float* __restrict__ gate_w,
               float2* __restrict__ gl, uint32_t* __restrict__ err) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t r_bytes = (uint32_t)P16 * D * 2;
  const uint32_t a_bytes = kTile * D * 2;
  const uint32_t s_r = sbase, s_a = sbase + r_bytes;
  // code staging: [128 rows][S words] of RACE codes, then 128 sort codes
  uint32_t* st_w = reinterpret_cast<uint32_t*>(smem + r_bytes + nbuf * a_bytes);
  uint16_t* st_code = reinterpret_cast<uint16_t*>(st_w + kTile * S);
  const uint32_t code_bytes = (uint32_t)((kTile * S * 4 + kTile * 2 + 15) / 16 * 16);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + r_bytes + nbuf * a_bytes + code_bytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((sbase & 1023u) != 0) {   // the swizzled tiles need a 1024-byte aligned base
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  const int64_t tiles = (2 * rows_per_tensor + kTile - 1) / kTile;
  if ((int64_t)blockIdx.x >= tiles) return;

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // resident hyperplanes in the column layout above; zero rows pad
  {
    constexpr int kChunks = D / 8;
    const int race_cols = 32 * Wr;
    for (int i = tid; i < P16 * kChunks; i += kThreads) {
      const int j = i / kChunks, ch = i % kChunks;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (j < race_cols) {
        const int t = j / cw, b = j - t * cw;
        if (b < kr) val = *reinterpret_cast<const uint4*>(r_race + (size_t)(t * kr + b) * D + ch * 8);
      } else if (j - race_cols < sort_bits) {
        val = *reinterpret_cast<const uint4*>(r_sort + (size_t)(j - race_cols) * D + ch * 8);
      } else if (j - race_cols >= 32) {
        // rounds 1 .. R - 1: 16 columns each
        const int x = j - race_cols - 32, t = 1 + x / 16, b = x % 16;
        if (t < rounds && b < sort_bits)
          val = *reinterpret_cast<const uint4*>(r_sort + ((size_t)t * sort_bits + b) * D +
                                                ch * 8);
      } else if (gl != nullptr && j - race_cols >= 16 && j - race_cols < 20) {
        // gate columns: w_s hi, w_s lo, w_r hi, w_r lo
        const int gc = j - race_cols - 16;
        const float* wrow = gate_w + (size_t)(gc >> 1) * D + ch * 8;
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          float x[2] = {wrow[e], wrow[e + 1]};
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const float hi = __bfloat162float(__float2bfloat16_rn(x[m]));
            x[m] = (gc & 1) ? x[m] - hi : hi;
          }
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(x[0], x[1]);
          pk[e >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        val = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      *reinterpret_cast<uint4*>(smem + (ch >> 3) * (P16 * 128) + sw128_off(j, ch & 7)) = val;
    }
  }
  load_tile<D, kThreads>(s_a, q, k, rows_per_tensor, blockIdx.x);
  cp_async_commit();
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const int npass = (P16 + kPass - 1) / kPass;
  uint32_t phase = 0;
  bool ok = true;
  int it = 0;
  for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++it) {
    const uint32_t buf = nbuf == 2 ? (uint32_t)(it & 1) : 0u;
    const int64_t next = tile + gridDim.x;
    if (nbuf == 2 && next < tiles) {
      load_tile<D, kThreads>(s_a + (buf ^ 1u) * a_bytes, q, k, rows_per_tensor, next);
      cp_async_commit();
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      cp_async_wait_all();
    }
    fence_async_smem();
    __syncthreads();
    for (int p = 0; p < npass; ++p) {
      const int ncol = min(kPass, P16 - p * kPass);
      if (tid == 0) {
        fence_after();
        const uint32_t idesc = idesc_bf16(128, ncol, false, false);
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const uint32_t koff = (s >> 2) * (kTile * 128) + (s & 3) * 32;
          const uint32_t roff = (s >> 2) * (P16 * 128) + p * kPass * 128 + (s & 3) * 32;
          mma_bf16_ss(tmem, sw128_desc(s_a + buf * a_bytes + koff, 16, 1024),
                      sw128_desc(s_r + roff, 16, 1024), idesc, s > 0);
        }
        mma_commit(bar);
      }
      ok = mbar_wait(bar, phase & 1, err);
      ++phase;
      if (__syncthreads_or(!ok)) {  // every thread leaves with ok false
        ok = false;
        break;
      }
      fence_after();
      for (int c0 = 0; c0 < ncol; c0 += 32) {
        const int w = (p * kPass + c0) >> 5;
        float v[32];
        tmem_ld32(tmem + lane_off + c0, v);
        tmem_ld_wait();
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) m |= (uint32_t)(__float_as_int(v[i]) > 0) << i;
        if (w < Wr) st_w[tid * S + w] = m;
        else if (w > Wr) {   // rounds 2 (w - Wr) - 1 and 2 (w - Wr)
          const int t = 2 * (w - Wr) - 1;
          const int64_t grow = tile * kTile + tid;
          code[(size_t)t * 2 * rows_per_tensor + grow] = (uint16_t)(m & 0xFFFFu);
          if (t + 1 < rounds)
            code[(size_t)(t + 1) * 2 * rows_per_tensor + grow] = (uint16_t)(m >> 16);
        } else if (w == Wr) {
          st_code[tid] = (uint16_t)(m & 0xFFFFu);
          const int64_t grow = tile * kTile + tid;
          if (gl != nullptr && grow < rows_per_tensor)   // a query row: its gate logits
            gl[grow] = make_float2(v[16] + v[17], v[18] + v[19]);
        }
      }
      fence_before();
      __syncthreads();
    }
    if (!ok) break;
    {
      const int64_t row0 = tile * kTile;   // the tile's rows lie in one unit (N % 128 = 0)
      // row-major: the tile's codes are one contiguous block of 128 Wr words
      uint32_t* gw = reinterpret_cast<uint32_t*>(rcode) + row0 * Wr;
      for (int g = tid; g < kTile * Wr; g += kThreads) {
        const int r = g / Wr, w = g - r * Wr;
        gw[g] = st_w[r * S + w];
      }
      code[row0 + tid] = st_code[tid];
      // table-major: lanes 4i .. 4i + 3 (rows 4i .. 4i + 3 of the warp) trade
      // bytes so that lane 4i + j holds table 4w + j of the four rows (16-bit
      // codes: lane pairs, table 2w + j of two rows); one 4-byte store each
      const int64_t u = row0 / N;
      const int n0 = (int)(row0 - u * N) + tid;
      uint8_t* tbase = reinterpret_cast<uint8_t*>(rcode_t) + (size_t)u * L * N * sizeof(CodeT);
      for (int w = 0; w < Wr; ++w) {
        const uint32_t mine = st_w[tid * S + w];
        if (sizeof(CodeT) == 1) {
          const int j = lane & 3, b0 = lane & ~3;
          const uint32_t v0 = __shfl_sync(0xffffffffu, mine, b0);
          const uint32_t v1 = __shfl_sync(0xffffffffu, mine, b0 + 1);
          const uint32_t v2 = __shfl_sync(0xffffffffu, mine, b0 + 2);
          const uint32_t v3 = __shfl_sync(0xffffffffu, mine, b0 + 3);
          const uint32_t sel = (uint32_t)j | ((uint32_t)(j + 4) << 4);
          const uint32_t out = __byte_perm(__byte_perm(v0, v1, sel), __byte_perm(v2, v3, sel), 0x5410);
          const int t = 4 * w + j;
          *reinterpret_cast<uint32_t*>(tbase + (size_t)t * N + (n0 - j)) = out;
        } else {
          const int j = lane & 1, b0 = lane & ~1;
          const uint32_t v0 = __shfl_sync(0xffffffffu, mine, b0);
          const uint32_t v1 = __shfl_sync(0xffffffffu, mine, b0 + 1);
          const uint32_t out = __byte_perm(v0, v1, j ? 0x7632 : 0x5410);
          const int t = 2 * w + j;
          *reinterpret_cast<uint32_t*>(tbase + ((size_t)t * N + (n0 - j)) * 2) = out;
        }
      }
    }
    if (nbuf == 1 && next < tiles) {
      load_tile<D, kThreads>(s_a, q, k, rows_per_tensor, next);
      cp_async_commit();
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

template <int D, typename CodeT>
cudaError_t run(const Geometry& g, const void* q, const void* k, const void* r_sort,
                const void* r_race, uint16_t* code, void* rcode, void* rcode_t,
                const float* gate_w, float2* gl, int rounds, uint32_t* err, cudaStream_t s) {
  const HashShape h = hash_shape(g, gl != nullptr, rounds);
  cudaError_t e = cudaFuncSetAttribute(hash_tc_kernel<D, CodeT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)h.dyn);
  if (e != cudaSuccess) return e;
  // let shared memory take the whole carveout so several CTAs fit per SM
  e = cudaFuncSetAttribute(hash_tc_kernel<D, CodeT>,
                           cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // CTAs per SM: shared memory (228 KB per SM, 1 KB reserved per CTA) and
  // TMEM (4 x 128 columns)
  int per_sm = (int)((228u * 1024u) / (h.dyn + 1024u));
  per_sm = per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm);
  const int64_t rows = (int64_t)g.BH * g.N;
  const int64_t tiles = (2 * rows + kTile - 1) / kTile;
  const int64_t want = (int64_t)sms * per_sm;
  const int grid = (int)(tiles < want ? tiles : want);
  hash_tc_kernel<D, CodeT><<<grid, kThreads, h.dyn, s>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(r_sort), static_cast<const __nv_bfloat16*>(r_race), rows,
      g.N, g.sort_bits, g.L, g.kr, h.cw, h.Wr, h.S, h.P16, h.nbuf, rounds, code,
      static_cast<CodeT*>(rcode), static_cast<CodeT*>(rcode_t), gate_w, gl, err);
  return cudaGetLastError();
}

bool aligned_layout_fits(const Geometry& g, bool gates, int rounds = 1) {
  // codes fill whole 32-bit words per row; 128-row tiles never straddle units
  if ((g.L * g.rcode_bytes) % 4 != 0 || g.N % kTile != 0 || g.sort_bits > 16) return false;
  return hash_shape(g, gates, rounds).dyn <= (uint32_t)kSmemLimit;
}

}  // namespace

bool hash_tc_gate_logits_supported(const Geometry& g) {
  return g.bf16 && (g.d == 64 || g.d == 128) &&
         (aligned_layout_fits(g, true) || hash_tc_stream_fits(g, true));
}

bool hash_tc_supported(const Geometry& g) {
  if (!g.bf16 || (g.d != 64 && g.d != 128)) return false;
  return aligned_layout_fits(g, false) || hash_tc_stream_fits(g, false);
}

bool hash_tc_rounds_supported(const Geometry& g, bool gates) {
  return g.rounds > 1 && hash_tc_supported(g) && aligned_layout_fits(g, gates, g.rounds);
}

cudaError_t launch_hash_tc(const Geometry& g, const void* q, const void* k, const void* r_sort,
                           const void* r_race, uint16_t* code, void* rcode, void* rcode_t,
                           const float* gate_w, float2* gl, int rounds, uint32_t* err,
                           cudaStream_t s) {
  if (gl != nullptr && !hash_tc_gate_logits_supported(g)) return cudaErrorInvalidValue;
  if (rounds > 1 && !aligned_layout_fits(g, gl != nullptr, rounds)) return cudaErrorInvalidValue;
  // the word-aligned layout first (measured faster where both fit: text-32k
  // 0.18 against 0.40 ms), the bit stream for the other shapes
  const bool al = aligned_layout_fits(g, gl != nullptr, rounds);
#define ELSAA_HASH(DD, CT)                                                                    \
  (al ? run<DD, CT>(g, q, k, r_sort, r_race, code, rcode, rcode_t, gate_w, gl, rounds, err, s) \
      : launch_hash_tc_stream(g, q, k, r_sort, r_race, code, rcode, rcode_t, gate_w, gl, err, s))
  if (g.d == 64) return g.rcode_bytes == 1 ? ELSAA_HASH(64, uint8_t) : ELSAA_HASH(64, uint16_t);
  return g.rcode_bytes == 1 ? ELSAA_HASH(128, uint8_t) : ELSAA_HASH(128, uint16_t);
#undef ELSAA_HASH
}

}  // namespace elsaa
