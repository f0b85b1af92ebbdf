// SimHash codes on tcgen05 tensor cores for shapes whose codes do not fill
// whole 32-bit words, or whose word-aligned hyperplanes do not fit shared
// memory (hash_tc.cu covers the rest).  "ELSAA: Efficient Low-Rank and Sparse
// Attention Approximation for Training Transformers" (overview) selects the
// sparse branch by LSH; the RACE branch ("Two Efficient Attentions, One
// Denominator Problem") buckets tokens by hash.  Bit j of a code is
// [x . r_j > 0] with weight 2^j; a row's P = sort_bits + L race_bits
// projections are one GEMM row against hyperplanes packed column after column.
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

// Shapes the word-aligned layout does not fit (its padded hyperplanes above
// shared memory, codes not filling whole words, tiles straddling units) take
// the bit-stream variant below: P = sort_bits + L race_bits packed columns.
// Every row's P sign bits are staged as a bit array of SW words, and each code
// is cut out of it where it is written.
constexpr int kStreamThreads = 512;    // 8 reader warps, then 8 writer warps
constexpr int kReaders = 256;
constexpr int kReaderWarps = kReaders / 32;
constexpr uint32_t kStreamTmemCols = 256;   // two 128-column pass buffers
// named barriers (0 is __syncthreads): the readers' own, then per bit array
// "full" (readers arrive, writers wait) and "empty" (writers arrive, readers wait)
constexpr int kBarRead = 1, kBarFull = 2, kBarEmpty = 4;

ELSAA_DEV void nbar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
ELSAA_DEV void nbar_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

struct StreamShape {
  int P, gcol, P16, SW, nbuf;
  uint32_t r_bytes, a_bytes, code_bytes, dyn;
};

// With learned gates, four more columns (w_s and w_r, each as a bf16 high
// part and the bf16 remainder: their fp32 sums are w . q to about 16
// significant bits) start at the first 32-column word after the codes, gcol.
StreamShape stream_shape(const Geometry& g, bool gates) {
  StreamShape h;
  h.P = g.sort_bits + g.L * g.kr;
  h.gcol = gates ? (h.P + 31) / 32 * 32 : -1;
  h.P16 = ((gates ? h.gcol + 4 : h.P) + 15) / 16 * 16;
  // words of 32 sign bits per row (whole 32-column reads) plus one zero word,
  // so every code's two-word window exists; odd, so rows fall on distinct banks
  h.SW = ((h.P16 + 31) / 32 + 1) | 1;
  h.r_bytes = (uint32_t)h.P16 * g.d * 2;
  h.a_bytes = (uint32_t)kTile * g.d * 2;
  h.code_bytes = (uint32_t)((2 * kTile * h.SW * 4 + 15) / 16 * 16);   // two tiles' bit arrays
  h.nbuf = (h.r_bytes + 2 * h.a_bytes + h.code_bytes + 64 <= (uint32_t)kSmemLimit) ? 2 : 1;
  h.dyn = h.r_bytes + h.nbuf * h.a_bytes + h.code_bytes + 64;
  return h;
}

// Roles: warps 0..7 read, warps 8..15 write.  Per tile the readers run the
// passes, whose MMAs alternate between two TMEM buffers (pass p + 1 computes
// while pass p is read); reader warp w reads lane quarter w % 4, 32-column
// words w / 4 and w / 4 + 2 of every pass, and stores each row's sign masks
// into one of two bit arrays; once the tile's last MMA has completed, the
// next tile's load starts (one A buffer).  Meanwhile the writers cut the
// previous tile's codes from the other bit array, twice: warps over rows for
// the row-major codes, warps over tables for the table-major ones, so both
// global writes are coalesced.  Named barriers hand each bit array from the
// readers to the writers ("full") and back ("empty").
template <int D, typename CodeT>
__global__ void __launch_bounds__(kStreamThreads, 1)
hash_tc_stream_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
               const __nv_bfloat16* __restrict__ r_sort, const __nv_bfloat16* __restrict__ r_race,
               int64_t rows_per_tensor, int N, int sort_bits, int L, int kr, int P, int gcol,
               int P16, int SW, int nbuf, uint16_t* __restrict__ code, CodeT* __restrict__ rcode,
               CodeT* __restrict__ rcode_t, const float* __restrict__ gate_w,
               float2* __restrict__ gl, uint32_t* __restrict__ err) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t r_bytes = (uint32_t)P16 * D * 2;
  const uint32_t a_bytes = kTile * D * 2;
  const uint32_t s_r = sbase, s_a = sbase + r_bytes;
  // two tiles' sign bits: [2][128 rows][SW words]
  uint32_t* st_w = reinterpret_cast<uint32_t*>(smem + r_bytes + nbuf * a_bytes);
  const uint32_t code_bytes = (uint32_t)((2 * kTile * SW * 4 + 15) / 16 * 16);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + r_bytes + nbuf * a_bytes + code_bytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((sbase & 1023u) != 0) {   // the swizzled tiles need a 1024-byte aligned base
    if (tid == 0) raise_error(err, ERR_CHECK);
    return;
  }
  const int64_t total = 2 * rows_per_tensor;
  const int64_t tiles = (total + kTile - 1) / kTile;
  if ((int64_t)blockIdx.x >= tiles) return;

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kStreamTmemCols);
    tmem_relinquish();
  }
  // resident hyperplanes: rows [0, sort_bits) from r_sort, then L*kr from r_race, zero padding
  {
    constexpr int kChunks = D / 8;
    for (int i = tid; i < P16 * kChunks; i += kStreamThreads) {
      const int j = i / kChunks, ch = i % kChunks;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (j < sort_bits) {
        val = *reinterpret_cast<const uint4*>(r_sort + (size_t)j * D + ch * 8);
      } else if (j < P) {
        val = *reinterpret_cast<const uint4*>(r_race + (size_t)(j - sort_bits) * D + ch * 8);
      } else if (gcol >= 0 && j >= gcol && j < gcol + 4) {
        // gate columns: w_s hi, w_s lo, w_r hi, w_r lo
        const int gc = j - gcol;
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
  // words no pass writes stay zero (the window of the last code reads one)
  for (int i = tid; i < 2 * kTile * SW; i += kStreamThreads) st_w[i] = 0u;
  // s_abort: a reader's wait gave up (read by the readers after their own
  // barrier); s_done[b]: the readers' outcome for the tile of bit array b,
  // written before they arrive on its "full" barrier, so every writer reads
  // the same value
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_done = s_abort + 1;
  if (tid == 0) *s_abort = 0;
  if (tid < kReaders) {
    load_tile<D, kReaders>(s_a, q, k, rows_per_tensor, blockIdx.x);
    cp_async_commit();
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const int npass = (P16 + kPass - 1) / kPass;
  // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int n_my = (int)((tiles - blockIdx.x + gridDim.x - 1) / gridDim.x);
  if (warp < kReaderWarps) {
    // ------------------------------------------------------------ readers
    // warp w reads lane quarter w % 4, words w / 4 and w / 4 + 2 of every pass
    const int quarter = warp & 3, wsel = warp >> 2;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int srow = quarter * 32 + lane;   // the row this thread reads out
    uint32_t ph = 0u;   // bit b: the phase parity of mbarrier b
    auto issue = [&](int p, uint32_t abuf) {   // one thread: pass p into TMEM buffer p & 1
      fence_after();
      const int ncol = min(kPass, P16 - p * kPass);
      const uint32_t idesc = idesc_bf16(128, ncol, false, false);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const uint32_t koff = (s >> 2) * (kTile * 128) + (s & 3) * 32;
        const uint32_t roff = (s >> 2) * (P16 * 128) + p * kPass * 128 + (s & 3) * 32;
        mma_bf16_ss(tmem + (uint32_t)(p & 1) * kPass, sw128_desc(s_a + abuf + koff, 16, 1024),
                    sw128_desc(s_r + roff, 16, 1024), idesc, s > 0);
      }
      mma_commit(bar + (p & 1));
    };
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++it) {
      const int sb = it & 1;
      uint32_t* bits = st_w + sb * kTile * SW;
      const uint32_t abuf = nbuf == 2 ? (uint32_t)sb * a_bytes : 0u;
      const int64_t next = tile + gridDim.x;
      // the writers are done with this bit array (tile it - 2)
      if (it >= 2) nbar_sync(kBarEmpty + sb, kStreamThreads);
      if (nbuf == 2 && next < tiles) {
        load_tile<D, kReaders>(s_a + (a_bytes - abuf), q, k, rows_per_tensor, next);
        cp_async_commit();
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        cp_async_wait_all();
      }
      fence_async_smem();
      nbar_sync(kBarRead, kReaders);
      if (tid == 0) issue(0, abuf);
      bool ok = true;
      for (int p = 0; p < npass; ++p) {
        // pass p + 1 goes into the other TMEM buffer, whose last read-out
        // ended before the barrier that closed the previous pass
        if (tid == 0 && p + 1 < npass) issue(p + 1, abuf);
        const int b = p & 1;
        // every reader waits for the pass itself (no block barrier before the
        // read-out; the outcome is uniform over the warp, as tcgen05.ld needs);
        // a give-up is shared at the barrier after it
        const bool wok = __all_sync(0xffffffffu, mbar_wait(bar + b, (ph >> b) & 1u, err));
        ph ^= 1u << b;
        if (!wok) *s_abort = 1;
        fence_after();
        if (wok && p + 1 == npass && nbuf == 1 && next < tiles) {
          // every MMA of the tile has completed: its A buffer takes the next tile
          load_tile<D, kReaders>(s_a, q, k, rows_per_tensor, next);
          cp_async_commit();
        }
#pragma unroll
        for (int h = 0; h < 2 && wok; ++h) {
          const int wd = wsel + 2 * h;
          const int c0 = p * kPass + wd * 32;
          if (c0 < P16) {   // uniform over the warp
            float v[32];
            tmem_ld32(tmem + lane_off + (uint32_t)b * kPass + wd * 32, v);
            tmem_ld_wait();
            const int valid = min(32, P - c0);
            uint32_t m4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int i = 0; i < 32; ++i) m4[i & 3] |= (v[i] > 0.f ? 1u : 0u) << i;
            uint32_t m = (m4[0] | m4[1]) | (m4[2] | m4[3]);
            if (valid <= 0) m = 0u;
            else if (valid < 32) m &= (1u << valid) - 1u;
            bits[srow * SW + (c0 >> 5)] = m;
            if (c0 == gcol) {   // a query row's gate logits
              const int64_t grow = tile * kTile + srow;
              if (grow < rows_per_tensor) gl[grow] = make_float2(v[0] + v[1], v[2] + v[3]);
            }
          }
        }
        fence_before();
        nbar_sync(kBarRead, kReaders);   // the buffer's read-out is done: pass p + 2 may reuse it
        if (*s_abort) {   // every reader sees the same flag after the barrier
          ok = false;
          break;
        }
      }
      // this tile's bits (or the abort) go to the writers
      if (tid == 0) s_done[sb] = ok ? 1 : 0;
      nbar_arrive(kBarFull + sb, kStreamThreads);
      if (!ok) {
        // take the writers' release of the other bit array (tile it - 1), so
        // that no barrier is left half-arrived
        if (it >= 1 && it + 1 < n_my) nbar_sync(kBarEmpty + (sb ^ 1), kStreamThreads);
        break;
      }
    }
  } else {
    // ------------------------------------------------------------ writers
    // codes cut from the bit array of the previous tile while the readers
    // run the next one: warps over rows for the row-major codes, warps over
    // tables for the table-major ones, so both global writes are coalesced
    const int ww = warp - kReaderWarps, wt = tid - kReaders;
    constexpr int kWriterWarps = (kStreamThreads - kReaders) / 32;
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++it) {
      const int sb = it & 1;
      const uint32_t* bits = st_w + sb * kTile * SW;
      nbar_sync(kBarFull + sb, kStreamThreads);
      if (s_done[sb] == 0) break;   // the readers gave up on this tile
      // bits [o, o + n) of row r, n <= 16
      auto cut = [&](int r, int o, int n) -> uint32_t {
        const uint32_t* row = bits + r * SW + (o >> 5);
        return __funnelshift_r(row[0], row[1], o & 31) & ((1u << n) - 1u);
      };
      const int64_t row0 = tile * kTile;
      const int nrows = (int)min((int64_t)kTile, total - row0);
      for (int r = wt; r < nrows; r += kStreamThreads - kReaders)
        code[row0 + r] = (uint16_t)cut(r, 0, sort_bits);
      for (int r = ww; r < nrows; r += kWriterWarps) {
        CodeT* dst = rcode + (row0 + r) * L;
        for (int t = lane; t < L; t += 32) dst[t] = (CodeT)cut(r, sort_bits + t * kr, kr);
      }
      // unit and position of each of the lane's rows (the tile's rows are
      // consecutive; consecutive rows of a unit are consecutive along N)
      int64_t off[kTile / 32];
#pragma unroll
      for (int j = 0; j < kTile / 32; ++j) {
        const int64_t gr = row0 + lane + 32 * j;
        const int64_t u = gr / N;
        off[j] = u * L * N + (gr - u * N);
      }
      for (int t = ww; t < L; t += kWriterWarps) {
#pragma unroll
        for (int j = 0; j < kTile / 32; ++j) {
          const int r = lane + 32 * j;
          if (r < nrows) rcode_t[off[j] + (int64_t)t * N] = (CodeT)cut(r, sort_bits + t * kr, kr);
        }
      }
      // the readers may overwrite this bit array for tile it + 2 (no arrival
      // when there is no such tile, so no barrier is left half-arrived)
      if (it + 2 < n_my) nbar_arrive(kBarEmpty + sb, kStreamThreads);
    }
  }
  cp_async_wait_all();
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    tmem_dealloc(tmem, kStreamTmemCols);
  }
}

template <int D, typename CodeT>
cudaError_t run_stream(const Geometry& g, const void* q, const void* k, const void* r_sort,
                       const void* r_race, uint16_t* code, void* rcode, void* rcode_t,
                       const float* gate_w, float2* gl, uint32_t* err, cudaStream_t s) {
  const StreamShape h = stream_shape(g, gl != nullptr);
  cudaError_t e = cudaFuncSetAttribute(hash_tc_stream_kernel<D, CodeT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)h.dyn);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(hash_tc_stream_kernel<D, CodeT>,
                           cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // CTAs per SM: shared memory (228 KB per SM, 1 KB reserved per CTA), TMEM
  // (2 x 256 columns) and threads (4 x 512)
  int per_sm = (int)((228u * 1024u) / (h.dyn + 1024u));
  per_sm = per_sm < 1 ? 1 : (per_sm > 2 ? 2 : per_sm);
  const int64_t rows = (int64_t)g.BH * g.N;
  const int64_t tiles = (2 * rows + kTile - 1) / kTile;
  const int64_t want = (int64_t)sms * per_sm;
  const int grid = (int)(tiles < want ? tiles : want);
  hash_tc_stream_kernel<D, CodeT><<<grid, kStreamThreads, h.dyn, s>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(r_sort), static_cast<const __nv_bfloat16*>(r_race), rows,
      g.N, g.sort_bits, g.L, g.kr, h.P, h.gcol, h.P16, h.SW, h.nbuf, code,
      static_cast<CodeT*>(rcode), static_cast<CodeT*>(rcode_t), gate_w, gl, err);
  return cudaGetLastError();
}

}  // namespace

bool hash_tc_stream_fits(const Geometry& g, bool gates) {
  if (!g.bf16 || (g.d != 64 && g.d != 128) || g.sort_bits > 16 || g.kr > 16) return false;
  const StreamShape h = stream_shape(g, gates);
  return h.P > 0 && h.dyn <= (uint32_t)kSmemLimit;
}

cudaError_t launch_hash_tc_stream(const Geometry& g, const void* q, const void* k,
                                  const void* r_sort, const void* r_race, uint16_t* code,
                                  void* rcode, void* rcode_t, const float* gate_w, float2* gl,
                                  uint32_t* err, cudaStream_t s) {
  if (!hash_tc_stream_fits(g, gl != nullptr)) return cudaErrorInvalidValue;
#define ELSAA_HASH_STREAM(DD, CT) \
  run_stream<DD, CT>(g, q, k, r_sort, r_race, code, rcode, rcode_t, gate_w, gl, err, s)
  if (g.d == 64)
    return g.rcode_bytes == 1 ? ELSAA_HASH_STREAM(64, uint8_t) : ELSAA_HASH_STREAM(64, uint16_t);
  return g.rcode_bytes == 1 ? ELSAA_HASH_STREAM(128, uint8_t) : ELSAA_HASH_STREAM(128, uint16_t);
#undef ELSAA_HASH_STREAM
}

}  // namespace elsaa
