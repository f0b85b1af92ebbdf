// Sort-LSH ordering: a stable LSD radix sort of the sort codes of every
// (tensor, batch, head) segment, ties kept in token order.
//
// The Sort-LSH hybrid of "Two Efficient Attentions, One Denominator Problem"
// (section "The ablation isolates the actual contribution") orders tokens by
// hash code so that a chunk of consecutive sorted tokens holds similar ones.
// Each pass sorts by a digit of at most 8 bits in three launches:
//   1. per-tile digit histograms (tiles of kSortTile keys, shared-memory counts);
//   2. per-segment exclusive scan over (digit, tile), digit-major, so a tile's
//      keys of one digit land after every earlier tile's keys of that digit;
//   3. a stable scatter: warps own consecutive runs of the tile, count their
//      digits, take per-warp bases, then rank equal digits within each
//      32-key round with __match_any_sync.
// Codes of up to 16 bits take two passes (the second reads the first's order).
// Gray order sorts by each code's position in the reflected binary Gray
// sequence (the prefix XOR of its bits from the top), computed where a code is
// read; local order writes token order without sorting.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace elsaa {
namespace {

constexpr int kWarps = kSortThreads / 32;
constexpr int kPerWarp = kSortTile / kWarps;   // 256 keys, 8 rounds of 32

// The sort key of a code: the code itself, or its Gray-sequence position.
ELSAA_DEV int sort_key(uint16_t code, int gray) {
  int b = code;
  if (gray) {
    b ^= b >> 1;
    b ^= b >> 2;
    b ^= b >> 4;
    b ^= b >> 8;
  }
  return b;
}

__global__ void __launch_bounds__(kSortThreads)
sort_hist_kernel(const uint16_t* __restrict__ code, const int32_t* __restrict__ order_in,
                 int N, int shift, int mask, int bins, int tiles, int gray,
                 int32_t* __restrict__ hist) {
  __shared__ int h[256];
  for (int i = threadIdx.x; i < bins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int seg = blockIdx.y, tile = blockIdx.x;
  const uint16_t* c = code + (size_t)seg * N;
  const int32_t* oin = order_in ? order_in + (size_t)seg * N : nullptr;
  const int p0 = tile * kSortTile, p1 = min(N, p0 + kSortTile);
  for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
    const int idx = oin ? oin[p] : p;
    atomicAdd(&h[(sort_key(c[idx], gray) >> shift) & mask], 1);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < bins; b += blockDim.x)
    hist[((size_t)seg * bins + b) * tiles + tile] = h[b];
}

// In-place exclusive scan of n counts per segment (one block per segment).
__global__ void __launch_bounds__(1024) sort_scan_kernel(int32_t* __restrict__ hist, int n) {
  __shared__ int warp_tot[32];
  int32_t* a = hist + (size_t)blockIdx.x * n;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int lo = threadIdx.x * per, hi = min(n, lo + per);
  int local = 0;
  for (int i = lo; i < hi; ++i) local += a[i];
  // block exclusive scan of `local`
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    int v = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
    warp_tot[lane] = v;   // inclusive over warps
  }
  __syncthreads();
  int run = incl - local + (w > 0 ? warp_tot[w - 1] : 0);
  for (int i = lo; i < hi; ++i) {
    const int t = a[i];
    a[i] = run;
    run += t;
  }
}

__global__ void __launch_bounds__(kSortThreads)
sort_scatter_kernel(const uint16_t* __restrict__ code, const int32_t* __restrict__ order_in,
                    int N, int shift, int mask, int bins, int tiles, int gray,
                    const int32_t* __restrict__ offs, int32_t* __restrict__ order_out) {
  __shared__ int cnt[kWarps][256];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = blockIdx.y, tile = blockIdx.x;
  const uint16_t* c = code + (size_t)seg * N;
  const int32_t* oin = order_in ? order_in + (size_t)seg * N : nullptr;
  int32_t* out = order_out + (size_t)seg * N;
  for (int i = threadIdx.x; i < kWarps * 256; i += blockDim.x) (&cnt[0][0])[i] = 0;
  __syncthreads();
  const int base_p = tile * kSortTile + w * kPerWarp;
  const unsigned lt = (1u << lane) - 1u;
  // pass A: digit counts of this warp's run
  for (int r = 0; r < kPerWarp / 32; ++r) {
    const int p = base_p + r * 32 + lane;
    const bool valid = p < N;
    const int idx = valid ? (oin ? oin[p] : p) : 0;
    const int key = valid ? ((sort_key(c[idx], gray) >> shift) & mask) : (bins + lane);
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (valid && lane == __ffs(peers) - 1) cnt[w][key] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per-warp bases: the tile's global offset for the digit plus earlier warps' counts
  for (int b = threadIdx.x; b < bins; b += blockDim.x) {
    int run = offs[((size_t)seg * bins + b) * tiles + tile];
    for (int ww = 0; ww < kWarps; ++ww) {
      const int t = cnt[ww][b];
      cnt[ww][b] = run;
      run += t;
    }
  }
  __syncthreads();
  // pass B: stable ranks inside each round, rounds in token order
  for (int r = 0; r < kPerWarp / 32; ++r) {
    const int p = base_p + r * 32 + lane;
    const bool valid = p < N;
    const int idx = valid ? (oin ? oin[p] : p) : 0;
    const int key = valid ? ((sort_key(c[idx], gray) >> shift) & mask) : (bins + lane);
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    int pos = 0;
    if (valid) pos = cnt[w][key] + __popc(peers & lt);
    __syncwarp();
    if (valid) {
      out[pos] = idx;
      if (lane == __ffs(peers) - 1) cnt[w][key] += __popc(peers);
    }
    __syncwarp();
  }
}

// perm[seg][i] = i: local windows keep token order.
__global__ void __launch_bounds__(256)
token_order_kernel(int64_t total, int N, int32_t* __restrict__ perm) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x)
    perm[i] = (int32_t)(i % N);
}

}  // namespace

cudaError_t launch_sort(const Geometry& g, const uint16_t* code, int32_t* perm, int32_t* hist,
                        int32_t* tmp, cudaStream_t s) {
  const int segs = 2 * g.BH;
  if (g.sort_order == ELSAA_SORT_LOCAL) {
    const int64_t total = (int64_t)segs * g.N;
    const int64_t want = (total + 255) / 256;
    token_order_kernel<<<(int)(want < 148 * 8 ? want : 148 * 8), 256, 0, s>>>(total, g.N, perm);
    return cudaGetLastError();
  }
  const int gray = g.sort_order == ELSAA_SORT_GRAY ? 1 : 0;
  const dim3 grid(g.sort_tiles, segs);
  const int mask = g.sort_bins - 1;
  for (int pass = 0; pass < g.sort_passes; ++pass) {
    const int shift = pass * g.sort_digit_bits;
    const int32_t* in = pass == 0 ? nullptr : tmp;
    int32_t* out = (pass == g.sort_passes - 1) ? perm : tmp;
    sort_hist_kernel<<<grid, kSortThreads, 0, s>>>(code, in, g.N, shift, mask, g.sort_bins,
                                                   g.sort_tiles, gray, hist);
    sort_scan_kernel<<<segs, 1024, 0, s>>>(hist, g.sort_bins * g.sort_tiles);
    sort_scatter_kernel<<<grid, kSortThreads, 0, s>>>(code, in, g.N, shift, mask, g.sort_bins,
                                                      g.sort_tiles, gray, hist, out);
  }
  return cudaGetLastError();
}

}  // namespace elsaa

// ---------------------------------------------------------------------------
// Sort-LSH order without any device allocation (elsaa_sort_codes_noalloc).
//
// Some callers cannot hand the library scratch memory: a serving process whose
// memory pool has already reserved all device memory at start-up, or a host
// framework whose allocator contract forbids cudaMalloc/cudaFree inside a step
// (both synchronise the device).  For them the radix sort's scratch (per-tile
// digit histograms and, for codes of more than 8 bits, the order after the
// first pass) lives in one fixed array in device memory that the library
// itself owns.  Every device that loads the library keeps these bytes until
// the process exits.
// ---------------------------------------------------------------------------

namespace elsaa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
constexpr int kMaxContexts = 64;

__device__ __align__(256) unsigned char g_sort_scratch[kNoAllocScratchBytes];

// Device addresses of g_sort_scratch, one per CUDA context that has called in.
// The address belongs to the module loaded into a context, so the cache is
// keyed on the context's unique ID (cuCtxGetId: never reused within a
// process), not on the device index: after cudaDeviceReset, or when the caller
// makes another context current on the same device, the module is loaded anew
// and the array can sit elsewhere, and that context looks the address up again.
std::mutex g_scratch_mu;
struct ScratchEntry {
  unsigned long long ctx_id;
  void* ptr;
};
ScratchEntry g_scratch[kMaxContexts] = {};
int g_scratch_n = 0;

// cuCtxGetCurrent and cuCtxGetId through the driver entry points the runtime
// resolves (the library makes no direct driver-API calls).
struct CtxFns {
  CUresult (*get_current)(CUcontext*) = nullptr;
  CUresult (*get_id)(CUcontext, unsigned long long*) = nullptr;
};
const CtxFns& ctx_fns() {
  static CtxFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<CUresult (*)(CUcontext*)>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<CUresult (*)(CUcontext, unsigned long long*)>(p);
  });
  return f;
}

// Device address of g_sort_scratch in the current context (the host-side
// symbol is only a stand-in and must never reach a kernel).
cudaError_t scratch_address(void** out) {
  const CtxFns& f = ctx_fns();
  if (!f.get_current || !f.get_id) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  void* ptr = nullptr;
  if (ctx == nullptr) {
    // no context yet: the symbol lookup makes the runtime's primary context current
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_sort_scratch);
    if (e != cudaSuccess) return e;
    if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
  }
  unsigned long long id = 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  for (int i = 0; i < g_scratch_n; ++i)
    if (g_scratch[i].ctx_id == id) {
      *out = g_scratch[i].ptr;
      return cudaSuccess;
    }
  if (ptr == nullptr) {
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_sort_scratch);
    if (e != cudaSuccess) return e;
  }
  if (g_scratch_n < kMaxContexts) g_scratch[g_scratch_n++] = {id, ptr};
  *out = ptr;
  return cudaSuccess;
}

}  // namespace
}  // namespace elsaa

extern "C" elsaa_status elsaa_sort_codes_noalloc(const elsaa_params* p, const uint16_t* code,
                                                 int32_t* perm, void* stream) {
  using namespace elsaa;
  Geometry g;
  elsaa_status why;
  if (!make_geometry(p, &g, &why)) return why;
  if (!code || !perm) return ELSAA_ERR_INVALID_ARG;
  if (((uintptr_t)code % 16) != 0 || ((uintptr_t)perm % 16) != 0) return ELSAA_ERR_INVALID_ARG;
  const size_t hist = align_up((size_t)2 * g.BH * g.sort_bins * g.sort_tiles * 4);
  const size_t tmp = g.sort_passes > 1 ? (size_t)2 * g.BH * g.N * 4 : 0;
  if (hist + tmp > kNoAllocScratchBytes) return ELSAA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return ELSAA_ERR_CUDA;
  char* base = static_cast<char*>(scratch);
  // every histogram slot and the intermediate order are fully written before
  // they are read, so nothing left from an earlier call needs clearing
  if (launch_sort(g, code, perm, reinterpret_cast<int32_t*>(base),
                  reinterpret_cast<int32_t*>(base + hist), (cudaStream_t)stream) != cudaSuccess)
    return ELSAA_ERR_CUDA;
  return ELSAA_OK;
}

