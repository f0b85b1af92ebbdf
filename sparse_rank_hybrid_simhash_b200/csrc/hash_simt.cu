// SimHash codes on CUDA cores.
//
// "ELSAA: Efficient Low-Rank and Sparse Attention Approximation for Training
// Transformers" (overview) selects the sparse branch by LSH, and the RACE
// branch of "Two Efficient Attentions, One Denominator Problem" buckets
// tokens by hash.  Both use SimHash: bit j of row x is [x . r_j > 0], bit j
// weighs 2^j.  One warp per row; each lane owns one hyperplane of a group of
// 32 and accumulates the dot product in fp64 (products of fp32 / bf16 inputs
// are exact in fp64), so a code differs from an exact evaluation only when a
// projection is within fp64 rounding of zero.  This kernel serves fp32 data
// and head dims the tensor-core hash does not tile.
#include "common.cuh"
#include "internal.h"

namespace elsaa {
namespace {

template <typename T, typename CodeT>
__global__ void __launch_bounds__(256)
hash_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                 const T* __restrict__ r_sort, const T* __restrict__ r_race,
                 int64_t rows_per_tensor, int N, int d, int sort_bits, int L, int kr,
                 uint16_t* __restrict__ code, CodeT* __restrict__ rcode,
                 CodeT* __restrict__ rcode_t) {
  extern __shared__ float smem[];
  const int warps = blockDim.x >> 5;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = sort_bits + L * kr;
  const int nwords = (P + 31) >> 5;
  float* xs = smem + w * d;
  uint32_t* words = reinterpret_cast<uint32_t*>(smem + warps * d) + w * nwords;
  const int64_t total = 2 * rows_per_tensor;
  for (int64_t row = (int64_t)blockIdx.x * warps + w; row < total;
       row += (int64_t)gridDim.x * warps) {
    const T* src = row < rows_per_tensor ? q + row * d : k + (row - rows_per_tensor) * d;
    for (int t = lane; t < d; t += 32) xs[t] = to_f32(src[t]);
    __syncwarp();
    for (int j0 = 0; j0 < P; j0 += 32) {
      const int j = j0 + lane;
      bool bit = false;
      if (j < P) {
        const T* r = j < sort_bits ? r_sort + (size_t)j * d
                                   : r_race + (size_t)(j - sort_bits) * d;
        double acc = 0.0;
        for (int t = 0; t < d; ++t) acc += (double)xs[t] * (double)to_f32(r[t]);
        bit = acc > 0.0;
      }
      const uint32_t m = __ballot_sync(0xffffffffu, bit);
      if (lane == 0) words[j0 >> 5] = m;
    }
    __syncwarp();
    auto field = [&](int start, int n) -> uint32_t {
      uint32_t v = 0;
      for (int b = 0; b < n; ++b) {
        const int p = start + b;
        v |= ((words[p >> 5] >> (p & 31)) & 1u) << b;
      }
      return v;
    };
    if (lane == 0) code[row] = (uint16_t)field(0, sort_bits);
    const int64_t u = row / N;
    CodeT* tdst = rcode_t + (size_t)u * L * N + (row - u * N);
    for (int l = lane; l < L; l += 32) {
      const CodeT c = (CodeT)field(sort_bits + l * kr, kr);
      rcode[row * L + l] = c;
      tdst[(size_t)l * N] = c;
    }
    __syncwarp();
  }
}

template <typename T, typename CodeT>
cudaError_t run(const Geometry& g, const void* q, const void* k, const void* r_sort,
                const void* r_race, uint16_t* code, void* rcode, void* rcode_t, cudaStream_t s) {
  const int threads = 256, warps = threads / 32;
  const int P = g.sort_bits + g.L * g.kr;
  const size_t smem = (size_t)warps * g.d * sizeof(float) + (size_t)warps * ((P + 31) / 32) * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(hash_simt_kernel<T, CodeT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t rows = (int64_t)g.BH * g.N;
  const int64_t blocks = (2 * rows + warps - 1) / warps;
  const int grid = (int)(blocks < 148 * 64 ? blocks : 148 * 64);
  hash_simt_kernel<T, CodeT><<<grid, threads, smem, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(r_sort),
      static_cast<const T*>(r_race), rows, g.N, g.d, g.sort_bits, g.L, g.kr, code,
      static_cast<CodeT*>(rcode), static_cast<CodeT*>(rcode_t));
  return cudaGetLastError();
}

// Sort codes of hash rounds 1 .. R-1 (several Sort-LSH rounds, an extension):
// one warp per Q or K row, lane j of a group of 32 owns projection j of the
// (R - 1) * sort_bits extra hyperplanes (round 1 + j / sort_bits, bit
// j % sort_bits), fp64 sums of exact products as above.  code: [R][2 rows].
template <typename T>
__global__ void __launch_bounds__(256)
hash_sort_rounds_kernel(const T* __restrict__ q, const T* __restrict__ k,
                        const T* __restrict__ r_sort, int64_t rows_per_tensor, int d,
                        int sort_bits, int rounds, uint16_t* __restrict__ code) {
  extern __shared__ float smem[];
  const int warps = blockDim.x >> 5;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = (rounds - 1) * sort_bits;   // <= 7 * 16 = 112: at most four words
  float* xs = smem + w * d;
  const int64_t total = 2 * rows_per_tensor;
  for (int64_t row = (int64_t)blockIdx.x * warps + w; row < total;
       row += (int64_t)gridDim.x * warps) {
    const T* src = row < rows_per_tensor ? q + row * d : k + (row - rows_per_tensor) * d;
    for (int t = lane; t < d; t += 32) xs[t] = to_f32(src[t]);
    __syncwarp();
    uint32_t words[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const int j = wi * 32 + lane;
      bool bit = false;
      if (j < P) {
        const T* r = r_sort + (size_t)(sort_bits + j) * d;   // rounds 1.. follow round 0
        double acc = 0.0;
        for (int t = 0; t < d; ++t) acc += (double)xs[t] * (double)to_f32(r[t]);
        bit = acc > 0.0;
      }
      words[wi] = __ballot_sync(0xffffffffu, bit);
    }
    if (lane < rounds - 1) {
      uint32_t v = 0;
      for (int b = 0; b < sort_bits; ++b) {
        const int p = lane * sort_bits + b;
        v |= ((words[p >> 5] >> (p & 31)) & 1u) << b;
      }
      code[(int64_t)(lane + 1) * total + row] = (uint16_t)v;
    }
    __syncwarp();
  }
}

// rank[seg][perm[seg][x]] = x
__global__ void __launch_bounds__(256)
rank_kernel(const int32_t* __restrict__ perm, int32_t* __restrict__ rank, int64_t total, int N) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t seg = i / N;
    const int p = perm[i];
    if (p >= 0 && p < N) rank[seg * N + p] = (int32_t)(i - seg * N);
  }
}

}  // namespace

cudaError_t launch_hash_sort_rounds(const Geometry& g, const void* q, const void* k,
                                    const void* r_sort, uint16_t* code, cudaStream_t s) {
  if (g.rounds <= 1) return cudaSuccess;
  const int64_t rows = (int64_t)g.BH * g.N;
  if (g.sort_bits == 0)   // zero-bit codes are all 0
    return cudaMemsetAsync(code + 2 * rows, 0, (size_t)(g.rounds - 1) * 2 * rows * 2, s);
  if ((g.rounds - 1) * g.sort_bits > 128) return cudaErrorInvalidValue;
  const int threads = 256, warps = threads / 32;
  const size_t smem = (size_t)warps * g.d * sizeof(float);
  const int64_t blocks = (2 * rows + warps - 1) / warps;
  const int grid = (int)(blocks < 148 * 64 ? blocks : 148 * 64);
  if (g.bf16)
    hash_sort_rounds_kernel<__nv_bfloat16><<<grid, threads, smem, s>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(r_sort), rows, g.d, g.sort_bits, g.rounds, code);
  else
    hash_sort_rounds_kernel<float><<<grid, threads, smem, s>>>(
        static_cast<const float*>(q), static_cast<const float*>(k),
        static_cast<const float*>(r_sort), rows, g.d, g.sort_bits, g.rounds, code);
  return cudaGetLastError();
}

cudaError_t launch_ranks(const Geometry& g, const int32_t* perm, int32_t* rank, int64_t segs,
                         cudaStream_t s) {
  const int64_t total = segs * g.N;
  const int64_t want = (total + 255) / 256;
  rank_kernel<<<(int)(want < 148 * 8 ? want : 148 * 8), 256, 0, s>>>(perm, rank, total, g.N);
  return cudaGetLastError();
}

cudaError_t launch_hash_simt(const Geometry& g, const void* q, const void* k, const void* r_sort,
                             const void* r_race, uint16_t* code, void* rcode, void* rcode_t,
                             cudaStream_t s) {
  if (g.bf16) {
    return g.rcode_bytes == 1
               ? run<__nv_bfloat16, uint8_t>(g, q, k, r_sort, r_race, code, rcode, rcode_t, s)
               : run<__nv_bfloat16, uint16_t>(g, q, k, r_sort, r_race, code, rcode, rcode_t, s);
  }
  return g.rcode_bytes == 1
             ? run<float, uint8_t>(g, q, k, r_sort, r_race, code, rcode, rcode_t, s)
             : run<float, uint16_t>(g, q, k, r_sort, r_race, code, rcode, rcode_t, s);
}

}  // namespace elsaa
