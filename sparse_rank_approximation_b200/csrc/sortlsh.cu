// sortLSH selector (ELSAA paper §3.2), non-causal: queries and keys are hashed with
// angular LSH, sorted by hash value and grouped into equal-size blocks; query block t
// attends exactly key block t.  Rows carry a b-bit code (bit c set when x . R_c > 0),
// are ordered by the position of the code in the reflected Gray sequence (neighbouring
// buckets differ in one bit) and then by row index.
//
// Non-causal RACE, the fusion and diagonal-block attention all commute with row
// permutations, so the selector runs the rest of the operator on row-permuted copies
// (queries by the query order, keys and values by the key order) with tile t selecting
// block t, and scatters the outputs back.  This file holds the hashing and sorting,
// the row gather / scatter and the diagonal selection.
#include "common.cuh"
#include "kernels.h"

namespace elsaa {

namespace {

constexpr int kSortThreads = 1024;

__device__ __forceinline__ uint32_t gray_position(uint32_t code) {
  uint32_t n = code;
  for (uint32_t s = code >> 1; s; s >>= 1) n ^= s;
  return n;
}

template <typename E>
__device__ __forceinline__ float to_f(E x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

}  // namespace

// grid (BH, 2: queries then keys), block 1024.  Shared memory: the planes [bits][d]
// (fp32) and one 64-bit key (Gray position << 32 | row) per row, padded to a power of
// two; a bitonic network sorts the keys, which are unique, so the order is stable.
template <typename E>
__global__ void __launch_bounds__(kSortThreads) sortlsh_order_kernel(const E* __restrict__ Q,
                                                                     const E* __restrict__ K,
                                                                     const float* __restrict__ planes, int bits,
                                                                     int npow2, int* __restrict__ order,
                                                                     int* __restrict__ codes, Geom g) {
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem);
  float* sR = reinterpret_cast<float*>(keys + npow2);          // [bits][d]
  const int side = blockIdx.y, bh = blockIdx.x;
  const E* X = (side == 0 ? Q : K) + (size_t)bh * g.N * g.d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < bits * g.d; i += kSortThreads) {
    const int c = i / g.d, k = i % g.d;
    sR[i] = planes[(size_t)k * bits + c];                        // planes are [d][bits]
  }
  __syncthreads();
  // one warp per row: lanes split the row, then reduce each plane's projection
  for (int row = warp; row < g.N; row += kSortThreads / 32) {
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = lane + 32 * e;
      x[e] = k < g.d ? to_f<E>(X[(size_t)row * g.d + k]) : 0.f;
    }
    uint32_t code = 0;
    for (int c = 0; c < bits; ++c) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = lane + 32 * e;
        if (k < g.d) s = fmaf(x[e], sR[c * g.d + k], s);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      code |= (s > 0.f ? 1u : 0u) << c;
    }
    if (lane == 0) {
      keys[row] = ((unsigned long long)gray_position(code) << 32) | (unsigned)row;
      if (codes) codes[((size_t)bh * 2 + side) * g.N + row] = (int)code;
    }
  }
  for (int i = g.N + tid; i < npow2; i += kSortThreads) keys[i] = ~0ull;
  __syncthreads();
  // bitonic sort, ascending
  for (int k = 2; k <= npow2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < npow2; i += kSortThreads) {
        const int l = i ^ j;
        if (l > i) {
          const unsigned long long a = keys[i], b = keys[l];
          const bool up = (i & k) == 0;
          if ((a > b) == up) {
            keys[i] = b;
            keys[l] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  int* out = order + ((size_t)bh * 2 + side) * g.N;
  for (int i = tid; i < g.N; i += kSortThreads) out[i] = (int)(keys[i] & 0xffffffffu);
}

// Rows of 16-byte units: dst[r] = src[perm[r]] (gather) or dst[perm[r]] = src[r]
// (scatter), for `rows_per_head` rows of `units` 16-byte units per head.
__global__ void permute_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                    const int* __restrict__ perm, int rows_per_head, int units, int BH,
                                    int perm_stride, int scatter) {
  const size_t total = (size_t)BH * rows_per_head * units;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const size_t row = e / units;
    const int u = (int)(e % units);
    const int bh = (int)(row / rows_per_head), r = (int)(row % rows_per_head);
    const size_t pr = (size_t)bh * rows_per_head + perm[(size_t)bh * perm_stride + r];
    if (scatter)
      dst[pr * units + u] = src[row * units + u];
    else
      dst[row * units + u] = src[pr * units + u];
  }
}

// Per-row float32 vectors (lambda, gates): dst[r] = src[perm[r]].
__global__ void gather_vec_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                  const int* __restrict__ perm, int N, int BH, int perm_stride) {
  const size_t total = (size_t)BH * N;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const int bh = (int)(e / N), r = (int)(e % N);
    dst[e] = src[(size_t)bh * N + perm[(size_t)bh * perm_stride + r]];
  }
}

// Tile t selects block t (the diagonal of the permuted score matrix).
__global__ void diag_select_kernel(int* __restrict__ idx, Geom g) {
  const size_t total = (size_t)g.BH * g.n_t;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    int* row = idx + e * g.k;
    row[0] = (int)(e % g.n_t);
    for (int c = 1; c < g.k; ++c) row[c] = -1;
  }
}

size_t sortlsh_smem_bytes(const Geom& g, int bits) {
  int npow2 = 1;
  while (npow2 < g.N) npow2 <<= 1;
  return (size_t)npow2 * 8 + (size_t)bits * g.d * 4;
}

cudaError_t launch_sortlsh_order(const void* Q, const void* K, bool bf16, const float* planes, int bits,
                                 int* order, int* codes, const Geom& g, cudaStream_t st) {
  int npow2 = 1;
  while (npow2 < g.N) npow2 <<= 1;
  const size_t smem = sortlsh_smem_bytes(g, bits);
  auto run = [&](auto kern, const auto* q, const auto* k) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ProfScope ps("sortlsh_order", st);
    kern<<<dim3(g.BH, 2), kSortThreads, smem, st>>>(q, k, planes, bits, npow2, order, codes, g);
    return cudaGetLastError();
  };
  if (bf16)
    return run(sortlsh_order_kernel<__nv_bfloat16>, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K);
  return run(sortlsh_order_kernel<float>, (const float*)Q, (const float*)K);
}

cudaError_t launch_permute_rows(const void* src, void* dst, const int* perm, int row_bytes, const Geom& g,
                                int perm_stride, bool scatter, cudaStream_t st) {
  const int units = row_bytes / 16;
  const size_t total = (size_t)g.BH * g.N * units;
  const int blocks = (int)std::min<size_t>((total + 255) / 256, 148 * 16);
  ProfScope ps(scatter ? "sortlsh_scatter" : "sortlsh_gather", st);
  permute_rows_kernel<<<blocks, 256, 0, st>>>((const uint4*)src, (uint4*)dst, perm, g.N, units, g.BH, perm_stride,
                                             scatter ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_gather_vec(const float* src, float* dst, const int* perm, const Geom& g, int perm_stride,
                              cudaStream_t st) {
  const size_t total = (size_t)g.BH * g.N;
  const int blocks = (int)std::min<size_t>((total + 255) / 256, 148 * 8);
  gather_vec_kernel<<<blocks, 256, 0, st>>>(src, dst, perm, g.N, g.BH, perm_stride);
  return cudaGetLastError();
}

cudaError_t launch_diag_select(int* idx, const Geom& g, cudaStream_t st) {
  const size_t total = (size_t)g.BH * g.n_t;
  diag_select_kernel<<<(int)std::min<size_t>((total + 255) / 256, 1024), 256, 0, st>>>(idx, g);
  return cudaGetLastError();
}

}  // namespace elsaa
