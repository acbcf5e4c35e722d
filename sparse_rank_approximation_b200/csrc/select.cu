// Top-k key-block selector of the sparse branch, and the key-block -> query-tile
// inverse map the backward uses.
//
// The ELSAA paper lets the sparse branch use any efficient important-key
// selector that returns an exact sparse output and a denominator (§3.3,
// Practical notes) and names top-k / large-entry selectors (§1, §3).  Here a
// tile's score for key block b is the mean-pooled logit
//   s_tb = scale * mean_{i in t} q_i . mean_{j in b} k_j,
// computed in float64 and rounded once to float32; ranking is on the float32
// value, highest first, lower block index on ties.  Causal tiles always keep
// their diagonal block and rank only earlier blocks.
#include "common.cuh"
#include "kernels.h"

namespace elsaa {

// Column means of consecutive groups of T rows (the last group may be short), in float64.
// grid (n_t, BH, 2): z = 0 pools Q, z = 1 pools K.  block 128.
template <typename E>
__global__ void __launch_bounds__(128) pool_means_kernel(const E* __restrict__ Q, const E* __restrict__ K,
                                                         double* __restrict__ qbar, double* __restrict__ kbar,
                                                         Geom g) {
  constexpr int VEC = 16 / sizeof(E);
  const int t = blockIdx.x, bh = blockIdx.y;
  const E* X = (blockIdx.z == 0 ? Q : K) + (size_t)bh * g.N * g.d;
  double* out = (blockIdx.z == 0 ? qbar : kbar) + ((size_t)bh * g.n_t + t) * g.d;
  const int tpr = g.d / VEC;              // threads per row
  const int rows_par = 128 / tpr;         // rows read in parallel
  const int c0 = (threadIdx.x % tpr) * VEC;
  const int rg = threadIdx.x / tpr;
  const int r0 = t * g.T;
  const int r1 = min(g.N, r0 + g.T);
  double acc[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) acc[v] = 0.0;
  for (int row = r0 + rg; row < r1; row += rows_par) {
    const uint4 raw = *reinterpret_cast<const uint4*>(X + (size_t)row * g.d + c0);
    const E* e = reinterpret_cast<const E*>(&raw);
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] += (double)ElemIO<E>::ld(e + v);
  }
  __shared__ double red[128 * 8];
  for (int v = 0; v < VEC; ++v) red[threadIdx.x * VEC + v] = acc[v];
  __syncthreads();
  const double inv = 1.0 / (double)(r1 - r0);
  for (int c = threadIdx.x; c < g.d; c += 128) {
    // column c lives in thread (c / VEC) % tpr of every row group
    const int tt = c / VEC, v = c % VEC;
    double s = 0.0;
    for (int q = 0; q < rows_par; ++q) s += red[(q * tpr + tt) * VEC + v];
    out[c] = s * inv;
  }
}

// scores[bh, t, b] = (float)(scale * qbar_t . kbar_b), float64 dot.  grid (ceil(n_t/32), ceil(n_t/32), BH), block 32x8.
__global__ void __launch_bounds__(256) block_scores_kernel(const double* __restrict__ qbar,
                                                           const double* __restrict__ kbar,
                                                           float* __restrict__ scores, Geom g) {
  __shared__ double sq[32][33], sk[32][33];
  const int bh = blockIdx.z;
  const int b0 = blockIdx.x * 32, t0 = blockIdx.y * 32;
  const double* qb = qbar + (size_t)bh * g.n_t * g.d;
  const double* kb = kbar + (size_t)bh * g.n_t * g.d;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int c0 = 0; c0 < g.d; c0 += 32) {
    for (int i = ty; i < 32; i += 8) {
      const int t = t0 + i, b = b0 + i;
      sq[i][tx] = t < g.n_t ? qb[(size_t)t * g.d + c0 + tx] : 0.0;
      sk[i][tx] = b < g.n_t ? kb[(size_t)b * g.d + c0 + tx] : 0.0;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {
      const double kv = sk[tx][c];
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] += sq[ty + 8 * j][c] * kv;
    }
    __syncthreads();
  }
  float* out = scores + (size_t)bh * g.n_t * g.n_t;
  const int b = b0 + tx;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int t = t0 + ty + 8 * j;
    if (t < g.n_t && b < g.n_t) out[(size_t)t * g.n_t + b] = (float)((double)g.scale * acc[j]);
  }
}

// One warp per tile row: the row's scores are read once into registers (lane l holds blocks
// l, l + 32, ..., n_t <= 1024), the best `need` candidates by (score desc, index asc) come out
// of repeated warp arg-max passes over them, and the set is emitted in ascending order.
// grid (ceil(n_t/8), BH), block 256.
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ scores, int* __restrict__ idx,
                                                   Geom g) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  const int bh = blockIdx.y;
  __shared__ uint32_t sel[8][32];          // bitmap of chosen blocks, n_t <= 1024
  if (t >= g.n_t) return;
  const float* row = scores + ((size_t)bh * g.n_t + t) * g.n_t;
  int* out = idx + ((size_t)bh * g.n_t + t) * g.k;
  sel[warp][lane] = 0u;
  __syncwarp();
  const int n_cand = g.causal ? t : g.n_t;     // eligible, apart from a forced diagonal
  int need = g.causal ? g.k - 1 : g.k;
  if (g.k == 0) need = 0;
  if (g.causal && g.k > 0 && lane == 0) sel[warp][t >> 5] |= 1u << (t & 31);
  __syncwarp();
  if (need >= n_cand) {
    for (int b = lane; b < n_cand; b += 32) atomicOr(&sel[warp][b >> 5], 1u << (b & 31));
  } else {
    const int nj = (n_cand + 31) >> 5;          // register slots in use (warp-uniform)
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j >= nj) break;
      const int b = lane + 32 * j;
      v[j] = b < n_cand ? row[b] : 0.f;
    }
    float last_s = __int_as_float(0x7f800000);   // +inf: everything ranks below
    int last_b = -1;
    for (int it = 0; it < need; ++it) {
      float bs = -__int_as_float(0x7f800000);
      int bb = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j >= nj) break;
        const int b = lane + 32 * j;
        const float s = v[j];
        const bool below = (s < last_s) || (s == last_s && b > last_b);
        const bool better = (s > bs) || (s == bs && b < bb);
        if (b < n_cand && below && better) { bs = s; bb = b; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, o);
        const int ob = __shfl_xor_sync(0xffffffffu, bb, o);
        if (os > bs || (os == bs && ob < bb)) { bs = os; bb = ob; }
      }
      if (bb >= n_cand) break;   // only reachable with NaN scores (undefined input)
      last_s = bs;
      last_b = bb;
      if (lane == 0) sel[warp][bb >> 5] |= 1u << (bb & 31);
    }
  }
  __syncwarp();
  // ascending compaction of the bitmap: lane w owns blocks [32w, 32w+32)
  const uint32_t word = sel[warp][lane];
  const int cnt = __popc(word);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int pos = incl - cnt;
  uint32_t w = word;
  while (w) {
    const int bit = __ffs(w) - 1;
    w &= w - 1;
    out[pos++] = lane * 32 + bit;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  for (int s = total + lane; s < g.k; s += 32) out[s] = -1;
}

// Inverse of the selection for the key-major backward: for each key block b the
// ascending list of query tiles that selected it.  grid (BH), block 256.
// Output per head: offs[n_t + 1] and tiles[n_t * k] (CSR), and order[n_t]: the key
// blocks by descending count, ties by ascending block (a longest-first launch
// order for the key-major backward).  Deterministic.
__global__ void __launch_bounds__(256) invert_selection_kernel(const int* __restrict__ idx,
                                                               int* __restrict__ offs, int* __restrict__ tiles,
                                                               int* __restrict__ order, Geom g) {
  extern __shared__ uint32_t bits[];      // n_t rows x words bitmap: bit (t, b)
  const int bh = blockIdx.x;
  const int words = (g.n_t + 31) >> 5;
  const int* id = idx + (size_t)bh * g.n_t * g.k;
  int* of = offs + (size_t)bh * (g.n_t + 1);
  int* tl = tiles + (size_t)bh * g.n_t * g.k;
  for (int i = threadIdx.x; i < g.n_t * words; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < g.n_t * g.k; i += blockDim.x) {
    const int b = id[i];
    if (b >= 0) atomicOr(&bits[(i / g.k) * words + (b >> 5)], 1u << (b & 31));
  }
  __syncthreads();
  // counts per key block: column popcounts (one warp per block b)
  __shared__ int cnt_s[1025];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int b = warp; b < g.n_t; b += nw) {
    int c = 0;
    for (int t = lane; t < g.n_t; t += 32) c += (bits[t * words + (b >> 5)] >> (b & 31)) & 1u;
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) cnt_s[b] = c;
  }
  __syncthreads();
  if (order) {
    int* od = order + (size_t)bh * g.n_t;
    for (int b = threadIdx.x; b < g.n_t; b += blockDim.x) {
      const int c = cnt_s[b];
      int rank = 0;
      for (int b2 = 0; b2 < g.n_t; ++b2) {
        const int c2 = cnt_s[b2];
        rank += (c2 > c) || (c2 == c && b2 < b);
      }
      od[rank] = b;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int b = 0; b < g.n_t; ++b) {
      const int c = cnt_s[b];
      cnt_s[b] = acc;
      of[b] = acc;
      acc += c;
    }
    of[g.n_t] = acc;
  }
  __syncthreads();
  for (int b = warp; b < g.n_t; b += nw) {
    int base = cnt_s[b];
    for (int t0 = 0; t0 < g.n_t; t0 += 32) {
      const int t = t0 + lane;
      const bool on = t < g.n_t && ((bits[t * words + (b >> 5)] >> (b & 31)) & 1u);
      const uint32_t m = __ballot_sync(0xffffffffu, on);
      if (on) tl[base + __popc(m & ((1u << lane) - 1u))] = t;
      base += __popc(m);
    }
  }
}

cudaError_t launch_select(const void* Q, const void* K, bool bf16, double* qbar, double* kbar, float* scores,
                          int* idx, const Geom& g, cudaStream_t st) {
  {
    ProfScope ps("pool_means", st);
    if (bf16)
      pool_means_kernel<__nv_bfloat16><<<dim3(g.n_t, g.BH, 2), 128, 0, st>>>(
          (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, qbar, kbar, g);
    else
      pool_means_kernel<float><<<dim3(g.n_t, g.BH, 2), 128, 0, st>>>((const float*)Q, (const float*)K, qbar, kbar,
                                                                       g);
  }
  const int nb = (g.n_t + 31) / 32;
  {
    ProfScope ps("block_scores", st);
    block_scores_kernel<<<dim3(nb, nb, g.BH), dim3(32, 8), 0, st>>>(qbar, kbar, scores, g);
  }
  if (g.k > 0) {
    ProfScope ps("topk", st);
    topk_kernel<<<dim3((g.n_t + 7) / 8, g.BH), 256, 0, st>>>(scores, idx, g);
  }
  return cudaGetLastError();
}

cudaError_t launch_invert_selection(const int* idx, int* offs, int* tiles, int* order, const Geom& g,
                                    cudaStream_t st) {
  const size_t smem = (size_t)g.n_t * ((g.n_t + 31) / 32) * 4;
  cudaError_t e = cudaFuncSetAttribute(invert_selection_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps("invert_selection", st);
  invert_selection_kernel<<<g.BH, 256, smem, st>>>(idx, offs, tiles, order, g);
  return cudaGetLastError();
}

}  // namespace elsaa
