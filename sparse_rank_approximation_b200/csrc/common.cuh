// Device helpers shared by the ELSAA kernels (the RACE corner probabilities, bf16 packing,
// warp sums) and the problem description passed to every launch.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace elsaa {

constexpr int kHashBits = 4;
constexpr int kCorners = 1 << kHashBits;   // buckets per RACE table
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNormFloor = 1e-12f;

// Geometry of one call; every kernel receives it by value.
struct Geom {
  int BH;         // batch * heads
  int N, d;
  int T;          // block size (queries per tile = keys per block)
  int n_t;        // tiles = blocks = ceil(N / T)
  int k;          // selected blocks per tile
  int r;          // RACE features (0: branch off)
  int rp;         // RACE feature columns as stored: r, or on the tensor-core path r padded to G * 128
  int G;          // tensor-core path: feature groups of 128 (8 tables each), processed one after another
  int L;          // RACE tables
  int C;          // RACE chunk length
  int n_c;        // RACE chunks = ceil(N / C)
  int seg;        // chunks per state segment
  int n_seg;      // segments = ceil(n_c / seg)
  int dp;         // state columns: d value columns + 8 (column d holds the key mass)
  int causal;
  int fixed_m;    // fusion without the denominator-aware weight: m = 1, default g_lr = 1
  int selector;   // 0: top-k key blocks; 1: sortLSH (the operator runs on row-permuted copies)
  int lsh_bits;
  int lsh_levels; // causal sortLSH: recursion levels run on sorted rows (log2(n_t) - 1; the deepest
                  // level and the leaves run in the base pass)
  float scale, lam, eps, tau;
  // bounded waits: limit of the tensor-core kernels' pipeline waits in ns (default 2 s),
  // and a test hook that makes the sparse forward's softmax warps first wait on a
  // barrier nothing completes, so that the give-up path runs
  unsigned long long wait_ns;
  int debug_stall;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// sigma(y) and sigma(-y) = 1 - sigma(y) without cancellation: with e = exp(-|y|),
// 1 / (1 + e) is the larger and e / (1 + e) the smaller of the two.
__device__ __forceinline__ void sigmoid_pair(float y, float& sp, float& sm) {
  const float e = __expf(-fabsf(y));
  const float r = __fdividef(1.f, 1.f + e);
  const float t = e * r;
  sp = y >= 0.f ? r : t;
  sm = y >= 0.f ? t : r;
}

// The 16 corner probabilities of one table, p_c = prod_b (bit b of c ? sp_b : sm_b) * scale,
// as a two-level product (pairs of bits, then the cross product).
__device__ __forceinline__ void corner_probs(const float (&sp)[4], const float (&sm)[4], float scale,
                                             float (&p)[16]) {
  float lo[4], hi[4];
#pragma unroll
  for (int c2 = 0; c2 < 4; ++c2) {
    lo[c2] = ((c2 & 1) ? sp[0] : sm[0]) * ((c2 & 2) ? sp[1] : sm[1]) * scale;
    hi[c2] = ((c2 & 1) ? sp[2] : sm[2]) * ((c2 & 2) ? sp[3] : sm[3]);
  }
#pragma unroll
  for (int c = 0; c < 16; ++c) p[c] = lo[c & 3] * hi[c >> 2];
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename E> struct ElemIO;
template <> struct ElemIO<float> {
  static __device__ __forceinline__ float ld(const float* p) { return *p; }
  static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
};
template <> struct ElemIO<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

}  // namespace elsaa
