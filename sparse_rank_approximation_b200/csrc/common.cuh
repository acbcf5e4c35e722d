// Device helpers shared by the ELSAA kernels: async copies, ldmatrix, bf16 MMA
// fragments, and the problem description passed to every launch.
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
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global->shared copy; when !pred the destination is zero-filled and
// nothing is read (src must still be a mapped address, callers clamp it).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
  const int n = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n"
               :: "r"(smem_u32(smem)), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" :: "n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r[0]), "=r"(r[1]) : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r[0]), "=r"(r[1]) : "r"(smem_u32(p)));
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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

// Fragment addressing for a warp's m16n8k16 tiles held in padded shared memory.
// A operand, row-major [16 x 16] at (row0, col0) of an array with `ld` elements per row.
__device__ __forceinline__ const __nv_bfloat16* a_frag_ptr(const __nv_bfloat16* base, int ld, int row0,
                                                         int col0, int lane) {
  return base + (row0 + (lane & 7) + ((lane >> 3) & 1) * 8) * ld + col0 + (lane >> 4) * 8;
}
// A operand given as its transpose stored [k][m] (m contiguous): use with ldsm_x4_t.
__device__ __forceinline__ const __nv_bfloat16* at_frag_ptr(const __nv_bfloat16* base, int ld, int m0,
                                                          int k0, int lane) {
  return base + (k0 + (lane & 7) + (lane >> 4) * 8) * ld + m0 + ((lane >> 3) & 1) * 8;
}
// B operand stored [n][k] (k contiguous), two n-blocks (n0, n0+8) x k16: ldsm_x4 gives
// {b0,b1} of n-block n0 then {b0,b1} of n-block n0+8.
__device__ __forceinline__ const __nv_bfloat16* bnk_frag_ptr(const __nv_bfloat16* base, int ld, int n0,
                                                           int k0, int lane) {
  return base + (n0 + (lane & 7) + (lane >> 4) * 8) * ld + k0 + ((lane >> 3) & 1) * 8;
}
// B operand stored [k][n] (n contiguous), k16 x two n-blocks: ldsm_x4_t gives
// {b0,b1} of n-block n0 then {b0,b1} of n-block n0+8.
__device__ __forceinline__ const __nv_bfloat16* bkn_frag_ptr(const __nv_bfloat16* base, int ld, int k0,
                                                           int n0, int lane) {
  return base + (k0 + (lane & 7) + ((lane >> 3) & 1) * 8) * ld + n0 + (lane >> 4) * 8;
}
// Single n-block variants for ldsm_x2 / ldsm_x2_t (lanes 0..15 supply addresses).
__device__ __forceinline__ const __nv_bfloat16* bnk_frag_ptr1(const __nv_bfloat16* base, int ld, int n0,
                                                            int k0, int lane) {
  return base + (n0 + (lane & 7)) * ld + k0 + ((lane >> 3) & 1) * 8;
}
__device__ __forceinline__ const __nv_bfloat16* bkn_frag_ptr1(const __nv_bfloat16* base, int ld, int k0,
                                                            int n0, int lane) {
  return base + (k0 + (lane & 7) + ((lane >> 3) & 1) * 8) * ld + n0;
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
