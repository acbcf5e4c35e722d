// RACE low-rank branch (ELSAA paper §3.1) read-out and backward on the 5th-generation
// tensor cores, for d = 128 and chunk C = 128, over the features in groups of 128 (8 tables of
// 16 corners; r up to 256, zero-padded to whole groups).  Each group is one launch; the read-out
// carries its running numerator and denominator from the first group to the last, the backward
// kernels add the later groups' parts to the fp32 accumulators.
// One CTA per (head, chunk of 128 rows); every accumulator lives in tensor memory.
//
// Read-out, chunk t (query rows i):
//   [N_lr,i ; d_lr,i] = Phi(q_i) [P^V ; p1] + sum_{j in t, j <= i} (Phi(q_i).Phi(k_j)) [v_j ; 1],
//   O_lr,i = N_lr,i / d_lr,i (bf16) and d_lr,i (fp32), with P the prefix statistics.
//
// Key side, chunk c (rows j):
//   kappa^T = Phi(K_c) Phi(Q_c)^T and X = V_c dO_c^T (causal intra-chunk terms),
//   dv_j    = R^V^T Phi(k_j) + sum_{i in c, i >= j} cl_i kappa_ij dO_i,
//   dPhi_kj = R^V v_j + r1 + sum_{i in c, i >= j} (cl_i <dO_i, v_j> + delta_i) Phi(q_i),
// with R the suffix statistics of the later chunks (sum of Phi(q_i) [cl_i dO_i; delta_i]^T).
// Query side, chunk t (rows i):
//   dPhi_qi = cl_i P^V dO_i + delta_i p1 + sum_{j in t, j <= i} (cl_i <dO_i, v_j> + delta_i) Phi(k_j),
// with P the prefix statistics of the earlier chunks.  Both then go through the
// corner softmax (dh_b = (1/tau) sum_c p_c (dp_c - <dp, p>) c_b, dp = dPhi / sqrt(L)),
// du = dh W^T and dx = (du - x <x, du> / |x|^2) / |x| into the fp32 accumulators.
//
// Work split: warp 0 issues the TMA loads (the chunk's tiles, its statistics as
// bf16 hi + lo halves written per chunk by the split kernel, and W as bf16 hi + lo),
// warp 1 the MMAs, warps 2..9 (256 threads, TMEM lane quarter = warp % 4, column
// half = (warp - 2) / 4) load the per-row scalars and run the element-wise passes.  The masked intra-chunk
// matrices (bf16) and dh (bf16 hi + lo) are written back into tensor memory over
// the fp32 values they replace and feed the next products as the A operand.
// Every mbarrier wait is bounded; a timeout sets a bit in the caller's error word.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace elsaa {

namespace {

constexpr int kC = 128;
constexpr int kR = 128;
constexpr int kNH = 32;                          // projection columns 4 L
constexpr uint32_t kSlab = 128 * 128;            // [128 rows][64 bf16], 128-byte swizzle
constexpr uint32_t kTile = 2 * kSlab;            // [128 rows][128 bf16]
constexpr uint32_t kWSlab = kNH * 128;           // [32 rows][64 bf16]
constexpr int kThreads = 320;
constexpr int kComputeThreads = 256;

// Byte offset of element (row, col) of a [rows][128] bf16 tile kept as two
// 64-column slabs of `slab` bytes with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw_off(int row, int col, uint32_t slab) {
  return (uint32_t)(col >> 6) * slab + (uint32_t)row * 128u + (uint32_t)((((col & 63) >> 3) ^ (row & 7)) << 4) +
         (uint32_t)(col & 7) * 2u;
}
__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }

// Operand descriptors, built once from the shared-memory base; an operand at byte offset
// `off` and its K = 16 step kk only move the start address (one 32-bit add per descriptor).
struct SDesc {
  uint64_t k16, mn, mn_w;
  __device__ explicit SDesc(uint32_t sb)
      : k16(tc::sw128_desc(sb, 16, 1024)), mn(tc::sw128_desc(sb, kSlab, 1024)), mn_w(tc::sw128_desc(sb, kWSlab, 1024)) {}
  // K-major operand, K = 16 step kk of a [rows][128] tile
  __device__ uint64_t k(uint32_t off, int kk) const {
    return tc::desc_adv(k16, off + (uint32_t)(kk >> 2) * kSlab + (uint32_t)(kk & 3) * 32u);
  }
  // MN-major operand: rows are K, 128 columns are N (64-column slabs kSlab apart)
  __device__ uint64_t kn(uint32_t off, int kk) const { return tc::desc_adv(mn, off + (uint32_t)kk * 2048u); }
  // MN-major with slabs kWSlab apart (the hash-projection weights)
  __device__ uint64_t kn_w(uint32_t off, int kk) const { return tc::desc_adv(mn_w, off + (uint32_t)kk * 2048u); }
};
// TMEM column of the K = 16 step kk of a packed bf16 operand whose K index
// 64 h + m (h = column half of the thread that wrote it) sits at column 64 h + m / 2.
__device__ __forceinline__ uint32_t packed_col(int kk) { return (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8); }

struct Bars {
  uint64_t in_main, s_full, p_full, acc_full, dh_full, du_full, x_full;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Bars* ms, uint32_t* err,
                                              uint32_t code) {
  if (*(volatile int*)&ms->abort_flag) return false;
  if (tc::mbar_wait(bar, parity)) return true;
  *(volatile int*)&ms->abort_flag = 1;
  if (err) atomicOr(err, code);
  return false;
}

__device__ __forceinline__ void split2(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Corner-softmax backward of one table: h (4 normalised projections), dp (16
// corner adjoints, already divided by sqrt(L)) -> dh (4 values).
__device__ __forceinline__ void corner_bwd(const float (&h)[4], const float (&dp)[16], float inv_tau,
                                           float (&dh)[4]) {
  float sp[4], sm[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) sigmoid_pair(2.f * h[b] * inv_tau, sp[b], sm[b]);
  float p[16], s = 0.f;
  corner_probs(sp, sm, 1.f, p);
#pragma unroll
  for (int c = 0; c < 16; ++c) s = fmaf(p[c], dp[c], s);
#pragma unroll
  for (int b = 0; b < 4; ++b) dh[b] = 0.f;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const float da = p[c] * (dp[c] - s);
#pragma unroll
    for (int b = 0; b < 4; ++b) dh[b] += ((c >> b) & 1) ? da : -da;
  }
#pragma unroll
  for (int b = 0; b < 4; ++b) dh[b] *= inv_tau;
}

// Corner pass for the 4 tables 4 hc .. 4 hc + 3 of one row: dPhi of those tables
// (fp32, 64 TMEM columns from `dphi_col`, plus the optional `cl * G + de * m1`
// terms), projections h (global, fp32), then dh as bf16 hi / lo into TMEM columns
// 8 hc (hi) and 16 + 8 hc (lo).
// The projections of this thread's 4 tables (tables 8 grp + 4 hc .. + 3 of a row whose 4 L
// projections start at hrow); tables past the last one (padding of the group) read as zero.
__device__ __forceinline__ void load_h(const float* __restrict__ hrow, int grp, int hc, int L, float (&h16)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int table = 8 * grp + 4 * hc + q;
    const float4 v = hrow && table < L ? __ldg(reinterpret_cast<const float4*>(hrow) + table)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
    h16[4 * q] = v.x; h16[4 * q + 1] = v.y; h16[4 * q + 2] = v.z; h16[4 * q + 3] = v.w;
  }
}
// Row `row` of a [128][D] bf16 tile that TMA wrote as 64-column slabs with the 128-byte
// swizzle: this thread's half (columns D/2 hc .. D/2 hc + D/2 - 1) as D/16 x 16 bytes.  Eight
// consecutive rows read eight different 16-byte positions, so a warp's reads do not conflict.
template <int D>
__device__ __forceinline__ void load_x(const unsigned char* tile, int row, int hc, bool valid, uint4 (&xr)[D / 16]) {
  const int c0 = (D / 2) * hc;                      // first column of this half
  const unsigned char* base = tile + (uint32_t)(c0 >> 6) * kSlab + (uint32_t)row * 128u;
#pragma unroll
  for (int q = 0; q < D / 16; ++q)
    xr[q] = valid ? *reinterpret_cast<const uint4*>(base + (((((c0 & 63) >> 3) + q) ^ (row & 7)) << 4))
                  : make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ void corner_pass(uint32_t tmem, uint32_t lane_base, int hc, uint32_t dphi_col,
                                            bool has_dphi, uint32_t g_col, float cl, float de, const float* m1,
                                            const float (&h16)[16], float inv_sqrt_L, float inv_tau) {
  float dh16[16];
#pragma unroll
  for (int tl = 0; tl < 4; ++tl) {
    float a[16], gg[16];
    const uint32_t col = 64u * hc + 16u * tl;
    if (has_dphi) tc::tmem_ld16(tmem + lane_base + dphi_col + col, a);
    if (g_col) tc::tmem_ld16(tmem + lane_base + g_col + col, gg);
    tc::tmem_wait_ld();
    float dp[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      float v = has_dphi ? a[c] : 0.f;
      if (g_col) v = fmaf(cl, gg[c], v);
      v = fmaf(de, m1[col + c], v);
      dp[c] = v * inv_sqrt_L;
    }
    float h[4] = {h16[4 * tl], h16[4 * tl + 1], h16[4 * tl + 2], h16[4 * tl + 3]}, dh[4];
    corner_bwd(h, dp, inv_tau, dh);
#pragma unroll
    for (int b = 0; b < 4; ++b) dh16[4 * tl + b] = dh[b];
  }
  uint32_t hi[8], lo[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) split2(dh16[2 * e], dh16[2 * e + 1], hi[e], lo[e]);
  tc::tmem_st8(tmem + lane_base + 8u * hc, hi);
  tc::tmem_st8(tmem + lane_base + 16u + 8u * hc, lo);
}

// du = dh W^T: three products (hi hi, hi lo, lo hi), K = 32 (two steps each), N = D.
template <int D>
__device__ __forceinline__ void issue_du(uint32_t tmem, uint32_t d_col, const SDesc& sd, uint32_t w_hi, uint32_t w_lo) {
  const uint32_t idG = tc::idesc_bf16(128, D, false, true);
#pragma unroll
  for (int part = 0; part < 3; ++part) {
    const uint32_t a_col = part == 2 ? 16u : 0u;
    const uint32_t wb = part == 1 ? w_lo : w_hi;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk)
      tc::mma_bf16_ts(tmem + d_col, tmem + a_col + 8u * kk, sd.kn_w(wb, kk), idG,
                      (part > 0 || kk > 0) ? 1u : 0u);
  }
}

// fp32 gradient rows leave through shared memory: each thread writes its row there (pitch
// D + 4 floats, so the 16-byte stores of 8 consecutive rows hit 8 different bank groups),
// then all compute threads copy the [128][D] tile out with coalesced 16-byte stores.  The
// staging area reuses operand tiles that no product reads any more.
template <int D> constexpr int stage_pitch() { return D + 4; }
template <int D> constexpr uint32_t stage_bytes() { return (uint32_t)kC * stage_pitch<D>() * 4; }

// `add`: the feature groups after the first add their part to what the earlier ones wrote.
template <int D>
__device__ __forceinline__ void copy_staged(const float* stage, float* __restrict__ out, int rows, int ct, bool add) {
  for (int idx = ct; idx < kC * (D / 4); idx += kComputeThreads) {
    const int r = idx / (D / 4), c4 = idx % (D / 4);
    if (r < rows) {
      float4 v = *reinterpret_cast<const float4*>(stage + r * stage_pitch<D>() + 4 * c4);
      float4* o = reinterpret_cast<float4*>(out + (size_t)r * D) + c4;
      if (add) {
        const float4 p = *o;
        v.x += p.x; v.y += p.y; v.z += p.z; v.w += p.w;
      }
      *o = v;
    }
  }
}

// dx = (du - x <x, du> / n^2) / n for one row, this thread's 64 columns; the two
// column halves of a row meet through `xch`.  Stores fp32 into out (row pointer).
// Every compute thread calls this (the exchange barrier); `alive` false skips the
// tensor-memory reads and the stores.
template <int D>
__device__ __forceinline__ void chain_pass(uint32_t tmem, uint32_t lane_base, int hc, int row_in_chunk,
                                           uint32_t du_col, const uint4 (&xr)[D / 16], float n, float* xch,
                                           float* stage, bool valid, bool alive) {
  constexpr int H = D / 2;                          // this thread's columns
  float du[H];
  if (alive) {
    tc::tc_fence_after();
#pragma unroll
    for (int h2 = 0; h2 < H / 32; ++h2)
      tc::tmem_ld32(tmem + lane_base + du_col + H * hc + 32u * h2, *reinterpret_cast<float(*)[32]>(du + 32 * h2));
  } else {
#pragma unroll
    for (int q = 0; q < H; ++q) du[q] = 0.f;
  }
  valid = valid && alive;
  if (alive) tc::tmem_wait_ld();
  float xd = 0.f;
#pragma unroll
  for (int q = 0; q < D / 16; ++q) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&xr[q]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(p[e]);
      xd = fmaf(x.x, du[8 * q + 2 * e], xd);
      xd = fmaf(x.y, du[8 * q + 2 * e + 1], xd);
    }
  }
  xch[2 * row_in_chunk + hc] = xd;
  compute_bar();
  xd = xch[2 * row_in_chunk] + xch[2 * row_in_chunk + 1];
  if (!valid) return;
  const float proj = n <= kNormFloor ? 0.f : xd / (n * n);
  const float inv = 1.f / n;
  float4* o = reinterpret_cast<float4*>(stage + row_in_chunk * stage_pitch<D>() + H * hc);
#pragma unroll
  for (int q = 0; q < D / 16; ++q) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&xr[q]);
    const float2 x0 = __bfloat1622float2(p[0]), x1 = __bfloat1622float2(p[1]);
    const float2 x2 = __bfloat1622float2(p[2]), x3 = __bfloat1622float2(p[3]);
    o[2 * q] = make_float4((du[8 * q] - x0.x * proj) * inv, (du[8 * q + 1] - x0.y * proj) * inv,
                           (du[8 * q + 2] - x1.x * proj) * inv, (du[8 * q + 3] - x1.y * proj) * inv);
    o[2 * q + 1] = make_float4((du[8 * q + 4] - x2.x * proj) * inv, (du[8 * q + 5] - x2.y * proj) * inv,
                               (du[8 * q + 6] - x3.x * proj) * inv, (du[8 * q + 7] - x3.y * proj) * inv);
  }
}

// ------------------------------- key side ------------------------------------
constexpr uint32_t K_PK = 0, K_PQ = kTile, K_V = 2 * kTile, K_DO = 3 * kTile, K_RH = 4 * kTile, K_RL = 5 * kTile;
constexpr uint32_t K_WH = 6 * kTile, K_WL = K_WH + 2 * kWSlab;
constexpr uint32_t K_CL = K_WL + 2 * kWSlab;            // cl [128], delta [128], r1 [128], exchange [256]
constexpr uint32_t K_BARS = K_CL + (3 * 128 + 256) * 4;
// TMEM columns
constexpr uint32_t TK_KAP = 0, TK_X = 128, TK_DV = 256, TK_DPHI = 384, TK_DU = 128;
// staged dV and dK rows, over the operand tiles once every product that reads them is done
constexpr uint32_t K_STAGE_V = 0;
template <int D> constexpr uint32_t k_stage_k() { return (stage_bytes<D>() + 1023u) & ~1023u; }
// the K rows of the chunk for dx, over the statistics tiles once their products are done
template <int D> constexpr uint32_t k_xs() { return (k_stage_k<D>() + stage_bytes<D>() + 1023u) & ~1023u; }
static_assert(k_xs<128>() + kTile <= K_WH && k_xs<64>() + kTile <= K_WH,
              "the staged rows and the K tile overlap only the chunk tiles");

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    race_k_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmPK, const __grid_constant__ CUtensorMap tmPQ,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                         const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmW,
                         const __grid_constant__ CUtensorMap tmX, BwdArgs a, Geom g, int grp, uint32_t* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  Bars* ms = reinterpret_cast<Bars*>(smem + K_BARS);
  float* sCl = reinterpret_cast<float*>(smem + K_CL);
  float* sDl = sCl + 128;
  float* sR1 = sCl + 256;
  float* sX = sCl + 384;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, bh = blockIdx.y;
  const size_t head = (size_t)bh * g.N;
  const bool causal = g.causal;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0 && err) atomicOr(err, 0x80000000u);
    return;
  }
  if (threadIdx.x == 0) {
    tc::mbar_init(&ms->in_main, 1);
    tc::mbar_init(&ms->s_full, 1);
    tc::mbar_init(&ms->p_full, kComputeThreads);
    tc::mbar_init(&ms->acc_full, 1);
    tc::mbar_init(&ms->dh_full, kComputeThreads);
    tc::mbar_init(&ms->du_full, 1);
    tc::mbar_init(&ms->x_full, 1);
    ms->abort_flag = 0;
    tc::fence_barrier_init();
    // the chunk's tiles do not depend on anything the set-up computes: their copies start first
    {
      // Phi tiles are [128][128]; V, dO, the statistics and W are D columns wide
      constexpr uint32_t kTD = 128u * D * 2, kWD = (uint32_t)kNH * D * 2;
      tc::mbar_arrive_expect_tx(&ms->in_main, (causal ? 2 : 1) * kTile + (causal ? 2 : 1) * kTD + 2 * kTD + 2 * kWD);
      const int z = (bh * g.n_c + c) * 2;
      for (int s = 0; s < 2; ++s) {
        tc::tma_load_3d(smem + K_PK + s * kSlab, &tmPK, &ms->in_main, 64 * s, c * kC, bh);
        if (causal) tc::tma_load_3d(smem + K_PQ + s * kSlab, &tmPQ, &ms->in_main, 64 * s, c * kC, bh);
      }
      for (int s = 0; s < D / 64; ++s) {
        tc::tma_load_3d(smem + K_V + s * kSlab, &tmV, &ms->in_main, 64 * s, c * kC, bh);
        if (causal) tc::tma_load_3d(smem + K_DO + s * kSlab, &tmdO, &ms->in_main, 64 * s, c * kC, bh);
        tc::tma_load_3d(smem + K_RH + s * kSlab, &tmR, &ms->in_main, 64 * s, 0, z);
        tc::tma_load_3d(smem + K_RL + s * kSlab, &tmR, &ms->in_main, 64 * s, 0, z + 1);
        tc::tma_load_3d(smem + K_WH + s * kWSlab, &tmW, &ms->in_main, 64 * s, kNH * grp, 0);
        tc::tma_load_3d(smem + K_WL + s * kWSlab, &tmW, &ms->in_main, 64 * s, kNH * grp, 1);
      }
    }
  }
  if (warp == 1) {
    tc::tmem_alloc(&ms->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      constexpr uint32_t kTD = 128u * D * 2;
      tc::mbar_wait(&ms->in_main, 0);
      // the K rows for dx, once every product but du has read the chunk tiles; waited for
      // here too, so no copy is in flight when the CTA exits
      if (wait_or_abort(&ms->acc_full, 0, ms, err, 0x10000u)) {
        tc::mbar_arrive_expect_tx(&ms->x_full, kTD);
        for (int s = 0; s < D / 64; ++s)
          tc::tma_load_3d(smem + k_xs<D>() + s * kSlab, &tmX, &ms->x_full, 64 * s, c * kC, bh);
        wait_or_abort(&ms->x_full, 0, ms, err, 0x20000u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idNN = tc::idesc_bf16(128, 128, false, false);
      const uint32_t idNM = tc::idesc_bf16(128, 128, false, true);
      const uint32_t idDM = tc::idesc_bf16(128, D, false, true);     // N = D, B MN-major
      const SDesc sd(smem_u32(smem));
      bool ok = wait_or_abort(&ms->in_main, 0, ms, err, 0x100u);
      if (ok && causal) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_bf16(tmem + TK_KAP, sd.k(K_PK, kk), sd.k(K_PQ, kk), idNN, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_bf16(tmem + TK_X, sd.k(K_V, kk), sd.k(K_DO, kk), idNN, kk > 0 ? 1u : 0u);
        tc::mma_commit(&ms->s_full);
      }
      if (ok) {
        // inter-chunk parts: dv = Phi_K R^V, dPhi = V R^V^T (R as bf16 hi + lo)
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t rb = part ? K_RL : K_RH;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_bf16(tmem + TK_DV, sd.k(K_PK, kk), sd.kn(rb, kk), idDM,
                         (part > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tc::mma_bf16(tmem + TK_DPHI, sd.k(K_V, kk), sd.k(rb, kk), idNN, (part > 0 || kk > 0) ? 1u : 0u);
        }
      }
      if (ok && causal) {
        ok = wait_or_abort(&ms->p_full, 0, ms, err, 0x400u);
        if (ok) {
          tc::tc_fence_after();
          // intra-chunk parts, A operands from tensor memory
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_bf16_ts(tmem + TK_DV, tmem + TK_KAP + packed_col(kk), sd.kn(K_DO, kk), idDM, 1u);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_bf16_ts(tmem + TK_DPHI, tmem + TK_X + packed_col(kk), sd.kn(K_PQ, kk), idNM, 1u);
        }
      }
      tc::mma_commit(&ms->acc_full);
      ok = ok && wait_or_abort(&ms->dh_full, 0, ms, err, 0x800u);
      if (ok) {
        tc::tc_fence_after();
        issue_du<D>(tmem, TK_DU, sd, K_WH, K_WL);
      }
      tc::mma_commit(&ms->du_full);
      tc::mbar_wait(&ms->du_full, 0);
    }
  } else {
    const int ct = threadIdx.x - 64;
    const int q4 = warp & 3, hc = (warp - 2) >> 2;
    const int j = 32 * q4 + lane;                     // row of the chunk (TMEM lane)
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const int row = c * kC + j;
    const bool valid = row < g.N;
    float* stage_v = reinterpret_cast<float*>(smem + K_STAGE_V);
    float* stage_k = reinterpret_cast<float*>(smem + k_stage_k<D>());
    // row data for the corner and chain passes, fetched up front
    float h16[16];
    load_h(valid ? a.hK + (head + row) * 4 * g.L : nullptr, grp, hc, g.L, h16);
    const float nrm = valid ? a.nK[head + row] : 1.f;
    // ---- per-row scalars of the chunk and the key-mass column of the suffix statistics ----
    if (ct < kC) {
      const int r = c * kC + ct;
      sCl[ct] = r < g.N ? a.rs.cl[head + r] : 0.f;
      sDl[ct] = r < g.N ? a.rs.delta[head + r] : 0.f;
      sR1[ct] = a.Rmass[(((size_t)grp * g.BH + bh) * g.n_c + c) * kR + ct];
    }
    compute_bar();
    bool alive = true;
    // ---- intra-chunk element-wise pass: (cl_i kappa_ji) and (cl_i X_ji + delta_i), i >= j ----
    if (causal) {
      alive = __all_sync(0xffffffffu, wait_or_abort(&ms->s_full, 0, ms, err, 0x1000u));
      if (alive) {
        tc::tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 16) {
          float kv[16], xv[16];
          tc::tmem_ld16(tmem + lane_base + TK_KAP + 64 * hc + c0, kv);
          tc::tmem_ld16(tmem + lane_base + TK_X + 64 * hc + c0, xv);
          tc::tmem_wait_ld();
          uint32_t wk[8], wx[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float pk[2], px[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int i = 64 * hc + c0 + e + u;
              const bool on = i >= j;
              const float cl = sCl[i];
              pk[u] = on ? cl * kv[e + u] : 0.f;
              px[u] = on ? fmaf(cl, xv[e + u], sDl[i]) : 0.f;
            }
            wk[e >> 1] = pack_bf16(pk[0], pk[1]);
            wx[e >> 1] = pack_bf16(px[0], px[1]);
          }
          tc::tmem_st8(tmem + lane_base + TK_KAP + 64 * hc + c0 / 2, wk);
          tc::tmem_st8(tmem + lane_base + TK_X + 64 * hc + c0 / 2, wx);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&ms->p_full);
      }
    }
    // ---- dv rows; corner softmax backward -> dh ----
    if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->acc_full, 0, ms, err, 0x2000u));
    if (alive) {
      tc::tc_fence_after();
#pragma unroll
      for (int h2 = 0; h2 < D / 64; ++h2) {
        float v[32];
        tc::tmem_ld32(tmem + lane_base + TK_DV + (D / 2) * hc + 32 * h2, v);
        tc::tmem_wait_ld();
        // every product has read the operand tiles: dV rows are staged over them
        float4* o = reinterpret_cast<float4*>(stage_v + j * stage_pitch<D>() + (D / 2) * hc + 32 * h2);
#pragma unroll
        for (int q = 0; q < 8; ++q) o[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      }
      corner_pass(tmem, lane_base, hc, TK_DPHI, true, 0u, 0.f, valid ? 1.f : 0.f, sR1, h16, rsqrtf((float)g.L),
                  1.f / g.tau);
      tc::tmem_wait_st();
      tc::tc_fence_before();
      tc::mbar_arrive(&ms->dh_full);
    }
    uint4 xr[D / 16];
    if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->x_full, 0, ms, err, 0x40000u));
    load_x<D>(smem + k_xs<D>(), j, hc, valid && alive, xr);
    if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->du_full, 0, ms, err, 0x4000u));
    chain_pass<D>(tmem, lane_base, hc, j, TK_DU, xr, nrm, sX, stage_k, valid, alive);
    compute_bar();
    if (!*(volatile int*)&ms->abort_flag) {
      const int rows = min(kC, g.N - c * kC);
      copy_staged<D>(stage_v, a.dVacc + (head + (size_t)c * kC) * D, rows, ct, grp > 0);
      copy_staged<D>(stage_k, a.dKacc + (head + (size_t)c * kC) * D, rows, ct, grp > 0);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------- query side ------------------------------------
namespace {
constexpr uint32_t Q_DO = 0, Q_V = kTile, Q_PK = 2 * kTile, Q_PH = 3 * kTile, Q_PL = 4 * kTile;
constexpr uint32_t Q_WH = 5 * kTile, Q_WL = Q_WH + 2 * kWSlab;
constexpr uint32_t Q_P1 = Q_WL + 2 * kWSlab;            // p1 [128], exchange [256]
constexpr uint32_t Q_BARS = Q_P1 + (128 + 256) * 4;
// the Q rows of the chunk for dx, after the staged dQ rows
template <int D> constexpr uint32_t q_xs() { return (Q_DO + stage_bytes<D>() + 1023u) & ~1023u; }
static_assert(q_xs<128>() + kTile <= Q_WH && q_xs<64>() + kTile <= Q_WH,
              "the staged dQ rows and the Q tile overlap only the chunk tiles");
constexpr uint32_t TQ_X = 0, TQ_INTRA = 128, TQ_G = 256, TQ_DU = 384;
}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    race_q_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmdO, const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmPK, const __grid_constant__ CUtensorMap tmP,
                         const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                         BwdArgs a, Geom g, int grp, uint32_t* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  Bars* ms = reinterpret_cast<Bars*>(smem + Q_BARS);
  float* sP1 = reinterpret_cast<float*>(smem + Q_P1);
  float* sX = sP1 + 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x, bh = blockIdx.y;
  const size_t head = (size_t)bh * g.N;
  const bool causal = g.causal;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0 && err) atomicOr(err, 0x80000000u);
    return;
  }
  if (threadIdx.x == 0) {
    tc::mbar_init(&ms->in_main, 1);
    tc::mbar_init(&ms->s_full, 1);
    tc::mbar_init(&ms->p_full, kComputeThreads);
    tc::mbar_init(&ms->acc_full, 1);
    tc::mbar_init(&ms->dh_full, kComputeThreads);
    tc::mbar_init(&ms->du_full, 1);
    tc::mbar_init(&ms->x_full, 1);
    ms->abort_flag = 0;
    tc::fence_barrier_init();
    // the chunk's tiles do not depend on anything the set-up computes: their copies start first
    {
      // Phi(K) is [128][128]; dO, V, the statistics and W are D columns wide
      constexpr uint32_t kTD = 128u * D * 2, kWD = (uint32_t)kNH * D * 2;
      tc::mbar_arrive_expect_tx(&ms->in_main, (causal ? kTile + 2 * kTD : kTD) + 2 * kTD + 2 * kWD);
      const int z = (bh * g.n_c + t) * 2;
      if (causal)
        for (int s = 0; s < 2; ++s) tc::tma_load_3d(smem + Q_PK + s * kSlab, &tmPK, &ms->in_main, 64 * s, t * kC, bh);
      for (int s = 0; s < D / 64; ++s) {
        tc::tma_load_3d(smem + Q_DO + s * kSlab, &tmdO, &ms->in_main, 64 * s, t * kC, bh);
        if (causal) tc::tma_load_3d(smem + Q_V + s * kSlab, &tmV, &ms->in_main, 64 * s, t * kC, bh);
        tc::tma_load_3d(smem + Q_PH + s * kSlab, &tmP, &ms->in_main, 64 * s, 0, z);
        tc::tma_load_3d(smem + Q_PL + s * kSlab, &tmP, &ms->in_main, 64 * s, 0, z + 1);
        tc::tma_load_3d(smem + Q_WH + s * kWSlab, &tmW, &ms->in_main, 64 * s, kNH * grp, 0);
        tc::tma_load_3d(smem + Q_WL + s * kWSlab, &tmW, &ms->in_main, 64 * s, kNH * grp, 1);
      }
    }
  }
  if (warp == 1) {
    tc::tmem_alloc(&ms->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      constexpr uint32_t kTD = 128u * D * 2;
      tc::mbar_wait(&ms->in_main, 0);
      // the Q rows for dx, once every product but du has read the chunk tiles; waited for
      // here too, so no copy is in flight when the CTA exits
      if (wait_or_abort(&ms->acc_full, 0, ms, err, 0x10000u)) {
        tc::mbar_arrive_expect_tx(&ms->x_full, kTD);
        for (int s = 0; s < D / 64; ++s)
          tc::tma_load_3d(smem + q_xs<D>() + s * kSlab, &tmX, &ms->x_full, 64 * s, t * kC, bh);
        wait_or_abort(&ms->x_full, 0, ms, err, 0x20000u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idNN = tc::idesc_bf16(128, 128, false, false);
      const uint32_t idNM = tc::idesc_bf16(128, 128, false, true);
      const SDesc sd(smem_u32(smem));
      bool ok = wait_or_abort(&ms->in_main, 0, ms, err, 0x100u);
      if (ok && causal) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_bf16(tmem + TQ_X, sd.k(Q_DO, kk), sd.k(Q_V, kk), idNN, kk > 0 ? 1u : 0u);
        tc::mma_commit(&ms->s_full);
      }
      if (ok) {
        // inter-chunk part: G = dO P^V^T (P as bf16 hi + lo)
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t pb = part ? Q_PL : Q_PH;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tc::mma_bf16(tmem + TQ_G, sd.k(Q_DO, kk), sd.k(pb, kk), idNN, (part > 0 || kk > 0) ? 1u : 0u);
        }
      }
      if (ok && causal) {
        ok = wait_or_abort(&ms->p_full, 0, ms, err, 0x400u);
        if (ok) {
          tc::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_bf16_ts(tmem + TQ_INTRA, tmem + TQ_X + packed_col(kk), sd.kn(Q_PK, kk), idNM,
                            kk > 0 ? 1u : 0u);
        }
      }
      tc::mma_commit(&ms->acc_full);
      ok = ok && wait_or_abort(&ms->dh_full, 0, ms, err, 0x800u);
      if (ok) {
        tc::tc_fence_after();
        issue_du<D>(tmem, TQ_DU, sd, Q_WH, Q_WL);
      }
      tc::mma_commit(&ms->du_full);
      tc::mbar_wait(&ms->du_full, 0);
    }
  } else {
    const int ct = threadIdx.x - 64;
    const int q4 = warp & 3, hc = (warp - 2) >> 2;
    const int i = 32 * q4 + lane;                     // row of the tile (TMEM lane)
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const int row = t * kC + i;
    const bool valid = row < g.N;
    const float cl = valid ? a.rs.cl[head + row] : 0.f;
    const float de = valid ? a.rs.delta[head + row] : 0.f;
    float h16[16];
    load_h(valid ? a.hQ + (head + row) * 4 * g.L : nullptr, grp, hc, g.L, h16);
    const float nrm = valid ? a.nQ[head + row] : 1.f;
    if (ct < kR) sP1[ct] = a.Pmass[(((size_t)grp * g.BH + bh) * g.n_c + t) * kR + ct];
    compute_bar();
    bool alive = true;
    // ---- intra-chunk element-wise pass: dkappa_ij = cl_i X_ij + delta_i, j <= i ----
    if (causal) {
      alive = __all_sync(0xffffffffu, wait_or_abort(&ms->s_full, 0, ms, err, 0x1000u));
      if (alive) {
        tc::tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 16) {
          float xv[16];
          tc::tmem_ld16(tmem + lane_base + TQ_X + 64 * hc + c0, xv);
          tc::tmem_wait_ld();
          uint32_t wx[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const int jj = 64 * hc + c0 + e;
            const float p0 = jj <= i ? fmaf(cl, xv[e], de) : 0.f;
            const float p1 = jj + 1 <= i ? fmaf(cl, xv[e + 1], de) : 0.f;
            wx[e >> 1] = pack_bf16(p0, p1);
          }
          tc::tmem_st8(tmem + lane_base + TQ_X + 64 * hc + c0 / 2, wx);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&ms->p_full);
      }
    }
    if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->acc_full, 0, ms, err, 0x2000u));
    if (alive) {
      tc::tc_fence_after();
      corner_pass(tmem, lane_base, hc, TQ_INTRA, causal, TQ_G, cl, de, sP1, h16, rsqrtf((float)g.L),
                  1.f / g.tau);
      tc::tmem_wait_st();
      tc::tc_fence_before();
      tc::mbar_arrive(&ms->dh_full);
    }
    uint4 xr[D / 16];
    if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->x_full, 0, ms, err, 0x40000u));
    load_x<D>(smem + q_xs<D>(), i, hc, valid && alive, xr);
    if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->du_full, 0, ms, err, 0x4000u));
    // every product is done: dQ rows are staged over the operand tiles
    float* stage_q = reinterpret_cast<float*>(smem + Q_DO);
    chain_pass<D>(tmem, lane_base, hc, i, TQ_DU, xr, nrm, sX, stage_q, valid, alive);
    compute_bar();
    if (!*(volatile int*)&ms->abort_flag)
      copy_staged<D>(stage_q, a.dQacc + (head + (size_t)t * kC) * D, min(kC, g.N - t * kC), ct, grp > 0);
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------- read-out ------------------------------------
namespace {
constexpr uint32_t R_PQ = 0, R_PK = kTile, R_V = 2 * kTile, R_PH = 3 * kTile, R_PL = 4 * kTile;
constexpr uint32_t R_P1 = 5 * kTile;                    // p1 [128], exchange [256]
constexpr uint32_t R_BARS = R_P1 + (128 + 256) * 4;
constexpr uint32_t TR_KAP = 0, TR_N = 128;
}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    race_readout_tc_kernel(const __grid_constant__ CUtensorMap tmPQ, const __grid_constant__ CUtensorMap tmPK,
                           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmOlr,
                           const __grid_constant__ CUtensorMap tmP, FwdArgs a, Geom g, int grp, int mode,
                           uint32_t* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  Bars* ms = reinterpret_cast<Bars*>(smem + R_BARS);
  float* sP1 = reinterpret_cast<float*>(smem + R_P1);
  float* sX = sP1 + 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = g.n_c - 1 - blockIdx.x, bh = blockIdx.y;
  const size_t head = (size_t)bh * g.N;
  const bool causal = g.causal;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0 && err) atomicOr(err, 0x80000000u);
    return;
  }
  if (threadIdx.x == 0) {
    tc::mbar_init(&ms->in_main, 1);
    tc::mbar_init(&ms->s_full, 1);
    tc::mbar_init(&ms->p_full, kComputeThreads);
    tc::mbar_init(&ms->acc_full, 1);
    ms->abort_flag = 0;
    tc::fence_barrier_init();
    // the chunk's tiles do not depend on anything the set-up computes: their copies start first
    {
      // Phi tiles are [128][128]; V and the statistics are D columns wide
      constexpr uint32_t kTD = 128u * D * 2;
      tc::mbar_arrive_expect_tx(&ms->in_main, (causal ? 2 * kTile + kTD : kTile) + 2 * kTD);
      const int z = (bh * g.n_c + t) * 2;
      for (int s = 0; s < 2; ++s) {
        tc::tma_load_3d(smem + R_PQ + s * kSlab, &tmPQ, &ms->in_main, 64 * s, t * kC, bh);
        if (causal) tc::tma_load_3d(smem + R_PK + s * kSlab, &tmPK, &ms->in_main, 64 * s, t * kC, bh);
      }
      for (int s = 0; s < D / 64; ++s) {
        if (causal) tc::tma_load_3d(smem + R_V + s * kSlab, &tmV, &ms->in_main, 64 * s, t * kC, bh);
        tc::tma_load_3d(smem + R_PH + s * kSlab, &tmP, &ms->in_main, 64 * s, 0, z);
        tc::tma_load_3d(smem + R_PL + s * kSlab, &tmP, &ms->in_main, 64 * s, 0, z + 1);
      }
    }
  }
  if (warp == 1) {
    tc::tmem_alloc(&ms->tmem_base, 256);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      tc::mbar_wait(&ms->in_main, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idNN = tc::idesc_bf16(128, 128, false, false);
      const uint32_t idNM = tc::idesc_bf16(128, D, false, true);       // N = D, B MN-major
      const SDesc sd(smem_u32(smem));
      bool ok = wait_or_abort(&ms->in_main, 0, ms, err, 0x100u);
      if (ok && causal) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_bf16(tmem + TR_KAP, sd.k(R_PQ, kk), sd.k(R_PK, kk), idNN, kk > 0 ? 1u : 0u);
        tc::mma_commit(&ms->s_full);
      }
      if (ok) {
        // inter-chunk part: N = Phi_Q P^V (P as bf16 hi + lo)
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t pb = part ? R_PL : R_PH;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_bf16(tmem + TR_N, sd.k(R_PQ, kk), sd.kn(pb, kk), idNM,
                         (part > 0 || kk > 0) ? 1u : 0u);
        }
      }
      if (ok && causal) {
        ok = wait_or_abort(&ms->p_full, 0, ms, err, 0x400u);
        if (ok) {
          tc::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_bf16_ts(tmem + TR_N, tmem + TR_KAP + packed_col(kk), sd.kn(R_V, kk), idNM, 1u);
        }
      }
      tc::mma_commit(&ms->acc_full);
      tc::mbar_wait(&ms->acc_full, 0);
    }
  } else {
    const int ct = threadIdx.x - 64;
    const int q4 = warp & 3, hc = (warp - 2) >> 2;
    const int i = 32 * q4 + lane;                     // row of the tile (TMEM lane)
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const int row = t * kC + i;
    const bool valid = row < g.N;
    if (ct < kR) sP1[ct] = a.Pmass[(((size_t)grp * g.BH + bh) * g.n_c + t) * kR + ct];
    compute_bar();
    bool alive = true;
    float mass = 0.f;                                  // this thread's share of d_lr
    // ---- intra-chunk kappa_ij, j <= i: bf16 into tensor memory, its row sum into the mass ----
    if (causal) {
      alive = __all_sync(0xffffffffu, wait_or_abort(&ms->s_full, 0, ms, err, 0x1000u));
      if (alive) {
        tc::tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 16) {
          float kv[16];
          tc::tmem_ld16(tmem + lane_base + TR_KAP + 64 * hc + c0, kv);
          tc::tmem_wait_ld();
          uint32_t wk[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const int jj = 64 * hc + c0 + e;
            wk[e >> 1] = pack_bf16(jj <= i ? kv[e] : 0.f, jj + 1 <= i ? kv[e + 1] : 0.f);
            // the mass uses the same bf16 values the product does
            const float2 r2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wk[e >> 1]));
            mass += r2.x + r2.y;
          }
          tc::tmem_st8(tmem + lane_base + TR_KAP + 64 * hc + c0 / 2, wk);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&ms->p_full);
      }
    }
    // inter-chunk mass: Phi(q_i) . p1 over this thread's 64 features (bf16 row from shared memory)
    if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->in_main, 0, ms, err, 0x8000u));
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const uint4 v = *reinterpret_cast<const uint4*>(smem + R_PQ + sw_off(i, 64 * hc + 8 * ch, kSlab));
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        mass = fmaf(f.x, sP1[64 * hc + 8 * ch + 2 * e], mass);
        mass = fmaf(f.y, sP1[64 * hc + 8 * ch + 2 * e + 1], mass);
      }
    }
    sX[2 * i + hc] = mass;
    if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->acc_full, 0, ms, err, 0x2000u));
    compute_bar();
    // several feature groups (mode 1: the first, 2: the last) carry N and d_lr between launches
    float* num = a.lr_num ? a.lr_num + (head + min(row, g.N - 1)) * D + (D / 2) * hc : nullptr;
    float dl = sX[2 * i] + sX[2 * i + 1];
    if (mode == 2 && valid) dl += a.lr_den[head + row];
    const float il = dl > 0.f ? 1.f / dl : 0.f;
    if (alive && mode == 1) {
      tc::tc_fence_after();
#pragma unroll
      for (int h2 = 0; h2 < D / 64; ++h2) {
        float v[32];
        tc::tmem_ld32(tmem + lane_base + TR_N + (D / 2) * hc + 32 * h2, v);
        tc::tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<float4*>(num + 32 * h2)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
      if (hc == 0 && valid) a.lr_den[head + row] = dl;
    } else if (alive) {
      tc::tc_fence_after();
      // O_lr = N / d_lr as bf16, staged (swizzled) over the Phi(K) tile, then one TMA store
#pragma unroll
      for (int h2 = 0; h2 < D / 64; ++h2) {
        float v[32];
        tc::tmem_ld32(tmem + lane_base + TR_N + (D / 2) * hc + 32 * h2, v);
        tc::tmem_wait_ld();
        if (mode == 2 && valid) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 p = reinterpret_cast<const float4*>(num + 32 * h2)[q];
            v[4 * q] += p.x; v[4 * q + 1] += p.y; v[4 * q + 2] += p.z; v[4 * q + 3] += p.w;
          }
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int col = (D / 2) * hc + 32 * h2 + 8 * ch;
          *reinterpret_cast<uint4*>(smem + R_PK + sw_off(i, col, kSlab)) =
              make_uint4(pack_bf16(v[8 * ch] * il, v[8 * ch + 1] * il), pack_bf16(v[8 * ch + 2] * il, v[8 * ch + 3] * il),
                         pack_bf16(v[8 * ch + 4] * il, v[8 * ch + 5] * il), pack_bf16(v[8 * ch + 6] * il, v[8 * ch + 7] * il));
        }
      }
      if (hc == 0 && valid) a.dlr[head + row] = dl;
    }
    tc::fence_proxy_async_smem();
    compute_bar();
    if (ct == 0 && mode != 1 && !*(volatile int*)&ms->abort_flag) {
      asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];\n"
                   :: "l"(reinterpret_cast<uint64_t>(&tmOlr)), "r"(smem_u32(smem + R_PK)), "r"(0), "r"(t * kC),
                      "r"(bh) : "memory");
      if (D == 128)
        asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];\n"
                     :: "l"(reinterpret_cast<uint64_t>(&tmOlr)), "r"(smem_u32(smem + R_PK + kSlab)), "r"(64),
                        "r"(t * kC), "r"(bh) : "memory");
      asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
// Feature group grp's 128 columns of Phi ([BH][N][rp]) and its per-chunk statistics
// ([G][BH][n_c][2][128][d]).
static const void* phi_group(const void* phi, int grp) {
  return static_cast<const __nv_bfloat16*>(phi) + (size_t)grp * kR;
}
static const void* split_group(const void* split, const Geom& g, int grp) {
  return static_cast<const __nv_bfloat16*>(split) + (size_t)grp * g.BH * g.n_c * 2 * kR * g.d;
}
// [BH][N][d] rows (d = D) in boxes of 64 columns x 128 rows
static bool map_d(CUtensorMap* m, const void* base, const Geom& g) {
  return tc::map_rows_bf16_pitch(m, base, g.d, g.d, g.N, g.BH, kC);
}

template <int D>
static cudaError_t readout_t(const FwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  const size_t smem = R_BARS + sizeof(Bars);
  static_assert(R_BARS + sizeof(Bars) <= 232448, "shared memory per CTA");
  cudaError_t e = cudaFuncSetAttribute(race_readout_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  for (int grp = 0; grp < g.G; ++grp) {
    CUtensorMap mpq, mpk, mv, mo, mp;
    if (!tc::map_rows_bf16_pitch(&mpq, phi_group(a.phiQ, grp), kR, g.rp, g.N, g.BH, kC) ||
        !tc::map_rows_bf16_pitch(&mpk, phi_group(a.phiK, grp), kR, g.rp, g.N, g.BH, kC) || !map_d(&mv, a.V, g) ||
        !map_d(&mo, a.Olr, g) ||
        !tc::map_rows_bf16_pitch(&mp, split_group(a.Psplit, g, grp), D, D, kR, g.BH * g.n_c * 2, kR))
      return cudaErrorInvalidValue;
    // modes: 0 the only group; 1 the first of two (keeps N and d_lr); 2 the last (adds them)
    const int mode = g.G == 1 ? 0 : grp == 0 ? 1 : 2;
    ProfScope ps("race_readout_tc", st);
    race_readout_tc_kernel<D><<<dim3(g.n_c, g.BH), kThreads, smem, st>>>(mpq, mpk, mv, mo, mp, a, g, grp, mode, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_race_readout_tc(const FwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  if (!race_bwd_tc_supported(g) || !a.Psplit || !a.Pmass || (g.G > 1 && (!a.lr_num || !a.lr_den)))
    return cudaErrorInvalidValue;
  return g.d == 64 ? readout_t<64>(a, g, err, st) : readout_t<128>(a, g, err, st);
}

bool race_bwd_tc_supported(const Geom& g) {
  return (g.d == 64 || g.d == 128) && g.C == kC && g.r > 0 && g.r <= 2 * kR && g.r % 16 == 0 && g.rp == kR * g.G &&
         g.dp == g.d + 8;
}

template <int D>
static cudaError_t race_bwd_t(const BwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  const int NW = (4 * g.L + 31) & ~31;                 // rows of each W half (4 L padded to 32)
  CUtensorMap mv, mdo, mw, mq, mk;
  if (!map_d(&mq, a.Q, g) || !map_d(&mk, a.K, g) || !map_d(&mv, a.V, g) || !map_d(&mdo, a.dO, g) ||
      !tc::map_rows_bf16_pitch(&mw, a.Wsplit, D, D, NW, 2, kNH))
    return cudaErrorInvalidValue;
  const size_t smem_q = Q_BARS + sizeof(Bars), smem_k = K_BARS + sizeof(Bars);
  static_assert(Q_BARS + sizeof(Bars) <= 232448, "shared memory per CTA");
  static_assert(K_BARS + sizeof(Bars) <= 232448, "shared memory per CTA");
  cudaError_t e = cudaFuncSetAttribute(race_q_bwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem_q);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(race_k_bwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_k);
  if (e != cudaSuccess) return e;
  // one launch per group of 128 features (8 tables); the later groups add their parts
  for (int grp = 0; grp < g.G; ++grp) {
    CUtensorMap mpk, mpq, mp, mr;
    if (!tc::map_rows_bf16_pitch(&mpk, phi_group(a.phiK, grp), kR, g.rp, g.N, g.BH, kC) ||
        !tc::map_rows_bf16_pitch(&mpq, phi_group(a.phiQ, grp), kR, g.rp, g.N, g.BH, kC) ||
        !tc::map_rows_bf16_pitch(&mp, split_group(a.Psplit, g, grp), D, D, kR, g.BH * g.n_c * 2, kR) ||
        !tc::map_rows_bf16_pitch(&mr, split_group(a.Rsplit, g, grp), D, D, kR, g.BH * g.n_c * 2, kR))
      return cudaErrorInvalidValue;
    {
      ProfScope ps("race_q_bwd_tc", st);
      race_q_bwd_tc_kernel<D><<<dim3(g.n_c, g.BH), kThreads, smem_q, st>>>(mdo, mv, mpk, mp, mw, mq, a, g, grp, err);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    ProfScope ps("race_k_bwd_tc", st);
    race_k_bwd_tc_kernel<D><<<dim3(g.n_c, g.BH), kThreads, smem_k, st>>>(mpk, mpq, mv, mdo, mr, mw, mk, a, g, grp,
                                                                         err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_race_bwd_tc(const BwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  if (!race_bwd_tc_supported(g) || !a.hQ || !a.hK || !a.nQ || !a.nK || !a.Psplit || !a.Pmass || !a.Rsplit ||
      !a.Rmass || !a.Wsplit)
    return cudaErrorInvalidValue;
  return g.d == 64 ? race_bwd_t<64>(a, g, err, st) : race_bwd_t<128>(a, g, err, st);
}

}  // namespace elsaa
