// Sparse-branch backward on the 5th-generation tensor cores (tcgen05 + TMEM),
// 128-query tiles (or pairs of 64-query tiles), head dimension 64 or 128 (ELSAA paper
// §3.2 with the Eq. 5 adjoint folded into the softmax delta):
//   P_ij  = exp(z_ij - log d_s,i)            (z = scale q.k, j in the selected blocks)
//   dz_ij = P_ij (cs_i <dO_i, v_j> - Delta_i)
//   dq_i  = scale sum_j dz_ij k_j,  dk_j = scale sum_i dz_ij q_i,  dv_j = sum_i P_ij cs_i dO_i
// plus the low-rank gradient parts accumulated in fp32 by the RACE backward.
//
// dq kernel: one CTA per (head, query tile); Q and dO stay in shared memory, the
// selected K and V blocks stream through TMA rings (3 and 2 stages); S = Q K^T and
// dP = dO V^T land in TMEM, 8 softmax warps write dS as bf16 pairs into one of two
// TMEM buffers, and dQ += dS K (dS as the tensor-memory operand) accumulates in TMEM.
// dkdv kernel: one CTA per (head, key block); K and V stay in shared memory, the
// query tiles that selected the block (from the selection inverse) stream through a
// 2-stage ring together with their per-row scalars (a warp rewrites those as three
// arrays); S^T = K Q^T and dP^T = V dO^T land in TMEM, the softmax warps write
// (P^T cs) and dS^T back over them as bf16 in two passes of 64 queries, and
// dV += (P^T cs) dO, dK += dS^T Q accumulate in TMEM (with d = 64 in two buffers, the
// next pass's scores computed while the softmax works).
// Both: the tile loads that need no selection data start with the barrier set-up; the
// softmax arithmetic runs in packed fp32 pairs; the fp32 low-rank rows are TMA-loaded
// into buffers the products are done with, for the epilogue.  No atomics: the results
// are deterministic.
// Every mbarrier wait is bounded; a timeout sets a bit in the caller's error word,
// the CTA drains its copies and MMAs, frees TMEM and exits.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace elsaa {

namespace {

constexpr int kT = 128;
constexpr int kD = 128;
constexpr uint32_t kSlab = kT * 128;     // [128 rows][64 bf16], 128-byte swizzle
constexpr uint32_t kTile = 2 * kSlab;    // [128 rows][128 bf16]
constexpr int kSoftmaxThreads = 256;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];\n"
               :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2) : "memory");
}
__device__ __forceinline__ void tma_store_wait() {
  asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
  asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
}

// ------------------------------- dq ----------------------------------------
constexpr uint32_t DQ_Q = 0, DQ_DO = kTile;
constexpr int kDqKStages = 3, kDqVStages = 2;
__host__ __device__ constexpr uint32_t dq_k(int s) { return kTile * (2 + s); }                 // K ring
__host__ __device__ constexpr uint32_t dq_v(int s) { return kTile * (2 + kDqKStages + s); }    // V ring
constexpr uint32_t DQ_MISC = kTile * (2 + kDqKStages + kDqVStages);
// TMEM: S and dP (fp32), the dQ accumulator, dS (bf16 pairs) double-buffered
constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DQ = 256, TM_DS = 384;
constexpr int kDqThreads = 352;          // Q/dO + K producer, MMA, 8 softmax warps, V producer
constexpr uint32_t kAccBox = 128 * 128;  // [128 rows][32 fp32] box of the low-rank dQ tile

struct DqMisc {
  uint64_t qd_full, k_full[kDqKStages], k_empty[kDqKStages], v_full[kDqVStages], v_empty[kDqVStages], s_full,
      st_free, ds_full[2], done, acc_full;
  uint32_t tmem_base;
  int abort_flag;
  int idx[2][32];         // selected blocks of the CTA's tile (PAIR: of its two tiles)
};

template <typename M>
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, M* ms, uint32_t* err, uint32_t code) {
  if (*(volatile int*)&ms->abort_flag) return false;
  if (tc::mbar_wait(bar, parity)) return true;
  *(volatile int*)&ms->abort_flag = 1;
  if (err) atomicOr(err, code);
  return false;
}

// dS = P (cs dP - Delta) for one thread's 64 keys of a query row, as bf16 pairs;
// MASK: keys after column `lim` get P = 0.
// Pairs of columns go through packed fp32 lanes (one f32x2 instruction per pair and step).
template <bool MASK>
__device__ __forceinline__ void dq_softmax_cols(const float (&sv)[64], const float (&dp)[64], float sl2, float lg2,
                                                float cs, float Dl, int lim, uint32_t (&w)[32]) {
  const uint64_t sl2x2 = tc::f2_pack(sl2, sl2), neg_lg2 = tc::f2_pack(-lg2, -lg2);
  const uint64_t cs2 = tc::f2_pack(cs, cs), neg_dl = tc::f2_pack(-Dl, -Dl);
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    float x0, x1;
    tc::f2_unpack(tc::f2_fma(tc::f2_pack(sv[c], sv[c + 1]), sl2x2, neg_lg2), x0, x1);
    float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
    if (MASK) {
      p0 = c > lim ? 0.f : p0;
      p1 = c + 1 > lim ? 0.f : p1;
    }
    float d0, d1;
    tc::f2_unpack(tc::f2_mul(tc::f2_pack(p0, p1), tc::f2_fma(cs2, tc::f2_pack(dp[c], dp[c + 1]), neg_dl)), d0, d1);
    w[c >> 1] = pack_bf16(d0, d1);
  }
}

}  // namespace

// D = 64 or 128.  PAIR (blocks of 64): the CTA's 128 query rows are the tiles 2u and 2u + 1,
// and the K / V stage of step j holds tile 2u's j-th block in rows 0-63 and tile 2u + 1's in
// rows 64-127; each query row masks the other tile's 64 keys (dS = 0 there).
template <int D, bool PAIR>
__global__ void __launch_bounds__(kDqThreads, 1)
    dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                 const __grid_constant__ CUtensorMap tmdQ, const __grid_constant__ CUtensorMap tmAcc, BwdArgs a,
                 Geom g, uint32_t* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  DqMisc* ms = reinterpret_cast<DqMisc*>(smem + DQ_MISC);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  constexpr int TB = PAIR ? 64 : 128;       // keys per block = queries per tile
  constexpr int H = D / 2;                  // dQ columns per thread (half a row)
  const int n_units = PAIR ? (g.n_t + 1) / 2 : g.n_t;
  const int unit = a.tile_list ? (PAIR ? a.tile_list[(size_t)bh * a.n_list + 2 * blockIdx.x] / 2
                                       : a.tile_list[(size_t)bh * a.n_list + blockIdx.x])
                               : n_units - 1 - (int)blockIdx.x;
  const int ta = PAIR ? 2 * unit : unit, tb = PAIR ? 2 * unit + 1 : unit;
  const int row0 = kT * unit;
  const size_t head = (size_t)bh * g.N;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0 && err) atomicOr(err, 0x80000000u);
    return;
  }
  const int* idx_a = a.idx + ((size_t)bh * g.n_t + ta) * g.k;
  const int* idx_b = a.idx + ((size_t)bh * g.n_t + tb) * g.k;
  if (threadIdx.x == 0) {
    tc::mbar_init(&ms->qd_full, 1);
    for (int s = 0; s < kDqKStages; ++s) {
      tc::mbar_init(&ms->k_full[s], 1);
      tc::mbar_init(&ms->k_empty[s], 1);
    }
    for (int s = 0; s < kDqVStages; ++s) {
      tc::mbar_init(&ms->v_full[s], 1);
      tc::mbar_init(&ms->v_empty[s], 1);
    }
    tc::mbar_init(&ms->s_full, 1);
    tc::mbar_init(&ms->st_free, kSoftmaxThreads);
    tc::mbar_init(&ms->ds_full[0], kSoftmaxThreads);
    tc::mbar_init(&ms->ds_full[1], kSoftmaxThreads);
    tc::mbar_init(&ms->done, 1);
    tc::mbar_init(&ms->acc_full, 1);
    ms->abort_flag = 0;
    tc::fence_barrier_init();
    // Q and dO do not depend on the selection: their copies start before anything else
    tc::mbar_arrive_expect_tx(&ms->qd_full, 2 * 128u * D * 2);
    for (int sl = 0; sl < D / 64; ++sl) {
      tc::tma_load_3d(smem + DQ_Q + sl * kSlab, &tmQ, &ms->qd_full, 64 * sl, row0, bh);
      tc::tma_load_3d(smem + DQ_DO + sl * kSlab, &tmdO, &ms->qd_full, 64 * sl, row0, bh);
    }
    // so do the first selected block's K and V (its index is the first of the tile's list):
    // the producers start at the second block
    const int b0[2] = {g.k > 0 ? idx_a[0] : -1, PAIR && tb < g.n_t && g.k > 0 ? idx_b[0] : -1};
    if (b0[0] >= 0 || b0[1] >= 0) {
      for (int kv = 0; kv < 2; ++kv) {
        uint64_t* full = kv ? &ms->v_full[0] : &ms->k_full[0];
        tc::mbar_arrive_expect_tx(full, 128u * D * 2);
        for (int h = 0; h < (PAIR ? 2 : 1); ++h)
          for (int sl = 0; sl < D / 64; ++sl)
            tc::tma_load_3d(smem + (kv ? dq_v(0) : dq_k(0)) + sl * kSlab + h * 64 * 128, kv ? &tmV : &tmK, full,
                            64 * sl, (b0[h] >= 0 ? b0[h] : 0) * TB, bh);
      }
    }
  }
  if (threadIdx.x < 32) {
    ms->idx[0][threadIdx.x] = threadIdx.x < g.k ? idx_a[threadIdx.x] : -1;
    ms->idx[1][threadIdx.x] = PAIR && tb < g.n_t && threadIdx.x < g.k ? idx_b[threadIdx.x] : -1;
  }
  if (warp == 1) {
    tc::tmem_alloc(&ms->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  // block j of tile half h: the first 32 from shared memory, any further ones from global memory
  auto sel = [&](int h, int j) -> int { return j < 32 ? ms->idx[h][j] : (h ? idx_b : idx_a)[j]; };
  int n_sel_a = 0, n_sel_b = 0;
  while (n_sel_a < g.k && sel(0, n_sel_a) >= 0) ++n_sel_a;
  while (PAIR && tb < g.n_t && n_sel_b < g.k && sel(1, n_sel_b) >= 0) ++n_sel_b;
  const int n_sel = max(n_sel_a, n_sel_b);          // steps

  if (warp == 0 || warp == 10) {
    // ---------------- TMA producers: warp 0 Q, dO and the K ring; warp 10 the V ring ----------------
    if (lane == 0) {
      const bool kside = warp == 0;
      const int NS = kside ? kDqKStages : kDqVStages;
      uint64_t* full = kside ? ms->k_full : ms->v_full;
      uint64_t* empty = kside ? ms->k_empty : ms->v_empty;
      constexpr uint32_t kTD = 128u * D * 2;      // bytes of a [128][D] tile
      int issued = n_sel > 0 ? 1 : 0;             // block 0 was issued with the barriers
      for (int j = issued; j < n_sel; ++j) {
        const int s = j % NS;
        if (j >= NS && !wait_or_abort(&empty[s], ((j / NS) - 1) & 1, ms, err, kside ? 1u : 2u)) break;
        unsigned char* dst = smem + (kside ? dq_k(s) : dq_v(s));
        tc::mbar_arrive_expect_tx(&full[s], kTD);
        for (int h = 0; h < (PAIR ? 2 : 1); ++h) {
          // PAIR: a tile with fewer blocks stages block 0 in its half (every score of it is masked)
          const int b = j < (h ? n_sel_b : n_sel_a) ? sel(h, j) : 0;
          for (int sl = 0; sl < D / 64; ++sl)
            tc::tma_load_3d(dst + sl * kSlab + h * 64 * 128, kside ? &tmK : &tmV, &full[s], 64 * sl, b * TB, bh);
        }
        issued = j + 1;
      }
      // the V ring is free once the last dP products are done: the tile's low-rank dQ rows
      // (fp32, 32-column boxes, 128-byte swizzle) go there for the epilogue
      bool acc_issued = false;
      if (!kside && a.dQacc && issued == n_sel) {
        bool free_ring = true;
        for (int j = (n_sel > NS ? n_sel - NS : 0); free_ring && j < n_sel; ++j)
          free_ring = wait_or_abort(&empty[j % NS], (j / NS) & 1, ms, err, 2u);
        if (free_ring) {
          tc::mbar_arrive_expect_tx(&ms->acc_full, 128u * D * 4);
          for (int b = 0; b < D / 32; ++b)
            tc::tma_load_3d(smem + dq_v(0) + b * kAccBox, &tmAcc, &ms->acc_full, 32 * b, row0, bh);
          acc_issued = true;
        }
      }
      if (kside) tc::mbar_wait(&ms->qd_full, 0);
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j) tc::mbar_wait(&full[j % NS], (j / NS) & 1);
      if (acc_issued) tc::mbar_wait(&ms->acc_full, 0);   // no copy in flight when the CTA exits
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idNN = tc::idesc_bf16(128, 128, false, false);   // both operands K-major
      const uint32_t idNM = tc::idesc_bf16(128, D, false, true);      // B MN-major, N = D
      const uint32_t sb = smem_u32(smem);
      // operand descriptors built once; a K step or a ring stage only moves the start address
      const uint64_t q_desc = tc::sw128_desc(sb + DQ_Q, 16, 1024), do_desc = tc::sw128_desc(sb + DQ_DO, 16, 1024);
      const uint64_t k_desc = tc::sw128_desc(sb + dq_k(0), 16, 1024), v_desc = tc::sw128_desc(sb + dq_v(0), 16, 1024);
      const uint64_t kmn_desc = tc::sw128_desc(sb + dq_k(0), kSlab, 1024);    // K as the MN-major B of dS K
      bool ok = wait_or_abort(&ms->qd_full, 0, ms, err, 4u);
      int dq_issued = 0;
      // dQ += dS K: dS (bf16 pairs, TMEM buffer jj & 1) is the A operand
      auto issue_dq = [&](int jj) -> bool {
        if (!wait_or_abort(&ms->ds_full[jj & 1], (jj >> 1) & 1, ms, err, 8u)) return false;
        tc::tc_fence_after();
        const int st = jj % kDqKStages;
        const uint64_t kb = tc::desc_adv(kmn_desc, (uint32_t)st * kTile);
        const uint32_t ds = tmem + TM_DS + 64u * (jj & 1);
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk)
          tc::mma_bf16_ts(tmem + TM_DQ, ds + 8u * kk, tc::desc_adv(kb, kk * 2048), idNM, (jj > 0 || kk > 0) ? 1u : 0u);
        tc::mma_commit(&ms->k_empty[st]);
        dq_issued = jj + 1;
        return true;
      };
      for (int j = 0; ok && j < n_sel; ++j) {
        const int sv = j % kDqVStages, sk = j % kDqKStages;
        if (!wait_or_abort(&ms->v_full[sv], (j / kDqVStages) & 1, ms, err, 16u)) break;
        if (j >= 1 && !wait_or_abort(&ms->st_free, (j - 1) & 1, ms, err, 32u)) break;
        tc::tc_fence_after();
        const uint64_t vb = tc::desc_adv(v_desc, (uint32_t)sv * kTile);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSlab + (kk & 3) * 32;
          tc::mma_bf16(tmem + TM_DP, tc::desc_adv(do_desc, off), tc::desc_adv(vb, off), idNN, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&ms->v_empty[sv]);              // V slot free once dP is done
        if (!wait_or_abort(&ms->k_full[sk], (j / kDqKStages) & 1, ms, err, 64u)) break;
        tc::tc_fence_after();
        const uint64_t kb = tc::desc_adv(k_desc, (uint32_t)sk * kTile);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSlab + (kk & 3) * 32;
          tc::mma_bf16(tmem + TM_S, tc::desc_adv(q_desc, off), tc::desc_adv(kb, off), idNN, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&ms->s_full);
        if (j >= 1 && !issue_dq(j - 1)) break;
      }
      if (n_sel > 0 && dq_issued == n_sel - 1) issue_dq(n_sel - 1);
      tc::mma_commit(&ms->done);
      tc::mbar_wait(&ms->done, 0);
    }
  } else {
    // ---------------- softmax: half a query row per thread ----------------
    const int q4 = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = 32 * q4 + lane;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const int qrow = row0 + row;
    const bool row_ok = qrow < g.N;
    // PAIR: rows 0-63 belong to tile ta and key columns 0-63, rows 64-127 to tile tb and
    // columns 64-127; a thread whose half holds the other tile's keys masks all of them
    const int mine = PAIR ? (row >= 64) : 0;
    const int my_tile = PAIR ? (mine ? tb : ta) : ta;
    const int my_n = mine ? n_sel_b : n_sel_a;
    const bool dead_half = PAIR && half != mine;
    const int qpos = PAIR ? (row & 63) : row;        // query position within its tile
    const float4 sc = row_ok ? a.rs.packed[head + qrow] : make_float4(INFINITY, 0.f, 0.f, 0.f);
    const float lg2 = sc.x, cs = sc.y, Dl = sc.z;
    const float sl2 = g.scale * kLog2e;
    bool alive = true;
    for (int j = 0; j < n_sel && alive; ++j) {
      float sv[64], dp[64];
      alive = __all_sync(0xffffffffu, wait_or_abort(&ms->s_full, j & 1, ms, err, 128u));
      if (!alive) break;
      tc::tc_fence_after();
      tc::tmem_ld32(tmem + lane_base + TM_S + 64 * half, *reinterpret_cast<float(*)[32]>(sv));
      tc::tmem_ld32(tmem + lane_base + TM_S + 64 * half + 32, *reinterpret_cast<float(*)[32]>(sv + 32));
      tc::tmem_ld32(tmem + lane_base + TM_DP + 64 * half, *reinterpret_cast<float(*)[32]>(dp));
      tc::tmem_ld32(tmem + lane_base + TM_DP + 64 * half + 32, *reinterpret_cast<float(*)[32]>(dp + 32));
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      tc::mbar_arrive(&ms->st_free);
      // key k of this half's 64 columns is key c0 + k of block b (no block: all masked)
      const bool none = dead_half || j >= my_n;
      const int b = none ? 0 : sel(PAIR ? half : 0, j);
      const int c0 = PAIR ? 0 : 64 * half;
      const int kvalid = g.N - b * TB;
      const bool diag = g.causal && b == my_tile;
      const bool mask = none || diag || kvalid < TB;
      const int lim = none ? -1 : min(kvalid - 1, diag ? qpos : TB - 1) - c0;
      uint32_t w[32];
      // block-uniform: only the diagonal block and a ragged last block need the mask
      if (mask)
        dq_softmax_cols<true>(sv, dp, sl2, lg2, cs, Dl, lim, w);
      else
        dq_softmax_cols<false>(sv, dp, sl2, lg2, cs, Dl, lim, w);
      // dS (keys 64 half .. 64 half + 63 of this row) into TMEM buffer j & 1; the product that
      // read this buffer (block j - 2) finished before S_j was computed
      const uint32_t dcol = TM_DS + 64u * (j & 1) + 32u * half;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t w8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w8[e] = w[8 * q + e];
        tc::tmem_st8(tmem + lane_base + dcol + 8 * q, w8);
      }
      tc::tmem_wait_st();
      tc::tc_fence_before();
      tc::mbar_arrive(&ms->ds_full[j & 1]);
    }
    // ---------------- epilogue: dQ = scale dQ_sparse + dQ_lowrank, bf16 TMA store ----------------
    const int col0 = H * half;                       // this thread's dQ columns [col0, col0 + H)
    bool have = false;
    if (alive && n_sel > 0) {
      alive = __all_sync(0xffffffffu, wait_or_abort(&ms->done, 0, ms, err, 256u));
      have = alive;
      if (have) tc::tc_fence_after();
    }
    // the low-rank part, brought into the V ring by the V producer
    if (alive && a.dQacc) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->acc_full, 0, ms, err, 512u));
    const bool use_acc = alive && row_ok && a.dQacc;
    // fp32 element (row, c) of the low-rank tile: box c / 32, 16-byte chunk (c % 32) / 4 swizzled by row
    auto acc4 = [&](int c) -> float4 {
      return *reinterpret_cast<const float4*>(smem + dq_v(0) + (uint32_t)(c >> 5) * kAccBox + (uint32_t)row * 128u +
                                              ((uint32_t)(((c & 31) >> 2) ^ (row & 7)) << 4));
    };
    // every product has completed: stage the bf16 tile in the Q buffer, 32 columns at a time
    // (with a row map, write each row straight to the caller's row instead)
    unsigned char* orow = smem + DQ_Q + (col0 >> 6) * kSlab + row * 128;
    const int ch0 = (col0 & 63) >> 3;
    uint4* grow = a.q_rows && row_ok && alive
                      ? reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.dQ) +
                                                 (head + a.q_rows[(size_t)bh * a.rows_stride + qrow]) * D + col0)
                      : nullptr;
#pragma unroll
    for (int c = 0; c < H / 32; ++c) {
      float o[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = 0.f;
      if (have) {
        tc::tmem_ld32(tmem + lane_base + TM_DQ + col0 + 32 * c, o);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= g.scale;
      }
      if (use_acc) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = acc4(col0 + 32 * c + 4 * q);
          o[4 * q] += v.x; o[4 * q + 1] += v.y; o[4 * q + 2] += v.z; o[4 * q + 3] += v.w;
        }
      }
      if (a.out_f32) {                                   // fp32 rows (level slots), no staging
        if (alive && row_ok) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.dQ) + (head + qrow) * D + col0 + 32 * c);
#pragma unroll
          for (int q = 0; q < 8; ++q) dst[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        }
        continue;
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int ch = 4 * c + cc;
        const uint4 val = make_uint4(pack_bf16(o[8 * cc], o[8 * cc + 1]), pack_bf16(o[8 * cc + 2], o[8 * cc + 3]),
                                     pack_bf16(o[8 * cc + 4], o[8 * cc + 5]), pack_bf16(o[8 * cc + 6], o[8 * cc + 7]));
        if (a.q_rows) {
          if (grow) grow[ch] = val;
        } else {
          *reinterpret_cast<uint4*>(orow + (((ch0 + ch) ^ (row & 7)) << 4)) = val;
        }
      }
    }
    if (!a.q_rows && !a.out_f32) {
      tc::fence_proxy_async_smem();
      softmax_bar();
      if (threadIdx.x == 64 && !*(volatile int*)&ms->abort_flag) {
        for (int sl = 0; sl < D / 64; ++sl) tma_store_3d(&tmdQ, smem + DQ_Q + sl * kSlab, 64 * sl, row0, bh);
        tma_store_wait();
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}


// ------------------------------- dkdv ------------------------------------------
namespace {
constexpr int kStages = 2;
constexpr uint32_t KV_K = 0, KV_V = kTile;
__host__ __device__ constexpr uint32_t kv_q(int s) { return 2 * kTile + s * 2 * kTile; }   // Q tile, stage s
__host__ __device__ constexpr uint32_t kv_do(int s) { return kv_q(s) + kTile; }            // dO tile, stage s
constexpr uint32_t KV_SC = 2 * kTile + kStages * 2 * kTile;                   // scalars [stage][128] float4
constexpr int kMaxUnits = 1024;
// the scalars as three arrays per stage (-log2 d_s, cs, -Delta), for 8-byte column-pair loads
constexpr uint32_t KV_SOA = KV_SC + kStages * 128 * 16;
constexpr uint32_t KV_UNITS = KV_SOA + kStages * 3 * 128 * 4;                 // query tiles of the block(s)
constexpr uint32_t KV_MISC = KV_UNITS + 2 * kMaxUnits * 4;
// TMEM columns 0-255 hold S^T [keys][queries] and dP^T (fp32) for the 128 queries of a tile,
// taken as two passes of 64 queries.  d = 128: S^T in columns 0-127 and dP^T in 128-255, both
// products at N = 128 once per tile.  d = 64 (products half as long, so the softmax warps
// dominate): two buffers of one pass each (columns 128 h: S^T, then dP^T 64 further), the
// products at N = 64 per pass, so the next pass's scores are computed while the softmax warps
// work on this one.  Once read, (P^T cs) and dS^T (bf16 pairs) overwrite the first 8 of every
// 16 columns and feed dV / dK as the tensor-memory A operand.
constexpr uint32_t TM_DV = 256, TM_DK = 384;
template <int D> struct KvTmem {
  static constexpr bool kTwoBuf = D == 64;
  static constexpr uint32_t kDp = kTwoBuf ? 64 : 128;             // dP^T columns after S^T
  __host__ __device__ static constexpr uint32_t st(int pass) { return (kTwoBuf ? 128u : 64u) * pass; }
};
constexpr int kKvThreads = 352;          // TMA producer, MMA, 8 softmax warps, scalar transposer

struct KvMisc {
  uint64_t kv_full, qd_full[kStages], qd_empty[kStages], s_full[2], p_half[2], done;
  uint64_t kv_read, st1_read, acck_full, accv_full;   // K / V and stage 1 free; low-rank rows landed
  uint64_t sc_ready[kStages];                          // the stage's scalars transposed
  uint32_t tmem_base;
  int abort_flag;
};

// One thread's 32 queries (columns q0 .. q0 + 31 of the unit) for its key row: S^T and dP^T
// (fp32, TMEM) -> (P^T cs) and dS^T as bf16 pairs in the first 8 of each 16 columns read.
// nx, cs, nd: -log2 d_s, cs and -Delta of those queries; pairs of columns go through packed
// fp32 lanes.  MASK: queries outside [lo, hi) (relative to q0) get P = 0.
template <bool MASK>
__device__ __forceinline__ void dkdv_softmax_cols(uint32_t tmem, uint32_t st_col, uint32_t dp_col, const float* nx,
                                                  const float* cs, const float* nd, float sl2, int lo, int hi) {
  const uint64_t sl2x2 = tc::f2_pack(sl2, sl2);
#pragma unroll
  for (int c0 = 0; c0 < 32; c0 += 16) {
    float sv[16], dp[16];
    tc::tmem_ld16(tmem + st_col + c0, sv);
    tc::tmem_ld16(tmem + dp_col + c0, dp);
    tc::tmem_wait_ld();
    uint32_t wp[8], wd[8];
#pragma unroll
    for (int c = 0; c < 16; c += 2) {
      const int q = c0 + c;
      const uint64_t x2 = *reinterpret_cast<const uint64_t*>(nx + q);
      const uint64_t y2 = *reinterpret_cast<const uint64_t*>(cs + q);
      const uint64_t z2 = *reinterpret_cast<const uint64_t*>(nd + q);
      float e0, e1;
      tc::f2_unpack(tc::f2_fma(tc::f2_pack(sv[c], sv[c + 1]), sl2x2, x2), e0, e1);
      float p0 = ex2_approx(e0), p1 = ex2_approx(e1);
      if (MASK) {
        if (q < lo || q >= hi) p0 = 0.f;
        if (q + 1 < lo || q + 1 >= hi) p1 = 0.f;
      }
      const uint64_t p2 = tc::f2_pack(p0, p1);
      float a0, a1, b0, b1;
      tc::f2_unpack(tc::f2_mul(p2, y2), a0, a1);
      tc::f2_unpack(tc::f2_mul(p2, tc::f2_fma(y2, tc::f2_pack(dp[c], dp[c + 1]), z2)), b0, b1);
      wp[c >> 1] = pack_bf16(a0, a1);
      wd[c >> 1] = pack_bf16(b0, b1);
    }
    tc::tmem_st8(tmem + st_col + c0, wp);
    tc::tmem_st8(tmem + dp_col + c0, wd);
  }
}
}  // namespace

// One CTA per (head, key block b): K_b and V_b stay in shared memory; the query tiles that
// selected b (ascending, from the selection inverse) stream through a 2-stage ring with
// their per-row scalars.  Per tile: S^T = K Q^T and dP^T = V dO^T into TMEM; the softmax
// warps turn them into (P^T cs) and dS^T in two passes of 64 queries, and after each pass
// dV += (P^T cs) dO and dK += dS^T Q over those 64 queries run on the tensor cores while the
// other pass is computed.  With d = 64 the scores are computed per pass into two buffers, so
// the next pass's scores also overlap the softmax work.
// D = 64 or 128.  PAIR (blocks of 64): the CTA's 128 key rows are blocks 2c (rows 0-63) and
// 2c + 1 (rows 64-127); unit u stages the u-th query tile of block 2c in query rows 0-63 and
// the u-th of block 2c + 1 in rows 64-127, and each key row masks the other block's queries.
template <int D, bool PAIR>
__global__ void __launch_bounds__(kKvThreads, 1)
    dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                   const __grid_constant__ CUtensorMap tmSc, const __grid_constant__ CUtensorMap tmdK,
                   const __grid_constant__ CUtensorMap tmdV, const __grid_constant__ CUtensorMap tmKacc,
                   const __grid_constant__ CUtensorMap tmVacc, BwdArgs a, Geom g, uint32_t* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  KvMisc* ms = reinterpret_cast<KvMisc*>(smem + KV_MISC);
  int* units = reinterpret_cast<int*>(smem + KV_UNITS);       // [2][kMaxUnits] query tiles of the block(s)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  constexpr int TB = PAIR ? 64 : 128;       // keys per block = queries per tile
  constexpr int H = D / 2;                  // dK / dV columns per thread (half a row)
  // heaviest key blocks of every head first (order from the selection inverse); PAIR: the
  // CTA takes entries 2y and 2y + 1 of that order, two blocks with about as many query tiles
  // (pb[1] = -1 past the last block)
  const int nb = a.n_kv ? a.n_kv : g.n_t;
  const int* kvo = a.kv_order ? a.kv_order + (size_t)bh * g.n_t : nullptr;
  const int y = blockIdx.y;
  const int b = PAIR ? (kvo ? kvo[2 * y] : 2 * y) : (kvo ? kvo[y] : y);
  const int pb[2] = {b, PAIR ? (2 * y + 1 < nb ? (kvo ? kvo[2 * y + 1] : 2 * y + 1) : -1) : b};
  const int key0 = kT * b;                   // first key row of the CTA (not PAIR)
  const size_t head = (size_t)bh * g.N;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0 && err) atomicOr(err, 0x80000000u);
    return;
  }
  if (threadIdx.x == 0) {
    tc::mbar_init(&ms->kv_full, 1);
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&ms->qd_full[s], 1);
      tc::mbar_init(&ms->qd_empty[s], 1);
    }
    tc::mbar_init(&ms->s_full[0], 1);
    tc::mbar_init(&ms->s_full[1], 1);
    tc::mbar_init(&ms->kv_read, 1);
    tc::mbar_init(&ms->st1_read, 1);
    tc::mbar_init(&ms->acck_full, 1);
    tc::mbar_init(&ms->accv_full, 1);
    for (int st = 0; st < kStages; ++st) tc::mbar_init(&ms->sc_ready[st], 1);
    tc::mbar_init(&ms->p_half[0], kSoftmaxThreads);
    tc::mbar_init(&ms->p_half[1], kSoftmaxThreads);
    tc::mbar_init(&ms->done, 1);
    ms->abort_flag = 0;
    tc::fence_barrier_init();
    // K and V of the block(s) do not depend on the query tiles: their copies start first
    constexpr uint32_t kTD = 128u * D * 2;
    tc::mbar_arrive_expect_tx(&ms->kv_full, 2 * kTD);
    // PAIR: block pb[0] in key rows 0-63, pb[1] in rows 64-127 (a missing one stages pb[0])
    for (int h = 0; h < (PAIR ? 2 : 1); ++h) {
      const int kr = PAIR ? 64 * (pb[h] >= 0 ? pb[h] : pb[0]) : key0;
      for (int sl = 0; sl < D / 64; ++sl) {
        tc::tma_load_3d(smem + KV_K + sl * kSlab + h * 64 * 128, &tmK, &ms->kv_full, 64 * sl, kr, bh);
        tc::tma_load_3d(smem + KV_V + sl * kSlab + h * 64 * 128, &tmV, &ms->kv_full, 64 * sl, kr, bh);
      }
    }
    // so do the first query tile's Q, dO and scalars (the first entries of the block(s)' tile
    // lists): the producer starts at the second tile
    if (g.k > 0) {
      const int* of = a.offs + (size_t)bh * (g.n_t + 1);
      const int* list = a.tiles + (size_t)bh * g.n_t * g.k;
      int t0[2] = {-1, -1};
      for (int h = 0; h < (PAIR ? 2 : 1); ++h) {
        if (pb[h] < 0) break;
        const int e0 = of[pb[h]];
        if (of[pb[h] + 1] > e0) t0[h] = list[e0];
      }
      if (t0[0] >= 0 || t0[1] >= 0) {
        tc::mbar_arrive_expect_tx(&ms->qd_full[0], 2 * kTD + 128 * 16);
        for (int h = 0; h < (PAIR ? 2 : 1); ++h) {
          const int qr = (t0[h] >= 0 ? t0[h] : 0) * TB;
          for (int sl = 0; sl < D / 64; ++sl) {
            tc::tma_load_3d(smem + kv_q(0) + sl * kSlab + h * 64 * 128, &tmQ, &ms->qd_full[0], 64 * sl, qr, bh);
            tc::tma_load_3d(smem + kv_do(0) + sl * kSlab + h * 64 * 128, &tmdO, &ms->qd_full[0], 64 * sl, qr, bh);
          }
          tc::tma_load_3d(smem + KV_SC + h * 64 * 16, &tmSc, &ms->qd_full[0], 0, qr, bh);
        }
      }
    }
  }
  int n_ut[2] = {0, 0};
  if (g.k > 0) {
    const int* of = a.offs + (size_t)bh * (g.n_t + 1);
    const int* list = a.tiles + (size_t)bh * g.n_t * g.k;
    for (int h = 0; h < (PAIR ? 2 : 1); ++h) {
      const int bb = pb[h];
      if (bb < 0) break;
      const int e0 = of[bb];
      n_ut[h] = min(of[bb + 1] - e0, kMaxUnits);
      for (int i = threadIdx.x; i < n_ut[h]; i += kKvThreads) units[h * kMaxUnits + i] = list[e0 + i];
    }
  }
  const int n_ua = n_ut[0], n_ub = n_ut[1];
  const int n_u = max(n_ua, n_ub);
  const int last1 = n_u >= 2 ? ((n_u - 1) & 1 ? n_u - 1 : n_u - 2) : -1;   // last tile staged in stage 1

  if (warp == 1) {
    tc::tmem_alloc(&ms->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      constexpr uint32_t kTD = 128u * D * 2;      // bytes of a [128][D] tile
      int issued = n_u > 0 ? 1 : 0;               // tile 0 was issued with the barriers
      for (int u = issued; u < n_u; ++u) {
        const int s = u % kStages;
        if (u >= kStages && !wait_or_abort(&ms->qd_empty[s], ((u / kStages) - 1) & 1, ms, err, 1u)) break;
        tc::mbar_arrive_expect_tx(&ms->qd_full[s], 2 * kTD + 128 * 16);
        for (int h = 0; h < (PAIR ? 2 : 1); ++h) {
          // PAIR: a block with fewer query tiles stages tile 0 in its half (all of it is masked)
          const int t = u < (h ? n_ub : n_ua) ? units[h * kMaxUnits + u] : 0;
          const int qr = t * TB;
          for (int sl = 0; sl < D / 64; ++sl) {
            tc::tma_load_3d(smem + kv_q(s) + sl * kSlab + h * 64 * 128, &tmQ, &ms->qd_full[s], 64 * sl, qr, bh);
            tc::tma_load_3d(smem + kv_do(s) + sl * kSlab + h * 64 * 128, &tmdO, &ms->qd_full[s], 64 * sl, qr, bh);
          }
          tc::tma_load_3d(smem + KV_SC + s * 128 * 16 + h * 64 * 16, &tmSc, &ms->qd_full[s], 0, qr, bh);
        }
        issued = u + 1;
      }
      // the block's fp32 low-rank rows for the epilogue (32-column boxes, 128-byte swizzle): dV's
      // into stage 1 once no tile reads it, dK's into the K / V tiles once the last scores are done
      bool accv = false, acck = false;
      auto load_acc = [&](const CUtensorMap* map, uint64_t* bar, uint32_t dst) {
        const int nh = PAIR ? (pb[1] >= 0 ? 2 : 1) : 1;
        tc::mbar_arrive_expect_tx(bar, (uint32_t)(D / 32) * nh * TB * 128u);
        for (int b = 0; b < D / 32; ++b)
          for (int h = 0; h < nh; ++h)
            tc::tma_load_3d(smem + dst + b * kAccBox + h * 64 * 128, map, bar, 32 * b, PAIR ? 64 * pb[h] : key0, bh);
      };
      if (issued == n_u && a.dVacc && (last1 < 0 || wait_or_abort(&ms->st1_read, 0, ms, err, 1u))) {
        load_acc(&tmVacc, &ms->accv_full, kv_q(1));
        accv = true;
      }
      // (with no tile, the K / V copies must have landed before their space is reused)
      if (issued == n_u && a.dKacc &&
          (n_u == 0 ? wait_or_abort(&ms->kv_full, 0, ms, err, 1u) : wait_or_abort(&ms->kv_read, 0, ms, err, 1u))) {
        load_acc(&tmKacc, &ms->acck_full, KV_K);
        acck = true;
      }
      tc::mbar_wait(&ms->kv_full, 0);
      for (int u = (issued > kStages ? issued - kStages : 0); u < issued; ++u)
        tc::mbar_wait(&ms->qd_full[u % kStages], (u / kStages) & 1);
      if (accv) tc::mbar_wait(&ms->accv_full, 0);      // no copy in flight when the CTA exits
      if (acck) tc::mbar_wait(&ms->acck_full, 0);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      using TL = KvTmem<D>;
      constexpr int NQ = TL::kTwoBuf ? 64 : 128;                       // queries per score product
      const uint32_t idS = tc::idesc_bf16(128, NQ, false, false);     // K (keys x d) x Q (queries x d)
      const uint32_t idG = tc::idesc_bf16(128, D, false, true);       // P^T / dS^T (TMEM) x (dO / Q, MN-major)
      const uint32_t sb = smem_u32(smem);
      // operand descriptors built once; a K step or a ring stage only moves the start address
      const uint64_t k_desc = tc::sw128_desc(sb + KV_K, 16, 1024), v_desc = tc::sw128_desc(sb + KV_V, 16, 1024);
      const uint64_t q_desc = tc::sw128_desc(sb + kv_q(0), 16, 1024), do_desc = tc::sw128_desc(sb + kv_do(0), 16, 1024);
      const uint64_t qmn_desc = tc::sw128_desc(sb + kv_q(0), kSlab, 1024);     // Q, dO as MN-major B
      const uint64_t domn_desc = tc::sw128_desc(sb + kv_do(0), kSlab, 1024);
      bool ok = wait_or_abort(&ms->kv_full, 0, ms, err, 2u);
      // pass i = 2u + h: queries 64 h .. 64 h + 63 of unit u.
      // dV += (P^T cs) dO and dK += dS^T Q over the 64 queries of pass i
      auto issue_grads = [&](int i) -> bool {
        const int u = i >> 1, h = i & 1, s = u % kStages;
        if (!wait_or_abort(&ms->p_half[h], u & 1, ms, err, 4u)) return false;
        tc::tc_fence_after();
        const uint32_t so = (uint32_t)s * 2 * kTile;
        const uint64_t domb = tc::desc_adv(domn_desc, so), qmb = tc::desc_adv(qmn_desc, so);
        const uint32_t pt = tmem + TL::st(h);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = 4 * h + k4;                 // queries 16 kk .. 16 kk + 15 of the unit
          tc::mma_bf16_ts(tmem + TM_DV, pt + 16 * k4, tc::desc_adv(domb, kk * 2048), idG, (u > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = 4 * h + k4;
          tc::mma_bf16_ts(tmem + TM_DK, pt + TL::kDp + 16 * k4, tc::desc_adv(qmb, kk * 2048), idG,
                          (u > 0 || kk > 0) ? 1u : 0u);
        }
        if (h == 1) tc::mma_commit(&ms->qd_empty[s]);   // the unit's Q / dO stage is read
        if (h == 1 && u == last1) tc::mma_commit(&ms->st1_read);
        return true;
      };
      if constexpr (!TL::kTwoBuf) {
        // one buffer: per tile, the scores (N = 128), then each pass's products once the softmax
        // warps have written it; the next tile's scores overwrite this tile's after them
        // (tcgen05 MMAs of one thread run in issue order)
        for (int u = 0; ok && u < n_u; ++u) {
          const int s = u % kStages;
          if (!wait_or_abort(&ms->qd_full[s], (u / kStages) & 1, ms, err, 8u)) break;
          tc::tc_fence_after();
          const uint32_t so = (uint32_t)s * 2 * kTile;             // stage offset of Q and dO
          const uint64_t qb = tc::desc_adv(q_desc, so), dob = tc::desc_adv(do_desc, so);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kSlab + (kk & 3) * 32;
            tc::mma_bf16(tmem, tc::desc_adv(k_desc, off), tc::desc_adv(qb, off), idS, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kSlab + (kk & 3) * 32;
            tc::mma_bf16(tmem + TL::kDp, tc::desc_adv(v_desc, off), tc::desc_adv(dob, off), idS, kk > 0 ? 1u : 0u);
          }
          tc::mma_commit(&ms->s_full[0]);
          if (u == n_u - 1) tc::mma_commit(&ms->kv_read);   // every score product has read K and V
          const uint64_t domb = tc::desc_adv(domn_desc, so), qmb = tc::desc_adv(qmn_desc, so);
          for (int h = 0; ok && h < 2; ++h) {
            ok = wait_or_abort(&ms->p_half[h], u & 1, ms, err, 4u);
            if (!ok) break;
            tc::tc_fence_after();
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int kk = 4 * h + k4;             // queries 16 kk .. 16 kk + 15
              tc::mma_bf16_ts(tmem + TM_DV, tmem + 16 * kk, tc::desc_adv(domb, kk * 2048), idG,
                              (u > 0 || kk > 0) ? 1u : 0u);
            }
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int kk = 4 * h + k4;
              tc::mma_bf16_ts(tmem + TM_DK, tmem + TL::kDp + 16 * kk, tc::desc_adv(qmb, kk * 2048), idG,
                              (u > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if (ok) tc::mma_commit(&ms->qd_empty[s]);
          if (ok && u == last1) tc::mma_commit(&ms->st1_read);
        }
      } else {
        // two buffers: the scores of pass i + 1 run on the tensor cores while the softmax warps
        // work on pass i
        int n_grads = 0;                                 // passes whose products are issued
        for (int i = 0; ok && i < 2 * n_u; ++i) {
          const int u = i >> 1, h = i & 1, s = u % kStages;
          if (h == 0 && !wait_or_abort(&ms->qd_full[s], (u / kStages) & 1, ms, err, 8u)) break;
          tc::tc_fence_after();
          // buffer h last held pass i - 2, whose products were issued before (in order) and
          // whose scores the softmax warps had read before they arrived on p_half[h]
          const uint32_t qo = (uint32_t)s * 2 * kTile + (uint32_t)h * 64 * 128;   // query rows 64 h ..
          const uint64_t qb = tc::desc_adv(q_desc, qo), dob = tc::desc_adv(do_desc, qo);
          const uint32_t st = tmem + TL::st(h);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kSlab + (kk & 3) * 32;
            tc::mma_bf16(st, tc::desc_adv(k_desc, off), tc::desc_adv(qb, off), idS, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kSlab + (kk & 3) * 32;
            tc::mma_bf16(st + TL::kDp, tc::desc_adv(v_desc, off), tc::desc_adv(dob, off), idS, kk > 0 ? 1u : 0u);
          }
          tc::mma_commit(&ms->s_full[h]);
          if (i == 2 * n_u - 1) tc::mma_commit(&ms->kv_read);   // every score product has read K and V
          // the previous pass's products, behind this pass's scores
          if (i >= 1) {
            ok = issue_grads(i - 1);
            if (!ok) break;
            n_grads = i;
          }
        }
        if (ok && n_u > 0 && n_grads == 2 * n_u - 1) issue_grads(2 * n_u - 1);
      }
      tc::mma_commit(&ms->done);
      tc::mbar_wait(&ms->done, 0);
    }
  } else if (warp == 10) {
    // ---------------- scalar transposer: each stage's per-query (log2 d_s, cs, Delta) as three
    // arrays (-log2 d_s, cs, -Delta) once the stage has landed.  The stage's previous tile is
    // done with them: its copy waited for that tile's products, which waited for its softmax.
    for (int u = 0; u < n_u; ++u) {
      const int s = u % kStages;
      if (!__all_sync(0xffffffffu, wait_or_abort(&ms->qd_full[s], (u / kStages) & 1, ms, err, 2048u))) break;
      const float4* src = reinterpret_cast<const float4*>(smem + KV_SC + s * 128 * 16);
      float* dst = reinterpret_cast<float*>(smem + KV_SOA + s * 3 * 128 * 4);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 v = src[lane + 32 * k];
        dst[lane + 32 * k] = -v.x;
        dst[128 + lane + 32 * k] = v.y;
        dst[256 + lane + 32 * k] = -v.z;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ms->sc_ready[s]);
    }
  } else {
    // ---------------- softmax: one key row; two passes of 32 queries per thread ----------------
    const int q4 = warp & 3;
    const int grp = (warp - 2) >> 2;                // queries 32 grp + 64 pass .. + 31
    const int row = 32 * q4 + lane;                 // key row within the CTA's 128
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    // PAIR: key rows 0-63 are block pb[0], rows 64-127 block pb[1]
    const int mine = PAIR ? (row >= 64) : 0;
    const int my_block = pb[mine];
    const int krow = PAIR ? 64 * my_block + (row & 63) : key0 + row;      // key row in the head
    const bool key_ok = my_block >= 0 && krow < g.N;
    const float sl2 = g.scale * kLog2e;
    // PAIR: key rows 0-63 see query rows 0-63 of a unit (pass 0), rows 64-127 query rows
    // 64-127 (pass 1)
    const int kpos = PAIR ? (row & 63) : row;       // key position within its block
    bool alive = true;
    for (int u = 0; u < n_u && alive; ++u) {
      const int s = u % kStages;
      // one buffer: both passes' scores arrive together; two: each pass's on its own
      alive = __all_sync(0xffffffffu, wait_or_abort(&ms->s_full[0], u & 1, ms, err, 32u));
      if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->sc_ready[s], (u / kStages) & 1, ms, err, 4096u));
      if (!alive) break;
      tc::tc_fence_after();
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        if (KvTmem<D>::kTwoBuf && pass == 1) {
          alive = __all_sync(0xffffffffu, wait_or_abort(&ms->s_full[1], u & 1, ms, err, 32u));
          if (!alive) break;
          tc::tc_fence_after();
        }
        const int q0 = 64 * pass + 32 * grp;        // first query (column of the unit) of this thread
        // the query tile of these columns and the first one's position in it
        const int h = PAIR ? pass : 0;
        const bool present = u < (h ? n_ub : n_ua);
        const int t = present ? units[h * kMaxUnits + u] : 0;
        const int qp0 = PAIR ? q0 - 64 * pass : q0;
        const bool dead = PAIR && (pass != mine || !present);
        const bool diag = g.causal && t == my_block;
        const int qvalid = g.N - t * TB - qp0;      // queries of this thread inside the sequence
        const bool masked = dead || !key_ok || qvalid < 32 || (diag && kpos > qp0);
        const int lo = diag ? kpos - qp0 : 0;
        const int hi = dead ? 0 : key_ok ? qvalid : 0;
        const float* nx = reinterpret_cast<const float*>(smem + KV_SOA + s * 3 * 128 * 4) + q0;
        const uint32_t st_col = lane_base + KvTmem<D>::st(pass) + 32 * grp;
        // masking only on the causal diagonal, at the end of the sequence and for padding keys
        if (__any_sync(0xffffffffu, masked))
          dkdv_softmax_cols<true>(tmem, st_col, st_col + KvTmem<D>::kDp, nx, nx + 128, nx + 256, sl2, lo, hi);
        else
          dkdv_softmax_cols<false>(tmem, st_col, st_col + KvTmem<D>::kDp, nx, nx + 128, nx + 256, sl2, lo, hi);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&ms->p_half[pass]);
      }
    }
    // ---------------- epilogue: dK = scale dK_sparse + dK_lowrank, dV likewise; TMA stores ----------------
    const int hq = grp;
    const int col0 = H * hq;                         // this thread's columns [col0, col0 + H)
    const int ch0 = (col0 & 63) >> 3;
    bool have = false;
    if (alive && n_u > 0) {
      alive = __all_sync(0xffffffffu, wait_or_abort(&ms->done, 0, ms, err, 512u));
      have = alive;
      if (have) tc::tc_fence_after();
    }
    // every product has completed: stage dK in the stage-0 Q buffer and dV in the stage-0 dO buffer
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const float mul = which == 0 ? g.scale : 1.f;
      // the low-rank part, brought into shared memory by the producer
      if (alive && (which == 0 ? a.dKacc : a.dVacc))
        alive = __all_sync(0xffffffffu,
                           wait_or_abort(which == 0 ? &ms->acck_full : &ms->accv_full, 0, ms, err, 1024u));
      const bool use_acc = (which == 0 ? a.dKacc : a.dVacc) && alive && key_ok;
      const uint32_t acc_base = which == 0 ? KV_K : kv_q(1);
      // fp32 element (row, c): box c / 32, 16-byte chunk (c % 32) / 4 swizzled by the row
      auto acc4 = [&](int cc) -> float4 {
        return *reinterpret_cast<const float4*>(smem + acc_base + (uint32_t)(cc >> 5) * kAccBox + (uint32_t)row * 128u +
                                                ((uint32_t)(((cc & 31) >> 2) ^ (row & 7)) << 4));
      };
      unsigned char* orow = smem + (which == 0 ? kv_q(0) : kv_do(0)) + (col0 >> 6) * kSlab + row * 128;
      // with a row map, write each key row straight to the caller's row instead
      uint4* grow = a.k_rows && key_ok && alive
                        ? reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(which == 0 ? a.dK : a.dV) +
                                                   (head + a.k_rows[(size_t)bh * a.rows_stride + krow]) * D +
                                                   col0)
                        : nullptr;
      // 32 columns at a time: TMEM -> scale -> + low-rank part -> bf16 -> swizzled row
#pragma unroll
      for (int c = 0; c < H / 32; ++c) {
        float o[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
        if (have) {
          tc::tmem_ld32(tmem + lane_base + (which == 0 ? TM_DK : TM_DV) + col0 + 32 * c, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= mul;
        }
        if (use_acc) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 x = acc4(col0 + 32 * c + 4 * q);
            o[4 * q] += x.x; o[4 * q + 1] += x.y; o[4 * q + 2] += x.z; o[4 * q + 3] += x.w;
          }
        }
        if (a.out_f32) {                                 // fp32 rows (level slots), no staging
          if (alive && key_ok) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(which == 0 ? a.dK : a.dV) +
                                                    (head + (size_t)krow) * D + col0 + 32 * c);
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          }
          continue;
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int ch = 4 * c + cc;
          const uint4 val =
              make_uint4(pack_bf16(o[8 * cc], o[8 * cc + 1]), pack_bf16(o[8 * cc + 2], o[8 * cc + 3]),
                         pack_bf16(o[8 * cc + 4], o[8 * cc + 5]), pack_bf16(o[8 * cc + 6], o[8 * cc + 7]));
          if (a.k_rows) {
            if (grow) grow[ch] = val;
          } else {
            *reinterpret_cast<uint4*>(orow + (((ch0 + ch) ^ (row & 7)) << 4)) = val;
          }
        }
      }
    }
    if (!a.k_rows && !a.out_f32) {
      tc::fence_proxy_async_smem();
      softmax_bar();
      if (threadIdx.x == 64 && !*(volatile int*)&ms->abort_flag) {
        for (int h = 0; h < (PAIR ? 2 : 1); ++h) {
          if (pb[h] < 0) continue;
          const int kr = PAIR ? 64 * pb[h] : key0;
          for (int sl = 0; sl < D / 64; ++sl) {
            tma_store_3d(&tmdK, smem + kv_q(0) + sl * kSlab + h * 64 * 128, 64 * sl, kr, bh);
            tma_store_3d(&tmdV, smem + kv_do(0) + sl * kSlab + h * 64 * 128, 64 * sl, kr, bh);
          }
        }
        tma_store_wait();
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [BH][N][128] bf16 as a 3-D tensor (d, row, head), boxes of 64 x rows x 1, 128-byte swizzle.
bool tc::map_rows_bf16(CUtensorMap* m, const void* base, int N, int BH, int rows) {
  return map_rows_bf16_pitch(m, base, kD, kD, N, BH, rows);
}

// `cols` columns of [BH][N][pitch] bf16 rows starting at `base` (all of them, or a column
// block of wider rows), in boxes of 64 columns.
bool tc::map_rows_bf16_pitch(CUtensorMap* m, const void* base, int cols, int pitch, int N, int BH, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)pitch * 2, (cuuint64_t)N * pitch * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool bwd_tc_supported(const Geom& g) { return (g.d == 64 || g.d == 128) && (g.T == 64 || g.T == 128); }

// [BH][N][d] bf16 rows in boxes of 64 columns x `rows` rows
static bool map_d(CUtensorMap* m, const void* base, const Geom& g, int rows) {
  return tc::map_rows_bf16_pitch(m, base, g.d, g.d, g.N, g.BH, rows);
}

// fp32 [BH][N][d] low-rank gradient rows in boxes of 32 columns x `rows` rows, 128-byte swizzle.
static bool map_acc_f32(CUtensorMap* m, const float* base, const Geom& g, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)g.d, (cuuint64_t)g.N, (cuuint64_t)g.BH};
  cuuint64_t strides[2] = {(cuuint64_t)g.d * 4, (cuuint64_t)g.N * g.d * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool PAIR>
static cudaError_t dq_t(const BwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  constexpr int TB = PAIR ? 64 : 128;
  if (PAIR && a.tile_list && (a.n_list & 1)) return cudaErrorInvalidValue;   // tile pairs
  CUtensorMap mq, mk, mv, mdo, mdq, macc;
  if (!map_d(&mq, a.Q, g, kT) || !map_d(&mk, a.K, g, TB) || !map_d(&mv, a.V, g, TB) || !map_d(&mdo, a.dO, g, kT) ||
      !map_d(&mdq, a.dQ, g, kT))
    return cudaErrorInvalidValue;
  if (a.dQacc) {
    if (!map_acc_f32(&macc, a.dQacc, g, kT)) return cudaErrorInvalidValue;
  } else {
    macc = mdq;                                      // not read without a low-rank part
  }
  const size_t smem = DQ_MISC + sizeof(DqMisc);
  static_assert(DQ_MISC + sizeof(DqMisc) <= 232448, "shared memory per CTA");
  auto kern = dq_tc_kernel<D, PAIR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int units = a.tile_list ? (PAIR ? a.n_list / 2 : a.n_list) : (PAIR ? (g.n_t + 1) / 2 : g.n_t);
  ProfScope ps("dq_tc", st);
  kern<<<dim3(units, g.BH), kDqThreads, smem, st>>>(mq, mk, mv, mdo, mdq, macc, a, g, err);
  return cudaGetLastError();
}

cudaError_t launch_dq_tc(const BwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  if (!bwd_tc_supported(g) || !a.rs.packed) return cudaErrorInvalidValue;
  if (g.d == 64) return g.T == 64 ? dq_t<64, true>(a, g, err, st) : dq_t<64, false>(a, g, err, st);
  return g.T == 64 ? dq_t<128, true>(a, g, err, st) : dq_t<128, false>(a, g, err, st);
}

// Per-row scalars (log2 d_s, cs, Delta, 0) as float32 [BH][N][4]; boxes of 4 x rows x 1.
static bool map_scalars(CUtensorMap* m, const void* base, int N, int BH, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {4, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {16, (cuuint64_t)N * 16};
  cuuint32_t box[3] = {4, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool PAIR>
static cudaError_t dkdv_t(const BwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  constexpr int TB = PAIR ? 64 : 128;
  CUtensorMap mk, mv, mq, mdo, msc, mdk, mdv, mka, mva;
  if (!map_d(&mk, a.K, g, TB) || !map_d(&mv, a.V, g, TB) || !map_d(&mq, a.Q, g, TB) || !map_d(&mdo, a.dO, g, TB) ||
      !map_scalars(&msc, a.rs.packed, g.N, g.BH, TB) || !map_d(&mdk, a.dK, g, TB) || !map_d(&mdv, a.dV, g, TB))
    return cudaErrorInvalidValue;
  // maps of the low-rank parts (not read when absent)
  if ((a.dKacc && !map_acc_f32(&mka, a.dKacc, g, TB)) || (a.dVacc && !map_acc_f32(&mva, a.dVacc, g, TB)))
    return cudaErrorInvalidValue;
  if (!a.dKacc) mka = mk;
  if (!a.dVacc) mva = mv;
  const size_t smem = KV_MISC + sizeof(KvMisc);
  static_assert(KV_MISC + sizeof(KvMisc) <= 232448, "shared memory per CTA");
  auto kern = dkdv_tc_kernel<D, PAIR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps("dkdv_tc", st);
  // with n_kv, only the first n_kv key blocks of kv_order (the ones with query tiles) run;
  // PAIR: two consecutive entries of that order per CTA
  const int nb = a.n_kv ? a.n_kv : g.n_t;
  const int ctas = PAIR ? (nb + 1) / 2 : nb;
  kern<<<dim3(g.BH, ctas), kKvThreads, smem, st>>>(mk, mv, mq, mdo, msc, mdk, mdv, mka, mva, a, g, err);
  return cudaGetLastError();
}

cudaError_t launch_dkdv_tc(const BwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  if (!bwd_tc_supported(g) || !a.rs.packed || g.n_t > kMaxUnits || (a.n_kv && !a.kv_order) || a.n_kv > g.n_t)
    return cudaErrorInvalidValue;
  if (g.d == 64) return g.T == 64 ? dkdv_t<64, true>(a, g, err, st) : dkdv_t<64, false>(a, g, err, st);
  return g.T == 64 ? dkdv_t<128, true>(a, g, err, st) : dkdv_t<128, false>(a, g, err, st);
}

}  // namespace elsaa
