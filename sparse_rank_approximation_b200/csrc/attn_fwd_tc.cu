// Sparse-branch forward on the 5th-generation tensor cores (tcgen05 + TMEM), fused
// with the denominator-aware fusion epilogue (ELSAA paper §3.2, §3.3 Eq. 5, §1 Eq. 4).
// Head dimension D = 64 or 128.  A CTA works on 128 query rows: one tile of 128 queries
// with 128-key blocks, or (PAIR, blocks of 64) the two adjacent 64-query tiles 2u and
// 2u + 1, whose selected blocks are staged side by side: the K and V stage of step j
// holds tile 2u's j-th block in rows 0-63 and tile 2u + 1's in rows 64-127, so every
// product stays M = N = 128 and each query row masks the other tile's 64 keys.
//
// Two CTAs share an SM (256 TMEM columns and under 113 KB of shared memory each), so one
// CTA's products run while the other's softmax warps work: within a CTA the chain
// S_j = Q K_j^T -> softmax_j -> O += P_j V_j -> S_j+1 is serial (S_j+1 overwrites P_j in
// tensor memory).  10 warps:
//   warp 0      TMA producer: Q, then K_j and V_j into their rings (one stage at d = 128,
//               two at d = 64) as the products free them, and at the end the tile's
//               low-rank output O_lr into the K stage for the epilogue;
//   warp 1      TMEM owner and MMA issuer;
//   warps 2-9   softmax: each query row is split over two warps (64 score columns each)
//               that exchange their partial row max; online softmax in fp32 with lazy
//               rescaling (O and l move only when the running max grows by more than
//               2^16); P_j goes back over the score columns it came from as bf16 hi + lo
//               pairs (hi + lo within 2^-15 of P, so O_s, and the backward's softmax delta
//               formed from it, carry no bf16 rounding of the weights) and is the A operand of the
//               two PV products; the epilogue normalises O, applies the fusion and writes O
//               (TMA store from shared memory) and the fp32 O_s (row stores).
// Operand tiles are 64-column slabs with 128-byte swizzle, as TMA writes them.
// Every mbarrier wait is bounded; a timeout sets a bit in the caller's error word,
// the CTA drains its copies and MMAs, frees TMEM and exits.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace elsaa {

namespace {

constexpr int kT = 128;                  // query rows of a CTA = keys of a K/V stage
constexpr uint32_t kSlab = kT * 128;     // one [128 rows][64 bf16] swizzled slab
template <int D> struct FwdLayout {
  static constexpr int kStages = D == 64 ? 2 : 1;                 // K and V ring depth
  static constexpr uint32_t kTileB = (D / 64) * kSlab;            // one [128][D] bf16 tile
  static constexpr uint32_t kQ = 0;
  __host__ __device__ static constexpr uint32_t k(int s) { return kTileB * (1 + s); }
  __host__ __device__ static constexpr uint32_t v(int s) { return kTileB * (1 + kStages + s); }
  static constexpr uint32_t kMisc = kTileB * (1 + 2 * kStages);
};
// P over the score columns it came from, 16 keys (16 fp32 columns) at a time: the bf16 hi
// pairs of keys 16 kk .. 16 kk + 15 in the first 8 of those columns, the lo pairs
// (bf16(P - P_hi)) in the next 8; so P of a group of 32 keys only overwrites its own scores
__host__ __device__ constexpr uint32_t p_col(int kk) { return (uint32_t)(16 * kk); }
constexpr uint32_t kPLo = 8;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t TM_O = 0, TM_S = 128;                 // output accumulator, scores / P
constexpr float kRescaleThreshold = 16.f;                // log2 units: P stays below 2^16
constexpr int kThreads = 320;
constexpr int kSoftmaxThreads = 256;
constexpr int kMaxStages = 2;

struct Misc {
  uint64_t q_full, k_full[kMaxStages], k_empty[kMaxStages], v_full[kMaxStages], v_empty[kMaxStages], s_full,
      p_full, pv_done;
  uint64_t olr_full, drain, never;
  unsigned long long limit_ns;
  uint32_t tmem_base;
  int abort_flag;
  int idx[2][32];         // selected blocks of the CTA's tile (PAIR: of its two tiles)
  float red[2][256];      // partial row maxima / sums exchanged by the two halves of a row
};
template <int D>
constexpr size_t smem_bytes() { return FwdLayout<D>::kMisc + sizeof(Misc); }
static_assert(smem_bytes<128>() <= 232448 / 2 - 1024, "two CTAs per SM");
static_assert(smem_bytes<64>() <= 232448 / 2 - 1024, "two CTAs per SM");

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// A pair (a, b) of non-negative floats as bf16 hi + lo pairs by truncation, with integer and
// FMA instructions only: hi keeps the top 16 bits of each float (sign, exponent, 7 mantissa
// bits), lo the top 16 bits of the exact remainder, so hi + lo is within 2^-15 of each value.
// a sits in the low half of each word, b in the high half.
// ab holds the same pair as packed fp32 lanes, so both remainders take one f32x2 subtraction.
__device__ __forceinline__ void split_trunc(float a, float b, uint64_t ab, uint32_t& hi, uint32_t& lo) {
  const uint32_t ua = __float_as_uint(a), ub = __float_as_uint(b);
  hi = __byte_perm(ua, ub, 0x7632);
  float ra, rb;
  tc::f2_unpack(tc::f2_sub(ab, tc::f2_pack(__uint_as_float(ua & 0xffff0000u), __uint_as_float(ub & 0xffff0000u))), ra,
                rb);
  lo = __byte_perm(__float_as_uint(ra), __float_as_uint(rb), 0x7632);
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Misc* ms, uint32_t* err,
                                              uint32_t code) {
  if (*(volatile int*)&ms->abort_flag) return false;
  if (tc::mbar_wait(bar, parity, ms->limit_ns)) return true;
  *(volatile int*)&ms->abort_flag = 1;
  if (err) atomicOr(err, code);
  return false;
}

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];\n"
               :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2) : "memory");
}

}  // namespace

template <int D, bool PAIR>
__global__ void __launch_bounds__(kThreads, 2)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmLr,
                       const __grid_constant__ CUtensorMap tmO, FwdArgs a, Geom g, uint32_t* err) {
  using L = FwdLayout<D>;
  constexpr int KS = L::kStages;
  extern __shared__ __align__(1024) unsigned char smem[];
  Misc* ms = reinterpret_cast<Misc*>(smem + L::kMisc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  constexpr int TB = PAIR ? 64 : 128;       // keys per block = queries per tile
  constexpr int H = D / 2;                  // output columns per thread (half a row)
  // the CTA's rows: tile t (128 rows), or tiles ta = 2u, tb = 2u + 1 (PAIR; tb may be past the end)
  const int n_units = PAIR ? (g.n_t + 1) / 2 : g.n_t;
  const int unit = a.tile_list ? (PAIR ? a.tile_list[(size_t)bh * a.n_list + 2 * blockIdx.x] / 2
                                       : a.tile_list[(size_t)bh * a.n_list + blockIdx.x])
                               : n_units - 1 - (int)blockIdx.x;
  const int ta = PAIR ? 2 * unit : unit, tb = PAIR ? 2 * unit + 1 : unit;
  const int row0 = kT * unit;
  const size_t head = (size_t)bh * g.N;
  if (smem_u32(smem) & 1023u) {            // the swizzled layouts need 1024-byte aligned tiles
    if (threadIdx.x == 0 && err) atomicOr(err, 0x80000000u);
    return;
  }

  // ---- set-up: barriers, selected blocks, TMEM
  const int* idx_a = a.idx + ((size_t)bh * g.n_t + ta) * g.k;
  const int* idx_b = a.idx + ((size_t)bh * g.n_t + tb) * g.k;
  if (threadIdx.x == 0) {
    tc::mbar_init(&ms->q_full, 1);
    for (int s = 0; s < KS; ++s) {
      tc::mbar_init(&ms->k_full[s], 1);
      tc::mbar_init(&ms->k_empty[s], 1);
      tc::mbar_init(&ms->v_full[s], 1);
      tc::mbar_init(&ms->v_empty[s], 1);
    }
    tc::mbar_init(&ms->s_full, 1);
    tc::mbar_init(&ms->p_full, kSoftmaxThreads);
    tc::mbar_init(&ms->pv_done, 1);
    tc::mbar_init(&ms->olr_full, 1);
    tc::mbar_init(&ms->drain, 1);
    tc::mbar_init(&ms->never, 1);
    ms->limit_ns = g.wait_ns;
    ms->abort_flag = 0;
    tc::fence_barrier_init();
    // Q does not depend on the selection: its copy starts before anything else
    tc::mbar_arrive_expect_tx(&ms->q_full, 128u * D * 2);
    for (int sl = 0; sl < D / 64; ++sl) tc::tma_load_3d(smem + L::kQ + sl * kSlab, &tmQ, &ms->q_full, 64 * sl, row0, bh);
    tc::prefetch_tensormap(&tmK);
    tc::prefetch_tensormap(&tmV);
  }
  if (threadIdx.x < 32) {
    ms->idx[0][threadIdx.x] = threadIdx.x < g.k ? idx_a[threadIdx.x] : -1;
    ms->idx[1][threadIdx.x] = PAIR && tb < g.n_t && threadIdx.x < g.k ? idx_b[threadIdx.x] : -1;
  }
  if (warp == 1) {
    tc::tmem_alloc(&ms->tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  // block j of tile half h: the first 32 from shared memory, any further ones from global memory
  auto sel = [&](int h, int j) -> int { return j < 32 ? ms->idx[h][j] : (h ? idx_b : idx_a)[j]; };
  int n_sel_t[2] = {0, 0};
  for (int h = 0; h < (PAIR ? 2 : 1); ++h)
    while (n_sel_t[h] < g.k && (h == 0 || tb < g.n_t) && sel(h, n_sel_t[h]) >= 0) ++n_sel_t[h];
  const int n_sel = max(n_sel_t[0], n_sel_t[1]);          // steps

  if (warp == 0) {
    // ================= TMA producer: Q, the K and V rings, O_lr =================
    if (lane == 0) {
      constexpr uint32_t kTD = 128u * D * 2;      // bytes of a [128][D] tile
      bool alive = true;
      int k_issued = 0, v_issued = 0;
      // K_j and V_j in consumption order; a stage is reloaded once the product that read it is done
      for (int j = 0; alive && j < n_sel; ++j) {
        const int s = j % KS;
        for (int kv = 0; kv < 2; ++kv) {
          uint64_t* full = kv ? ms->v_full : ms->k_full;
          uint64_t* empty = kv ? ms->v_empty : ms->k_empty;
          if (j >= KS && !wait_or_abort(&empty[s], ((j / KS) - 1) & 1, ms, err, kv ? 512u : 1u)) {
            alive = false;
            break;
          }
          unsigned char* dst = smem + (kv ? L::v(s) : L::k(s));
          tc::mbar_arrive_expect_tx(&full[s], kTD);
          for (int h = 0; h < (PAIR ? 2 : 1); ++h) {
            // PAIR: a tile with fewer blocks stages block 0 in its half (every score of it is masked)
            const int b = j < (h ? n_sel_t[1] : n_sel_t[0]) ? sel(h, j) : 0;
            for (int sl = 0; sl < D / 64; ++sl)
              tc::tma_load_3d(dst + sl * kSlab + h * 64 * 128, kv ? &tmV : &tmK, &full[s], 64 * sl, b * TB, bh);
          }
          if (kv) v_issued = j + 1; else k_issued = j + 1;
        }
      }
      bool lr_issued = false;
      if (alive) {
        // the low-rank output goes into K stage 0 once every score MMA has read its K tile
        for (int j = (n_sel > KS ? n_sel - KS : 0); alive && j < n_sel; ++j)
          alive = wait_or_abort(&ms->k_empty[j % KS], (j / KS) & 1, ms, err, 2048u);
        if (alive) {
          tc::mbar_arrive_expect_tx(&ms->olr_full, kTD);
          for (int sl = 0; sl < D / 64; ++sl)
            tc::tma_load_3d(smem + L::k(0) + sl * kSlab, &tmLr, &ms->olr_full, 64 * sl, row0, bh);
          lr_issued = true;
        }
      }
      // drain: every copy this thread started has landed before the CTA may exit
      tc::mbar_wait(&ms->q_full, 0);
      if (lr_issued) tc::mbar_wait(&ms->olr_full, 0);
      for (int j = (k_issued > KS ? k_issued - KS : 0); j < k_issued; ++j) tc::mbar_wait(&ms->k_full[j % KS], (j / KS) & 1);
      for (int j = (v_issued > KS ? v_issued - KS : 0); j < v_issued; ++j) tc::mbar_wait(&ms->v_full[j % KS], (j / KS) & 1);
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t idS = tc::idesc_bf16(128, 128, false, false);   // Q (K-major) x K (K-major)
      const uint32_t idPV = tc::idesc_bf16(128, D, false, true);     // P (TMEM) x V (MN-major)
      const uint32_t sbase = smem_u32(smem);
      // operand descriptors built once; a K step or a ring stage only moves the start address
      const uint64_t q_desc = tc::sw128_desc(sbase + L::kQ, 16, 1024);
      const uint64_t k_desc = tc::sw128_desc(sbase + L::k(0), 16, 1024);
      const uint64_t v_desc = tc::sw128_desc(sbase + L::v(0), kSlab, 1024);   // V as the MN-major B of P V
      bool ok = wait_or_abort(&ms->q_full, 0, ms, err, 2u);
      // S_j overwrites P_{j-1}: the PV product that reads it was issued earlier, and tcgen05
      // MMAs of one thread run in issue order
      for (int j = 0; ok && j < n_sel; ++j) {
        const int s = j % KS;
        if (!wait_or_abort(&ms->k_full[s], (j / KS) & 1, ms, err, 8u)) break;
        tc::tc_fence_after();
        const uint64_t kb = tc::desc_adv(k_desc, L::k(s) - L::k(0));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSlab + (kk & 3) * 32;
          tc::mma_bf16(tmem + TM_S, tc::desc_adv(q_desc, off), tc::desc_adv(kb, off), idS, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&ms->s_full);
        tc::mma_commit(&ms->k_empty[s]);
        // O += P_hi V + P_lo V once the softmax warps have written P_j
        if (!wait_or_abort(&ms->p_full, j & 1, ms, err, 4u)) break;
        if (!wait_or_abort(&ms->v_full[s], (j / KS) & 1, ms, err, 1024u)) break;
        tc::tc_fence_after();
        const uint64_t vb = tc::desc_adv(v_desc, L::v(s) - L::v(0));
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk) {
          const uint64_t bd = tc::desc_adv(vb, kk * 2048);
          const uint32_t pa = tmem + TM_S + p_col(kk);
          tc::mma_bf16_ts(tmem + TM_O, pa, bd, idPV, (j > 0 || kk > 0) ? 1u : 0u);
          tc::mma_bf16_ts(tmem + TM_O, pa + kPLo, bd, idPV, 1u);
        }
        tc::mma_commit(&ms->v_empty[s]);
        tc::mma_commit(&ms->pv_done);
      }
      // drain: all MMAs this thread issued have completed
      tc::mma_commit(&ms->drain);
      tc::mbar_wait(&ms->drain, 0);
    }
  } else {
    // ================= softmax / epilogue: half a query row per thread =================
    const int q4 = warp & 3;
    const int half = (warp - 2) >> 2;                // score columns [64 half, +64), output [H half, +H)
    const int row = 32 * q4 + lane;
    const int sid = half * 128 + row;                // slot in the exchange arrays
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const float sl2 = g.scale * kLog2e;
    const int qrow = row0 + row;
    // PAIR: rows 0-63 belong to tile ta and score columns 0-63, rows 64-127 to tile tb and
    // columns 64-127; a thread whose half holds the other tile's keys masks all of them
    const int mine = PAIR ? (row >= 64) : 0;
    const int my_tile = PAIR ? (mine ? tb : ta) : ta;
    const int my_n = mine ? n_sel_t[1] : n_sel_t[0];
    const bool dead_half = PAIR && half != mine;
    const int qpos = PAIR ? (row & 63) : row;        // query position within its tile
    float m_used = -INFINITY, lp = 0.f;              // running max (scaled log2 units), partial row sum
    bool alive = true;                               // warp-uniform; every barrier below is still taken
    // test hook: a wait on a barrier nothing completes, so the give-up path runs
    if (g.debug_stall) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->never, 0, ms, err, 0x40000u));
    for (int j = 0; j < n_sel; ++j) {
      const int s = j & 1;                           // exchange buffer
      float sv[32];
      if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->s_full, j & 1, ms, err, 32u));
      // key k of this half's 64 columns is key c0 + k of block b (no block: all masked)
      const bool none = dead_half || j >= my_n;
      const int b = none ? 0 : sel(PAIR ? half : 0, j);
      const int c0 = PAIR ? 0 : 64 * half;
      const int kvalid = g.N - b * TB;
      const bool diag = g.causal && b == my_tile;
      const int lim = none ? -1 : (diag || kvalid < TB) ? min(kvalid - 1, diag ? qpos : TB - 1) - c0 : 64;
      // scores of this thread's 64 columns in two parts of 32; the row max over part 0 first, then
      // over part 1, which stays in registers; part 0 is read again after the exchange
      auto load_part = [&](int part) {
        tc::tmem_ld32(tmem + lane_base + TM_S + 64 * half + 32 * part, sv);
        tc::tmem_wait_ld();
        if (lim < 64) {
#pragma unroll
          for (int c = 0; c < 32; ++c) sv[c] = 32 * part + c > lim ? -INFINITY : sv[c];
        }
      };
      auto part_max = [&]() {
        float m4[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
        for (int c = 4; c < 32; c += 4) {
          m4[0] = fmaxf(m4[0], sv[c]);
          m4[1] = fmaxf(m4[1], sv[c + 1]);
          m4[2] = fmaxf(m4[2], sv[c + 2]);
          m4[3] = fmaxf(m4[3], sv[c + 3]);
        }
        return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      };
      if (alive) {
        tc::tc_fence_after();
        load_part(0);
        const float m0 = part_max();
        load_part(1);
        ms->red[s][sid] = fmaxf(m0, part_max());
      }
      softmax_bar();
      if (alive) {
        const float mx = fmaxf(ms->red[s][row], ms->red[s][128 + row]) * sl2;
        // lazy rescaling: move the reference max only when the row max grew by > 2^16
        const float m_new = fmaxf(m_used, mx);
        const bool resc = m_new > m_used + kRescaleThreshold;     // false while both are -inf
        float alpha = 1.f;
        if (resc) {
          alpha = (m_used == -INFINITY) ? 0.f : exp2f(m_used - m_new);
          lp *= alpha;
          m_used = m_new;
        }
        // P_j as bf16 hi + lo pairs, part 1 (in registers) and then part 0 (read again)
        const float msub = m_used == -INFINITY ? 0.f : m_used;
        // pairs of columns in packed fp32 lanes: x = s sl2 - m, the row sum and the lo remainder
        // each take one f32x2 instruction per pair
        const uint64_t sl2x2 = tc::f2_pack(sl2, sl2), negm2 = tc::f2_pack(-msub, -msub);
        uint64_t rs2 = tc::f2_pack(0.f, 0.f);
#pragma unroll 1
        for (int part = 1; part >= 0; --part) {
          if (part == 0) load_part(0);
#pragma unroll
          for (int q = 0; q < 2; ++q) {              // 16 keys: 8 hi pairs, then 8 lo pairs
            uint32_t w[8], wl[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float x0, x1;
              tc::f2_unpack(tc::f2_fma(tc::f2_pack(sv[16 * q + 2 * e], sv[16 * q + 2 * e + 1]), sl2x2, negm2), x0, x1);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              const uint64_t p2 = tc::f2_pack(p0, p1);
              rs2 = tc::f2_add(rs2, p2);
              split_trunc(p0, p1, p2, w[e], wl[e]);
            }
            const uint32_t col = tmem + lane_base + TM_S + 64 * half + 32 * part + 16 * q;
            tc::tmem_st8(col, w);
            tc::tmem_st8(col + kPLo, wl);
          }
        }
        float rs0, rs1;
        tc::f2_unpack(rs2, rs0, rs1);
        lp += rs0 + rs1;
        // O holds the products through block j-1 (complete: S_j was issued after them and its
        // completion was signalled); a moved reference max rescales this half of its columns
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int c = 0; c < H / 32; ++c) {
            float tmp[32];
            tc::tmem_ld32(tmem + lane_base + TM_O + H * half + 32 * c, tmp);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) tmp[i] *= alpha;
            tc::tmem_st32(tmem + lane_base + TM_O + H * half + 32 * c, tmp);
          }
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&ms->p_full);
      }
    }
    // ---- epilogue: O_s = O / l, log d_s, fusion (Eq. 5, Eq. 4); O through shared memory and a
    // TMA store (or straight to the caller's row with a row map), O_s as fp32 row stores
    const int rb = n_sel & 1;                         // exchange buffer not read in the last loop step
    ms->red[rb][sid] = lp;
    bool have = false;
    if (alive && n_sel > 0) {
      alive = __all_sync(0xffffffffu, wait_or_abort(&ms->pv_done, (n_sel - 1) & 1, ms, err, 128u));
      have = alive;
    }
    if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->olr_full, 0, ms, err, 4096u));
    softmax_bar();
    const float l = ms->red[rb][row] + ms->red[rb][128 + row];
    // every PV product is done: the V stage holds the outgoing O, the K stage the incoming O_lr
    if (alive) {
      if (have) tc::tc_fence_after();
      const size_t ri = head + min(qrow, g.N - 1);
      const float dl = a.dlr[ri];
      const float lam = a.lam ? a.lam[ri] : g.lam;
      const float gs = a.gs ? a.gs[ri] : 1.f;
      const float glr_in = a.glr ? a.glr[ri] : -1.f;
      const float logd = l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const float mf = g.fixed_m ? 1.f : logd == -INFINITY ? 0.f : 1.f / (1.f + (lam * dl + g.eps) * expf(-logd));
      const float gl = a.glr ? glr_in : g.fixed_m ? 1.f : 1.f - mf;
      const float cs = gs * mf;
      const bool row_ok = qrow < g.N;
      // this thread's output columns [col0, col0 + H), 16-byte chunks of 8 bf16 from chunk ch0
      // of their 64-column slab
      const int col0 = H * half, ch0 = (col0 & 63) >> 3;
      const unsigned char* lrow = smem + L::k(0) + (col0 >> 6) * kSlab + row * 128;
      unsigned char* orow = smem + L::v(0) + (col0 >> 6) * kSlab + row * 128;
      // with a row map, O goes straight to the caller's row (8 bf16 per 16-byte unit)
      uint4* grow = a.q_rows && row_ok
                        ? reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.O) +
                                                   (head + a.q_rows[(size_t)bh * a.rows_stride + qrow]) * D + col0)
                        : nullptr;
      float4* srow = row_ok ? reinterpret_cast<float4*>(static_cast<float*>(a.Os) + (head + qrow) * D + col0) : nullptr;
#pragma unroll 1
      for (int c2 = 0; c2 < H / 32; ++c2) {
        float o[32];
        if (have) {
          tc::tmem_ld32(tmem + lane_base + TM_O + col0 + 32 * c2, o);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int ch = 4 * c2 + cc;
          const int sw = ((ch0 + ch) ^ (row & 7)) << 4;
          const uint4 lr = *reinterpret_cast<const uint4*>(lrow + sw);
          const __nv_bfloat16* lv = reinterpret_cast<const __nv_bfloat16*>(&lr);
          uint32_t wo[4];
          float sv8[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float s0 = o[8 * cc + 2 * e] * inv_l, s1 = o[8 * cc + 2 * e + 1] * inv_l;
            sv8[2 * e] = s0;
            sv8[2 * e + 1] = s1;
            wo[e] = pack_bf16(cs * s0 + gl * __bfloat162float(lv[2 * e]), cs * s1 + gl * __bfloat162float(lv[2 * e + 1]));
          }
          if (a.q_rows) {
            if (grow) grow[ch] = make_uint4(wo[0], wo[1], wo[2], wo[3]);
          } else {
            *reinterpret_cast<uint4*>(orow + sw) = make_uint4(wo[0], wo[1], wo[2], wo[3]);
          }
          // O_s in fp32 (the backward's softmax delta is formed from it)
          if (srow) {
            srow[2 * ch] = make_float4(sv8[0], sv8[1], sv8[2], sv8[3]);
            srow[2 * ch + 1] = make_float4(sv8[4], sv8[5], sv8[6], sv8[7]);
          }
        }
      }
      if (half == 0 && row_ok) {
        a.logd[head + qrow] = logd;
        a.m[head + qrow] = mf;
      }
    }
    tc::fence_proxy_async_smem();
    softmax_bar();
    if (threadIdx.x == 64 && !*(volatile int*)&ms->abort_flag && !a.q_rows && a.O) {
      for (int sl = 0; sl < D / 64; ++sl) tma_store_3d(&tmO, smem + L::v(0) + sl * kSlab, 64 * sl, row0, bh);
      asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch.
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

// [BH][N][d] bf16 viewed as a 3-D tensor (column, row, head); boxes of 64 columns x `rows`
// rows, 128-byte swizzle; loads past row N read zeros, stores past row N are dropped.
static bool make_map(CUtensorMap* m, const void* base, int d, int N, int BH, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool attn_fwd_tc_supported(const Geom& g) { return (g.d == 64 || g.d == 128) && (g.T == 64 || g.T == 128); }

template <int D, bool PAIR>
static cudaError_t fwd_t(const FwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  constexpr int TB = PAIR ? 64 : 128;
  if (PAIR && a.tile_list && (a.n_list & 1)) return cudaErrorInvalidValue;   // tile pairs
  CUtensorMap mq, mk, mv, mlr, mo;
  if (!make_map(&mq, a.Q, D, g.N, g.BH, kT) || !make_map(&mk, a.K, D, g.N, g.BH, TB) ||
      !make_map(&mv, a.V, D, g.N, g.BH, TB) || !make_map(&mlr, a.Olr, D, g.N, g.BH, kT) ||
      !make_map(&mo, a.O ? a.O : a.Q, D, g.N, g.BH, kT))    // without O the map is not used
    return cudaErrorInvalidValue;
  auto kern = attn_fwd_tc_kernel<D, PAIR>;
  constexpr size_t smem = smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int units = a.tile_list ? (PAIR ? a.n_list / 2 : a.n_list) : (PAIR ? (g.n_t + 1) / 2 : g.n_t);
  ProfScope ps("attn_fwd_tc", st);
  kern<<<dim3(units, g.BH), kThreads, smem, st>>>(mq, mk, mv, mlr, mo, a, g, err);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_tc(const FwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  if (!attn_fwd_tc_supported(g)) return cudaErrorInvalidValue;
  if (g.d == 64) return g.T == 64 ? fwd_t<64, true>(a, g, err, st) : fwd_t<64, false>(a, g, err, st);
  return g.T == 64 ? fwd_t<128, true>(a, g, err, st) : fwd_t<128, false>(a, g, err, st);
}

}  // namespace elsaa
