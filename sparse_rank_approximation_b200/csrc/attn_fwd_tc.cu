// Sparse-branch forward on the 5th-generation tensor cores (tcgen05 + TMEM), fused
// with the denominator-aware fusion epilogue (ELSAA paper §3.2, §3.3 Eq. 5, §1 Eq. 4).
// Head dimension D = 64 or 128.  A CTA works on 128 query rows: one tile of 128 queries
// with 128-key blocks, or (PAIR, blocks of 64) the two adjacent 64-query tiles 2u and
// 2u + 1, whose selected blocks are staged side by side: the K and V stage of step j
// holds tile 2u's j-th block in rows 0-63 and tile 2u + 1's in rows 64-127, so every
// product stays M = N = 128 and each query row masks the other tile's 64 keys.
//
// One CTA per (head, 128 query rows), 11 warps:
//   warp 0      TMA producer of Q and of the K ring (3 stages); once the last
//               score MMA is done it prefetches the tile's low-rank output O_lr
//               into a K stage for the epilogue;
//   warp 1      TMEM owner and MMA issuer: S_j = Q K_j^T into one of two TMEM
//               score buffers, then O += P_{j-1} V_{j-1} into the TMEM output
//               with P_{j-1} read from tensor memory;
//   warp 2      TMA producer of the V ring (3 stages);
//   warps 3-10  softmax: each query row is split over two warps, one per half
//               of the key columns; each half keeps its own running max, row
//               sum and output accumulator O_h = sum over its keys of P V (the
//               PV product of a block is two products of 64 keys, one per
//               half), so the halves never wait on each other inside the loop;
//               online softmax in fp32 with lazy rescaling (O_h and l_h are
//               rescaled only when the half's running max grows by more than
//               2^16, after P_j is written and just before it is released);
//               P_j (bf16 pairs) overwrites the score columns it came from and
//               is the A operand of the PV product; the epilogue merges the two
//               halves (one exchange of max and sum), normalises O, applies the
//               fusion and writes O and O_s through shared memory with TMA stores.
// Operand tiles are 64-column slabs with 128-byte swizzle, as TMA writes them.
// Every mbarrier wait is bounded; a timeout sets a bit in the caller's error
// word, the CTA drains its copies and MMAs, frees TMEM and exits.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace elsaa {

namespace {

constexpr int kT = 128;                  // query rows of a CTA = keys of a K/V stage
constexpr uint32_t kSlab = kT * 128;     // one [128 rows][64 bf16] swizzled slab
constexpr uint32_t kTile = 2 * kSlab;    // 128 x 128 bf16
constexpr uint32_t OFF_Q = 0;
constexpr int kStages = 3;                 // K and V ring depth
__host__ __device__ constexpr uint32_t off_k(int s) { return kTile * (1 + s); }              // K stage s
__host__ __device__ constexpr uint32_t off_v(int s) { return kTile * (1 + kStages + s); }    // V stage s
constexpr uint32_t OFF_MISC = (1 + 2 * kStages) * kTile;
// column of the K = 16 step kk of P_hi (key 64 h + m of a row sits at column 64 h + m / 2);
// P_lo = bf16(P - P_hi) sits 32 columns further, over score columns already read
__host__ __device__ constexpr uint32_t p_col(int kk) { return (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8); }
constexpr uint32_t kPLo = 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t TM_O0 = 0, TM_O1 = 384;                 // output accumulators of the two key halves
__host__ __device__ constexpr uint32_t tm_s(int s) { return 128u + 128u * s; }         // score buffer s
constexpr float kRescaleThreshold = 16.f;                // log2 units: P stays below 2^16
constexpr int kThreads = 352;
constexpr int kSoftmaxThreads = 256;

struct Misc {
  uint64_t q_full, k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages], s_full[2],
      p_full[2][2], pv_done[2][2];       // [score buffer][key half]
  uint64_t olr_full, drain, never;
  unsigned long long limit_ns;
  uint32_t tmem_base;
  int abort_flag;
  int idx[2][32];         // selected blocks of the CTA's tile (PAIR: of its two tiles)
  float mx_half[256], l_half[256];   // each half's reference max and row sum, for the merge
};
constexpr size_t kSmemBytes = OFF_MISC + sizeof(Misc);
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
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
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmLr,
                       const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmS, FwdArgs a,
                       Geom g, uint32_t* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  Misc* ms = reinterpret_cast<Misc*>(smem + OFF_MISC);
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
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&ms->k_full[s], 1);
      tc::mbar_init(&ms->k_empty[s], 1);
      tc::mbar_init(&ms->v_full[s], 1);
      tc::mbar_init(&ms->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&ms->s_full[s], 1);
      for (int h = 0; h < 2; ++h) {
        tc::mbar_init(&ms->p_full[s][h], kSoftmaxThreads / 2);
        tc::mbar_init(&ms->pv_done[s][h], 1);
      }
    }
    tc::mbar_init(&ms->olr_full, 1);
    tc::mbar_init(&ms->drain, 1);
    tc::mbar_init(&ms->never, 1);
    ms->limit_ns = g.wait_ns;
    ms->abort_flag = 0;
    tc::fence_barrier_init();
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

  if (warp == 0 || warp == 2) {
    // ================= TMA producers: warp 0 Q, K ring, O_lr; warp 2 the V ring =================
    if (lane == 0) {
      const bool is_k = warp == 0;
      uint64_t* full = is_k ? ms->k_full : ms->v_full;
      uint64_t* empty = is_k ? ms->k_empty : ms->v_empty;
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      int issued = 0;
      constexpr uint32_t kTD = 128u * D * 2;      // bytes of a [128][D] tile
      if (is_k) {
        tc::mbar_arrive_expect_tx(&ms->q_full, kTD);
        for (int sl = 0; sl < D / 64; ++sl) tc::tma_load_3d(smem + OFF_Q + sl * kSlab, &tmQ, &ms->q_full, 64 * sl, row0, bh);
      }
      bool alive = true;
      for (int j = 0; j < n_sel; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !wait_or_abort(&empty[s], ((j / kStages) - 1) & 1, ms, err, is_k ? 1u : 512u)) {
          alive = false;
          break;
        }
        unsigned char* dst = smem + (is_k ? off_k(s) : off_v(s));
        tc::mbar_arrive_expect_tx(&full[s], kTD);
        for (int h = 0; h < (PAIR ? 2 : 1); ++h) {
          // PAIR: a tile with fewer blocks stages block 0 in its half (every score of it is masked)
          const int b = j < (h ? n_sel_t[1] : n_sel_t[0]) ? sel(h, j) : 0;
          for (int sl = 0; sl < D / 64; ++sl)
            tc::tma_load_3d(dst + sl * kSlab + h * 64 * 128, map, &full[s], 64 * sl, b * TB, bh);
        }
        issued = j + 1;
      }
      bool lr_issued = false;
      if (is_k && alive) {
        // the low-rank output goes into K stage 0 once every score MMA has read its K tile
        for (int j = (n_sel > kStages ? n_sel - kStages : 0); alive && j < n_sel; ++j)
          alive = wait_or_abort(&ms->k_empty[j % kStages], (j / kStages) & 1, ms, err, 2048u);
        if (alive) {
          tc::mbar_arrive_expect_tx(&ms->olr_full, kTD);
          for (int sl = 0; sl < D / 64; ++sl)
            tc::tma_load_3d(smem + off_k(0) + sl * kSlab, &tmLr, &ms->olr_full, 64 * sl, row0, bh);
          lr_issued = true;
        }
      }
      // drain: every copy this thread started has landed before the CTA may exit
      if (is_k) tc::mbar_wait(&ms->q_full, 0);
      if (lr_issued) tc::mbar_wait(&ms->olr_full, 0);
      for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
        tc::mbar_wait(&full[j % kStages], (j / kStages) & 1);
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t idS = tc::idesc_bf16(128, 128, false, false);   // Q (K-major) x K (K-major)
      const uint32_t idPV = tc::idesc_bf16(128, D, false, true);     // P (TMEM) x V (MN-major)
      const uint32_t sbase = smem_u32(smem);
      bool ok = wait_or_abort(&ms->q_full, 0, ms, err, 2u);
      int pv_issued = 0;
      // O_h += P_jj[:, keys of half h] V_jj[keys of half h, :], each half as soon as its P is
      // written
      auto issue_pv = [&](int jj) -> bool {
        const uint32_t vb = sbase + off_v(jj % kStages);
        for (int h = 0; h < 2; ++h) {
          if (!wait_or_abort(&ms->p_full[jj & 1][h], (jj >> 1) & 1, ms, err, 4u)) return false;
          if (h == 0 && !wait_or_abort(&ms->v_full[jj % kStages], (jj / kStages) & 1, ms, err, 1024u)) return false;
          tc::tc_fence_after();
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int kk = 4 * h + k4;                  // keys 16 kk .. 16 kk + 15
            const uint64_t bd = tc::sw128_desc(vb + kk * 2048, kSlab, 1024);
            const uint32_t pa = tmem + tm_s(jj & 1) + p_col(kk);
            tc::mma_bf16_ts(tmem + (h ? TM_O1 : TM_O0), pa, bd, idPV, (jj > 0 || k4 > 0) ? 1u : 0u);
            tc::mma_bf16_ts(tmem + (h ? TM_O1 : TM_O0), pa + kPLo, bd, idPV, 1u);
          }
          tc::mma_commit(&ms->pv_done[jj & 1][h]);
        }
        tc::mma_commit(&ms->v_empty[jj % kStages]);
        pv_issued = jj + 1;
        return true;
      };
      // S_j reuses the TMEM columns of P_{j-2}: the PV product that reads them was issued
      // earlier, and tcgen05 MMAs of one thread run in issue order
      for (int j = 0; ok && j < n_sel; ++j) {
        const int s = j & 1, sk = j % kStages;
        if (!wait_or_abort(&ms->k_full[sk], (j / kStages) & 1, ms, err, 8u)) break;
        tc::tc_fence_after();
        const uint32_t kb = sbase + off_k(sk);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = tc::sw128_desc(sbase + OFF_Q + (kk >> 2) * kSlab + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = tc::sw128_desc(kb + (kk >> 2) * kSlab + (kk & 3) * 32, 16, 1024);
          tc::mma_bf16(tmem + tm_s(s), ad, bd, idS, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&ms->s_full[s]);
        tc::mma_commit(&ms->k_empty[sk]);
        if (j >= 1 && !issue_pv(j - 1)) break;
      }
      if (n_sel > 0 && pv_issued == n_sel - 1) issue_pv(n_sel - 1);
      // drain: all MMAs this thread issued have completed
      tc::mma_commit(&ms->drain);
      tc::mbar_wait(&ms->drain, 0);
    }
  } else {
    // ================= softmax / epilogue: half a query row per thread =================
    const int q4 = warp & 3;
    const int half = (warp - 3) >> 2;                // score columns [64 half, +64), output [H half, +H)
    const int row = 32 * q4 + lane;
    const int sid = half * 128 + row;                // slot in the merge arrays
    const uint32_t o_mine = half ? TM_O1 : TM_O0;    // this half's output accumulator
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
    const size_t ri = head + min(qrow, g.N - 1);
    // per-row fusion inputs, fetched now so their latency hides behind the main loop
    const float dl = a.dlr[ri];
    const float lam = a.lam ? a.lam[ri] : g.lam;
    const float gs = a.gs ? a.gs[ri] : 1.f;
    const float glr_in = a.glr ? a.glr[ri] : -1.f;
    float m_used = -INFINITY, lp = 0.f;              // this half's reference max (scaled log2 units), row sum
    bool alive = true;                               // warp-uniform; every barrier below is still taken
    // test hook: a wait on a barrier nothing completes, so the give-up path runs
    if (g.debug_stall) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->never, 0, ms, err, 0x40000u));
    for (int j = 0; j < n_sel; ++j) {
      const int s = j & 1;
      float sv[64];
      if (alive) {
        alive = __all_sync(0xffffffffu, wait_or_abort(&ms->s_full[s], (j >> 1) & 1, ms, err, 32u));
      }
      if (alive) {
        tc::tc_fence_after();
        float tmp[32];
        tc::tmem_ld32(tmem + lane_base + tm_s(s) + 64 * half, tmp);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[i] = tmp[i];
        tc::tmem_ld32(tmem + lane_base + tm_s(s) + 64 * half + 32, tmp);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[32 + i] = tmp[i];
        tc::tmem_wait_ld();
        // key k of this half's 64 columns is key c0 + k of block b (no block: all masked)
        const bool none = dead_half || j >= my_n;
        const int b = none ? 0 : sel(PAIR ? half : 0, j);
        const int c0 = PAIR ? 0 : 64 * half;
        const int kvalid = g.N - b * TB;
        const bool diag = g.causal && b == my_tile;
        if (none) {
#pragma unroll
          for (int c = 0; c < 64; ++c) sv[c] = -INFINITY;
        } else if (diag || kvalid < TB) {            // only the diagonal / ragged block masks
          const int lim = min(kvalid - 1, diag ? qpos : TB - 1) - c0;
#pragma unroll
          for (int c = 0; c < 64; ++c) sv[c] = c > lim ? -INFINITY : sv[c];
        }
        float m4[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
        for (int c = 4; c < 64; c += 4) {
          m4[0] = fmaxf(m4[0], sv[c]);
          m4[1] = fmaxf(m4[1], sv[c + 1]);
          m4[2] = fmaxf(m4[2], sv[c + 2]);
          m4[3] = fmaxf(m4[3], sv[c + 3]);
        }
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
        // lazy rescaling: move the reference max only when this half's max grew by > 2^16
        const float m_new = fmaxf(m_used, mx);
        const bool resc = m_new > m_used + kRescaleThreshold;     // false while both are -inf
        float alpha = 1.f;
        if (resc) {
          alpha = (m_used == -INFINITY) ? 0.f : exp2f(m_used - m_new);
          lp *= alpha;
          m_used = m_new;
        }
        // P_j as bf16 hi + lo pairs (16 significant bits, so O_s and the backward's softmax delta
        // formed from it carry no bf16 rounding of the weights) over this thread's score
        // columns: the PV product of block j-2 read that buffer before S_j was written into it
        const float msub = m_used == -INFINITY ? 0.f : m_used;
        float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t w[8], wl[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float p0 = ex2_approx(fmaf(sv[16 * ch + 2 * e], sl2, -msub));
            const float p1 = ex2_approx(fmaf(sv[16 * ch + 2 * e + 1], sl2, -msub));
            rs0 += p0;
            rs1 += p1;
            w[e] = pack_bf16(p0, p1);
            wl[e] = pack_bf16(p0 - __uint_as_float(w[e] << 16), p1 - __uint_as_float(w[e] & 0xffff0000u));
          }
          tc::tmem_st8(tmem + lane_base + tm_s(s) + 64 * half + 8 * ch, w);
          tc::tmem_st8(tmem + lane_base + tm_s(s) + 64 * half + kPLo + 8 * ch, wl);
        }
        lp += rs0 + rs1;
        tc::tmem_wait_st();
        // O_h holds this half's products through block j-1; a moved reference max rescales it
        // once that product is done, before P_j is released to the MMA warp
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
          alive = __all_sync(0xffffffffu, wait_or_abort(&ms->pv_done[(j - 1) & 1][half], ((j - 1) >> 1) & 1, ms,
                                                        err, 64u));
          if (alive) {
            tc::tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              float tmp[32];
              tc::tmem_ld32(tmem + lane_base + o_mine + 32 * c, tmp);
              tc::tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) tmp[i] *= alpha;
              tc::tmem_st32(tmem + lane_base + o_mine + 32 * c, tmp);
            }
            tc::tmem_wait_st();
          }
        }
        if (alive) {
          tc::tc_fence_before();
          tc::mbar_arrive(&ms->p_full[s][half]);
        }
      }
    }
    // ---- epilogue: merge the two halves (O = f0 O_0 + f1 O_1, l = f0 l_0 + f1 l_1 with
    // f_h = 2^(m_h - max(m_0, m_1))), O_s = O / l, log d_s, fusion (Eq. 5, Eq. 4), TMA stores
    // from shared memory
    ms->mx_half[sid] = m_used;
    ms->l_half[sid] = lp;
    bool have = false;
    if (alive && n_sel > 0) {
      const int jl = n_sel - 1;
      alive = __all_sync(0xffffffffu, wait_or_abort(&ms->pv_done[jl & 1][0], (jl >> 1) & 1, ms, err, 128u));
      if (alive)
        alive = __all_sync(0xffffffffu, wait_or_abort(&ms->pv_done[jl & 1][1], (jl >> 1) & 1, ms, err, 128u));
      have = alive;
    }
    if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->olr_full, 0, ms, err, 4096u));
    softmax_bar();
    const float m0 = ms->mx_half[row], m1 = ms->mx_half[128 + row];
    const float mm = fmaxf(m0, m1);
    const float f0 = m0 == -INFINITY ? 0.f : exp2f(m0 - mm);
    const float f1 = m1 == -INFINITY ? 0.f : exp2f(m1 - mm);
    const float l = f0 * ms->l_half[row] + f1 * ms->l_half[128 + row];
    float o[H];
#pragma unroll
    for (int c = 0; c < H; ++c) o[c] = 0.f;
    if (have && alive) {
      tc::tc_fence_after();
#pragma unroll
      for (int c2 = 0; c2 < H / 32; ++c2) {
        float t0[32], t1[32];
        tc::tmem_ld32(tmem + lane_base + TM_O0 + H * half + 32 * c2, t0);
        tc::tmem_ld32(tmem + lane_base + TM_O1 + H * half + 32 * c2, t1);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[32 * c2 + i] = f0 * t0[i] + f1 * t1[i];
      }
    }
    // every PV product is done: V stage 0 holds the outgoing O, V stages 1 (and 2) the fp32 O_s
    if (alive) {
      const float logd = l > 0.f ? (mm + log2f(l)) * kLn2 : -INFINITY;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const float mf = g.fixed_m ? 1.f : logd == -INFINITY ? 0.f : 1.f / (1.f + (lam * dl + g.eps) * expf(-logd));
      const float gl = a.glr ? glr_in : g.fixed_m ? 1.f : 1.f - mf;
      const float cs = gs * mf;
      // this thread's output columns [col0, col0 + H), 16-byte chunks of 8 bf16 from chunk ch0
      // of their 64-column slab
      const int col0 = H * half, ch0 = (col0 & 63) >> 3;
      const unsigned char* lrow = smem + off_k(0) + (col0 >> 6) * kSlab + row * 128;
      unsigned char* orow = smem + off_v(0) + (col0 >> 6) * kSlab + row * 128;
      // with a row map, O goes straight to the caller's row (8 bf16 per 16-byte unit)
      uint4* grow = a.q_rows && qrow < g.N
                        ? reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.O) +
                                                   (head + a.q_rows[(size_t)bh * a.rows_stride + qrow]) * D + col0)
                        : nullptr;
#pragma unroll
      for (int ch = 0; ch < H / 8; ++ch) {
        const int sw = ((ch0 + ch) ^ (row & 7)) << 4;
        const uint4 lr = *reinterpret_cast<const uint4*>(lrow + sw);
        const __nv_bfloat16* lv = reinterpret_cast<const __nv_bfloat16*>(&lr);
        uint32_t wo[4];
        float sv[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float s0 = o[8 * ch + 2 * e] * inv_l, s1 = o[8 * ch + 2 * e + 1] * inv_l;
          sv[2 * e] = s0;
          sv[2 * e + 1] = s1;
          wo[e] = pack_bf16(cs * s0 + gl * __bfloat162float(lv[2 * e]), cs * s1 + gl * __bfloat162float(lv[2 * e + 1]));
        }
        if (a.q_rows) {
          if (grow) grow[ch] = make_uint4(wo[0], wo[1], wo[2], wo[3]);
        } else {
          *reinterpret_cast<uint4*>(orow + sw) = make_uint4(wo[0], wo[1], wo[2], wo[3]);
        }
        // O_s in fp32 (the backward's softmax delta is formed from it): boxes of [128 rows][32
        // floats] with the 128-byte swizzle over the V stages after the first; column fc sits
        // in box fc / 32, 16-byte chunk (fc % 32) / 4
        const int fc = col0 + 8 * ch;
        unsigned char* sbox = smem + off_v(1) + (fc >> 5) * kSlab + row * 128;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int cc = ((fc & 31) >> 2) + e;
          *reinterpret_cast<float4*>(sbox + ((cc ^ (row & 7)) << 4)) =
              make_float4(sv[4 * e], sv[4 * e + 1], sv[4 * e + 2], sv[4 * e + 3]);
        }
      }
      if (half == 0 && qrow < g.N) {
        a.logd[head + qrow] = logd;
        a.m[head + qrow] = mf;
      }
    }
    tc::fence_proxy_async_smem();
    softmax_bar();
    if (threadIdx.x == 96 && !*(volatile int*)&ms->abort_flag) {
      if (!a.q_rows)
        for (int sl = 0; sl < D / 64; ++sl) tma_store_3d(&tmO, smem + off_v(0) + sl * kSlab, 64 * sl, row0, bh);
      for (int b = 0; b < D / 32; ++b) tma_store_3d(&tmS, smem + off_v(1) + b * kSlab, 32 * b, row0, bh);
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

// [BH][N][d] fp32 viewed as (column, row, head); boxes of 32 x 128 x 1 (128-byte rows),
// 128-byte swizzle; stores past row N are dropped.
static bool make_map_f32(CUtensorMap* m, void* base, int d, int N, int BH) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)N * d * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)kT, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool attn_fwd_tc_supported(const Geom& g) { return (g.d == 64 || g.d == 128) && (g.T == 64 || g.T == 128); }

template <int D, bool PAIR>
static cudaError_t fwd_t(const FwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  constexpr int TB = PAIR ? 64 : 128;
  if (PAIR && a.tile_list && (a.n_list & 1)) return cudaErrorInvalidValue;   // tile pairs
  CUtensorMap mq, mk, mv, mlr, mo, ms;
  if (!make_map(&mq, a.Q, D, g.N, g.BH, kT) || !make_map(&mk, a.K, D, g.N, g.BH, TB) ||
      !make_map(&mv, a.V, D, g.N, g.BH, TB) || !make_map(&mlr, a.Olr, D, g.N, g.BH, kT) ||
      !make_map(&mo, a.O, D, g.N, g.BH, kT) || !make_map_f32(&ms, a.Os, D, g.N, g.BH))
    return cudaErrorInvalidValue;
  auto kern = attn_fwd_tc_kernel<D, PAIR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int units = a.tile_list ? (PAIR ? a.n_list / 2 : a.n_list) : (PAIR ? (g.n_t + 1) / 2 : g.n_t);
  ProfScope ps("attn_fwd_tc", st);
  kern<<<dim3(units, g.BH), kThreads, kSmemBytes, st>>>(mq, mk, mv, mlr, mo, ms, a, g, err);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_tc(const FwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  if (!attn_fwd_tc_supported(g)) return cudaErrorInvalidValue;
  if (g.d == 64) return g.T == 64 ? fwd_t<64, true>(a, g, err, st) : fwd_t<64, false>(a, g, err, st);
  return g.T == 64 ? fwd_t<128, true>(a, g, err, st) : fwd_t<128, false>(a, g, err, st);
}

}  // namespace elsaa
