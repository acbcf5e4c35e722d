// RACE chunk statistics on the 5th-generation tensor cores (ELSAA paper §3.1: causal
// chunks read the prefix sums of the bucket statistics of the chunks before them), for
// d = 64 or 128, chunk C = 128, and the features in groups of 128 (one launch pair per group).
//
// Chunk c contributes S_c = Phi_c^T [Y_c | w_c]: the value statistics (r x d) and the
// mass column (r) of every bucket.  Forward: Phi = Phi(K), Y = V, w = 1, and chunk c
// reads the exclusive prefix P_c = sum_{c' < c} S_c' (all chunks' sum when non-causal).
// Backward: Phi = Phi(Q), Y = cl dO, w = delta, and chunk c reads the exclusive suffix
// R_c = sum_{c' > c} S_c'.  The consumers (read-out and the two backward kernels) load
// each chunk's statistics as bf16 hi + lo halves [r][d] and the mass in fp32.
//
// Two launches around a scan of the segment totals:
//   totals   one CTA per segment of `seg` chunks: S summed over the segment in tensor
//            memory (the mass on the CUDA cores), written once as fp32 [r][d + 8];
//   (race_scan_kernel turns the totals into each segment's exclusive prefix / suffix)
//   emit     one CTA per segment again: the running statistics start at the segment's
//            carry, stay in registers in fp32, and before each chunk's S_c is added the
//            running value goes out as that chunk's bf16 hi + lo tiles (TMA stores) and
//            mass.  No per-chunk fp32 prefix is ever written.
// S_c = Phi_c^T Y_c is one M = r, N = d, K = C product with both operands MN-major, as
// TMA writes the [C rows][r] and [C rows][d] tiles; the mass Phi_c^T w_c is a second, N = 16
// product against a K-major tile whose rows 0 and 1 hold w as bf16 hi and lo (the rest zero),
// so the mass carries w to 16 significant bits.
// Warps: 0 TMA producer, 1 TMEM owner and MMA issuer, 2-9 (256 threads) compute: TMEM
// lane quarter = warp % 4 (bucket row f of the statistics), column half = (warp - 2) / 4;
// the first 128 of them write the chunk's weight tile.
// Every mbarrier wait is bounded; a timeout sets a bit in the caller's error word, the CTA
// drains its copies and products, frees its tensor memory and exits.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace elsaa {

namespace {

constexpr int kC = 128;                           // chunk rows
constexpr int kR = 128;                           // buckets (r = 16 L)
constexpr uint32_t kSlab = 128 * 128;             // [128 rows][64 bf16], 128-byte swizzle
constexpr uint32_t kTile = 2 * kSlab;             // [128 rows][128 bf16]
constexpr int kThreads = 320;
constexpr int kComputeThreads = 256;
constexpr int kMaxStages = 3;

constexpr uint32_t kWTile = 2 * 16 * 128;         // weight tile: [16 rows][128 rows of the chunk], K-major
template <bool EMIT>
struct StatsLayout {
  static constexpr int stages = EMIT ? 2 : 3;     // emit keeps 64 KB of staging for the stores
  static constexpr uint32_t phi(int s) { return (uint32_t)s * 2 * kTile; }
  static constexpr uint32_t y(int s) { return phi(s) + kTile; }
  static constexpr uint32_t hi = (uint32_t)stages * 2 * kTile;       // staging of the outgoing tiles
  static constexpr uint32_t lo = hi + kTile;
  static constexpr uint32_t wt0 = EMIT ? lo + kTile : hi;            // weight tiles [stages]
  static constexpr uint32_t wt(int s) { return wt0 + (uint32_t)s * kWTile; }
  static constexpr uint32_t bars = wt0 + (uint32_t)kMaxStages * kWTile;
  // TMEM: the S accumulator(s) at 0 (and 128), the mass accumulator(s) after them
  static constexpr uint32_t tmem_cols = EMIT ? 512 : 256;
  static constexpr uint32_t mass_col(int b) { return (EMIT ? 256u : 128u) + 16u * b; }
};

struct StatBars {
  uint64_t full[kMaxStages], empty[kMaxStages], w_full[kMaxStages], x_full[2], x_free[2], drain;
  unsigned long long limit_ns;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, StatBars* ms, uint32_t* err,
                                              uint32_t code) {
  if (*(volatile int*)&ms->abort_flag) return false;
  if (tc::mbar_wait(bar, parity, ms->limit_ns)) return true;
  *(volatile int*)&ms->abort_flag = 1;
  if (err) atomicOr(err, code);
  return false;
}

__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }

// Operand descriptors are built once from the shared-memory base (`d0`, with the layout's
// leading offset); an operand at byte offset `off` and its K = 16 step kk only move the start
// address.
// MN-major operand: K = 16 rows per step, 64-element M (or N) atoms kSlab bytes apart.
__device__ __forceinline__ uint64_t desc_mn(uint64_t d0, uint32_t off, int kk) {
  return tc::desc_adv(d0, off + (uint32_t)kk * 2048u);
}

// K-major operand, K = 16 step kk of a tile of 128-byte rows kept as 64-column slabs.
__device__ __forceinline__ uint64_t desc_k(uint64_t d0, uint32_t off, int kk, uint32_t slab) {
  return tc::desc_adv(d0, off + (uint32_t)(kk >> 2) * slab + (uint32_t)(kk & 3) * 32u);
}

// bf16 element (row, col) of a [128][128] tile kept as two 64-column slabs with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
  return (uint32_t)(col >> 6) * kSlab + (uint32_t)row * 128u + (uint32_t)((((col & 63) >> 3) ^ (row & 7)) << 4) +
         (uint32_t)(col & 7) * 2u;
}

__device__ __forceinline__ void split2(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];\n"
               :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2) : "memory");
}

}  // namespace

// grid (n_seg, BH), kThreads threads.  bwd: chunks walk in descending order, the carry is the
// suffix slot.  w: per-row mass weights [BH][N] (null: 1).  Atot: [BH][n_seg + 1][r][d + 8]
// fp32 (totals: slot seg + 1 written; emit: the scanned carry read).
template <bool EMIT, int D>
__global__ void __launch_bounds__(kThreads, 1)
    race_stats_tc_kernel(const __grid_constant__ CUtensorMap tmPhi, const __grid_constant__ CUtensorMap tmY,
                         const __grid_constant__ CUtensorMap tmOut, const float* __restrict__ w,
                         float* __restrict__ Atot, float* __restrict__ mass_out, int bwd, Geom g, uint32_t* err) {
  using Lay = StatsLayout<EMIT>;
  constexpr int NS = Lay::stages;
  extern __shared__ __align__(1024) unsigned char smem[];
  StatBars* ms = reinterpret_cast<StatBars*>(smem + Lay::bars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int c_begin = seg * g.seg, c_end = min(g.n_c, c_begin + g.seg);
  const int n_here = max(0, c_end - c_begin);
  const bool accumulate = !EMIT || g.causal;     // emit without causality: every chunk gets the total
  const int n_load = accumulate ? n_here : 0;
  const size_t state = (size_t)kR * g.dp;
  auto chunk_of = [&](int s) { return bwd ? c_end - 1 - s : c_begin + s; };
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0 && err) atomicOr(err, 0x80000000u);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(&ms->full[s], 1);
      tc::mbar_init(&ms->empty[s], 1);                     // the products' commit
      tc::mbar_init(&ms->w_full[s], 128);                  // the weight tile's 128 writers
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&ms->x_full[b], 1);
      tc::mbar_init(&ms->x_free[b], kComputeThreads);
    }
    tc::mbar_init(&ms->drain, 1);
    ms->limit_ns = g.wait_ns;
    ms->abort_flag = 0;
    tc::fence_barrier_init();
  }
  // weight tiles: rows 2-15 stay zero (rows 0 and 1 are rewritten for every chunk)
  for (int i = threadIdx.x; i < (int)(NS * kWTile / 16); i += kThreads)
    reinterpret_cast<uint4*>(smem + Lay::wt0)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (warp == 1) {
    tc::tmem_alloc(&ms->tmem_base, Lay::tmem_cols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer: the chunk's Phi and Y tiles ----------------
    if (lane == 0) {
      int issued = 0;
      for (int s = 0; s < n_load; ++s) {
        const int st = s % NS;
        if (s >= NS && !wait_or_abort(&ms->empty[st], ((s / NS) - 1) & 1, ms, err, 0x100000u)) break;
        const int c = chunk_of(s);
        tc::mbar_arrive_expect_tx(&ms->full[st], kTile + 128u * D * 2);
        for (int h = 0; h < 2; ++h)
          tc::tma_load_3d(smem + Lay::phi(st) + h * kSlab, &tmPhi, &ms->full[st], 64 * h, c * kC, bh);
        for (int h = 0; h < D / 64; ++h)
          tc::tma_load_3d(smem + Lay::y(st) + h * kSlab, &tmY, &ms->full[st], 64 * h, c * kC, bh);
        issued = s + 1;
      }
      // drain: every copy this thread started has landed before the CTA may exit
      for (int s = (issued > NS ? issued - NS : 0); s < issued; ++s) tc::mbar_wait(&ms->full[s % NS], (s / NS) & 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: S_c = Phi_c^T Y_c ----------------
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(128, D, true, true);    // A = Phi^T and B = Y, both MN-major
      const uint32_t idm = tc::idesc_bf16(128, 16, true, false);    // A = Phi^T, B = the weight tile (K-major)
      const uint32_t sb = smem_u32(smem);
      const uint64_t dmn = tc::sw128_desc(sb, kSlab, 1024), dk = tc::sw128_desc(sb, 16, 1024);
      for (int s = 0; s < n_load; ++s) {
        const int st = s % NS, buf = EMIT ? (s & 1) : 0;
        if (!wait_or_abort(&ms->full[st], (s / NS) & 1, ms, err, 0x200000u)) break;
        if (!wait_or_abort(&ms->w_full[st], (s / NS) & 1, ms, err, 0x200000u)) break;
        if (EMIT && s >= 2 && !wait_or_abort(&ms->x_free[buf], ((s >> 1) - 1) & 1, ms, err, 0x400000u)) break;
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk) {
          const uint32_t acc = (EMIT ? kk > 0 : (s > 0 || kk > 0)) ? 1u : 0u;
          tc::mma_bf16(tmem + 128u * buf, desc_mn(dmn, Lay::phi(st), kk), desc_mn(dmn, Lay::y(st), kk), idesc, acc);
          tc::mma_bf16(tmem + Lay::mass_col(buf), desc_mn(dmn, Lay::phi(st), kk), desc_k(dk, Lay::wt(st), kk, 2048u),
                       idm, acc);
        }
        tc::mma_commit(&ms->empty[st]);
        if (EMIT) tc::mma_commit(&ms->x_full[buf]);
      }
      if (!EMIT) tc::mma_commit(&ms->x_full[0]);                       // the segment's sum is complete
      tc::mma_commit(&ms->drain);
      tc::mbar_wait(&ms->drain, 0);
    }
  } else {
    // ---------------- compute: bucket row f, columns 64 hc .. 64 hc + 63 ----------------
    const int ct = threadIdx.x - 64;
    const int q4 = warp & 3, hc = (warp - 2) >> 2;
    const int f = 32 * q4 + lane;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const size_t head = (size_t)bh * g.N;
    constexpr int H = D / 2;                         // this thread's columns
    float run[H];
    float run_mass = 0.f;
#pragma unroll
    for (int i = 0; i < H; ++i) run[i] = 0.f;
    if (EMIT) {
      // the carry: the exclusive prefix (suffix) of the other segments, after the scan
      const int slot = bwd ? (g.causal ? seg + 1 : 0) : (g.causal ? seg : g.n_seg);
      const float* a = Atot + ((size_t)bh * (g.n_seg + 1) + slot) * state + (size_t)f * g.dp;
#pragma unroll
      for (int q = 0; q < H / 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(a + H * hc + 4 * q);
        run[4 * q] = v.x; run[4 * q + 1] = v.y; run[4 * q + 2] = v.z; run[4 * q + 3] = v.w;
      }
      run_mass = a[D];
    }
    bool alive = true;
    for (int s = 0; s < n_here; ++s) {
      const int c = chunk_of(s);
      if (EMIT) {
        // chunk c's statistics: the running value, as bf16 hi + lo tiles and the fp32 mass
        if (ct == 0) asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
        compute_bar();                                   // the staging is free again
        if (alive) {
#pragma unroll
          for (int ch = 0; ch < H / 8; ++ch) {
            uint32_t h[4], l[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) split2(run[8 * ch + 2 * e], run[8 * ch + 2 * e + 1], h[e], l[e]);
            const uint32_t off = sw_off(f, H * hc + 8 * ch);
            *reinterpret_cast<uint4*>(smem + Lay::hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4*>(smem + Lay::lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
          }
          if (hc == 0) mass_out[((size_t)bh * g.n_c + c) * kR + f] = run_mass;
        }
        tc::fence_proxy_async_smem();
        compute_bar();
        if (ct == 0 && alive) {
          const int z = (bh * g.n_c + c) * 2;
          for (int h = 0; h < D / 64; ++h) {
            tma_store_3d(&tmOut, smem + Lay::hi + h * kSlab, 64 * h, 0, z);
            tma_store_3d(&tmOut, smem + Lay::lo + h * kSlab, 64 * h, 0, z + 1);
          }
          asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
        }
      }
      if (!accumulate) continue;
      const int st = s % NS;
      // the chunk's weight tile (rows 0 and 1: w as bf16 hi and lo, zero past the last row),
      // once the products that read this stage's previous tile are done
      if (ct < kC) {
        if (s >= NS && alive)
          alive = wait_or_abort(&ms->empty[st], ((s / NS) - 1) & 1, ms, err, 0x800000u);
        const int row = c * kC + ct;
        const float wv = row < g.N ? (w ? w[head + row] : 1.f) : 0.f;
        const __nv_bfloat16 whi = __float2bfloat16_rn(wv);
        const __nv_bfloat16 wlo = __float2bfloat16_rn(wv - __bfloat162float(whi));
        unsigned char* t = smem + Lay::wt(st) + (uint32_t)(ct >> 6) * 2048u;
        const uint32_t cb = (uint32_t)(((ct & 63) >> 3) << 4) + (uint32_t)(ct & 7) * 2u;
        *reinterpret_cast<__nv_bfloat16*>(t + 0 * 128 + (cb ^ (0u << 4))) = whi;
        *reinterpret_cast<__nv_bfloat16*>(t + 1 * 128 + (cb ^ (1u << 4))) = wlo;
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(&ms->w_full[st]);
      }
      if (EMIT && alive) {
        const int buf = s & 1;
        alive = __all_sync(0xffffffffu, wait_or_abort(&ms->x_full[buf], (s >> 1) & 1, ms, err, 0x1000000u));
        if (alive) {
          tc::tc_fence_after();
          float x[32];
#pragma unroll
          for (int h2 = 0; h2 < H / 32; ++h2) {
            tc::tmem_ld32(tmem + lane_base + 128u * buf + H * hc + 32u * h2, x);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) run[32 * h2 + i] += x[i];
          }
          float m2[16];
          tc::tmem_ld16(tmem + lane_base + Lay::mass_col(buf), m2);
          tc::tmem_wait_ld();
          run_mass += m2[0] + m2[1];
          tc::tc_fence_before();
          tc::mbar_arrive(&ms->x_free[buf]);
        }
      }
    }
    if (!EMIT) {
      // the segment's total: S from tensor memory, the mass from the CUDA cores
      if (alive && n_here > 0) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->x_full[0], 0, ms, err, 0x2000000u));
      if (alive) {
        tc::tc_fence_after();
        float* o = Atot + ((size_t)bh * (g.n_seg + 1) + seg + 1) * state + (size_t)f * g.dp;
        float x[32];
#pragma unroll
        for (int h2 = 0; h2 < H / 32; ++h2) {
          if (n_here > 0) {
            tc::tmem_ld32(tmem + lane_base + H * hc + 32u * h2, x);
            tc::tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = 0.f;
          }
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(o + H * hc + 32 * h2 + 4 * q) =
                make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        }
        if (hc == 0) {
          float m2[16];
          if (n_here > 0) {
            tc::tmem_ld16(tmem + lane_base + Lay::mass_col(0), m2);
            tc::tmem_wait_ld();
          } else {
            m2[0] = m2[1] = 0.f;
          }
          o[D] = m2[0] + m2[1];
          for (int e = D + 1; e < g.dp; ++e) o[e] = 0.f;
        }
      }
    } else if (ct == 0) {
      asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, Lay::tmem_cols);
  }
}

static cudaError_t launch_race_stats_group(const void* phi, const void* Y, const float* w, bool bwd, float* Atot,
                                           void* out, float* mass, const Geom& g, uint32_t* err, cudaStream_t st);

bool race_stats_tc_supported(const Geom& g) {
  return (g.d == 64 || g.d == 128) && g.C == kC && g.r > 0 && g.rp == kR * g.G && g.dp == g.d + 8;
}

// Totals, scan, per-chunk emission, for each group of 128 features in turn.  phi: [BH][N][rp]
// bf16; Y: [BH][N][d] bf16; w: [BH][N] fp32 or null (1); Atot: fp32 [BH][n_seg + 1][128][dp]
// scratch (reused by the groups); out: bf16 [G][BH][n_c][2][128][d]; mass: fp32 [G][BH][n_c][128].
cudaError_t launch_race_stats_tc(const void* phi, const void* Y, const float* w, bool bwd, float* Atot, void* out,
                                 float* mass, const Geom& g, uint32_t* err, cudaStream_t st) {
  if (!race_stats_tc_supported(g)) return cudaErrorInvalidValue;
  for (int grp = 0; grp < g.G; ++grp) {
    cudaError_t e = launch_race_stats_group(
        static_cast<const __nv_bfloat16*>(phi) + (size_t)grp * kR, Y, w, bwd, Atot,
        static_cast<__nv_bfloat16*>(out) + (size_t)grp * g.BH * g.n_c * 2 * kR * g.d,
        mass + (size_t)grp * g.BH * g.n_c * kR, g, err, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int D>
static cudaError_t stats_group_t(const void* phi, const void* Y, const float* w, bool bwd, float* Atot, void* out,
                                 float* mass, const Geom& g, uint32_t* err, cudaStream_t st) {
  CUtensorMap mphi, my, mo;
  if (!tc::map_rows_bf16_pitch(&mphi, phi, kR, g.rp, g.N, g.BH, kC) ||
      !tc::map_rows_bf16_pitch(&my, Y, D, D, g.N, g.BH, kC) ||
      !tc::map_rows_bf16_pitch(&mo, out, D, D, kR, g.BH * g.n_c * 2, kR))
    return cudaErrorInvalidValue;
  const size_t smem_t = StatsLayout<false>::bars + sizeof(StatBars);
  const size_t smem_e = StatsLayout<true>::bars + sizeof(StatBars);
  static_assert(StatsLayout<false>::bars + sizeof(StatBars) <= 232448, "shared memory per CTA");
  static_assert(StatsLayout<true>::bars + sizeof(StatBars) <= 232448, "shared memory per CTA");
  cudaError_t e = cudaFuncSetAttribute(race_stats_tc_kernel<false, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem_t);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(race_stats_tc_kernel<true, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_e);
  if (e != cudaSuccess) return e;
  {
    ProfScope ps(bwd ? "race_stats_bwd_totals" : "race_stats_fwd_totals", st);
    race_stats_tc_kernel<false, D><<<dim3(g.n_seg, g.BH), kThreads, smem_t, st>>>(mphi, my, mo, w, Atot, mass,
                                                                                    bwd ? 1 : 0, g, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  e = launch_race_scan(Atot, kR, bwd, g, st);
  if (e != cudaSuccess) return e;
  ProfScope ps(bwd ? "race_stats_bwd_emit" : "race_stats_fwd_emit", st);
  race_stats_tc_kernel<true, D><<<dim3(g.n_seg, g.BH), kThreads, smem_e, st>>>(mphi, my, mo, w, Atot, mass,
                                                                                 bwd ? 1 : 0, g, err);
  return cudaGetLastError();
}

static cudaError_t launch_race_stats_group(const void* phi, const void* Y, const float* w, bool bwd, float* Atot,
                                           void* out, float* mass, const Geom& g, uint32_t* err, cudaStream_t st) {
  return g.d == 64 ? stats_group_t<64>(phi, Y, w, bwd, Atot, out, mass, g, err, st)
                   : stats_group_t<128>(phi, Y, w, bwd, Atot, out, mass, g, err, st);
}

}  // namespace elsaa
