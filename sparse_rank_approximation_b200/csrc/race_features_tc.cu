// RACE soft-hash features on the 5th-generation tensor cores (ELSAA paper §3.1: keys and
// queries are softly assigned to hypercube buckets; sketch size S_R = L 2^gamma, §6).
//
// For a row x (d = 64 or 128): u = x / max(|x|, 1e-12); table l projects h_l = W_l^T u
// (gamma = 4 values); corner c in {-1,1}^4 has probability softmax_c(<c, h_l> / tau), which
// factorises into prod_b sigmoid(2 c_b h_lb / tau); Phi(x) = [p_l(c|x) / sqrt(L)] (r = 16 L
// columns, stored zero-padded to rp).
//
// One CTA per (128-row chunk, head, side Q / K).  The projections X W^T of the chunk are one
// M = 128, N = NW (4 L padded to 32), K = d product on the tensor cores, with W split into
// bf16 hi + lo halves (two accumulating products: X is exact in bf16, W nearly exact).  Warp 0
// issues the TMA loads, warp 1 owns TMEM and issues the products, warps 2-5 (one row per
// thread, TMEM lane quarter = warp % 4) divide by the row norm (from the staged bf16 row), run
// the corner probabilities, stage Phi (bf16, zero-padded to rp columns) over the operand tiles
// the products no longer need and write it with TMA stores; the normalised projections h (fp32)
// and the norm go out as row stores.  Every mbarrier wait is bounded; a timeout sets a bit in
// the caller's error word.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace elsaa {

namespace {

constexpr int kC = 128;                           // rows per CTA
constexpr uint32_t kSlab = 128 * 128;             // [128 rows][64 bf16], 128-byte swizzle
constexpr int kThreads = 192;
constexpr int kMaxNW = 64;                        // projections per row: 4 L <= 64
// Shared memory for NW projections: the X tile (2 slabs), W hi and W lo ([NW][d], 2 slabs of
// NW rows each), the barriers after them; Phi (rp / 64 slabs, rp = 2 NW) is staged over X and
// W once the products have read them.  NW = 32: 48 KB, four CTAs per SM.
constexpr uint32_t F_X = 0;
template <int NW> struct FeatLayout {
  static constexpr uint32_t kWSlab = (uint32_t)NW * 128;
  static constexpr uint32_t kWH = 2 * kSlab;
  static constexpr uint32_t kWL = kWH + 2 * kWSlab;
  static constexpr uint32_t kBars = kWL + 2 * kWSlab;
  static_assert(kBars >= (uint32_t)(2 * NW / 64) * kSlab, "Phi staging over the X and W tiles");
};

struct FeatBars {
  uint64_t in_full, acc_full;
  unsigned long long limit_ns;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, FeatBars* ms, uint32_t* err,
                                              uint32_t code) {
  if (*(volatile int*)&ms->abort_flag) return false;
  if (tc::mbar_wait(bar, parity, ms->limit_ns)) return true;
  *(volatile int*)&ms->abort_flag = 1;
  if (err) atomicOr(err, code);
  return false;
}

// K-major operand at byte offset `off`, K = 16 step kk of a tile of 128-byte rows kept as
// 64-column slabs; `d0` is the descriptor of offset 0, built once by the issuing thread.
__device__ __forceinline__ uint64_t desc_k(uint64_t d0, uint32_t off, int kk, uint32_t slab) {
  return tc::desc_adv(d0, off + (uint32_t)(kk >> 2) * slab + (uint32_t)(kk & 3) * 32u);
}

__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, 128;\n" ::: "memory"); }

}  // namespace

template <int D, int NW>
__global__ void __launch_bounds__(kThreads, NW == 32 ? 4 : 1)
    race_features_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmPQ,
                            const __grid_constant__ CUtensorMap tmPK, float* __restrict__ hQ, float* __restrict__ hK,
                            float* __restrict__ nQ, float* __restrict__ nK, Geom g, uint32_t* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  using FL = FeatLayout<NW>;
  FeatBars* ms = reinterpret_cast<FeatBars*>(smem + FL::kBars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, bh = blockIdx.y, side = blockIdx.z;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0 && err) atomicOr(err, 0x80000000u);
    return;
  }
  if (threadIdx.x == 0) {
    tc::mbar_init(&ms->in_full, 1);
    tc::mbar_init(&ms->acc_full, 1);
    ms->limit_ns = g.wait_ns;
    ms->abort_flag = 0;
    tc::fence_barrier_init();
    // the chunk's tiles do not depend on anything the set-up computes: their copies start first
    {
      constexpr uint32_t kWD = (uint32_t)NW * D * 2;
      tc::mbar_arrive_expect_tx(&ms->in_full, 128u * D * 2 + 2 * kWD);
      for (int s = 0; s < D / 64; ++s) {
        tc::tma_load_3d(smem + F_X + s * kSlab, side ? &tmK : &tmQ, &ms->in_full, 64 * s, c * kC, bh);
        tc::tma_load_3d(smem + FL::kWH + s * FL::kWSlab, &tmW, &ms->in_full, 64 * s, 0, 0);
        tc::tma_load_3d(smem + FL::kWL + s * FL::kWSlab, &tmW, &ms->in_full, 64 * s, 0, 1);
      }
    }
  }
  if (warp == 1) {
    tc::tmem_alloc(&ms->tmem_base, NW < 32 ? 32 : NW);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      tc::mbar_wait(&ms->in_full, 0);                 // no copy in flight when the CTA exits
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(128, NW, false, false);   // X (K-major) x W (K-major)
      const uint64_t d0 = tc::sw128_desc(smem_u32(smem), 16, 1024);
      if (wait_or_abort(&ms->in_full, 0, ms, err, 0x4000000u)) {
        tc::tc_fence_after();
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tc::mma_bf16(tmem, desc_k(d0, F_X, kk, kSlab), desc_k(d0, part ? FL::kWL : FL::kWH, kk, FL::kWSlab), idesc,
                         (part > 0 || kk > 0) ? 1u : 0u);
      }
      tc::mma_commit(&ms->acc_full);
      tc::mbar_wait(&ms->acc_full, 0);
    }
  } else {
    const int q4 = warp & 3;
    const int i = 32 * q4 + lane;                    // row of the chunk (TMEM lane)
    const int row = c * kC + i;
    const bool valid = row < g.N;
    const size_t grow = (size_t)bh * g.N + row;
    bool alive = __all_sync(0xffffffffu, wait_or_abort(&ms->in_full, 0, ms, err, 0x8000000u));
    // row norm from the staged bf16 row (fp32 sum of squares of the exact values)
    float ss = 0.f;
    if (alive) {
#pragma unroll
      for (int s = 0; s < D / 64; ++s)
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 v = *reinterpret_cast<const uint4*>(smem + F_X + s * kSlab + i * 128 + ((q ^ (i & 7)) << 4));
          const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(p[e]);
            ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
          }
        }
    }
    const float n = fmaxf(sqrtf(ss), kNormFloor);
    if (alive) alive = __all_sync(0xffffffffu, wait_or_abort(&ms->acc_full, 0, ms, err, 0x10000000u));
    if (alive) {
      tc::tc_fence_after();
      float hp[NW];
#pragma unroll
      for (int q = 0; q < NW / 32; ++q) {
        float tmp[32];
        tc::tmem_ld32(tmem + ((uint32_t)(32 * q4) << 16) + 32u * q, tmp);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) hp[32 * q + e] = tmp[e];
      }
      // Phi of this row into the staging tile (64-column slabs, 128-byte swizzle): the products
      // have read X and W, and this thread alone has read X row i
      float* hout = (side ? hK : hQ) + grow * (size_t)(4 * g.L);
      const float inv_n = 1.f / n, inv_sqrt_L = rsqrtf((float)g.L), two_over_tau = 2.f / g.tau;
      auto stage16 = [&](int col, const uint32_t (&w)[8]) {      // 16 bf16 at column col (multiple of 16)
        unsigned char* base = smem + F_X + (uint32_t)(col >> 6) * kSlab + (uint32_t)i * 128u;
        const int ch = (col & 63) >> 3;
        *reinterpret_cast<uint4*>(base + ((ch ^ (i & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(base + (((ch + 1) ^ (i & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
      };
#pragma unroll
      for (int l = 0; l < NW / 4; ++l) {
        if (l >= g.L) break;
        float sp[kHashBits], sm[kHashBits], hv[kHashBits];
#pragma unroll
        for (int b = 0; b < kHashBits; ++b) {
          hv[b] = hp[4 * l + b] * inv_n;
          sigmoid_pair(two_over_tau * hv[b], sp[b], sm[b]);   // P(c_b = +1), P(c_b = -1)
        }
        if (valid) reinterpret_cast<float4*>(hout)[l] = make_float4(hv[0], hv[1], hv[2], hv[3]);
        float pc[kCorners];
        corner_probs(sp, sm, inv_sqrt_L, pc);
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = pack_bf16(pc[2 * e], pc[2 * e + 1]);
        stage16(16 * l, w);
      }
      // stored rows are padded to rp columns with zeros
      const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      for (int col = 16 * g.L; col < g.rp; col += 16) stage16(col, z);
      if (valid) (side ? nK : nQ)[grow] = n;
    }
    // every row staged: one thread writes the tile (rows past N are dropped by the store)
    tc::fence_proxy_async_smem();
    compute_bar();
    if (threadIdx.x == 64 && !*(volatile int*)&ms->abort_flag) {
      const CUtensorMap* map = side ? &tmPK : &tmPQ;
      for (int sl = 0; sl < g.rp / 64; ++sl)
        asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];\n"
                     :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(smem + F_X + sl * kSlab)), "r"(64 * sl),
                        "r"(c * kC), "r"(bh) : "memory");
      asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, NW < 32 ? 32 : NW);
  }
}

template <int D, int NW>
static cudaError_t features_t(const void* Q, const void* K, const void* wsplit, void* phiQ, void* phiK, float* hQ,
                              float* hK, float* nQ, float* nK, const Geom& g, uint32_t* err, cudaStream_t st) {
  CUtensorMap mq, mk, mw, mpq, mpk;
  if (!tc::map_rows_bf16_pitch(&mq, Q, D, D, g.N, g.BH, kC) || !tc::map_rows_bf16_pitch(&mk, K, D, D, g.N, g.BH, kC) ||
      !tc::map_rows_bf16_pitch(&mw, wsplit, D, D, NW, 2, NW) ||
      !tc::map_rows_bf16_pitch(&mpq, phiQ, g.rp, g.rp, g.N, g.BH, kC) ||
      !tc::map_rows_bf16_pitch(&mpk, phiK, g.rp, g.rp, g.N, g.BH, kC))
    return cudaErrorInvalidValue;
  const size_t smem = FeatLayout<NW>::kBars + sizeof(FeatBars);
  static_assert(FeatLayout<NW>::kBars + sizeof(FeatBars) <= 232448, "shared memory per CTA");
  auto kern = race_features_tc_kernel<D, NW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps("race_features_tc", st);
  kern<<<dim3(g.n_c, g.BH, 2), kThreads, smem, st>>>(mq, mk, mw, mpq, mpk, hQ, hK, nQ, nK, g, err);
  return cudaGetLastError();
}

// wsplit: bf16 [2][NW][d] (hi, lo) written by launch_race_w_split, NW = 4 L padded to 32.
cudaError_t launch_race_features_tc(const void* Q, const void* K, const void* wsplit, void* phiQ, void* phiK,
                                    float* hQ, float* hK, float* nQ, float* nK, const Geom& g, uint32_t* err,
                                    cudaStream_t st) {
  const int NW = (4 * g.L + 31) & ~31;
  // Phi is staged as rp / 64 slabs over the 64 KB of operand tiles: rp = 128 (r <= 128) or 256
  if ((g.d != 64 && g.d != 128) || NW > kMaxNW || g.C != kC || g.rp < g.r || (g.rp != 128 && g.rp != 256) ||
      (g.rp == 256) != (NW == 64))
    return cudaErrorInvalidValue;
  if (g.d == 64)
    return NW == 32 ? features_t<64, 32>(Q, K, wsplit, phiQ, phiK, hQ, hK, nQ, nK, g, err, st)
                    : features_t<64, 64>(Q, K, wsplit, phiQ, phiK, hQ, hK, nQ, nK, g, err, st);
  return NW == 32 ? features_t<128, 32>(Q, K, wsplit, phiQ, phiK, hQ, hK, nQ, nK, g, err, st)
                  : features_t<128, 64>(Q, K, wsplit, phiQ, phiK, hQ, hK, nQ, nK, g, err, st);
}

}  // namespace elsaa
