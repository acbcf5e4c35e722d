// Sparse-branch forward on the 5th-generation tensor cores (tcgen05 + TMEM), for
// 128-query tiles, 128-key blocks and head dimension 128, fused with the
// denominator-aware fusion epilogue (ELSAA paper §3.2, §3.3 Eq. 5, §1 Eq. 4).
//
// One CTA per (head, query tile), 6 warps:
//   warp 0     TMA producer: Q tile once, then K and V of each selected block
//              into a 2-stage ring (128-byte swizzled 64-column slabs);
//   warp 1     TMEM owner and MMA issuer: S_j = Q K_j^T into one of two TMEM
//              score buffers, then O += P_{j-1} V_{j-1} into the TMEM output;
//   warps 2-5  one query row per thread: read S_j from TMEM, mask, online
//              softmax in fp32 (lazy rescaling: O and l are rescaled only when
//              the running max grows by more than 2^8), write P_j as bf16 to
//              shared memory in the swizzled K-major layout; finally read O,
//              normalise, fuse with the low-rank output and store.
// Every mbarrier wait is bounded; a timeout sets a bit in the caller's error
// word, the CTA drains its outstanding copies and MMAs, frees TMEM and exits.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace elsaa {

namespace {

constexpr int kT = 128;                  // tile rows = keys per block
constexpr int kD = 128;                  // head dimension
constexpr uint32_t kSlab = kT * 128;     // one [128 rows][64 bf16] swizzled slab
constexpr uint32_t kTile = 2 * kSlab;    // 128 x 128 bf16
constexpr uint32_t OFF_Q = 0;
__host__ __device__ constexpr uint32_t off_k(int s) { return kTile * (1 + 2 * s); }   // K stage s
__host__ __device__ constexpr uint32_t off_v(int s) { return kTile * (2 + 2 * s); }   // V stage s
__host__ __device__ constexpr uint32_t off_p(int b) { return kTile * (5 + b); }      // P buffer b
constexpr uint32_t OFF_MISC = 7 * kTile;
constexpr size_t kSmemBytes = OFF_MISC + 512 + 1024;     // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t TM_O = 0;
__host__ __device__ constexpr uint32_t tm_s(int s) { return 128u + 128u * s; }        // score buffer s
constexpr float kRescaleThreshold = 8.f;                 // log2 units

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

struct Misc {
  uint64_t q_full, kv_full[2], kv_empty[2], s_full[2], s_free[2], p_full[2], pv_done[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  int idx[32];
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Misc* ms, uint32_t* err,
                                              uint32_t code) {
  if (*(volatile int*)&ms->abort_flag) return false;
  if (tc::mbar_wait(bar, parity)) return true;
  *(volatile int*)&ms->abort_flag = 1;
  if (err) atomicOr(err, code);
  return false;
}

}  // namespace

__global__ void __launch_bounds__(192, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, FwdArgs a, Geom g, uint32_t* err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Misc* ms = reinterpret_cast<Misc*>(smem + OFF_MISC);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = g.n_t - 1 - blockIdx.x;
  const int bh = blockIdx.y;
  const size_t head = (size_t)bh * g.N;

  // ---- set-up: barriers, selected blocks, TMEM
  const int* my_idx = a.idx + ((size_t)bh * g.n_t + t) * g.k;
  if (threadIdx.x == 0) {
    tc::mbar_init(&ms->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&ms->kv_full[s], 1);
      tc::mbar_init(&ms->kv_empty[s], 1);
      tc::mbar_init(&ms->s_full[s], 1);
      tc::mbar_init(&ms->s_free[s], 128);
      tc::mbar_init(&ms->p_full[s], 128);
      tc::mbar_init(&ms->pv_done[s], 1);
    }
    tc::mbar_init(&ms->drain, 1);
    ms->abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (threadIdx.x < 32) ms->idx[threadIdx.x] = threadIdx.x < g.k ? my_idx[threadIdx.x] : -1;
  if (warp == 1) {
    tc::tmem_alloc(&ms->tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  int n_sel = 0;
  while (n_sel < g.k && n_sel < 32 && ms->idx[n_sel] >= 0) ++n_sel;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      int issued = 0;
      tc::mbar_arrive_expect_tx(&ms->q_full, kTile);
      tc::tma_load_3d(smem + OFF_Q, &tmQ, &ms->q_full, 0, t * kT, bh);
      tc::tma_load_3d(smem + OFF_Q + kSlab, &tmQ, &ms->q_full, 64, t * kT, bh);
      for (int j = 0; j < n_sel; ++j) {
        const int s = j & 1;
        if (j >= 2 && !wait_or_abort(&ms->kv_empty[s], ((j >> 1) + 1) & 1, ms, err, 1u)) break;
        const int b = ms->idx[j];
        tc::mbar_arrive_expect_tx(&ms->kv_full[s], 2 * kTile);
        tc::tma_load_3d(smem + off_k(s), &tmK, &ms->kv_full[s], 0, b * kT, bh);
        tc::tma_load_3d(smem + off_k(s) + kSlab, &tmK, &ms->kv_full[s], 64, b * kT, bh);
        tc::tma_load_3d(smem + off_v(s), &tmV, &ms->kv_full[s], 0, b * kT, bh);
        tc::tma_load_3d(smem + off_v(s) + kSlab, &tmV, &ms->kv_full[s], 64, b * kT, bh);
        issued = j + 1;
      }
      // drain: every copy this thread started has landed before the CTA may exit
      tc::mbar_wait(&ms->q_full, 0);
      for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j) tc::mbar_wait(&ms->kv_full[j & 1], (j >> 1) & 1);
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t idS = tc::idesc_bf16(128, 128, false, false);   // Q (K-major) x K (K-major)
      const uint32_t idPV = tc::idesc_bf16(128, kD, false, true);    // P (K-major) x V (MN-major)
      const uint32_t sbase = smem_u32(smem);
      bool ok = wait_or_abort(&ms->q_full, 0, ms, err, 2u);
      int pv_issued = 0;
      auto issue_pv = [&](int jj) -> bool {
        if (!wait_or_abort(&ms->p_full[jj & 1], (jj >> 1) & 1, ms, err, 4u)) return false;
        tc::tc_fence_after();
        const uint32_t vb = sbase + off_v(jj & 1);
        const uint32_t pb = sbase + off_p(jj & 1);
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk) {
          const uint64_t ad = tc::sw128_desc(pb + (kk >> 2) * kSlab + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = tc::sw128_desc(vb + kk * 2048, kSlab, 1024);
          tc::mma_bf16(tmem + TM_O, ad, bd, idPV, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(&ms->kv_empty[jj & 1]);
        tc::mma_commit(&ms->pv_done[jj & 1]);
        pv_issued = jj + 1;
        return true;
      };
      for (int j = 0; ok && j < n_sel; ++j) {
        const int s = j & 1;
        if (!wait_or_abort(&ms->kv_full[s], (j >> 1) & 1, ms, err, 8u)) break;
        if (j >= 2 && !wait_or_abort(&ms->s_free[s], ((j >> 1) + 1) & 1, ms, err, 16u)) break;
        tc::tc_fence_after();
        const uint32_t kb = sbase + off_k(s);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t ad = tc::sw128_desc(sbase + OFF_Q + (kk >> 2) * kSlab + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = tc::sw128_desc(kb + (kk >> 2) * kSlab + (kk & 3) * 32, 16, 1024);
          tc::mma_bf16(tmem + tm_s(s), ad, bd, idS, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&ms->s_full[s]);
        if (j >= 1 && !issue_pv(j - 1)) break;
      }
      if (n_sel > 0 && pv_issued == n_sel - 1) issue_pv(n_sel - 1);
      // drain: all MMAs this thread issued have completed
      tc::mma_commit(&ms->drain);
      tc::mbar_wait(&ms->drain, 0);
    }
  } else {
    // ================= softmax / epilogue: one query row per thread =================
    const int q4 = warp & 3;
    const int row = 32 * q4 + lane;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const float sl2 = g.scale * kLog2e;
    float m_used = -INFINITY, l = 0.f;     // running max (log2 units, scaled) and row sum
    bool ok = true;
    for (int j = 0; j < n_sel; ++j) {
      const int s = j & 1;
      ok = wait_or_abort(&ms->s_full[s], (j >> 1) & 1, ms, err, 32u);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc::tc_fence_after();
      float sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float tmp[32];
        tc::tmem_ld32(tmem + lane_base + tm_s(s) + 32 * c, tmp);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[32 * c + i] = tmp[i];
      }
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      tc::mbar_arrive(&ms->s_free[s]);
      const int b = ms->idx[j];
      const int kvalid = g.N - b * kT;            // keys of this block inside the sequence
      if ((g.causal && b == t) || kvalid < kT) {  // block-uniform: only the diagonal / ragged block masks
        const int lim = min(kvalid - 1, (g.causal && b == t) ? row : kT - 1);
#pragma unroll
        for (int c = 0; c < 128; ++c) sv[c] = c > lim ? -INFINITY : sv[c];
      }
      float m4[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
      for (int c = 4; c < 128; c += 4) {
        m4[0] = fmaxf(m4[0], sv[c]);
        m4[1] = fmaxf(m4[1], sv[c + 1]);
        m4[2] = fmaxf(m4[2], sv[c + 2]);
        m4[3] = fmaxf(m4[3], sv[c + 3]);
      }
      const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
      // lazy rescaling: move the reference max only when the row max grew by > 2^8
      const float m_new = fmaxf(m_used, mx);
      const bool resc = m_new > m_used + kRescaleThreshold;     // false while both are -inf
      float alpha = 1.f;
      if (resc) {
        alpha = (m_used == -INFINITY) ? 0.f : exp2f(m_used - m_new);
        l *= alpha;
        m_used = m_new;
      }
      if (j > 0 && __any_sync(0xffffffffu, resc)) {
        // O holds the products through block j-1: wait for the last one, rescale (warp-collective)
        ok = wait_or_abort(&ms->pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, ms, err, 64u);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc::tc_fence_after();
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          float tmp[32];
          tc::tmem_ld32(tmem + lane_base + TM_O + 32 * c, tmp);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) tmp[i] *= alpha;
          tc::tmem_st32(tmem + lane_base + TM_O + 32 * c, tmp);
        }
        tc::tmem_wait_st();
      }
      // P buffer j&1 is free once the PV product of block j-2 has finished
      if (j >= 2) {
        ok = wait_or_abort(&ms->pv_done[s], ((j >> 1) + 1) & 1, ms, err, 256u);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      }
      const float msub = m_used == -INFINITY ? 0.f : m_used;
      float rs0 = 0.f, rs1 = 0.f;
      unsigned char* prow = smem + off_p(s) + row * 128;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = ex2_approx(fmaf(sv[8 * ch + 2 * e], sl2, -msub));
          const float p1 = ex2_approx(fmaf(sv[8 * ch + 2 * e + 1], sl2, -msub));
          rs0 += p0;
          rs1 += p1;
          w[e] = pack_bf16(p0, p1);
        }
        const int phys = (ch & 7) ^ (row & 7);
        *reinterpret_cast<uint4*>(prow + (ch >> 3) * kSlab + phys * 16) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      l += rs0 + rs1;
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(&ms->p_full[s]);
    }
    // ---- epilogue: O_s = O / l, log d_s, fusion (Eq. 5, Eq. 4), coalesced stores via smem
    float o[kD];
#pragma unroll
    for (int c = 0; c < kD; ++c) o[c] = 0.f;
    if (ok && n_sel > 0) {
      ok = wait_or_abort(&ms->pv_done[(n_sel - 1) & 1], ((n_sel - 1) >> 1) & 1, ms, err, 128u);
      if (__all_sync(0xffffffffu, ok)) {
        tc::tc_fence_after();
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          float tmp[32];
          tc::tmem_ld32(tmem + lane_base + TM_O + 32 * c, tmp);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[32 * c + i] = tmp[i];
        }
        tc::tmem_wait_ld();
      } else {
        ok = false;
      }
    }
    // every PV product is done (or abandoned): K/V stage 0 and both P buffers are free.
    // Tiles are [128 rows][256 bytes] with 16-byte chunk c of row r stored at chunk c ^ (r & 15).
    const int tid = threadIdx.x - 64;                      // 0..127 among the softmax warps
    unsigned char* sLr = smem + off_p(0);
    unsigned char* sO = smem + off_p(1);
    unsigned char* sS = smem + off_k(0);
    const int rows_here = min(kT, g.N - t * kT);
    const __nv_bfloat16* olr_g = static_cast<const __nv_bfloat16*>(a.Olr) + (head + (size_t)t * kT) * kD;
#pragma unroll 4
    for (int i = tid; i < kT * 16; i += 128) {
      const int r = i >> 4, c = i & 15;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < rows_here) v = *reinterpret_cast<const uint4*>(olr_g + (size_t)r * kD + c * 8);
      *reinterpret_cast<uint4*>(sLr + r * 256 + ((c ^ (r & 15)) << 4)) = v;
    }
    asm volatile("bar.sync 1, 128;\n" ::: "memory");
    const int qrow = t * kT + row;
    float logd = -INFINITY, mf = 0.f;
    if (qrow < g.N) {
      const size_t ri = head + qrow;
      logd = l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const float dl = a.dlr[ri];
      const float lam = a.lam ? a.lam[ri] : g.lam;
      mf = logd == -INFINITY ? 0.f : 1.f / (1.f + (lam * dl + g.eps) * expf(-logd));
      const float gs = a.gs ? a.gs[ri] : 1.f;
      const float gl = a.glr ? a.glr[ri] : 1.f - mf;
      const float cs = gs * mf;
#pragma unroll
      for (int ch = 0; ch < kD / 8; ++ch) {
        const int off = row * 256 + ((ch ^ (row & 15)) << 4);
        const uint4 lr = *reinterpret_cast<const uint4*>(sLr + off);
        const __nv_bfloat16* lv = reinterpret_cast<const __nv_bfloat16*>(&lr);
        uint32_t wo[4], ws[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float s0 = o[8 * ch + 2 * e] * inv_l, s1 = o[8 * ch + 2 * e + 1] * inv_l;
          ws[e] = pack_bf16(s0, s1);
          wo[e] = pack_bf16(cs * s0 + gl * __bfloat162float(lv[2 * e]), cs * s1 + gl * __bfloat162float(lv[2 * e + 1]));
        }
        *reinterpret_cast<uint4*>(sO + off) = make_uint4(wo[0], wo[1], wo[2], wo[3]);
        *reinterpret_cast<uint4*>(sS + off) = make_uint4(ws[0], ws[1], ws[2], ws[3]);
      }
      a.logd[ri] = logd;
      a.m[ri] = mf;
    }
    asm volatile("bar.sync 1, 128;\n" ::: "memory");
    if (ok) {
      __nv_bfloat16* o_g = static_cast<__nv_bfloat16*>(a.O) + (head + (size_t)t * kT) * kD;
      __nv_bfloat16* s_g = static_cast<__nv_bfloat16*>(a.Os) + (head + (size_t)t * kT) * kD;
#pragma unroll 4
      for (int i = tid; i < kT * 16; i += 128) {
        const int r = i >> 4, c = i & 15;
        if (r < rows_here) {
          const int off = r * 256 + ((c ^ (r & 15)) << 4);
          *reinterpret_cast<uint4*>(o_g + (size_t)r * kD + c * 8) = *reinterpret_cast<const uint4*>(sO + off);
          *reinterpret_cast<uint4*>(s_g + (size_t)r * kD + c * 8) = *reinterpret_cast<const uint4*>(sS + off);
        }
      }
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

// [BH][N][128] bf16 viewed as a 3-D tensor (d, row, head); boxes of 64 x 128 x 1,
// 128-byte swizzle; rows past N read as zeros.
static bool make_map(CUtensorMap* m, const void* base, int N, int BH) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)N * kD * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)kT, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool attn_fwd_tc_supported(const Geom& g) { return g.d == kD && g.T == kT && g.k <= 32; }

cudaError_t launch_attn_fwd_tc(const FwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st) {
  if (!attn_fwd_tc_supported(g)) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.Q, g.N, g.BH) || !make_map(&mk, a.K, g.N, g.BH) || !make_map(&mv, a.V, g.N, g.BH))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  ProfScope ps("attn_fwd_tc", st);
  attn_fwd_tc_kernel<<<dim3(g.n_t, g.BH), 192, kSmemBytes, st>>>(mq, mk, mv, a, g, err);
  return cudaGetLastError();
}

}  // namespace elsaa
