// RACE low-rank read-out as its own pass (ELSAA paper §3.1): for each query
// tile, [N_lr ; d_lr] = Phi_Q P_t (prefix bucket statistics, bf16 hi + lo) plus,
// when causal, the masked diagonal-chunk term sum_{j <= i} (Phi(q_i).Phi(k_j)) [v_j ; 1].
// Writes O_lr = N_lr / d_lr (bf16) and d_lr (fp32).  Used ahead of the tcgen05
// sparse-branch kernel, whose epilogue applies the fusion.  grid (n_t, BH), block 2T.
#include "common.cuh"
#include "kernels.h"

namespace elsaa {

template <int D, int T>
struct ReadoutSmem {
  static constexpr int LD = D + 8;
  static constexpr int LDV1 = D + 16;
  static constexpr int RC = 64;
  static constexpr int LDF = RC + 8;
  static constexpr size_t off_fa = 0;
  static constexpr size_t off_fb = off_fa + (size_t)T * LDF * 2;
  static constexpr size_t off_ph = off_fb + (size_t)T * LDF * 2;
  static constexpr size_t off_pl = off_ph + (size_t)RC * LDV1 * 2;
  static constexpr size_t off_vd = off_pl + (size_t)RC * LDV1 * 2;
  static constexpr size_t off_out = off_vd + (size_t)T * LDV1 * 2;
  static constexpr size_t bytes = off_out + (size_t)T * LD * 2;
};

template <int D, int T>
__global__ void __launch_bounds__(2 * T) race_readout_bf16_kernel(
    const __nv_bfloat16* __restrict__ V, const __nv_bfloat16* __restrict__ phiQ,
    const __nv_bfloat16* __restrict__ phiK, const float* __restrict__ Ast, const float* __restrict__ Bst,
    __nv_bfloat16* __restrict__ Olr_out, float* __restrict__ dlr_out, Geom g) {
  using S = ReadoutSmem<D, T>;
  constexpr int LD = S::LD;
  constexpr int NT = 2 * T;
  constexpr int NBD = D / 8;
  constexpr int NBT = T / 8;
  constexpr int NBP = NBD + 1;
  extern __shared__ __align__(16) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int t = g.n_t - 1 - blockIdx.x;
  const int bh = blockIdx.y;
  const int row0 = warp * 16;
  const size_t head = (size_t)bh * g.N;
  const int rl[2] = {row0 + g4, row0 + g4 + 8};

  // ---- RACE read-out
  float acc[NBP][4];
#pragma unroll
  for (int nb = 0; nb < NBP; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
  if (g.r > 0) {
    __nv_bfloat16* sFa = reinterpret_cast<__nv_bfloat16*>(smem + S::off_fa);
    __nv_bfloat16* sFb = reinterpret_cast<__nv_bfloat16*>(smem + S::off_fb);
    __nv_bfloat16* sPh = reinterpret_cast<__nv_bfloat16*>(smem + S::off_ph);
    __nv_bfloat16* sPl = reinterpret_cast<__nv_bfloat16*>(smem + S::off_pl);
    __nv_bfloat16* sVd = reinterpret_cast<__nv_bfloat16*>(smem + S::off_vd);
    constexpr int LDF = S::LDF, LDV1 = S::LDV1, RC = S::RC;
    const int DP = g.dp;
    const int sidx = t / g.seg;
    const float* pa = Ast + ((size_t)bh * (g.n_seg + 1) + (g.causal ? sidx : g.n_seg)) * g.r * DP;
    const float* pb = g.causal ? Bst + ((size_t)bh * g.n_c + t) * g.r * DP : nullptr;
    const __nv_bfloat16* fq = phiQ + head * g.r;
    const __nv_bfloat16* fk = phiK + head * g.r;

    auto load_feat = [&](__nv_bfloat16* dst, const __nv_bfloat16* src, int rc, int rcw) {
      const int ch = rcw / 8;
      for (int i = tid; i < T * ch; i += NT) {
        const int r = i / ch, c = (i % ch) * 8;
        const int row = t * T + r;
        cp_async16(dst + r * LDF + c, src + (size_t)min(row, g.N - 1) * g.r + rc + c, row < g.N);
      }
    };

    // inter-chunk term: Phi_Q (P_hi + P_lo), P = prefix statistics in fp32
    for (int rc = 0; rc < g.r; rc += RC) {
      const int rcw = min(RC, g.r - rc);
      load_feat(sFa, fq, rc, rcw);
      cp_async_commit();
      const int q4 = DP / 4;
      const int total = rcw * q4;
      // loads batched 4 deep per thread before conversion, so their latencies overlap
#pragma unroll 1
      for (int i0 = tid; i0 < total; i0 += 4 * NT) {
        float4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i = i0 + k * NT;
          v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (i < total) {
            const int r = i / q4, c = (i % q4) * 4;
            v[k] = __ldg(reinterpret_cast<const float4*>(pa + (size_t)(rc + r) * DP + c));
            if (pb) {
              const float4 w = __ldg(reinterpret_cast<const float4*>(pb + (size_t)(rc + r) * DP + c));
              v[k].x += w.x; v[k].y += w.y; v[k].z += w.z; v[k].w += w.w;
            }
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i = i0 + k * NT;
          if (i >= total) break;
          const int r = i / q4, c = (i % q4) * 4;
          const float vv[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
          __align__(8) __nv_bfloat16 hi[4], lo[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            hi[j] = __float2bfloat16_rn(vv[j]);
            lo[j] = __float2bfloat16_rn(vv[j] - __bfloat162float(hi[j]));
          }
          *reinterpret_cast<uint2*>(sPh + r * LDV1 + c) = *reinterpret_cast<const uint2*>(hi);
          *reinterpret_cast<uint2*>(sPl + r * LDV1 + c) = *reinterpret_cast<const uint2*>(lo);
        }
      }
      cp_async_wait<0>();
      __syncthreads();
      for (int kk = 0; kk < rcw / 16; ++kk) {
        uint32_t a[4];
        ldsm_x4(a, a_frag_ptr(sFa, LDF, row0, kk * 16, lane));
#pragma unroll
        for (int nb2 = 0; nb2 < NBP / 2; ++nb2) {
          uint32_t bh_[4], bl_[4];
          ldsm_x4_t(bh_, bkn_frag_ptr(sPh, LDV1, kk * 16, nb2 * 16, lane));
          ldsm_x4_t(bl_, bkn_frag_ptr(sPl, LDV1, kk * 16, nb2 * 16, lane));
          mma16816(acc[2 * nb2], a, bh_[0], bh_[1]);
          mma16816(acc[2 * nb2 + 1], a, bh_[2], bh_[3]);
          mma16816(acc[2 * nb2], a, bl_[0], bl_[1]);
          mma16816(acc[2 * nb2 + 1], a, bl_[2], bl_[3]);
        }
        uint32_t b2[2];
        ldsm_x2_t(b2, bkn_frag_ptr1(sPh, LDV1, kk * 16, (NBP - 1) * 8, lane));
        mma16816(acc[NBP - 1], a, b2[0], b2[1]);
        ldsm_x2_t(b2, bkn_frag_ptr1(sPl, LDV1, kk * 16, (NBP - 1) * 8, lane));
        mma16816(acc[NBP - 1], a, b2[0], b2[1]);
      }
      __syncthreads();
    }

    if (g.causal) {
      // intra-chunk term: kappa = Phi_Q Phi_K^T on the diagonal block, masked j <= i
      float kap[NBT][4];
#pragma unroll
      for (int nb = 0; nb < NBT; ++nb) kap[nb][0] = kap[nb][1] = kap[nb][2] = kap[nb][3] = 0.f;
      // V of the diagonal block with the key-mass column block
      for (int i = tid; i < T * (D / 8); i += NT) {
        const int r = i / (D / 8), c = (i % (D / 8)) * 8;
        const int row = t * T + r;
        cp_async16(sVd + r * LDV1 + c, V + (head + min(row, g.N - 1)) * D + c, row < g.N);
      }
      for (int r = tid; r < T; r += NT) {
        __nv_bfloat16* o1 = sVd + r * LDV1 + D;
        o1[0] = __float2bfloat16_rn(t * T + r < g.N ? 1.f : 0.f);
#pragma unroll
        for (int j = 1; j < 8; ++j) o1[j] = __float2bfloat16_rn(0.f);
      }
      for (int rc = 0; rc < g.r; rc += RC) {
        const int rcw = min(RC, g.r - rc);
        load_feat(sFa, fq, rc, rcw);
        load_feat(sFb, fk, rc, rcw);
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        for (int kk = 0; kk < rcw / 16; ++kk) {
          uint32_t a[4];
          ldsm_x4(a, a_frag_ptr(sFa, LDF, row0, kk * 16, lane));
#pragma unroll
          for (int nb2 = 0; nb2 < NBT / 2; ++nb2) {
            uint32_t bf[4];
            ldsm_x4(bf, bnk_frag_ptr(sFb, LDF, nb2 * 16, kk * 16, lane));
            mma16816(kap[2 * nb2], a, bf[0], bf[1]);
            mma16816(kap[2 * nb2 + 1], a, bf[2], bf[3]);
          }
        }
        __syncthreads();
      }
#pragma unroll
      for (int nb = 0; nb < NBT; ++nb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = nb * 8 + t4 * 2 + (e & 1);
          if (col > rl[e >> 1]) kap[nb][e] = 0.f;
        }
      }
#pragma unroll
      for (int kk = 0; kk < T / 16; ++kk) {
        uint32_t a[4];
        a[0] = pack_bf16(kap[2 * kk][0], kap[2 * kk][1]);
        a[1] = pack_bf16(kap[2 * kk][2], kap[2 * kk][3]);
        a[2] = pack_bf16(kap[2 * kk + 1][0], kap[2 * kk + 1][1]);
        a[3] = pack_bf16(kap[2 * kk + 1][2], kap[2 * kk + 1][3]);
#pragma unroll
        for (int nb2 = 0; nb2 < NBP / 2; ++nb2) {
          uint32_t bf[4];
          ldsm_x4_t(bf, bkn_frag_ptr(sVd, LDV1, kk * 16, nb2 * 16, lane));
          mma16816(acc[2 * nb2], a, bf[0], bf[1]);
          mma16816(acc[2 * nb2 + 1], a, bf[2], bf[3]);
        }
        uint32_t b2[2];
        ldsm_x2_t(b2, bkn_frag_ptr1(sVd, LDV1, kk * 16, (NBP - 1) * 8, lane));
        mma16816(acc[NBP - 1], a, b2[0], b2[1]);
      }
    }
  }

  float dl[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) dl[h] = __shfl_sync(0xffffffffu, acc[NBP - 1][2 * h], lane & ~3);
  __syncthreads();
  __nv_bfloat16* sO = reinterpret_cast<__nv_bfloat16*>(smem + S::off_out);
#pragma unroll
  for (int nb = 0; nb < NBD; ++nb) {
    const int col = nb * 8 + t4 * 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float il = dl[h] > 0.f ? 1.f / dl[h] : 0.f;
      *reinterpret_cast<uint32_t*>(sO + rl[h] * LD + col) = pack_bf16(acc[nb][2 * h] * il, acc[nb][2 * h + 1] * il);
    }
  }
  if (t4 == 0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int qi = t * T + rl[h];
      if (qi < g.N) dlr_out[head + qi] = dl[h];
    }
  }
  __syncthreads();
  for (int i = tid; i < T * (D / 8); i += NT) {
    const int r = i / (D / 8), c = (i % (D / 8)) * 8;
    const int row = t * T + r;
    if (row < g.N)
      *reinterpret_cast<uint4*>(Olr_out + (head + row) * D + c) = *reinterpret_cast<const uint4*>(sO + r * LD + c);
  }
}

template <int D, int T>
static cudaError_t readout_t(const FwdArgs& a, const Geom& g, cudaStream_t st) {
  const size_t smem = ReadoutSmem<D, T>::bytes;
  auto kern = race_readout_bf16_kernel<D, T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps("race_readout", st);
  kern<<<dim3(g.n_t, g.BH), 2 * T, smem, st>>>((const __nv_bfloat16*)a.V, (const __nv_bfloat16*)a.phiQ,
                                                (const __nv_bfloat16*)a.phiK, a.Ast, a.Bst,
                                                (__nv_bfloat16*)a.Olr, a.dlr, g);
  return cudaGetLastError();
}

cudaError_t launch_race_readout_bf16(const FwdArgs& a, const Geom& g, cudaStream_t st) {
  if (g.d == 64 && g.T == 64) return readout_t<64, 64>(a, g, st);
  if (g.d == 64 && g.T == 128) return readout_t<64, 128>(a, g, st);
  if (g.d == 128 && g.T == 64) return readout_t<128, 64>(a, g, st);
  if (g.d == 128 && g.T == 128) return readout_t<128, 128>(a, g, st);
  return cudaErrorInvalidValue;
}

}  // namespace elsaa
