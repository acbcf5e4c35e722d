// Fused forward tile kernel: sparse branch over the selected key blocks, RACE
// read-out, denominator-aware fusion and the output store.
//
//   sparse branch (ELSAA paper §3.2, §3.3 Practical notes): for query i of tile t
//     and keys j of the selected blocks (j <= i when causal),
//     d_s,i = sum_j exp(z_ij), O_s,i = sum_j exp(z_ij) v_j / d_s,i, z = scale q.k,
//     with an online (running max) softmax in fp32 and bf16 tensor-core MMAs;
//   low-rank read-out (§3.1): [N_lr ; d_lr]_i = Phi(q_i) P_t + sum_{j in chunk t,
//     j <= i} (Phi(q_i).Phi(k_j)) [v_j ; 1], P_t the prefix bucket statistics;
//   fusion (Eq. 5, Eq. 4): m = d_s / (d_s + lambda d_lr + eps),
//     O = g_s m O_s + g_lr N_lr / d_lr  (default g_s = 1, g_lr = 1 - m).
//
// One CTA per (head, query tile), T/16 warps, each warp 16 query rows.  K/V
// blocks are double-buffered in shared memory with cp.async; heavy (late)
// causal tiles are launched first.  The RACE stage reuses the K/V buffers.
#include "common.cuh"
#include "kernels.h"

namespace elsaa {

template <int D, int T>
struct FwdSmem {
  static constexpr int LD = D + 8;            // bf16 row pitch of Q/K/V tiles
  static constexpr int LDV1 = D + 16;         // V tile with the key-mass column block
  static constexpr int RC = 64;               // feature columns per RACE pass
  static constexpr int LDF = RC + 8;
  static constexpr int LDO = D + 8;           // fp32 pitch of the O_s stash
  static constexpr size_t sparse_bytes = (size_t)5 * T * LD * 2;
  // RACE stage layout (bytes, from 0): Os stash | PhiQ | PhiK | P hi | P lo | V+1
  static constexpr size_t off_os = 0;
  static constexpr size_t off_fa = off_os + (size_t)T * LDO * 4;
  static constexpr size_t off_fb = off_fa + (size_t)T * LDF * 2;
  static constexpr size_t off_ph = off_fb + (size_t)T * LDF * 2;
  static constexpr size_t off_pl = off_ph + (size_t)RC * LDV1 * 2;
  static constexpr size_t off_vd = off_pl + (size_t)RC * LDV1 * 2;
  static constexpr size_t race_bytes = off_vd + (size_t)T * LDV1 * 2;
  static constexpr size_t bytes = sparse_bytes > race_bytes ? sparse_bytes : race_bytes;
  // the epilogue stages three bf16 [T][LD] tiles from off_fa while the O_s stash is live
  static_assert(off_fa + (size_t)3 * T * LD * 2 <= bytes, "epilogue staging overflows shared memory");
};

template <int D, int T>
__global__ void __launch_bounds__(2 * T) attn_fwd_bf16_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, const int* __restrict__ idx,
    const __nv_bfloat16* __restrict__ phiQ, const __nv_bfloat16* __restrict__ phiK,
    const float* __restrict__ Ast, const float* __restrict__ Bst, const float* __restrict__ lam_vec,
    const float* __restrict__ gs_vec, const float* __restrict__ glr_vec, __nv_bfloat16* __restrict__ O,
    __nv_bfloat16* __restrict__ Os_out, float* __restrict__ logd_out, float* __restrict__ dlr_out,
    float* __restrict__ m_out, __nv_bfloat16* __restrict__ Olr_out, Geom g) {
  using S = FwdSmem<D, T>;
  constexpr int LD = S::LD;
  constexpr int NT = 2 * T;                   // threads
  constexpr int NBD = D / 8;                  // n-blocks of the output
  constexpr int NBT = T / 8;                  // n-blocks of a score row
  constexpr int NBP = NBD + 1;                // n-blocks of [value | key mass]
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sK = sQ + T * LD;            // [2][T][LD]
  __nv_bfloat16* sV = sK + 2 * T * LD;        // [2][T][LD]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int t = g.n_t - 1 - blockIdx.x;
  const int bh = blockIdx.y;
  const int row0 = warp * 16;
  const size_t head = (size_t)bh * g.N;
  const int* my_idx = idx + ((size_t)bh * g.n_t + t) * g.k;

  // ---- Q tile
  for (int i = tid; i < T * (D / 8); i += NT) {
    const int r = i / (D / 8), c = (i % (D / 8)) * 8;
    const int row = t * T + r;
    cp_async16(sQ + r * LD + c, Q + (head + min(row, g.N - 1)) * D + c, row < g.N);
  }
  cp_async_commit();
  int n_sel = 0;
  while (n_sel < g.k && my_idx[n_sel] >= 0) ++n_sel;

  auto load_kv = [&](int buf, int b) {
    __nv_bfloat16* dK = sK + buf * T * LD;
    __nv_bfloat16* dV = sV + buf * T * LD;
    for (int i = tid; i < T * (D / 8); i += NT) {
      const int r = i / (D / 8), c = (i % (D / 8)) * 8;
      const int row = b * T + r;
      const size_t src = (head + min(row, g.N - 1)) * D + c;
      cp_async16(dK + r * LD + c, K + src, row < g.N);
      cp_async16(dV + r * LD + c, V + src, row < g.N);
    }
  };
  if (n_sel > 0) {
    load_kv(0, my_idx[0]);
    cp_async_commit();
    cp_async_wait<1>();
  } else {
    cp_async_wait<0>();
  }
  __syncthreads();

  uint32_t qf[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) ldsm_x4(qf[kk], a_frag_ptr(sQ, LD, row0, kk * 16, lane));

  float o[NBD][4];
#pragma unroll
  for (int nb = 0; nb < NBD; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const float sl2 = g.scale * kLog2e;
  const int rl[2] = {row0 + g4, row0 + g4 + 8};

  for (int it = 0; it < n_sel; ++it) {
    if (it + 1 < n_sel) {
      load_kv((it + 1) & 1, my_idx[it + 1]);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int b = my_idx[it];
    const __nv_bfloat16* cK = sK + (it & 1) * T * LD;
    const __nv_bfloat16* cV = sV + (it & 1) * T * LD;
    float s[NBT][4];
#pragma unroll
    for (int nb = 0; nb < NBT; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int nb2 = 0; nb2 < NBT / 2; ++nb2) {
        uint32_t bf[4];
        ldsm_x4(bf, bnk_frag_ptr(cK, LD, nb2 * 16, kk * 16, lane));
        mma16816(s[2 * nb2], qf[kk], bf[0], bf[1]);
        mma16816(s[2 * nb2 + 1], qf[kk], bf[2], bf[3]);
      }
    }
    const bool diag = g.causal && b == t;
    const bool ragged = (b + 1) * T > g.N;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nb = 0; nb < NBT; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nb * 8 + t4 * 2 + (e & 1);
        float v = s[nb][e] * sl2;
        if ((diag && col > rl[e >> 1]) || (ragged && b * T + col >= g.N)) v = -INFINITY;
        s[nb][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
    float alpha[2], msub[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
      const float mnew = fmaxf(mrow[h], mx[h]);
      msub[h] = mnew == -INFINITY ? 0.f : mnew;
      alpha[h] = exp2f(mrow[h] - msub[h]);
      mrow[h] = mnew;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nb = 0; nb < NBT; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[nb][e] - msub[e >> 1]);
        s[nb][e] = p;
        rs[e >> 1] += p;
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) lrow[h] = lrow[h] * alpha[h] + rs[h];
#pragma unroll
    for (int nb = 0; nb < NBD; ++nb) {
      o[nb][0] *= alpha[0];
      o[nb][1] *= alpha[0];
      o[nb][2] *= alpha[1];
      o[nb][3] *= alpha[1];
    }
#pragma unroll
    for (int kk = 0; kk < T / 16; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nb2 = 0; nb2 < NBD / 2; ++nb2) {
        uint32_t bf[4];
        ldsm_x4_t(bf, bkn_frag_ptr(cV, LD, kk * 16, nb2 * 16, lane));
        mma16816(o[2 * nb2], a, bf[0], bf[1]);
        mma16816(o[2 * nb2 + 1], a, bf[2], bf[3]);
      }
    }
    __syncthreads();
  }

  // ---- finish the sparse branch: O_s and log d_s per row
  float logd[2], inv_l[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 1);
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 2);
    inv_l[h] = lrow[h] > 0.f ? 1.f / lrow[h] : 0.f;
    logd[h] = lrow[h] > 0.f ? (mrow[h] + log2f(lrow[h])) * kLn2 : -INFINITY;
  }
  __syncthreads();   // every warp is done with the Q/K/V buffers
  float* sOs = reinterpret_cast<float*>(smem + S::off_os);
#pragma unroll
  for (int nb = 0; nb < NBD; ++nb) {
    const int col = nb * 8 + t4 * 2;
    *reinterpret_cast<float2*>(sOs + rl[0] * S::LDO + col) = make_float2(o[nb][0] * inv_l[0], o[nb][1] * inv_l[0]);
    *reinterpret_cast<float2*>(sOs + rl[1] * S::LDO + col) = make_float2(o[nb][2] * inv_l[1], o[nb][3] * inv_l[1]);
  }

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

  // ---- fusion epilogue (Eq. 5, Eq. 4)
  float dl[2], mfac[2], cs[2], cl[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    dl[h] = __shfl_sync(0xffffffffu, acc[NBP - 1][2 * h], lane & ~3);
    const int qi = t * T + rl[h];
    const int qc = min(qi, g.N - 1);
    const float lam = lam_vec ? lam_vec[head + qc] : g.lam;
    const float c = lam * dl[h] + g.eps;
    mfac[h] = g.fixed_m ? 1.f : logd[h] == -INFINITY ? 0.f : 1.f / (1.f + c * expf(-logd[h]));
    const float gs = gs_vec ? gs_vec[head + qc] : 1.f;
    const float gl = glr_vec ? glr_vec[head + qc] : g.fixed_m ? 1.f : 1.f - mfac[h];
    cs[h] = gs * mfac[h];
    cl[h] = dl[h] > 0.f ? gl / dl[h] : 0.f;
  }
  __syncthreads();   // RACE buffers are free; stage bf16 outputs there
  __nv_bfloat16* sO = reinterpret_cast<__nv_bfloat16*>(smem + S::off_fa);   // [T][LD]
  __nv_bfloat16* sS = sO + T * LD;                                           // [T][LD]
  __nv_bfloat16* sL = sS + T * LD;                                           // [T][LD]
  const float* sOs2 = reinterpret_cast<const float*>(smem + S::off_os);
#pragma unroll
  for (int nb = 0; nb < NBD; ++nb) {
    const int col = nb * 8 + t4 * 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float2 os = *reinterpret_cast<const float2*>(sOs2 + rl[h] * S::LDO + col);
      const float o0 = cs[h] * os.x + cl[h] * acc[nb][2 * h];
      const float o1 = cs[h] * os.y + cl[h] * acc[nb][2 * h + 1];
      *reinterpret_cast<uint32_t*>(sO + rl[h] * LD + col) = pack_bf16(o0, o1);
      *reinterpret_cast<uint32_t*>(sS + rl[h] * LD + col) = pack_bf16(os.x, os.y);
      const float il = dl[h] > 0.f ? 1.f / dl[h] : 0.f;
      *reinterpret_cast<uint32_t*>(sL + rl[h] * LD + col) = pack_bf16(acc[nb][2 * h] * il, acc[nb][2 * h + 1] * il);
    }
  }
  if (t4 == 0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int qi = t * T + rl[h];
      if (qi < g.N) {
        logd_out[head + qi] = logd[h];
        dlr_out[head + qi] = dl[h];
        m_out[head + qi] = mfac[h];
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < T * (D / 8); i += NT) {
    const int r = i / (D / 8), c = (i % (D / 8)) * 8;
    const int row = t * T + r;
    if (row < g.N) {
      *reinterpret_cast<uint4*>(O + (head + row) * D + c) = *reinterpret_cast<const uint4*>(sO + r * LD + c);
      *reinterpret_cast<uint4*>(Os_out + (head + row) * D + c) = *reinterpret_cast<const uint4*>(sS + r * LD + c);
      *reinterpret_cast<uint4*>(Olr_out + (head + row) * D + c) = *reinterpret_cast<const uint4*>(sL + r * LD + c);
    }
  }
}

template <int D, int T>
static cudaError_t launch_fwd_t(const FwdArgs& a, const Geom& g, cudaStream_t st) {
  const size_t smem = FwdSmem<D, T>::bytes;
  auto kern = attn_fwd_bf16_kernel<D, T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps("attn_fwd", st);
  kern<<<dim3(g.n_t, g.BH), 2 * T, smem, st>>>(
      (const __nv_bfloat16*)a.Q, (const __nv_bfloat16*)a.K, (const __nv_bfloat16*)a.V, a.idx,
      (const __nv_bfloat16*)a.phiQ, (const __nv_bfloat16*)a.phiK, a.Ast, a.Bst, a.lam, a.gs, a.glr,
      (__nv_bfloat16*)a.O, (__nv_bfloat16*)a.Os, a.logd, a.dlr, a.m, (__nv_bfloat16*)a.Olr, g);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_bf16(const FwdArgs& a, const Geom& g, cudaStream_t st) {
  if (g.d == 64 && g.T == 64) return launch_fwd_t<64, 64>(a, g, st);
  if (g.d == 64 && g.T == 128) return launch_fwd_t<64, 128>(a, g, st);
  if (g.d == 128 && g.T == 64) return launch_fwd_t<128, 64>(a, g, st);
  if (g.d == 128 && g.T == 128) return launch_fwd_t<128, 128>(a, g, st);
  return cudaErrorInvalidValue;
}

}  // namespace elsaa
