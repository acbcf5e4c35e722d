// Backward of the ELSAA operator: exact gradients of sum(dO * O) with respect to
// Q, K and V through the fusion (Eq. 4, Eq. 5 of the ELSAA paper), the sparse
// softmax over the selected blocks (§3.2) and the RACE read-out and features
// (§3.1).  Selection and the hash hyperplanes are constants.
//
// Per row i (default gates g_s = 1, g_lr = 1 - m):
//   dm      = g_s <dO, O_s> - <dO, O_lr>              (the -<dO,O_lr> term only for the default g_lr)
//   dO_s    = cs dO,  cs = g_s m;      dN = cl dO,  cl = g_lr / d_lr
//   Delta   = cs <dO, O_s> - dm m (1 - m)            (the d_s adjoint folded into the softmax delta)
//   delta   = -dm lam d_s / D^2 - cl <dO, O_lr>,     D = d_s + lam d_lr + eps
// Sparse:   dz_ij = P_ij (cs <dO_i, v_j> - Delta_i),  dq += scale dz k, dk += scale dz q, dv += P cs dO.
// RACE:     e_i = [cl dO_i ; delta_i];  dkappa_ij = e_i . [v_j ; 1];
//           dPhi(q_i) = S_i e_i  (S_i: forward prefix statistics incl. own chunk),
//           dPhi(k_j) = U_j [v_j ; 1],  dv_j += U_j^V' Phi(k_j)  (U_j: suffix of Phi(q_i) e_i^T),
//           then through the corner softmax, h = W^T u and u = x / |x|.
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace elsaa {

template <typename E>
__device__ __forceinline__ void load8(const E* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 raw = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = __bfloat162float(e[j]);
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 x = reinterpret_cast<const float4*>(p)[0];
  const float4 y = reinterpret_cast<const float4*>(p)[1];
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
}

// Row scalars (see the header comment).  grid (ceil(N / rows_per_block), BH), block 256;
// d/8 threads per row, 8 elements each.  The scalar algebra runs in float64.
template <typename E>
__global__ void __launch_bounds__(256) row_scalars_kernel(BwdArgs a, Geom g) {
  const int tpr = g.d / 8;
  const int rpb = 256 / tpr;
  const int sub = threadIdx.x % tpr;
  const int row = blockIdx.x * rpb + threadIdx.x / tpr;
  const size_t i = (size_t)blockIdx.y * g.N + min(row, g.N - 1);
  float dO[8], os[8], ol[8];
  load8<E>((const E*)a.dO + i * g.d + sub * 8, dO);
  load8<E>((const E*)a.Os + i * g.d + sub * 8, os);
  load8<E>((const E*)a.Olr + i * g.d + sub * 8, ol);
  float A = 0.f, Bv = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    A += dO[j] * os[j];
    Bv += dO[j] * ol[j];
  }
  for (int o = 1; o < tpr; o <<= 1) {
    A += __shfl_xor_sync(0xffffffffu, A, o);
    Bv += __shfl_xor_sync(0xffffffffu, Bv, o);
  }
  if (sub != 0 || row >= g.N) return;
  const double logd = a.logd[i], dl = a.dlr[i];
  const double lam = a.lam ? a.lam[i] : g.lam;
  const double gs = a.gs ? a.gs[i] : 1.0;
  const double ds = exp(logd);
  const double c = lam * dl + (double)g.eps;
  const double D = ds + c;
  const double m = D > 0.0 ? ds / D : 0.0;
  const double one_m = D > 0.0 ? c / D : 1.0;
  const double gl = a.glr ? (double)a.glr[i] : one_m;
  const double dm = gs * A - (a.glr ? 0.0 : (double)Bv);
  const double cs = gs * m;
  const double cl = dl > 0.0 ? gl / dl : 0.0;
  const double ddlr = D > 0.0 ? -dm * lam * ds / (D * D) : 0.0;
  a.rs.cs[i] = (float)cs;
  a.rs.Delta[i] = (float)(cs * A - dm * m * one_m);
  a.rs.cl[i] = (float)cl;
  a.rs.delta[i] = (float)(ddlr - cl * Bv);
}

cudaError_t launch_row_scalars(const BwdArgs& a, bool bf16, const Geom& g, cudaStream_t st) {
  const int rpb = 256 / (g.d / 8);
  dim3 grid((g.N + rpb - 1) / rpb, g.BH);
  ProfScope ps("row_scalars", st);
  if (bf16) row_scalars_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a, g);
  else row_scalars_kernel<float><<<grid, 256, 0, st>>>(a, g);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Shared pieces of the RACE backward (bf16 path).
// ---------------------------------------------------------------------------

// Pull dPhi of one table through the corner softmax for the 4 corners this
// thread holds (n-blocks 2tl and 2tl+1 of a 16 x 64 fragment, row half h):
// returns dh_b (b = 0..3) reduced over the quad, already divided by tau.
__device__ __forceinline__ void corner_softmax_bwd(const float (&G)[8][4], int tl, int h, const float* hrow,
                                                   float inv_sqrt_L, float tau, int t4, float (&dh)[4]) {
  float sp[4], sm[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const float y = 2.f * hrow[b] / tau;
    sp[b] = 1.f / (1.f + expf(-y));
    sm[b] = 1.f / (1.f + expf(y));
  }
  float p[4], dp[4];
  int cidx[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int nb = 2 * tl + (q >> 1);
    const int c = (q >> 1) * 8 + 2 * t4 + (q & 1);
    cidx[q] = c;
    float pv = 1.f;
#pragma unroll
    for (int b = 0; b < 4; ++b) pv *= ((c >> b) & 1) ? sp[b] : sm[b];
    p[q] = pv;
    dp[q] = G[nb][2 * h + (q & 1)] * inv_sqrt_L;
  }
  float s = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) s += dp[q] * p[q];
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
#pragma unroll
  for (int b = 0; b < 4; ++b) dh[b] = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float da = p[q] * (dp[q] - s);
#pragma unroll
    for (int b = 0; b < 4; ++b) dh[b] += ((cidx[q] >> b) & 1) ? da : -da;
  }
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    dh[b] += __shfl_xor_sync(0xffffffffu, dh[b], 1);
    dh[b] += __shfl_xor_sync(0xffffffffu, dh[b], 2);
    dh[b] /= tau;
  }
}

// du = W dh (all tables), dx = (du - u <u, du>) / n with u = x / n.  One warp per
// row of the tile; writes the fp32 gradient rows.  sdh: [T][ldh] fp32.
template <int D, int T>
__device__ __forceinline__ void feature_chain_rows(const float* sdh, int ldh, const float* __restrict__ W,
                                                   const __nv_bfloat16* __restrict__ X, const float* __restrict__ nrm,
                                                   float* __restrict__ out, int row_base, const Geom& g) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int NH = g.L * kHashBits;
  constexpr int NJ = D / 32;
  for (int r = warp; r < T; r += nw) {
    const int row = row_base + r;
    if (row >= g.N) break;
    float du[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) du[j] = 0.f;
    for (int n = 0; n < NH; ++n) {
      const float dh = sdh[r * ldh + n];
      const float* w = W + (size_t)(n >> 2) * D * kHashBits + (n & 3);
#pragma unroll
      for (int j = 0; j < NJ; ++j) du[j] += dh * w[(size_t)(lane + 32 * j) * kHashBits];
    }
    const float nv = nrm[row];
    float x[NJ], xd = 0.f;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      x[j] = __bfloat162float(X[(size_t)row * D + lane + 32 * j]);
      xd += x[j] * du[j];
    }
    xd = warp_sum(xd);
    const bool floored = nv <= kNormFloor;
    const float proj = floored ? 0.f : xd / (nv * nv);
#pragma unroll
    for (int j = 0; j < NJ; ++j) out[(size_t)row * D + lane + 32 * j] = (du[j] - x[j] * proj) / nv;
  }
}

// Load rows [f0, f0+64) of a float32 state [r][dp] (sum of up to two sources) as
// bf16 hi/lo halves [64][ld] (columns 0..D-1) and the key-mass column as fp32.
// Rows at or beyond `rows` are zero-filled without being read.
template <int D>
__device__ __forceinline__ void load_state_chunk(const float* __restrict__ s0, const float* __restrict__ s1, int f0,
                                                 int rows, int dp, __nv_bfloat16* sh, __nv_bfloat16* sl,
                                                 float* s1col, int ld, int nthr) {
  const int q4 = D / 4;
  for (int i = threadIdx.x; i < 64 * q4; i += nthr) {
    const int r = i / q4, c = (i % q4) * 4;
    if (r >= rows) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sh[r * ld + c + j] = __float2bfloat16_rn(0.f);
        sl[r * ld + c + j] = __float2bfloat16_rn(0.f);
      }
      continue;
    }
    float4 v = *reinterpret_cast<const float4*>(s0 + (size_t)(f0 + r) * dp + c);
    if (s1) {
      const float4 w = *reinterpret_cast<const float4*>(s1 + (size_t)(f0 + r) * dp + c);
      v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
    }
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(vv[j]);
      sh[r * ld + c + j] = hi;
      sl[r * ld + c + j] = __float2bfloat16_rn(vv[j] - __bfloat162float(hi));
    }
  }
  for (int r = threadIdx.x; r < 64; r += nthr) {
    float v = 0.f;
    if (r < rows) {
      v = s0[(size_t)(f0 + r) * dp + D];
      if (s1) v += s1[(size_t)(f0 + r) * dp + D];
    }
    s1col[r] = v;
  }
}

template <int T>
__device__ __forceinline__ void load_rows_bf16(__nv_bfloat16* dst, int ld, const __nv_bfloat16* __restrict__ src,
                                               int src_ld, int col0, int width, int row_base, int N, int nthr) {
  const int ch = width / 8;
  for (int i = threadIdx.x; i < T * ch; i += nthr) {
    const int r = i / ch, c = (i % ch) * 8;
    const int row = row_base + r;
    cp_async16(dst + r * ld + c, src + (size_t)min(row, N - 1) * src_ld + col0 + c, row < N);
  }
}

// ---------------------------------------------------------------------------
// RACE backward, query side: dQacc = chain(dPhi(q)) for one tile of rows.
// grid (n_t, BH), block 2T.
// ---------------------------------------------------------------------------
template <int D, int T>
struct RaceBwdSmem {
  static constexpr int LD = D + 8;
  static constexpr int LDF = 72;
  static constexpr size_t off_a = 0;                                   // dO (q side) / V (k side) [T][LD]
  static constexpr size_t off_b = off_a + (size_t)T * LD * 2;          // V diag (q) / dO (k)     [T][LD]
  static constexpr size_t off_h = off_b + (size_t)T * LD * 2;          // state hi [64][LD]
  static constexpr size_t off_l = off_h + (size_t)64 * LD * 2;         // state lo [64][LD]
  static constexpr size_t off_f1 = off_l + (size_t)64 * LD * 2;        // features [T][LDF]
  static constexpr size_t off_f2 = off_f1 + (size_t)T * LDF * 2;       // features [T][LDF]
  static constexpr size_t off_s1 = off_f2 + (size_t)T * LDF * 2;       // key-mass column [64]
  static constexpr size_t off_cl = off_s1 + 64 * 4;                    // cl [T]
  static constexpr size_t off_dl = off_cl + (size_t)T * 4;             // delta [T]
  static constexpr size_t off_dh = off_dl + (size_t)T * 4;             // dh [T][65]
  static constexpr int LDH = 65;
  static constexpr size_t bytes = off_dh + (size_t)T * LDH * 4;
};

template <int D, int T>
__global__ void __launch_bounds__(2 * T) race_q_bwd_bf16_kernel(BwdArgs a, Geom g) {
  using S = RaceBwdSmem<D, T>;
  constexpr int LD = S::LD, LDF = S::LDF, NT = 2 * T;
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* sdO = reinterpret_cast<__nv_bfloat16*>(smem + S::off_a);
  __nv_bfloat16* sVt = reinterpret_cast<__nv_bfloat16*>(smem + S::off_b);
  __nv_bfloat16* sPh = reinterpret_cast<__nv_bfloat16*>(smem + S::off_h);
  __nv_bfloat16* sPl = reinterpret_cast<__nv_bfloat16*>(smem + S::off_l);
  __nv_bfloat16* sF = reinterpret_cast<__nv_bfloat16*>(smem + S::off_f1);
  float* sp1 = reinterpret_cast<float*>(smem + S::off_s1);
  float* scl = reinterpret_cast<float*>(smem + S::off_cl);
  float* sdel = reinterpret_cast<float*>(smem + S::off_dl);
  float* sdh = reinterpret_cast<float*>(smem + S::off_dh);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g4 = lane >> 2, t4 = lane & 3;
  const int t = blockIdx.x, bh = blockIdx.y;
  const size_t head = (size_t)bh * g.N;
  const int row0 = warp * 16;
  const int rl[2] = {row0 + g4, row0 + g4 + 8};
  const __nv_bfloat16* dO = (const __nv_bfloat16*)a.dO + head * D;
  const __nv_bfloat16* V = (const __nv_bfloat16*)a.V + head * D;

  load_rows_bf16<T>(sdO, LD, dO, D, 0, D, t * T, g.N, NT);
  if (g.causal) load_rows_bf16<T>(sVt, LD, V, D, 0, D, t * T, g.N, NT);
  cp_async_commit();
  for (int r = tid; r < T; r += NT) {
    const int row = t * T + r;
    scl[r] = row < g.N ? a.rs.cl[head + row] : 0.f;
    sdel[r] = row < g.N ? a.rs.delta[head + row] : 0.f;
  }
  cp_async_wait<0>();
  __syncthreads();

  // intra-chunk adjoint dkappa_ij = cl_i <dO_i, v_j> + delta_i (j <= i), as bf16 A fragments
  uint32_t dk_pk[T / 16][4];
  if (g.causal) {
    float X[T / 8][4];
#pragma unroll
    for (int nb = 0; nb < T / 8; ++nb) X[nb][0] = X[nb][1] = X[nb][2] = X[nb][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t af[4];
      ldsm_x4(af, a_frag_ptr(sdO, LD, row0, kk * 16, lane));
#pragma unroll
      for (int nb2 = 0; nb2 < T / 16; ++nb2) {
        uint32_t bf[4];
        ldsm_x4(bf, bnk_frag_ptr(sVt, LD, nb2 * 16, kk * 16, lane));
        mma16816(X[2 * nb2], af, bf[0], bf[1]);
        mma16816(X[2 * nb2 + 1], af, bf[2], bf[3]);
      }
    }
#pragma unroll
    for (int nb = 0; nb < T / 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nb * 8 + 2 * t4 + (e & 1);
        const int r = rl[e >> 1];
        X[nb][e] = col <= r ? scl[r] * X[nb][e] + sdel[r] : 0.f;
      }
    }
#pragma unroll
    for (int kk = 0; kk < T / 16; ++kk) {
      dk_pk[kk][0] = pack_bf16(X[2 * kk][0], X[2 * kk][1]);
      dk_pk[kk][1] = pack_bf16(X[2 * kk][2], X[2 * kk][3]);
      dk_pk[kk][2] = pack_bf16(X[2 * kk + 1][0], X[2 * kk + 1][1]);
      dk_pk[kk][3] = pack_bf16(X[2 * kk + 1][2], X[2 * kk + 1][3]);
    }
  }

  const float* pa = a.Ast + ((size_t)bh * (g.n_seg + 1) + (g.causal ? t / g.seg : g.n_seg)) * g.r * g.dp;
  const float* pb = g.causal ? a.Bst + ((size_t)bh * g.n_c + t) * g.r * g.dp : nullptr;
  const __nv_bfloat16* fk = (const __nv_bfloat16*)a.phiK + head * g.r;
  const float inv_sqrt_L = rsqrtf((float)g.L);
  for (int rc = 0; rc < g.r; rc += 64) {
    const int rcw = min(64, g.r - rc);
    __syncthreads();
    if (g.causal) {
      load_rows_bf16<T>(sF, LDF, fk, g.r, rc, rcw, t * T, g.N, NT);
      cp_async_commit();
    }
    load_state_chunk<D>(pa, pb, rc, rcw, g.dp, sPh, sPl, sp1, LD, NT);
    cp_async_wait<0>();
    __syncthreads();
    float G[8][4];
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) G[nb][0] = G[nb][1] = G[nb][2] = G[nb][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t af[4];
      ldsm_x4(af, a_frag_ptr(sdO, LD, row0, kk * 16, lane));
#pragma unroll
      for (int nb2 = 0; nb2 < 4; ++nb2) {
        if (nb2 * 16 >= rcw) break;
        uint32_t bh_[4], bl_[4];
        ldsm_x4(bh_, bnk_frag_ptr(sPh, LD, nb2 * 16, kk * 16, lane));
        ldsm_x4(bl_, bnk_frag_ptr(sPl, LD, nb2 * 16, kk * 16, lane));
        mma16816(G[2 * nb2], af, bh_[0], bh_[1]);
        mma16816(G[2 * nb2 + 1], af, bh_[2], bh_[3]);
        mma16816(G[2 * nb2], af, bl_[0], bl_[1]);
        mma16816(G[2 * nb2 + 1], af, bl_[2], bl_[3]);
      }
    }
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int f = nb * 8 + 2 * t4 + (e & 1);
        const int r = rl[e >> 1];
        G[nb][e] = scl[r] * G[nb][e] + (f < rcw ? sdel[r] * sp1[f] : 0.f);
      }
    }
    if (g.causal) {
#pragma unroll
      for (int kk = 0; kk < T / 16; ++kk) {
#pragma unroll
        for (int nb2 = 0; nb2 < 4; ++nb2) {
          if (nb2 * 16 >= rcw) break;
          uint32_t bf[4];
          ldsm_x4_t(bf, bkn_frag_ptr(sF, LDF, kk * 16, nb2 * 16, lane));
          mma16816(G[2 * nb2], dk_pk[kk], bf[0], bf[1]);
          mma16816(G[2 * nb2 + 1], dk_pk[kk], bf[2], bf[3]);
        }
      }
    }
    // through the corner softmax, one table (16 features) per n-block pair
#pragma unroll
    for (int tl = 0; tl < 4; ++tl) {
      if (tl * 16 >= rcw) break;
      const int l = rc / 16 + tl;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = min(t * T + rl[h], g.N - 1);
        const float* hrow = a.hQ + (head + row) * (g.L * kHashBits) + l * kHashBits;
        float hv[4] = {hrow[0], hrow[1], hrow[2], hrow[3]};
        float dh[4];
        corner_softmax_bwd(G, tl, h, hv, inv_sqrt_L, g.tau, t4, dh);
        if (t4 == 0) {
#pragma unroll
          for (int b = 0; b < 4; ++b) sdh[rl[h] * S::LDH + l * kHashBits + b] = dh[b];
        }
      }
    }
  }
  __syncthreads();
  feature_chain_rows<D, T>(sdh, S::LDH, a.W, (const __nv_bfloat16*)a.Q + head * D, a.nQ + head,
                           a.dQacc + head * D, t * T, g);
}

// ---------------------------------------------------------------------------
// RACE backward, key side: dKacc = chain(dPhi(k)), dVacc = low-rank value
// gradient, for one key chunk (== block).  grid (n_t, BH), block 2T.
// ---------------------------------------------------------------------------
template <int D, int T>
__global__ void __launch_bounds__(2 * T) race_k_bwd_bf16_kernel(BwdArgs a, Geom g) {
  using S = RaceBwdSmem<D, T>;
  constexpr int LD = S::LD, LDF = S::LDF, NT = 2 * T, NBD = D / 8;
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + S::off_a);
  __nv_bfloat16* sdO = reinterpret_cast<__nv_bfloat16*>(smem + S::off_b);
  __nv_bfloat16* sRh = reinterpret_cast<__nv_bfloat16*>(smem + S::off_h);
  __nv_bfloat16* sRl = reinterpret_cast<__nv_bfloat16*>(smem + S::off_l);
  __nv_bfloat16* sFk = reinterpret_cast<__nv_bfloat16*>(smem + S::off_f1);
  __nv_bfloat16* sFq = reinterpret_cast<__nv_bfloat16*>(smem + S::off_f2);
  float* sr1 = reinterpret_cast<float*>(smem + S::off_s1);
  float* scl = reinterpret_cast<float*>(smem + S::off_cl);
  float* sdel = reinterpret_cast<float*>(smem + S::off_dl);
  float* sdh = reinterpret_cast<float*>(smem + S::off_dh);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g4 = lane >> 2, t4 = lane & 3;
  const int c = blockIdx.x, bh = blockIdx.y;
  const size_t head = (size_t)bh * g.N;
  const int row0 = warp * 16;
  const int rl[2] = {row0 + g4, row0 + g4 + 8};
  const __nv_bfloat16* dO = (const __nv_bfloat16*)a.dO + head * D;
  const __nv_bfloat16* V = (const __nv_bfloat16*)a.V + head * D;
  const __nv_bfloat16* fk = (const __nv_bfloat16*)a.phiK + head * g.r;
  const __nv_bfloat16* fq = (const __nv_bfloat16*)a.phiQ + head * g.r;

  load_rows_bf16<T>(sV, LD, V, D, 0, D, c * T, g.N, NT);
  if (g.causal) load_rows_bf16<T>(sdO, LD, dO, D, 0, D, c * T, g.N, NT);
  cp_async_commit();
  for (int r = tid; r < T; r += NT) {
    const int row = c * T + r;
    scl[r] = row < g.N ? a.rs.cl[head + row] : 0.f;
    sdel[r] = row < g.N ? a.rs.delta[head + row] : 0.f;
  }
  cp_async_wait<0>();
  __syncthreads();

  uint32_t dkT[T / 16][4], kT[T / 16][4];
  if (g.causal) {
    // dkappa^T[j][i] = cl_i <dO_i, v_j> + delta_i for i >= j (rows j: keys, cols i: queries)
    float X[T / 8][4];
#pragma unroll
    for (int nb = 0; nb < T / 8; ++nb) X[nb][0] = X[nb][1] = X[nb][2] = X[nb][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t af[4];
      ldsm_x4(af, a_frag_ptr(sV, LD, row0, kk * 16, lane));
#pragma unroll
      for (int nb2 = 0; nb2 < T / 16; ++nb2) {
        uint32_t bf[4];
        ldsm_x4(bf, bnk_frag_ptr(sdO, LD, nb2 * 16, kk * 16, lane));
        mma16816(X[2 * nb2], af, bf[0], bf[1]);
        mma16816(X[2 * nb2 + 1], af, bf[2], bf[3]);
      }
    }
#pragma unroll
    for (int nb = 0; nb < T / 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nb * 8 + 2 * t4 + (e & 1);
        X[nb][e] = col >= rl[e >> 1] ? scl[col] * X[nb][e] + sdel[col] : 0.f;
      }
    }
#pragma unroll
    for (int kk = 0; kk < T / 16; ++kk) {
      dkT[kk][0] = pack_bf16(X[2 * kk][0], X[2 * kk][1]);
      dkT[kk][1] = pack_bf16(X[2 * kk][2], X[2 * kk][3]);
      dkT[kk][2] = pack_bf16(X[2 * kk + 1][0], X[2 * kk + 1][1]);
      dkT[kk][3] = pack_bf16(X[2 * kk + 1][2], X[2 * kk + 1][3]);
    }
    // kappa^T[j][i] = Phi(k_j).Phi(q_i), i >= j, scaled by cl_i
#pragma unroll
    for (int nb = 0; nb < T / 8; ++nb) X[nb][0] = X[nb][1] = X[nb][2] = X[nb][3] = 0.f;
    for (int rc = 0; rc < g.r; rc += 64) {
      const int rcw = min(64, g.r - rc);
      __syncthreads();
      load_rows_bf16<T>(sFk, LDF, fk, g.r, rc, rcw, c * T, g.N, NT);
      load_rows_bf16<T>(sFq, LDF, fq, g.r, rc, rcw, c * T, g.N, NT);
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
      for (int kk = 0; kk < rcw / 16; ++kk) {
        uint32_t af[4];
        ldsm_x4(af, a_frag_ptr(sFk, LDF, row0, kk * 16, lane));
#pragma unroll
        for (int nb2 = 0; nb2 < T / 16; ++nb2) {
          uint32_t bf[4];
          ldsm_x4(bf, bnk_frag_ptr(sFq, LDF, nb2 * 16, kk * 16, lane));
          mma16816(X[2 * nb2], af, bf[0], bf[1]);
          mma16816(X[2 * nb2 + 1], af, bf[2], bf[3]);
        }
      }
    }
#pragma unroll
    for (int nb = 0; nb < T / 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nb * 8 + 2 * t4 + (e & 1);
        X[nb][e] = col >= rl[e >> 1] ? scl[col] * X[nb][e] : 0.f;
      }
    }
#pragma unroll
    for (int kk = 0; kk < T / 16; ++kk) {
      kT[kk][0] = pack_bf16(X[2 * kk][0], X[2 * kk][1]);
      kT[kk][1] = pack_bf16(X[2 * kk][2], X[2 * kk][3]);
      kT[kk][2] = pack_bf16(X[2 * kk + 1][0], X[2 * kk + 1][1]);
      kT[kk][3] = pack_bf16(X[2 * kk + 1][2], X[2 * kk + 1][3]);
    }
  }

  // dV_lr = kappa^T (cl dO) [intra] + Phi_K R^V [inter]
  float dv[NBD][4];
#pragma unroll
  for (int nb = 0; nb < NBD; ++nb) dv[nb][0] = dv[nb][1] = dv[nb][2] = dv[nb][3] = 0.f;
  if (g.causal) {
#pragma unroll
    for (int kk = 0; kk < T / 16; ++kk) {
#pragma unroll
      for (int nb2 = 0; nb2 < NBD / 2; ++nb2) {
        uint32_t bf[4];
        ldsm_x4_t(bf, bkn_frag_ptr(sdO, LD, kk * 16, nb2 * 16, lane));
        mma16816(dv[2 * nb2], kT[kk], bf[0], bf[1]);
        mma16816(dv[2 * nb2 + 1], kT[kk], bf[2], bf[3]);
      }
    }
  }
  const float* ra = a.RA + ((size_t)bh * (g.n_seg + 1) + (g.causal ? c / g.seg + 1 : 0)) * g.r * g.dp;
  const float* rb = g.causal ? a.RB + ((size_t)bh * g.n_c + c) * g.r * g.dp : nullptr;
  const float inv_sqrt_L = rsqrtf((float)g.L);
  for (int rc = 0; rc < g.r; rc += 64) {
    const int rcw = min(64, g.r - rc);
    __syncthreads();
    load_rows_bf16<T>(sFk, LDF, fk, g.r, rc, rcw, c * T, g.N, NT);
    if (g.causal) load_rows_bf16<T>(sFq, LDF, fq, g.r, rc, rcw, c * T, g.N, NT);
    cp_async_commit();
    load_state_chunk<D>(ra, rb, rc, rcw, g.dp, sRh, sRl, sr1, LD, NT);
    cp_async_wait<0>();
    __syncthreads();
    // inter-chunk value gradient: Phi_K[:, rc:rc+64] R^V[rc:rc+64, :]
    for (int kk = 0; kk < rcw / 16; ++kk) {
      uint32_t af[4];
      ldsm_x4(af, a_frag_ptr(sFk, LDF, row0, kk * 16, lane));
#pragma unroll
      for (int nb2 = 0; nb2 < NBD / 2; ++nb2) {
        uint32_t bh_[4], bl_[4];
        ldsm_x4_t(bh_, bkn_frag_ptr(sRh, LD, kk * 16, nb2 * 16, lane));
        ldsm_x4_t(bl_, bkn_frag_ptr(sRl, LD, kk * 16, nb2 * 16, lane));
        mma16816(dv[2 * nb2], af, bh_[0], bh_[1]);
        mma16816(dv[2 * nb2 + 1], af, bh_[2], bh_[3]);
        mma16816(dv[2 * nb2], af, bl_[0], bl_[1]);
        mma16816(dv[2 * nb2 + 1], af, bl_[2], bl_[3]);
      }
    }
    // dPhi(k_j) for this feature chunk: R^V v_j + R^1 + sum_{i >= j} dkappa_ij Phi(q_i)
    float G[8][4];
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) G[nb][0] = G[nb][1] = G[nb][2] = G[nb][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t af[4];
      ldsm_x4(af, a_frag_ptr(sV, LD, row0, kk * 16, lane));
#pragma unroll
      for (int nb2 = 0; nb2 < 4; ++nb2) {
        if (nb2 * 16 >= rcw) break;
        uint32_t bh_[4], bl_[4];
        ldsm_x4(bh_, bnk_frag_ptr(sRh, LD, nb2 * 16, kk * 16, lane));
        ldsm_x4(bl_, bnk_frag_ptr(sRl, LD, nb2 * 16, kk * 16, lane));
        mma16816(G[2 * nb2], af, bh_[0], bh_[1]);
        mma16816(G[2 * nb2 + 1], af, bh_[2], bh_[3]);
        mma16816(G[2 * nb2], af, bl_[0], bl_[1]);
        mma16816(G[2 * nb2 + 1], af, bl_[2], bl_[3]);
      }
    }
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int f = nb * 8 + 2 * t4 + (e & 1);
        const int row = c * T + rl[e >> 1];
        if (f < rcw && row < g.N) G[nb][e] += sr1[f];
      }
    }
    if (g.causal) {
#pragma unroll
      for (int kk = 0; kk < T / 16; ++kk) {
#pragma unroll
        for (int nb2 = 0; nb2 < 4; ++nb2) {
          if (nb2 * 16 >= rcw) break;
          uint32_t bf[4];
          ldsm_x4_t(bf, bkn_frag_ptr(sFq, LDF, kk * 16, nb2 * 16, lane));
          mma16816(G[2 * nb2], dkT[kk], bf[0], bf[1]);
          mma16816(G[2 * nb2 + 1], dkT[kk], bf[2], bf[3]);
        }
      }
    }
#pragma unroll
    for (int tl = 0; tl < 4; ++tl) {
      if (tl * 16 >= rcw) break;
      const int l = rc / 16 + tl;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = min(c * T + rl[h], g.N - 1);
        const float* hrow = a.hK + (head + row) * (g.L * kHashBits) + l * kHashBits;
        float hv[4] = {hrow[0], hrow[1], hrow[2], hrow[3]};
        float dh[4];
        corner_softmax_bwd(G, tl, h, hv, inv_sqrt_L, g.tau, t4, dh);
        if (t4 == 0) {
#pragma unroll
          for (int b = 0; b < 4; ++b) sdh[rl[h] * S::LDH + l * kHashBits + b] = dh[b];
        }
      }
    }
  }
  // value gradient rows
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = c * T + rl[h];
    if (row < g.N) {
#pragma unroll
      for (int nb = 0; nb < NBD; ++nb) {
        const int col = nb * 8 + 2 * t4;
        *reinterpret_cast<float2*>(a.dVacc + (head + row) * D + col) = make_float2(dv[nb][2 * h], dv[nb][2 * h + 1]);
      }
    }
  }
  __syncthreads();
  feature_chain_rows<D, T>(sdh, S::LDH, a.W, (const __nv_bfloat16*)a.K + head * D, a.nK + head,
                           a.dKacc + head * D, c * T, g);
}

// ---------------------------------------------------------------------------
// Sparse branch backward, query side: dQ = scale sum_j dz_ij k_j (+ low-rank part).
// Each selected key block is processed in halves of 64 keys.  grid (n_t, BH), block 2T.
// ---------------------------------------------------------------------------
template <int D, int T>
__global__ void __launch_bounds__(2 * T) sparse_dq_bf16_kernel(BwdArgs a, Geom g) {
  constexpr int LD = D + 8, NT = 2 * T, NBD = D / 8, HK = 64;
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sdO = sQ + T * LD;
  __nv_bfloat16* sK = sdO + T * LD;     // [2][T][LD]
  __nv_bfloat16* sV = sK + 2 * T * LD;  // [2][T][LD]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g4 = lane >> 2, t4 = lane & 3;
  const int t = g.n_t - 1 - blockIdx.x, bh = blockIdx.y;
  const size_t head = (size_t)bh * g.N;
  const int row0 = warp * 16;
  const int rl[2] = {row0 + g4, row0 + g4 + 8};
  const __nv_bfloat16* Q = (const __nv_bfloat16*)a.Q + head * D;
  const __nv_bfloat16* K = (const __nv_bfloat16*)a.K + head * D;
  const __nv_bfloat16* V = (const __nv_bfloat16*)a.V + head * D;
  const __nv_bfloat16* dO = (const __nv_bfloat16*)a.dO + head * D;
  const int* my_idx = a.idx + ((size_t)bh * g.n_t + t) * g.k;
  int n_sel = 0;
  while (n_sel < g.k && my_idx[n_sel] >= 0) ++n_sel;

  load_rows_bf16<T>(sQ, LD, Q, D, 0, D, t * T, g.N, NT);
  load_rows_bf16<T>(sdO, LD, dO, D, 0, D, t * T, g.N, NT);
  cp_async_commit();
  auto load_kv = [&](int buf, int b) {
    load_rows_bf16<T>(sK + buf * T * LD, LD, K, D, 0, D, b * T, g.N, NT);
    load_rows_bf16<T>(sV + buf * T * LD, LD, V, D, 0, D, b * T, g.N, NT);
  };
  float lg2[2], cs[2], Dl[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = t * T + rl[h];
    const bool ok = row < g.N;
    lg2[h] = ok ? a.logd[head + row] * kLog2e : INFINITY;
    cs[h] = ok ? a.rs.cs[head + row] : 0.f;
    Dl[h] = ok ? a.rs.Delta[head + row] : 0.f;
  }
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
  float dq[NBD][4];
#pragma unroll
  for (int nb = 0; nb < NBD; ++nb) dq[nb][0] = dq[nb][1] = dq[nb][2] = dq[nb][3] = 0.f;
  const float sl2 = g.scale * kLog2e;

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
    const bool diag = g.causal && b == t;
#pragma unroll 1
    for (int hk = 0; hk < T / HK; ++hk) {
      const int k0 = hk * HK;
      float s[8][4], dp[8][4];
#pragma unroll
      for (int nb = 0; nb < 8; ++nb) {
        s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
        dp[nb][0] = dp[nb][1] = dp[nb][2] = dp[nb][3] = 0.f;
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t af[4];
        ldsm_x4(af, a_frag_ptr(sdO, LD, row0, kk * 16, lane));
#pragma unroll
        for (int nb2 = 0; nb2 < 4; ++nb2) {
          uint32_t bk[4], bv[4];
          ldsm_x4(bk, bnk_frag_ptr(cK, LD, k0 + nb2 * 16, kk * 16, lane));
          ldsm_x4(bv, bnk_frag_ptr(cV, LD, k0 + nb2 * 16, kk * 16, lane));
          mma16816(s[2 * nb2], qf[kk], bk[0], bk[1]);
          mma16816(s[2 * nb2 + 1], qf[kk], bk[2], bk[3]);
          mma16816(dp[2 * nb2], af, bv[0], bv[1]);
          mma16816(dp[2 * nb2 + 1], af, bv[2], bv[3]);
        }
      }
#pragma unroll
      for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = e >> 1;
          const int col = k0 + nb * 8 + 2 * t4 + (e & 1);
          const bool masked = (diag && col > rl[h]) || (b * T + col >= g.N);
          const float p = masked ? 0.f : exp2f(s[nb][e] * sl2 - lg2[h]);
          s[nb][e] = p * (cs[h] * dp[nb][e] - Dl[h]);
        }
      }
#pragma unroll
      for (int kk = 0; kk < HK / 16; ++kk) {
        uint32_t af[4];
        af[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
        af[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
        af[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        af[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int nb2 = 0; nb2 < NBD / 2; ++nb2) {
          uint32_t bf[4];
          ldsm_x4_t(bf, bkn_frag_ptr(cK, LD, k0 + kk * 16, nb2 * 16, lane));
          mma16816(dq[2 * nb2], af, bf[0], bf[1]);
          mma16816(dq[2 * nb2 + 1], af, bf[2], bf[3]);
        }
      }
    }
    __syncthreads();
  }
  // epilogue: dQ = scale * dq (+ low-rank part), bf16, staged for 16-byte stores
  __nv_bfloat16* sO = sK;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = t * T + rl[h];
    const int rowc = min(row, g.N - 1);
#pragma unroll
    for (int nb = 0; nb < NBD; ++nb) {
      const int col = nb * 8 + 2 * t4;
      float x0 = g.scale * dq[nb][2 * h], x1 = g.scale * dq[nb][2 * h + 1];
      if (a.dQacc) {
        const float2 l = *reinterpret_cast<const float2*>(a.dQacc + (head + rowc) * D + col);
        x0 += l.x;
        x1 += l.y;
      }
      *reinterpret_cast<uint32_t*>(sO + rl[h] * LD + col) = pack_bf16(x0, x1);
    }
  }
  __syncthreads();
  __nv_bfloat16* out = (__nv_bfloat16*)a.dQ + head * D;
  for (int i = tid; i < T * (D / 8); i += NT) {
    const int r = i / (D / 8), cc = (i % (D / 8)) * 8;
    const int row = t * T + r;
    if (row < g.N) *reinterpret_cast<uint4*>(out + (size_t)row * D + cc) = *reinterpret_cast<const uint4*>(sO + r * LD + cc);
  }
}

// ---------------------------------------------------------------------------
// Sparse branch backward, key side: for key block b, loop over the query tiles
// that selected it (ascending, deterministic, no atomics), in halves of 64
// queries:  dV += P^T (cs dO),  dK += scale dz^T Q.  grid (n_t, BH), block 2T.
// ---------------------------------------------------------------------------
template <int D, int T>
__global__ void __launch_bounds__(2 * T) sparse_dkdv_bf16_kernel(BwdArgs a, Geom g) {
  constexpr int LD = D + 8, NT = 2 * T, NBD = D / 8, HQ = 64;
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sV = sK + T * LD;
  __nv_bfloat16* sQ = sV + T * LD;       // [2][T][LD]
  __nv_bfloat16* sdO = sQ + 2 * T * LD;  // [2][T][LD]
  float* ssc = reinterpret_cast<float*>(sdO + 2 * T * LD);   // [2][3][T]: log2 d_s, cs, Delta
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g4 = lane >> 2, t4 = lane & 3;
  const int b = blockIdx.x, bh = blockIdx.y;
  const size_t head = (size_t)bh * g.N;
  const int row0 = warp * 16;
  const int rl[2] = {row0 + g4, row0 + g4 + 8};
  const __nv_bfloat16* Q = (const __nv_bfloat16*)a.Q + head * D;
  const __nv_bfloat16* K = (const __nv_bfloat16*)a.K + head * D;
  const __nv_bfloat16* V = (const __nv_bfloat16*)a.V + head * D;
  const __nv_bfloat16* dO = (const __nv_bfloat16*)a.dO + head * D;
  int l0 = 0, l1 = 0;
  const int* list = nullptr;
  if (g.k > 0) {
    const int* of = a.offs + (size_t)bh * (g.n_t + 1);
    l0 = of[b];
    l1 = of[b + 1];
    list = a.tiles + (size_t)bh * g.n_t * g.k;
  }
  const int n_list = l1 - l0;

  load_rows_bf16<T>(sK, LD, K, D, 0, D, b * T, g.N, NT);
  load_rows_bf16<T>(sV, LD, V, D, 0, D, b * T, g.N, NT);
  cp_async_commit();
  auto load_q = [&](int buf, int t) {
    load_rows_bf16<T>(sQ + buf * T * LD, LD, Q, D, 0, D, t * T, g.N, NT);
    load_rows_bf16<T>(sdO + buf * T * LD, LD, dO, D, 0, D, t * T, g.N, NT);
    float* sc = ssc + buf * 3 * T;
    for (int r = tid; r < T; r += NT) {
      const int row = t * T + r;
      const bool ok = row < g.N;
      sc[r] = ok ? a.logd[head + row] * kLog2e : INFINITY;
      sc[T + r] = ok ? a.rs.cs[head + row] : 0.f;
      sc[2 * T + r] = ok ? a.rs.Delta[head + row] : 0.f;
    }
  };
  if (n_list > 0) {
    load_q(0, list[l0]);
    cp_async_commit();
  }
  float dk[NBD][4], dv[NBD][4];
#pragma unroll
  for (int nb = 0; nb < NBD; ++nb) {
    dk[nb][0] = dk[nb][1] = dk[nb][2] = dk[nb][3] = 0.f;
    dv[nb][0] = dv[nb][1] = dv[nb][2] = dv[nb][3] = 0.f;
  }
  const float sl2 = g.scale * kLog2e;
  for (int it = 0; it < n_list; ++it) {
    if (it + 1 < n_list) {
      load_q((it + 1) & 1, list[l0 + it + 1]);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int t = list[l0 + it];
    const __nv_bfloat16* cQ = sQ + (it & 1) * T * LD;
    const __nv_bfloat16* cdO = sdO + (it & 1) * T * LD;
    const float* sc = ssc + (it & 1) * 3 * T;
    const bool diag = g.causal && t == b;
#pragma unroll 1
    for (int hq = 0; hq < T / HQ; ++hq) {
      const int q0 = hq * HQ;
      float s[8][4], dp[8][4];
#pragma unroll
      for (int nb = 0; nb < 8; ++nb) {
        s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
        dp[nb][0] = dp[nb][1] = dp[nb][2] = dp[nb][3] = 0.f;
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t ak[4], av[4];
        ldsm_x4(ak, a_frag_ptr(sK, LD, row0, kk * 16, lane));
        ldsm_x4(av, a_frag_ptr(sV, LD, row0, kk * 16, lane));
#pragma unroll
        for (int nb2 = 0; nb2 < 4; ++nb2) {
          uint32_t bq[4], bo[4];
          ldsm_x4(bq, bnk_frag_ptr(cQ, LD, q0 + nb2 * 16, kk * 16, lane));
          ldsm_x4(bo, bnk_frag_ptr(cdO, LD, q0 + nb2 * 16, kk * 16, lane));
          mma16816(s[2 * nb2], ak, bq[0], bq[1]);
          mma16816(s[2 * nb2 + 1], ak, bq[2], bq[3]);
          mma16816(dp[2 * nb2], av, bo[0], bo[1]);
          mma16816(dp[2 * nb2 + 1], av, bo[2], bo[3]);
        }
      }
      // P^T[j][i] and dz^T[j][i]; the P^T operand of dV carries cs_i
#pragma unroll
      for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = q0 + nb * 8 + 2 * t4 + (e & 1);   // query (local)
          const int key = rl[e >> 1];                       // key (local)
          const bool masked = (diag && key > col) || (b * T + key >= g.N);
          const float p = masked ? 0.f : exp2f(s[nb][e] * sl2 - sc[col]);
          const float c = sc[T + col];
          s[nb][e] = p * c;
          dp[nb][e] = p * (c * dp[nb][e] - sc[2 * T + col]);
        }
      }
#pragma unroll
      for (int kk = 0; kk < HQ / 16; ++kk) {
        uint32_t ap[4], as[4];
        ap[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
        ap[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
        ap[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        ap[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
        as[0] = pack_bf16(dp[2 * kk][0], dp[2 * kk][1]);
        as[1] = pack_bf16(dp[2 * kk][2], dp[2 * kk][3]);
        as[2] = pack_bf16(dp[2 * kk + 1][0], dp[2 * kk + 1][1]);
        as[3] = pack_bf16(dp[2 * kk + 1][2], dp[2 * kk + 1][3]);
#pragma unroll
        for (int nb2 = 0; nb2 < NBD / 2; ++nb2) {
          uint32_t bo[4], bq[4];
          ldsm_x4_t(bo, bkn_frag_ptr(cdO, LD, q0 + kk * 16, nb2 * 16, lane));
          ldsm_x4_t(bq, bkn_frag_ptr(cQ, LD, q0 + kk * 16, nb2 * 16, lane));
          mma16816(dv[2 * nb2], ap, bo[0], bo[1]);
          mma16816(dv[2 * nb2 + 1], ap, bo[2], bo[3]);
          mma16816(dk[2 * nb2], as, bq[0], bq[1]);
          mma16816(dk[2 * nb2 + 1], as, bq[2], bq[3]);
        }
      }
    }
    __syncthreads();
  }
  if (n_list == 0) cp_async_wait<0>();
  __syncthreads();
  // epilogue: dK = scale dk (+ low-rank), dV = dv (+ low-rank); stage in the Q buffers
  __nv_bfloat16* sOk = sQ;
  __nv_bfloat16* sOv = sQ + T * LD;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int rowc = min(b * T + rl[h], g.N - 1);
#pragma unroll
    for (int nb = 0; nb < NBD; ++nb) {
      const int col = nb * 8 + 2 * t4;
      float k0 = g.scale * dk[nb][2 * h], k1 = g.scale * dk[nb][2 * h + 1];
      float v0 = dv[nb][2 * h], v1 = dv[nb][2 * h + 1];
      if (a.dKacc) {
        const float2 lk = *reinterpret_cast<const float2*>(a.dKacc + (head + rowc) * D + col);
        const float2 lv = *reinterpret_cast<const float2*>(a.dVacc + (head + rowc) * D + col);
        k0 += lk.x; k1 += lk.y; v0 += lv.x; v1 += lv.y;
      }
      *reinterpret_cast<uint32_t*>(sOk + rl[h] * LD + col) = pack_bf16(k0, k1);
      *reinterpret_cast<uint32_t*>(sOv + rl[h] * LD + col) = pack_bf16(v0, v1);
    }
  }
  __syncthreads();
  __nv_bfloat16* outk = (__nv_bfloat16*)a.dK + head * D;
  __nv_bfloat16* outv = (__nv_bfloat16*)a.dV + head * D;
  for (int i = tid; i < T * (D / 8); i += NT) {
    const int r = i / (D / 8), cc = (i % (D / 8)) * 8;
    const int row = b * T + r;
    if (row < g.N) {
      *reinterpret_cast<uint4*>(outk + (size_t)row * D + cc) = *reinterpret_cast<const uint4*>(sOk + r * LD + cc);
      *reinterpret_cast<uint4*>(outv + (size_t)row * D + cc) = *reinterpret_cast<const uint4*>(sOv + r * LD + cc);
    }
  }
}

template <typename KernT>
static cudaError_t launch2(const char* name, KernT kern, size_t smem, int T, const BwdArgs& a, const Geom& g,
                           cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(name, st);
  kern<<<dim3(g.n_t, g.BH), 2 * T, smem, st>>>(a, g);
  return cudaGetLastError();
}

template <int D, int T>
static cudaError_t bwd_t(const BwdArgs& a0, const Geom& g, cudaStream_t st) {
  BwdArgs a = a0;
  cudaError_t e;
  if (g.r > 0) {
    e = launch2("race_q_bwd", race_q_bwd_bf16_kernel<D, T>, RaceBwdSmem<D, T>::bytes, T, a, g, st);
    if (e != cudaSuccess) return e;
    e = launch2("race_k_bwd", race_k_bwd_bf16_kernel<D, T>, RaceBwdSmem<D, T>::bytes, T, a, g, st);
    if (e != cudaSuccess) return e;
  } else {
    a.dQacc = a.dKacc = a.dVacc = nullptr;
  }
  const size_t lds = (size_t)(D + 8) * 2;
  e = launch2("sparse_dq", sparse_dq_bf16_kernel<D, T>, (size_t)6 * T * lds, T, a, g, st);
  if (e != cudaSuccess) return e;
  return launch2("sparse_dkdv", sparse_dkdv_bf16_kernel<D, T>, (size_t)6 * T * lds + (size_t)6 * T * 4, T, a, g, st);
}

cudaError_t launch_bwd_bf16(const BwdArgs& a, const Geom& g, cudaStream_t st) {
  if (g.d == 64 && g.T == 64) return bwd_t<64, 64>(a, g, st);
  if (g.d == 64 && g.T == 128) return bwd_t<64, 128>(a, g, st);
  if (g.d == 128 && g.T == 64) return bwd_t<128, 64>(a, g, st);
  if (g.d == 128 && g.T == 128) return bwd_t<128, 128>(a, g, st);
  return cudaErrorInvalidValue;
}

}  // namespace elsaa
