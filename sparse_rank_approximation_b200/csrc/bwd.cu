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

// Row scalars (see the header comment).  grid (ceil(N / rows_per_block), BH), block 256.
// d/8 threads per row reduce the row's <dO, O_s> and <dO, O_lr> (8 elements each); then
// one thread per row (the block's first rows_per_block threads, so a warp covers 16 or 32
// consecutive rows) runs the scalar algebra in float64 and writes the per-row outputs;
// cl comes back through shared memory for the cl dO rows.
template <typename E>
__global__ void __launch_bounds__(256) row_scalars_kernel(BwdArgs a, Geom g) {
  __shared__ float sA[32], sB[32], sCl[32];
  const int tpr = g.d / 8;
  const int rpb = 256 / tpr;
  const int sub = threadIdx.x % tpr;
  const int lr = threadIdx.x / tpr;
  const int row = blockIdx.x * rpb + lr;
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
  if (sub == 0) {
    sA[lr] = A;
    sB[lr] = Bv;
  }
  __syncthreads();
  if ((int)threadIdx.x < rpb) {
    const int r = blockIdx.x * rpb + threadIdx.x;
    float clv = 0.f;
    if (r < g.N) {
      const size_t k = (size_t)blockIdx.y * g.N + r;
      const double Ar = sA[threadIdx.x], Br = sB[threadIdx.x];
      const double logd = a.logd[k], dl = a.dlr[k];
      const double lam = a.lam ? a.lam[k] : g.lam;
      const double gs = a.gs ? a.gs[k] : 1.0;
      const double ds = exp(logd);
      const double c = lam * dl + (double)g.eps;
      const double D = ds + c;
      // fixed_m: the ablation without denominator-aware fusion (m = 1, default g_lr = 1, no dm)
      const double m = g.fixed_m ? 1.0 : D > 0.0 ? ds / D : 0.0;
      const double one_m = g.fixed_m ? 0.0 : D > 0.0 ? c / D : 1.0;
      const double gl = a.glr ? (double)a.glr[k] : g.fixed_m ? 1.0 : one_m;
      const double dm = g.fixed_m ? 0.0 : gs * Ar - (a.glr ? 0.0 : Br);
      const double cs = gs * m;
      const double cl = dl > 0.0 ? gl / dl : 0.0;
      const double ddlr = D > 0.0 ? -dm * lam * ds / (D * D) : 0.0;
      const double Dl = cs * Ar - dm * m * one_m;
      a.rs.cs[k] = (float)cs;
      a.rs.Delta[k] = (float)Dl;
      if (a.rs.packed) a.rs.packed[k] = make_float4((float)(logd * 1.4426950408889634), (float)cs, (float)Dl, 0.f);
      a.rs.cl[k] = (float)cl;
      a.rs.delta[k] = (float)(ddlr - cl * Br);
      clv = (float)cl;
    }
    sCl[threadIdx.x] = clv;
  }
  // the rows cl dO (bf16) feed the RACE suffix statistics
  if (a.dOcl) {
    __syncthreads();
    if (row < g.N) {
      const float clf = sCl[lr];
      uint4 w;
      w.x = pack_bf16(clf * dO[0], clf * dO[1]);
      w.y = pack_bf16(clf * dO[2], clf * dO[3]);
      w.z = pack_bf16(clf * dO[4], clf * dO[5]);
      w.w = pack_bf16(clf * dO[6], clf * dO[7]);
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dOcl) + i * g.d + sub * 8) = w;
    }
  }
}

// Per-row gradients of sum(dO * O) with respect to lambda, g_s and g_lr (Eq. 5 / Eq. 4):
// dlambda = -dm d_s d_lr / D^2 (0 when m is held at 1), dg_s = m <dO, O_s>, dg_lr = <dO, O_lr>,
// dm = g_s <dO, O_s> - [g_lr defaulted] <dO, O_lr>.  Same row layout as the row scalars.
template <typename E>
__global__ void __launch_bounds__(256) fusion_grads_kernel(const E* __restrict__ dO_, const E* __restrict__ Os_,
                                                           const E* __restrict__ Olr_, const float* __restrict__ logd_,
                                                           const float* __restrict__ dlr_, const float* lamv,
                                                           const float* gsv, const float* glrv, float* dlam,
                                                           float* dgs, float* dglr, const int* perm,
                                                           int perm_stride, Geom g) {
  const int tpr = g.d / 8;
  const int rpb = 256 / tpr;
  const int sub = threadIdx.x % tpr;
  const int row = blockIdx.x * rpb + threadIdx.x / tpr;
  const size_t i = (size_t)blockIdx.y * g.N + min(row, g.N - 1);    // row of the saved state
  // the caller's row: the same, or where the sortLSH order put this one
  const size_t io = perm ? (size_t)blockIdx.y * g.N + perm[(size_t)blockIdx.y * perm_stride + min(row, g.N - 1)] : i;
  float dO[8], os[8], ol[8];
  load8<E>(dO_ + io * g.d + sub * 8, dO);
  load8<E>(Os_ + i * g.d + sub * 8, os);
  load8<E>(Olr_ + i * g.d + sub * 8, ol);
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
  const double dl = dlr_[i], ds = exp((double)logd_[i]);
  const double lam = lamv ? lamv[io] : g.lam;
  const double gs = gsv ? gsv[io] : 1.0;
  const double D = ds + lam * dl + (double)g.eps;
  const double m = g.fixed_m ? 1.0 : D > 0.0 ? ds / D : 0.0;
  const double dm = g.fixed_m ? 0.0 : gs * A - (glrv ? 0.0 : (double)Bv);
  if (dlam) dlam[io] = (g.fixed_m || !(D > 0.0)) ? 0.f : (float)(-dm * ds * dl / (D * D));
  if (dgs) dgs[io] = (float)(m * A);
  if (dglr) dglr[io] = Bv;
}

cudaError_t launch_fusion_grads(const void* dO, const void* Os, const void* Olr, const float* logd, const float* dlr,
                                const float* lam, const float* gs, const float* glr, float* dlam, float* dgs,
                                float* dglr, const int* perm, int perm_stride, bool bf16, const Geom& g,
                                cudaStream_t st) {
  const int rpb = 256 / (g.d / 8);
  dim3 grid((g.N + rpb - 1) / rpb, g.BH);
  ProfScope ps("fusion_grads", st);
  if (bf16)
    fusion_grads_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)dO, (const __nv_bfloat16*)Os,
                                                             (const __nv_bfloat16*)Olr, logd, dlr, lam, gs, glr,
                                                             dlam, dgs, dglr, perm, perm_stride, g);
  else
    fusion_grads_kernel<float><<<grid, 256, 0, st>>>((const float*)dO, (const float*)Os, (const float*)Olr, logd, dlr,
                                                     lam, gs, glr, dlam, dgs, dglr, perm, perm_stride, g);
  return cudaGetLastError();
}

cudaError_t launch_row_scalars(const BwdArgs& a, bool bf16, const Geom& g, cudaStream_t st) {
  const int rpb = 256 / (g.d / 8);
  dim3 grid((g.N + rpb - 1) / rpb, g.BH);
  ProfScope ps("row_scalars", st);
  if (bf16) row_scalars_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a, g);
  else row_scalars_kernel<float><<<grid, 256, 0, st>>>(a, g);
  return cudaGetLastError();
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
    if (a.rs.packed) {                // (log2 d_s, cs, Delta) in one row (also the gathered rows of sortLSH)
      const float4 p = ok ? a.rs.packed[head + row] : make_float4(INFINITY, 0.f, 0.f, 0.f);
      lg2[h] = p.x;
      cs[h] = p.y;
      Dl[h] = p.z;
    } else {
      lg2[h] = ok ? a.logd[head + row] * kLog2e : INFINITY;
      cs[h] = ok ? a.rs.cs[head + row] : 0.f;
      Dl[h] = ok ? a.rs.Delta[head + row] : 0.f;
    }
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
      if (a.rs.packed) {
        const float4 p = ok ? a.rs.packed[head + row] : make_float4(INFINITY, 0.f, 0.f, 0.f);
        sc[r] = p.x;
        sc[T + r] = p.y;
        sc[2 * T + r] = p.z;
      } else {
        sc[r] = ok ? a.logd[head + row] * kLog2e : INFINITY;
        sc[T + r] = ok ? a.rs.cs[head + row] : 0.f;
        sc[2 * T + r] = ok ? a.rs.Delta[head + row] : 0.f;
      }
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
static cudaError_t bwd_t(const BwdArgs& a0, const Geom& g, int parts, cudaStream_t st) {
  BwdArgs a = a0;
  cudaError_t e;
  // the sparse kernels add the fp32 accumulators when they are given (null: nothing to add)
  if (g.r > 0 && (parts & 1)) {
    e = launch_race_bwd_bf16(a, g, st);
    if (e != cudaSuccess) return e;
  }
  const size_t lds = (size_t)(D + 8) * 2;
  if (parts & 2) {
    e = launch2("sparse_dq", sparse_dq_bf16_kernel<D, T>, (size_t)6 * T * lds, T, a, g, st);
    if (e != cudaSuccess) return e;
  }
  if (parts & 4)
    return launch2("sparse_dkdv", sparse_dkdv_bf16_kernel<D, T>, (size_t)6 * T * lds + (size_t)6 * T * 4, T, a, g, st);
  return cudaSuccess;
}

// parts: bit 0 RACE backward, bit 1 sparse dQ, bit 2 sparse dK/dV (mma.sync kernels).
cudaError_t launch_bwd_bf16(const BwdArgs& a, const Geom& g, int parts, cudaStream_t st) {
  if (g.d == 64 && g.T == 64) return bwd_t<64, 64>(a, g, parts, st);
  if (g.d == 64 && g.T == 128) return bwd_t<64, 128>(a, g, parts, st);
  if (g.d == 128 && g.T == 64) return bwd_t<128, 64>(a, g, parts, st);
  if (g.d == 128 && g.T == 128) return bwd_t<128, 128>(a, g, parts, st);
  return cudaErrorInvalidValue;
}

}  // namespace elsaa
