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
// d/8 threads per row reduce the row's <dO, O_s> and <dO, O_lr> (8 elements each; the
// butterfly leaves both sums in every one of them); each of those threads then runs the
// scalar algebra in fp32 (no block barrier, so the memory traffic of other rows keeps
// flowing), the row's first thread writes the per-row outputs and all of them write
// their 8 elements of cl dO.
template <typename E>
__global__ void __launch_bounds__(256) row_scalars_kernel(BwdArgs a, Geom g) {
  const int tpr = g.d / 8;
  const int rpb = 256 / tpr;
  const int sub = threadIdx.x % tpr;
  const int row = blockIdx.x * rpb + threadIdx.x / tpr;
  const size_t i = (size_t)blockIdx.y * g.N + min(row, g.N - 1);
  float dO[8], os[8], ol[8];
  load8<E>((const E*)a.dO + i * g.d + sub * 8, dO);
  load8<float>((const float*)a.Os + i * g.d + sub * 8, os);     // O_s is saved in fp32
  load8<E>((const E*)a.Olr + i * g.d + sub * 8, ol);
  const float logd = a.logd[i], dl = a.dlr[i];
  const float lam = a.lam ? a.lam[i] : g.lam;
  const float gs = a.gs ? a.gs[i] : 1.f;
  const float glr = a.glr ? a.glr[i] : 0.f;
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
  if (row >= g.N) return;
  const float ds = expf(logd);
  const float c = lam * dl + g.eps;
  const float D = ds + c;
  // fixed_m: the ablation without denominator-aware fusion (m = 1, default g_lr = 1, no dm)
  const float m = g.fixed_m ? 1.f : D > 0.f ? ds / D : 0.f;
  const float one_m = g.fixed_m ? 0.f : D > 0.f ? c / D : 1.f;
  const float gl = a.glr ? glr : g.fixed_m ? 1.f : one_m;
  const float dm = g.fixed_m ? 0.f : gs * A - (a.glr ? 0.f : Bv);
  const float cs = gs * m;
  const float cl = dl > 0.f ? gl / dl : 0.f;
  const float ddlr = D > 0.f ? -dm * lam * ds / (D * D) : 0.f;
  const float Dl = cs * A - dm * m * one_m;
  if (sub == 0) {
    a.rs.cs[i] = cs;
    a.rs.Delta[i] = Dl;
    if (a.rs.packed) a.rs.packed[i] = make_float4(logd * 1.44269504f, cs, Dl, 0.f);
    a.rs.cl[i] = cl;
    a.rs.delta[i] = ddlr - cl * Bv;
  }
  // the rows cl dO (bf16) feed the RACE suffix statistics
  if (a.dOcl) {
    uint4 w;
    w.x = pack_bf16(cl * dO[0], cl * dO[1]);
    w.y = pack_bf16(cl * dO[2], cl * dO[3]);
    w.z = pack_bf16(cl * dO[4], cl * dO[5]);
    w.w = pack_bf16(cl * dO[6], cl * dO[7]);
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dOcl) + i * g.d + sub * 8) = w;
  }
}

// Per-row gradients of sum(dO * O) with respect to lambda, g_s and g_lr (Eq. 5 / Eq. 4):
// dlambda = -dm d_s d_lr / D^2 (0 when m is held at 1), dg_s = m <dO, O_s>, dg_lr = <dO, O_lr>,
// dm = g_s <dO, O_s> - [g_lr defaulted] <dO, O_lr>.  Same row layout as the row scalars.
template <typename E>
__global__ void __launch_bounds__(256) fusion_grads_kernel(const E* __restrict__ dO_, const float* __restrict__ Os_,
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
  load8<float>(Os_ + i * g.d + sub * 8, os);
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
    fusion_grads_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)dO, (const float*)Os,
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

}  // namespace elsaa
