// float32 path: SIMT kernels for small problems (block size 1 allowed).  Same
// operator as the bf16 tensor-core path (sparse branch §3.2, RACE §3.1, fusion
// Eq. 5 / Eq. 4 of the ELSAA paper), one warp per row, exact fp32 arithmetic
// with an online softmax.  RACE chunks here have their own length g.C.
#include "common.cuh"
#include "kernels.h"

namespace elsaa {

constexpr int kMaxD = 128;
constexpr int kMaxR = 256;

// Forward, one warp per query row.  grid (ceil(N/8), BH), block 256.
__global__ void __launch_bounds__(256) attn_fwd_f32_kernel(FwdArgs a, Geom g) {
  __shared__ float sphi[8][kMaxR];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qi = blockIdx.x * 8 + warp;
  const int bh = blockIdx.y;
  if (qi >= g.N) return;
  const size_t head = (size_t)bh * g.N;
  const float* Q = (const float*)a.Q + head * g.d;
  const float* K = (const float*)a.K + head * g.d;
  const float* V = (const float*)a.V + head * g.d;
  constexpr int NJ = kMaxD / 32;
  float q[NJ], o[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int c = lane + 32 * j;
    q[j] = c < g.d ? Q[(size_t)qi * g.d + c] : 0.f;
    o[j] = 0.f;
  }
  const int t = qi / g.T;
  const int* my_idx = a.idx + ((size_t)bh * g.n_t + t) * g.k;
  float m = -INFINITY, l = 0.f;
  for (int s = 0; s < g.k; ++s) {
    const int b = my_idx[s];
    if (b < 0) break;
    const int j1 = min(g.N, (b + 1) * g.T);
    for (int j = b * g.T; j < j1; ++j) {
      if (g.causal && j > qi) break;
      float part = 0.f;
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) {
        const int c = lane + 32 * jj;
        if (c < g.d) part += q[jj] * K[(size_t)j * g.d + c];
      }
      const float z = warp_sum(part) * g.scale;
      const float mn = fmaxf(m, z);
      const float al = expf(m - mn);
      const float p = expf(z - mn);
      l = l * al + p;
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) {
        const int c = lane + 32 * jj;
        o[jj] = o[jj] * al + (c < g.d ? p * V[(size_t)j * g.d + c] : 0.f);
      }
      m = mn;
    }
  }
  const float inv_l = l > 0.f ? 1.f / l : 0.f;
  const float logd = l > 0.f ? m + logf(l) : -INFINITY;

  // RACE read-out: [N_lr; d_lr] = Phi_q P_chunk + sum_{j in chunk, j <= i} kappa_ij [v_j; 1]
  constexpr int NP = (kMaxD + 8 + 31) / 32;
  float acc[NP];
#pragma unroll
  for (int j = 0; j < NP; ++j) acc[j] = 0.f;
  if (g.r > 0) {
    const float* fq = (const float*)a.phiQ + (head + qi) * g.r;
    for (int f = lane; f < g.r; f += 32) sphi[warp][f] = fq[f];
    __syncwarp();
    const int c = qi / g.C;
    const int sidx = c / g.seg;
    const float* pa = a.Ast + ((size_t)bh * (g.n_seg + 1) + (g.causal ? sidx : g.n_seg)) * g.r * g.dp;
    const float* pb = g.causal ? a.Bst + ((size_t)bh * g.n_c + c) * g.r * g.dp : nullptr;
#pragma unroll
    for (int jj = 0; jj < NP; ++jj) {
      const int col = lane + 32 * jj;
      if (col > g.d) continue;
      float s = 0.f;
      for (int f = 0; f < g.r; ++f) {
        float pv = pa[(size_t)f * g.dp + col];
        if (pb) pv += pb[(size_t)f * g.dp + col];
        s += sphi[warp][f] * pv;
      }
      acc[jj] = s;
    }
    if (g.causal) {
      const float* fk = (const float*)a.phiK + head * g.r;
      for (int j = c * g.C; j <= qi; ++j) {
        float part = 0.f;
        for (int f = lane; f < g.r; f += 32) part += sphi[warp][f] * fk[(size_t)j * g.r + f];
        const float kap = warp_sum(part);
#pragma unroll
        for (int jj = 0; jj < NP; ++jj) {
          const int col = lane + 32 * jj;
          if (col < g.d) acc[jj] += kap * V[(size_t)j * g.d + col];
          else if (col == g.d) acc[jj] += kap;
        }
      }
    }
  }
  const float dl = __shfl_sync(0xffffffffu, acc[g.d / 32], g.d % 32);
  const float lam = a.lam ? a.lam[head + qi] : g.lam;
  const float cc = lam * dl + g.eps;
  const float mf = g.fixed_m ? 1.f : logd == -INFINITY ? 0.f : 1.f / (1.f + cc * expf(-logd));
  const float gs = a.gs ? a.gs[head + qi] : 1.f;
  const float gl = a.glr ? a.glr[head + qi] : g.fixed_m ? 1.f : 1.f - mf;
  const float cs = gs * mf, cl = dl > 0.f ? gl / dl : 0.f;
  float* O = (float*)a.O + (head + qi) * g.d;
  float* Os = (float*)a.Os + (head + qi) * g.d;
  float* Olr = (float*)a.Olr + (head + qi) * g.d;
#pragma unroll
  for (int jj = 0; jj < NJ; ++jj) {
    const int c = lane + 32 * jj;
    if (c < g.d) {
      const float os = o[jj] * inv_l;
      O[c] = cs * os + cl * acc[jj];
      Os[c] = os;
      Olr[c] = dl > 0.f ? acc[jj] / dl : 0.f;
    }
  }
  if (lane == 0) {
    a.logd[head + qi] = logd;
    a.dlr[head + qi] = dl;
    a.m[head + qi] = mf;
  }
}

cudaError_t launch_attn_fwd_f32(const FwdArgs& a, const Geom& g, cudaStream_t st) {
  ProfScope ps("attn_fwd_f32", st);
  attn_fwd_f32_kernel<<<dim3((g.N + 7) / 8, g.BH), 256, 0, st>>>(a, g);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Backward, float32 path.  Row scalars, the suffix statistics and the selection
// inverse are computed by the shared kernels first.
// ---------------------------------------------------------------------------

// Chain dPhi (lanes hold features f = lane + 32 m) through the corner softmax of
// each table into dh (per warp, smem), then dx = (du - u <u,du>) / n.
__device__ void f32_feature_chain(const float (&dphi)[kMaxR / 32], const float* __restrict__ hrow,
                                  const float* __restrict__ W, const float* __restrict__ x, float nrm,
                                  float* sdh, float (&dx)[kMaxD / 32], const Geom& g) {
  const int lane = threadIdx.x & 31;
  const float inv_sqrt_L = rsqrtf((float)g.L);
  const int cidx = lane & 15;
#pragma unroll
  for (int mm = 0; mm < kMaxR / 32; ++mm) {
    const int f0 = 32 * mm;
    if (f0 >= g.r) break;
    const int f = f0 + lane;
    const int l = f >> 4;
    const bool ok = f < g.r;
    float p = 0.f, dp = 0.f;
    if (ok) {
      p = 1.f;
      for (int b = 0; b < kHashBits; ++b) {
        const float y = 2.f * hrow[l * kHashBits + b] / g.tau;
        p *= ((cidx >> b) & 1) ? 1.f / (1.f + expf(-y)) : 1.f / (1.f + expf(y));
      }
      dp = dphi[mm] * inv_sqrt_L;
    }
    float s = dp * p;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float da = p * (dp - s);
#pragma unroll
    for (int b = 0; b < kHashBits; ++b) {
      float v = ((cidx >> b) & 1) ? da : -da;
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (ok && cidx == 0) sdh[l * kHashBits + b] = v / g.tau;
    }
  }
  __syncwarp();
  const int NH = g.L * kHashBits;
  float xd = 0.f;
#pragma unroll
  for (int jj = 0; jj < kMaxD / 32; ++jj) {
    const int c = lane + 32 * jj;
    float du = 0.f;
    if (c < g.d) {
      for (int n = 0; n < NH; ++n) du += sdh[n] * W[((size_t)(n >> 2) * g.d + c) * kHashBits + (n & 3)];
      xd += x[c] * du;
    }
    dx[jj] = du;
  }
  xd = warp_sum(xd);
  const float proj = nrm <= kNormFloor ? 0.f : xd / (nrm * nrm);
#pragma unroll
  for (int jj = 0; jj < kMaxD / 32; ++jj) {
    const int c = lane + 32 * jj;
    dx[jj] = c < g.d ? (dx[jj] - x[c] * proj) / nrm : 0.f;
  }
  __syncwarp();
}

// dQ, one warp per query row.  grid (ceil(N/8), BH), block 256.
__global__ void __launch_bounds__(256) bwd_dq_f32_kernel(BwdArgs a, Geom g) {
  __shared__ float se[8][kMaxD + 8];
  __shared__ float sdh[8][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qi = blockIdx.x * 8 + warp;
  const int bh = blockIdx.y;
  if (qi >= g.N) return;
  const size_t head = (size_t)bh * g.N;
  const float* Q = (const float*)a.Q + head * g.d;
  const float* K = (const float*)a.K + head * g.d;
  const float* V = (const float*)a.V + head * g.d;
  const float* dO = (const float*)a.dO + head * g.d;
  constexpr int NJ = kMaxD / 32;
  float q[NJ], go[NJ], dq[NJ];
#pragma unroll
  for (int jj = 0; jj < NJ; ++jj) {
    const int c = lane + 32 * jj;
    q[jj] = c < g.d ? Q[(size_t)qi * g.d + c] : 0.f;
    go[jj] = c < g.d ? dO[(size_t)qi * g.d + c] : 0.f;
    dq[jj] = 0.f;
  }
  const size_t ri = head + qi;
  const float logd = a.logd[ri], cs = a.rs.cs[ri], Dl = a.rs.Delta[ri], cl = a.rs.cl[ri], del = a.rs.delta[ri];
  const int t = qi / g.T;
  const int* my_idx = a.idx + ((size_t)bh * g.n_t + t) * g.k;
  for (int s = 0; s < g.k; ++s) {
    const int b = my_idx[s];
    if (b < 0) break;
    const int j1 = min(g.N, (b + 1) * g.T);
    for (int j = b * g.T; j < j1; ++j) {
      if (g.causal && j > qi) break;
      float zp = 0.f, vp = 0.f;
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) {
        const int c = lane + 32 * jj;
        if (c < g.d) {
          zp += q[jj] * K[(size_t)j * g.d + c];
          vp += go[jj] * V[(size_t)j * g.d + c];
        }
      }
      const float z = warp_sum(zp) * g.scale;
      const float dpv = warp_sum(vp);
      const float p = expf(z - logd);
      const float ds = p * (cs * dpv - Dl);
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) {
        const int c = lane + 32 * jj;
        if (c < g.d) dq[jj] += g.scale * ds * K[(size_t)j * g.d + c];
      }
    }
  }
  if (g.r > 0) {
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj) {
      const int c = lane + 32 * jj;
      if (c < g.d) se[warp][c] = cl * go[jj];
    }
    if (lane == 0) se[warp][g.d] = del;
    __syncwarp();
    const int c = qi / g.C;
    const float* pa = a.Ast + ((size_t)bh * (g.n_seg + 1) + (g.causal ? c / g.seg : g.n_seg)) * g.r * g.dp;
    const float* pb = g.causal ? a.Bst + ((size_t)bh * g.n_c + c) * g.r * g.dp : nullptr;
    float dphi[kMaxR / 32];
#pragma unroll
    for (int mm = 0; mm < kMaxR / 32; ++mm) {
      const int f = lane + 32 * mm;
      float acc = 0.f;
      if (f < g.r) {
        for (int col = 0; col <= g.d; ++col) {
          float pv = pa[(size_t)f * g.dp + col];
          if (pb) pv += pb[(size_t)f * g.dp + col];
          acc += pv * se[warp][col];
        }
      }
      dphi[mm] = acc;
    }
    if (g.causal) {
      const float* fk = (const float*)a.phiK + head * g.r;
      for (int j = c * g.C; j <= qi; ++j) {
        float vp = 0.f;
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) {
          const int cc = lane + 32 * jj;
          if (cc < g.d) vp += go[jj] * V[(size_t)j * g.d + cc];
        }
        const float dk = cl * warp_sum(vp) + del;
#pragma unroll
        for (int mm = 0; mm < kMaxR / 32; ++mm) {
          const int f = lane + 32 * mm;
          if (f < g.r) dphi[mm] += dk * fk[(size_t)j * g.r + f];
        }
      }
    }
    float dx[NJ];
    f32_feature_chain(dphi, a.hQ + ri * (g.L * kHashBits), a.W, Q + (size_t)qi * g.d, a.nQ[ri], sdh[warp], dx, g);
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj) dq[jj] += dx[jj];
  }
  float* out = (float*)a.dQ + ri * g.d;
#pragma unroll
  for (int jj = 0; jj < NJ; ++jj) {
    const int c = lane + 32 * jj;
    if (c < g.d) out[c] = dq[jj];
  }
}

// dK, dV, one warp per key row.  grid (ceil(N/8), BH), block 256.
__global__ void __launch_bounds__(256) bwd_dkdv_f32_kernel(BwdArgs a, Geom g) {
  __shared__ float sv[8][kMaxD + 8];
  __shared__ float sdh[8][64];
  __shared__ float sfk[8][kMaxR];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kj = blockIdx.x * 8 + warp;
  const int bh = blockIdx.y;
  if (kj >= g.N) return;
  const size_t head = (size_t)bh * g.N;
  const float* Q = (const float*)a.Q + head * g.d;
  const float* K = (const float*)a.K + head * g.d;
  const float* V = (const float*)a.V + head * g.d;
  const float* dO = (const float*)a.dO + head * g.d;
  constexpr int NJ = kMaxD / 32;
  float kv[NJ], vv[NJ], dk[NJ], dv[NJ];
#pragma unroll
  for (int jj = 0; jj < NJ; ++jj) {
    const int c = lane + 32 * jj;
    kv[jj] = c < g.d ? K[(size_t)kj * g.d + c] : 0.f;
    vv[jj] = c < g.d ? V[(size_t)kj * g.d + c] : 0.f;
    dk[jj] = dv[jj] = 0.f;
  }
  const int b = kj / g.T;
  if (g.k > 0) {
    const int* of = a.offs + (size_t)bh * (g.n_t + 1);
    const int* list = a.tiles + (size_t)bh * g.n_t * g.k;
    for (int e = of[b]; e < of[b + 1]; ++e) {
      const int t = list[e];
      const int i1 = min(g.N, (t + 1) * g.T);
      for (int i = t * g.T; i < i1; ++i) {
        if (g.causal && i < kj) continue;
        float zp = 0.f, vp = 0.f;
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) {
          const int c = lane + 32 * jj;
          if (c < g.d) {
            zp += kv[jj] * Q[(size_t)i * g.d + c];
            vp += vv[jj] * dO[(size_t)i * g.d + c];
          }
        }
        const float z = warp_sum(zp) * g.scale;
        const float dpv = warp_sum(vp);
        const size_t ri = head + i;
        const float p = expf(z - a.logd[ri]);
        const float cs = a.rs.cs[ri];
        const float ds = p * (cs * dpv - a.rs.Delta[ri]);
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) {
          const int c = lane + 32 * jj;
          if (c < g.d) {
            dk[jj] += g.scale * ds * Q[(size_t)i * g.d + c];
            dv[jj] += p * cs * dO[(size_t)i * g.d + c];
          }
        }
      }
    }
  }
  const size_t rj = head + kj;
  if (g.r > 0) {
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj) {
      const int c = lane + 32 * jj;
      if (c < g.d) sv[warp][c] = vv[jj];
    }
    if (lane == 0) sv[warp][g.d] = 1.f;
    const float* fkr = (const float*)a.phiK + rj * g.r;
    for (int f = lane; f < g.r; f += 32) sfk[warp][f] = fkr[f];
    __syncwarp();
    const int c = kj / g.C;
    const float* ra = a.RA + ((size_t)bh * (g.n_seg + 1) + (g.causal ? c / g.seg + 1 : 0)) * g.r * g.dp;
    const float* rb = g.causal ? a.RB + ((size_t)bh * g.n_c + c) * g.r * g.dp : nullptr;
    float dphi[kMaxR / 32];
#pragma unroll
    for (int mm = 0; mm < kMaxR / 32; ++mm) {
      const int f = lane + 32 * mm;
      float acc = 0.f;
      if (f < g.r) {
        for (int col = 0; col <= g.d; ++col) {
          float rv = ra[(size_t)f * g.dp + col];
          if (rb) rv += rb[(size_t)f * g.dp + col];
          acc += rv * sv[warp][col];
        }
      }
      dphi[mm] = acc;
    }
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj) {
      const int col = lane + 32 * jj;
      if (col < g.d) {
        float acc = 0.f;
        for (int f = 0; f < g.r; ++f) {
          float rv = ra[(size_t)f * g.dp + col];
          if (rb) rv += rb[(size_t)f * g.dp + col];
          acc += sfk[warp][f] * rv;
        }
        dv[jj] += acc;
      }
    }
    if (g.causal) {
      const float* fq = (const float*)a.phiQ + head * g.r;
      const int i1 = min(g.N, (c + 1) * g.C);
      for (int i = kj; i < i1; ++i) {
        const size_t ri = head + i;
        float vp = 0.f, kp = 0.f;
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) {
          const int cc = lane + 32 * jj;
          if (cc < g.d) vp += vv[jj] * dO[(size_t)i * g.d + cc];
        }
        for (int f = lane; f < g.r; f += 32) kp += sfk[warp][f] * fq[(size_t)i * g.r + f];
        const float cl = a.rs.cl[ri];
        const float dkap = cl * warp_sum(vp) + a.rs.delta[ri];
        const float kap = warp_sum(kp);
#pragma unroll
        for (int mm = 0; mm < kMaxR / 32; ++mm) {
          const int f = lane + 32 * mm;
          if (f < g.r) dphi[mm] += dkap * fq[(size_t)i * g.r + f];
        }
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) {
          const int cc = lane + 32 * jj;
          if (cc < g.d) dv[jj] += kap * cl * dO[(size_t)i * g.d + cc];
        }
      }
    }
    float dx[NJ];
    f32_feature_chain(dphi, a.hK + rj * (g.L * kHashBits), a.W, K + (size_t)kj * g.d, a.nK[rj], sdh[warp], dx, g);
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj) dk[jj] += dx[jj];
  }
  float* ok = (float*)a.dK + rj * g.d;
  float* ov = (float*)a.dV + rj * g.d;
#pragma unroll
  for (int jj = 0; jj < NJ; ++jj) {
    const int c = lane + 32 * jj;
    if (c < g.d) {
      ok[c] = dk[jj];
      ov[c] = dv[jj];
    }
  }
}

cudaError_t launch_bwd_f32(const BwdArgs& a, const Geom& g, cudaStream_t st) {
  const dim3 grid((g.N + 7) / 8, g.BH);
  {
    ProfScope ps("bwd_dq_f32", st);
    bwd_dq_f32_kernel<<<grid, 256, 0, st>>>(a, g);
  }
  ProfScope ps("bwd_dkdv_f32", st);
  bwd_dkdv_f32_kernel<<<grid, 256, 0, st>>>(a, g);
  return cudaGetLastError();
}

}  // namespace elsaa
