// RACE low-rank branch, the pieces outside the tensor-core kernels (ELSAA paper §3.1;
// sketch size S_R = L 2^gamma, §6): W split into bf16 hi + lo rows for the tensor-core
// products, the scan over segment totals, and the float32 path (SIMT) of the features and
// the chunked prefix summaries.
//
// Features.  For a row x: u = x / max(|x|, 1e-12); table l projects
// h_l = W_l^T u (gamma = 4 values); the probability of corner c in {-1,1}^4 is
// the softmax of <c, h_l>/tau over the 16 corners, which factorises into
// prod_b sigmoid(2 c_b h_lb / tau); Phi(x) = [p_l(c|x) / sqrt(L)] (r = 16 L).
//
// Summaries.  Chunk c of length C contributes S_c = Phi(K_c)^T [V_c | 1]
// (r x (d+1): the value statistics and the key mass of every bucket).  A causal
// query of chunk c reads the exclusive prefix P_c = sum_{c' < c} S_c' plus its
// own chunk, masked; a non-causal query reads the total.  P_c is split into a
// per-segment part (a CTA walks `seg` chunks in order, carrying the sum in
// registers) and the exclusive prefix of segment totals (a short scan).
// State layout: float32 [r][dp], dp = d + 8, column d = key mass, d+1..d+7 = 0.
#include "common.cuh"
#include "kernels.h"

namespace elsaa {

// ---------------------------------------------------------------------------
// Features, bf16 inputs.  grid (ceil(N/64), BH, 2: Q then K), block 128.
// H = X (W_hi + W_lo) on the tensor cores (X is exact in bf16, W split into two
// bf16 halves), then the corner probabilities per (row, table) in fp32.
// Writes Phi (bf16 [BH,N,r]), the normalised projections h (fp32 [BH,N,4L]) and
// the row norms n (fp32 [BH,N]).
// ---------------------------------------------------------------------------
// W[l][k][b] (fp32) -> rows n = 4 l + b of bf16 hi and lo [NW][D] (zero rows beyond 4 L).
__global__ void race_w_split_kernel(const float* __restrict__ W, __nv_bfloat16* __restrict__ out, int D, int NH,
                                    int NW) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < NW * D; i += gridDim.x * blockDim.x) {
    const int n = i / D, k = i % D;
    const float w = n < NH ? W[((size_t)(n >> 2) * D + k) * kHashBits + (n & 3)] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    out[i] = hi;
    out[(size_t)NW * D + i] = __float2bfloat16_rn(w - __bfloat162float(hi));
  }
}

// Forward: exclusive prefix over segment totals, in place.  Afterwards slot s
// holds sum_{s' < s} total_{s'} and slot n_seg the grand total.
// Backward: exclusive suffix, in place.  Afterwards slot s + 1 holds
// sum_{s' > s} total_{s'} and slot 0 the grand total.
// (total_s is written to slot s + 1 by the state kernel.)  States hold `rows` feature rows of
// dp columns.  grid (ceil(rows*dp/256), BH).
__global__ void race_scan_kernel(float* __restrict__ A, Geom g, int rows, int reverse) {
  const int e = blockIdx.x * 256 + threadIdx.x;
  const int n = rows * g.dp;
  if (e >= n) return;
  float* a = A + (size_t)blockIdx.y * (g.n_seg + 1) * n + e;
  constexpr int kB = 8;          // loads in flight per thread
  float acc = 0.f;
  if (!reverse) {
    a[0] = 0.f;
    for (int s0 = 1; s0 <= g.n_seg; s0 += kB) {
      float v[kB];
#pragma unroll
      for (int q = 0; q < kB; ++q) v[q] = s0 + q <= g.n_seg ? a[(size_t)(s0 + q) * n] : 0.f;
#pragma unroll
      for (int q = 0; q < kB; ++q)
        if (s0 + q <= g.n_seg) {
          acc += v[q];
          a[(size_t)(s0 + q) * n] = acc;
        }
    }
  } else {
    for (int s0 = g.n_seg - 1; s0 >= 0; s0 -= kB) {
      float v[kB];
#pragma unroll
      for (int q = 0; q < kB; ++q) v[q] = s0 - q >= 0 ? a[(size_t)(s0 - q + 1) * n] : 0.f;
#pragma unroll
      for (int q = 0; q < kB; ++q)
        if (s0 - q >= 0) {
          a[(size_t)(s0 - q + 1) * n] = acc;
          acc += v[q];
        }
    }
    a[0] = acc;
  }
}

// ---------------------------------------------------------------------------
// float32 path (small problems, block size 1 allowed): SIMT versions.
// ---------------------------------------------------------------------------

// grid (ceil(N/8), BH, 2), block 256: one warp per row.
__global__ void __launch_bounds__(256) race_features_f32_kernel(const float* __restrict__ Q,
                                                                const float* __restrict__ K,
                                                                const float* __restrict__ W,
                                                                float* __restrict__ phiQ, float* __restrict__ phiK,
                                                                float* __restrict__ hQ, float* __restrict__ hK,
                                                                float* __restrict__ nQ, float* __restrict__ nK,
                                                                Geom g) {
  __shared__ float sx[8][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= g.N) return;
  const int side = blockIdx.z;
  const float* x = (side == 0 ? Q : K) + ((size_t)blockIdx.y * g.N + row) * g.d;
  float* phi = (side == 0 ? phiQ : phiK) + ((size_t)blockIdx.y * g.N + row) * g.r;
  const int NH = g.L * kHashBits;
  float* hout = (side == 0 ? hQ : hK) + ((size_t)blockIdx.y * g.N + row) * NH;
  float* nout = (side == 0 ? nQ : nK) + (size_t)blockIdx.y * g.N + row;
  float ss = 0.f;
  for (int c = lane; c < g.d; c += 32) {
    const float v = x[c];
    sx[warp][c] = v;
    ss += v * v;
  }
  ss = warp_sum(ss);
  const float n = fmaxf(sqrtf(ss), kNormFloor);
  __syncwarp();
  const float inv_sqrt_L = rsqrtf((float)g.L);
  for (int l = lane; l < g.L; l += 32) {
    float sp[kHashBits], sm[kHashBits];
    for (int b = 0; b < kHashBits; ++b) {
      float acc = 0.f;
      for (int c = 0; c < g.d; ++c) acc += sx[warp][c] * W[((size_t)l * g.d + c) * kHashBits + b];
      const float h = acc / n;
      hout[l * kHashBits + b] = h;
      const float y = 2.f * h / g.tau;
      sp[b] = 1.f / (1.f + expf(-y));
      sm[b] = 1.f / (1.f + expf(y));
    }
    for (int c = 0; c < kCorners; ++c) {
      float p = inv_sqrt_L;
      for (int b = 0; b < kHashBits; ++b) p *= ((c >> b) & 1) ? sp[b] : sm[b];
      phi[l * kCorners + c] = p;
    }
  }
  if (lane == 0) *nout = n;
}

// grid (n_seg, BH, ceil(r*dp/256)), block 256: each thread owns one state entry.
// Same two modes and slot conventions as the bf16 state kernel.
template <bool BWD>
__global__ void __launch_bounds__(256) race_state_f32_kernel(const float* __restrict__ phi,
                                                             const float* __restrict__ Y,
                                                             const float* __restrict__ rscale,
                                                             const float* __restrict__ rextra,
                                                             float* __restrict__ Atot, float* __restrict__ Bpart,
                                                             Geom g) {
  const int e = blockIdx.z * 256 + threadIdx.x;
  const int n = g.r * g.dp;
  if (e >= n) return;
  const int f = e / g.dp, col = e % g.dp;
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int c_begin = seg * g.seg, c_end = min(g.n_c, c_begin + g.seg);
  const float* pk = phi + (size_t)bh * g.N * g.r;
  const float* vv = Y + (size_t)bh * g.N * g.d;
  const size_t rowbase = (size_t)bh * g.N;
  float acc = 0.f;
  for (int step = 0; step < c_end - c_begin; ++step) {
    const int c = BWD ? c_end - 1 - step : c_begin + step;
    if (g.causal) Bpart[((size_t)bh * g.n_c + c) * n + e] = acc;
    const int j1 = min(g.N, (c + 1) * g.C);
    for (int j = c * g.C; j < j1; ++j) {
      float val;
      if (col < g.d) val = vv[(size_t)j * g.d + col] * (BWD ? rscale[rowbase + j] : 1.f);
      else val = col == g.d ? (BWD ? rextra[rowbase + j] : 1.f) : 0.f;
      acc += pk[(size_t)j * g.r + f] * val;
    }
  }
  Atot[((size_t)bh * (g.n_seg + 1) + seg + 1) * n + e] = acc;
}

cudaError_t launch_race_w_split(const float* W, void* out, const Geom& g, cudaStream_t st) {
  const int NW = (g.L * kHashBits + 31) & ~31;
  race_w_split_kernel<<<(NW * g.d + 255) / 256, 256, 0, st>>>(W, (__nv_bfloat16*)out, g.d, g.L * kHashBits, NW);
  return cudaGetLastError();
}

cudaError_t launch_race_features_f32(const float* Q, const float* K, const float* W, float* phiQ, float* phiK,
                                     float* hQ, float* hK, float* nQ, float* nK, const Geom& g, cudaStream_t st) {
  if (g.r == 0) return cudaSuccess;
  ProfScope ps("race_features_f32", st);
  race_features_f32_kernel<<<dim3((g.N + 7) / 8, g.BH, 2), 256, 0, st>>>(Q, K, W, phiQ, phiK, hQ, hK, nQ, nK, g);
  return cudaGetLastError();
}

cudaError_t launch_race_scan(float* Atot, int rows, bool bwd, const Geom& g, cudaStream_t st) {
  ProfScope ps(bwd ? "race_scan_bwd" : "race_scan_fwd", st);
  race_scan_kernel<<<dim3((rows * g.dp + 255) / 256, g.BH), 256, 0, st>>>(Atot, g, rows, bwd ? 1 : 0);
  return cudaGetLastError();
}

template <bool BWD>
static cudaError_t run_state_f32(const float* phi, const float* Y, const float* rsc, const float* rex, float* Atot,
                                 float* Bpart, const Geom& g, cudaStream_t st) {
  const int n = g.r * g.dp;
  ProfScope ps(BWD ? "race_state_bwd_f32" : "race_state_fwd_f32", st);
  race_state_f32_kernel<BWD><<<dim3(g.n_seg, g.BH, (n + 255) / 256), 256, 0, st>>>(phi, Y, rsc, rex, Atot, Bpart, g);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_race_scan(Atot, g.r, BWD, g, st);
}

cudaError_t launch_race_state_fwd_f32(const float* phiK, const float* V, float* Ast, float* Bst, const Geom& g,
                                      cudaStream_t st) {
  if (g.r == 0) return cudaSuccess;
  return run_state_f32<false>(phiK, V, nullptr, nullptr, Ast, Bst, g, st);
}

cudaError_t launch_race_state_bwd_f32(const BwdArgs& a, const Geom& g, cudaStream_t st) {
  if (g.r == 0) return cudaSuccess;
  return run_state_f32<true>((const float*)a.phiQ, (const float*)a.dO, a.rs.cl, a.rs.delta, a.RA, a.RB, g, st);
}

}  // namespace elsaa
