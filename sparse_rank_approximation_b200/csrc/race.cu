// RACE low-rank branch: soft hypercube-bucket features and the chunked prefix
// summaries the read-out uses (ELSAA paper §3.1; sketch size S_R = L 2^gamma, §6).
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

template <int D>
__global__ void __launch_bounds__(128) race_features_bf16_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ Wsplit,
    __nv_bfloat16* __restrict__ phiQ, __nv_bfloat16* __restrict__ phiK, float* __restrict__ hQ,
    float* __restrict__ hK, float* __restrict__ nQ, float* __restrict__ nK, Geom g) {
  constexpr int LDX = D + 8;
  const int NH = g.L * kHashBits;              // projection columns
  const int NW = (NH + 15) & ~15;              // padded to whole n-block pairs
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* sX = reinterpret_cast<__nv_bfloat16*>(smem);           // [64][LDX]
  __nv_bfloat16* sWh = sX + 64 * LDX;                                     // [NW][LDX]
  __nv_bfloat16* sWl = sWh + NW * LDX;                                    // [NW][LDX]
  float* sH = reinterpret_cast<float*>(sWl + NW * LDX);                  // [64][NW+1]
  float* sN = sH + 64 * (NW + 1);                                         // [64]

  const int side = blockIdx.z;
  const __nv_bfloat16* X = (side == 0 ? Q : K) + (size_t)blockIdx.y * g.N * D;
  __nv_bfloat16* phi = (side == 0 ? phiQ : phiK) + (size_t)blockIdx.y * g.N * g.r;
  // h and the norms are kept for the backward when the caller passes buffers for them
  float* hout = (side == 0 ? hQ : hK);
  float* nout = (side == 0 ? nQ : nK);
  if (hout) hout += (size_t)blockIdx.y * g.N * NH;
  if (nout) nout += (size_t)blockIdx.y * g.N;
  const int row_base = blockIdx.x * 64;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int i = tid; i < 64 * (D / 8); i += 128) {
    const int r = i / (D / 8), c = (i % (D / 8)) * 8;
    const int row = row_base + r;
    cp_async16(sX + r * LDX + c, X + (size_t)min(row, g.N - 1) * D + c, row < g.N);
  }
  // W already split into bf16 hi + lo rows n = 4 l + b (race_w_split_kernel), [NW][D] each
  for (int i = tid; i < 2 * NW * (D / 8); i += 128) {
    const int half = i / (NW * (D / 8)), r = (i / (D / 8)) % NW, c = (i % (D / 8)) * 8;
    cp_async16((half ? sWl : sWh) + r * LDX + c, Wsplit + ((size_t)half * NW + r) * D + c, true);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  // row norms (fp32 sum of squares of the exact bf16 values)
  if (tid < 64) {
    float s = 0.f;
    for (int c = 0; c < D; ++c) {
      const float v = __bfloat162float(sX[tid * LDX + c]);
      s += v * v;
    }
    sN[tid] = fmaxf(sqrtf(s), kNormFloor);
  }
  // projections: each warp 16 rows x NW columns
  for (int nb2 = 0; nb2 < NW / 16; ++nb2) {
    float acc[2][4] = {};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a[4], bh_[4], bl_[4];
      ldsm_x4(a, a_frag_ptr(sX, LDX, warp * 16, kk * 16, lane));
      ldsm_x4(bh_, bnk_frag_ptr(sWh, LDX, nb2 * 16, kk * 16, lane));
      ldsm_x4(bl_, bnk_frag_ptr(sWl, LDX, nb2 * 16, kk * 16, lane));
      mma16816(acc[0], a, bh_[0], bh_[1]);
      mma16816(acc[1], a, bh_[2], bh_[3]);
      mma16816(acc[0], a, bl_[0], bl_[1]);
      mma16816(acc[1], a, bl_[2], bl_[3]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int col = nb2 * 16 + h * 8 + (lane & 3) * 2;
      const int r0 = warp * 16 + (lane >> 2);
      sH[r0 * (NW + 1) + col] = acc[h][0];
      sH[r0 * (NW + 1) + col + 1] = acc[h][1];
      sH[(r0 + 8) * (NW + 1) + col] = acc[h][2];
      sH[(r0 + 8) * (NW + 1) + col + 1] = acc[h][3];
    }
  }
  __syncthreads();

  const float inv_sqrt_L = rsqrtf((float)g.L);
  const float two_over_tau = 2.f / g.tau;
  for (int item = tid; item < 64 * g.L; item += 128) {
    const int r = item / g.L, l = item % g.L;
    const int row = row_base + r;
    if (row >= g.N) continue;
    const float inv_n = 1.f / sN[r];
    float sp[kHashBits], sm[kHashBits], hv[kHashBits];
#pragma unroll
    for (int b = 0; b < kHashBits; ++b) {
      hv[b] = sH[r * (NW + 1) + l * kHashBits + b] * inv_n;
      sigmoid_pair(two_over_tau * hv[b], sp[b], sm[b]);   // P(c_b = +1), P(c_b = -1)
    }
    if (hout) *reinterpret_cast<float4*>(hout + (size_t)row * NH + l * kHashBits) = make_float4(hv[0], hv[1], hv[2], hv[3]);
    float pc[kCorners];
    corner_probs(sp, sm, inv_sqrt_L, pc);
    __align__(16) __nv_bfloat16 out[kCorners];
#pragma unroll
    for (int c = 0; c < kCorners; ++c) out[c] = __float2bfloat16_rn(pc[c]);
    uint4* dst = reinterpret_cast<uint4*>(phi + (size_t)row * g.r + l * kCorners);
    dst[0] = reinterpret_cast<const uint4*>(out)[0];
    dst[1] = reinterpret_cast<const uint4*>(out)[1];
    if (l == 0 && nout) nout[row] = sN[r];
  }
}

// ---------------------------------------------------------------------------
// Segment summaries, bf16 path.  grid (n_seg, BH), block 32 * (r/16): warp w
// owns state rows [16w, 16w+16) x all dp columns in registers.
//   forward (BWD = false): walk the segment's chunks in order; for each chunk c
//     (causal) write the running in-segment exclusive prefix to Bst[c], then add
//     S_c = Phi(K_c)^T [V_c | 1].  The segment total goes to Ast[seg + 1].
//   backward (BWD = true): the same over Phi(Q_c)^T [cl dO_c | delta] walking
//     the chunks in reverse, giving in-segment exclusive suffixes (RB) and the
//     segment totals (RA[seg + 1]).
// Chunk length C == block size (64/128).
// ---------------------------------------------------------------------------
template <int D, int C, bool BWD>
__global__ void __launch_bounds__(512) race_state_bf16_kernel(const __nv_bfloat16* __restrict__ phi,
                                                              const __nv_bfloat16* __restrict__ Y,
                                                              const float* __restrict__ rscale,
                                                              const float* __restrict__ rextra,
                                                              float* __restrict__ Atot, float* __restrict__ Bpart,
                                                              Geom g) {
  constexpr int DP = D + 8;
  constexpr int NB = DP / 8;         // n-blocks of the state (odd)
  constexpr int LDV = D + 16;
  const int LDP = g.r + 8;
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* sP = reinterpret_cast<__nv_bfloat16*>(smem);     // [2][C][LDP]
  __nv_bfloat16* sV = sP + 2 * C * LDP;                            // [2][C][LDV]
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int c_begin = seg * g.seg, c_end = min(g.n_c, c_begin + g.seg);
  const int n_here = c_end - c_begin;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthr = blockDim.x;
  const __nv_bfloat16* pk = phi + (size_t)bh * g.N * g.r;
  const __nv_bfloat16* vv = Y + (size_t)bh * g.N * D;
  const float* rsc = BWD && rscale ? rscale + (size_t)bh * g.N : nullptr;
  const float* rex = BWD ? rextra + (size_t)bh * g.N : nullptr;

  auto load = [&](int buf, int c) {
    __nv_bfloat16* dP = sP + buf * C * LDP;
    __nv_bfloat16* dV = sV + buf * C * LDV;
    const int rchunks = g.r / 8;
    for (int i = tid; i < C * rchunks; i += nthr) {
      const int r = i / rchunks, cc = (i % rchunks) * 8;
      const int row = c * C + r;
      cp_async16(dP + r * LDP + cc, pk + (size_t)min(row, g.N - 1) * g.r + cc, row < g.N);
    }
    if (!BWD || !rsc) {
      // forward rows, or backward rows already scaled by cl
      for (int i = tid; i < C * (D / 8); i += nthr) {
        const int r = i / (D / 8), cc = (i % (D / 8)) * 8;
        const int row = c * C + r;
        cp_async16(dV + r * LDV + cc, vv + (size_t)min(row, g.N - 1) * D + cc, row < g.N);
      }
    } else {
      for (int i = tid; i < C * (D / 8); i += nthr) {
        const int r = i / (D / 8), cc = (i % (D / 8)) * 8;
        const int row = c * C + r;
        uint4 raw = make_uint4(0u, 0u, 0u, 0u);
        if (row < g.N) {
          raw = *reinterpret_cast<const uint4*>(vv + (size_t)row * D + cc);
          const float sc = rsc[row];
          __nv_bfloat16* e = reinterpret_cast<__nv_bfloat16*>(&raw);
#pragma unroll
          for (int j = 0; j < 8; ++j) e[j] = __float2bfloat16_rn(sc * __bfloat162float(e[j]));
        }
        *reinterpret_cast<uint4*>(dV + r * LDV + cc) = raw;
      }
    }
    for (int r = tid; r < C; r += nthr) {
      const int row = c * C + r;
      __nv_bfloat16* o = dV + r * LDV + D;
      const float x = row < g.N ? (BWD ? rex[row] : 1.f) : 0.f;
      o[0] = __float2bfloat16_rn(x);
#pragma unroll
      for (int j = 1; j < 8; ++j) o[j] = __float2bfloat16_rn(0.f);
    }
  };

  float acc[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;

  auto store_state = [&](float* dst) {
    const int r0 = warp * 16 + (lane >> 2);
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int col = nb * 8 + (lane & 3) * 2;
      *reinterpret_cast<float2*>(dst + (size_t)r0 * DP + col) = make_float2(acc[nb][0], acc[nb][1]);
      *reinterpret_cast<float2*>(dst + (size_t)(r0 + 8) * DP + col) = make_float2(acc[nb][2], acc[nb][3]);
    }
  };
  auto chunk_of = [&](int step) { return BWD ? c_end - 1 - step : c_begin + step; };

  if (n_here > 0) {
    load(0, chunk_of(0));
    cp_async_commit();
  }
  for (int step = 0; step < n_here; ++step) {
    const int c = chunk_of(step);
    const int buf = step & 1;
    if (step + 1 < n_here) {
      load(buf ^ 1, chunk_of(step + 1));
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (g.causal) store_state(Bpart + ((size_t)bh * g.n_c + c) * g.r * DP);
    const __nv_bfloat16* cP = sP + buf * C * LDP;
    const __nv_bfloat16* cV = sV + buf * C * LDV;
#pragma unroll 2
    for (int kk = 0; kk < C / 16; ++kk) {
      uint32_t a[4];
      ldsm_x4_t(a, at_frag_ptr(cP, LDP, warp * 16, kk * 16, lane));
#pragma unroll
      for (int nb2 = 0; nb2 < NB / 2; ++nb2) {
        uint32_t b[4];
        ldsm_x4_t(b, bkn_frag_ptr(cV, LDV, kk * 16, nb2 * 16, lane));
        mma16816(acc[2 * nb2], a, b[0], b[1]);
        mma16816(acc[2 * nb2 + 1], a, b[2], b[3]);
      }
      uint32_t b2[2];
      ldsm_x2_t(b2, bkn_frag_ptr1(cV, LDV, kk * 16, (NB - 1) * 8, lane));
      mma16816(acc[NB - 1], a, b2[0], b2[1]);
    }
    __syncthreads();
  }
  store_state(Atot + ((size_t)bh * (g.n_seg + 1) + seg + 1) * g.r * DP);
}

// Forward: exclusive prefix over segment totals, in place.  Afterwards slot s
// holds sum_{s' < s} total_{s'} and slot n_seg the grand total.
// Backward: exclusive suffix, in place.  Afterwards slot s + 1 holds
// sum_{s' > s} total_{s'} and slot 0 the grand total.
// (total_s is written to slot s + 1 by the state kernel.)  grid (ceil(r*dp/256), BH).
__global__ void race_scan_kernel(float* __restrict__ A, Geom g, int reverse) {
  const int e = blockIdx.x * 256 + threadIdx.x;
  const int n = g.r * g.dp;
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

// Statistics of chunk c for the tensor-core RACE kernels: S = A[slot] + B[c] (fp32 [r][dp])
// as bf16 hi and lo halves, row-major [r][d] each, stored [BH][n_c][2][r][d], and the
// key-mass column [BH][n_c][r] in fp32.  Forward: slot = the segment's exclusive prefix;
// backward: the exclusive suffix of the later segments.  grid (n_c, BH), block 256.
__global__ void __launch_bounds__(256) race_state_split_kernel(const float* __restrict__ A,
                                                               const float* __restrict__ B, int bwd,
                                                               __nv_bfloat16* __restrict__ out,
                                                               float* __restrict__ mass, Geom g) {
  const int c = blockIdx.x, bh = blockIdx.y;
  const size_t state = (size_t)g.r * g.dp;
  const int slot = bwd ? (g.causal ? c / g.seg + 1 : 0) : (g.causal ? c / g.seg : g.n_seg);
  const float* a = A + ((size_t)bh * (g.n_seg + 1) + slot) * state;
  const float* b = g.causal ? B + ((size_t)bh * g.n_c + c) * state : nullptr;
  __nv_bfloat16* hi = out + ((size_t)bh * g.n_c + c) * 2 * g.r * g.d;
  __nv_bfloat16* lo = hi + (size_t)g.r * g.d;
  const int q4 = g.d / 4;
#pragma unroll 4
  for (int i = threadIdx.x; i < g.r * q4; i += blockDim.x) {
    const int f = i / q4, e = (i % q4) * 4;
    float4 v = *reinterpret_cast<const float4*>(a + (size_t)f * g.dp + e);
    if (b) {
      const float4 w = *reinterpret_cast<const float4*>(b + (size_t)f * g.dp + e);
      v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
    }
    __nv_bfloat16 h[4], l[4];
    const float x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      h[k] = __float2bfloat16_rn(x[k]);
      l[k] = __float2bfloat16_rn(x[k] - __bfloat162float(h[k]));
    }
    *reinterpret_cast<uint2*>(hi + (size_t)f * g.d + e) = *reinterpret_cast<const uint2*>(h);
    *reinterpret_cast<uint2*>(lo + (size_t)f * g.d + e) = *reinterpret_cast<const uint2*>(l);
  }
  for (int f = threadIdx.x; f < g.r; f += blockDim.x)
    mass[((size_t)bh * g.n_c + c) * g.r + f] = a[(size_t)f * g.dp + g.d] + (b ? b[(size_t)f * g.dp + g.d] : 0.f);
}

cudaError_t launch_race_state_split(const float* A, const float* B, bool bwd, void* out, float* mass, const Geom& g,
                                    cudaStream_t st) {
  ProfScope ps(bwd ? "race_split_bwd" : "race_split_fwd", st);
  race_state_split_kernel<<<dim3(g.n_c, g.BH), 256, 0, st>>>(A, B, bwd ? 1 : 0, (__nv_bfloat16*)out, mass, g);
  return cudaGetLastError();
}

cudaError_t launch_race_w_split(const float* W, void* out, const Geom& g, cudaStream_t st) {
  const int NW = (g.L * kHashBits + 15) & ~15;
  race_w_split_kernel<<<(NW * g.d + 255) / 256, 256, 0, st>>>(W, (__nv_bfloat16*)out, g.d, g.L * kHashBits, NW);
  return cudaGetLastError();
}

static size_t features_smem(const Geom& g) {
  const int NW = (g.L * kHashBits + 15) & ~15;
  return (size_t)(64 + 2 * NW) * (g.d + 8) * 2 + (size_t)64 * (NW + 1) * 4 + 64 * 4;
}

cudaError_t launch_race_features(const void* Q, const void* K, const float* W, void* wsplit, bool bf16, void* phiQ,
                                 void* phiK, float* hQ, float* hK, float* nQ, float* nK, const Geom& g,
                                 cudaStream_t st) {
  if (g.r == 0) return cudaSuccess;
  if (!bf16) {
    ProfScope ps("race_features_f32", st);
    race_features_f32_kernel<<<dim3((g.N + 7) / 8, g.BH, 2), 256, 0, st>>>(
        (const float*)Q, (const float*)K, W, (float*)phiQ, (float*)phiK, hQ, hK, nQ, nK, g);
    return cudaGetLastError();
  }
  const size_t smem = features_smem(g);
  const int NW = (g.L * kHashBits + 15) & ~15;
  race_w_split_kernel<<<(NW * g.d + 255) / 256, 256, 0, st>>>(W, (__nv_bfloat16*)wsplit, g.d, g.L * kHashBits, NW);
  auto run = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ProfScope ps("race_features", st);
    kern<<<dim3((g.N + 63) / 64, g.BH, 2), 128, smem, st>>>(
        (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)wsplit, (__nv_bfloat16*)phiQ,
        (__nv_bfloat16*)phiK, hQ, hK, nQ, nK, g);
    return cudaGetLastError();
  };
  if (g.d == 64) return run(race_features_bf16_kernel<64>);
  return run(race_features_bf16_kernel<128>);
}

template <bool BWD>
static cudaError_t run_state(const void* phi, const void* Y, const float* rsc, const float* rex, bool bf16,
                             float* Atot, float* Bpart, const Geom& g, cudaStream_t st) {
  if (!bf16) {
    const int n = g.r * g.dp;
    ProfScope ps(BWD ? "race_state_bwd_f32" : "race_state_fwd_f32", st);
    race_state_f32_kernel<BWD><<<dim3(g.n_seg, g.BH, (n + 255) / 256), 256, 0, st>>>(
        (const float*)phi, (const float*)Y, rsc, rex, Atot, Bpart, g);
  } else {
    const size_t smem = (size_t)2 * g.C * (g.r + 8) * 2 + (size_t)2 * g.C * (g.d + 16) * 2;
    auto go = [&](auto kern) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      ProfScope ps(BWD ? "race_state_bwd" : "race_state_fwd", st);
      kern<<<dim3(g.n_seg, g.BH), 32 * (g.r / 16), smem, st>>>(
          (const __nv_bfloat16*)phi, (const __nv_bfloat16*)Y, rsc, rex, Atot, Bpart, g);
      return cudaGetLastError();
    };
    cudaError_t e;
    if (g.d == 64 && g.C == 64) e = go(race_state_bf16_kernel<64, 64, BWD>);
    else if (g.d == 64) e = go(race_state_bf16_kernel<64, 128, BWD>);
    else if (g.C == 64) e = go(race_state_bf16_kernel<128, 64, BWD>);
    else e = go(race_state_bf16_kernel<128, 128, BWD>);
    if (e != cudaSuccess) return e;
  }
  {
    ProfScope ps(BWD ? "race_scan_bwd" : "race_scan_fwd", st);
    race_scan_kernel<<<dim3((g.r * g.dp + 255) / 256, g.BH), 256, 0, st>>>(Atot, g, BWD ? 1 : 0);
  }
  return cudaGetLastError();
}

cudaError_t launch_race_state_fwd(const void* phiK, const void* V, bool bf16, float* Ast, float* Bst,
                                  const Geom& g, cudaStream_t st) {
  if (g.r == 0) return cudaSuccess;
  return run_state<false>(phiK, V, nullptr, nullptr, bf16, Ast, Bst, g, st);
}

cudaError_t launch_race_state_bwd(const BwdArgs& a, bool bf16, const Geom& g, cudaStream_t st) {
  if (g.r == 0) return cudaSuccess;
  // bf16: the row scalars already wrote cl dO, so the rows stream in with cp.async
  if (bf16 && a.dOcl) return run_state<true>(a.phiQ, a.dOcl, nullptr, a.rs.delta, bf16, a.RA, a.RB, g, st);
  return run_state<true>(a.phiQ, a.dO, a.rs.cl, a.rs.delta, bf16, a.RA, a.RB, g, st);
}

}  // namespace elsaa
