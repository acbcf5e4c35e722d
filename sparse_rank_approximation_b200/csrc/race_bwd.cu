// RACE low-rank branch backward (ELSAA paper §3.1), bf16 tensor-core path.
//
// Query side, per tile t of query rows i:
//   dPhi(q_i) = cl_i P^V_t dO_i + delta_i p1_t + sum_{j in chunk t, j <= i} dkappa_ij Phi(k_j),
//   dkappa_ij = cl_i <dO_i, v_j> + delta_i,
// with P_t the forward prefix statistics (P^V its value columns, p1 its key-mass column).
// Key side, per chunk c of key rows j:
//   dPhi(k_j) = R^V_{>c} v_j + r1_{>c} + sum_{i in chunk c, i >= j} dkappa_ij Phi(q_i),
//   dv_j      = (R^V_{>c})^T Phi(k_j) + sum_{i in chunk c, i >= j} kappa_ij cl_i dO_i,
// with R_{>c} = sum over later chunks of Phi(q_i) [cl_i dO_i ; delta_i]^T (suffix statistics).
// Both then pull dPhi back through the features: per table the corner softmax
// (dh_b = (1/tau) sum_c p_c (dp_c - <dp, p>) c_b, dp = dPhi / sqrt(L)), then
// du = W dh and dx = (du - u <u, du>) / |x|.  The projections h = W^T u are
// recomputed from the staged rows (bf16 rows times W as bf16 hi + lo halves), and
// du = dh W^T runs on the tensor cores with dh and W split into hi + lo halves.
#include "common.cuh"
#include "kernels.h"

namespace elsaa {

namespace {

constexpr int kMaxNH = 64;          // projection columns 4L, r <= 256
constexpr int kLDF = 72;            // feature chunk pitch (64 + 8)
constexpr int kLDH = kMaxNH + 4;    // dh pitch (fp32)

template <int D, int T>
struct RBSmem {
  static constexpr int LD = D + 8;
  static constexpr int SR = T > 128 ? T : 128;                       // rows of the tile/state region
  static constexpr size_t off_x = 0;                                   // Q or K rows      [T][LD]
  static constexpr size_t off_a = off_x + (size_t)T * LD * 2;          // dO (q) / V (k)   [T][LD]
  static constexpr size_t off_b = off_a + (size_t)T * LD * 2;          // V / dO, then state hi+lo
  static constexpr size_t off_wh = off_b + (size_t)SR * LD * 2;        // W hi [kMaxNH][LD]
  static constexpr size_t off_wl = off_wh + (size_t)kMaxNH * LD * 2;   // W lo
  static constexpr size_t off_f1 = off_wl + (size_t)kMaxNH * LD * 2;   // features [T][kLDF]
  static constexpr size_t off_f2 = off_f1 + (size_t)T * kLDF * 2;      // features [T][kLDF]
  static constexpr size_t off_s1 = off_f2 + (size_t)T * kLDF * 2;      // key-mass column [64]
  static constexpr size_t off_cl = off_s1 + 64 * 4;                    // cl [T]
  static constexpr size_t off_dl = off_cl + (size_t)T * 4;             // delta [T]
  static constexpr size_t off_dh = off_dl + (size_t)T * 4;             // dh [T][kLDH]
  static constexpr size_t bytes = off_dh + (size_t)T * kLDH * 4;
};

__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// W[l][k][b] (fp32, [L][D][4]) -> rows n = 4l + b of [kMaxNH][LD] hi/lo bf16, zero beyond 4L.
// Loads are issued in batches of 8 before any conversion so their latencies overlap.
template <int D, int NT>
__device__ void stage_w(const float* __restrict__ W, int NH, __nv_bfloat16* sWh, __nv_bfloat16* sWl) {
  constexpr int LD = D + 8;
  constexpr int PER = kMaxNH * D / NT;
  static_assert(PER % 8 == 0, "W staging batch");
#pragma unroll 1
  for (int k0 = 0; k0 < PER; k0 += 8) {
    float w[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = threadIdx.x + (k0 + k) * NT;
      const int n = i / D, col = i % D;
      w[k] = n < NH ? __ldg(W + ((size_t)(n >> 2) * D + col) * kHashBits + (n & 3)) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = threadIdx.x + (k0 + k) * NT;
      const int n = i / D, col = i % D;
      split_bf16(w[k], sWh[n * LD + col], sWl[n * LD + col]);
    }
  }
}

template <int T>
__device__ __forceinline__ void load_rows(__nv_bfloat16* dst, int ld, const __nv_bfloat16* __restrict__ src,
                                          int src_ld, int col0, int width, int row_base, int N, int nthr) {
  const int ch = width / 8;
  for (int i = threadIdx.x; i < T * ch; i += nthr) {
    const int r = i / ch, c = (i % ch) * 8;
    const int row = row_base + r;
    cp_async16(dst + r * ld + c, src + (size_t)min(row, N - 1) * src_ld + col0 + c, row < N);
  }
}

// Rows [f0, f0 + 64) of a float32 state [r][dp] (sum of up to two sources) as bf16
// hi/lo [64][LD] (value columns) and the key-mass column; rows >= `rows` are zero.
// Each thread issues its loads in batches of 4 float4 before converting.
template <int D, int NT>
__device__ void load_state(const float* __restrict__ s0, const float* __restrict__ s1, int f0, int rows, int dp,
                           __nv_bfloat16* sh, __nv_bfloat16* sl, float* s1col) {
  constexpr int LD = D + 8;
  constexpr int Q4 = D / 4;
  constexpr int PER = 64 * Q4 / NT;
  static_assert(PER % 4 == 0, "state staging batch");
#pragma unroll 1
  for (int k0 = 0; k0 < PER; k0 += 4) {
    float4 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = threadIdx.x + (k0 + k) * NT;
      const int r = i / Q4, c = (i % Q4) * 4;
      v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < rows) {
        v[k] = __ldg(reinterpret_cast<const float4*>(s0 + (size_t)(f0 + r) * dp + c));
        if (s1) {
          const float4 w = __ldg(reinterpret_cast<const float4*>(s1 + (size_t)(f0 + r) * dp + c));
          v[k].x += w.x; v[k].y += w.y; v[k].z += w.z; v[k].w += w.w;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = threadIdx.x + (k0 + k) * NT;
      const int r = i / Q4, c = (i % Q4) * 4;
      __nv_bfloat16 h[4], l[4];
      split_bf16(v[k].x, h[0], l[0]);
      split_bf16(v[k].y, h[1], l[1]);
      split_bf16(v[k].z, h[2], l[2]);
      split_bf16(v[k].w, h[3], l[3]);
      *reinterpret_cast<uint2*>(sh + r * LD + c) = *reinterpret_cast<const uint2*>(h);
      *reinterpret_cast<uint2*>(sl + r * LD + c) = *reinterpret_cast<const uint2*>(l);
    }
  }
  for (int r = threadIdx.x; r < 64; r += NT) {
    float v = 0.f;
    if (r < rows) {
      v = s0[(size_t)(f0 + r) * dp + D];
      if (s1) v += s1[(size_t)(f0 + r) * dp + D];
    }
    s1col[r] = v;
  }
}

// H = X (W_hi + W_lo) for the warp's 16 rows (all projection columns) and the row
// norms max(|x|, 1e-12) of rows g4 and g4 + 8.
template <int D>
__device__ __forceinline__ void project_rows(const __nv_bfloat16* sX, const __nv_bfloat16* sWh,
                                             const __nv_bfloat16* sWl, int NH, int row0, float (&H)[8][4],
                                             float (&nrm)[2]) {
  constexpr int LD = D + 8;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int nb = 0; nb < 8; ++nb) H[nb][0] = H[nb][1] = H[nb][2] = H[nb][3] = 0.f;
  float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4(a, a_frag_ptr(sX, LD, row0, kk * 16, lane));
    const float2 x0 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&a[0]));
    const float2 x1 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&a[1]));
    const float2 x2 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&a[2]));
    const float2 x3 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&a[3]));
    ss0 += x0.x * x0.x + x0.y * x0.y + x2.x * x2.x + x2.y * x2.y;
    ss1 += x1.x * x1.x + x1.y * x1.y + x3.x * x3.x + x3.y * x3.y;
#pragma unroll
    for (int nb2 = 0; nb2 < 4; ++nb2) {
      if (nb2 * 16 >= NH) break;
      uint32_t bh[4], bl[4];
      ldsm_x4(bh, bnk_frag_ptr(sWh, LD, nb2 * 16, kk * 16, lane));
      ldsm_x4(bl, bnk_frag_ptr(sWl, LD, nb2 * 16, kk * 16, lane));
      mma16816(H[2 * nb2], a, bh[0], bh[1]);
      mma16816(H[2 * nb2 + 1], a, bh[2], bh[3]);
      mma16816(H[2 * nb2], a, bl[0], bl[1]);
      mma16816(H[2 * nb2 + 1], a, bl[2], bl[3]);
    }
  }
  ss0 += __shfl_xor_sync(0xffffffffu, ss0, 1);
  ss0 += __shfl_xor_sync(0xffffffffu, ss0, 2);
  ss1 += __shfl_xor_sync(0xffffffffu, ss1, 1);
  ss1 += __shfl_xor_sync(0xffffffffu, ss1, 2);
  nrm[0] = fmaxf(sqrtf(ss0), kNormFloor);
  nrm[1] = fmaxf(sqrtf(ss1), kNormFloor);
}

// The 4 normalised projections of table l (compile-time after unrolling) for row
// half hh, gathered from the quad's H fragments.
__device__ __forceinline__ void table_h(const float (&H)[8][4], int l, int hh, float n, float (&h)[4]) {
  const int lane = threadIdx.x & 31;
  const int nb = l >> 1, p = l & 1;
  const int base = lane & ~3;
  const float a0 = __shfl_sync(0xffffffffu, H[nb][2 * hh], base | (2 * p));
  const float a1 = __shfl_sync(0xffffffffu, H[nb][2 * hh + 1], base | (2 * p));
  const float a2 = __shfl_sync(0xffffffffu, H[nb][2 * hh], base | (2 * p + 1));
  const float a3 = __shfl_sync(0xffffffffu, H[nb][2 * hh + 1], base | (2 * p + 1));
  const float inv = 1.f / n;
  h[0] = a0 * inv;
  h[1] = a1 * inv;
  h[2] = a2 * inv;
  h[3] = a3 * inv;
}

// Corner-softmax backward of one table for the 4 features this thread holds in a
// 16 x 64 fragment G (n-blocks 2tl, 2tl+1; row half hh).  Returns dh_b (quad-reduced).
__device__ __forceinline__ void corner_bwd(const float (&G)[8][4], int tl, int hh, const float (&h)[4],
                                           float inv_sqrt_L, float inv_tau, float (&dh)[4]) {
  const int t4 = threadIdx.x & 3;
  float sp[4], sm[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const float y = 2.f * h[b] * inv_tau;
    sp[b] = 1.f / (1.f + expf(-y));
    sm[b] = 1.f / (1.f + expf(y));
  }
  float p[4], dp[4];
  int cidx[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = (q >> 1) * 8 + 2 * t4 + (q & 1);
    cidx[q] = c;
    float pv = 1.f;
#pragma unroll
    for (int b = 0; b < 4; ++b) pv *= ((c >> b) & 1) ? sp[b] : sm[b];
    p[q] = pv;
    dp[q] = G[2 * tl + (q >> 1)][2 * hh + (q & 1)] * inv_sqrt_L;
  }
  float s = dp[0] * p[0] + dp[1] * p[1] + dp[2] * p[2] + dp[3] * p[3];
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
    dh[b] *= inv_tau;
  }
}

// Corner softmax for every table of a 64-feature chunk; writes dh to sdh.
__device__ __forceinline__ void chunk_corner_bwd(const float (&G)[8][4], const float (&H)[8][4],
                                                 const float (&nrm)[2], int chunk, int rcw, int row0,
                                                 float inv_sqrt_L, float inv_tau, float* sdh) {
  const int lane = threadIdx.x & 31, g4 = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int tl = 0; tl < 4; ++tl) {
    if (tl * 16 >= rcw) break;
    const int l = chunk * 4 + tl;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float h[4], dh[4];
      table_h(H, l, hh, nrm[hh], h);
      corner_bwd(G, tl, hh, h, inv_sqrt_L, inv_tau, dh);
      sdh[(row0 + g4 + 8 * hh) * kLDH + l * 4 + t4] = t4 == 0 ? dh[0] : t4 == 1 ? dh[1] : t4 == 2 ? dh[2] : dh[3];
    }
  }
}

// du = dh W^T (hi/lo split of both, three MMAs per step), then
// dx = (du - x <x, du> / n^2) / n, stored as fp32 rows [row_base + r][D].
template <int D>
__device__ __forceinline__ void chain_rows(const float* sdh, const __nv_bfloat16* sWh, const __nv_bfloat16* sWl,
                                           const __nv_bfloat16* sX, int NH, int row0, const float (&nrm)[2],
                                           float* __restrict__ out, int row_base, int N) {
  constexpr int LD = D + 8;
  constexpr int NBD = D / 8;
  const int lane = threadIdx.x & 31, g4 = lane >> 2, t4 = lane & 3;
  float du[NBD][4];
#pragma unroll
  for (int nb = 0; nb < NBD; ++nb) du[nb][0] = du[nb][1] = du[nb][2] = du[nb][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < kMaxNH / 16; ++kk) {
    if (kk * 16 >= NH) break;
    uint32_t ah[4], al[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = row0 + g4 + 8 * (q & 1);
      const int c = kk * 16 + 8 * (q >> 1) + 2 * t4;
      const float x0 = sdh[r * kLDH + c], x1 = sdh[r * kLDH + c + 1];
      __nv_bfloat16 h0, l0, h1, l1;
      split_bf16(x0, h0, l0);
      split_bf16(x1, h1, l1);
      __nv_bfloat162 hv(h0, h1), lv(l0, l1);
      ah[q] = *reinterpret_cast<uint32_t*>(&hv);
      al[q] = *reinterpret_cast<uint32_t*>(&lv);
    }
#pragma unroll
    for (int nb2 = 0; nb2 < NBD / 2; ++nb2) {
      uint32_t bh[4], bl[4];
      ldsm_x4_t(bh, bkn_frag_ptr(sWh, LD, kk * 16, nb2 * 16, lane));
      ldsm_x4_t(bl, bkn_frag_ptr(sWl, LD, kk * 16, nb2 * 16, lane));
      mma16816(du[2 * nb2], ah, bh[0], bh[1]);
      mma16816(du[2 * nb2 + 1], ah, bh[2], bh[3]);
      mma16816(du[2 * nb2], ah, bl[0], bl[1]);
      mma16816(du[2 * nb2 + 1], ah, bl[2], bl[3]);
      mma16816(du[2 * nb2], al, bh[0], bh[1]);
      mma16816(du[2 * nb2 + 1], al, bh[2], bh[3]);
    }
  }
  float xd[2] = {0.f, 0.f};
#pragma unroll
  for (int nb = 0; nb < NBD; ++nb) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const float2 x = __bfloat1622float2(
          *reinterpret_cast<const __nv_bfloat162*>(sX + (row0 + g4 + 8 * hh) * LD + nb * 8 + 2 * t4));
      xd[hh] += x.x * du[nb][2 * hh] + x.y * du[nb][2 * hh + 1];
    }
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    xd[hh] += __shfl_xor_sync(0xffffffffu, xd[hh], 1);
    xd[hh] += __shfl_xor_sync(0xffffffffu, xd[hh], 2);
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int r = row0 + g4 + 8 * hh;
    const int row = row_base + r;
    if (row >= N) continue;
    const float n = nrm[hh];
    const float proj = n <= kNormFloor ? 0.f : xd[hh] / (n * n);
    const float inv = 1.f / n;
#pragma unroll
    for (int nb = 0; nb < NBD; ++nb) {
      const int col = nb * 8 + 2 * t4;
      const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sX + r * LD + col));
      *reinterpret_cast<float2*>(out + (size_t)row * D + col) =
          make_float2((du[nb][2 * hh] - x.x * proj) * inv, (du[nb][2 * hh + 1] - x.y * proj) * inv);
    }
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// Query side: dQacc rows of tile t.  grid (n_t, BH), block 2T.
// ---------------------------------------------------------------------------
template <int D, int T>
__global__ void __launch_bounds__(2 * T) race_q_bwd_bf16_kernel(BwdArgs a, Geom g) {
  using S = RBSmem<D, T>;
  constexpr int LD = S::LD, NT = 2 * T;
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* sX = reinterpret_cast<__nv_bfloat16*>(smem + S::off_x);
  __nv_bfloat16* sdO = reinterpret_cast<__nv_bfloat16*>(smem + S::off_a);
  __nv_bfloat16* sU = reinterpret_cast<__nv_bfloat16*>(smem + S::off_b);     // V, then state hi
  __nv_bfloat16* sPl = sU + 64 * LD;                                          // state lo
  __nv_bfloat16* sWh = reinterpret_cast<__nv_bfloat16*>(smem + S::off_wh);
  __nv_bfloat16* sWl = reinterpret_cast<__nv_bfloat16*>(smem + S::off_wl);
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
  const int NH = g.L * kHashBits;

  load_rows<T>(sX, LD, (const __nv_bfloat16*)a.Q + head * D, D, 0, D, t * T, g.N, NT);
  load_rows<T>(sdO, LD, (const __nv_bfloat16*)a.dO + head * D, D, 0, D, t * T, g.N, NT);
  if (g.causal) load_rows<T>(sU, LD, (const __nv_bfloat16*)a.V + head * D, D, 0, D, t * T, g.N, NT);
  cp_async_commit();
  stage_w<D, NT>(a.W, NH, sWh, sWl);
  for (int i = tid; i < T * kLDH; i += NT) sdh[i] = 0.f;
  for (int r = tid; r < T; r += NT) {
    const int row = t * T + r;
    scl[r] = row < g.N ? a.rs.cl[head + row] : 0.f;
    sdel[r] = row < g.N ? a.rs.delta[head + row] : 0.f;
  }
  cp_async_wait<0>();
  __syncthreads();

  float H[8][4], nrm[2];
  project_rows<D>(sX, sWh, sWl, NH, row0, H, nrm);

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
        ldsm_x4(bf, bnk_frag_ptr(sU, LD, nb2 * 16, kk * 16, lane));
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
  const float cl_r[2] = {scl[rl[0]], scl[rl[1]]};
  const float de_r[2] = {sdel[rl[0]], sdel[rl[1]]};

  const float* pa = a.Ast + ((size_t)bh * (g.n_seg + 1) + (g.causal ? t / g.seg : g.n_seg)) * g.r * g.dp;
  const float* pb = g.causal ? a.Bst + ((size_t)bh * g.n_c + t) * g.r * g.dp : nullptr;
  const __nv_bfloat16* fk = (const __nv_bfloat16*)a.phiK + head * g.r;
  const float inv_sqrt_L = rsqrtf((float)g.L), inv_tau = 1.f / g.tau;
#pragma unroll
  for (int ci = 0; ci < 4; ++ci) {
    const int rc = ci * 64;
    if (rc >= g.r) break;
    const int rcw = min(64, g.r - rc);
    __syncthreads();
    if (g.causal) {
      load_rows<T>(sF, kLDF, fk, g.r, rc, rcw, t * T, g.N, NT);
      cp_async_commit();
    }
    load_state<D, NT>(pa, pb, rc, rcw, g.dp, sU, sPl, sp1);
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
        ldsm_x4(bh_, bnk_frag_ptr(sU, LD, nb2 * 16, kk * 16, lane));
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
        G[nb][e] = cl_r[e >> 1] * G[nb][e] + de_r[e >> 1] * sp1[f];
      }
    }
    if (g.causal) {
#pragma unroll
      for (int kk = 0; kk < T / 16; ++kk) {
#pragma unroll
        for (int nb2 = 0; nb2 < 4; ++nb2) {
          if (nb2 * 16 >= rcw) break;
          uint32_t bf[4];
          ldsm_x4_t(bf, bkn_frag_ptr(sF, kLDF, kk * 16, nb2 * 16, lane));
          mma16816(G[2 * nb2], dk_pk[kk], bf[0], bf[1]);
          mma16816(G[2 * nb2 + 1], dk_pk[kk], bf[2], bf[3]);
        }
      }
    }
    chunk_corner_bwd(G, H, nrm, ci, rcw, row0, inv_sqrt_L, inv_tau, sdh);
  }
  __syncthreads();
  chain_rows<D>(sdh, sWh, sWl, sX, NH, row0, nrm, a.dQacc + head * D, t * T, g.N);
}

// ---------------------------------------------------------------------------
// Key side: dKacc and dVacc rows of chunk c.  grid (n_t, BH), block 2T.
// ---------------------------------------------------------------------------
template <int D, int T>
__global__ void __launch_bounds__(2 * T) race_k_bwd_bf16_kernel(BwdArgs a, Geom g) {
  using S = RBSmem<D, T>;
  constexpr int LD = S::LD, NT = 2 * T, NBD = D / 8;
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* sX = reinterpret_cast<__nv_bfloat16*>(smem + S::off_x);      // K rows
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + S::off_a);
  __nv_bfloat16* sdO = reinterpret_cast<__nv_bfloat16*>(smem + S::off_b);     // dO, then state hi
  __nv_bfloat16* sRl = sdO + 64 * LD;                                          // state lo
  __nv_bfloat16* sWh = reinterpret_cast<__nv_bfloat16*>(smem + S::off_wh);
  __nv_bfloat16* sWl = reinterpret_cast<__nv_bfloat16*>(smem + S::off_wl);
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
  const int NH = g.L * kHashBits;
  const __nv_bfloat16* dO = (const __nv_bfloat16*)a.dO + head * D;
  const __nv_bfloat16* fk = (const __nv_bfloat16*)a.phiK + head * g.r;
  const __nv_bfloat16* fq = (const __nv_bfloat16*)a.phiQ + head * g.r;

  load_rows<T>(sX, LD, (const __nv_bfloat16*)a.K + head * D, D, 0, D, c * T, g.N, NT);
  load_rows<T>(sV, LD, (const __nv_bfloat16*)a.V + head * D, D, 0, D, c * T, g.N, NT);
  if (g.causal) load_rows<T>(sdO, LD, dO, D, 0, D, c * T, g.N, NT);
  cp_async_commit();
  stage_w<D, NT>(a.W, NH, sWh, sWl);
  for (int i = tid; i < T * kLDH; i += NT) sdh[i] = 0.f;
  for (int r = tid; r < T; r += NT) {
    const int row = c * T + r;
    scl[r] = row < g.N ? a.rs.cl[head + row] : 0.f;
    sdel[r] = row < g.N ? a.rs.delta[head + row] : 0.f;
  }
  cp_async_wait<0>();
  __syncthreads();

  float H[8][4], nrm[2];
  project_rows<D>(sX, sWh, sWl, NH, row0, H, nrm);

  float dv[NBD][4];
#pragma unroll
  for (int nb = 0; nb < NBD; ++nb) dv[nb][0] = dv[nb][1] = dv[nb][2] = dv[nb][3] = 0.f;
  uint32_t dkT[T / 16][4];
  if (g.causal) {
    float X[T / 8][4];
    // kappa^T[j][i] = Phi(k_j).Phi(q_i), i >= j, scaled by cl_i; dv += kappa^T dO
#pragma unroll
    for (int nb = 0; nb < T / 8; ++nb) X[nb][0] = X[nb][1] = X[nb][2] = X[nb][3] = 0.f;
#pragma unroll
    for (int ci = 0; ci < 4; ++ci) {
      const int rc = ci * 64;
      if (rc >= g.r) break;
      const int rcw = min(64, g.r - rc);
      __syncthreads();
      load_rows<T>(sFk, kLDF, fk, g.r, rc, rcw, c * T, g.N, NT);
      load_rows<T>(sFq, kLDF, fq, g.r, rc, rcw, c * T, g.N, NT);
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        if (kk * 16 >= rcw) break;
        uint32_t af[4];
        ldsm_x4(af, a_frag_ptr(sFk, kLDF, row0, kk * 16, lane));
#pragma unroll
        for (int nb2 = 0; nb2 < T / 16; ++nb2) {
          uint32_t bf[4];
          ldsm_x4(bf, bnk_frag_ptr(sFq, kLDF, nb2 * 16, kk * 16, lane));
          mma16816(X[2 * nb2], af, bf[0], bf[1]);
          mma16816(X[2 * nb2 + 1], af, bf[2], bf[3]);
        }
      }
    }
#pragma unroll
    for (int kk = 0; kk < T / 16; ++kk) {
      uint32_t ap[4];
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int nb = 2 * kk + (e >> 2);
        const int col = nb * 8 + 2 * t4 + (e & 1);
        v[e] = col >= rl[(e >> 1) & 1] ? scl[col] * X[nb][e & 3] : 0.f;
      }
      ap[0] = pack_bf16(v[0], v[1]);
      ap[1] = pack_bf16(v[2], v[3]);
      ap[2] = pack_bf16(v[4], v[5]);
      ap[3] = pack_bf16(v[6], v[7]);
#pragma unroll
      for (int nb2 = 0; nb2 < NBD / 2; ++nb2) {
        uint32_t bf[4];
        ldsm_x4_t(bf, bkn_frag_ptr(sdO, LD, kk * 16, nb2 * 16, lane));
        mma16816(dv[2 * nb2], ap, bf[0], bf[1]);
        mma16816(dv[2 * nb2 + 1], ap, bf[2], bf[3]);
      }
    }
    // dkappa^T[j][i] = cl_i <dO_i, v_j> + delta_i for i >= j
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
  }

  const float* ra = a.RA + ((size_t)bh * (g.n_seg + 1) + (g.causal ? c / g.seg + 1 : 0)) * g.r * g.dp;
  const float* rb = g.causal ? a.RB + ((size_t)bh * g.n_c + c) * g.r * g.dp : nullptr;
  const float inv_sqrt_L = rsqrtf((float)g.L), inv_tau = 1.f / g.tau;
  const bool valid[2] = {c * T + rl[0] < g.N, c * T + rl[1] < g.N};
#pragma unroll
  for (int ci = 0; ci < 4; ++ci) {
    const int rc = ci * 64;
    if (rc >= g.r) break;
    const int rcw = min(64, g.r - rc);
    __syncthreads();
    load_rows<T>(sFk, kLDF, fk, g.r, rc, rcw, c * T, g.N, NT);
    if (g.causal) load_rows<T>(sFq, kLDF, fq, g.r, rc, rcw, c * T, g.N, NT);
    cp_async_commit();
    load_state<D, NT>(ra, rb, rc, rcw, g.dp, sdO, sRl, sr1);
    cp_async_wait<0>();
    __syncthreads();
    // inter-chunk value gradient: Phi_K[:, rc:rc+64] R^V[rc:rc+64, :]
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      if (kk * 16 >= rcw) break;
      uint32_t af[4];
      ldsm_x4(af, a_frag_ptr(sFk, kLDF, row0, kk * 16, lane));
#pragma unroll
      for (int nb2 = 0; nb2 < NBD / 2; ++nb2) {
        uint32_t bh_[4], bl_[4];
        ldsm_x4_t(bh_, bkn_frag_ptr(sdO, LD, kk * 16, nb2 * 16, lane));
        ldsm_x4_t(bl_, bkn_frag_ptr(sRl, LD, kk * 16, nb2 * 16, lane));
        mma16816(dv[2 * nb2], af, bh_[0], bh_[1]);
        mma16816(dv[2 * nb2 + 1], af, bh_[2], bh_[3]);
        mma16816(dv[2 * nb2], af, bl_[0], bl_[1]);
        mma16816(dv[2 * nb2 + 1], af, bl_[2], bl_[3]);
      }
    }
    // dPhi(k_j), this chunk: R^V v_j + r1 + sum_{i >= j} dkappa_ij Phi(q_i)
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
        ldsm_x4(bh_, bnk_frag_ptr(sdO, LD, nb2 * 16, kk * 16, lane));
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
        if (valid[e >> 1]) G[nb][e] += sr1[f];
      }
    }
    if (g.causal) {
#pragma unroll
      for (int kk = 0; kk < T / 16; ++kk) {
#pragma unroll
        for (int nb2 = 0; nb2 < 4; ++nb2) {
          if (nb2 * 16 >= rcw) break;
          uint32_t bf[4];
          ldsm_x4_t(bf, bkn_frag_ptr(sFq, kLDF, kk * 16, nb2 * 16, lane));
          mma16816(G[2 * nb2], dkT[kk], bf[0], bf[1]);
          mma16816(G[2 * nb2 + 1], dkT[kk], bf[2], bf[3]);
        }
      }
    }
    chunk_corner_bwd(G, H, nrm, ci, rcw, row0, inv_sqrt_L, inv_tau, sdh);
  }
  // value gradient rows
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int row = c * T + rl[hh];
    if (row < g.N) {
#pragma unroll
      for (int nb = 0; nb < NBD; ++nb) {
        const int col = nb * 8 + 2 * t4;
        *reinterpret_cast<float2*>(a.dVacc + (head + row) * D + col) = make_float2(dv[nb][2 * hh], dv[nb][2 * hh + 1]);
      }
    }
  }
  __syncthreads();
  chain_rows<D>(sdh, sWh, sWl, sX, NH, row0, nrm, a.dKacc + head * D, c * T, g.N);
}

template <typename KernT>
static cudaError_t launch_rb(const char* name, KernT kern, size_t smem, int T, const BwdArgs& a, const Geom& g,
                             cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(name, st);
  kern<<<dim3(g.n_t, g.BH), 2 * T, smem, st>>>(a, g);
  return cudaGetLastError();
}

template <int D, int T>
static cudaError_t race_bwd_t(const BwdArgs& a, const Geom& g, cudaStream_t st) {
  cudaError_t e = launch_rb("race_q_bwd", race_q_bwd_bf16_kernel<D, T>, RBSmem<D, T>::bytes, T, a, g, st);
  if (e != cudaSuccess) return e;
  return launch_rb("race_k_bwd", race_k_bwd_bf16_kernel<D, T>, RBSmem<D, T>::bytes, T, a, g, st);
}

cudaError_t launch_race_bwd_bf16(const BwdArgs& a, const Geom& g, cudaStream_t st) {
  if (g.d == 64 && g.T == 64) return race_bwd_t<64, 64>(a, g, st);
  if (g.d == 64 && g.T == 128) return race_bwd_t<64, 128>(a, g, st);
  if (g.d == 128 && g.T == 64) return race_bwd_t<128, 64>(a, g, st);
  if (g.d == 128 && g.T == 128) return race_bwd_t<128, 128>(a, g, st);
  return cudaErrorInvalidValue;
}

}  // namespace elsaa
