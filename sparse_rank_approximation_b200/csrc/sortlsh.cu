// sortLSH selector (ELSAA paper §3.2): queries and keys are hashed with angular LSH,
// sorted by hash value and grouped into equal-size blocks; query block t attends exactly
// key block t.  Rows carry a b-bit code (bit c set when x . R_c > 0), are ordered by the
// position of the code in the reflected Gray sequence (neighbouring buckets differ in one
// bit) and then by row index.
//
// Non-causal: RACE, the fusion and diagonal-block attention all commute with row
// permutations, so the selector runs the rest of the operator on row-permuted copies
// (queries by the query order, keys and values by the key order) with tile t selecting
// block t, and scatters the outputs back.
// Causal: the paper's recursion.  Every level's future-half queries meet its past-half
// keys by sorted blocks; the levels run as extra heads of the sparse kernels on gathered
// rows, and their partial softmaxes are merged by log-sum-exp before the fusion.
// This file holds the hashing and sorting, the row gathers and scatters, the selections
// and the recursion's merge and gradient collection.
#include "common.cuh"
#include "kernels.h"

namespace elsaa {

namespace {

constexpr int kSortThreads = 1024;
constexpr int kSmemSortRows = 16384;     // shared-memory sort: items packed (position << 14 | row)

__device__ __forceinline__ uint32_t gray_position(uint32_t code) {
  uint32_t n = code;
  for (uint32_t s = code >> 1; s; s >>= 1) n ^= s;
  return n;
}

}  // namespace

// Hashing: eight lanes per row, each a d/8-element slice (one or two 16-byte loads), and
// each lane hashes four rows (16 rows per warp), so every plane value read from shared
// memory serves four rows.  The planes sit there as [bits][d/8][8], so the eight slices
// of one element index fall in eight banks.  Each row's Gray position goes to `pos` (the
// sort's input) and, if asked, its code to `codes`; both [BH][2][N].
constexpr int kHashRows = 4;

template <typename E, int EPL>
__global__ void __launch_bounds__(256) sortlsh_hash_kernel(const E* __restrict__ Q, const E* __restrict__ K,
                                                           const float* __restrict__ planes, int bits,
                                                           int* __restrict__ pos, int* __restrict__ codes, Geom g) {
  extern __shared__ __align__(16) float sR[];                   // [bits][d/8][8]
  constexpr int epl = EPL;                                      // elements per lane: d / 8
  for (int i = threadIdx.x; i < bits * g.d; i += blockDim.x) {
    const int c = i / g.d, k = i % g.d;                         // plane c, element k = sub * epl + e
    const int sub = k / epl, e = k % epl;
    sR[(c * epl + e) * 8 + sub] = planes[(size_t)k * bits + c];   // planes are [d][bits]
  }
  __syncthreads();
  // blockIdx.y: the (head, side) segment; the blocks of a segment stride over its rows
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const int seg = blockIdx.y, bh = seg >> 1, side = seg & 1;
  const E* base = (side ? K : Q) + (size_t)bh * g.N * g.d + sub * epl;
  const int groups = (g.N + 4 * kHashRows - 1) / (4 * kHashRows);
  for (int grp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; grp < groups; grp += (gridDim.x * blockDim.x) >> 5) {
    int row[kHashRows];
    float v[kHashRows][epl];
#pragma unroll
    for (int m = 0; m < kHashRows; ++m) {
      row[m] = grp * 4 * kHashRows + 4 * m + (lane >> 3);
      const E* x = base + (size_t)min(row[m], g.N - 1) * g.d;
      if constexpr (sizeof(E) == 2) {
#pragma unroll
        for (int u = 0; u < epl / 8; ++u) {
          const uint4 w = *reinterpret_cast<const uint4*>(x + 8 * u);
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(h[j]);
            v[m][8 * u + 2 * j] = f.x;
            v[m][8 * u + 2 * j + 1] = f.y;
          }
        }
      } else {
#pragma unroll
        for (int u = 0; u < epl / 4; ++u) {
          const float4 w = *reinterpret_cast<const float4*>(x + 4 * u);
          v[m][4 * u] = w.x; v[m][4 * u + 1] = w.y; v[m][4 * u + 2] = w.z; v[m][4 * u + 3] = w.w;
        }
      }
    }
    uint32_t code[kHashRows] = {};
    for (int c = 0; c < bits; ++c) {
      const float* pc = sR + c * epl * 8 + sub;
      float acc[kHashRows] = {};
#pragma unroll
      for (int e = 0; e < epl; ++e) {
        const float w = pc[e * 8];
#pragma unroll
        for (int m = 0; m < kHashRows; ++m) acc[m] = fmaf(v[m][e], w, acc[m]);
      }
#pragma unroll
      for (int m = 0; m < kHashRows; ++m) {
        float t = acc[m];
        t += __shfl_xor_sync(0xffffffffu, t, 1);
        t += __shfl_xor_sync(0xffffffffu, t, 2);
        t += __shfl_xor_sync(0xffffffffu, t, 4);
        code[m] |= (t > 0.f ? 1u : 0u) << c;
      }
    }
    if (sub == 0) {
#pragma unroll
      for (int m = 0; m < kHashRows; ++m) {
        if (row[m] >= g.N) continue;
        pos[(size_t)seg * g.N + row[m]] = (int)gray_position(code[m]);
        if (codes) codes[(size_t)seg * g.N + row[m]] = (int)code[m];
      }
    }
  }
}

// Stable sort of n items by Gray position, in shared memory: least-significant digit
// first, 8 bits per pass, each pass a counting sort.  Items are packed
// (position << 14 | local row), so n <= 16384.  Warp w owns the rows of the w-th
// contiguous slice; counts are kept per (digit, warp) and scanned digit-major,
// warp-minor, and within a warp equal digits are ranked by lane (match_any), which
// keeps every pass stable.  `bufA` holds the items on entry; returns the buffer that
// holds them sorted.  Called by all kSortThreads threads.
__device__ uint32_t* block_counting_sort(uint32_t* bufA, uint32_t* bufB, int* cnt, int* wsum, int n, int bits) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slice = (n + 31) / 32;
  const int r0 = warp * slice, r1 = min(n, r0 + slice);
  uint32_t* src = bufA;
  uint32_t* dst = bufB;
  for (int shift = 0; shift < bits; shift += 8) {
    for (int i = tid; i < 256 * 32; i += kSortThreads) cnt[i] = 0;
    __syncthreads();
    // 1: per-warp digit counts
    for (int base = r0; base < r1; base += 32) {
      const int i = base + lane;
      const bool live = i < r1;
      const uint32_t dig = live ? (src[i] >> (14 + shift)) & 255u : 256u + lane;
      const unsigned peers = __match_any_sync(0xffffffffu, dig);
      if (live && lane == __ffs(peers) - 1) cnt[dig * 32 + warp] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
    // 2: exclusive scan over (digit, warp); thread t owns entries 8t .. 8t + 7
    {
      int loc[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        loc[j] = cnt[8 * tid + j];
        sum += loc[j];
      }
      int inc = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
      }
      if (lane == 31) wsum[warp] = inc;
      __syncthreads();
      if (warp == 0) {
        int w = wsum[lane], wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, wi, o);
          if (lane >= o) wi += t;
        }
        wsum[lane] = wi - w;
      }
      __syncthreads();
      int run = wsum[warp] + inc - sum;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[8 * tid + j] = run;
        run += loc[j];
      }
    }
    __syncthreads();
    // 3: stable scatter, each warp through its slice in row order
    for (int base = r0; base < r1; base += 32) {
      const int i = base + lane;
      const bool live = i < r1;
      const uint32_t item = live ? src[i] : 0u;
      const uint32_t dig = live ? (item >> (14 + shift)) & 255u : 256u + lane;
      const unsigned peers = __match_any_sync(0xffffffffu, dig);
      if (live) {
        const int at = cnt[dig * 32 + warp] + __popc(peers & ((1u << lane) - 1u));
        dst[at] = item;
      }
      __syncwarp();
      if (live && lane == __ffs(peers) - 1) cnt[dig * 32 + warp] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
    uint32_t* t = src;
    src = dst;
    dst = t;
  }
  return src;
}

// The same stable LSD counting sort for segments longer than shared memory holds
// (n > kSmemSortRows): the rows move between two global buffers, 8 bits per pass; the
// per-(digit, warp) counts stay in shared memory, scanned digit-major, warp-minor, and
// equal digits within a warp are ranked by lane, so every pass is stable.  pos holds the
// positions of the segment's rows (indexed from 0); the last pass writes first + row to
// out and, if inv is not null, the sorted position first + at of every row to
// inv[first + row].  tmp holds n ints.  Called by all kSortThreads threads.
__device__ void global_counting_sort(const int* __restrict__ pos, int* __restrict__ tmp, int* __restrict__ out,
                                     int* __restrict__ inv, int first, int n, int bits, int* cnt, int* wsum) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slice = (n + 31) / 32;
  const int r0 = warp * slice, r1 = min(n, r0 + slice);
  const int passes = (bits + 7) / 8;
  for (int p = 0; p < passes; ++p) {
    const int shift = 8 * p;
    const bool last = p == passes - 1;
    const int* src = p == 0 ? nullptr : tmp;          // pass 0 reads the rows in order
    int* dst = last ? nullptr : tmp;                  // (2 passes: rows -> tmp -> out)
    for (int i = tid; i < 256 * 32; i += kSortThreads) cnt[i] = 0;
    __syncthreads();
    for (int base = r0; base < r1; base += 32) {
      const int i = base + lane;
      const bool live = i < r1;
      const int r = live ? (src ? src[i] : i) : 0;
      const uint32_t dig = live ? ((uint32_t)pos[r] >> shift) & 255u : 256u + lane;
      const unsigned peers = __match_any_sync(0xffffffffu, dig);
      if (live && lane == __ffs(peers) - 1) cnt[dig * 32 + warp] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
    {
      int loc[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        loc[j] = cnt[8 * tid + j];
        sum += loc[j];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      if (lane == 31) wsum[warp] = incl;
      __syncthreads();
      if (warp == 0) {
        int w = wsum[lane], wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, wi, o);
          if (lane >= o) wi += t;
        }
        wsum[lane] = wi - w;
      }
      __syncthreads();
      int run = wsum[warp] + incl - sum;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[8 * tid + j] = run;
        run += loc[j];
      }
    }
    __syncthreads();
    for (int base = r0; base < r1; base += 32) {
      const int i = base + lane;
      const bool live = i < r1;
      const int r = live ? (src ? src[i] : i) : 0;
      const uint32_t dig = live ? ((uint32_t)pos[r] >> shift) & 255u : 256u + lane;
      const unsigned peers = __match_any_sync(0xffffffffu, dig);
      if (live) {
        const int at = cnt[dig * 32 + warp] + __popc(peers & ((1u << lane) - 1u));
        if (last) {
          out[at] = first + r;
          if (inv) inv[first + r] = first + at;
        } else {
          dst[at] = r;
        }
      }
      __syncwarp();
      if (live && lane == __ffs(peers) - 1) cnt[dig * 32 + warp] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
  }
}

// Long heads (N > kSmemSortRows), grid (BH, 2): positions from `pos` ([BH][2][N]), the sorted
// rows into `order`; tmp ([BH][2][N]) holds the pass in between.
__global__ void __launch_bounds__(kSortThreads) sortlsh_sort_global_kernel(const int* __restrict__ pos,
                                                                           int* __restrict__ order,
                                                                           int* __restrict__ tmp, int bits, Geom g) {
  __shared__ int cnt[256 * 32];
  __shared__ int wsum[32];
  const size_t off = ((size_t)blockIdx.x * 2 + blockIdx.y) * g.N;
  global_counting_sort(pos + off, tmp + off, order + off, nullptr, 0, g.N, bits, cnt, wsum);
}

// One (head, side) per CTA, grid (BH, 2): reads its `order` segment (the Gray
// positions) whole, then writes the sorted rows over it.
__global__ void __launch_bounds__(kSortThreads) sortlsh_sort_kernel(int* __restrict__ order, int bits, Geom g) {
  extern __shared__ __align__(16) unsigned char smem[];
  int* cnt = reinterpret_cast<int*>(smem);                          // [256 digits][32 warps]
  uint32_t* bufA = reinterpret_cast<uint32_t*>(cnt + 256 * 32);
  uint32_t* bufB = bufA + g.N;
  __shared__ int wsum[32];
  int* seg = order + ((size_t)blockIdx.x * 2 + blockIdx.y) * g.N;
  for (int i = threadIdx.x; i < g.N; i += kSortThreads) bufA[i] = ((uint32_t)seg[i] << 14) | (uint32_t)i;
  const uint32_t* out = block_counting_sort(bufA, bufB, cnt, wsum, g.N, bits);
  for (int i = threadIdx.x; i < g.N; i += kSortThreads) seg[i] = (int)(out[i] & 0x3fffu);
}

// Causal recursion, one level: rows are cut into half-segments of h rows (a past half
// 2s and a future half 2s + 1 per segment).  grid (BH, 2, N / 2h): side 0 sorts the
// queries of future half 2s + 1, side 1 the keys of past half 2s, by Gray position
// (stable); the other half of each side's order is the identity.  pos and order are
// [BH][2][N]; order holds row indices.  inv, if not null, receives for every row of a
// future half its position in the sorted query order ([BH][N]).
__global__ void __launch_bounds__(kSortThreads) sortlsh_level_sort_kernel(const int* __restrict__ pos,
                                                                          int* __restrict__ order,
                                                                          int* __restrict__ inv, int h, int bits,
                                                                          Geom g) {
  extern __shared__ __align__(16) unsigned char smem[];
  int* cnt = reinterpret_cast<int*>(smem);
  uint32_t* bufA = reinterpret_cast<uint32_t*>(cnt + 256 * 32);
  uint32_t* bufB = bufA + h;
  __shared__ int wsum[32];
  const int side = blockIdx.y, s = blockIdx.z;
  const size_t off = ((size_t)blockIdx.x * 2 + side) * g.N;
  const int sorted0 = (2 * s + (side == 0 ? 1 : 0)) * h;       // first row of the half this CTA sorts
  const int ident0 = (2 * s + (side == 0 ? 0 : 1)) * h;
  for (int i = threadIdx.x; i < h; i += kSortThreads) {
    bufA[i] = ((uint32_t)pos[off + sorted0 + i] << 14) | (uint32_t)i;
    order[off + ident0 + i] = ident0 + i;
  }
  const uint32_t* out = block_counting_sort(bufA, bufB, cnt, wsum, h, bits);
  for (int i = threadIdx.x; i < h; i += kSortThreads) {
    const int r = sorted0 + (int)(out[i] & 0x3fffu);
    order[off + sorted0 + i] = r;
    // queries: where each future-half row sits in the sorted order ([BH][N])
    if (inv && side == 0) inv[(size_t)blockIdx.x * g.N + r] = sorted0 + i;
  }
}

// The level sort for halves longer than shared memory holds (h > kSmemSortRows); tmp is
// [BH][2][N] (each CTA uses its own half's range).
__global__ void __launch_bounds__(kSortThreads) sortlsh_level_sort_global_kernel(const int* __restrict__ pos,
                                                                                 int* __restrict__ order,
                                                                                 int* __restrict__ inv,
                                                                                 int* __restrict__ tmp, int h,
                                                                                 int bits, Geom g) {
  __shared__ int cnt[256 * 32];
  __shared__ int wsum[32];
  const int side = blockIdx.y, s = blockIdx.z;
  const size_t off = ((size_t)blockIdx.x * 2 + side) * g.N;
  const int sorted0 = (2 * s + (side == 0 ? 1 : 0)) * h;
  const int ident0 = (2 * s + (side == 0 ? 0 : 1)) * h;
  for (int i = threadIdx.x; i < h; i += kSortThreads) order[off + ident0 + i] = ident0 + i;
  global_counting_sort(pos + off + sorted0, tmp + off + sorted0, order + off + sorted0,
                       inv && side == 0 ? inv + (size_t)blockIdx.x * g.N : nullptr, sorted0, h, bits, cnt, wsum);
}

// Base-pass selection of the causal recursion (the caller's row order, causal): tile t
// takes its own block and, when t is odd, block t - 1 (the deepest level, whose halves
// are single blocks and need no sort); ascending, -1 padded, k = 2.
__global__ void causal_lsh_select_kernel(int* __restrict__ idx, Geom g) {
  const size_t total = (size_t)g.BH * g.n_t;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(e % g.n_t);
    idx[2 * e] = (t & 1) ? t - 1 : t;
    idx[2 * e + 1] = (t & 1) ? t : -1;
  }
}

// Log-sum-exp merge of the recursion's sparse partials, then the fusion (Eq. 5 weight,
// Eq. 4 output) with the low-rank branch, per row.  The base pass's partial (O_s, log d_s)
// is in row order; level l's is in its sorted query order, at position inv_l[row], and
// exists for the rows of its future halves (halves of h_l = N >> (l + 1) rows).  Then
// m = 1 / (1 + (lambda d_lr + eps) e^{-log d_s}) (1 when m is held), O = g_s m O_s + g_lr O_lr
// with g_lr = 1 - m by default (1 when m is held).  Writes O, the saved fp32 O_s, log d_s
// and m.  One thread per 8 columns; partials and the merge are fp32.
constexpr int kMaxLevels = 10;            // n_t <= 1024 tiles: at most 9 sorted levels

__global__ void lsh_fuse_kernel(const float* __restrict__ Os0, const float* __restrict__ logd0,
                                const float* __restrict__ Os_lv, const float* __restrict__ logd_lv,
                                const int* __restrict__ inv_lv, int levels, const __nv_bfloat16* __restrict__ Olr,
                                const float* __restrict__ dlr, const float* lamv, const float* gsv, const float* glrv,
                                __nv_bfloat16* __restrict__ O, float* __restrict__ Os,
                                float* __restrict__ logd_out, float* __restrict__ m_out, int units_log2, Geom g) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (g.N << units_log2)) return;
  const int r = e >> units_log2, u = e & ((1 << units_log2) - 1);
  const size_t rows = (size_t)g.BH * g.N;
  const size_t row = (size_t)bh * g.N + r;
  // the partials this row has: base (slot 0), then one per level where it is in a future
  // half; first their log-denominators (and slot rows), for the common maximum
  size_t pos[kMaxLevels];
  float lg[kMaxLevels + 1];
  lg[0] = logd0[row];
#pragma unroll
  for (int l = 0; l < kMaxLevels; ++l) {
    lg[l + 1] = -INFINITY;
    pos[l] = 0;
    const int hl = 31 - __clz(g.N >> (l + 1));      // log2 of the half length
    if (l < levels && ((r >> hl) & 1)) {
      pos[l] = (size_t)l * rows + (size_t)bh * g.N + inv_lv[(size_t)l * rows + row];
      lg[l + 1] = logd_lv[pos[l]];
    }
  }
  float L = -INFINITY;
#pragma unroll
  for (int j = 0; j <= kMaxLevels; ++j) L = fmaxf(L, lg[j]);
  float sum = 0.f, s[8] = {};
  if (L > -INFINITY) {
    // then the rows, weighted by e^{log d - L} as they arrive
#pragma unroll
    for (int j = 0; j <= kMaxLevels; ++j) {
      if (lg[j] == -INFINITY) continue;
      const float wj = __expf(lg[j] - L);
      sum += wj;
      const float4* src = reinterpret_cast<const float4*>((j ? Os_lv + pos[j - 1] * g.d : Os0 + row * g.d) + 8 * u);
      const float4 w0 = src[0], w1 = src[1];
      s[0] = fmaf(wj, w0.x, s[0]); s[1] = fmaf(wj, w0.y, s[1]); s[2] = fmaf(wj, w0.z, s[2]); s[3] = fmaf(wj, w0.w, s[3]);
      s[4] = fmaf(wj, w1.x, s[4]); s[5] = fmaf(wj, w1.y, s[5]); s[6] = fmaf(wj, w1.z, s[6]); s[7] = fmaf(wj, w1.w, s[7]);
    }
    const float inv_sum = 1.f / sum;
#pragma unroll
    for (int k = 0; k < 8; ++k) s[k] *= inv_sum;
    L += __logf(sum);
  }
  const float lam = lamv ? lamv[row] : g.lam;
  const float gs = gsv ? gsv[row] : 1.f;
  const float mf = g.fixed_m ? 1.f : L == -INFINITY ? 0.f : 1.f / (1.f + (lam * dlr[row] + g.eps) * __expf(-L));
  const float gl = glrv ? glrv[row] : g.fixed_m ? 1.f : 1.f - mf;
  const float cs = gs * mf;
  const uint4 wl = *reinterpret_cast<const uint4*>(Olr + row * g.d + 8 * u);
  const __nv_bfloat162* lv = reinterpret_cast<const __nv_bfloat162*>(&wl);
  uint32_t wo[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(lv[j]);
    const __nv_bfloat162 o = __floats2bfloat162_rn(cs * s[2 * j] + gl * f.x, cs * s[2 * j + 1] + gl * f.y);
    wo[j] = *reinterpret_cast<const uint32_t*>(&o);
  }
  *reinterpret_cast<uint4*>(O + row * g.d + 8 * u) = make_uint4(wo[0], wo[1], wo[2], wo[3]);
  reinterpret_cast<float4*>(Os + row * g.d + 8 * u)[0] = make_float4(s[0], s[1], s[2], s[3]);
  reinterpret_cast<float4*>(Os + row * g.d + 8 * u)[1] = make_float4(s[4], s[5], s[6], s[7]);
  if (u == 0) {
    logd_out[row] = L;
    m_out[row] = mf;
  }
}

// Inverse of every level's two orders: inv[l][bh][side][order[l][bh][side][p]] = p.
__global__ void lsh_invert_orders_kernel(const int* __restrict__ order, int* __restrict__ inv, size_t total, int N) {
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const size_t seg = e / N;
    inv[seg * N + order[e]] = (int)(e % N);
  }
}

// The recursion's sparse gradient parts, per row of the caller's order: acc[row] += the
// sum over the levels where the row is in a future half (queries: want = 1) or a past
// half (keys: want = 0) of src_l at the row's sorted position.  Up to two tensors (dK
// and dV) share the key side's positions.  src slots are fp32 [levels][BH][N][d]; inv
// [levels][BH][2][N].
__global__ void lsh_collect_kernel(const float* __restrict__ src0, float* __restrict__ acc0,
                                   const float* __restrict__ src1, float* __restrict__ acc1,
                                   const int* __restrict__ inv, int levels, int side, int want, int units_log2,
                                   Geom g) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (g.N << units_log2)) return;
  const int r = e >> units_log2, u = e & ((1 << units_log2) - 1);
  const size_t rows = (size_t)g.BH * g.N;
  const size_t row = (size_t)bh * g.N + r;
  float s0[8] = {}, s1[8] = {};
  bool any = false;
  // every level's slot row is loaded as soon as its position is known (predicated, unrolled)
#pragma unroll
  for (int l = 0; l < kMaxLevels; ++l) {
    const int hl = 31 - __clz(g.N >> (l + 1));      // log2 of the half length
    if (l < levels && ((r >> hl) & 1) == want) {
      any = true;
      const size_t p = (size_t)l * rows + (size_t)bh * g.N + inv[(((size_t)l * g.BH + bh) * 2 + side) * g.N + r];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t == 1 && !src1) break;
        const float4* w = reinterpret_cast<const float4*>((t ? src1 : src0) + p * g.d + 8 * u);
        const float4 w0 = w[0], w1 = w[1];
        float* sv = t ? s1 : s0;
        sv[0] += w0.x; sv[1] += w0.y; sv[2] += w0.z; sv[3] += w0.w;
        sv[4] += w1.x; sv[5] += w1.y; sv[6] += w1.z; sv[7] += w1.w;
      }
    }
  }
  if (!any) return;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (t == 1 && !src1) break;
    float4* a = reinterpret_cast<float4*>((t ? acc1 : acc0) + row * g.d + 8 * u);
    const float* sv = t ? s1 : s0;
    const float4 a0 = a[0], a1 = a[1];
    a[0] = make_float4(a0.x + sv[0], a0.y + sv[1], a0.z + sv[2], a0.w + sv[3]);
    a[1] = make_float4(a1.x + sv[4], a1.y + sv[5], a1.z + sv[6], a1.w + sv[7]);
  }
}

// Every level's sorted rows, gathered into level slots: for level l (halves of
// h_l = N >> (l + 1) rows; its orders at perm + l BH 2N, one side of [BH][2][N]),
// dst_t[l][bh][p] = src_t[bh][perm_l[p]] for up to four tensors, 16-byte units; half >= 0
// moves only the positions in the past (0) or future (1) halves.
struct RowMoves {
  const uint4* src[4];
  uint4* dst[4];
  int n;
};

// One level-major virtual head per blockIdx.y (level l, head bh); x covers the rows it moves
// (with half >= 0 only the rows of that half of each length-(N >> (l + 1)) pair of halves,
// taken in order) times their 16-byte units.  N and the unit count are powers of two.
__global__ void gather_rows_kernel(RowMoves mv, const int* __restrict__ perm, int units_log2, int half, Geom g) {
  const int vh = blockIdx.y;
  const int l = vh / g.BH, bh = vh - l * g.BH;
  const int nrows = half >= 0 ? g.N >> 1 : g.N;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (nrows << units_log2)) return;
  const int c = e >> units_log2, u = e & ((1 << units_log2) - 1);
  int r = c;
  if (half >= 0) {
    const int hl = 31 - __clz(g.N >> (l + 1));      // log2 of the half length
    r = ((c >> hl) << (hl + 1)) | (half << hl) | (c & ((1 << hl) - 1));
  }
  const size_t pr = (size_t)bh * g.N + perm[((size_t)l * g.BH + bh) * 2 * g.N + r];
  const size_t row = (size_t)vh * g.N + r;         // slot row: [levels][BH][N]
  const size_t units = (size_t)1 << units_log2;
#pragma unroll
  for (int t = 0; t < 4; ++t)
    if (t < mv.n) mv.dst[t][row * units + u] = mv.src[t][pr * units + u];
}

// Every level's selection and future tiles (halves of hb_l = n_t >> (l + 1) blocks): idx
// [levels][BH][n_t] (a future tile takes the block hb_l before it, a past tile none) and
// tile_list [levels][BH][n_t / 2] (the future tiles, in block order).
__global__ void causal_lsh_select_levels_kernel(int* __restrict__ idx, int* __restrict__ tile_list, int levels,
                                                Geom g) {
  const size_t total = (size_t)levels * g.BH * g.n_t;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const size_t vh = e / g.n_t;                      // level-major virtual head
    const int l = (int)(vh / g.BH), t = (int)(e % g.n_t);
    const int hb = g.n_t >> (l + 1);
    const bool future = (t / hb) & 1;
    idx[e] = future ? t - hb : -1;
    if (future) tile_list[vh * (g.n_t / 2) + (t / (2 * hb)) * hb + (t % hb)] = t;
  }
}

// Rows of 16-byte units: dst[r] = src[perm[r]] (gather) or dst[perm[r]] = src[r]
// (scatter), for `rows_per_head` rows of `units` 16-byte units per head.
__global__ void permute_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                    const int* __restrict__ perm, int rows_per_head, int units, int BH,
                                    int perm_stride, int scatter) {
  const size_t total = (size_t)BH * rows_per_head * units;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const size_t row = e / units;
    const int u = (int)(e % units);
    const int bh = (int)(row / rows_per_head), r = (int)(row % rows_per_head);
    const size_t pr = (size_t)bh * rows_per_head + perm[(size_t)bh * perm_stride + r];
    if (scatter)
      dst[pr * units + u] = src[row * units + u];
    else
      dst[row * units + u] = src[pr * units + u];
  }
}

// Per-row float32 vectors (lambda, gates): dst[r] = src[perm[r]].
__global__ void gather_vec_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                  const int* __restrict__ perm, int N, int BH, int perm_stride) {
  const size_t total = (size_t)BH * N;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const int bh = (int)(e / N), r = (int)(e % N);
    dst[e] = src[(size_t)bh * N + perm[(size_t)bh * perm_stride + r]];
  }
}

// Tile t selects block t (the diagonal of the permuted score matrix).
__global__ void diag_select_kernel(int* __restrict__ idx, Geom g) {
  const size_t total = (size_t)g.BH * g.n_t;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    int* row = idx + e * g.k;
    row[0] = (int)(e % g.n_t);
    for (int c = 1; c < g.k; ++c) row[c] = -1;
  }
}

size_t sortlsh_smem_bytes(const Geom& g, int bits) {
  (void)bits;
  return (size_t)256 * 32 * 4 + (size_t)2 * g.N * 4;
}

size_t sortlsh_scratch_ints(const Geom& g) {
  if (g.lsh_bits == 0) return 0;                  // not the sortLSH selector
  // non-causal: positions and the pass buffer of the whole heads; causal: the pass buffer of
  // the level sorts (their positions are computed once into the workspace)
  if (!g.causal) return g.N > kSmemSortRows ? (size_t)2 * g.BH * 2 * g.N : 0;
  return g.N / 2 > kSmemSortRows ? (size_t)g.BH * 2 * g.N : 0;
}

cudaError_t launch_sortlsh_hash(const void* Q, const void* K, bool bf16, const float* planes, int bits, int* pos,
                                int* codes, const Geom& g, cudaStream_t st) {
  const size_t hsmem = (size_t)bits * g.d * 4;
  const int per_seg_max = (g.N + 8 * 4 * kHashRows - 1) / (8 * 4 * kHashRows);   // one iteration each
  const int per_seg = std::max(1, std::min(per_seg_max, (148 * 8 + 2 * g.BH - 1) / (2 * g.BH)));
  const dim3 hgrid(per_seg, 2 * g.BH);
  ProfScope ps("sortlsh_hash", st);
  auto run = [&](auto kern, const auto* q, const auto* k) {
    kern<<<hgrid, 256, hsmem, st>>>(q, k, planes, bits, pos, codes, g);
  };
  const auto* q16 = (const __nv_bfloat16*)Q;
  const auto* k16 = (const __nv_bfloat16*)K;
  const auto* q32 = (const float*)Q;
  const auto* k32 = (const float*)K;
  if (bf16 && g.d == 128) run(sortlsh_hash_kernel<__nv_bfloat16, 16>, q16, k16);
  else if (bf16) run(sortlsh_hash_kernel<__nv_bfloat16, 8>, q16, k16);
  else if (g.d == 128) run(sortlsh_hash_kernel<float, 16>, q32, k32);
  else run(sortlsh_hash_kernel<float, 8>, q32, k32);
  return cudaGetLastError();
}

cudaError_t launch_sortlsh_level_sort(const int* pos, int* order, int* inv, int h, int bits, int* scratch,
                                      const Geom& g, cudaStream_t st) {
  if (h > kSmemSortRows) {
    if (!scratch) return cudaErrorInvalidValue;
    ProfScope ps("sortlsh_level_sort", st);
    sortlsh_level_sort_global_kernel<<<dim3(g.BH, 2, g.N / (2 * h)), kSortThreads, 0, st>>>(pos, order, inv, scratch,
                                                                                            h, bits, g);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)256 * 32 * 4 + (size_t)2 * h * 4;
  cudaError_t e = cudaFuncSetAttribute(sortlsh_level_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps("sortlsh_level_sort", st);
  sortlsh_level_sort_kernel<<<dim3(g.BH, 2, g.N / (2 * h)), kSortThreads, smem, st>>>(pos, order, inv, h, bits, g);
  return cudaGetLastError();
}

static int elementwise_blocks(size_t total) { return (int)std::min<size_t>((total + 255) / 256, 148 * 16); }

cudaError_t launch_causal_lsh_select(int* idx, const Geom& g, cudaStream_t st) {
  causal_lsh_select_kernel<<<elementwise_blocks((size_t)g.BH * g.n_t), 256, 0, st>>>(idx, g);
  return cudaGetLastError();
}

cudaError_t launch_lsh_fuse(const void* Os0, const float* logd0, const void* Os_lv, const float* logd_lv,
                            const int* inv_lv, int levels, const void* Olr, const float* dlr, const float* lam,
                            const float* gs, const float* glr, void* O, void* Os, float* logd, float* m, const Geom& g,
                            cudaStream_t st) {
  if (levels > kMaxLevels) return cudaErrorInvalidValue;
  const int units = g.d / 8;
  if ((units & (units - 1)) || (g.N & (g.N - 1)) || g.BH > 65535) return cudaErrorInvalidValue;
  const int units_log2 = 31 - __builtin_clz((unsigned)units);
  ProfScope ps("lsh_fuse", st);
  lsh_fuse_kernel<<<dim3((unsigned)(((size_t)g.N * units + 255) / 256), g.BH), 256, 0, st>>>(
      (const float*)Os0, logd0, (const float*)Os_lv, logd_lv, inv_lv, levels,
      (const __nv_bfloat16*)Olr, dlr, lam, gs, glr, (__nv_bfloat16*)O, (float*)Os, logd, m, units_log2, g);
  return cudaGetLastError();
}

cudaError_t launch_lsh_invert_orders(const int* order, int* inv, int levels, const Geom& g, cudaStream_t st) {
  const size_t total = (size_t)levels * g.BH * 2 * g.N;
  lsh_invert_orders_kernel<<<elementwise_blocks(total), 256, 0, st>>>(order, inv, total, g.N);
  return cudaGetLastError();
}

cudaError_t launch_lsh_collect(const void* src0, float* acc0, const void* src1, float* acc1, const int* inv,
                               int levels, bool keys, const Geom& g, cudaStream_t st) {
  if (levels > kMaxLevels) return cudaErrorInvalidValue;
  const int units = g.d / 8;
  if ((units & (units - 1)) || (g.N & (g.N - 1)) || g.BH > 65535) return cudaErrorInvalidValue;
  const int units_log2 = 31 - __builtin_clz((unsigned)units);
  ProfScope ps("lsh_collect", st);
  lsh_collect_kernel<<<dim3((unsigned)(((size_t)g.N * units + 255) / 256), g.BH), 256, 0, st>>>(
      (const float*)src0, acc0, (const float*)src1, acc1, inv, levels, keys ? 1 : 0, keys ? 0 : 1, units_log2, g);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* const* src, void* const* dst, int n, const int* perm, int row_bytes,
                               int levels, int half, const Geom& g, cudaStream_t st) {
  if (n < 1 || n > 4) return cudaErrorInvalidValue;
  RowMoves mv{};
  for (int t = 0; t < n; ++t) {
    mv.src[t] = (const uint4*)src[t];
    mv.dst[t] = (uint4*)dst[t];
  }
  mv.n = n;
  const int units = row_bytes / 16;
  if (units < 1 || (units & (units - 1)) || (g.N & (g.N - 1)) || levels < 1 || (size_t)levels * g.BH > 65535)
    return cudaErrorInvalidValue;
  const int units_log2 = 31 - __builtin_clz((unsigned)units);
  const int nrows = half >= 0 ? g.N / 2 : g.N;
  ProfScope ps("sortlsh_gather", st);
  gather_rows_kernel<<<dim3((unsigned)(((size_t)nrows * units + 255) / 256), levels * g.BH), 256, 0, st>>>(
      mv, perm, units_log2, half, g);
  return cudaGetLastError();
}

cudaError_t launch_causal_lsh_select_levels(int* idx, int* tile_list, int levels, const Geom& g, cudaStream_t st) {
  causal_lsh_select_levels_kernel<<<elementwise_blocks((size_t)levels * g.BH * g.n_t), 256, 0, st>>>(idx, tile_list,
                                                                                                     levels, g);
  return cudaGetLastError();
}

cudaError_t launch_sortlsh_order(const void* Q, const void* K, bool bf16, const float* planes, int bits,
                                 int* order, int* codes, int* scratch, const Geom& g, cudaStream_t st) {
  if (g.N > kSmemSortRows) {
    // long heads: positions into scratch, the sort through global memory
    if (!scratch) return cudaErrorInvalidValue;
    int* pos = scratch;
    int* tmp = scratch + (size_t)g.BH * 2 * g.N;
    const cudaError_t eh = launch_sortlsh_hash(Q, K, bf16, planes, bits, pos, codes, g, st);
    if (eh != cudaSuccess) return eh;
    ProfScope ps("sortlsh_sort", st);
    sortlsh_sort_global_kernel<<<dim3(g.BH, 2), kSortThreads, 0, st>>>(pos, order, tmp, bits, g);
    return cudaGetLastError();
  }
  const cudaError_t eh = launch_sortlsh_hash(Q, K, bf16, planes, bits, order, codes, g, st);
  if (eh != cudaSuccess) return eh;
  const size_t smem = sortlsh_smem_bytes(g, bits);
  cudaError_t e = cudaFuncSetAttribute(sortlsh_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps("sortlsh_sort", st);
  sortlsh_sort_kernel<<<dim3(g.BH, 2), kSortThreads, smem, st>>>(order, bits, g);
  return cudaGetLastError();
}

cudaError_t launch_permute_rows(const void* src, void* dst, const int* perm, int row_bytes, const Geom& g,
                                int perm_stride, bool scatter, cudaStream_t st) {
  const int units = row_bytes / 16;
  const size_t total = (size_t)g.BH * g.N * units;
  const int blocks = (int)std::min<size_t>((total + 255) / 256, 148 * 16);
  ProfScope ps(scatter ? "sortlsh_scatter" : "sortlsh_gather", st);
  permute_rows_kernel<<<blocks, 256, 0, st>>>((const uint4*)src, (uint4*)dst, perm, g.N, units, g.BH, perm_stride,
                                             scatter ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_gather_vec(const float* src, float* dst, const int* perm, const Geom& g, int perm_stride,
                              cudaStream_t st) {
  const size_t total = (size_t)g.BH * g.N;
  const int blocks = (int)std::min<size_t>((total + 255) / 256, 148 * 8);
  gather_vec_kernel<<<blocks, 256, 0, st>>>(src, dst, perm, g.N, g.BH, perm_stride);
  return cudaGetLastError();
}

cudaError_t launch_diag_select(int* idx, const Geom& g, cudaStream_t st) {
  const size_t total = (size_t)g.BH * g.n_t;
  diag_select_kernel<<<(int)std::min<size_t>((total + 255) / 256, 1024), 256, 0, st>>>(idx, g);
  return cudaGetLastError();
}

}  // namespace elsaa
