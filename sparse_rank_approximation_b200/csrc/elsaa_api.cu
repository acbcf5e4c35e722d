// C ABI of libelsaa.so: argument validation, the layout of the caller-owned
// `saved` and `workspace` buffers, and the launch sequence of the forward and
// backward passes.  The operator is defined in include/elsaa.h.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/elsaa.h"
#include "kernels.h"

using namespace elsaa;

namespace {

thread_local std::string g_last_error;

// test hook (elsaa_debug_set_wait_limit): pipeline-wait limit and the forward stall
std::atomic<unsigned long long> g_wait_ns{0};
std::atomic<int> g_debug_stall{0};
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;

elsaa_status fail(elsaa_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
elsaa_status fail(elsaa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Sequential sub-allocator over a caller buffer (or a null base to measure).
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    off = align_up(off);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

bool tc_race(const Geom& g, bool bf16);

bool make_geom(const elsaa_params* p, Geom* g, elsaa_status* st) {
  *st = ELSAA_OK;
  if (!p) { *st = fail(ELSAA_ERR_INVALID_ARG, "params is NULL"); return false; }
  if (p->B < 1 || p->H < 1 || p->N < 1) {
    *st = fail(ELSAA_ERR_INVALID_ARG, "B, H, N must be >= 1 (got %d, %d, %d)", p->B, p->H, p->N);
    return false;
  }
  if (p->dtype != ELSAA_DTYPE_F32 && p->dtype != ELSAA_DTYPE_BF16) {
    *st = fail(ELSAA_ERR_INVALID_ARG, "dtype %d is not an elsaa_dtype", p->dtype);
    return false;
  }
  if (p->causal != 0 && p->causal != 1) { *st = fail(ELSAA_ERR_INVALID_ARG, "causal must be 0 or 1"); return false; }
  if (!(std::isfinite(p->scale) && std::isfinite(p->lambda) && std::isfinite(p->eps) && p->eps >= 0.f &&
        std::isfinite(p->tau) && p->tau > 0.f)) {
    *st = fail(ELSAA_ERR_INVALID_ARG, "scale/lambda must be finite, eps >= 0, tau > 0");
    return false;
  }
  if (p->hash_bits != kHashBits) {
    *st = fail(ELSAA_ERR_UNSUPPORTED, "hash_bits %d unsupported (4 only)", p->hash_bits);
    return false;
  }
  if (p->rank_r < 0 || p->rank_r > 256 || p->rank_r % 16) {
    *st = fail(ELSAA_ERR_UNSUPPORTED, "rank_r %d unsupported (multiple of 16 in [0, 256])", p->rank_r);
    return false;
  }
  if (p->d != 64 && p->d != 128) { *st = fail(ELSAA_ERR_UNSUPPORTED, "d %d unsupported (64 or 128)", p->d); return false; }
  const bool bf16 = p->dtype == ELSAA_DTYPE_BF16;
  const int T = p->block_size;
  if (bf16 ? (T != 64 && T != 128) : (T != 1 && T != 64 && T != 128)) {
    *st = fail(ELSAA_ERR_UNSUPPORTED, "block_size %d unsupported for %s", T, bf16 ? "bf16 (64, 128)" : "f32 (1, 64, 128)");
    return false;
  }
  if (T == 1 && p->N > 4096) {
    *st = fail(ELSAA_ERR_UNSUPPORTED, "block_size 1 needs N <= 4096 (got %d)", p->N);
    return false;
  }
  const int n_t = (p->N + T - 1) / T;
  if (n_t > 1024) { *st = fail(ELSAA_ERR_UNSUPPORTED, "ceil(N / block_size) = %d > 1024", n_t); return false; }
  if (p->selector != ELSAA_SEL_TOPK_BLOCKS && p->selector != ELSAA_SEL_SORTLSH) {
    *st = fail(ELSAA_ERR_INVALID_ARG, "selector %d is not an elsaa_selector", p->selector);
    return false;
  }
  const bool lsh = p->selector == ELSAA_SEL_SORTLSH;
  int lsh_levels = 0;
  if (lsh) {
    if (T == 1) { *st = fail(ELSAA_ERR_UNSUPPORTED, "sortLSH needs block_size 64 or 128"); return false; }
    if (p->lsh_bits < 1 || p->lsh_bits > 16) {
      *st = fail(ELSAA_ERR_INVALID_ARG, "lsh_bits %d outside [1, 16]", p->lsh_bits);
      return false;
    }
    if (p->causal) {
      // the recursion runs on the bf16 tensor-core sparse kernels, halving down
      // to single blocks
      if (!bf16) {
        *st = fail(ELSAA_ERR_UNSUPPORTED, "causal sortLSH needs bf16");
        return false;
      }
      if (p->N % T || (n_t & (n_t - 1))) {
        *st = fail(ELSAA_ERR_UNSUPPORTED, "causal sortLSH needs N = block_size * 2^L (got N = %d)", p->N);
        return false;
      }
      while ((2 << lsh_levels) < n_t) ++lsh_levels;               // log2(n_t) - 1 sorted levels
    }
    if ((long)p->B * p->H > 32767) { *st = fail(ELSAA_ERR_UNSUPPORTED, "sortLSH: B * H <= 32767"); return false; }
  }
  if (!lsh && (p->topk < 0 || p->topk > n_t)) {
    *st = fail(ELSAA_ERR_INVALID_ARG, "topk %d outside [0, %d]", p->topk, n_t);
    return false;
  }
  g->BH = p->B * p->H;
  g->N = p->N;
  g->d = p->d;
  g->T = T;
  g->n_t = n_t;
  // sortLSH: tile t selects block t of the sorted orders; causal: the base pass takes the
  // tile's own block and, for odd t, block t - 1
  g->k = lsh ? (p->causal ? 2 : 1) : p->topk;
  g->r = p->rank_r;
  g->L = p->rank_r >> kHashBits;
  // RACE chunk length: 128 rows on the bf16 (tensor-core) path whatever the block size, 64 on the
  // fp32 path (the result does not depend on it)
  g->C = bf16 ? 128 : 64;
  g->n_c = (p->N + g->C - 1) / g->C;
  long want = ((long)g->BH * g->n_c + 295) / 296;   // about two segments per SM
  g->seg = (int)std::max(1L, std::min(16L, want));
  g->n_seg = (g->n_c + g->seg - 1) / g->seg;
  g->dp = p->d + 8;
  g->causal = p->causal;
  g->fixed_m = p->fixed_m != 0;
  g->selector = p->selector;
  g->lsh_bits = lsh ? p->lsh_bits : 0;
  g->lsh_levels = lsh_levels;
  g->scale = p->scale;
  g->lam = p->lambda;
  g->eps = p->eps;
  g->tau = p->tau;
  g->rp = g->r;
  g->G = 1;
  if (tc_race(*g, bf16)) {          // decided by dtype and r alone: the shape checks above admit
                                     // only shapes the tensor-core RACE kernels take
    // the tensor-core RACE kernels take the features in groups of 128 (8 tables), zero-padded
    g->G = (g->r + 127) / 128;
    g->rp = 128 * g->G;
    // the tensor-core statistics walk a segment per CTA, one CTA per SM: about one wave
    const int per_head = std::max(1, 148 / g->BH);
    g->seg = std::max(1, (g->n_c + per_head - 1) / per_head);
    g->n_seg = (g->n_c + g->seg - 1) / g->seg;
  }
  const unsigned long long wn = g_wait_ns.load();
  g->wait_ns = wn ? wn : kDefaultWaitNs;
  g->debug_stall = g_debug_stall.load();
  return true;
}

// The tensor-core RACE path (statistics, read-out, backward): every bf16 problem with a low-rank
// branch (d = 64 or 128, chunks of 128 rows, r up to 256 in groups of 128 features).  The
// launchers check the geometry (race_bwd_tc_supported) and refuse anything else.
bool tc_race(const Geom& g, bool bf16) { return bf16 && g.r > 0; }

struct Saved {
  int* idx;
  float *logd, *dlr, *m;
  void *Os, *Olr;
  void *phiQ, *phiK;
  float *hQ, *hK, *nQ, *nK;
  float *Ast, *Bst;
  void* Psplit;
  float* Pmass;
  int* lsh_order;          // sortLSH: sorted query and key orders [BH][2][N] (causal: one per level)
  // sortLSH: the rows the operator runs on, gathered by the forward and read again by the
  // backward.  Non-causal: Q by the query order, K and V by the key order ([BH][N][d]).
  // Causal: every level's future-half queries and past-half keys and values ([levels][BH][N][d]).
  void *lvQ, *lvK, *lvV;
};

Saved carve_saved(void* base, const Geom& g, size_t esz, size_t* bytes) {
  Carver c(base);
  Saved s;
  const size_t rows = (size_t)g.BH * g.N;
  const bool split = tc_race(g, esz == 2);
  // a state holds the statistics of r features, or on the tensor-core path of one group of 128
  // (the groups run one after another and reuse it)
  const size_t state = (size_t)(split ? 128 : g.r) * g.dp;
  s.idx = c.take<int>((size_t)g.BH * g.n_t * std::max(g.k, 1));
  s.logd = c.take<float>(rows);
  s.dlr = c.take<float>(rows);
  s.m = c.take<float>(rows);
  s.Os = c.take<float>(rows * g.d);          // fp32 on every path: the backward's softmax delta reads it
  s.Olr = c.take<char>(rows * g.d * esz);
  s.phiQ = c.take<char>(rows * g.rp * esz);
  s.phiK = c.take<char>(rows * g.rp * esz);
  s.hQ = c.take<float>(rows * g.L * kHashBits);
  s.hK = c.take<float>(rows * g.L * kHashBits);
  s.nQ = c.take<float>(rows);
  s.nK = c.take<float>(rows);
  s.Ast = c.take<float>((size_t)g.BH * (g.n_seg + 1) * state);
  // the in-segment prefix is kept only by the fp32 statistics
  s.Bst = c.take<float>(g.causal && !split ? (size_t)g.BH * g.n_c * state : 0);
  s.Psplit = split ? c.take<char>((size_t)g.BH * g.n_c * 2 * g.rp * g.d * 2) : nullptr;
  s.Pmass = split ? c.take<float>((size_t)g.BH * g.n_c * g.rp) : nullptr;
  const size_t orders = g.selector != ELSAA_SEL_SORTLSH ? 0 : g.causal ? (size_t)g.lsh_levels : 1;
  s.lsh_order = orders ? c.take<int>(orders * g.BH * 2 * g.N) : nullptr;
  const size_t lv_count = g.selector != ELSAA_SEL_SORTLSH ? 0 : g.causal ? (size_t)g.lsh_levels : 1;
  const bool lv_rows = lv_count > 0;
  const size_t lv_mat = lv_count * rows * g.d * esz;
  s.lvQ = lv_rows ? c.take<char>(lv_mat) : nullptr;
  s.lvK = lv_rows ? c.take<char>(lv_mat) : nullptr;
  s.lvV = lv_rows ? c.take<char>(lv_mat) : nullptr;
  *bytes = align_up(c.off);
  return s;
}

// sortLSH: row-permuted copies of the inputs and outputs (the operator runs on them).
struct PermBufs {
  void *Q, *K, *V, *X, *dQ, *dK, *dV;     // X: O (forward) or dO (backward)
  float *lam, *gs, *glr;
  // causal recursion: every sorted level is one more block of heads ("level slots",
  // [levels][BH][N][d]).  Q, K, V (and dO, dQ, dK, dV in the backward) are slotted; idx
  // and tile_list hold every level's selection and future tiles; offs, tiles, order the
  // selection inverse over the level heads.  Forward: the base pass's O_s, log d_s (X is
  // its scratch output), the levels' partial O_s and log d_s, the future rows' positions
  // inv ([levels][BH][N]), the Gray positions.  Backward: the orders' inverses inv
  // ([levels][BH][2][N]) and the sorted rows' packed backward scalars.
  void *Os, *Os_lv;
  float *logd, *m, *logd_lv;
  int *idx, *tile_list, *offs, *tiles, *order, *pos, *inv;
  float4* packed;
  // the sparse-only passes' low-rank inputs: the forward kernel reads O_lr and d_lr, whose
  // contents do not matter there (m is held at 1 and the fused output is not used)
  void* Olr;
  float* dlr;
};

PermBufs carve_perm(Carver& c, const Geom& g, size_t esz, bool backward) {
  PermBufs b{};
  if (g.selector != ELSAA_SEL_SORTLSH) return b;
  const size_t rows = (size_t)g.BH * g.N, mat = rows * g.d * esz;
  if (!g.causal) {
    // (the sorted Q, K and V are kept in the saved buffer)
    b.X = c.take<char>(mat);
    if (backward) {
      b.dQ = c.take<char>(mat);
      b.dK = c.take<char>(mat);
      b.dV = c.take<char>(mat);
    }
    b.lam = c.take<float>(rows);
    b.gs = c.take<float>(rows);
    b.glr = c.take<float>(rows);
    return b;
  }
  // (the levels' gathered Q, K and V are kept in the saved buffer)
  const size_t lv = (size_t)g.lsh_levels, vheads = lv * g.BH;
  b.idx = c.take<int>(vheads * g.n_t);
  b.tile_list = c.take<int>(vheads * (g.n_t / 2));
  if (backward) {
    b.X = c.take<char>(lv * mat);
    // the level gradients stay fp32 until the base pass's single bf16 rounding
    b.dQ = c.take<float>(lv * rows * g.d);
    b.dK = c.take<float>(lv * rows * g.d);
    b.dV = c.take<float>(lv * rows * g.d);
    b.packed = c.take<float4>(lv * rows);
    b.offs = c.take<int>(vheads * (g.n_t + 1));
    b.tiles = c.take<int>(vheads * g.n_t);
    b.order = c.take<int>(vheads * g.n_t);
    b.inv = c.take<int>(lv * rows * 2);
    return b;
  }
  b.X = c.take<char>(mat);
  b.Os = c.take<float>(rows * g.d);
  b.logd = c.take<float>(rows);
  b.m = c.take<float>(std::max<size_t>(lv, 1) * rows);
  b.Olr = c.take<char>(std::max<size_t>(lv, 1) * mat);
  b.dlr = c.take<float>(std::max<size_t>(lv, 1) * rows);
  b.Os_lv = c.take<float>(lv * rows * g.d);
  b.logd_lv = c.take<float>(lv * rows);
  b.inv = c.take<int>(lv * rows);
  b.pos = c.take<int>(rows * 2);
  return b;
}

struct FwdWs {
  uint32_t* flag;
  double *qbar, *kbar;
  float* scores;
  void* wsplit;
  float *lr_num, *lr_den;
  int* lsh_scratch;        // sortLSH sorts longer than shared memory takes (else null)
  PermBufs pm;
};

FwdWs carve_fwd_ws(void* base, const Geom& g, size_t esz, size_t* bytes) {
  Carver c(base);
  FwdWs w;
  w.flag = c.take<uint32_t>(64);
  w.qbar = c.take<double>((size_t)g.BH * g.n_t * g.d);
  w.kbar = c.take<double>((size_t)g.BH * g.n_t * g.d);
  w.scores = c.take<float>((size_t)g.BH * g.n_t * g.n_t);
  w.wsplit = c.take<char>((size_t)2 * ((g.L * kHashBits + 31) & ~31) * g.d * 2);
  // tensor-core read-out over several feature groups: the running numerator and denominator
  const bool groups = g.G > 1 && tc_race(g, esz == 2);
  w.lr_num = groups ? c.take<float>((size_t)g.BH * g.N * g.d) : nullptr;
  w.lr_den = groups ? c.take<float>((size_t)g.BH * g.N) : nullptr;
  w.pm = carve_perm(c, g, esz, false);
  const size_t scr = sortlsh_scratch_ints(g);
  w.lsh_scratch = scr ? c.take<int>(scr) : nullptr;
  *bytes = align_up(c.off);
  return w;
}

struct BwdWs {
  uint32_t* flag;
  RowScalars rs;
  float *RA, *RB;
  int *offs, *tiles, *order;
  float *dQacc, *dKacc, *dVacc;
  void* dOcl;
  void *Rsplit, *Wsplit;
  float* Rmass;
  PermBufs pm;
};

BwdWs carve_bwd_ws(void* base, const Geom& g, bool bf16, size_t* bytes) {
  Carver c(base);
  BwdWs w;
  const size_t rows = (size_t)g.BH * g.N;
  const size_t state = (size_t)(tc_race(g, bf16) ? 128 : g.r) * g.dp;
  w.flag = c.take<uint32_t>(64);
  w.rs.cs = c.take<float>(rows);
  w.rs.Delta = c.take<float>(rows);
  w.rs.cl = c.take<float>(rows);
  w.rs.delta = c.take<float>(rows);
  w.rs.packed = bf16 ? c.take<float4>(rows) : nullptr;
  w.RA = c.take<float>((size_t)g.BH * (g.n_seg + 1) * state);
  w.RB = c.take<float>(g.causal && !tc_race(g, bf16) ? (size_t)g.BH * g.n_c * state : 0);
  w.offs = c.take<int>((size_t)g.BH * (g.n_t + 1));
  w.tiles = c.take<int>((size_t)g.BH * g.n_t * std::max(g.k, 1));
  w.order = c.take<int>((size_t)g.BH * g.n_t);
  const bool causal_lsh = g.selector == ELSAA_SEL_SORTLSH && g.causal;
  const size_t acc = bf16 && (g.r > 0 || causal_lsh) ? rows * g.d : 0;
  w.dQacc = acc ? c.take<float>(acc) : nullptr;
  w.dKacc = acc ? c.take<float>(acc) : nullptr;
  w.dVacc = acc ? c.take<float>(acc) : nullptr;
  w.dOcl = c.take<char>(bf16 && g.r > 0 ? rows * g.d * 2 : 0);
  const bool split = tc_race(g, bf16);
  w.Rsplit = split ? c.take<char>((size_t)g.BH * g.n_c * 2 * g.rp * g.d * 2) : nullptr;
  w.Rmass = split ? c.take<float>((size_t)g.BH * g.n_c * g.rp) : nullptr;
  w.Wsplit = split ? c.take<char>((size_t)2 * ((g.L * kHashBits + 31) & ~31) * g.d * 2) : nullptr;
  w.pm = carve_perm(c, g, bf16 ? 2 : 4, true);
  *bytes = align_up(c.off);
  return w;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

elsaa_status check_ptr(const void* p, const char* name, bool required = true) {
  if (!p) return required ? fail(ELSAA_ERR_INVALID_ARG, "%s is NULL", name) : ELSAA_OK;
  if (!aligned16(p)) return fail(ELSAA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return ELSAA_OK;
}

elsaa_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return ELSAA_OK;
  return fail(ELSAA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define ELSAA_TRY(expr)                   \
  do {                                    \
    elsaa_status _s = (expr);             \
    if (_s != ELSAA_OK) return _s;        \
  } while (0)

// ---- a second stream for the block selection --------------------------------
// The selection does not depend on the RACE branch, so a forward runs it on a second stream
// (one per host thread and device, created on first use) while the features, statistics and
// read-out run on the caller's stream; one event pair forks and joins them before the sparse
// forward.  Both are stream-ordered, so a CUDA-graph capture of the caller's stream takes the
// forked work in as well.  If the stream cannot be created, the selection stays on the caller's.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool failed = false;
};
constexpr int kMaxSideDevices = 64;
SideStream* side_stream() {
  thread_local SideStream per_dev[kMaxSideDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSideDevices) return nullptr;
  SideStream& x = per_dev[dev];
  if (!x.s && !x.failed) {
    if (cudaStreamCreateWithFlags(&x.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming) != cudaSuccess) {
      x.failed = true;
      x.s = nullptr;
      cudaGetLastError();
    }
  }
  return x.s ? &x : nullptr;
}

// Joins the selection stream back into the caller's stream exactly once: on the normal path
// before the sparse forward, or, if a launch fails after the fork, when the forward returns,
// so no work queued on the second stream outlives the call.  The join event is recorded on
// the second stream by this guard (never a record left over from an earlier call: inside a
// graph capture, a wait on an event recorded outside the capture would invalidate it).
struct JoinGuard {
  SideStream* side = nullptr;
  cudaStream_t caller = nullptr;
  bool recorded = false, done = true;
  JoinGuard() = default;
  JoinGuard(const JoinGuard&) = delete;
  JoinGuard& operator=(const JoinGuard&) = delete;
  void arm(SideStream* s, cudaStream_t c) {
    side = s;
    caller = c;
    recorded = false;
    done = false;
  }
  cudaError_t record() {
    if (done || recorded) return cudaSuccess;
    recorded = true;
    return cudaEventRecord(side->join, side->s);
  }
  cudaError_t join() {
    if (done) return cudaSuccess;
    cudaError_t e = record();
    done = true;
    return e != cudaSuccess ? e : cudaStreamWaitEvent(caller, side->join, 0);
  }
  ~JoinGuard() {
    if (join() != cudaSuccess) cudaGetLastError();
  }
};

// ---- opt-in per-kernel profiler ------------------------------------------
struct ProfRec {
  const char* name;
  int slot;
};
struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> ev;    // 2 events per slot, created on first use
  std::vector<ProfRec> recs;
  int used = 0;
};
Profiler& prof() {
  static Profiler p;
  return p;
}
constexpr int kMaxProfSlots = 16384;

}  // namespace

namespace elsaa {
void record_error(const char* msg) { g_last_error = msg; }

ProfScope::ProfScope(const char* name, cudaStream_t st) : slot(-1), stream(st) {
  Profiler& p = prof();
  if (!p.on) return;
  std::lock_guard<std::mutex> lk(p.mu);
  if (p.used >= kMaxProfSlots) return;
  const int s = p.used;
  while ((int)p.ev.size() < 2 * (s + 1)) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return;
    p.ev.push_back(e);
  }
  p.used++;
  slot = s;
  p.recs.push_back({name, s});
  cudaEventRecord(p.ev[2 * s], st);
}
ProfScope::~ProfScope() {
  if (slot < 0) return;
  cudaEventRecord(prof().ev[2 * slot + 1], stream);
}
}  // namespace elsaa

// sortLSH: gather the inputs into the sorted orders (queries by the query order, keys and values
// by the key order, per-row vectors by the query order).  The forward sorts first and gathers Q,
// K and V into the saved buffer (qkv); the backward reuses those and gathers only dO and the
// per-row vectors.
elsaa_status lsh_gather(const elsaa_params* p, const Geom& g, bool bf16, const int* order, bool forward, int* scratch,
                        const void* Q, const void* K, const void* V, const void* X, const float* lam,
                        const float* gs, const float* glr, void* const (&qkv)[3], const PermBufs& b,
                        cudaStream_t st) {
  const int row_bytes = g.d * (bf16 ? 2 : 4), stride = 2 * g.N;
  const int* oq = order;
  const int* ok = order + g.N;
  if (forward) {
    ELSAA_TRY(cuda_status(launch_sortlsh_order(Q, K, bf16, p->lsh_planes, p->lsh_bits, const_cast<int*>(order),
                                               nullptr, scratch, g, st), "sortLSH order"));
    ELSAA_TRY(cuda_status(launch_permute_rows(Q, qkv[0], oq, row_bytes, g, stride, false, st), "sortLSH gather Q"));
    ELSAA_TRY(cuda_status(launch_permute_rows(K, qkv[1], ok, row_bytes, g, stride, false, st), "sortLSH gather K"));
    ELSAA_TRY(cuda_status(launch_permute_rows(V, qkv[2], ok, row_bytes, g, stride, false, st), "sortLSH gather V"));
  }
  if (X) ELSAA_TRY(cuda_status(launch_permute_rows(X, b.X, oq, row_bytes, g, stride, false, st), "sortLSH gather dO"));
  if (lam) ELSAA_TRY(cuda_status(launch_gather_vec(lam, b.lam, oq, g, stride, st), "sortLSH gather lambda"));
  if (gs) ELSAA_TRY(cuda_status(launch_gather_vec(gs, b.gs, oq, g, stride, st), "sortLSH gather g_sparse"));
  if (glr) ELSAA_TRY(cuda_status(launch_gather_vec(glr, b.glr, oq, g, stride, st), "sortLSH gather g_lr"));
  return ELSAA_OK;
}

// ---- causal sortLSH: the recursion of the paper's §3.2 on the tensor-core kernels ----
//
// Level l (1 .. lsh_levels) cuts the rows into half-segments of h = N >> l rows; the
// future half's sorted query blocks meet the past half's sorted key blocks.  Each level
// gathers its sorted rows, runs the sparse kernel alone (no low-rank branch, m held at 1,
// so its O_s and log d_s are the level's exact partial softmax) and merges that into the
// running result by log-sum-exp.  The deepest level (halves of one block) needs no sort:
// it joins the leaves in the base pass, tile t taking block t under the mask j <= i and,
// for odd t, block t - 1.  The fusion then runs on the merged sparse branch.  In the
// backward every level's sparse gradient uses the merged log d_s and Delta, so the levels
// are independent: each one's dQ, dK, dV (sorted order) are added to the fp32
// accumulators that the base pass folds into its single bf16 rounding.

Geom sparse_only(const Geom& g, bool causal, int k) {
  Geom s = g;
  s.r = 0;
  s.L = 0;
  s.fixed_m = 1;
  s.causal = causal ? 1 : 0;
  s.k = k;
  return s;
}

elsaa_status causal_lsh_forward(const elsaa_params* p, const Geom& g, const void* Q, const void* K, const void* V,
                                const float* W, const float* lam, const float* gs, const float* glr, void* O,
                                const Saved& s, const FwdWs& w, cudaStream_t st) {
  const PermBufs& b = w.pm;
  const size_t rows = (size_t)g.BH * g.N;
  const int rb = g.d * 2, stride = 2 * g.N;
  ELSAA_TRY(cuda_status(cudaMemsetAsync(w.flag, 0, 4, st), "flag reset"));
  // the low-rank branch, causal, in the caller's row order
  if (g.r > 0) {
    ELSAA_TRY(cuda_status(launch_race_w_split(W, w.wsplit, g, st), "W split"));
    ELSAA_TRY(cuda_status(launch_race_features_tc(Q, K, w.wsplit, s.phiQ, s.phiK, s.hQ, s.hK, s.nQ, s.nK, g, w.flag,
                                                  st),
                          "tcgen05 race features"));
    FwdArgs ra{Q, K, V, s.idx, s.phiQ, s.phiK, s.Ast, s.Bst, lam, gs, glr, O, s.Os, s.logd, s.dlr, s.m, s.Olr,
               s.Psplit, s.Pmass};
    ra.lr_num = w.lr_num;
    ra.lr_den = w.lr_den;
    ELSAA_TRY(cuda_status(launch_race_stats_tc(s.phiK, V, nullptr, false, s.Ast, s.Psplit, s.Pmass, g, w.flag, st),
                          "tcgen05 race statistics"));
    ELSAA_TRY(cuda_status(launch_race_readout_tc(ra, g, w.flag, st), "tcgen05 race read-out"));
  } else {
    ELSAA_TRY(cuda_status(cudaMemsetAsync(s.Olr, 0, rows * rb, st), "O_lr"));
    ELSAA_TRY(cuda_status(cudaMemsetAsync(s.dlr, 0, rows * 4, st), "d_lr"));
  }
  // sparse-only passes write O_s and log d_s into the level buffers; their fused output
  // and m are not used (the low-rank input they read is scratch)
  FwdArgs sa{};
  sa.idx = s.idx;
  sa.O = b.X;
  sa.Olr = b.Olr;
  sa.Os = b.Os;
  sa.logd = b.logd;
  sa.dlr = b.dlr;
  sa.m = b.m;
  // base pass: the leaves and the deepest level, in the caller's order
  const Geom gb = sparse_only(g, true, 2);
  auto sparse_pass = [&](const FwdArgs& fa, const Geom& fg) { return launch_attn_fwd_tc(fa, fg, w.flag, st); };
  ELSAA_TRY(cuda_status(launch_causal_lsh_select(s.idx, g, st), "causal sortLSH base selection"));
  sa.Q = Q; sa.K = K; sa.V = V;
  ELSAA_TRY(cuda_status(sparse_pass(sa, gb), "causal sortLSH base pass"));
  if (g.lsh_levels > 0) {
    const int lv = g.lsh_levels;
    ELSAA_TRY(cuda_status(launch_sortlsh_hash(Q, K, true, p->lsh_planes, p->lsh_bits, b.pos, nullptr, g, st),
                          "sortLSH hash"));
    for (int lev = 0; lev < lv; ++lev)
      ELSAA_TRY(cuda_status(launch_sortlsh_level_sort(b.pos, s.lsh_order + (size_t)lev * g.BH * stride,
                                                      b.inv + lev * rows, g.N >> (lev + 1), p->lsh_bits,
                                                      w.lsh_scratch, g, st),
                            "sortLSH level sort"));
    // only the future halves' queries and the past halves' keys and values are read
    const void* qs[1] = {Q};
    void* qd[1] = {s.lvQ};
    const void* kvs[2] = {K, V};
    void* kvd[2] = {s.lvK, s.lvV};
    ELSAA_TRY(cuda_status(launch_gather_rows(qs, qd, 1, s.lsh_order, rb, lv, 1, g, st), "sortLSH gather Q"));
    ELSAA_TRY(cuda_status(launch_gather_rows(kvs, kvd, 2, s.lsh_order + g.N, rb, lv, 0, g, st),
                          "sortLSH gather K, V"));
    ELSAA_TRY(cuda_status(launch_causal_lsh_select_levels(b.idx, b.tile_list, lv, g, st), "sortLSH level selection"));
    // all levels in one launch, as lv * BH heads (the tcgen05 kernel over their future
    // tiles only); the fused output is not used and not written, so the gathered rows stay
    // intact for the backward
    Geom gv = sparse_only(g, false, 1);
    gv.BH = lv * g.BH;
    sa.Q = s.lvQ; sa.K = s.lvK; sa.V = s.lvV; sa.idx = b.idx;
    sa.O = nullptr;
    sa.Os = b.Os_lv;
    sa.logd = b.logd_lv;
    sa.tile_list = b.tile_list;
    sa.n_list = g.n_t / 2;
    ELSAA_TRY(cuda_status(sparse_pass(sa, gv), "sortLSH level pass"));
  }
  return cuda_status(launch_lsh_fuse(b.Os, b.logd, b.Os_lv, b.logd_lv, b.inv, g.lsh_levels, s.Olr, s.dlr, lam, gs,
                                     glr, O, s.Os, s.logd, s.m, g, st),
                     "merge and fusion");
}

elsaa_status causal_lsh_backward(const Geom& g, BwdArgs a, const Saved& s, const BwdWs& w, cudaStream_t st) {
  const PermBufs& b = w.pm;
  const size_t rows = (size_t)g.BH * g.N;
  const int rb = g.d * 2, stride = 2 * g.N;
  ELSAA_TRY(cuda_status(cudaMemsetAsync(w.flag, 0, 4, st), "flag reset"));
  ELSAA_TRY(cuda_status(launch_row_scalars(a, true, g, st), "row scalars"));
  if (g.r > 0) {
    ELSAA_TRY(cuda_status(launch_race_stats_tc(a.phiQ, a.dOcl, w.rs.delta, true, w.RA, w.Rsplit, w.Rmass, g,
                                               w.flag, st),
                          "tcgen05 race statistics"));
    ELSAA_TRY(cuda_status(launch_race_w_split(a.W, w.Wsplit, g, st), "W split"));
    ELSAA_TRY(cuda_status(launch_race_bwd_tc(a, g, w.flag, st), "tcgen05 race backward"));
  } else {
    ELSAA_TRY(cuda_status(cudaMemsetAsync(w.dQacc, 0, rows * g.d * 4, st), "dQ accumulator"));
    ELSAA_TRY(cuda_status(cudaMemsetAsync(w.dKacc, 0, rows * g.d * 4, st), "dK accumulator"));
    ELSAA_TRY(cuda_status(cudaMemsetAsync(w.dVacc, 0, rows * g.d * 4, st), "dV accumulator"));
  }
  if (g.lsh_levels > 0) {
    const int lv = g.lsh_levels;
    // Q, K and V of the levels are the forward's gathered rows (saved); dO and the row scalars
    // are gathered here
    const void* qs[1] = {a.dO};
    void* qd[1] = {b.X};
    const void* ps[1] = {w.rs.packed};
    void* pd[1] = {b.packed};
    ELSAA_TRY(cuda_status(launch_gather_rows(qs, qd, 1, s.lsh_order, rb, lv, 1, g, st), "sortLSH gather dO"));
    ELSAA_TRY(cuda_status(launch_gather_rows(ps, pd, 1, s.lsh_order, 16, lv, 1, g, st), "sortLSH gather row scalars"));
    ELSAA_TRY(cuda_status(launch_causal_lsh_select_levels(b.idx, b.tile_list, lv, g, st), "sortLSH level selection"));
    Geom gv = sparse_only(g, false, 1);
    gv.BH = lv * g.BH;
    ELSAA_TRY(cuda_status(launch_invert_selection(b.idx, b.offs, b.tiles, b.order, gv, st), "selection inverse"));
    // all levels in one launch each: dQ over the future tiles, dK/dV over the key blocks
    // that have a tile (the past halves, first in the longest-first order)
    BwdArgs la{};
    la.Q = s.lvQ; la.K = s.lvK; la.V = s.lvV; la.dO = b.X;
    la.idx = b.idx; la.offs = b.offs; la.tiles = b.tiles; la.kv_order = b.order;
    la.rs.packed = b.packed;
    la.dQ = b.dQ; la.dK = b.dK; la.dV = b.dV;
    la.out_f32 = 1;
    la.tile_list = b.tile_list;
    la.n_list = g.n_t / 2;
    la.n_kv = g.n_t / 2;
    ELSAA_TRY(cuda_status(launch_dq_tc(la, gv, w.flag, st), "sortLSH level dq"));
    ELSAA_TRY(cuda_status(launch_dkdv_tc(la, gv, w.flag, st), "sortLSH level dkdv"));
    ELSAA_TRY(cuda_status(launch_lsh_invert_orders(s.lsh_order, b.inv, lv, g, st), "order inverses"));
    ELSAA_TRY(cuda_status(launch_lsh_collect(b.dQ, w.dQacc, nullptr, nullptr, b.inv, lv, false, g, st), "sortLSH dQ"));
    ELSAA_TRY(cuda_status(launch_lsh_collect(b.dK, w.dKacc, b.dV, w.dVacc, b.inv, lv, true, g, st),
                          "sortLSH dK, dV"));
  }
  // base pass in the caller's order: adds the accumulators before the single rounding
  const Geom gb = sparse_only(g, true, 2);
  ELSAA_TRY(cuda_status(launch_invert_selection(s.idx, w.offs, w.tiles, w.order, gb, st), "selection inverse"));
  a.idx = s.idx; a.offs = w.offs; a.tiles = w.tiles; a.kv_order = w.order;
  a.dQacc = w.dQacc; a.dKacc = w.dKacc; a.dVacc = w.dVacc;
  ELSAA_TRY(cuda_status(launch_dq_tc(a, gb, w.flag, st), "causal sortLSH base dq"));
  return cuda_status(launch_dkdv_tc(a, gb, w.flag, st), "causal sortLSH base dkdv");
}

extern "C" {

elsaa_status elsaa_profile_begin(void) {
  g_last_error.clear();
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  p.recs.clear();
  p.used = 0;
  p.on = true;
  return ELSAA_OK;
}

int elsaa_profile_end(const char** names, double* total_ms, int* launches, int max_entries) {
  g_last_error.clear();
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  p.on = false;
  int n = 0;
  for (const ProfRec& r : p.recs) {
    if (cudaEventSynchronize(p.ev[2 * r.slot + 1]) != cudaSuccess) {
      fail(ELSAA_ERR_CUDA, "profile event sync failed");
      return -1;
    }
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, p.ev[2 * r.slot], p.ev[2 * r.slot + 1]) != cudaSuccess) {
      fail(ELSAA_ERR_CUDA, "profile event timing failed");
      return -1;
    }
    int k = 0;
    while (k < n && strcmp(names[k], r.name) != 0) ++k;
    if (k == n) {
      if (n >= max_entries) continue;
      names[n] = r.name;
      total_ms[n] = 0.0;
      launches[n] = 0;
      ++n;
    }
    total_ms[k] += ms;
    launches[k] += 1;
  }
  p.recs.clear();
  p.used = 0;
  return n;
}

size_t elsaa_saved_bytes(const elsaa_params* p) {
  Geom g;
  elsaa_status st;
  if (!make_geom(p, &g, &st)) return 0;
  size_t bytes = 0;
  carve_saved(nullptr, g, p->dtype == ELSAA_DTYPE_BF16 ? 2 : 4, &bytes);
  return bytes;
}

size_t elsaa_workspace_bytes(const elsaa_params* p, int for_backward) {
  Geom g;
  elsaa_status st;
  if (!make_geom(p, &g, &st)) return 0;
  size_t bytes = 0;
  if (for_backward) carve_bwd_ws(nullptr, g, p->dtype == ELSAA_DTYPE_BF16, &bytes);
  else carve_fwd_ws(nullptr, g, p->dtype == ELSAA_DTYPE_BF16 ? 2 : 4, &bytes);
  return bytes;
}

elsaa_status elsaa_forward(const elsaa_params* p, const void* Q, const void* K, const void* V, const float* W,
                           const float* lam, const float* gs, const float* glr, void* O, void* saved,
                           void* workspace, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  Geom g;
  elsaa_status st;
  if (!make_geom(p, &g, &st)) return st;
  ELSAA_TRY(check_ptr(Q, "Q"));
  ELSAA_TRY(check_ptr(K, "K"));
  ELSAA_TRY(check_ptr(V, "V"));
  ELSAA_TRY(check_ptr(O, "O"));
  ELSAA_TRY(check_ptr(saved, "saved"));
  ELSAA_TRY(check_ptr(workspace, "workspace"));
  ELSAA_TRY(check_ptr(W, "W_hash", g.r > 0));
  ELSAA_TRY(check_ptr(lam, "lambda_vec", false));
  ELSAA_TRY(check_ptr(gs, "g_sparse", false));
  ELSAA_TRY(check_ptr(glr, "g_lr", false));
  const bool bf16 = p->dtype == ELSAA_DTYPE_BF16;
  size_t need = 0;
  FwdWs w = carve_fwd_ws(workspace, g, bf16 ? 2 : 4, &need);
  if (ws_bytes < need) return fail(ELSAA_ERR_WORKSPACE, "workspace %zu bytes < %zu required", ws_bytes, need);
  size_t sb = 0;
  Saved s = carve_saved(saved, g, bf16 ? 2 : 4, &sb);
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  const bool lsh = g.selector == ELSAA_SEL_SORTLSH;
  if (lsh && g.causal) {
    ELSAA_TRY(check_ptr(p->lsh_planes, "lsh_planes"));
    return causal_lsh_forward(p, g, Q, K, V, W, lam, gs, glr, O, s, w, st_);
  }
  void* O_out = O;
  if (lsh) {
    // the operator runs on the sorted rows (non-causal RACE, the fusion and diagonal-block
    // attention commute with row permutations); O is scattered back at the end
    ELSAA_TRY(check_ptr(p->lsh_planes, "lsh_planes"));
    void* const qkv[3] = {s.lvQ, s.lvK, s.lvV};
    ELSAA_TRY(lsh_gather(p, g, bf16, s.lsh_order, true, w.lsh_scratch, Q, K, V, nullptr, lam, gs, glr, qkv, w.pm,
                         st_));
    Q = s.lvQ; K = s.lvK; V = s.lvV; O = w.pm.X;
    if (lam) lam = w.pm.lam;
    if (gs) gs = w.pm.gs;
    if (glr) glr = w.pm.glr;
  }

  ELSAA_TRY(cuda_status(cudaMemsetAsync(w.flag, 0, 4, st_), "flag reset"));
  // the selection on the second stream, joined before the sparse forward
  SideStream* side = bf16 ? side_stream() : nullptr;
  cudaStream_t sel_st = st_;
  JoinGuard joined;                   // an early return still makes the caller's stream wait
  if (side) {
    ELSAA_TRY(cuda_status(cudaEventRecord(side->fork, st_), "selection fork"));
    ELSAA_TRY(cuda_status(cudaStreamWaitEvent(side->s, side->fork, 0), "selection fork"));
    sel_st = side->s;
    joined.arm(side, st_);
  }
  if (lsh)
    ELSAA_TRY(cuda_status(launch_diag_select(s.idx, g, sel_st), "selection"));
  else
    ELSAA_TRY(cuda_status(launch_select(Q, K, bf16, w.qbar, w.kbar, w.scores, s.idx, g, sel_st), "selection"));
  ELSAA_TRY(cuda_status(joined.record(), "selection join"));
  if (g.r > 0 && bf16) {
    ELSAA_TRY(cuda_status(launch_race_w_split(W, w.wsplit, g, st_), "W split"));
    ELSAA_TRY(cuda_status(launch_race_features_tc(Q, K, w.wsplit, s.phiQ, s.phiK, s.hQ, s.hK, s.nQ, s.nK, g, w.flag,
                                                  st_),
                          "tcgen05 race features"));
  } else if (g.r > 0) {
    ELSAA_TRY(cuda_status(launch_race_features_f32((const float*)Q, (const float*)K, W, (float*)s.phiQ,
                                                   (float*)s.phiK, s.hQ, s.hK, s.nQ, s.nK, g, st_),
                          "race features"));
  }
  // per-chunk bf16 hi/lo statistics for the tensor-core read-out and query-side backward (bf16),
  // or the segment and in-segment prefixes the fp32 read-out combines
  if (g.r > 0 && bf16)
    ELSAA_TRY(cuda_status(launch_race_stats_tc(s.phiK, V, nullptr, false, s.Ast, s.Psplit, s.Pmass, g, w.flag, st_),
                          "tcgen05 race statistics"));
  else if (g.r > 0)
    ELSAA_TRY(cuda_status(launch_race_state_fwd_f32((const float*)s.phiK, (const float*)V, s.Ast, s.Bst, g, st_),
                          "race summaries"));
  FwdArgs a{Q, K, V, s.idx, s.phiQ, s.phiK, s.Ast, s.Bst, lam, gs, glr, O, s.Os, s.logd, s.dlr, s.m, s.Olr,
            s.Psplit, s.Pmass};
  a.lr_num = w.lr_num;
  a.lr_den = w.lr_den;
  bool scattered = false;
  if (bf16) {
    if (g.r > 0) {
      ELSAA_TRY(cuda_status(launch_race_readout_tc(a, g, w.flag, st_), "tcgen05 race read-out"));
    } else {                          // no low-rank branch: the fusion reads O_lr = 0, d_lr = 0
      ELSAA_TRY(cuda_status(cudaMemsetAsync(s.Olr, 0, (size_t)g.BH * g.N * g.d * 2, st_), "O_lr"));
      ELSAA_TRY(cuda_status(cudaMemsetAsync(s.dlr, 0, (size_t)g.BH * g.N * 4, st_), "d_lr"));
    }
    ELSAA_TRY(cuda_status(joined.join(), "selection join"));
    FwdArgs at = a;
    if (lsh) {                        // the epilogue writes O straight into the caller's row order
      at.O = O_out;
      at.q_rows = s.lsh_order;
      at.rows_stride = 2 * g.N;
      scattered = true;
    }
    ELSAA_TRY(cuda_status(launch_attn_fwd_tc(at, g, w.flag, st_), "tcgen05 forward"));
  } else {
    ELSAA_TRY(cuda_status(launch_attn_fwd_f32(a, g, st_), "fused forward"));
  }
  if (lsh && !scattered)
    ELSAA_TRY(cuda_status(launch_permute_rows(O, O_out, s.lsh_order, g.d * (bf16 ? 2 : 4), g, 2 * g.N, true, st_),
                          "sortLSH scatter O"));
  return ELSAA_OK;
}

elsaa_status elsaa_backward(const elsaa_params* p, const void* Q, const void* K, const void* V, const float* W,
                            const float* lam, const float* gs, const float* glr, const void* dO,
                            const void* saved, void* dQ, void* dK, void* dV, void* workspace, size_t ws_bytes,
                            void* stream) {
  g_last_error.clear();
  Geom g;
  elsaa_status st;
  if (!make_geom(p, &g, &st)) return st;
  ELSAA_TRY(check_ptr(Q, "Q"));
  ELSAA_TRY(check_ptr(K, "K"));
  ELSAA_TRY(check_ptr(V, "V"));
  ELSAA_TRY(check_ptr(dO, "dO"));
  ELSAA_TRY(check_ptr(saved, "saved"));
  ELSAA_TRY(check_ptr(dQ, "dQ"));
  ELSAA_TRY(check_ptr(dK, "dK"));
  ELSAA_TRY(check_ptr(dV, "dV"));
  ELSAA_TRY(check_ptr(workspace, "workspace"));
  ELSAA_TRY(check_ptr(W, "W_hash", g.r > 0));
  ELSAA_TRY(check_ptr(lam, "lambda_vec", false));
  ELSAA_TRY(check_ptr(gs, "g_sparse", false));
  ELSAA_TRY(check_ptr(glr, "g_lr", false));
  const bool bf16 = p->dtype == ELSAA_DTYPE_BF16;
  size_t need = 0;
  BwdWs w = carve_bwd_ws(workspace, g, bf16, &need);
  if (ws_bytes < need) return fail(ELSAA_ERR_WORKSPACE, "workspace %zu bytes < %zu required", ws_bytes, need);
  size_t sb = 0;
  Saved s = carve_saved(const_cast<void*>(saved), g, bf16 ? 2 : 4, &sb);
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  const bool lsh = g.selector == ELSAA_SEL_SORTLSH;
  if (lsh && g.causal) {
    BwdArgs a{};
    a.Q = Q; a.K = K; a.V = V; a.dO = dO; a.W = W;
    a.lam = lam; a.gs = gs; a.glr = glr;
    a.logd = s.logd; a.dlr = s.dlr; a.m = s.m;
    a.Os = s.Os; a.Olr = s.Olr; a.phiQ = s.phiQ; a.phiK = s.phiK;
    a.hQ = s.hQ; a.hK = s.hK; a.nQ = s.nQ; a.nK = s.nK;
    a.Ast = s.Ast; a.Bst = s.Bst; a.RA = w.RA; a.RB = w.RB;
    a.rs = w.rs;
    a.dQacc = w.dQacc; a.dKacc = w.dKacc; a.dVacc = w.dVacc;
    a.dOcl = g.r > 0 ? w.dOcl : nullptr;
    a.Psplit = s.Psplit; a.Pmass = s.Pmass; a.Rsplit = w.Rsplit; a.Rmass = w.Rmass; a.Wsplit = w.Wsplit;
    a.dQ = dQ; a.dK = dK; a.dV = dV;
    return causal_lsh_backward(g, a, s, w, st_);
  }
  void *dQ_out = dQ, *dK_out = dK, *dV_out = dV;
  if (lsh) {
    // the forward ran on the sorted rows and saved its state in that order; so does this,
    // and the gradients are scattered back at the end
    void* const qkv[3] = {s.lvQ, s.lvK, s.lvV};
    ELSAA_TRY(lsh_gather(p, g, bf16, s.lsh_order, false, nullptr, Q, K, V, dO, lam, gs, glr, qkv, w.pm, st_));
    Q = s.lvQ; K = s.lvK; V = s.lvV; dO = w.pm.X;
    dQ = w.pm.dQ; dK = w.pm.dK; dV = w.pm.dV;
    if (lam) lam = w.pm.lam;
    if (gs) gs = w.pm.gs;
    if (glr) glr = w.pm.glr;
  }
  BwdArgs a{};
  a.Q = Q; a.K = K; a.V = V; a.dO = dO; a.W = W;
  a.lam = lam; a.gs = gs; a.glr = glr;
  a.idx = s.idx; a.logd = s.logd; a.dlr = s.dlr; a.m = s.m;
  a.Os = s.Os; a.Olr = s.Olr; a.phiQ = s.phiQ; a.phiK = s.phiK;
  a.hQ = s.hQ; a.hK = s.hK; a.nQ = s.nQ; a.nK = s.nK;
  a.Ast = s.Ast; a.Bst = s.Bst; a.RA = w.RA; a.RB = w.RB;
  a.offs = w.offs; a.tiles = w.tiles; a.kv_order = g.k > 0 ? w.order : nullptr; a.rs = w.rs;
  a.dQacc = w.dQacc; a.dKacc = w.dKacc; a.dVacc = w.dVacc;
  a.dOcl = bf16 && g.r > 0 ? w.dOcl : nullptr;
  a.Psplit = s.Psplit; a.Pmass = s.Pmass; a.Rsplit = w.Rsplit; a.Rmass = w.Rmass; a.Wsplit = w.Wsplit;
  a.dQ = dQ; a.dK = dK; a.dV = dV;

  bool scattered = false;
  ELSAA_TRY(cuda_status(cudaMemsetAsync(w.flag, 0, 4, st_), "flag reset"));
  ELSAA_TRY(cuda_status(launch_row_scalars(a, bf16, g, st_), "row scalars"));
  const bool race_tc = tc_race(g, bf16);
  if (race_tc)
    ELSAA_TRY(cuda_status(launch_race_stats_tc(a.phiQ, a.dOcl, w.rs.delta, true, w.RA, w.Rsplit, w.Rmass, g, w.flag,
                                               st_),
                          "tcgen05 race statistics"));
  else if (!bf16)
    ELSAA_TRY(cuda_status(launch_race_state_bwd_f32(a, g, st_), "race suffix summaries"));
  if (g.k > 0) ELSAA_TRY(cuda_status(launch_invert_selection(s.idx, w.offs, w.tiles, w.order, g, st_), "selection inverse"));
  if (bf16) {
    BwdArgs at = a;
    if (g.r == 0) at.dQacc = at.dKacc = at.dVacc = nullptr;
    if (race_tc) {
      ELSAA_TRY(cuda_status(launch_race_w_split(W, w.Wsplit, g, st_), "W split"));
      ELSAA_TRY(cuda_status(launch_race_bwd_tc(a, g, w.flag, st_), "tcgen05 race backward"));
    }
    if (lsh) {                        // the epilogues write straight into the caller's row orders
      at.dQ = dQ_out;
      at.dK = dK_out;
      at.dV = dV_out;
      at.q_rows = s.lsh_order;
      at.k_rows = s.lsh_order + g.N;
      at.rows_stride = 2 * g.N;
      scattered = true;
    }
    ELSAA_TRY(cuda_status(launch_dq_tc(at, g, w.flag, st_), "tcgen05 dq"));
    ELSAA_TRY(cuda_status(launch_dkdv_tc(at, g, w.flag, st_), "tcgen05 dkdv"));
  } else {
    ELSAA_TRY(cuda_status(launch_bwd_f32(a, g, st_), "backward"));
  }
  if (lsh && !scattered) {
    const int rb = g.d * (bf16 ? 2 : 4);
    ELSAA_TRY(cuda_status(launch_permute_rows(dQ, dQ_out, s.lsh_order, rb, g, 2 * g.N, true, st_), "sortLSH dQ"));
    ELSAA_TRY(cuda_status(launch_permute_rows(dK, dK_out, s.lsh_order + g.N, rb, g, 2 * g.N, true, st_),
                          "sortLSH dK"));
    ELSAA_TRY(cuda_status(launch_permute_rows(dV, dV_out, s.lsh_order + g.N, rb, g, 2 * g.N, true, st_),
                          "sortLSH dV"));
  }
  return ELSAA_OK;
}

elsaa_status elsaa_step_host(const elsaa_params* p, const void* const* host_in, void* const* host_out,
                             void* const* dev_in, void* const* dev_out, void* saved, void* workspace,
                             size_t ws_bytes, void* stream, void* h2d_stream, void* d2h_stream,
                             void* const* events) {
  g_last_error.clear();
  Geom g;
  elsaa_status st;
  if (!make_geom(p, &g, &st)) return st;
  if (!host_in || !host_out || !dev_in || !dev_out || !events)
    return fail(ELSAA_ERR_INVALID_ARG, "host_in, host_out, dev_in, dev_out and events must not be NULL");
  static const char* in_names[5] = {"host Q", "host K", "host V", "host dO", "host W_hash"};
  static const char* out_names[4] = {"host O", "host dQ", "host dK", "host dV"};
  for (int i = 0; i < 5; ++i) {
    if (i == 4 && g.r == 0) continue;
    if (!host_in[i]) return fail(ELSAA_ERR_INVALID_ARG, "%s is NULL", in_names[i]);
    ELSAA_TRY(check_ptr(dev_in[i], "device input"));
  }
  for (int i = 0; i < 4; ++i) {
    if (!host_out[i]) return fail(ELSAA_ERR_INVALID_ARG, "%s is NULL", out_names[i]);
    ELSAA_TRY(check_ptr(dev_out[i], "device output"));
  }
  for (int i = 0; i < 3; ++i)
    if (!events[i]) return fail(ELSAA_ERR_INVALID_ARG, "event %d is NULL", i);
  const bool lsh = g.selector == ELSAA_SEL_SORTLSH;
  if (lsh && (!host_in[5] || !p->lsh_planes))
    return fail(ELSAA_ERR_INVALID_ARG, "sortLSH: host planes (host_in[5]) and params->lsh_planes are required");
  const size_t mat = (size_t)g.BH * g.N * g.d * (p->dtype == ELSAA_DTYPE_BF16 ? 2 : 4);
  const size_t wbytes = (size_t)g.L * g.d * kHashBits * sizeof(float);
  cudaStream_t sc = static_cast<cudaStream_t>(stream), si = static_cast<cudaStream_t>(h2d_stream),
               so = static_cast<cudaStream_t>(d2h_stream);
  cudaEvent_t in_ready = static_cast<cudaEvent_t>(events[0]), computed = static_cast<cudaEvent_t>(events[1]),
              out_done = static_cast<cudaEvent_t>(events[2]);
  // inputs in, once this set's previous step has read them
  ELSAA_TRY(cuda_status(cudaStreamWaitEvent(si, computed, 0), "wait for the set's previous step"));
  for (int i = 0; i < 5; ++i) {
    if (i == 4 && g.r == 0) continue;
    ELSAA_TRY(cuda_status(cudaMemcpyAsync(dev_in[i], host_in[i], i == 4 ? wbytes : mat, cudaMemcpyHostToDevice, si),
                          "input copy"));
  }
  ELSAA_TRY(cuda_status(cudaEventRecord(in_ready, si), "inputs landed"));
  // the step, once its inputs have landed and the set's previous results have left
  ELSAA_TRY(cuda_status(cudaStreamWaitEvent(sc, in_ready, 0), "wait for the inputs"));
  ELSAA_TRY(cuda_status(cudaStreamWaitEvent(sc, out_done, 0), "wait for the previous results"));
  if (lsh)      // the planes live at one address: copied in stream order with the steps that read them
    ELSAA_TRY(cuda_status(cudaMemcpyAsync(const_cast<float*>(p->lsh_planes), host_in[5],
                                          (size_t)g.d * p->lsh_bits * sizeof(float), cudaMemcpyHostToDevice, sc),
                          "planes copy"));
  const float* W = g.r > 0 ? static_cast<const float*>(dev_in[4]) : nullptr;
  ELSAA_TRY(elsaa_forward(p, dev_in[0], dev_in[1], dev_in[2], W, nullptr, nullptr, nullptr, dev_out[0], saved,
                          workspace, ws_bytes, stream));
  ELSAA_TRY(elsaa_backward(p, dev_in[0], dev_in[1], dev_in[2], W, nullptr, nullptr, nullptr, dev_in[3], saved,
                           dev_out[1], dev_out[2], dev_out[3], workspace, ws_bytes, stream));
  ELSAA_TRY(cuda_status(cudaEventRecord(computed, sc), "step computed"));
  // results out
  ELSAA_TRY(cuda_status(cudaStreamWaitEvent(so, computed, 0), "wait for the step"));
  for (int i = 0; i < 4; ++i)
    ELSAA_TRY(cuda_status(cudaMemcpyAsync(host_out[i], dev_out[i], mat, cudaMemcpyDeviceToHost, so), "result copy"));
  return cuda_status(cudaEventRecord(out_done, so), "results left");
}

elsaa_status elsaa_fusion_grads(const elsaa_params* p, const float* lam, const float* gs, const float* glr,
                                const void* dO, const void* saved, float* dlam, float* dgs, float* dglr,
                                void* stream) {
  g_last_error.clear();
  Geom g;
  elsaa_status st;
  if (!make_geom(p, &g, &st)) return st;
  ELSAA_TRY(check_ptr(dO, "dO"));
  ELSAA_TRY(check_ptr(saved, "saved"));
  ELSAA_TRY(check_ptr(lam, "lambda_vec", false));
  ELSAA_TRY(check_ptr(gs, "g_sparse", false));
  ELSAA_TRY(check_ptr(glr, "g_lr", false));
  ELSAA_TRY(check_ptr(dlam, "dlambda", false));
  ELSAA_TRY(check_ptr(dgs, "dg_sparse", false));
  ELSAA_TRY(check_ptr(dglr, "dg_lr", false));
  const bool bf16 = p->dtype == ELSAA_DTYPE_BF16;
  size_t sb = 0;
  Saved s = carve_saved(const_cast<void*>(saved), g, bf16 ? 2 : 4, &sb);
  if (!dlam && !dgs && !dglr) return ELSAA_OK;
  // sortLSH: the saved state is in the sorted query order; each row maps back through it
  // (the causal recursion fuses in the caller's order)
  const int* perm = g.selector == ELSAA_SEL_SORTLSH && !g.causal ? s.lsh_order : nullptr;
  return cuda_status(launch_fusion_grads(dO, s.Os, s.Olr, s.logd, s.dlr, lam, gs, glr, dlam, dgs, dglr, perm,
                                         2 * g.N, bf16, g, static_cast<cudaStream_t>(stream)),
                     "fusion gradients");
}

elsaa_status elsaa_debug_select(const elsaa_params* p, const void* Q, const void* K, float* scores, int32_t* idx,
                                void* workspace, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  Geom g;
  elsaa_status st;
  if (!make_geom(p, &g, &st)) return st;
  if (g.selector != ELSAA_SEL_TOPK_BLOCKS)
    return fail(ELSAA_ERR_UNSUPPORTED, "elsaa_debug_select is for the top-k selector (see elsaa_debug_sortlsh)");
  ELSAA_TRY(check_ptr(Q, "Q"));
  ELSAA_TRY(check_ptr(K, "K"));
  ELSAA_TRY(check_ptr(scores, "scores"));
  ELSAA_TRY(check_ptr(idx, "idx", g.k > 0));
  ELSAA_TRY(check_ptr(workspace, "workspace"));
  size_t need = 0;
  FwdWs w = carve_fwd_ws(workspace, g, p->dtype == ELSAA_DTYPE_BF16 ? 2 : 4, &need);
  if (ws_bytes < need) return fail(ELSAA_ERR_WORKSPACE, "workspace %zu bytes < %zu required", ws_bytes, need);
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_select(Q, K, p->dtype == ELSAA_DTYPE_BF16, w.qbar, w.kbar, scores, idx, g, st_),
                     "selection");
}

elsaa_status elsaa_debug_sortlsh(const elsaa_params* p, const void* Q, const void* K, int32_t* codes,
                                 int32_t* order, void* stream) {
  g_last_error.clear();
  Geom g;
  elsaa_status st;
  if (!make_geom(p, &g, &st)) return st;
  if (g.selector != ELSAA_SEL_SORTLSH) return fail(ELSAA_ERR_INVALID_ARG, "params.selector is not ELSAA_SEL_SORTLSH");
  ELSAA_TRY(check_ptr(Q, "Q"));
  ELSAA_TRY(check_ptr(K, "K"));
  ELSAA_TRY(check_ptr(p->lsh_planes, "lsh_planes"));
  ELSAA_TRY(check_ptr(order, "order"));
  ELSAA_TRY(check_ptr(codes, "codes", false));
  // long heads sort through global memory: scratch allocated and freed on the stream
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  Geom gs = g;
  gs.causal = 0;                       // the whole-sequence orders, as for the non-causal selector
  const size_t scr_n = sortlsh_scratch_ints(gs);
  int* scratch = nullptr;
  if (scr_n) ELSAA_TRY(cuda_status(cudaMallocAsync(reinterpret_cast<void**>(&scratch), scr_n * 4, st_), "sortLSH scratch"));
  const elsaa_status r = cuda_status(launch_sortlsh_order(Q, K, p->dtype == ELSAA_DTYPE_BF16, p->lsh_planes,
                                                          p->lsh_bits, order, codes, scratch, gs, st_),
                                     "sortLSH order");
  if (scratch) cudaFreeAsync(scratch, st_);
  return r;
}

elsaa_status elsaa_debug_set_wait_limit(unsigned long long wait_ns, int stall) {
  g_last_error.clear();
  if (stall != 0 && stall != 1) return fail(ELSAA_ERR_INVALID_ARG, "stall must be 0 or 1");
  g_wait_ns.store(wait_ns);
  g_debug_stall.store(stall);
  return ELSAA_OK;
}

elsaa_status elsaa_check_device_flags(void* workspace, void* stream) {
  g_last_error.clear();
  if (!workspace) return fail(ELSAA_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  uint32_t flag = 0;
  ELSAA_TRY(cuda_status(cudaStreamSynchronize(st_), "stream sync"));
  ELSAA_TRY(cuda_status(cudaMemcpy(&flag, workspace, 4, cudaMemcpyDeviceToHost), "flag read"));
  ELSAA_TRY(cuda_status(cudaMemset(workspace, 0, 4), "flag clear"));
  if (flag) return fail(ELSAA_ERR_TIMEOUT, "a kernel gave up a bounded wait (flag 0x%x)", flag);
  return ELSAA_OK;
}

const char* elsaa_status_string(elsaa_status s) {
  switch (s) {
    case ELSAA_OK: return "ok";
    case ELSAA_ERR_INVALID_ARG: return "invalid argument";
    case ELSAA_ERR_UNSUPPORTED: return "unsupported shape or option";
    case ELSAA_ERR_WORKSPACE: return "workspace too small";
    case ELSAA_ERR_CUDA: return "CUDA error";
    case ELSAA_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* elsaa_last_error_message(void) { return g_last_error.c_str(); }

}  // extern "C"
