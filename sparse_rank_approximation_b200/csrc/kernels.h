// Internal launch interface between the C ABI (elsaa_api.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>
#include "common.cuh"

namespace elsaa {

// Opt-in per-kernel timing (elsaa_profile_begin / elsaa_profile_end): when
// enabled, every kernel launch is bracketed by a pair of CUDA events recorded on
// the launching stream.  Costs one branch per launch when disabled.
struct ProfScope {
  ProfScope(const char* name, cudaStream_t st);
  ~ProfScope();
  int slot;
  cudaStream_t stream;
};

struct FwdArgs {
  const void *Q, *K, *V;
  const int* idx;
  const void *phiQ, *phiK;
  const float *Ast, *Bst;
  const float *lam, *gs, *glr;
  void *O, *Os;
  float *logd, *dlr, *m;
  void* Olr;      // O_lr saved for the backward
  const void* Psplit;  // prefix statistics per chunk as bf16 hi/lo [G][BH][n_c][2][128][d] (tensor-core RACE
                       // path; one block per group of 128 features)
  const float* Pmass;  // their key-mass column [G][BH][n_c][128]
  // optional: the query tiles to run, n_list per head ([BH][n_list]); null runs all tiles
  const int* tile_list;
  int n_list;
  // optional (tensor-core kernel): O row r of head bh goes to row q_rows[bh * rows_stride + r]
  // of the caller's O instead of row r (the sortLSH orders); O_s stays in row order
  const int* q_rows;
  int rows_stride;
  // tensor-core read-out over several feature groups: the running numerator (fp32 [BH][N][d])
  // and denominator ([BH][N]) between the groups' launches
  float *lr_num, *lr_den;
};

// Per-row adjoint scalars of the fusion (Eq. 4 / Eq. 5), float32 [BH, N] each.
struct RowScalars {
  float* cs;      // g_s m: dO_s = cs dO
  float* Delta;   // <dO_s, O_s> - dd_s d_s   (sparse softmax delta)
  float* cl;      // g_lr / d_lr: dN = cl dO
  float* delta;   // dd_lr - cl <dO, O_lr>      (RACE key-mass adjoint)
  float4* packed; // (log2 d_s, cs, Delta, 0) per row, for the tensor-core backward
};

struct BwdArgs {
  const void *Q, *K, *V, *dO;
  const float* W;
  const float *lam, *gs, *glr;
  const int* idx;
  const float *logd, *dlr, *m;
  const void *Os, *Olr;
  const void *phiQ, *phiK;
  const float *hQ, *hK, *nQ, *nK;
  const float *Ast, *Bst;        // forward prefix statistics
  float *RA, *RB;                // backward suffix statistics
  const int *offs, *tiles;       // key block -> query tiles
  const int* kv_order;           // per head, key blocks by descending tile count (ties: lower block first)
  RowScalars rs;
  float *dQacc, *dKacc, *dVacc;  // fp32 low-rank gradient parts (bf16 path)
  void* dOcl;                    // cl dO rows (bf16 path), written by the row scalars
  const void* Psplit;            // prefix statistics per chunk, bf16 hi/lo [G][BH][n_c][2][128][d] (tensor-core RACE)
  const float* Pmass;            //   key-mass column [G][BH][n_c][128]
  const void* Rsplit;            // suffix statistics per chunk, same layout
  const float* Rmass;
  const void* Wsplit;            // W as bf16 hi/lo rows n = 4 l + b, [2][NW][d]
  void *dQ, *dK, *dV;
  // optional (tensor-core sparse kernels): the query tiles dQ runs, n_list per head
  // ([BH][n_list], null: all), and how many key blocks dK/dV runs in kv_order (0: all)
  const int* tile_list;
  int n_list;
  int n_kv;
  // optional (tensor-core kernels): dQ row r goes to row q_rows[bh * rows_stride + r], dK and
  // dV row r to row k_rows[bh * rows_stride + r] of the caller's outputs (the sortLSH orders)
  const int *q_rows, *k_rows;
  int rows_stride;
  // optional (sparse kernels, no row maps): write dQ, dK, dV as fp32 rows instead of bf16 (the
  // causal sortLSH recursion's level slots, summed before the single bf16 rounding)
  int out_f32;
};

// sortLSH selector: per head the sorted query and key orders, int32 [BH][2][N]
// (codes, if not null, receive the hash codes in the same layout).  Heads longer than a
// shared-memory sort takes (N > 16384) sort through global memory in `scratch`
// (sortlsh_scratch_ints ints; null is refused there).
cudaError_t launch_sortlsh_order(const void* Q, const void* K, bool bf16, const float* planes, int bits,
                                 int* order, int* codes, int* scratch, const Geom& g, cudaStream_t st);
size_t sortlsh_smem_bytes(const Geom& g, int bits);
size_t sortlsh_scratch_ints(const Geom& g);
// Hash only: Gray positions (and, if not null, codes) [BH][2][N].
cudaError_t launch_sortlsh_hash(const void* Q, const void* K, bool bf16, const float* planes, int bits, int* pos,
                                int* codes, const Geom& g, cudaStream_t st);
// Causal recursion: one level's orders [BH][2][N] (queries sorted in the future halves,
// keys in the past halves of h rows; identity elsewhere) and, if inv is not null, the
// future-half rows' positions [BH][N]; the base-pass selection; the final
// log-sum-exp merge of the partials with the fusion; the orders' inverses; the level
// gradients collected into the fp32 accumulators; multi-tensor half-row gathers.
cudaError_t launch_sortlsh_level_sort(const int* pos, int* order, int* inv, int h, int bits, int* scratch,
                                      const Geom& g, cudaStream_t st);
cudaError_t launch_causal_lsh_select(int* idx, const Geom& g, cudaStream_t st);
cudaError_t launch_lsh_fuse(const void* Os0, const float* logd0, const void* Os_lv, const float* logd_lv,
                            const int* inv_lv, int levels, const void* Olr, const float* dlr, const float* lam,
                            const float* gs, const float* glr, void* O, void* Os, float* logd, float* m, const Geom& g,
                            cudaStream_t st);
cudaError_t launch_lsh_invert_orders(const int* order, int* inv, int levels, const Geom& g, cudaStream_t st);
cudaError_t launch_lsh_collect(const void* src0, float* acc0, const void* src1, float* acc1, const int* inv,
                               int levels, bool keys, const Geom& g, cudaStream_t st);
cudaError_t launch_gather_rows(const void* const* src, void* const* dst, int n, const int* perm, int row_bytes,
                               int levels, int half, const Geom& g, cudaStream_t st);
// Every level's selection ([levels][BH][n_t], k = 1) and its future tiles ([levels][BH][n_t / 2]).
cudaError_t launch_causal_lsh_select_levels(int* idx, int* tile_list, int levels, const Geom& g, cudaStream_t st);
// Row permutation of [BH][N] rows of row_bytes (a multiple of 16): gather dst[r] = src[perm[r]]
// or scatter dst[perm[r]] = src[r]; perm advances by perm_stride per head.
cudaError_t launch_permute_rows(const void* src, void* dst, const int* perm, int row_bytes, const Geom& g,
                                int perm_stride, bool scatter, cudaStream_t st);
cudaError_t launch_gather_vec(const float* src, float* dst, const int* perm, const Geom& g, int perm_stride,
                              cudaStream_t st);
// idx[t] = {t, -1, ...}: tile t selects block t.
cudaError_t launch_diag_select(int* idx, const Geom& g, cudaStream_t st);

// Sets the message elsaa_last_error_message() returns on this thread.
void record_error(const char* msg);

cudaError_t launch_select(const void* Q, const void* K, bool bf16, double* qbar, double* kbar, float* scores,
                          int* idx, const Geom& g, cudaStream_t st);
cudaError_t launch_invert_selection(const int* idx, int* offs, int* tiles, int* order, const Geom& g,
                                    cudaStream_t st);
// fp32 path: RACE features and the chunked prefix / suffix summaries (SIMT).
cudaError_t launch_race_features_f32(const float* Q, const float* K, const float* W, float* phiQ, float* phiK,
                                     float* hQ, float* hK, float* nQ, float* nK, const Geom& g, cudaStream_t st);
cudaError_t launch_race_state_fwd_f32(const float* phiK, const float* V, float* Ast, float* Bst, const Geom& g,
                                      cudaStream_t st);
cudaError_t launch_race_state_bwd_f32(const BwdArgs& a, const Geom& g, cudaStream_t st);
// In place over the segment totals [BH][n_seg + 1][rows][dp] (total of segment s in slot s + 1):
// forward, slot s becomes the exclusive prefix of the segments before s and slot n_seg the
// grand total; backward, slot s + 1 the exclusive suffix of the segments after s and slot 0
// the grand total.
cudaError_t launch_race_scan(float* Atot, int rows, bool bwd, const Geom& g, cudaStream_t st);
// RACE chunk statistics on the tensor cores (d = 64 or 128, chunks of 128 rows, features in groups
// of 128): segment totals in tensor memory, the scan, then every chunk's exclusive prefix
// (forward: Phi = Phi(K), Y = V, w = null for 1) or suffix (backward: Phi = Phi(Q), Y = cl dO,
// w = delta) written as bf16 hi/lo [G][BH][n_c][2][128][d] with its fp32 mass [G][BH][n_c][128].
// Atot is fp32 scratch [BH][n_seg + 1][128][dp], reused by the groups.
bool race_stats_tc_supported(const Geom& g);
cudaError_t launch_race_stats_tc(const void* phi, const void* Y, const float* w, bool bwd, float* Atot, void* out,
                                 float* mass, const Geom& g, uint32_t* err, cudaStream_t st);
// W[l][d][4] -> bf16 hi/lo rows n = 4 l + b, [2][NW][d] with NW = 4L rounded up to 32.
cudaError_t launch_race_w_split(const float* W, void* out, const Geom& g, cudaStream_t st);
// RACE features on the tensor cores (bf16, d = 64 or 128, L <= 16): Phi (bf16 [BH][N][rp], zero
// padded), the normalised projections h (fp32 [BH][N][4L]) and the row norms; wsplit is the W
// split written by launch_race_w_split.
cudaError_t launch_race_features_tc(const void* Q, const void* K, const void* wsplit, void* phiQ, void* phiK,
                                    float* hQ, float* hK, float* nQ, float* nK, const Geom& g, uint32_t* err,
                                    cudaStream_t st);
// tcgen05 sparse-branch forward + fusion epilogue (d = 64 or 128, blocks of 64 or 128 keys);
// reads the low-rank output written by launch_race_readout_tc (zeros without a low-rank branch).
bool attn_fwd_tc_supported(const Geom& g);
cudaError_t launch_attn_fwd_tc(const FwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st);
// tcgen05 RACE read-out (same shapes as race_bwd_tc_supported): O_lr (bf16) and d_lr.
cudaError_t launch_race_readout_tc(const FwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st);
cudaError_t launch_attn_fwd_f32(const FwdArgs& a, const Geom& g, cudaStream_t st);
cudaError_t launch_row_scalars(const BwdArgs& a, bool bf16, const Geom& g, cudaStream_t st);
// Per-row gradients of the fusion parameters lambda, g_s, g_lr (any output may be null).
// With perm (sortLSH), row r of the saved state belongs to input row perm[r] (stride
// perm_stride per head): dO, lambda and the gates are read there and the results written there.
cudaError_t launch_fusion_grads(const void* dO, const void* Os, const void* Olr, const float* logd, const float* dlr,
                                const float* lam, const float* gs, const float* glr, float* dlam, float* dgs,
                                float* dglr, const int* perm, int perm_stride, bool bf16, const Geom& g,
                                cudaStream_t st);
// tcgen05 sparse-branch backward (d = 64 or 128, blocks of 64 or 128 keys): dQ (query-major) and
// dK/dV (key-major through the selection inverse), adding the low-rank accumulators.
bool bwd_tc_supported(const Geom& g);
// tcgen05 RACE backward (d = 64 or 128, chunks of 128 rows, r <= 256 in groups of 128 features):
// low-rank parts of dQ, dK, dV into the fp32 accumulators; needs the saved projections and
// row norms.
bool race_bwd_tc_supported(const Geom& g);
cudaError_t launch_race_bwd_tc(const BwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st);
cudaError_t launch_dq_tc(const BwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st);
cudaError_t launch_dkdv_tc(const BwdArgs& a, const Geom& g, uint32_t* err, cudaStream_t st);
cudaError_t launch_bwd_f32(const BwdArgs& a, const Geom& g, cudaStream_t st);

}  // namespace elsaa
