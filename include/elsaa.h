/*
 * elsaa.h — C ABI of libelsaa.so: the ELSAA attention operator (sparse top-k
 * block branch + RACE low-rank branch + denominator-aware fusion), forward and
 * backward, on one NVIDIA B200 (sm_100a).
 *
 * Source of every definition: the paper page "ELSAA: Efficient Low-Rank and
 * Sparse Attention Approximation for Training Transformers" (arXiv 2607.20214):
 *   - dense per-head attention and the per-head procedure ........ §3
 *   - low-rank branch: RACE soft hash-bucket summaries, normalised
 *     ratio form giving O_lr and d_lr; causal chunked prefix ...... §3.1
 *   - sparse branch: exact attention over a selected support,
 *     returning O_sparse and d_sparse .............................. §3.2, §3.3 Practical notes
 *   - fusion weight m = d_s / (d_s + lambda d_lr + eps) ............ §3.3, Eq. 5
 *   - output O = g_s m O_s + g_lr O_lr ............................. §1, Eq. 4
 *   - sketch size S_R = L 2^gamma (so r = L * 2^gamma) ............. §6
 * Readings this library takes where the page is silent:
 *   - selector: top-k key blocks per query tile (block size T = queries per
 *     tile = keys per block), block score = scale * mean(Q_tile) . mean(K_block),
 *     ties to the lower block index; causal: the diagonal block is always
 *     selected, then the best k-1 earlier blocks, keys j > i masked;
 *   - RACE features: u = x / max(|x|, 1e-12), h_l = W_l^T u, bucket
 *     probabilities p_l(c|x) = softmax over corners c in {-1,1}^gamma of
 *     <c, h_l> / tau, Phi(x) = [p_l(c|x) / sqrt(L)];
 *     kappa(q, k) = Phi(q) . Phi(k); O_lr,i = sum_j kappa v_j / d_lr,i over
 *     all keys (j <= i when causal), d_lr,i = sum_j kappa;
 *   - default gates g_s = 1, g_lr = 1 - m; gradients flow to Q, K, V only
 *     (selection, W_hash, lambda and the gates are constants).
 *
 * Conventions shared by every entry point:
 *   - Ownership: the caller owns every buffer and stream.  The library never
 *     allocates or frees device memory and keeps no state between calls
 *     (apart from the opt-in profiler below).
 *   - Pointers: all tensor pointers are DEVICE pointers, 16-byte aligned,
 *     except where a function says otherwise.
 *   - Layout: Q, K, V, O, dO, dQ, dK, dV are contiguous row-major [B, H, N, d]
 *     in the element type given by params->dtype (float32 or bfloat16).
 *     W_hash is float32 [L, d, gamma] (L = rank_r >> hash_bits), shared by all
 *     batches and heads.  lambda_vec, g_sparse, g_lr are float32 [B, H, N] or
 *     NULL (NULL: scalar params->lambda; g_s = 1; g_lr = 1 - m).
 *   - Streams: calls are asynchronous on `stream` (a cudaStream_t, may be 0).
 *     They do not synchronise, except elsaa_check_device_flags.
 *   - Errors: invalid arguments return before any launch with
 *     ELSAA_ERR_INVALID_ARG / ELSAA_ERR_UNSUPPORTED / ELSAA_ERR_WORKSPACE;
 *     a failed launch returns ELSAA_ERR_CUDA.  elsaa_last_error_message()
 *     returns a one-line description of the last failure on this thread.
 *   - Supported: N >= 1 (a last tile shorter than block_size is allowed);
 *     d in {64, 128}; hash_bits == 4; rank_r a multiple of 16 with
 *     0 <= rank_r <= 256; 0 <= topk <= ceil(N / block_size) <= 1024.
 *     bfloat16: block_size in {64, 128}.  float32: block_size in {1, 64, 128}
 *     (block_size 1 only with N <= 4096).
 */
#ifndef ELSAA_H_
#define ELSAA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ELSAA_API __attribute__((visibility("default")))
#else
#define ELSAA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ELSAA_OK = 0,
  ELSAA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned buffer */
  ELSAA_ERR_UNSUPPORTED = 2,   /* valid operator, shape outside the supported set */
  ELSAA_ERR_WORKSPACE = 3,     /* workspace or saved buffer smaller than required */
  ELSAA_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
  ELSAA_ERR_TIMEOUT = 5        /* a device-side bounded wait gave up (see elsaa_check_device_flags) */
} elsaa_status;

typedef enum { ELSAA_DTYPE_F32 = 0, ELSAA_DTYPE_BF16 = 1 } elsaa_dtype;

/* Sparse-branch selector.  TOPK_BLOCKS: per query tile the top-k key blocks by
 * mean-pooled logit (§3.3 Practical notes allow any important-key selector).
 * SORTLSH: the paper's sortLSH (§3.2); topk is not used.  Rows are hashed with
 * angular LSH (lsh_bits hyperplanes, bit c set when x . R_c > 0) and ordered by the
 * code's position in the reflected Gray sequence, then by row.
 *   causal = 0: the sorted queries and keys are cut into blocks of block_size and
 *     query block t attends key block t exactly.  block_size 64 or 128.
 *   causal = 1: the paper's recursion ("For the causal setting", §3.2).  A segment
 *     splits on a block boundary into past and future halves (an odd block count
 *     gives the extra block to the past); each half recurses; the future queries
 *     attend the past keys by non-causal sortLSH on the two halves; the future
 *     half's results merge by log-sum-exp; a single block is attended exactly under
 *     j <= i.  Needs bf16 and N = block_size * 2^L.
 *   Heads of up to 16384 rows (halves of up to 16384 rows in the recursion) are sorted
 *   in shared memory, longer ones through global memory in the workspace. */
typedef enum { ELSAA_SEL_TOPK_BLOCKS = 0, ELSAA_SEL_SORTLSH = 1 } elsaa_selector;

typedef struct {
  int32_t B, H, N, d;     /* batch, heads, sequence length, head dimension */
  int32_t dtype;          /* elsaa_dtype of Q, K, V, O, dO, dQ, dK, dV */
  int32_t causal;         /* 0 or 1 */
  int32_t rank_r;         /* r = L * 2^hash_bits RACE features; 0 disables the low-rank branch */
  int32_t hash_bits;      /* gamma: bits per RACE table (4) */
  int32_t block_size;     /* T: queries per tile = keys per block */
  int32_t topk;           /* k: key blocks selected per query tile; 0 disables the sparse branch */
  float scale;            /* logit scale, normally 1/sqrt(d) */
  float lambda;           /* Eq. 5 lambda when lambda_vec == NULL */
  float eps;              /* Eq. 5 epsilon (>= 0) */
  float tau;              /* RACE soft-assignment temperature (> 0) */
  int32_t fixed_m;        /* 0: denominator-aware fusion (Eq. 5).  1: the paper's ablation without it
                             (Sort_Lsh_RACE, §6 "Attention variants"): m = 1 and g_lr defaults to 1,
                             so O = g_s O_s + g_lr O_lr.  Must match between forward and backward. */
  int32_t selector;       /* elsaa_selector */
  int32_t lsh_bits;       /* SORTLSH: hash bits b, 1..16 */
  const float* lsh_planes;/* SORTLSH: device float32 [d, lsh_bits] hyperplanes R, caller-owned */
} elsaa_params;

/* Bytes of the caller-owned `saved` buffer the forward fills and the backward
 * reads (selection, per-row denominators, the fusion weight, O_sparse, RACE
 * features and prefix summaries; with SORTLSH also the sorted orders, one pair per
 * recursion level when causal, and the rows the operator ran on, which the backward
 * reuses: the sorted Q, K, V, or with the causal recursion every level's gathered
 * query, key and value rows, 3 * levels * B * H * N * d elements).  O_sparse is kept in float32 for every dtype: the
 * backward forms the softmax delta <dO_s, O_s> from it, and a bf16 copy would put
 * the rounding of O_s into every dS of a row whose mass sits on a few keys.
 * Returns 0 when params are invalid. */
ELSAA_API size_t elsaa_saved_bytes(const elsaa_params* params);

/* Bytes of scratch device memory a forward (for_backward = 0) or backward
 * (for_backward = 1) call needs.  With SORTLSH this includes the row-permuted copies
 * of O (forward) or dO and the gradients (backward) and, when causal, every recursion
 * level's partial results and gradients at once.  Returns 0 when params are invalid. */
ELSAA_API size_t elsaa_workspace_bytes(const elsaa_params* params, int for_backward);

/* Forward: O = g_s m O_s + g_lr O_lr for every (b, h) [Eq. 4, Eq. 5, §3.1, §3.2].
 *   Q, K, V      in   [B,H,N,d] dtype
 *   W_hash       in   float32 [L, d, hash_bits]
 *   lambda_vec, g_sparse, g_lr  in  float32 [B,H,N] or NULL
 *   O            out  [B,H,N,d] dtype
 *   saved        out  elsaa_saved_bytes() bytes, consumed by elsaa_backward
 *   workspace    scratch, elsaa_workspace_bytes(params, 0) bytes */
ELSAA_API elsaa_status elsaa_forward(const elsaa_params* params,
                           const void* Q, const void* K, const void* V,
                           const float* W_hash, const float* lambda_vec,
                           const float* g_sparse, const float* g_lr,
                           void* O, void* saved,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Backward: exact gradients of sum(dO * O) with respect to Q, K and V through
 * Eq. 4, Eq. 5, the sparse softmax and the RACE features, given the `saved`
 * buffer of the forward call with the same params and inputs.
 *   dO           in   [B,H,N,d] dtype
 *   dQ, dK, dV   out  [B,H,N,d] dtype (overwritten)
 *   workspace    scratch, elsaa_workspace_bytes(params, 1) bytes */
ELSAA_API elsaa_status elsaa_backward(const elsaa_params* params,
                            const void* Q, const void* K, const void* V,
                            const float* W_hash, const float* lambda_vec,
                            const float* g_sparse, const float* g_lr,
                            const void* dO, const void* saved,
                            void* dQ, void* dK, void* dV,
                            void* workspace, size_t workspace_bytes, void* stream);

/* One forward + backward step from pinned host memory: the end-to-end path a training
 * loop takes when its batches live on the host.  Copies the step's inputs host -> device
 * on `h2d_stream`, runs elsaa_forward and elsaa_backward on `stream` (default lambda and
 * gates), and copies O, dQ, dK, dV device -> host on `d2h_stream`; everything is
 * asynchronous and the call allocates nothing.
 *   host_in   in   pinned host pointers {Q, K, V, dO (each [B,H,N,d] dtype), W_hash (float32
 *                  [L, d, hash_bits]; may be NULL when rank_r = 0), sortLSH planes (float32
 *                  [d, lsh_bits], copied into params->lsh_planes in `stream` order; NULL otherwise)}
 *   host_out  out  pinned host pointers {O, dQ, dK, dV}, [B,H,N,d] dtype
 *   dev_in, dev_out    one set of caller-owned device buffers of the same shapes {Q, K, V, dO,
 *                  W_hash} and {O, dQ, dK, dV}; alternate two sets between consecutive calls so
 *                  that one step's copies overlap the other's compute
 *   saved, workspace   as elsaa_forward / elsaa_backward (elsaa_saved_bytes(), and the larger of
 *                  the two elsaa_workspace_bytes() sizes), shared by every call in `stream` order
 *   events    three caller-owned CUDA events (cudaEvent_t) of this device set: {inputs landed,
 *                  step computed, results left}.  The input copies first wait for "step computed"
 *                  of the set's previous use, the step for "inputs landed" and the set's previous
 *                  "results left", the result copies for "step computed".  The caller waits on
 *                  "results left" before reading host_out.
 * NULL arrays, inputs or events return ELSAA_ERR_INVALID_ARG before any copy; otherwise the
 * status of the copies, the forward and the backward. */
ELSAA_API elsaa_status elsaa_step_host(const elsaa_params* params, const void* const* host_in,
                                       void* const* host_out, void* const* dev_in, void* const* dev_out,
                                       void* saved, void* workspace, size_t workspace_bytes, void* stream,
                                       void* h2d_stream, void* d2h_stream, void* const* events);

/* Per-row gradients of sum(dO * O) with respect to the fusion parameters of Eq. 5 /
 * Eq. 4 (the paper's optional learnable lambda, §1 contribution 3, and the two gates):
 *   dlambda[i] = -dm_i d_s,i d_lr,i / D_i^2     (0 when fixed_m = 1)
 *   dg_sparse[i] = m_i <dO_i, O_s,i>,  dg_lr[i] = <dO_i, O_lr,i>
 * with dm_i = g_s,i <dO_i, O_s,i> - [g_lr == NULL] <dO_i, O_lr,i> and D_i = d_s,i + lambda_i d_lr,i + eps.
 * A gate passed as NULL gets the derivative at its default value.  For a scalar lambda
 * (lambda_vec == NULL) its gradient is the sum of dlambda over all rows.
 *   lambda_vec, g_sparse, g_lr  in   float32 [B,H,N] or NULL, as given to the forward
 *   dO                          in   [B,H,N,d] dtype
 *   saved                       in   the forward's `saved` buffer
 *   dlambda, dg_sparse, dg_lr   out  float32 [B,H,N]; any may be NULL (not written)
 * Asynchronous on `stream`; allocates nothing and needs no workspace. */
ELSAA_API elsaa_status elsaa_fusion_grads(const elsaa_params* params, const float* lambda_vec,
                                          const float* g_sparse, const float* g_lr, const void* dO,
                                          const void* saved, float* dlambda, float* dg_sparse, float* dg_lr,
                                          void* stream);

/* sortLSH selector only: the hash code of every row and the two sorted orders, for
 * inspection.  codes and order are int32 [B,H,2,N] (index 0: queries, 1: keys): codes
 * hold the lsh_bits-bit hash, order[.., s, p] the row at sorted position p of the whole
 * sequence (the causal recursion sorts each half-segment by the same key, so its orders
 * follow from the codes).  Needs no workspace; asynchronous on `stream`.  For N > 16384
 * the sort goes through global memory: its scratch (2 B H 2 N int32) is allocated and
 * freed on `stream` (stream-ordered; not for use inside a graph capture). */
ELSAA_API elsaa_status elsaa_debug_sortlsh(const elsaa_params* params, const void* Q, const void* K,
                                           int32_t* codes, int32_t* order, void* stream);

/* Selection only: the float32 block scores the selector ranks and the chosen
 * blocks, for checking the selector against an external implementation.
 *   scores  out  float32 [B, H, n_t, n_t]  (n_t = ceil(N / block_size)); every
 *                entry is written, including blocks a causal tile may not select
 *   idx     out  int32 [B, H, n_t, topk], ascending block order, -1 padding
 *   workspace    scratch, elsaa_workspace_bytes(params, 0) bytes */
ELSAA_API elsaa_status elsaa_debug_select(const elsaa_params* params, const void* Q, const void* K,
                                float* scores, int32_t* idx,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Selection with no caller scratch and no allocation (the paper has no
 * counterpart; this is a deployment convenience).  Same result as the idx
 * output of elsaa_debug_select, for callers that cannot allocate device memory
 * when they need it: code inside a region being captured into a CUDA graph,
 * programs whose device memory is reserved up front by a pool or another
 * framework, and runtimes that forbid allocation after start-up.
 *   Q, K    in   [B,H,N,d] dtype, device pointers
 *   idx     out  int32 [B, H, n_t, topk] (device), as elsaa_debug_select
 * The pooled means and block scores live in one static device array of
 * 16 MiB compiled into the library, which every GPU that loads the library
 * holds until the process exits.  A problem needing more,
 * B*H*n_t*(16*d + 4*n_t) bytes plus alignment (n_t = ceil(N / block_size)),
 * is rejected with ELSAA_ERR_UNSUPPORTED before any launch.  The first call on
 * each device resolves the array's device address (cudaGetSymbolAddress) with
 * that device current; make that first call before any stream capture.  All
 * calls share the array: calls whose work can overlap on the GPU (other
 * streams, other host threads on the same device) race and must be
 * serialised by the caller.  The function allocates and frees nothing. */
ELSAA_API elsaa_status elsaa_select_noalloc(const elsaa_params* params, const void* Q, const void* K,
                                           int32_t* idx, void* stream);

/* Synchronises `stream`, then reads and clears the device error flag kept at
 * the start of `workspace`.  Returns ELSAA_ERR_TIMEOUT if a kernel gave up a
 * bounded wait since the last check, else ELSAA_OK (or ELSAA_ERR_CUDA). */
ELSAA_API elsaa_status elsaa_check_device_flags(void* workspace, void* stream);

/* Test hook for the bounded device waits (failure detection without a GPU fault).
 * Every pipeline wait of the tensor-core kernels gives up after a time limit,
 * records a code in the error word at the start of the call's workspace, drains
 * the copies and products its block has in flight, frees its tensor memory and
 * returns; elsaa_check_device_flags then reports ELSAA_ERR_TIMEOUT.
 *   wait_ns  the limit for calls made from now on; 0 restores the default (2 s)
 *   stall    1: the tensor-core sparse forward's softmax warps first wait on a
 *            barrier that nothing completes, so every such launch takes the
 *            give-up path once the limit has passed (code 0x40000 in the error
 *            word); 0: normal operation
 * Process-wide, read when a call starts; not for concurrent use with other
 * calls.  Returns ELSAA_ERR_INVALID_ARG for stall outside {0, 1}. */
ELSAA_API elsaa_status elsaa_debug_set_wait_limit(unsigned long long wait_ns, int stall);

/* Opt-in kernel timing.  After elsaa_profile_begin() every kernel the library
 * launches (from any thread, on any stream) is bracketed by two CUDA events
 * recorded on its launch stream.  elsaa_profile_end() waits for those events,
 * turns profiling off and reports, per kernel name, the summed device time in
 * milliseconds and the number of launches; it fills at most max_entries rows of
 * the caller's arrays (names point to static strings) and returns the number of
 * rows, or -1 on a CUDA error.  Profiling is the only state the library keeps
 * between calls; it holds up to 16384 launches per session. */
ELSAA_API elsaa_status elsaa_profile_begin(void);
ELSAA_API int elsaa_profile_end(const char** names, double* total_ms, int* launches, int max_entries);

/* Static English name of a status code. */
ELSAA_API const char* elsaa_status_string(elsaa_status status);

/* One-line description of the last failed call on this thread ("" if none). */
ELSAA_API const char* elsaa_last_error_message(void);

#ifdef __cplusplus
}
#endif
#endif /* ELSAA_H_ */
