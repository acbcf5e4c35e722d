// Selection without caller-provided scratch: the same pooling, block-score and
// top-k kernels as elsaa_debug_select, with their scratch (pooled means and the
// block-score matrix) in a fixed array compiled into the library.
//
// Some callers cannot call cudaMalloc at the moment they need the selection:
// code running inside a region that is being captured into a CUDA graph,
// programs whose memory is fully reserved up front by a pool or another
// framework, and embedded or real-time runtimes that forbid device allocation
// after start-up.  They can call elsaa_select_noalloc, which needs only the
// inputs and the output.
//
// The scratch is one static device array of kNoAllocScratchBytes.  Every GPU
// that loads the library keeps it until the process exits.  All calls share it,
// so calls whose work overlaps on the GPU (different streams, or different host
// threads on the same device) race; serialise them.  Nothing in it needs to
// start at zero: the kernels write every entry they later read.
#include <cuda.h>

#include <mutex>
#include <string>

#include "../../include/elsaa.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};   // the context each cached address belongs to

// The current driver context, or null when it cannot be read.  A device reset or a
// different (non-primary) context on the same ordinal loads the module again, at a
// new address, so the cached address is only reused under the context it came from.
CUcontext current_context() {
  using Fn = CUresult (*)(CUcontext*);
  static Fn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<Fn>(p);
  }
  CUcontext ctx = nullptr;
  if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

elsaa_status noalloc_fail(elsaa_status s, const std::string& msg) {
  elsaa::record_error(msg.c_str());   // read back with elsaa_last_error_message()
  return s;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" {

elsaa_status elsaa_select_noalloc(const elsaa_params* p, const void* Q, const void* K, int32_t* idx,
                                  void* stream) {
  elsaa::record_error("");
  if (!p) return noalloc_fail(ELSAA_ERR_INVALID_ARG, "params is NULL");
  // The size query validates the parameters without touching the GPU.
  if (elsaa_workspace_bytes(p, 0) == 0)
    return noalloc_fail(ELSAA_ERR_INVALID_ARG, std::string("invalid params: ") + elsaa_last_error_message());
  if (p->selector != ELSAA_SEL_TOPK_BLOCKS)
    return noalloc_fail(ELSAA_ERR_UNSUPPORTED, "elsaa_select_noalloc is the top-k block selection");
  if (!Q || !K || (p->topk > 0 && !idx)) return noalloc_fail(ELSAA_ERR_INVALID_ARG, "Q, K or idx is NULL");
  if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(idx)) & 15u)
    return noalloc_fail(ELSAA_ERR_INVALID_ARG, "Q, K and idx must be 16-byte aligned");

  elsaa::Geom g{};
  g.BH = p->B * p->H;
  g.N = p->N;
  g.d = p->d;
  g.T = p->block_size;
  g.n_t = (p->N + p->block_size - 1) / p->block_size;
  g.k = p->topk;
  g.causal = p->causal;
  g.scale = p->scale;
  const size_t means = align256((size_t)g.BH * g.n_t * g.d * sizeof(double));
  const size_t scores = align256((size_t)g.BH * g.n_t * g.n_t * sizeof(float));
  const size_t need = 2 * means + scores;
  if (need > kNoAllocScratchBytes)
    return noalloc_fail(ELSAA_ERR_UNSUPPORTED,
                        "selection needs " + std::to_string(need) + " bytes of scratch; the static scratch holds " +
                            std::to_string(kNoAllocScratchBytes) + " (B*H*ceil(N/block)*(16*d + 4*ceil(N/block)))");

  // One-time set-up per device and context (with that device current): the host-side
  // name of the array is not a device address, so resolve the address and cache it.
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return noalloc_fail(ELSAA_ERR_CUDA, "cudaGetDevice failed or device ordinal out of range");
  const CUcontext ctx = current_context();
  char* base = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev] || !ctx || g_scratch_ctx[dev] != ctx) {
      void* ptr = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&ptr, g_select_scratch);
      if (e != cudaSuccess || !ptr)
        return noalloc_fail(ELSAA_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
      g_scratch_ptr[dev] = ptr;
      // with the context unknown the address is resolved again on every call
      g_scratch_ctx[dev] = ctx;
    }
    base = static_cast<char*>(g_scratch_ptr[dev]);
  }
  double* qbar = reinterpret_cast<double*>(base);
  double* kbar = reinterpret_cast<double*>(base + means);
  float* sc = reinterpret_cast<float*>(base + 2 * means);
  const cudaError_t e = elsaa::launch_select(Q, K, p->dtype == ELSAA_DTYPE_BF16, qbar, kbar, sc, idx, g,
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return noalloc_fail(ELSAA_ERR_CUDA, std::string("selection: ") + cudaGetErrorString(e));
  return ELSAA_OK;
}

}  // extern "C"
