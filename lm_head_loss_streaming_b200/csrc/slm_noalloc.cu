// slm_noalloc.cu - a forward entry point for callers that cannot allocate device memory.
//
// slm_loss_fwd needs a caller-provided workspace for its scratch (the per-row partial
// statistics of every vocabulary run, the label logits, the reduction buffers and the
// device status word).  Some callers cannot provide one: a plain C host that links this
// library without a framework allocator, a runtime whose enqueue path must not call
// cudaMalloc (it can synchronise the whole device), or a process that works inside a
// fixed memory budget.  slm_loss_fwd_noalloc serves them with scratch that lives in a
// file-scope __device__ array of fixed size, allocated once per GPU when the library's
// device code is loaded there and held until the process exits.
//
// The array's name is only a host-side stand-in for the symbol; its device address is
// looked up with cudaGetSymbolAddress, with the device current, on the first call that runs
// on a device, and kept for that device's CUDA context.  A context that is torn down and
// re-created (cudaDeviceReset, or a primary context released and retained again) reloads
// the library's device code at another address, so the cached address is keyed on the
// context's unique id and looked up again when the current context is a different one.
// The lookup may load the library's device code, so the first call on each device (and
// the first after a context is re-created) should come before any stream capture.
//
// Every call shares the one array and leaves its contents behind.  The forward rewrites
// everything it reads before reading it (the status word is cleared on entry, the partials,
// label logits and reduction buffers are fully written by the kernels that later read
// them), so no state carries over between calls.  Calls that overlap on the GPU (two
// streams at once, or two host threads on different streams) race on the array and must be
// serialised by the caller.
//
// Nothing here allocates: no cudaMalloc, no cudaFree, no allocating library routine.

#include <cuda.h>

#include <mutex>

#include "../../include/slm.h"
#include "slm_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SLM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
struct ScratchAddr {
  unsigned long long ctx_id;  // unique id of the context the address belongs to (0: none)
  void* ptr;
};
ScratchAddr g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the current CUDA context, or 0 when there is none or it cannot be read.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array in the current device's current context: looked up
// once per device and context (again whenever the context's id cannot be read).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SLM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long id = current_context_id();
  if (id == 0 || g_scratch[dev].ctx_id != id || g_scratch[dev].ptr == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return SLM_ERR_CUDA;
    // The lookup creates the primary context when there was none: key on the id after it.
    g_scratch[dev] = ScratchAddr{current_context_id(), p};
  }
  *out = g_scratch[dev].ptr;
  return SLM_OK;
}

}  // namespace

extern "C" SLM_API int slm_loss_fwd_noalloc(int kind, const void* Hq, const void* Hp,
                                            const void* W, const int32_t* labels,
                                            int32_t ignore_index, int64_t N, int64_t d,
                                            int64_t V, float* loss_tok, float* alpha_tok,
                                            double* loss_sum, int64_t* n_valid,
                                            float* loss_mean, float* stats, int* device_flags,
                                            void* stream) {
  // Reject an unknown kind or an invalid shape before touching the device.
  if (slm_workspace_bytes(kind, N, d, V, 1) == 0) {
    if (kind < SLM_CE || kind > SLM_CE_ARGMAX_P) return SLM_ERR_KIND;
    return SLM_ERR_SHAPE;
  }
  void* scratch = nullptr;
  int st = scratch_address(&scratch);
  if (st != SLM_OK) return st;
  // slm_loss_fwd rejects (SLM_ERR_WORKSPACE) any size whose scratch exceeds the array.
  st = slm_loss_fwd(kind, Hq, Hp, W, labels, ignore_index, N, d, V, loss_tok, alpha_tok,
                    loss_sum, n_valid, loss_mean, stats, scratch, SLM_NOALLOC_SCRATCH_BYTES,
                    stream);
  if (st != SLM_OK) return st;
  if (device_flags) {
    if (cudaMemcpyAsync(device_flags, scratch, sizeof(int), cudaMemcpyDeviceToDevice,
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
      return SLM_ERR_CUDA;
  }
  return SLM_OK;
}
