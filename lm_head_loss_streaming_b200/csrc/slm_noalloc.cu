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
// looked up with cudaGetSymbolAddress, once per device, with that device current, on the
// first call that runs on it.  That lookup may load the library's device code, so the first
// call on each device should come before any stream capture.
//
// Every call shares the one array and leaves its contents behind.  The forward rewrites
// everything it reads before reading it (the status word is cleared on entry, the partials,
// label logits and reduction buffers are fully written by the kernels that later read
// them), so no state carries over between calls.  Calls that overlap on the GPU (two
// streams at once, or two host threads on different streams) race on the array and must be
// serialised by the caller.
//
// Nothing here allocates: no cudaMalloc, no cudaFree, no allocating library routine.

#include <mutex>

#include "../../include/slm.h"
#include "slm_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SLM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SLM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return SLM_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
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
    if (kind < SLM_CE || kind > SLM_LK_HYBRID) return SLM_ERR_KIND;
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
