// slm_api.cu - the C ABI of the streaming LM-head loss (declared in include/slm.h).
//
// Host-side orchestration only: argument validation, workspace carving, TMA tensor-map
// encoding and the launch sequence.  All arithmetic runs in the kernels of
// slm_kernels.cu.  Nothing here allocates device memory or synchronises (except
// slm_device_status).
//
// Launch sequence ("Training speculative decoders: removing the logits and attention
// bottlenecks", "Streaming Cross Entropy" and "Backward pass"):
//   forward   memset(status) -> LM-head GEMM with the online softmax-statistics epilogue
//             (vocabulary-tiled, one pass for CE / KL) -> per-row combine -> [alpha
//             losses: second GEMM pass for alpha and S -> combine] -> fixed-order loss
//             reduction (loss_sum, n_valid, mean).
//   backward  for each token chunk: GEMM recompute of the chunk's logits with the
//             logits-gradient epilogue (bf16 chunk buffer) -> dH = dZ W -> dW (+)= dZ^T H.

#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/slm.h"
#include "slm_internal.h"
#include "slm_schedule.h"

namespace slm {
namespace {

constexpr size_t kAlign = 256;
// Kernel classes of slm_trace_read (the order of SLM_TRACE_* in slm.h).
enum TraceClass : int {
  kTrFwdGemm = 0,    // forward statistics GEMMs (pass 1; flatness)
  kTrPass2Gemm = 1,  // second-pass GEMMs (alpha / S, JSD halves)
  kTrDzGemm = 2,     // backward logits recompute + logits-gradient GEMMs
  kTrDhGemm = 3,     // dH = dZ W
  kTrDwGemm = 4,     // dW (+)= dZ^T H
  kTrBwdFused = 5,   // the persistent fused backward (dZ, dH and dW in one launch)
  kTrLogitsRow = 6,  // row kernels over kept logits (fused single call)
  kTrRow = 7,        // combines, reductions, counts, alignment
  kTraceClasses = 8
};
constexpr int kMaxReserveSms = 128;  // slm_loss_bwd_overlap's reserve_sms, at most
constexpr long long kTimeoutCycles = 4000000000LL;  // ~2 s at the B200's boost clock

// Test hooks set through slm_debug_set (process-wide, read at every launch).
std::atomic<int> g_fault{0};
// Backward launch shape (slm_set_backward_mode): 1 = one persistent launch per chunk
// (bwd_fused_kernel), 0 = three launches per chunk (logits gradient, dH, dW).
std::atomic<int> g_bwd_mode{1};
std::atomic<long long> g_timeout{kTimeoutCycles};

DevCtl make_ctl(int* status) {
  return DevCtl{status, g_timeout.load(), g_fault.load()};
}

// Kernel-class timing (slm_trace_enable / slm_trace_read).  While enabled, every kernel
// launch of the library is bracketed by two CUDA events on its stream; reading
// synchronises on the recorded events and sums their elapsed times per class.  Events
// come from a per-device pool that is created on first use and reused; nothing is
// recorded (one relaxed atomic load per launch) while tracing is off.
constexpr size_t kMaxTraceRecords = size_t(1) << 16;
std::atomic<int> g_trace_on{0};
std::mutex g_trace_mu;
struct TraceRec {
  int cls;
  cudaEvent_t a, b;
};
std::vector<TraceRec> g_trace_recs;
std::vector<std::pair<int, cudaEvent_t>> g_trace_pool;  // (device, free event)
long long g_trace_dropped = 0;

// A free event of the current device (under g_trace_mu), or nullptr.
cudaEvent_t trace_event() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  for (size_t i = 0; i < g_trace_pool.size(); ++i) {
    if (g_trace_pool[i].first == dev) {
      cudaEvent_t e = g_trace_pool[i].second;
      g_trace_pool[i] = g_trace_pool.back();
      g_trace_pool.pop_back();
      return e;
    }
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

void trace_release(cudaEvent_t e) {
  int dev = 0;
  cudaGetDevice(&dev);
  g_trace_pool.emplace_back(dev, e);
}

// Brackets the launches of one kernel class in a scope.
class Trace {
 public:
  Trace(int cls, cudaStream_t s) : cls_(cls), s_(s) {
    if (!g_trace_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(g_trace_mu);
    if (g_trace_recs.size() >= kMaxTraceRecords) {
      ++g_trace_dropped;
      return;
    }
    a_ = trace_event();
    if (a_ && cudaEventRecord(a_, s_) != cudaSuccess) {
      trace_release(a_);
      a_ = nullptr;
    }
  }
  ~Trace() {
    if (!a_) return;
    std::lock_guard<std::mutex> lock(g_trace_mu);
    cudaEvent_t b = trace_event();
    if (b && cudaEventRecord(b, s_) == cudaSuccess) {
      g_trace_recs.push_back(TraceRec{cls_, a_, b});
      return;
    }
    trace_release(a_);
    if (b) trace_release(b);
  }
  Trace(const Trace&) = delete;
  Trace& operator=(const Trace&) = delete;

 private:
  int cls_;
  cudaStream_t s_;
  cudaEvent_t a_ = nullptr;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool valid_kind(int k) { return k >= SLM_CE && k <= SLM_CE_ARGMAX_P; }
// Kinds whose loss needs the final log-sum-exps: a second pass over the vocabulary.
bool two_pass_kind(int k) {
  return k == SLM_TV || k == SLM_NLA || k == SLM_LK_HYBRID || k == SLM_JSD;
}

int64_t default_chunk(int64_t N, int64_t d, int64_t chunk_tokens) {
  if (N <= 0) return 0;
  int64_t c = chunk_tokens > 0 ? chunk_tokens : align_up(static_cast<size_t>(2 * d), kBM);
  return std::max<int64_t>(1, std::min<int64_t>(c, N));
}

// Counters of the persistent fused backward (bwd_fused_kernel): one per 256-row M tile of a
// chunk and one per vocabulary run of its logits-gradient schedule.
size_t fused_ctr_count(int64_t C) {
  return 1 + static_cast<size_t>(std::max<int64_t>(1, ceil_div(C, kPairM))) + kMaxRuns + 1;
}

struct Layout {
  size_t status_off, red_off, nblk, ctr_off, big_off, part_off, zy_off, dz_off, ldz;
  size_t fwd_total;  // bytes the forward uses
  size_t bwd_total;  // bytes the backward uses with this chunk size
  size_t total;      // max of the two
};

Layout layout(int kind, int64_t N, int64_t d, int64_t V, int64_t chunk_tokens) {
  Layout L{};
  L.status_off = 0;
  L.nblk = static_cast<size_t>(std::max<int64_t>(1, ceil_div(N, kCombineThreads)));
  L.red_off = kAlign;
  size_t off = align_up(L.red_off + L.nblk * (sizeof(double) + sizeof(long long)), kAlign);
  L.ctr_off = off;
  off = align_up(off + fused_ctr_count(default_chunk(N, d, chunk_tokens)) * sizeof(int), kAlign);
  L.big_off = off;
  const FwdSched f = fwd_sched(kind, V);
  const size_t part = static_cast<size_t>(f.slots) * f.fields * static_cast<size_t>(N) * 4;
  L.part_off = off;
  L.zy_off = align_up(L.part_off + part, kAlign);
  const size_t fwd_end = align_up(L.zy_off + static_cast<size_t>(N) * 4, kAlign);
  L.ldz = align_up(static_cast<size_t>(V), 8);
  L.dz_off = off;  // the backward's chunk buffer reuses the forward's partials region
  const size_t bwd_end =
      align_up(L.dz_off + static_cast<size_t>(default_chunk(N, d, chunk_tokens)) * L.ldz * 2,
               kAlign);
  L.fwd_total = fwd_end;
  L.bwd_total = bwd_end;
  L.total = std::max(fwd_end, bwd_end);
  return L;
}

// ---------------------------------------------------------------------------------------
// Device checks and tensor maps.
// ---------------------------------------------------------------------------------------
int check_device() {
  static int cache[64];
  static std::once_flag once;
  std::call_once(once, [] {
    for (int i = 0; i < 64; ++i) cache[i] = -1;
  });
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SLM_ERR_CUDA;
  if (cache[dev] < 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return SLM_ERR_CUDA;
    cache[dev] = (major == 10 && minor == 0) ? SLM_OK : SLM_ERR_UNSUPPORTED_ARCH;
  }
  return cache[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [outer, inner] matrix with `ld` elements per row;
// box {box_inner, box_outer}, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t ld,
              int box_inner, int box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The same for an fp32 matrix (the fused path's kept logits).
bool make_map_f32(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t ld,
                  int box_inner, int box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 4};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool misaligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; }

// `backward` selects which pass's workspace needs are checked.
int common_checks(int kind, const void* Hq, const void* Hp, const void* W, const int32_t* labels,
                  int64_t N, int64_t d, int64_t V, const void* workspace, size_t ws_bytes,
                  int64_t chunk_tokens, bool backward) {
  if (!valid_kind(kind)) return SLM_ERR_KIND;
  if (N < 0 || d <= 0 || V <= 0 || (d % 8) != 0) return SLM_ERR_SHAPE;
  if (N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31) || d >= (int64_t(1) << 31))
    return SLM_ERR_SHAPE;
  if (!W || !workspace) return SLM_ERR_NULL;
  if (N > 0) {
    if (!Hq) return SLM_ERR_NULL;
    if (dual_kind(kind) && !Hp) return SLM_ERR_NULL;
    if (kind == SLM_CE && !labels) return SLM_ERR_NULL;
  }
  if (misaligned(W, 16) || (Hq && misaligned(Hq, 16)) || (dual_kind(kind) && Hp && misaligned(Hp, 16)))
    return SLM_ERR_ALIGN;
  if (misaligned(workspace, kAlign)) return SLM_ERR_WORKSPACE;
  const Layout L = layout(kind, N, d, V, chunk_tokens);
  if (ws_bytes < (backward ? L.bwd_total : L.fwd_total)) return SLM_ERR_WORKSPACE;
  return SLM_OK;
}

// Weighted combinations: a workspace laid out like the single-kind one, with union
// partials (kUnionFields per slot), the label logits, the per-term losses [kNumKinds][N],
// and per-block sums of the total and of every term.
struct ComboLayout {
  size_t status_off, red_off, nblk, cnt_off, ctr_off, part_off, zy_off, tl_off, dz_off, ldz;
  size_t fwd_total, bwd_total, total;
};

ComboLayout combo_layout(int64_t N, int64_t d, int64_t V, int64_t chunk_tokens) {
  ComboLayout L{};
  L.status_off = 0;
  L.nblk = static_cast<size_t>(std::max<int64_t>(1, ceil_div(N, kCombineThreads)));
  L.red_off = kAlign;
  L.cnt_off = align_up(L.red_off + L.nblk * (1 + kNumKinds) * sizeof(double), 16);
  L.ctr_off = align_up(L.cnt_off + L.nblk * sizeof(long long), kAlign);
  const size_t big = align_up(
      L.ctr_off + fused_ctr_count(default_chunk(N, d, chunk_tokens)) * sizeof(int), kAlign);
  const FwdSched f = fwd_sched(SLM_KL, V);
  L.part_off = big;
  const size_t part = static_cast<size_t>(f.slots) * kUnionFields * static_cast<size_t>(N) * 4;
  L.zy_off = align_up(L.part_off + part, kAlign);
  L.tl_off = align_up(L.zy_off + static_cast<size_t>(N) * 4, kAlign);
  L.fwd_total = align_up(L.tl_off + static_cast<size_t>(kNumKinds) * N * 4, kAlign);
  L.ldz = align_up(static_cast<size_t>(V), 8);
  L.dz_off = big;
  L.bwd_total =
      align_up(L.dz_off + static_cast<size_t>(default_chunk(N, d, chunk_tokens)) * L.ldz * 2,
               kAlign);
  L.total = std::max(L.fwd_total, L.bwd_total);
  return L;
}

// Validates a weight vector; fills the device copy and reports which operands it needs.
int combo_weights(const float* weights, ComboW* cw, bool* needs_p, bool* needs_labels,
                  bool* two_pass) {
  if (!weights) return SLM_ERR_NULL;
  bool any = false;
  *needs_p = false;
  for (int k = 0; k < kNumKinds; ++k) {
    const float w = weights[k];
    if (!(w == w) || w > 3.0e38f || w < -3.0e38f) return SLM_ERR_KIND;  // NaN or inf
    cw->w[k] = w;
    if (w != 0.f) {
      any = true;
      if (k != SLM_CE) *needs_p = true;
    }
  }
  if (!any) return SLM_ERR_KIND;
  *needs_labels = weights[SLM_CE] != 0.f;
  *two_pass = weights[SLM_TV] != 0.f || weights[SLM_NLA] != 0.f ||
              weights[SLM_LK_HYBRID] != 0.f || weights[SLM_JSD] != 0.f;
  return SLM_OK;
}

int combo_checks(const float* weights, ComboW* cw, bool* two_pass, const void* Hq,
                 const void* Hp, const void* W, const int32_t* labels, int64_t N, int64_t d,
                 int64_t V, const void* workspace, size_t ws_bytes, int64_t chunk_tokens,
                 bool backward) {
  bool needs_p = false, needs_labels = false;
  int st = combo_weights(weights, cw, &needs_p, &needs_labels, two_pass);
  if (st != SLM_OK) return st;
  if (N < 0 || d <= 0 || V <= 0 || (d % 8) != 0) return SLM_ERR_SHAPE;
  if (N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31) || d >= (int64_t(1) << 31))
    return SLM_ERR_SHAPE;
  if (!W || !workspace) return SLM_ERR_NULL;
  if (N > 0) {
    if (!Hq) return SLM_ERR_NULL;
    if (needs_p && !Hp) return SLM_ERR_NULL;
    if (needs_labels && !labels) return SLM_ERR_NULL;
  }
  if (misaligned(W, 16) || (Hq && misaligned(Hq, 16)) || (Hp && misaligned(Hp, 16)))
    return SLM_ERR_ALIGN;
  if (misaligned(workspace, kAlign)) return SLM_ERR_WORKSPACE;
  const ComboLayout L = combo_layout(N, d, V, chunk_tokens);
  if (ws_bytes < (backward ? L.bwd_total : L.fwd_total)) return SLM_ERR_WORKSPACE;
  return SLM_OK;
}

// Fused forward + backward: per chunk of C token rows, the forward GEMM stores the chunk's
// fp32 logits (draft, and target for the dual kinds) and the logits gradient and the second
// pass read them back.  C is a multiple of 256 (the row blocks of the loss reduction).
int64_t fused_chunk(int64_t N, int64_t chunk_tokens) {
  if (N <= 0) return 0;
  int64_t c = chunk_tokens > 0 ? static_cast<int64_t>(align_up(static_cast<size_t>(chunk_tokens), 256))
                               : 4096;
  return std::min<int64_t>(c, N);
}

struct FusedLayout {
  size_t status_off, red_off, nblk, ctr_off, part_off, zy_off, lq_off, lp_off, dz_off, ldl, ldz,
      total;
};

FusedLayout fused_layout(int kind, int64_t N, int64_t V, int64_t chunk_tokens) {
  FusedLayout L{};
  L.status_off = 0;
  L.nblk = static_cast<size_t>(std::max<int64_t>(1, ceil_div(N, kCombineThreads)));
  L.red_off = kAlign;
  size_t off = align_up(L.red_off + L.nblk * (sizeof(double) + sizeof(long long)), kAlign);
  L.ctr_off = off;  // the claim counter of the persistent dH + dW launch
  off += kAlign;
  const size_t C = static_cast<size_t>(fused_chunk(N, chunk_tokens));
  const FwdSched f = fwd_sched(kind, V);
  L.part_off = off;
  off = align_up(off + static_cast<size_t>(f.slots) * f.fields * C * 4, kAlign);
  L.zy_off = off;
  off = align_up(off + C * 4, kAlign);
  L.ldl = align_up(static_cast<size_t>(V), 4);
  L.lq_off = off;
  off = align_up(off + C * L.ldl * 4, kAlign);
  L.lp_off = off;
  if (dual_kind(kind) && kind != SLM_CE_ARGMAX_P) off = align_up(off + C * L.ldl * 4, kAlign);
  L.ldz = align_up(static_cast<size_t>(V), 8);
  L.dz_off = off;
  off = align_up(off + C * L.ldz * 2, kAlign);
  L.total = off;
  return L;
}

#define SLM_TRY_CUDA(expr)                  \
  do {                                      \
    if ((expr) != cudaSuccess) return SLM_ERR_CUDA; \
  } while (0)

// A kernel launch of the given trace class on the function's stream `s`.
#define SLM_LAUNCH(cls, expr)                         \
  do {                                                \
    Trace slm_trace_scope_(cls, s);                   \
    if ((expr) != cudaSuccess) return SLM_ERR_CUDA;   \
  } while (0)

}  // namespace
}  // namespace slm

using namespace slm;

extern "C" {

int slm_version(void) { return 100; }

const char* slm_status_string(int s) {
  switch (s) {
    case SLM_OK: return "SLM_OK";
    case SLM_ERR_NULL: return "SLM_ERR_NULL: a required pointer is NULL";
    case SLM_ERR_SHAPE: return "SLM_ERR_SHAPE: invalid N, d or V (d must be a positive multiple of 8)";
    case SLM_ERR_ALIGN: return "SLM_ERR_ALIGN: a tensor base is not 16-byte aligned";
    case SLM_ERR_KIND: return "SLM_ERR_KIND: unknown loss kind";
    case SLM_ERR_WORKSPACE: return "SLM_ERR_WORKSPACE: workspace NULL, misaligned or too small";
    case SLM_ERR_LABEL_RANGE: return "SLM_ERR_LABEL_RANGE: a label outside [0, V) (row masked)";
    case SLM_ERR_TIMEOUT: return "SLM_ERR_TIMEOUT: a device pipeline wait ran out of time";
    case SLM_ERR_CUDA: return "SLM_ERR_CUDA: a CUDA call or launch failed";
    case SLM_ERR_UNSUPPORTED_ARCH: return "SLM_ERR_UNSUPPORTED_ARCH: needs compute capability 10.0 (B200)";
    default: return "SLM: unknown status";
  }
}

size_t slm_stats_floats(int kind) {
  if (!valid_kind(kind)) return 0;
  if (kind == SLM_CE) return 1;
  if (kind == SLM_CE_ARGMAX_P) return 2;
  if (kind == SLM_KL || kind == SLM_RKL) return 3;
  return 5;
}

size_t slm_workspace_bytes(int kind, int64_t N, int64_t d, int64_t V, int64_t chunk_tokens) {
  if (!valid_kind(kind) || N < 0 || d <= 0 || V <= 0 || (d % 8) != 0) return 0;
  return layout(kind, N, d, V, chunk_tokens).total;
}

int slm_loss_fwd(int kind, const void* Hq, const void* Hp, const void* W, const int32_t* labels,
                 int32_t ignore_index, int64_t N, int64_t d, int64_t V, float* loss_tok,
                 float* alpha_tok, double* loss_sum, int64_t* n_valid, float* loss_mean,
                 float* stats, void* workspace, size_t ws_bytes, void* stream) {
  int st = common_checks(kind, Hq, Hp, W, labels, N, d, V, workspace, ws_bytes, 0, false);
  if (st != SLM_OK) return st;
  if (!loss_sum || !n_valid || (N > 0 && !stats)) return SLM_ERR_NULL;
  if ((st = check_device()) != SLM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Layout L = layout(kind, N, d, V, 0);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws + L.status_off);
  double* blk_sum = reinterpret_cast<double*>(ws + L.red_off);
  long long* blk_cnt = reinterpret_cast<long long*>(blk_sum + L.nblk);
  float* part = reinterpret_cast<float*>(ws + L.part_off);
  float* zy = reinterpret_cast<float*>(ws + L.zy_off);
  SLM_TRY_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  const DevCtl ctl = make_ctl(status);

  if (N > 0) {
    const FwdSched f = fwd_sched(kind, V);
    const GemmGeom g = geom(N, V, d, f.bn, f.vc, kGroupPairs, kPairM,
                             SLM_SYNC_KB_V, SLM_SYNC_SLACK_V);
    CUtensorMap tHq, tHp, tW;
    if (!make_map(&tHq, Hq, d, N, d, kBK, kBM)) return SLM_ERR_CUDA;
    if (!make_map(&tW, W, d, V, d, kBK, 128)) return SLM_ERR_CUDA;
    FwdParams p{labels, ignore_index, N, V, part, zy, stats, kind == SLM_JSD ? 1 : 0,
                nullptr, nullptr, 0};
    if (!dual_kind(kind)) {
      SLM_LAUNCH(kTrFwdGemm, launch_fwd_ce(tHq, tW, g, p, ctl, s));
    } else {
      if (!make_map(&tHp, Hp, d, N, d, kBK, kBM)) return SLM_ERR_CUDA;
      if (kind == SLM_CE_ARGMAX_P)
        SLM_LAUNCH(kTrFwdGemm, launch_fwd_argmax(tHq, tHp, tW, g, p, ctl, s));
      else
        SLM_LAUNCH(kTrFwdGemm, launch_fwd_dual(tHq, tHp, tW, g, p, ctl, kind == SLM_RKL, s));
    }
    SLM_LAUNCH(kTrRow, launch_combine(kind, 1, part, f.slots, zy, labels, ignore_index, N, V,
                                loss_tok, alpha_tok, stats, blk_sum, blk_cnt, status, s));
    if (two_pass_kind(kind)) {
      if (kind == SLM_JSD)
        SLM_LAUNCH(kTrPass2Gemm, launch_jsd(tHq, tHp, tW, g, p, ctl, s));
      else
        SLM_LAUNCH(kTrPass2Gemm, launch_alpha(tHq, tHp, tW, g, p, ctl, s));
      SLM_LAUNCH(kTrRow, launch_combine(kind, 2, part, f.slots, zy, labels, ignore_index, N, V,
                                  loss_tok, alpha_tok, stats, blk_sum, blk_cnt, status, s));
    }
    SLM_LAUNCH(kTrRow, launch_finalize(blk_sum, blk_cnt, static_cast<int>(L.nblk), loss_sum, n_valid,
                                 loss_mean, s));
  } else {
    SLM_TRY_CUDA(cudaMemsetAsync(blk_sum, 0, L.nblk * (sizeof(double) + sizeof(long long)), s));
    SLM_LAUNCH(kTrRow, launch_finalize(blk_sum, blk_cnt, static_cast<int>(L.nblk), loss_sum, n_valid,
                                 loss_mean, s));
  }
  return SLM_OK;
}

// One chunk of the backward as one persistent launch (bwd_fused_kernel): the chunk's
// logits gradient (zkind 0: CE, 1: divergences, 2: weighted combination; -1: dZ is already
// in the chunk buffer, only dH and dW run), then dH and dW, ordered by the counters at
// `ctr` (zeroed here).
static int launch_chunk_fused(int zkind, const CUtensorMap& tHq, const CUtensorMap& tHp,
                       const CUtensorMap& tWk, const CUtensorMap& tDzK, const CUtensorMap& tWmn,
                       const CUtensorMap& tDzMn, const CUtensorMap& tHmn, const FwdSched& f,
                       int64_t rows, int64_t d, int64_t V, int* ctr, const DzParams& pz,
                       const DhParams& ph, const DwParams& pw, const DevCtl& ctl,
                       cudaStream_t s) {
  BwdFusedGeom fg{};
  fg.claim = ctr;
  if (zkind >= 0) {
    fg.gz = geom(rows, V, d, f.bn, f.vc, kGroupPairs, kPairM, SLM_SYNC_KB_V, SLM_SYNC_SLACK_V);
    fg.bn_z = f.bn;
    fg.rows_done = ctr + 1;
    fg.runs_done = ctr + 1 + fg.gz.num_m;
  }
  SLM_TRY_CUDA(
      cudaMemsetAsync(ctr, 0, (1 + fg.gz.num_m + fg.gz.units_n) * sizeof(int), s));
  fg.num_mh = static_cast<int>(ceil_div(rows, kPairM));
  fg.num_nh = static_cast<int>(ceil_div(d, kTileDh));
  fg.kb_h = static_cast<int>(ceil_div(V, kBK));
  fg.num_mw = static_cast<int>(ceil_div(V, kPairM));
  fg.num_nw = static_cast<int>(ceil_div(d, kTileDw));
  fg.kb_w = static_cast<int>(ceil_div(rows, kBK));
  fg.group_h = std::max(1, std::min(group_b(fg.num_nh), fg.num_mh));
  fg.group_w = std::max(1, std::min(group_b(fg.num_nw), fg.num_mw));
  SLM_LAUNCH(kTrBwdFused, launch_bwd_fused(zkind < 0 ? 0 : zkind, tHq, tHp, tWk, tDzK, tWmn,
                                           tDzMn, tHmn, fg, pz, ph, pw, ctl, s));
  return SLM_OK;
}

// The backward of slm_loss_bwd and slm_loss_bwd_overlap.  With `overlap`, the last chunk
// runs its dW GEMM before its dH GEMM, records `dw_ready` (if given) between the two, and
// launches that dH GEMM on `reserve_pairs` fewer CTA pairs.
static int loss_bwd(int kind, const void* Hq, const void* Hp, const void* W,
                    const int32_t* labels, int32_t ignore_index, int64_t N, int64_t d, int64_t V,
                    const float* grad_tok, const float* grad_scale, const int64_t* n_valid,
                    const float* stats, void* dHq, float* dW, int accumulate_dW,
                    int64_t chunk_tokens, void* workspace, size_t ws_bytes, void* stream,
                    bool overlap, cudaEvent_t dw_ready, int reserve_pairs) {
  int st = common_checks(kind, Hq, Hp, W, labels, N, d, V, workspace, ws_bytes, chunk_tokens,
                         true);
  if (st != SLM_OK) return st;
  if (!dW || (N > 0 && (!dHq || !stats))) return SLM_ERR_NULL;
  if ((N > 0 && misaligned(dHq, 16)) || misaligned(dW, 16)) return SLM_ERR_ALIGN;
  if ((st = check_device()) != SLM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Layout L = layout(kind, N, d, V, chunk_tokens);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws + L.status_off);
  __nv_bfloat16* dz = reinterpret_cast<__nv_bfloat16*>(ws + L.dz_off);
  int* ctr = reinterpret_cast<int*>(ws + L.ctr_off);
  SLM_TRY_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  const DevCtl ctl = make_ctl(status);

  if (N == 0) {
    if (!accumulate_dW) SLM_LAUNCH(kTrRow, launch_zero_f32(dW, V * d, s));
    if (dw_ready) SLM_TRY_CUDA(cudaEventRecord(dw_ready, s));
    return SLM_OK;
  }
  const int64_t C = default_chunk(N, d, chunk_tokens);
  // CE against argmax p needs only the draft logits in the backward: it runs the CE
  // logits-gradient kernel with the forward's argmax targets (ignore_index on masked rows)
  // as labels.
  const bool argmax_kind = kind == SLM_CE_ARGMAX_P;
  const int dz_kind = argmax_kind ? SLM_CE : kind;
  const int32_t* dz_labels =
      argmax_kind ? reinterpret_cast<const int32_t*>(stats + N) : labels;
  const FwdSched f = fwd_sched(dz_kind, V);
  CUtensorMap tW_k, tW_mn;
  if (!make_map(&tW_k, W, d, V, d, kBK, 128)) return SLM_ERR_CUDA;
  if (!make_map(&tW_mn, W, d, V, d, 64, 64)) return SLM_ERR_CUDA;
  const int64_t ldz = static_cast<int64_t>(L.ldz);

  for (int64_t c0 = 0; c0 < N; c0 += C) {
    const int64_t rows = std::min<int64_t>(C, N - c0);
    const __nv_bfloat16* hq = static_cast<const __nv_bfloat16*>(Hq) + c0 * d;
    // 1) Recompute the chunk's logits and write its logits gradient dZ [rows, V] (bf16).
    CUtensorMap tHq, tHp;
    if (!make_map(&tHq, hq, d, rows, d, kBK, kBM)) return SLM_ERR_CUDA;
    const GemmGeom gz = geom(rows, V, d, f.bn, f.vc, kGroupPairs, kPairM,
                             SLM_SYNC_KB_V, SLM_SYNC_SLACK_V);
    DzParams pz{dz_kind, dz_labels, ignore_index, c0, rows, N, V, stats, grad_tok, grad_scale,
                n_valid, dz, ldz, ComboW{}};
    // The epilogue stores dZ in 32-row x 64-column blocks through this map.
    if (!make_map(&pz.dz_map, dz, V, rows, ldz, 64, 32)) return SLM_ERR_CUDA;
    CUtensorMap tDz_k, tDz_mn, tH_mn;
    if (!make_map(&tDz_k, dz, V, rows, ldz, kBK, kBM)) return SLM_ERR_CUDA;
    if (!make_map(&tDz_mn, dz, V, rows, ldz, 64, 64)) return SLM_ERR_CUDA;
    if (!make_map(&tH_mn, hq, d, rows, d, 64, 64)) return SLM_ERR_CUDA;
    DhParams ph{static_cast<__nv_bfloat16*>(dHq), c0, rows, d};
    DwParams pw{dW, V, d, (accumulate_dW || c0 > 0) ? 1 : 0};
    const bool last_overlapped = overlap && c0 + rows >= N;
    if (!last_overlapped && g_bwd_mode.load() == 1) {
      // 1-3) in one persistent launch (with the overlap, every chunk but the last: that
      // one runs its dW GEMM before its dH GEMM, below).
      if (dual_kind(dz_kind)) {
        const __nv_bfloat16* hp = static_cast<const __nv_bfloat16*>(Hp) + c0 * d;
        if (!make_map(&tHp, hp, d, rows, d, kBK, kBM)) return SLM_ERR_CUDA;
      } else {
        tHp = tHq;
      }
      st = launch_chunk_fused(dual_kind(dz_kind) ? 1 : 0, tHq, tHp, tW_k, tDz_k, tW_mn, tDz_mn,
                              tH_mn, f, rows, d, V, ctr, pz, ph, pw, ctl, s);
      if (st != SLM_OK) return st;
      continue;
    }
    // 1) as its own launch.
    if (!dual_kind(dz_kind)) {
      SLM_LAUNCH(kTrDzGemm, launch_dz_ce(tHq, tW_k, gz, pz, ctl, s));
    } else {
      const __nv_bfloat16* hp = static_cast<const __nv_bfloat16*>(Hp) + c0 * d;
      if (!make_map(&tHp, hp, d, rows, d, kBK, kBM)) return SLM_ERR_CUDA;
      SLM_LAUNCH(kTrDzGemm, launch_dz_dual(tHq, tHp, tW_k, gz, pz, ctl, s));
    }
    // 2) dH[chunk] = dZ W   (M = rows, N = d, K = V; W read MN-major).
    GemmGeom gh = geom(rows, d, V, kTileDh, 1, 1, kPairM, SLM_SYNC_KB_B, SLM_SYNC_SLACK_B);
    // 3) dW (+)= dZ^T H[chunk]   (M = V, N = d, K = rows; both operands MN-major).
    const GemmGeom gw = geom(V, d, rows, kTileDw, 1, 1, kPairM,
                              SLM_SYNC_KB_B, SLM_SYNC_SLACK_B);
    if (last_overlapped) {
      // Last chunk: dW is final once its GEMM is done; the dH GEMM that follows leaves
      // SMs free for the caller's reduction of dW.
      SLM_LAUNCH(kTrDwGemm, launch_dw(tDz_mn, tH_mn, gw, pw, ctl, s));
      if (dw_ready) SLM_TRY_CUDA(cudaEventRecord(dw_ready, s));
      gh.reserve_pairs = reserve_pairs;
      SLM_LAUNCH(kTrDhGemm, launch_dh(tDz_k, tW_mn, gh, ph, ctl, s));
    } else {
      SLM_LAUNCH(kTrDhGemm, launch_dh(tDz_k, tW_mn, gh, ph, ctl, s));
      SLM_LAUNCH(kTrDwGemm, launch_dw(tDz_mn, tH_mn, gw, pw, ctl, s));
    }
  }
  return SLM_OK;
}

int slm_loss_bwd(int kind, const void* Hq, const void* Hp, const void* W, const int32_t* labels,
                 int32_t ignore_index, int64_t N, int64_t d, int64_t V, const float* grad_tok,
                 const float* grad_scale, const int64_t* n_valid, const float* stats, void* dHq,
                 float* dW, int accumulate_dW, int64_t chunk_tokens, void* workspace,
                 size_t ws_bytes, void* stream) {
  return loss_bwd(kind, Hq, Hp, W, labels, ignore_index, N, d, V, grad_tok, grad_scale,
                  n_valid, stats, dHq, dW, accumulate_dW, chunk_tokens, workspace, ws_bytes,
                  stream, false, nullptr, 0);
}

int slm_loss_bwd_overlap(int kind, const void* Hq, const void* Hp, const void* W,
                         const int32_t* labels, int32_t ignore_index, int64_t N, int64_t d,
                         int64_t V, const float* grad_tok, const float* grad_scale,
                         const int64_t* n_valid, const float* stats, void* dHq, float* dW,
                         int accumulate_dW, int64_t chunk_tokens, void* workspace,
                         size_t ws_bytes, void* stream, void* dw_ready_event, int reserve_sms) {
  if (reserve_sms < 0 || reserve_sms > kMaxReserveSms) return SLM_ERR_SHAPE;
  return loss_bwd(kind, Hq, Hp, W, labels, ignore_index, N, d, V, grad_tok, grad_scale,
                  n_valid, stats, dHq, dW, accumulate_dW, chunk_tokens, workspace, ws_bytes,
                  stream, true, static_cast<cudaEvent_t>(dw_ready_event), (reserve_sms + 1) / 2);
}

int slm_align_labels(const int32_t* tokens, const uint8_t* loss_mask, const int32_t* seq_ids,
                     int64_t B, int64_t S, int32_t shift, int32_t ignore_index,
                     int32_t* labels, void* stream) {
  if (B < 0 || S < 0 || shift < 0 || B * S >= (int64_t(1) << 40)) return SLM_ERR_SHAPE;
  if (B * S == 0) return SLM_OK;
  if (!tokens || !labels) return SLM_ERR_NULL;
  int st = check_device();
  if (st != SLM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SLM_LAUNCH(kTrRow, launch_align_labels(tokens, loss_mask, seq_ids, B, S, shift, ignore_index,
                                         labels, s));
  return SLM_OK;
}

size_t slm_flatness_workspace_bytes(int64_t N, int64_t d, int64_t V) {
  if (N < 0 || d <= 0 || V <= 0 || (d % 8) != 0) return 0;
  const FwdSched f = fwd_sched(SLM_CE, V);
  return kAlign + align_up(static_cast<size_t>(f.slots) * kFlatFields *
                               static_cast<size_t>(std::max<int64_t>(N, 1)) * 4,
                           kAlign);
}

int slm_target_flatness(const void* Hp, const void* W, int64_t N, int64_t d, int64_t V,
                        float* flat, void* workspace, size_t ws_bytes, void* stream) {
  if (N < 0 || d <= 0 || V <= 0 || (d % 8) != 0) return SLM_ERR_SHAPE;
  if (N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31)) return SLM_ERR_SHAPE;
  if (N == 0) return SLM_OK;
  if (!Hp || !W || !flat || !workspace) return SLM_ERR_NULL;
  if (misaligned(Hp, 16) || misaligned(W, 16)) return SLM_ERR_ALIGN;
  if (misaligned(workspace, kAlign) || ws_bytes < slm_flatness_workspace_bytes(N, d, V))
    return SLM_ERR_WORKSPACE;
  int st = check_device();
  if (st != SLM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  float* part = reinterpret_cast<float*>(ws + kAlign);
  SLM_TRY_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  const DevCtl ctl = make_ctl(status);
  const FwdSched f = fwd_sched(SLM_CE, V);
  const GemmGeom g = geom(N, V, d, f.bn, f.vc, kGroupPairs, kPairM,
                             SLM_SYNC_KB_V, SLM_SYNC_SLACK_V);
  CUtensorMap tHp, tW;
  if (!make_map(&tHp, Hp, d, N, d, kBK, kBM)) return SLM_ERR_CUDA;
  if (!make_map(&tW, W, d, V, d, kBK, 128)) return SLM_ERR_CUDA;
  FwdParams p{nullptr, 0, N, V, part, nullptr, nullptr, 0, nullptr, nullptr, 0};
  SLM_LAUNCH(kTrFwdGemm, launch_fwd_flat(tHp, tW, g, p, ctl, s));
  SLM_LAUNCH(kTrRow, launch_flat_combine(part, f.slots, N, V, flat, s));
  return SLM_OK;
}

size_t slm_fused_workspace_bytes(int kind, int64_t N, int64_t d, int64_t V,
                                 int64_t chunk_tokens) {
  if (!valid_kind(kind) || N < 0 || d <= 0 || V <= 0 || (d % 8) != 0) return 0;
  return fused_layout(kind, N, V, chunk_tokens).total;
}

int64_t slm_chunk_for_budget(int kind, int64_t N, int64_t d, int64_t V, size_t budget_bytes,
                             int fused) {
  if (!valid_kind(kind) || N <= 0 || d <= 0 || V <= 0 || (d % 8) != 0) return 0;
  const int64_t step = fused ? 256 : kBM;
  auto ws = [&](int64_t c) {
    return fused ? slm_fused_workspace_bytes(kind, N, d, V, c)
                 : slm_workspace_bytes(kind, N, d, V, c);
  };
  if (ws(step) > budget_bytes) return 0;
  // The workspace grows with the chunk: bisect over multiples of `step` up to all N rows.
  int64_t lo = 1, hi = ceil_div(N, step);
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) / 2;
    if (ws(mid * step) <= budget_bytes)
      lo = mid;
    else
      hi = mid - 1;
  }
  // A chunk of all N rows is the largest that can be used: never report more.
  return std::min<int64_t>(lo * step, N);
}

int slm_loss_fwd_bwd(int kind, const void* Hq, const void* Hp, const void* W,
                     const int32_t* labels, int32_t ignore_index, int64_t N, int64_t d,
                     int64_t V, const float* grad_tok, const float* grad_scale, float* loss_tok,
                     float* alpha_tok, double* loss_sum, int64_t* n_valid, float* loss_mean,
                     float* stats, void* dHq, float* dW, int accumulate_dW,
                     int64_t chunk_tokens, void* workspace, size_t ws_bytes, void* stream) {
  // Shapes, pointers and alignment as for the two-call path; the workspace is checked below.
  int st = common_checks(kind, Hq, Hp, W, labels, N, d, V, workspace, SIZE_MAX, 0, false);
  if (st != SLM_OK) return st;
  if (!loss_sum || !n_valid || !dW || (N > 0 && (!stats || !dHq))) return SLM_ERR_NULL;
  if ((N > 0 && misaligned(dHq, 16)) || misaligned(dW, 16)) return SLM_ERR_ALIGN;
  const FusedLayout L = fused_layout(kind, N, V, chunk_tokens);
  if (ws_bytes < L.total) return SLM_ERR_WORKSPACE;
  if ((st = check_device()) != SLM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws + L.status_off);
  double* blk_sum = reinterpret_cast<double*>(ws + L.red_off);
  long long* blk_cnt = reinterpret_cast<long long*>(blk_sum + L.nblk);
  float* part = reinterpret_cast<float*>(ws + L.part_off);
  float* zy = reinterpret_cast<float*>(ws + L.zy_off);
  float* lq = reinterpret_cast<float*>(ws + L.lq_off);
  float* lp = reinterpret_cast<float*>(ws + L.lp_off);
  __nv_bfloat16* dz = reinterpret_cast<__nv_bfloat16*>(ws + L.dz_off);
  const int64_t ldl = static_cast<int64_t>(L.ldl);
  const int64_t ldz = static_cast<int64_t>(L.ldz);
  SLM_TRY_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  const DevCtl ctl = make_ctl(status);
  if (N == 0) {
    SLM_TRY_CUDA(cudaMemsetAsync(blk_sum, 0, L.nblk * (sizeof(double) + sizeof(long long)), s));
    SLM_LAUNCH(kTrRow, launch_finalize(blk_sum, blk_cnt, static_cast<int>(L.nblk), loss_sum, n_valid,
                                 loss_mean, s));
    if (!accumulate_dW) SLM_LAUNCH(kTrRow, launch_zero_f32(dW, V * d, s));
    return SLM_OK;
  }
  // The mean's denominator is needed before the first chunk's gradient.
  SLM_LAUNCH(kTrRow, launch_count_valid(labels, ignore_index, N, V, kind == SLM_CE ? 1 : 0, n_valid, s));
  const int64_t C = fused_chunk(N, chunk_tokens);
  const FwdSched f = fwd_sched(kind, V);
  const bool argmax_kind = kind == SLM_CE_ARGMAX_P;
  const int dz_kind = argmax_kind ? SLM_CE : kind;
  const int32_t* dz_labels = argmax_kind ? reinterpret_cast<const int32_t*>(stats + N) : labels;
  CUtensorMap tW, tW_mn;
  if (!make_map(&tW, W, d, V, d, kBK, 128)) return SLM_ERR_CUDA;
  if (!make_map(&tW_mn, W, d, V, d, 64, 64)) return SLM_ERR_CUDA;
  for (int64_t c0 = 0; c0 < N; c0 += C) {
    const int64_t rows = std::min<int64_t>(C, N - c0);
    const __nv_bfloat16* hq = static_cast<const __nv_bfloat16*>(Hq) + c0 * d;
    CUtensorMap tHq, tHp, tDz_k, tDz_mn, tH_mn;
    if (!make_map(&tHq, hq, d, rows, d, kBK, kBM)) return SLM_ERR_CUDA;
    // 1) Logits of the chunk: statistics in the epilogue, fp32 logits kept.
    const GemmGeom g = geom(rows, V, d, f.bn, f.vc, kGroupPairs, kPairM,
                             SLM_SYNC_KB_V, SLM_SYNC_SLACK_V);
    FwdParams p{labels ? labels + c0 : nullptr, ignore_index, rows, V, part, zy, nullptr, 0,
                lq, (dual_kind(kind) && !argmax_kind) ? lp : nullptr, ldl};
    // The epilogue stores the kept logits in 32 x 32 blocks through these maps.
    if (!make_map_f32(&p.lq_map, lq, V, rows, ldl, 32, 32)) return SLM_ERR_CUDA;
    if (p.lp_out && !make_map_f32(&p.lp_map, lp, V, rows, ldl, 32, 32)) return SLM_ERR_CUDA;
    if (!dual_kind(kind)) {
      SLM_LAUNCH(kTrFwdGemm, launch_fwd_ce(tHq, tW, g, p, ctl, s));
    } else {
      const __nv_bfloat16* hp = static_cast<const __nv_bfloat16*>(Hp) + c0 * d;
      if (!make_map(&tHp, hp, d, rows, d, kBK, kBM)) return SLM_ERR_CUDA;
      if (argmax_kind)
        SLM_LAUNCH(kTrFwdGemm, launch_fwd_argmax(tHq, tHp, tW, g, p, ctl, s));
      else
        SLM_LAUNCH(kTrFwdGemm, launch_fwd_dual(tHq, tHp, tW, g, p, ctl, kind == SLM_RKL, s));
    }
    SLM_LAUNCH(kTrRow, launch_combine(kind, 1, part, f.slots, zy, labels, ignore_index, rows, V,
                                loss_tok, alpha_tok, stats, blk_sum, blk_cnt, status, s, c0, N));
    // 2) Second pass of the alpha losses / JSD over the kept logits.
    if (two_pass_kind(kind)) {
      SLM_LAUNCH(kTrLogitsRow, launch_logits_pass2(kind, lq, lp, ldl, stats, c0, N, rows, V, part, s));
      SLM_LAUNCH(kTrRow, launch_combine(kind, 2, part, 1, zy, labels, ignore_index, rows, V, loss_tok,
                                  alpha_tok, stats, blk_sum, blk_cnt, status, s, c0, N));
    }
    // 3) Logits gradient of the chunk from the kept logits.
    DzParams pz{dz_kind, dz_labels, ignore_index, c0, rows, N, V, stats, grad_tok, grad_scale,
                n_valid, dz, ldz, ComboW{}};
    SLM_LAUNCH(kTrLogitsRow, launch_logits_dz(pz, lq, lp, ldl, s));
    // 4) dH[chunk] = dZ W and dW (+)= dZ^T H[chunk].
    if (!make_map(&tDz_k, dz, V, rows, ldz, kBK, kBM)) return SLM_ERR_CUDA;
    if (!make_map(&tDz_mn, dz, V, rows, ldz, 64, 64)) return SLM_ERR_CUDA;
    if (!make_map(&tH_mn, hq, d, rows, d, 64, 64)) return SLM_ERR_CUDA;
    DhParams ph{static_cast<__nv_bfloat16*>(dHq), c0, rows, d};
    DwParams pw{dW, V, d, (accumulate_dW || c0 > 0) ? 1 : 0};
    if (g_bwd_mode.load() == 1) {
      // Both GEMMs in one persistent launch (dZ is already complete: no counters).
      st = launch_chunk_fused(-1, tHq, tHq, tW, tDz_k, tW_mn, tDz_mn, tH_mn, f, rows, d, V,
                              reinterpret_cast<int*>(ws + L.ctr_off), pz, ph, pw, ctl, s);
      if (st != SLM_OK) return st;
      continue;
    }
    const GemmGeom gh = geom(rows, d, V, kTileDh, 1, 1, kPairM,
                              SLM_SYNC_KB_B, SLM_SYNC_SLACK_B);
    SLM_LAUNCH(kTrDhGemm, launch_dh(tDz_k, tW_mn, gh, ph, ctl, s));
    const GemmGeom gw = geom(V, d, rows, kTileDw, 1, 1, kPairM,
                              SLM_SYNC_KB_B, SLM_SYNC_SLACK_B);
    SLM_LAUNCH(kTrDwGemm, launch_dw(tDz_mn, tH_mn, gw, pw, ctl, s));
  }
  SLM_LAUNCH(kTrRow, launch_finalize(blk_sum, blk_cnt, static_cast<int>(L.nblk), loss_sum, n_valid,
                               loss_mean, s));
  return SLM_OK;
}

size_t slm_combo_workspace_bytes(int64_t N, int64_t d, int64_t V, int64_t chunk_tokens) {
  if (N < 0 || d <= 0 || V <= 0 || (d % 8) != 0) return 0;
  return combo_layout(N, d, V, chunk_tokens).total;
}

int slm_combo_fwd(const float* weights, const void* Hq, const void* Hp, const void* W,
                  const int32_t* labels, int32_t ignore_index, int64_t N, int64_t d, int64_t V,
                  float* loss_tok, float* term_loss_tok, double* loss_sum,
                  double* term_loss_sum, int64_t* n_valid, float* loss_mean, float* stats,
                  void* workspace, size_t ws_bytes, void* stream) {
  ComboW cw;
  bool two_pass = false;
  int st = combo_checks(weights, &cw, &two_pass, Hq, Hp, W, labels, N, d, V, workspace,
                        ws_bytes, 0, false);
  if (st != SLM_OK) return st;
  if (!loss_sum || !n_valid || (N > 0 && !stats)) return SLM_ERR_NULL;
  if ((st = check_device()) != SLM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ComboLayout L = combo_layout(N, d, V, 0);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws + L.status_off);
  double* blk_sums = reinterpret_cast<double*>(ws + L.red_off);
  long long* blk_cnt = reinterpret_cast<long long*>(ws + L.cnt_off);
  float* part = reinterpret_cast<float*>(ws + L.part_off);
  float* zy = reinterpret_cast<float*>(ws + L.zy_off);
  float* tl = reinterpret_cast<float*>(ws + L.tl_off);
  SLM_TRY_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  const DevCtl ctl = make_ctl(status);
  if (N > 0) {
    const FwdSched f = fwd_sched(SLM_KL, V);
    const GemmGeom g = geom(N, V, d, f.bn, f.vc, kGroupPairs, kPairM,
                             SLM_SYNC_KB_V, SLM_SYNC_SLACK_V);
    // A CE-only combination has no target: the draft stands in for it (its statistics are
    // computed and unused).
    const void* hp = Hp ? Hp : Hq;
    CUtensorMap tHq, tHp, tW;
    if (!make_map(&tHq, Hq, d, N, d, kBK, kBM)) return SLM_ERR_CUDA;
    if (!make_map(&tHp, hp, d, N, d, kBK, kBM)) return SLM_ERR_CUDA;
    if (!make_map(&tW, W, d, V, d, kBK, 128)) return SLM_ERR_CUDA;
    FwdParams p{labels, ignore_index, N, V, part, zy, stats, cw.w[SLM_JSD] != 0.f ? 1 : 0,
                nullptr, nullptr, 0};
    SLM_LAUNCH(kTrFwdGemm, launch_fwd_union(tHq, tHp, tW, g, p, ctl, s));
    SLM_LAUNCH(kTrRow, launch_combo_combine(1, cw, part, f.slots, zy, labels, ignore_index, N, V,
                                      stats, tl, status, s));
    if (two_pass) {
      SLM_LAUNCH(kTrPass2Gemm, launch_pass2_union(tHq, tHp, tW, g, p, ctl, s));
      SLM_LAUNCH(kTrRow, launch_combo_combine(2, cw, part, f.slots, zy, labels, ignore_index, N, V,
                                        stats, tl, status, s));
    }
  }
  SLM_LAUNCH(kTrRow, launch_combo_total(cw, tl, labels, ignore_index, N, V, loss_tok, term_loss_tok,
                                  blk_sums, blk_cnt, s));
  SLM_LAUNCH(kTrRow, launch_combo_finalize(blk_sums, blk_cnt, static_cast<int>(L.nblk), loss_sum,
                                     term_loss_sum, n_valid, loss_mean, s));
  return SLM_OK;
}

int slm_combo_bwd(const float* weights, const void* Hq, const void* Hp, const void* W,
                  const int32_t* labels, int32_t ignore_index, int64_t N, int64_t d, int64_t V,
                  const float* grad_tok, const float* grad_scale, const int64_t* n_valid,
                  const float* stats, void* dHq, float* dW, int accumulate_dW,
                  int64_t chunk_tokens, void* workspace, size_t ws_bytes, void* stream) {
  ComboW cw;
  bool two_pass = false;
  int st = combo_checks(weights, &cw, &two_pass, Hq, Hp, W, labels, N, d, V, workspace,
                        ws_bytes, chunk_tokens, true);
  if (st != SLM_OK) return st;
  if (!dW || (N > 0 && (!dHq || !stats))) return SLM_ERR_NULL;
  if ((N > 0 && misaligned(dHq, 16)) || misaligned(dW, 16)) return SLM_ERR_ALIGN;
  if ((st = check_device()) != SLM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ComboLayout L = combo_layout(N, d, V, chunk_tokens);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws + L.status_off);
  __nv_bfloat16* dz = reinterpret_cast<__nv_bfloat16*>(ws + L.dz_off);
  int* ctr = reinterpret_cast<int*>(ws + L.ctr_off);
  SLM_TRY_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  const DevCtl ctl = make_ctl(status);
  if (N == 0) {
    if (!accumulate_dW) SLM_LAUNCH(kTrRow, launch_zero_f32(dW, V * d, s));
    return SLM_OK;
  }
  const int64_t C = default_chunk(N, d, chunk_tokens);
  const FwdSched f = fwd_sched(SLM_KL, V);
  const int64_t ldz = static_cast<int64_t>(L.ldz);
  const void* hp_all = Hp ? Hp : Hq;
  CUtensorMap tW_k, tW_mn;
  if (!make_map(&tW_k, W, d, V, d, kBK, 128)) return SLM_ERR_CUDA;
  if (!make_map(&tW_mn, W, d, V, d, 64, 64)) return SLM_ERR_CUDA;
  for (int64_t c0 = 0; c0 < N; c0 += C) {
    const int64_t rows = std::min<int64_t>(C, N - c0);
    const __nv_bfloat16* hq = static_cast<const __nv_bfloat16*>(Hq) + c0 * d;
    const __nv_bfloat16* hp = static_cast<const __nv_bfloat16*>(hp_all) + c0 * d;
    CUtensorMap tHq, tHp, tDz_k, tDz_mn, tH_mn;
    if (!make_map(&tHq, hq, d, rows, d, kBK, kBM)) return SLM_ERR_CUDA;
    if (!make_map(&tHp, hp, d, rows, d, kBK, kBM)) return SLM_ERR_CUDA;
    const GemmGeom gz = geom(rows, V, d, f.bn, f.vc, kGroupPairs, kPairM,
                             SLM_SYNC_KB_V, SLM_SYNC_SLACK_V);
    DzParams pz{-1, labels, ignore_index, c0, rows, N, V, stats, grad_tok, grad_scale,
                n_valid, dz, ldz, cw};
    if (!make_map(&tDz_k, dz, V, rows, ldz, kBK, kBM)) return SLM_ERR_CUDA;
    if (!make_map(&tDz_mn, dz, V, rows, ldz, 64, 64)) return SLM_ERR_CUDA;
    if (!make_map(&tH_mn, hq, d, rows, d, 64, 64)) return SLM_ERR_CUDA;
    DhParams ph{static_cast<__nv_bfloat16*>(dHq), c0, rows, d};
    DwParams pw{dW, V, d, (accumulate_dW || c0 > 0) ? 1 : 0};
    if (g_bwd_mode.load() == 1) {
      st = launch_chunk_fused(2, tHq, tHp, tW_k, tDz_k, tW_mn, tDz_mn, tH_mn, f, rows, d, V,
                              ctr, pz, ph, pw, ctl, s);
      if (st != SLM_OK) return st;
      continue;
    }
    SLM_LAUNCH(kTrDzGemm, launch_dz_combo(tHq, tHp, tW_k, gz, pz, ctl, s));
    const GemmGeom gh = geom(rows, d, V, kTileDh, 1, 1, kPairM,
                              SLM_SYNC_KB_B, SLM_SYNC_SLACK_B);
    SLM_LAUNCH(kTrDhGemm, launch_dh(tDz_k, tW_mn, gh, ph, ctl, s));
    const GemmGeom gw = geom(V, d, rows, kTileDw, 1, 1, kPairM,
                              SLM_SYNC_KB_B, SLM_SYNC_SLACK_B);
    SLM_LAUNCH(kTrDwGemm, launch_dw(tDz_mn, tH_mn, gw, pw, ctl, s));
  }
  return SLM_OK;
}

int slm_count_valid(int kind, const int32_t* labels, int32_t ignore_index, int64_t N,
                    int64_t V, int64_t* n_valid, void* stream) {
  if (!valid_kind(kind)) return SLM_ERR_KIND;
  if (N < 0 || V <= 0 || N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31))
    return SLM_ERR_SHAPE;
  if (!n_valid || (kind == SLM_CE && N > 0 && !labels)) return SLM_ERR_NULL;
  int st = check_device();
  if (st != SLM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SLM_LAUNCH(kTrRow, launch_count_valid(N > 0 ? labels : nullptr, ignore_index, N, V,
                                        kind == SLM_CE ? 1 : 0, n_valid, s));
  return SLM_OK;
}

int slm_set_backward_mode(int mode) {
  if (mode < 0 || mode > 1) return -1;
  return g_bwd_mode.exchange(mode);
}

int slm_trace_enable(int on) {
  g_trace_on.store(on ? 1 : 0);
  return SLM_OK;
}

int slm_trace_read(double* ms, int64_t* launches, int n_classes) {
  if (n_classes < 0 || ((!ms || !launches) && n_classes > 0)) return SLM_ERR_NULL;
  std::lock_guard<std::mutex> lock(g_trace_mu);
  for (int c = 0; c < n_classes; ++c) {
    ms[c] = 0.0;
    launches[c] = 0;
  }
  int st = SLM_OK;
  for (const TraceRec& r : g_trace_recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      st = SLM_ERR_CUDA;
    else if (r.cls < n_classes) {
      ms[r.cls] += t;
      launches[r.cls] += 1;
    }
    trace_release(r.a);
    trace_release(r.b);
  }
  g_trace_recs.clear();
  if (g_trace_dropped != 0 && st == SLM_OK) st = SLM_ERR_WORKSPACE;
  g_trace_dropped = 0;
  return st;
}

int slm_debug_exp2(const float* x, float* y_fma, float* y_mufu, int64_t n, void* stream) {
  if (n < 0 || n >= (int64_t(1) << 31)) return SLM_ERR_SHAPE;
  if (n == 0) return SLM_OK;
  if (!x || !y_fma || !y_mufu) return SLM_ERR_NULL;
  int st = check_device();
  if (st != SLM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SLM_LAUNCH(kTrRow, launch_exp2_pair(x, y_fma, y_mufu, n, s));
  return SLM_OK;
}

int slm_debug_set(int fault_mode, long long timeout_cycles) {
  if (fault_mode < 0 || fault_mode > 2 || timeout_cycles < 0) return SLM_ERR_SHAPE;
  g_fault.store(fault_mode);
  g_timeout.store(timeout_cycles > 0 ? timeout_cycles : kTimeoutCycles);
  return SLM_OK;
}

int slm_device_status(const void* workspace, void* stream) {
  if (!workspace) return SLM_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SLM_ERR_CUDA;
  int flags = 0;
  int* status = reinterpret_cast<int*>(const_cast<void*>(workspace));
  if (cudaMemcpy(&flags, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SLM_ERR_CUDA;
  if (flags != 0 && cudaMemset(status, 0, sizeof(int)) != cudaSuccess) return SLM_ERR_CUDA;
  if (flags & kFlagTimeout) return SLM_ERR_TIMEOUT;
  if (flags & kFlagLabelRange) return SLM_ERR_LABEL_RANGE;
  return SLM_OK;
}

}  // extern "C"
