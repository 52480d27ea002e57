// slm_kernels.cu - sm_100a kernels of the streaming LM-head loss.
//
// One warp-specialised persistent GEMM skeleton serves every contraction of the path.  A
// cluster of two CTAs (one per SM) shares each tensor-core MMA (tcgen05.mma.cta_group::2,
// M = 256): CTA r of the pair holds rows [128 r, 128 r + 128) of the A operand tile and
// half of every B slice in its own shared memory, and receives its 128 accumulator rows
// in its own tensor memory (TMEM).
//   warp 0      TMA producer (both CTAs): 2-D tiled loads with 128-byte swizzle into a
//               ring of shared-memory stages; both CTAs' copies complete on the leader
//               CTA's "full" barrier;
//   warp 1      MMA issuer (leader CTA only): one lane issues the pair's MMAs (bf16 x bf16
//               -> fp32) and releases ring stages and accumulators in both CTAs with
//               multicast tcgen05.commit;
//   warps 2..   epilogue (both CTAs): one or two warpgroups, one thread per tile row, each
//               warpgroup over its share of the tile's columns, reading TMEM with
//               tcgen05.ld and applying the fused epilogue.  Epilogues that write wide
//               outputs stage each warp's block in swizzled shared memory and hand it to
//               one TMA bulk store.
// Work units (M tile, run of N tiles[, K slice]) go to the pairs round robin; the pairs of
// the GEMMs over the vocabulary keep a loose lockstep so that W tiles are shared in L2.
// The epilogues are what make the path streaming ("Training speculative decoders:
// removing the logits and attention bottlenecks", "Streaming Cross Entropy" and
// "Backward pass"): logits tiles live only in TMEM and registers.
//   EpiFwdCE    online row max / sum of exp and the label logit          (CE forward)
//   EpiFwdDualT the same for target and draft plus the forward-KL (A) and/or reverse-KL
//               (B) accumulator                                          (KL / RKL forward,
//               first pass of the alpha losses and of JSD)
//   EpiFwdArgmax draft log-sum-exp plus the target's running argmax      (CE against argmax p)
//   EpiAlpha    alpha = sum min(p, q) and S = sum_{q<p} q                 (second pass)
//   EpiJsd      the two halves of the Jensen-Shannon divergence         (second pass)
//   EpiDz       the logits gradient, rounded to bf16 into the chunk buffer (backward)
//   EpiDh       dH chunk rows (bf16)                                      (dH = dZ W)
//   EpiDwT      fp32 read-add-write of disjoint dW tiles, no atomics      (dW += dZ^T H)
//   EpiFwdUnion, EpiPass2Union, EpiDzCombo   the same for weighted combinations
//   EpiFlat     sum of exp and of its square                             (target flatness)
// In the fused single call the forward epilogues also store the chunk's fp32 logits.
// Every pipeline wait is bounded: on expiry the kernel records kFlagTimeout, lets its own
// copies and MMAs finish, frees TMEM and returns.

#include <math.h>

#include <algorithm>
#include <atomic>
#include <utility>

#include "slm_internal.h"
#include "sm100.cuh"

namespace slm {
using namespace sm100;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kTmemCols = 512;

// Bounded wait executed by all 32 lanes of a warp; the result is warp-uniform.
// honor_abort = false is used for the final waits on a CTA's own in-flight work.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          const DevCtl& ctl, bool honor_abort = true) {
  const uint32_t a = smem_u32(bar);
  bool done = mbar_try_wait(a, parity);
  if (!done) {
    const long long t0 = clock64();
    while (true) {
      done = mbar_try_wait(a, parity);
      if (done) break;
      if (honor_abort && *abort) break;
      if (clock64() - t0 > ctl.timeout_cycles) {
        *abort = 1;
        atomicOr(ctl.status, kFlagTimeout);
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, done);
}

// Work unit u -> (pair M tile mt, vocabulary run j).  Units are handed to the pairs round
// robin, so the pairs that start together share B tiles only while their units have the
// same length.  The runs of vc tiles come first, in raster groups of group_m M tiles with M
// fastest (the pairs running the same run j at once read the same W tiles); the short last
// run of every row (when vc does not divide num_n) is deferred to the end of the schedule,
// where its small units also even out the pairs' finishing times.
__device__ __forceinline__ void unit_coords(const GemmGeom& g, int u, int& mt, int& j) {
  const int full_runs = (g.num_n % g.vc) != 0 ? g.units_n - 1 : g.units_n;
  const int n_full = g.num_m * full_runs;
  if (u >= n_full) {
    mt = u - n_full;
    j = full_runs;
    return;
  }
  const int per_group = g.group_m * full_runs;
  const int grp = u / per_group;
  const int r = u - grp * per_group;
  const int gm = min(g.group_m, g.num_m - grp * g.group_m);
  j = r / gm;
  mt = grp * g.group_m + (r - j * gm);
}

// Loose lockstep of the pairs.  Pairs that read the same W tiles at nearly the same time
// share them in L2; left alone they drift apart by more than a tile's L2 residency, and W
// is then fetched from DRAM once per pair.  The leader CTA's producer of every pair records
// its progress (K blocks issued, in steps of g.sync_kb) under the launch's tag and lets no
// pair run more than g.slack steps ahead of the slowest started pair.
constexpr int kMaxSyncPairs = 128;
constexpr long long kSyncSpinCycles = 1LL << 21;
__device__ unsigned long long g_pair_progress[kMaxSyncPairs];

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Records that this pair begins progress step `step` (from 1) and waits until every started
// pair of this launch has begun step `step - slack`.  Pairs with no record under this
// launch's tag (not resident yet) and finished pairs (step 0xffffffff) hold nobody back.
// The wait only shapes performance: after kSyncSpinCycles it gives up, marks this pair as
// finished for the others and returns false, and the caller stops synchronising.
// Warp-collective.
__device__ __forceinline__ bool lockstep(const GemmGeom& g, int pair, int npairs,
                                         uint32_t step, const DevCtl& ctl) {
  // Test hook (fault == 2): give up at the first wait, as a pair held back too long would.
  const long long spin = ctl.fault == 2 ? 0 : kSyncSpinCycles;
  const int lane = threadIdx.x & 31;
  const unsigned long long tag = static_cast<unsigned long long>(g.epoch) << 32;
  if (lane == 0) st_relaxed_u64(&g_pair_progress[pair], tag | step);
  __syncwarp();
  if (step <= static_cast<uint32_t>(g.slack)) return true;
  const uint32_t need = step - static_cast<uint32_t>(g.slack);
  const long long t0 = clock64();
  while (true) {
    uint32_t mn = 0xffffffffu;
    for (int i = lane; i < npairs; i += 32) {
      const unsigned long long v = ld_relaxed_u64(&g_pair_progress[i]);
      if ((v >> 32) == g.epoch) mn = min(mn, static_cast<uint32_t>(v));
    }
    mn = __reduce_min_sync(0xffffffffu, mn);
    if (mn >= need) return true;
    if (__any_sync(0xffffffffu, clock64() - t0 >= spin)) {
      if (lane == 0) st_relaxed_u64(&g_pair_progress[pair], tag | 0xffffffffull);
      __syncwarp();
      return false;
    }
    __nanosleep(128);
  }
}

// ----------------------------------------------------------------------------------------
// Pair GEMM configuration.
//   BNI    N of one MMA instruction (<= 256); each CTA holds BNI / 2 of it ("B slice")
//   NSUB   MMA instructions along N per accumulator: tile N = NSUB * BNI
//   NUM_A  A operands sharing the B tile, one accumulator each (1, or 2 for target+draft)
//   NBUF   TMEM accumulator buffers (2: the epilogue of one tile overlaps the next tile's
//          MMAs; 1: wider tiles, fewer bytes from L2 per flop)
//   NWG    epilogue warpgroups, each over 1/NWG of the tile's columns
// ----------------------------------------------------------------------------------------
template <int STAGES>
struct PairCtl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t fin;
  uint32_t tmem_base;
  int abort;
};

template <int BNI, int NSUB, int NUM_A, int NBUF, int NWG, bool A_MN, bool B_MN, int STAGES>
struct PairCfg {
  static constexpr int kTileN = NSUB * BNI;
  static constexpr int kSliceN = BNI / 2;
  static constexpr uint32_t kABytes = kBM * kBK * 2;
  static constexpr uint32_t kSliceBytes = kSliceN * kBK * 2;
  static constexpr uint32_t kStageBytes = NUM_A * kABytes + NSUB * kSliceBytes;
  static constexpr uint32_t kAccCols = NUM_A * kTileN;  // TMEM columns per buffer
  static constexpr int kThreads = 64 + 128 * NWG;
  static constexpr int kEpiCols = kTileN / NWG;  // columns per epilogue warpgroup
  static constexpr size_t kSmem =
      1024 + STAGES * static_cast<size_t>(kStageBytes) + sizeof(PairCtl<STAGES>);
  static_assert(NBUF * kAccCols <= kTmemCols, "accumulator buffers must fit in TMEM");
  static_assert(BNI % 128 == 0 && BNI <= 256, "UMMA N (M = 256) and whole 64-wide B boxes");
  static_assert(kEpiCols % 32 == 0, "epilogue column share");
  // The bytes the leader's "full" barrier expects per CTA equal the boxes the producer
  // issues per stage: per A operand one 64 x 128 box (K-major) or two 64 x 64 boxes
  // (MN-major), per B slice one 64 x kSliceN box (K-major) or kSliceN / 64 boxes of 64 x 64
  // (MN-major); bf16 throughout.
  static constexpr uint32_t kABoxBytes = A_MN ? 2u * 64u * 64u * 2u : 64u * kBM * 2u;
  static constexpr uint32_t kBBoxBytes =
      B_MN ? static_cast<uint32_t>(kSliceN / 64) * 64u * 64u * 2u : 64u * kSliceN * 2u;
  static_assert(NUM_A * kABoxBytes + NSUB * kBBoxBytes == kStageBytes,
                "expect_tx must count exactly the bytes the producer loads");
  static_assert(kSmem <= 232448, "shared memory per CTA");
};

// Bytes of shared staging per epilogue warp an epilogue asks for (kStageBytesPerWarp).
template <class E, class = void>
struct EpiStageBytes {
  static constexpr int value = 0;
};
template <class E>
struct EpiStageBytes<E, decltype(void(E::kStageBytesPerWarp))> {
  static constexpr int value = E::kStageBytesPerWarp;
};

// Epilogues that set kSplitHalves take a single-buffered two-sub-tile accumulator in two
// halves (see gemm_pair_kernel): each warpgroup drains its share of the first sub-tile,
// releases it, then drains its share of the second.  Their tile() must accept any
// 32-column-aligned sub-range [c0, c1) and not depend on the order in which ranges come.
template <class E, class = void>
struct EpiSplit {
  static constexpr bool value = false;
};
template <class E>
struct EpiSplit<E, decltype(void(E::kSplitHalves))> {
  static constexpr bool value = E::kSplitHalves;
};

// Epilogues with asynchronous work of their own (bulk stores) declare finish(), which the
// kernel calls once after the epilogue's last tile.
template <class E, class = void>
struct EpiHasFinish {
  static constexpr bool value = false;
};
template <class E>
struct EpiHasFinish<E, decltype(std::declval<E&>().finish())> {
  static constexpr bool value = true;
};

template <int BNI, int NSUB, int NUM_A, int NBUF, int NWG, bool A_MN, bool B_MN, int STAGES,
          class Epi>
__global__ void __launch_bounds__(64 + 128 * NWG, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0,
                     const __grid_constant__ CUtensorMap tmA1,
                     const __grid_constant__ CUtensorMap tmB, const GemmGeom g,
                     const __grid_constant__ typename Epi::Params ep, const DevCtl ctl) {
  using C = PairCfg<BNI, NSUB, NUM_A, NBUF, NWG, A_MN, B_MN, STAGES>;
  constexpr int kTileN = C::kTileN;
  constexpr int kSliceN = C::kSliceN;
  constexpr uint32_t kABytes = C::kABytes;
  constexpr uint32_t kSliceBytes = C::kSliceBytes;
  constexpr uint32_t kStageBytes = C::kStageBytes;
  constexpr uint32_t kAccCols = C::kAccCols;
  constexpr uint32_t kIdesc = idesc_bf16_f32(2 * kBM, BNI, A_MN, B_MN);
  // Split accumulator (single buffer, two N sub-tiles, an epilogue that takes halves): the
  // sub-tiles have their own "empty" barriers, so the next tile's MMAs for sub-tile 0 start
  // while the epilogue still drains sub-tile 1.  (Halving the N = 256 MMAs of the
  // two-operand tiles the same way measured slower: N = 128 MMAs read each A tile from
  // shared memory twice per K step, which with the TMA writes exceeds the shared-memory
  // port.)
  constexpr bool kSplit = NBUF == 1 && NSUB == 2 && EpiSplit<Epi>::value;
  static_assert(!kSplit || (!A_MN && !B_MN), "split accumulators: K-major operands");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  PairCtl<STAGES>* pc = reinterpret_cast<PairCtl<STAGES>*>(smem + STAGES * kStageBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&pc->full[s], 1);
      mbar_init(&pc->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&pc->tfull[b], 1);
      mbar_init(&pc->tempty[b], 2 * 4 * NWG);  // one arrive per epilogue warp, both CTAs
    }
    mbar_init(&pc->fin, 1);
    pc->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    if (NUM_A == 2) tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(&pc->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  // Both CTAs' barriers exist before either CTA touches the other's.
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = pc->tmem_base;
  volatile int* abort = &pc->abort;

  if (warp == 0) {
    // ------------------------------ TMA producer (both CTAs) ------------------------------
    uint32_t it = 0;
    bool ok = true;
    const bool sync_pub = g.epoch != 0 && leader && pair < kMaxSyncPairs && npairs <= kMaxSyncPairs;
    bool sync_on = sync_pub;
    uint32_t sync_step = 0;
    for (int u = pair; ok && u < g.num_units; u += npairs) {
      int mt, j;
      unit_coords(g, u, mt, j);
      const int mrow = mt * 2 * kBM + static_cast<int>(rank) * kBM;
      const int n_end = min((j + 1) * g.vc, g.num_n);
      for (int nt = j * g.vc; ok && nt < n_end; ++nt) {
        for (int kb = 0; kb < g.k_blocks; ++kb, ++it) {
          if (sync_on && it % static_cast<uint32_t>(g.sync_kb) == 0)
            sync_on = lockstep(g, pair, npairs, ++sync_step, ctl);
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_warp(&pc->empty[s], ph ^ 1u, abort, ctl)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            uint8_t* st = smem + s * kStageBytes;
            if (leader) mbar_arrive_expect_tx(&pc->full[s], 2 * kStageBytes);
            const int k0 = kb * kBK;
#pragma unroll
            for (int a = 0; a < NUM_A; ++a) {
              const CUtensorMap* map = (a == 0) ? &tmA0 : &tmA1;
              uint8_t* dst = st + a * kABytes;
              if (A_MN) {
                tma_load_2d_pair(dst, map, &pc->full[s], mrow, k0);
                tma_load_2d_pair(dst + 8192, map, &pc->full[s], mrow + 64, k0);
              } else {
                tma_load_2d_pair(dst, map, &pc->full[s], k0, mrow);
              }
            }
#pragma unroll
            for (int sub = 0; sub < NSUB; ++sub) {
              uint8_t* bdst = st + NUM_A * kABytes + sub * kSliceBytes;
              const int ncol = nt * kTileN + sub * BNI + static_cast<int>(rank) * kSliceN;
              if (B_MN) {
#pragma unroll
                for (int jb = 0; jb < kSliceN / 64; ++jb)
                  tma_load_2d_pair(bdst + jb * 8192, &tmB, &pc->full[s], ncol + jb * 64, k0);
              } else {
                tma_load_2d_pair(bdst, &tmB, &pc->full[s], k0, ncol);
              }
            }
          }
          __syncwarp();
        }
      }
    }
    if (sync_pub && lane == 0)
      st_relaxed_u64(&g_pair_progress[pair],
                     (static_cast<unsigned long long>(g.epoch) << 32) | 0xffffffffull);
    if (ok) {
      // Producer tail: the leader's MMA warp releases every stage of BOTH CTAs with a
      // multicast commit that arrives on this CTA's "empty" barrier once the stage's MMAs
      // are done.  Wait for the releases of the last STAGES stages, so that no such remote
      // arrive can reach this CTA's shared memory after it has exited.
      // If the pair is aborting, the last releases may never come: then give the ones in
      // flight a moment instead.
      const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
      bool tail_ok = true;
      for (uint32_t i = first; tail_ok && i < it; ++i)
        tail_ok = wait_warp(&pc->empty[i % STAGES], (i / STAGES) & 1u, abort, ctl);
      if (!tail_ok)
        for (int i = 0; i < 100; ++i) __nanosleep(1000);
    } else {
      if (leader) {
        // The full barriers count both CTAs' copies: waiting on them lets the pair's
        // copies in flight land before either CTA leaves the final cluster barrier.
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
        for (uint32_t i = first; i < it; ++i)
          wait_warp(&pc->full[i % STAGES], (i / STAGES) & 1u, abort, ctl, false);
      } else {
        // The non-leader's copies complete on the leader's barriers, which this CTA cannot
        // wait on: give any copy still in flight (issued at most STAGES stages ahead of the
        // last one the leader counted) time to land before the final cluster barrier.
        for (int i = 0; i < 100; ++i) __nanosleep(1000);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (leader only) ------------------------------
    if (leader) {
      uint32_t it = 0, t = 0;
      bool ok = true;
      for (int u = pair; ok && u < g.num_units; u += npairs) {
        int mt, j;
        unit_coords(g, u, mt, j);
        const int n_end = min((j + 1) * g.vc, g.num_n);
        for (int nt = j * g.vc; ok && nt < n_end; ++nt, ++t) {
          const int b = (NBUF == 2) ? static_cast<int>(t & 1u) : 0;
          const uint32_t ub = (NBUF == 2) ? ((t >> 1) & 1u) : (t & 1u);
          if (!wait_warp(&pc->tempty[b], ub ^ 1u, abort, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dcol = tmem + b * kAccCols;
          if constexpr (kSplit) {
            // Sub-tile h's MMAs of one stage (first = the tile's first K block).
            auto issue_half = [&](int st, int h, bool first) {
              const uint32_t a_addr = smem_u32(smem + st * kStageBytes);
              const uint32_t bs = a_addr + NUM_A * kABytes + h * kSliceBytes;
#pragma unroll
              for (int kk = 0; kk < kBK / 16; ++kk) {
                const uint64_t bd = smem_desc_sw128(bs + kk * 32, 16, 1024);
#pragma unroll
                for (int a = 0; a < NUM_A; ++a) {
                  const uint64_t ad = smem_desc_sw128(a_addr + a * kABytes + kk * 32, 16, 1024);
                  umma_bf16_pair(dcol + (a * NSUB + h) * BNI, ad, bd, kIdesc,
                                 (!first || kk != 0) ? 1u : 0u);
                }
              }
            };
            // Sub-tile 0 over the first `pre` K blocks (the stages the producer filled while
            // the epilogue drained), then, once sub-tile 1 is free, its MMAs for those K
            // blocks with each stage's release, then both sub-tiles per K block.
            const int pre = min(STAGES, g.k_blocks);
            const uint32_t it0 = it;
            for (int kb = 0; ok && kb < pre; ++kb) {
              const int st = (it0 + kb) % STAGES;
              if (!wait_warp(&pc->full[st], ((it0 + kb) / STAGES) & 1u, abort, ctl)) {
                ok = false;
                break;
              }
              tc_fence_after();
              if (lane == 0) issue_half(st, 0, kb == 0);
              __syncwarp();
            }
            if (!ok) break;
            if (!wait_warp(&pc->tempty[1], ub ^ 1u, abort, ctl)) {
              ok = false;
              break;
            }
            tc_fence_after();
            for (int kb = 0; kb < pre; ++kb) {
              const int st = (it0 + kb) % STAGES;
              if (lane == 0) {
                issue_half(st, 1, kb == 0);
                umma_commit_pair_mc(&pc->empty[st], 0x3);
              }
              __syncwarp();
            }
            it = it0 + pre;
            for (int kb = pre; kb < g.k_blocks; ++kb, ++it) {
              const int st = it % STAGES;
              if (!wait_warp(&pc->full[st], (it / STAGES) & 1u, abort, ctl)) {
                ok = false;
                break;
              }
              tc_fence_after();
              if (lane == 0) {
                issue_half(st, 0, false);
                issue_half(st, 1, false);
                umma_commit_pair_mc(&pc->empty[st], 0x3);
              }
              __syncwarp();
            }
          } else {
            for (int kb = 0; kb < g.k_blocks; ++kb, ++it) {
              const int s = it % STAGES;
              const uint32_t ph = (it / STAGES) & 1u;
              if (!wait_warp(&pc->full[s], ph, abort, ctl)) {
                ok = false;
                break;
              }
              tc_fence_after();
              if (lane == 0) {
                const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
                const uint32_t b_addr = a_addr + NUM_A * kABytes;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
                  for (int sub = 0; sub < NSUB; ++sub) {
                    const uint32_t bs = b_addr + sub * kSliceBytes;
                    const uint64_t bd = B_MN ? smem_desc_sw128(bs + kk * 2048, 8192, 1024)
                                             : smem_desc_sw128(bs + kk * 32, 16, 1024);
#pragma unroll
                    for (int a = 0; a < NUM_A; ++a) {
                      const uint32_t aa = a_addr + a * kABytes;
                      const uint64_t ad = A_MN ? smem_desc_sw128(aa + kk * 2048, 8192, 1024)
                                               : smem_desc_sw128(aa + kk * 32, 16, 1024);
                      umma_bf16_pair(dcol + (a * NSUB + sub) * BNI, ad, bd, kIdesc,
                                     (kb | kk) != 0 ? 1u : 0u);
                    }
                  }
                }
                umma_commit_pair_mc(&pc->empty[s], 0x3);
              }
              __syncwarp();
            }
          }
          if (!ok) break;
          if (lane == 0) umma_commit_pair_mc(&pc->tfull[b], 0x3);
          __syncwarp();
        }
      }
      // Every MMA must be complete (in both CTAs' TMEM) before TMEM is released.
      if (lane == 0) umma_commit_pair_mc(&pc->fin, 0x1);
      __syncwarp();
      wait_warp(&pc->fin, 0u, abort, ctl, false);
    }
  } else {
    // ------------------------------ epilogue (both CTAs) ------------------------------
    const int q = warp & 3;  // a warp may only touch TMEM lanes [32 * (warp % 4), +32)
    const int wg = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(q * 32) << 16;
    const int c0 = wg * C::kEpiCols;
    const int c1 = c0 + C::kEpiCols;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&pc->tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&pc->tempty[1]), 0);
    Epi epi;
    if constexpr (EpiStageBytes<Epi>::value > 0) {
      // Per-warp staging buffers live after the control block, 1024-byte aligned so that
      // their rows follow the 128-byte swizzle pattern of the tensor maps.
      uint8_t* st = reinterpret_cast<uint8_t*>(
          (reinterpret_cast<uintptr_t>(pc + 1) + 1023) & ~static_cast<uintptr_t>(1023));
      epi.stage = reinterpret_cast<float*>(st + (warp - 2) * EpiStageBytes<Epi>::value);
    }
    uint32_t t = 0;
    bool ok = true;
    for (int u = pair; ok && u < g.num_units; u += npairs) {
      int mt, j;
      unit_coords(g, u, mt, j);
      const int row0 = mt * 2 * kBM + static_cast<int>(rank) * kBM;
      const int n_end = min((j + 1) * g.vc, g.num_n);
      epi.unit_begin(ep, row0, row);
      for (int nt = j * g.vc; nt < n_end; ++nt, ++t) {
        const int b = (NBUF == 2) ? static_cast<int>(t & 1u) : 0;
        const uint32_t ub = (NBUF == 2) ? ((t >> 1) & 1u) : (t & 1u);
        if (!wait_warp(&pc->tfull[b], ub, abort, ctl)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Test hook (fault == 1): withhold the release of the first accumulator, so that the
        // MMA issuer's bounded wait for it runs out and the kernel unwinds with a timeout.
        const bool withhold = ctl.fault == 1 && t == 0;
        if constexpr (kSplit) {
          // This warpgroup's share of each sub-tile in turn, each released once drained.
          constexpr int kHalf = kTileN / 2, kPer = kHalf / NWG;
          static_assert(kPer % 32 == 0, "split epilogue share");
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            const int ch = h * kHalf + wg * kPer;
            epi.template tile<kTileN>(ep, tmem + lane_bits, row0,
                                      static_cast<int64_t>(nt) * kTileN, ch, ch + kPer, row);
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && !(withhold && h == 0))
              mbar_arrive_cluster(h ? tempty_leader1 : tempty_leader0);
          }
        } else {
          epi.template tile<kTileN>(ep, tmem + lane_bits + b * kAccCols, row0,
                                    static_cast<int64_t>(nt) * kTileN, c0, c1, row);
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && !withhold) mbar_arrive_cluster(b ? tempty_leader1 : tempty_leader0);
        }
      }
      if (!ok) break;
      epi.unit_end(ep, row0, j * NWG + wg, row);
    }
    if constexpr (EpiHasFinish<Epi>::value) epi.finish();
  }

  // Neither CTA leaves while the other may still signal its barriers or use its TMEM.
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

// ----------------------------------------------------------------------------------------
// Epilogues.  tile<TN>(p, tb, row0, n0, c0, c1, row): this thread owns row `row0 + row`
// of the M operand; accumulator a's column c (of the TN-wide tile that starts at global
// column n0) is at TMEM address tb + a * TN + c; the thread's warpgroup covers columns
// [c0, c1).  unit_end receives the partial slot of (vocabulary run, warpgroup).
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ float max32(const float (&v)[32]) {
  float m0 = fmaxf(v[0], v[1]), m1 = fmaxf(v[2], v[3]);
#pragma unroll
  for (int i = 4; i < 32; i += 4) {
    m0 = fmaxf(m0, fmaxf(v[i], v[i + 1]));
    m1 = fmaxf(m1, fmaxf(v[i + 2], v[i + 3]));
  }
  return fmaxf(m0, m1);
}

// Packed fp32 pairs (sm_100 fma / add / sub / mul .f32x2): two independent fp32 operations,
// each rounded to nearest as its scalar form, in one instruction.  SLM_PACKED_EPI = 0 selects
// the scalar forms (same results, except where a packed pair of partial sums replaces one
// running sum).
#ifndef SLM_PACKED_EPI
#define SLM_PACKED_EPI 1
#endif
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 exp2_2(float2 a) { return make_float2(exp2f(a.x), exp2f(a.y)); }
// log2 of a pair of sums of probabilities; a sum of 0 (both terms underflowed or masked)
// gives -126 instead of -inf, so that the terms it multiplies stay 0.
__device__ __forceinline__ float2 log2_2(float2 a) {
  return make_float2(log2f(fmaxf(a.x, 1.1754944e-38f)), log2f(fmaxf(a.y, 1.1754944e-38f)));
}

// 2^x for x <= 0 on the FMA pipe instead of the MUFU pipe, for a pair of values.  The
// epilogues' exponentials are MUFU-bound while the FMA pipe idles, so a share of them is
// computed this way (a share of the column pairs, see exp2_mix).  x = j + r with j = round(x) (adding 1.5 * 2^23 rounds to an
// integer) and r in [-0.5, 0.5]; 2^r is a degree-5 polynomial in r whose coefficients were
// fitted here to 2^r on [-0.5, 0.5] (relative error weighted least squares on Chebyshev
// nodes: 7.5e-8 in exact arithmetic, 2.2e-7 in fp32 Horner form); 2^j is added into the
// exponent field.  Arguments are clamped at -126 so that the exponent field stays
// non-negative: the result is then at most 2^-126, which only ever enters sums of terms
// >= 1.  Not for -inf arguments (the tail chunks, with masked columns, keep exp2f).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 kr = make_float2(kRound, kRound);
  const float2 t = add2(x, kr);
  const float2 r = sub2(x, sub2(t, kr));
  float2 p = fma2(make_float2(0.001327647129073739f, 0.001327647129073739f), r,
                  make_float2(0.009675540961325169f, 0.009675540961325169f));
  p = fma2(p, r, make_float2(0.05550713092088699f, 0.05550713092088699f));
  p = fma2(p, r, make_float2(0.24022120237350464f, 0.24022120237350464f));
  p = fma2(p, r, make_float2(0.6931469440460205f, 0.6931469440460205f));
  p = fma2(p, r, make_float2(1.0000001192092896f, 1.0000001192092896f));
  const int jx = __float_as_int(t.x) - 0x4B400000;  // j, from the rounded sum's low bits
  const int jy = __float_as_int(t.y) - 0x4B400000;
  return make_float2(__int_as_float(__float_as_int(p.x) + (jx << 23)),
                     __int_as_float(__float_as_int(p.y) + (jy << 23)));
}

// exp2_2 or exp2_fma2 for column pair `pair` of a 32-column chunk: pairs with
// (pair % 8) < eighths take the FMA-pipe form.  `pair` is a constant once the chunk loop is
// unrolled, so the choice costs nothing at run time.
__device__ __forceinline__ float2 exp2_mix(int pair, int eighths, float2 x) {
  return (pair & 7) < eighths ? exp2_fma2(x) : exp2_2(x);
}
// Shares for the kernels with two exponentials per column (target and draft: the second one
// is mixed) and with one (hard-label CE).
#ifndef SLM_EXP2_FMA_DUAL
#define SLM_EXP2_FMA_DUAL 6
#endif
#ifndef SLM_EXP2_FMA_CE
#define SLM_EXP2_FMA_CE 0
#endif

__device__ __forceinline__ void mask_tail(float (&v)[32], int64_t col0, int64_t V,
                                          float fill = -INFINITY) {
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (col0 + i >= V) v[i] = fill;
}

// Fused path: this warp's 32 rows x 32 columns of fp32 logits (each lane holds its row's
// 32 values; `grow` is the lane's row) go to the warp's 4 KB staging block in the 128-byte
// swizzle layout of the store map (16-byte chunk k of row r at position k ^ (r % 8)), and
// from there to global memory with one TMA bulk store.  Columns >= V and rows beyond the
// launch's rows fall outside the map and are not written.  The staging block is rewritten
// only once the previous store has read it.  Warp-collective.
__device__ __forceinline__ void stage_store_f32(float* stage, const CUtensorMap* map,
                                                const float (&v)[32], int64_t col0,
                                                int64_t grow) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
  float4* srow = reinterpret_cast<float4*>(stage + lane * 32);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    srow[k ^ (lane & 7)] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, stage, static_cast<int32_t>(col0), static_cast<int32_t>(grow));
    bulk_commit();
  }
}

// Waits for the warp's outstanding bulk stores (the end of an epilogue that issued some).
__device__ __forceinline__ void finish_bulk_stores() {
  if ((threadIdx.x & 31) == 0) bulk_wait_all();
  __syncwarp();
}

// CE forward: per row, online max m (log2 units) and s = sum 2^(z log2e - m) over the
// warpgroup's columns of the unit's vocabulary run, plus the label logit z_y when the
// label falls there.
struct EpiFwdCE {
  using Params = FwdParams;
  static constexpr bool kSplitHalves = true;
  static constexpr int kStageBytesPerWarp = 4096;
  float* stage;  // this warp's staging buffer (fused path stores)
  float m, s, zyv;
  int32_t lab;
  bool has_zy, row_ok;
  int64_t grow;

  __device__ __forceinline__ void unit_begin(const Params& p, int row0, int row) {
    m = -INFINITY;
    s = 0.f;
    has_zy = false;
    zyv = 0.f;
    grow = static_cast<int64_t>(row0) + row;
    row_ok = grow < p.N;
    lab = row_ok ? p.labels[grow] : -1;
  }

  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int, int64_t n0, int c0,
                                       int c1, int) {
    const int64_t rel = static_cast<int64_t>(lab) - n0;
#pragma unroll 1
    for (int c = c0; c < c1; c += 32) {
      float v[32];
      tmem_ld32(tb + c, v);
      tmem_ld_wait();
      if (n0 + c + 32 > p.V) mask_tail(v, n0 + c, p.V);
      if (p.lq_out && n0 + c < p.V)
        stage_store_f32(stage, &p.lq_map, v, n0 + c, grow - (threadIdx.x & 31));
      if (static_cast<uint64_t>(rel - c) < 32u) {
        const int o = static_cast<int>(rel - c);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i == o) zyv = v[i];
        has_zy = true;
      }
      const float mx = max32(v) * kLog2e;
      if (mx > m) {
        s *= exp2f(m - mx);
        m = mx;
      }
      if (m != -INFINITY) {
#if SLM_PACKED_EPI
        const float2 l2 = make_float2(kLog2e, kLog2e), nm = make_float2(-m, -m);
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 32; i += 2)
          a = add2(a, exp2_mix(i / 2, SLM_EXP2_FMA_CE, fma2(make_float2(v[i], v[i + 1]), l2, nm)));
        s += a.x + a.y;
#else
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          a0 += exp2f(fmaf(v[i], kLog2e, -m));
          a1 += exp2f(fmaf(v[i + 1], kLog2e, -m));
        }
        s += a0 + a1;
#endif
      }
    }
  }

  __device__ __forceinline__ void finish() { finish_bulk_stores(); }

  __device__ __forceinline__ void unit_end(const Params& p, int, int slot, int) {
    if (!row_ok) return;
    p.part[(static_cast<int64_t>(slot) * 2 + 0) * p.N + grow] = m;
    p.part[(static_cast<int64_t>(slot) * 2 + 1) * p.N + grow] = s;
    if (has_zy) p.zy[grow] = zyv;
  }
};

// KL / RKL forward (and the first pass of the alpha losses and of JSD): per row and for
// both the draft (q, accumulator 0) and the target (p, accumulator 1): online max and sum
// of exp; plus A = sum_v 2^(z_p log2e - m_p) (z_p - z_q), rescaled whenever m_p grows, and
// B = sum_v 2^(z_q log2e - m_q) (z_q - z_p), rescaled whenever m_q grows.
// ACC selects the divergence accumulators: 1 = forward KL (A), 2 = reverse KL (B), 3 = both.
template <int ACC>
struct EpiFwdDualT {
  using Params = FwdParams;
  static constexpr int kStageBytesPerWarp = 4096;
  float* stage;  // this warp's staging buffer (fused path stores)
  float mq, sq, mp, sp, A, B;
  bool row_ok;
  int64_t grow;

  __device__ __forceinline__ void unit_begin(const Params& p, int row0, int row) {
    mq = mp = -INFINITY;
    sq = sp = A = B = 0.f;
    grow = static_cast<int64_t>(row0) + row;
    row_ok = grow < p.N;
  }

  template <bool TAIL>
  __device__ __forceinline__ void chunk(float (&vq)[32], float (&vp)[32]) {
    const float xq = max32(vq) * kLog2e;
    const float xp = max32(vp) * kLog2e;
    if (xq > mq) {
      const float r = exp2f(mq - xq);
      sq *= r;
      if (ACC & 2) B *= r;
      mq = xq;
    }
    if (xp > mp) {
      const float r = exp2f(mp - xp);
      sp *= r;
      if (ACC & 1) A *= r;
      mp = xp;
    }
    if (mq == -INFINITY || mp == -INFINITY) return;
#if SLM_PACKED_EPI
    if (!TAIL) {
      // Column pairs: each sum runs as two partial sums (even and odd columns), added at
      // the end of the 32 columns.
      const float2 l2 = make_float2(kLog2e, kLog2e);
      const float2 nmq = make_float2(-mq, -mq), nmp = make_float2(-mp, -mp);
      float2 sq2 = make_float2(0.f, 0.f), sp2 = sq2, a2 = sq2, b2 = sq2;
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float2 zq = make_float2(vq[i], vq[i + 1]);
        const float2 zp = make_float2(vp[i], vp[i + 1]);
        const float2 eq = exp2_2(fma2(zq, l2, nmq));
        const float2 e = exp2_mix(i / 2, SLM_EXP2_FMA_DUAL, fma2(zp, l2, nmp));
        sq2 = add2(sq2, eq);
        sp2 = add2(sp2, e);
        if (ACC & 1) a2 = fma2(e, sub2(zp, zq), a2);
        if (ACC & 2) b2 = fma2(eq, sub2(zq, zp), b2);
      }
      sq += sq2.x + sq2.y;
      sp += sp2.x + sp2.y;
      if (ACC & 1) A += a2.x + a2.y;
      if (ACC & 2) B += b2.x + b2.y;
      return;
    }
#endif
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float eq = exp2f(fmaf(vq[i], kLog2e, -mq));
      const float e = exp2f(fmaf(vp[i], kLog2e, -mp));
      sq += eq;
      sp += e;
      if (TAIL) {
        // Masked columns are -inf in both: their weights are 0 and their difference NaN.
        if ((ACC & 1) && e > 0.f) A = fmaf(e, vp[i] - vq[i], A);
        if ((ACC & 2) && eq > 0.f) B = fmaf(eq, vq[i] - vp[i], B);
      } else {
        const float dpq = vp[i] - vq[i];
        if (ACC & 1) A = fmaf(e, dpq, A);
        if (ACC & 2) B = fmaf(-eq, dpq, B);
      }
    }
  }

  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int, int64_t n0, int c0,
                                       int c1, int) {
#pragma unroll 1
    for (int c = c0; c < c1; c += 32) {
      float vq[32], vp[32];
      tmem_ld32(tb + c, vq);
      tmem_ld32(tb + TN + c, vp);
      tmem_ld_wait();
      const bool tail = n0 + c + 32 > p.V;
      if (tail) {
        mask_tail(vq, n0 + c, p.V);
        mask_tail(vp, n0 + c, p.V);
      }
      // Fused path: the draft block's store overlaps this chunk's arithmetic, which reads
      // vq and vp only; the target block follows.
      const bool store = p.lq_out && n0 + c < p.V;
      const int64_t wrow = grow - (threadIdx.x & 31);
      if (store) stage_store_f32(stage, &p.lq_map, vq, n0 + c, wrow);
      if (tail)
        chunk<true>(vq, vp);
      else
        chunk<false>(vq, vp);
      if (store && p.lp_out) stage_store_f32(stage, &p.lp_map, vp, n0 + c, wrow);
    }
  }

  __device__ __forceinline__ void finish() { finish_bulk_stores(); }

  __device__ __forceinline__ void unit_end(const Params& p, int, int slot, int) {
    if (!row_ok) return;
    float* base = p.part + static_cast<int64_t>(slot) * kDualFields * p.N + grow;
    base[0 * p.N] = mq;
    base[1 * p.N] = sq;
    base[2 * p.N] = mp;
    base[3 * p.N] = sp;
    base[4 * p.N] = A;
    base[5 * p.N] = B;
  }
};

using EpiFwdDual = EpiFwdDualT<3>;

// CE against argmax p (forward): online max / sum of exp of the draft logits, and the
// target's running argmax over the slot's columns (the first, i.e. lowest, column wins
// ties: columns are visited in increasing order and only a strictly larger value
// replaces), with the draft logit at that column.
struct EpiFwdArgmax {
  using Params = FwdParams;
  static constexpr int kStageBytesPerWarp = 4096;
  float* stage;  // this warp's staging buffer (fused path stores)
  float mq, sq, pmax, zqa;
  int pidx;
  bool row_ok;
  int64_t grow;

  __device__ __forceinline__ void unit_begin(const Params& p, int row0, int row) {
    mq = pmax = -INFINITY;
    sq = zqa = 0.f;
    pidx = -1;
    grow = static_cast<int64_t>(row0) + row;
    row_ok = grow < p.N;
  }

  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int, int64_t n0, int c0,
                                       int c1, int) {
#pragma unroll 1
    for (int c = c0; c < c1; c += 32) {
      float vq[32], vp[32];
      tmem_ld32(tb + c, vq);
      tmem_ld32(tb + TN + c, vp);
      tmem_ld_wait();
      if (n0 + c + 32 > p.V) {
        mask_tail(vq, n0 + c, p.V);
        mask_tail(vp, n0 + c, p.V);
      }
      if (p.lq_out && n0 + c < p.V)
        stage_store_f32(stage, &p.lq_map, vq, n0 + c, grow - (threadIdx.x & 31));
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (vp[i] > pmax) {
          pmax = vp[i];
          pidx = static_cast<int>(n0 + c + i);
          zqa = vq[i];
        }
      }
      const float mx = max32(vq) * kLog2e;
      if (mx > mq) {
        sq *= exp2f(mq - mx);
        mq = mx;
      }
      if (mq != -INFINITY) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          a0 += exp2f(fmaf(vq[i], kLog2e, -mq));
          a1 += exp2f(fmaf(vq[i + 1], kLog2e, -mq));
        }
        sq += a0 + a1;
      }
    }
  }

  __device__ __forceinline__ void unit_end(const Params& p, int, int slot, int) {
    if (!row_ok) return;
    float* base = p.part + static_cast<int64_t>(slot) * kArgmaxFields * p.N + grow;
    base[0 * p.N] = mq;
    base[1 * p.N] = sq;
    base[2 * p.N] = pmax;
    base[3 * p.N] = __int_as_float(pidx);
    base[4 * p.N] = zqa;
  }

  __device__ __forceinline__ void finish() { finish_bulk_stores(); }
};

// Second pass of the alpha losses: with the final log-sum-exps L_q and L_p known,
// alpha += min(p_v, q_v) and S += q_v where q_v < p_v.
struct EpiAlpha {
  using Params = FwdParams;
  float lq2, lp2, al, S;
  bool row_ok;
  int64_t grow;

  __device__ __forceinline__ void unit_begin(const Params& p, int row0, int row) {
    al = S = 0.f;
    grow = static_cast<int64_t>(row0) + row;
    row_ok = grow < p.N;
    lq2 = row_ok ? p.stats[grow] * kLog2e : 0.f;
    lp2 = row_ok ? p.stats[p.N + grow] * kLog2e : 0.f;
  }

  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int, int64_t n0, int c0,
                                       int c1, int) {
#pragma unroll 1
    for (int c = c0; c < c1; c += 32) {
      float vq[32], vp[32];
      tmem_ld32(tb + c, vq);
      tmem_ld32(tb + TN + c, vp);
      tmem_ld_wait();
      if (n0 + c + 32 > p.V) {
        mask_tail(vq, n0 + c, p.V);
        mask_tail(vp, n0 + c, p.V);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float qv = exp2f(fmaf(vq[i], kLog2e, -lq2));
        const float pv = exp2f(fmaf(vp[i], kLog2e, -lp2));
        al += fminf(pv, qv);
        S += (qv < pv) ? qv : 0.f;
      }
    }
  }

  __device__ __forceinline__ void unit_end(const Params& p, int, int slot, int) {
    if (!row_ok) return;
    p.part[(static_cast<int64_t>(slot) * 2 + 0) * p.N + grow] = al;
    p.part[(static_cast<int64_t>(slot) * 2 + 1) * p.N + grow] = S;
  }
};

// Second pass of JSD: with L_q and L_p known, per column p, q and M = (p + q) / 2;
// jp += p (log p - log M) and jq += q (log q - log M), where log p = z_p - L_p exactly.
// JSD = (jp + jq) / 2; the backward also needs T = sum_v q_v a_v = jq / 2 with
// a_v = (log q_v - log M_v) / 2.
struct EpiJsd {
  using Params = FwdParams;
  float lq, lp, lq2, lp2, jp, jq;
  bool row_ok;
  int64_t grow;

  __device__ __forceinline__ void unit_begin(const Params& p, int row0, int row) {
    jp = jq = 0.f;
    grow = static_cast<int64_t>(row0) + row;
    row_ok = grow < p.N;
    lq = row_ok ? p.stats[grow] : 0.f;
    lp = row_ok ? p.stats[p.N + grow] : 0.f;
    lq2 = lq * kLog2e;
    lp2 = lp * kLog2e;
  }

  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int, int64_t n0, int c0,
                                       int c1, int) {
#pragma unroll 1
    for (int c = c0; c < c1; c += 32) {
      float vq[32], vp[32];
      tmem_ld32(tb + c, vq);
      tmem_ld32(tb + TN + c, vp);
      tmem_ld_wait();
      if (n0 + c + 32 > p.V) {
        // A finite fill: both exponentials of a masked column are 0 and so are its terms
        // (a -inf logit would give 0 * -inf).
        mask_tail(vq, n0 + c, p.V, -1e30f);
        mask_tail(vp, n0 + c, p.V, -1e30f);
      }
      const float2 l2 = make_float2(kLog2e, kLog2e);
      const float2 nq = make_float2(-lq2, -lq2), np = make_float2(-lp2, -lp2);
      float2 ap2 = make_float2(0.f, 0.f), aq2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float2 a = fma2(make_float2(vp[i], vp[i + 1]), l2, np);  // log2 p
        const float2 b = fma2(make_float2(vq[i], vq[i + 1]), l2, nq);  // log2 q
        // log2 p - log2 M = a + w and log2 q - log2 M = b + w, w = 1 - log2(p + q).
        const float2 pv = exp2_2(a), qv = exp2_2(b);
        const float2 w = sub2(make_float2(1.f, 1.f), log2_2(add2(pv, qv)));
        ap2 = fma2(pv, add2(a, w), ap2);
        aq2 = fma2(qv, add2(b, w), aq2);
      }
      jp += ap2.x + ap2.y;
      jq += aq2.x + aq2.y;
    }
  }

  // jp and jq were summed in log2 units.
  __device__ __forceinline__ void unit_end(const Params& p, int, int slot, int) {
    if (!row_ok) return;
    p.part[(static_cast<int64_t>(slot) * 2 + 0) * p.N + grow] = jp * kLn2;
    p.part[(static_cast<int64_t>(slot) * 2 + 1) * p.N + grow] = jq * kLn2;
  }
};

// Upstream gradient of one row: valid * grad_tok * grad_scale / max(n_valid, 1).
__device__ __forceinline__ float row_grad(const DzParams& p, int64_t n, bool valid) {
  if (!valid) return 0.f;
  float g = p.grad_tok ? p.grad_tok[n] : 1.f;
  if (p.grad_scale) g *= *p.grad_scale;
  if (p.n_valid) {
    const long long nv = static_cast<long long>(*p.n_valid);
    g /= static_cast<float>(nv > 0 ? nv : 1);
  }
  return g;
}

__device__ __forceinline__ void store_bf16_row32(__nv_bfloat16* dst, const float (&v)[32],
                                                 int64_t col0, int64_t limit) {
  if (col0 + 32 <= limit) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t w[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * k + 2 * h], v[8 * k + 2 * h + 1]);
        w[h] = *reinterpret_cast<uint32_t*>(&b2);
      }
      d4[k] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (col0 + i < limit) dst[i] = __float2bfloat16_rn(v[i]);
  }
}

// Backward logits-gradient tile: recomputed logits -> dZ (bf16) of the token chunk.
//   CE (and CE against argmax p, whose targets come from the forward):
//            dz_j = g (q_j - [j = y])
//   KL, TV, NLA, LK (mode 0):  dz_j = ck (q_j - p_j) + cm q_j (m_j - S),  m_j = [q_j < p_j]
//            KL: ck = g, cm = 0;  TV: ck = 0, cm = -g;  NLA: ck = 0, cm = -g / alpha;
//            LK: ck = g lambda, cm = -g (1 - lambda), lambda = exp(-3 alpha) (detached).
//   RKL (mode 1):  dz_j = g q_j (log q_j - log p_j - RKL) = g q_j (z_q - z_p - c),
//            c = L_q - L_p + RKL.
//   JSD (mode 2):  dz_j = g q_j (a_j - T),  a_j = (log q_j - log M_j) / 2.
template <bool DUAL>
struct EpiDz {
  using Params = DzParams;
  // Per warp: a 32-row x 64-column bf16 block of dZ, laid out as the dZ tensor map's
  // 128-byte swizzle expects (16-byte chunk k of row r at position k ^ (r % 8)), written to
  // the chunk buffer by one TMA store.
  static constexpr int kStageBytesPerWarp = 4096;
  float* stage;
  float lq, lp, lq2, lp2, g, ck, cm, S;
  int32_t lab;
  int mode;
  bool row_ok;
  int64_t lrow;

  __device__ __forceinline__ void unit_begin(const Params& p, int row0, int row) {
    lrow = static_cast<int64_t>(row0) + row;
    row_ok = lrow < p.rows;
    const int64_t n = p.row0 + lrow;
    lq = lp = lq2 = lp2 = g = ck = cm = S = 0.f;
    lab = -1;
    mode = 0;
    if (!row_ok) return;
    bool valid = true;
    if (p.labels) {
      lab = p.labels[n];
      valid = lab != p.ignore_index;
      if (!DUAL && (lab < 0 || lab >= p.V)) valid = false;
    }
    g = row_grad(p, n, valid);
    lq = p.stats[n];
    lq2 = lq * kLog2e;
    if (DUAL) {
      lp = p.stats[p.N + n];
      lp2 = lp * kLog2e;
      if (p.kind == kKL) {
        ck = g;  // mode 0: dz = g (q - p)
      } else if (p.kind == kRKL) {
        mode = 1;
        ck = g;
        cm = lq - lp + p.stats[2 * p.N + n];  // c
      } else if (p.kind == kJSD) {
        mode = 2;
        ck = g;
        S = p.stats[4 * p.N + n];  // T
      } else {
        mode = 3;
        const float al = p.stats[3 * p.N + n];
        S = p.stats[4 * p.N + n];
        if (p.kind == kTV) {
          cm = -g;
        } else if (p.kind == kNLA) {
          cm = -g / fmaxf(al, 1e-30f);
        } else {
          const float lam = expf(-3.f * al);
          ck = g * lam;
          cm = -g * (1.f - lam);
        }
      }
    }
  }

  // vq (draft logits of columns [col0, col0 + 32)) becomes dz; vp holds the target logits
  // of the same columns (unused for CE).
  // fma_cols: which columns take the FMA-pipe 2^x for the target (KL): -1 = element i is
  // column col0 + i with col0 a multiple of 32 (the GEMM epilogue), so the share rule of
  // exp2_mix applies by position; 0 / 1 = every element of this call is / is not in such a
  // column (the row kernel, whose elements come from columns with one rule per thread).
  // Either way a column's exponential is computed the same way on both paths.
  __device__ __forceinline__ void apply(float (&vq)[32], const float (&vp)[32], int64_t col0,
                                        int fma_cols = -1) const {
    if (DUAL) {
      {
        if (mode == 0) {
#if SLM_PACKED_EPI
          const float2 l2 = make_float2(kLog2e, kLog2e);
          const float2 nq = make_float2(-lq2, -lq2), np = make_float2(-lp2, -lp2);
          const float2 ck2 = make_float2(ck, ck);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 qv = exp2_2(fma2(make_float2(vq[i], vq[i + 1]), l2, nq));
            const float2 ap = fma2(make_float2(vp[i], vp[i + 1]), l2, np);
            const float2 pv = fma_cols < 0 ? exp2_mix(i / 2, SLM_EXP2_FMA_DUAL, ap)
                                           : (fma_cols ? exp2_fma2(ap) : exp2_2(ap));
            const float2 r = mul2(ck2, sub2(qv, pv));
            vq[i] = r.x;
            vq[i + 1] = r.y;
          }
#else
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float qv = exp2f(fmaf(vq[i], kLog2e, -lq2));
            const float pv = exp2f(fmaf(vp[i], kLog2e, -lp2));
            vq[i] = ck * (qv - pv);
          }
#endif
        } else if (mode == 3) {
          // alpha-based kinds: dz = ck (q - p) + cm q ([q < p] - S), two columns at a time.
          const float2 l2 = make_float2(kLog2e, kLog2e);
          const float2 nq = make_float2(-lq2, -lq2), np = make_float2(-lp2, -lp2);
          const float2 ck2 = make_float2(ck, ck), cm2 = make_float2(cm, cm);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 qv = exp2_2(fma2(make_float2(vq[i], vq[i + 1]), l2, nq));
            const float2 pv = exp2_2(fma2(make_float2(vp[i], vp[i + 1]), l2, np));
            const float2 mS = make_float2(((qv.x < pv.x) ? 1.f : 0.f) - S,
                                          ((qv.y < pv.y) ? 1.f : 0.f) - S);
            const float2 r = fma2(ck2, sub2(qv, pv), mul2(mul2(cm2, qv), mS));
            vq[i] = r.x;
            vq[i + 1] = r.y;
          }
        } else if (mode == 1) {
          // Reverse KL: dz = ck q ((z_q - z_p) - c), two columns at a time.
          const float2 l2 = make_float2(kLog2e, kLog2e), nq = make_float2(-lq2, -lq2);
          const float2 ck2 = make_float2(ck, ck), cm2 = make_float2(cm, cm);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 z = make_float2(vq[i], vq[i + 1]);
            const float2 qv = exp2_2(fma2(z, l2, nq));
            const float2 r =
                mul2(mul2(ck2, qv), sub2(sub2(z, make_float2(vp[i], vp[i + 1])), cm2));
            vq[i] = r.x;
            vq[i + 1] = r.y;
          }
        } else {
          // JSD: dz = g q ((log q - log M) / 2 - T), M = (p + q) / 2.  In log2 units, with
          // b = log2 q: log2 q - log2 M = b + w, w = 1 - log2(p + q), so
          // dz = q (k1 (b + w) - g T), k1 = g ln2 / 2.  Two columns at a time, no branch.
          const float2 l2 = make_float2(kLog2e, kLog2e);
          const float2 nq = make_float2(-lq2, -lq2), np = make_float2(-lp2, -lp2);
          const float2 k1 = make_float2(0.5f * kLn2 * ck, 0.5f * kLn2 * ck);
          const float2 gt = make_float2(ck * S, ck * S);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 a = fma2(make_float2(vp[i], vp[i + 1]), l2, np);  // log2 p
            const float2 b = fma2(make_float2(vq[i], vq[i + 1]), l2, nq);  // log2 q
            // log2 q - log2 M = b + w, w = 1 - log2(p + q).
            const float2 q = exp2_2(b);
            const float2 w = sub2(make_float2(1.f, 1.f), log2_2(add2(exp2_2(a), q)));
            const float2 r = mul2(q, sub2(mul2(k1, add2(b, w)), gt));
            vq[i] = r.x;
            vq[i + 1] = r.y;
          }
        }
      }
    } else {
      const int64_t rel = static_cast<int64_t>(lab) - col0;
#if SLM_PACKED_EPI
      const float2 l2 = make_float2(kLog2e, kLog2e), nq = make_float2(-lq2, -lq2);
      const float2 g2 = make_float2(g, g);
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float2 qv =
            exp2_mix(i / 2, SLM_EXP2_FMA_CE, fma2(make_float2(vq[i], vq[i + 1]), l2, nq));
        const float2 oh = make_float2(rel == i ? 1.f : 0.f, rel == i + 1 ? 1.f : 0.f);
        const float2 r = mul2(g2, sub2(qv, oh));
        vq[i] = r.x;
        vq[i + 1] = r.y;
      }
#else
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float qv = exp2f(fmaf(vq[i], kLog2e, -lq2));
        vq[i] = g * (qv - (rel == i ? 1.f : 0.f));
      }
#endif
    }
  }

  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int row0, int64_t n0,
                                       int c0, int c1, int row) {
    const int lane = threadIdx.x & 31;
    uint8_t* srow = reinterpret_cast<uint8_t*>(stage) + lane * 128;
    const int wrow0 = row0 + row - lane;  // chunk row of this warp's first row
#pragma unroll 1
    for (int c = c0; c < c1; c += 64) {
      // The staging block is free once the previous block's store has read it.
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float vq[32], vp[32];
        tmem_ld32(tb + c + 32 * h, vq);
        if (DUAL) tmem_ld32(tb + TN + c + 32 * h, vp);
        tmem_ld_wait();
        apply(vq, vp, n0 + c + 32 * h);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 b2 =
                __floats2bfloat162_rn(vq[8 * k + 2 * e], vq[8 * k + 2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          *reinterpret_cast<uint4*>(srow + (((4 * h + k) ^ (lane & 7)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      // Columns >= V and rows beyond the chunk fall outside the map and are not written.
      if (lane == 0 && n0 + c < p.V) {
        tma_store_2d(&p.dz_map, stage, static_cast<int32_t>(n0 + c), wrow0);
        bulk_commit();
      }
    }
  }

  __device__ __forceinline__ void unit_end(const Params&, int, int, int) {}

  // Every store has landed before the kernel's shared memory goes away.
  __device__ __forceinline__ void finish() {
    if ((threadIdx.x & 31) == 0) bulk_wait_all();
    __syncwarp();
  }
};

// dH rows of the chunk: fp32 accumulator -> bf16.
struct EpiDh {
  using Params = DhParams;
  __device__ __forceinline__ void unit_begin(const Params&, int, int) {}
  __device__ __forceinline__ void unit_end(const Params&, int, int, int) {}
  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int row0, int64_t n0,
                                       int c0, int c1, int row) {
    const int64_t lrow = static_cast<int64_t>(row0) + row;
    const bool ok = lrow < p.rows;
    __nv_bfloat16* out = p.dH + (p.row0 + lrow) * p.d + n0;
#pragma unroll 1
    for (int c = c0; c < c1; c += 32) {
      float v[32];
      tmem_ld32(tb + c, v);
      tmem_ld_wait();
      if (ok && n0 + c < p.d) store_bf16_row32(out + c, v, n0 + c, p.d);
    }
  }
};

// dW tile: fp32 read-add-write (or plain write) of rows this CTA owns exclusively, without
// atomics.
//   STAGED = true: each warp passes its 32 rows x 32 columns through a 4 KB shared-memory
//     stage (16-byte chunk k of row r at position k ^ (r % 8), so that neither the writes
//     nor the reads conflict), so that each global load and store instruction covers four
//     whole 128-byte row segments, 8 lanes per row.  The persistent fused backward uses it.
//   STAGED = false: each lane adds its own row's 32 columns, a 16-byte piece at a time.  The
//     standalone dW GEMM uses it: there, with one epilogue warpgroup, the staged form was
//     about 1% slower, while in the fused backward it made the kernel 1.4% faster.
template <bool STAGED>
struct EpiDwT {
  using Params = DwParams;
  static constexpr int kStageBytesPerWarp = STAGED ? 4096 : 0;
  float* stage;
  __device__ __forceinline__ void unit_begin(const Params&, int, int) {}
  __device__ __forceinline__ void unit_end(const Params&, int, int, int) {}
  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int row0, int64_t n0,
                                       int c0, int c1, int row) {
    const int lane = threadIdx.x & 31;
    float4* st = reinterpret_cast<float4*>(stage);
    const int64_t wrow0 = static_cast<int64_t>(row0) + row - lane;  // the warp's first row
    const int sub = lane >> 3;  // row within each group of four
    const int k = lane & 7;     // 16-byte chunk within the row's 32 columns
#pragma unroll 1
    for (int c = c0; c < c1; c += 32) {
      float x[32];
      tmem_ld32(tb + c, x);
      tmem_ld_wait();
      if (!STAGED) {
        const int64_t v = static_cast<int64_t>(row0) + row;
        if (v >= p.V || n0 + c >= p.d) continue;
        float* out = p.dW + v * p.d + n0 + c;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (n0 + c + 4 * q >= p.d) break;
          float4* dst = reinterpret_cast<float4*>(out + 4 * q);
          float4 r = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
          if (p.beta) {
            const float4 o = *dst;
            r.x += o.x;
            r.y += o.y;
            r.z += o.z;
            r.w += o.w;
          }
          *dst = r;
        }
        continue;
      }
      const int64_t col = n0 + c + 4 * k;
      if (n0 + c >= p.d) continue;  // the whole block lies past d (warp-uniform)
      __syncwarp();                 // every lane has read the previous block
#pragma unroll
      for (int q = 0; q < 8; ++q)
        st[lane * 8 + (q ^ (lane & 7))] =
            make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
      __syncwarp();
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) {
        const int r = rr * 4 + sub;
        const int64_t v = wrow0 + r;
        const float4 a = st[r * 8 + (k ^ (r & 7))];
        // d % 8 == 0: a 4-column chunk that starts below d ends within the row.
        if (v < p.V && col < p.d) {
          float4* dst = reinterpret_cast<float4*>(p.dW + v * p.d + col);
          float4 out = a;
          if (p.beta) {
            const float4 o = *dst;
            out.x = a.x + o.x;
            out.y = a.y + o.y;
            out.z = a.z + o.z;
            out.w = a.w + o.w;
          }
          *dst = out;
        }
      }
    }
  }
};
using EpiDw = EpiDwT<false>;
using EpiDwStaged = EpiDwT<true>;

// ----------------------------------------------------------------------------------------
// Target flatness ("Flatter Tokens are More Valuable for Speculative Draft Model
// Training"): cos(p, uniform) = 1 / (sqrt(V) ||p||_2).  Per row and vocabulary slot the
// online max m, s = sum 2^(z log2e - m) and s2 = sum 2^(2 (z log2e - m)).
// ----------------------------------------------------------------------------------------
struct EpiFlat {
  using Params = FwdParams;
  static constexpr bool kSplitHalves = true;
  float m, s, s2;
  bool row_ok;
  int64_t grow;

  __device__ __forceinline__ void unit_begin(const Params& p, int row0, int row) {
    m = -INFINITY;
    s = s2 = 0.f;
    grow = static_cast<int64_t>(row0) + row;
    row_ok = grow < p.N;
  }

  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int, int64_t n0, int c0,
                                       int c1, int) {
#pragma unroll 1
    for (int c = c0; c < c1; c += 32) {
      float v[32];
      tmem_ld32(tb + c, v);
      tmem_ld_wait();
      if (n0 + c + 32 > p.V) mask_tail(v, n0 + c, p.V);
      const float mx = max32(v) * kLog2e;
      if (mx > m) {
        const float r = exp2f(m - mx);
        s *= r;
        s2 *= r * r;
        m = mx;
      }
      if (m != -INFINITY) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float e = exp2f(fmaf(v[i], kLog2e, -m));
          s += e;
          s2 = fmaf(e, e, s2);
        }
      }
    }
  }

  __device__ __forceinline__ void unit_end(const Params& p, int, int slot, int) {
    if (!row_ok) return;
    float* base = p.part + static_cast<int64_t>(slot) * kFlatFields * p.N + grow;
    base[0] = m;
    base[p.N] = s;
    base[2 * p.N] = s2;
  }
};

// ----------------------------------------------------------------------------------------
// Weighted combinations ("Loss Functions", "Weighted Combinations"): every term shares one
// logit pass.  Pass 1 gathers the union of the one-pass statistics; pass 2 (only when a
// term needs the final log-sum-exps) the union of alpha, S and the JSD halves; the
// backward forms sum_k w_k dz_k in one epilogue.
// ----------------------------------------------------------------------------------------
struct EpiFwdUnion {
  using Params = FwdParams;
  EpiFwdDual dual;
  float pmax, zqa, zyv;
  int pidx;
  int32_t lab;
  bool has_zy;

  __device__ __forceinline__ void unit_begin(const Params& p, int row0, int row) {
    dual.unit_begin(p, row0, row);
    pmax = -INFINITY;
    zqa = zyv = 0.f;
    pidx = -1;
    has_zy = false;
    lab = (dual.row_ok && p.labels) ? p.labels[dual.grow] : -1;
  }

  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int, int64_t n0, int c0,
                                       int c1, int) {
    const int64_t rel = static_cast<int64_t>(lab) - n0;
#pragma unroll 1
    for (int c = c0; c < c1; c += 32) {
      float vq[32], vp[32];
      tmem_ld32(tb + c, vq);
      tmem_ld32(tb + TN + c, vp);
      tmem_ld_wait();
      const bool tail = n0 + c + 32 > p.V;
      if (tail) {
        mask_tail(vq, n0 + c, p.V);
        mask_tail(vp, n0 + c, p.V);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (vp[i] > pmax) {
          pmax = vp[i];
          pidx = static_cast<int>(n0 + c + i);
          zqa = vq[i];
        }
      }
      if (static_cast<uint64_t>(rel - c) < 32u) {
        const int o = static_cast<int>(rel - c);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i == o) zyv = vq[i];
        has_zy = true;
      }
      if (tail)
        dual.template chunk<true>(vq, vp);
      else
        dual.template chunk<false>(vq, vp);
    }
  }

  __device__ __forceinline__ void unit_end(const Params& p, int, int slot, int) {
    if (!dual.row_ok) return;
    float* base = p.part + static_cast<int64_t>(slot) * kUnionFields * p.N + dual.grow;
    base[0 * p.N] = dual.mq;
    base[1 * p.N] = dual.sq;
    base[2 * p.N] = dual.mp;
    base[3 * p.N] = dual.sp;
    base[4 * p.N] = dual.A;
    base[5 * p.N] = dual.B;
    base[6 * p.N] = pmax;
    base[7 * p.N] = __int_as_float(pidx);
    base[8 * p.N] = zqa;
    if (has_zy) p.zy[dual.grow] = zyv;
  }
};

struct EpiPass2Union {
  using Params = FwdParams;
  float lq, lp, lq2, lp2, al, S, jp, jq;
  bool row_ok;
  int64_t grow;

  __device__ __forceinline__ void unit_begin(const Params& p, int row0, int row) {
    al = S = jp = jq = 0.f;
    grow = static_cast<int64_t>(row0) + row;
    row_ok = grow < p.N;
    lq = row_ok ? p.stats[grow] : 0.f;
    lp = row_ok ? p.stats[p.N + grow] : 0.f;
    lq2 = lq * kLog2e;
    lp2 = lp * kLog2e;
  }

  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int, int64_t n0, int c0,
                                       int c1, int) {
#pragma unroll 1
    for (int c = c0; c < c1; c += 32) {
      float vq[32], vp[32];
      tmem_ld32(tb + c, vq);
      tmem_ld32(tb + TN + c, vp);
      tmem_ld_wait();
      if (n0 + c + 32 > p.V) {
        mask_tail(vq, n0 + c, p.V);
        mask_tail(vp, n0 + c, p.V);
      }
      if (p.with_jsd) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float qv = exp2f(fmaf(vq[i], kLog2e, -lq2));
          const float pv = exp2f(fmaf(vp[i], kLog2e, -lp2));
          al += fminf(pv, qv);
          S += (qv < pv) ? qv : 0.f;
          const float ms = pv + qv;
          if (ms > 0.f) {
            const float lm = log2f(0.5f * ms) * kLn2;
            jp = fmaf(pv, (vp[i] - lp) - lm, jp);
            jq = fmaf(qv, (vq[i] - lq) - lm, jq);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float qv = exp2f(fmaf(vq[i], kLog2e, -lq2));
          const float pv = exp2f(fmaf(vp[i], kLog2e, -lp2));
          al += fminf(pv, qv);
          S += (qv < pv) ? qv : 0.f;
        }
      }
    }
  }

  __device__ __forceinline__ void unit_end(const Params& p, int, int slot, int) {
    if (!row_ok) return;
    float* base = p.part + static_cast<int64_t>(slot) * kPass2Fields * p.N + grow;
    base[0 * p.N] = al;
    base[1 * p.N] = S;
    base[2 * p.N] = jp;
    base[3 * p.N] = jq;
  }
};

// Logits gradient of a weighted combination:
//   dz_j = g [ q_j (a0 + a1 (m_j - S) + a2 (z_q,j - z_p,j) + a3 (a_j - T)) - beta p_j
//              - w_ce [j = y] - w_am [j = y_am] ],   a_j = (log q_j - log M_j) / 2,
// with a0 = w_ce + w_am + w_kl + w_lk lambda - w_rkl (L_q - L_p + RKL),
//      a1 = -(w_tv + w_nla / alpha + w_lk (1 - lambda)),  a2 = w_rkl,  a3 = w_jsd,
//      beta = w_kl + w_lk lambda:  the sum of the per-kind gradients of EpiDz.
struct EpiDzCombo {
  using Params = DzParams;
  float lq, lq2, lp2, a0, a1, a2, a3, beta, S, T, wce, wam;
  int32_t yce, yam;
  bool row_ok;
  int64_t lrow;

  __device__ __forceinline__ void unit_begin(const Params& p, int row0, int row) {
    lrow = static_cast<int64_t>(row0) + row;
    row_ok = lrow < p.rows;
    const int64_t n = p.row0 + lrow;
    lq = lq2 = lp2 = a0 = a1 = a2 = a3 = beta = S = T = wce = wam = 0.f;
    yce = yam = -1;
    if (!row_ok) return;
    const float* w = p.cw.w;
    bool valid = true;
    int32_t lab = -1;
    if (p.labels) {
      lab = p.labels[n];
      valid = lab != p.ignore_index;
      if (w[kCE] != 0.f && (lab < 0 || lab >= p.V)) valid = false;
    }
    const float g = row_grad(p, n, valid);
    lq = p.stats[n];
    const float lp = p.stats[p.N + n];
    lq2 = lq * kLog2e;
    lp2 = lp * kLog2e;
    const float rkl = p.stats[3 * p.N + n];
    const float al = p.stats[4 * p.N + n];
    S = p.stats[5 * p.N + n];
    T = p.stats[7 * p.N + n];
    const float lam = (w[kLK] != 0.f) ? expf(-3.f * al) : 0.f;
    a0 = g * (w[kCE] + w[kCEArgmax] + w[kKL] + w[kLK] * lam - w[kRKL] * (lq - lp + rkl));
    a1 = -g * (w[kTV] + ((w[kNLA] != 0.f) ? w[kNLA] / fmaxf(al, 1e-30f) : 0.f) +
               w[kLK] * (1.f - lam));
    a2 = g * w[kRKL];
    a3 = g * w[kJSD];
    beta = g * (w[kKL] + w[kLK] * lam);
    wce = g * w[kCE];
    wam = g * w[kCEArgmax];
    yce = (w[kCE] != 0.f) ? lab : -1;
    yam = (w[kCEArgmax] != 0.f) ? __float_as_int(p.stats[8 * p.N + n]) : -1;
  }

  template <int TN>
  __device__ __forceinline__ void tile(const Params& p, uint32_t tb, int, int64_t n0, int c0,
                                       int c1, int) {
    const float* w = p.cw.w;
    // Uniform across the launch: which terms need the indicator and log M.
    const bool need_m = w[kTV] != 0.f || w[kNLA] != 0.f || w[kLK] != 0.f;
    const bool need_lm = w[kJSD] != 0.f;
    __nv_bfloat16* out = p.dz + lrow * p.ldz + n0;
#pragma unroll 1
    for (int c = c0; c < c1; c += 32) {
      float vq[32], vp[32];
      tmem_ld32(tb + c, vq);
      tmem_ld32(tb + TN + c, vp);
      tmem_ld_wait();
      const int64_t rce = static_cast<int64_t>(yce) - (n0 + c);
      const int64_t ram = static_cast<int64_t>(yam) - (n0 + c);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float qv = exp2f(fmaf(vq[i], kLog2e, -lq2));
        const float pv = exp2f(fmaf(vp[i], kLog2e, -lp2));
        float t = fmaf(a2, vq[i] - vp[i], a0);
        if (need_m) t = fmaf(a1, ((qv < pv) ? 1.f : 0.f) - S, t);
        if (need_lm) {
          const float ms = pv + qv;
          if (ms > 0.f) {
            const float lm = log2f(0.5f * ms) * kLn2;
            t = fmaf(a3, 0.5f * ((vq[i] - lq) - lm) - T, t);
          }
        }
        float dz = fmaf(qv, t, -beta * pv);
        if (rce == i) dz -= wce;
        if (ram == i) dz -= wam;
        vq[i] = dz;
      }
      if (row_ok && n0 + c < p.V) store_bf16_row32(out + c, vq, n0 + c, p.V);
    }
  }

  __device__ __forceinline__ void unit_end(const Params&, int, int, int) {}
};

// ----------------------------------------------------------------------------------------
// Launchers: persistent 2-SM launches with clusters of two CTAs, at most as many clusters
// as can be resident at once (so the static unit schedule never waits for a second wave).
// ----------------------------------------------------------------------------------------
int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

template <int BNI, int NSUB, int NUM_A, int NBUF, int NWG, bool A_MN, bool B_MN, int STAGES,
          class Epi>
static cudaError_t launch_pair(const CUtensorMap& a0, const CUtensorMap& a1,
                               const CUtensorMap& b, const GemmGeom& g,
                               const typename Epi::Params& p, const DevCtl& c, cudaStream_t s) {
  using Cfg = PairCfg<BNI, NSUB, NUM_A, NBUF, NWG, A_MN, B_MN, STAGES>;
  constexpr size_t kStage = EpiStageBytes<Epi>::value;
  constexpr size_t kSmem = Cfg::kSmem + (kStage ? 1024 + kStage * 4 * NWG : 0);
  static_assert(kSmem <= 232448, "shared memory per CTA");
  auto kern = gemm_pair_kernel<BNI, NSUB, NUM_A, NBUF, NWG, A_MN, B_MN, STAGES, Epi>;
  cudaError_t e = cudaSuccess;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  // Per device, once: the shared-memory opt-in and the number of co-resident pairs.  Later
  // launches make no such calls, so that they can be captured into a CUDA graph.
  static bool smem_set[64] = {false};
  if (!smem_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmem));
    if (e != cudaSuccess) return e;
    smem_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int max_clusters[64] = {0};
  if (max_clusters[dev] == 0) {
    int n = 0;
    cfg.gridDim = dim3(2 * 512, 1, 1);
    if ((e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg)) != cudaSuccess) return e;
    max_clusters[dev] = n > 0 ? n : 1;
  }
  const int cap = std::max(1, max_clusters[dev] - std::max(0, g.reserve_pairs));
  const int pairs = std::max(1, std::min(g.num_units, cap));
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  GemmGeom gg = g;
  gg.epoch = 0;
  if (g.sync_kb > 0 && g.slack >= 0 && pairs > 1 && pairs <= kMaxSyncPairs) {
    // A fresh tag per launch: records left by earlier launches are ignored.
    static std::atomic<uint32_t> next_epoch{1};
    uint32_t e = next_epoch.fetch_add(1);
    if (e == 0) e = next_epoch.fetch_add(1);
    gg.epoch = e;
  }
  return cudaLaunchKernelEx(&cfg, kern, a0, a1, b, gg, p, c);
}

// Forward statistics and logits gradient: A = hidden states (K-major), B = W (K-major).
//   CE:   one accumulator, tile 256 x 512 (two 256-wide MMAs), single TMEM buffer
//   dual: target + draft accumulators, tile 256 x 256 each, single TMEM buffer
// dH: A = dZ (K-major), B = W (MN-major), tile 256 x 512, single buffer.
// dW: A = dZ^T (MN-major), B = H (MN-major), tile 256 x 256, double-buffered (its fp32
//     read-add-write epilogue overlaps the next tile's MMAs).
cudaError_t launch_fwd_ce(const CUtensorMap& tH, const CUtensorMap& tW, const GemmGeom& g,
                          const FwdParams& p, const DevCtl& c, cudaStream_t s) {
  return launch_pair<256, 2, 1, 1, 2, false, false, 4, EpiFwdCE>(tH, tH, tW, g, p, c, s);
}
cudaError_t launch_fwd_dual(const CUtensorMap& tHq, const CUtensorMap& tHp, const CUtensorMap& tW,
                            const GemmGeom& g, const FwdParams& p, const DevCtl& c, bool rkl,
                            cudaStream_t s) {
  // Reverse KL needs only the accumulator B, every other kind only A.
  if (rkl)
    return launch_pair<256, 1, 2, 1, 2, false, false, 4, EpiFwdDualT<2>>(tHq, tHp, tW, g, p, c,
                                                                         s);
  return launch_pair<256, 1, 2, 1, 2, false, false, 4, EpiFwdDualT<1>>(tHq, tHp, tW, g, p, c, s);
}
cudaError_t launch_fwd_argmax(const CUtensorMap& tHq, const CUtensorMap& tHp,
                              const CUtensorMap& tW, const GemmGeom& g, const FwdParams& p,
                              const DevCtl& c, cudaStream_t s) {
  return launch_pair<256, 1, 2, 1, 2, false, false, 4, EpiFwdArgmax>(tHq, tHp, tW, g, p, c, s);
}
cudaError_t launch_jsd(const CUtensorMap& tHq, const CUtensorMap& tHp, const CUtensorMap& tW,
                       const GemmGeom& g, const FwdParams& p, const DevCtl& c, cudaStream_t s) {
  return launch_pair<256, 1, 2, 1, 2, false, false, 4, EpiJsd>(tHq, tHp, tW, g, p, c, s);
}
cudaError_t launch_fwd_flat(const CUtensorMap& tHp, const CUtensorMap& tW, const GemmGeom& g,
                            const FwdParams& p, const DevCtl& c, cudaStream_t s) {
  return launch_pair<256, 2, 1, 1, 2, false, false, 4, EpiFlat>(tHp, tHp, tW, g, p, c, s);
}
cudaError_t launch_fwd_union(const CUtensorMap& tHq, const CUtensorMap& tHp,
                             const CUtensorMap& tW, const GemmGeom& g, const FwdParams& p,
                             const DevCtl& c, cudaStream_t s) {
  return launch_pair<256, 1, 2, 1, 2, false, false, 4, EpiFwdUnion>(tHq, tHp, tW, g, p, c, s);
}
cudaError_t launch_pass2_union(const CUtensorMap& tHq, const CUtensorMap& tHp,
                               const CUtensorMap& tW, const GemmGeom& g, const FwdParams& p,
                               const DevCtl& c, cudaStream_t s) {
  return launch_pair<256, 1, 2, 1, 2, false, false, 4, EpiPass2Union>(tHq, tHp, tW, g, p, c, s);
}
cudaError_t launch_dz_combo(const CUtensorMap& tHq, const CUtensorMap& tHp,
                            const CUtensorMap& tW, const GemmGeom& g, const DzParams& p,
                            const DevCtl& c, cudaStream_t s) {
  return launch_pair<256, 1, 2, 1, 2, false, false, 4, EpiDzCombo>(tHq, tHp, tW, g, p, c, s);
}
cudaError_t launch_alpha(const CUtensorMap& tHq, const CUtensorMap& tHp, const CUtensorMap& tW,
                         const GemmGeom& g, const FwdParams& p, const DevCtl& c,
                         cudaStream_t s) {
  return launch_pair<256, 1, 2, 1, 2, false, false, 4, EpiAlpha>(tHq, tHp, tW, g, p, c, s);
}
cudaError_t launch_dz_ce(const CUtensorMap& tH, const CUtensorMap& tW, const GemmGeom& g,
                         const DzParams& p, const DevCtl& c, cudaStream_t s) {
  return launch_pair<256, 2, 1, 1, 2, false, false, 4, EpiDz<false>>(tH, tH, tW, g, p, c, s);
}
cudaError_t launch_dz_dual(const CUtensorMap& tHq, const CUtensorMap& tHp, const CUtensorMap& tW,
                           const GemmGeom& g, const DzParams& p, const DevCtl& c,
                           cudaStream_t s) {
  return launch_pair<256, 1, 2, 1, 2, false, false, 4, EpiDz<true>>(tHq, tHp, tW, g, p, c, s);
}
cudaError_t launch_dh(const CUtensorMap& tDz, const CUtensorMap& tW, const GemmGeom& g,
                      const DhParams& p, const DevCtl& c, cudaStream_t s) {
  return launch_pair<256, 2, 1, 1, 2, false, true, 4, EpiDh>(tDz, tDz, tW, g, p, c, s);
}
cudaError_t launch_dw(const CUtensorMap& tDzT, const CUtensorMap& tH, const GemmGeom& g,
                      const DwParams& p, const DevCtl& c, cudaStream_t s) {
  return launch_pair<256, 1, 1, 2, 1, true, true, 6, EpiDw>(tDzT, tDzT, tH, g, p, c, s);
}

// ----------------------------------------------------------------------------------------
// Row combines: merge the per-unit partials of each row into the final statistics and the
// per-token loss, then reduce the block's loss sum and valid count in a fixed order.
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ void block_reduce_store(double v, long long c, double* blk_sum,
                                                   long long* blk_cnt) {
  __shared__ double ss[kCombineThreads / 32];
  __shared__ long long sc[kCombineThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v += __shfl_down_sync(0xffffffffu, v, o);
    c += __shfl_down_sync(0xffffffffu, c, o);
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    ss[w] = v;
    sc[w] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    long long k = 0;
    for (int i = 0; i < kCombineThreads / 32; ++i) {
      t += ss[i];
      k += sc[i];
    }
    blk_sum[blockIdx.x] = t;
    blk_cnt[blockIdx.x] = k;
  }
}

__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(int kind, int pass, const float* __restrict__ part, int nch,
                   const float* __restrict__ zy, const int32_t* __restrict__ labels,
                   int32_t ignore_index, int64_t N, int64_t V, float* loss_tok,
                   float* alpha_tok, float* stats, double* blk_sum, long long* blk_cnt,
                   int* status, int64_t row0, int64_t ldN) {
  // n: row within this launch (partials and label logits are indexed by it);
  // gn = row0 + n: the row of the whole batch (labels, statistics, per-token outputs).
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kCombineThreads + threadIdx.x;
  const int64_t gn = row0 + n;
  double lsum = 0.0;
  long long cnt = 0;
  if (n < N) {
    bool valid = true;
    int32_t y = 0;
    if (labels) {
      y = labels[gn];
      valid = y != ignore_index;
      if (kind == kCE && valid && (y < 0 || y >= V)) {
        atomicOr(status, kFlagLabelRange);
        valid = false;
      }
    }
    float loss = 0.f;
    if (kind == kCE) {
      float M = -INFINITY;
      for (int j = 0; j < nch; ++j) M = fmaxf(M, part[(2 * (int64_t)j) * N + n]);
      float S = 0.f;
      for (int j = 0; j < nch; ++j)
        S += part[(2 * (int64_t)j + 1) * N + n] * exp2f(part[(2 * (int64_t)j) * N + n] - M);
      const float L = (M + log2f(S)) * kLn2;
      stats[gn] = L;
      loss = valid ? (L - zy[n]) : 0.f;
    } else if (kind == kCEArgmax) {
      // Log-sum-exp of the draft; the target's argmax over all slots (the largest value,
      // the lowest column on ties) and the draft logit there.
      float Mq = -INFINITY, best = -INFINITY, zq_best = 0.f;
      int idx = -1;
      for (int j = 0; j < nch; ++j) {
        const float* b = part + (int64_t)j * kArgmaxFields * N + n;
        Mq = fmaxf(Mq, b[0]);
        const float v = b[2 * N];
        const int k = __float_as_int(b[3 * N]);
        if (k >= 0 && (v > best || (v == best && k < idx))) {
          best = v;
          idx = k;
          zq_best = b[4 * N];
        }
      }
      float Sq = 0.f;
      for (int j = 0; j < nch; ++j) {
        const float* b = part + (int64_t)j * kArgmaxFields * N + n;
        Sq += b[N] * exp2f(b[0] - Mq);
      }
      const float Lq = (Mq + log2f(Sq)) * kLn2;
      if (idx < 0) valid = false;
      stats[gn] = Lq;
      stats[ldN + gn] = __int_as_float(valid ? idx : ignore_index);
      loss = valid ? (Lq - zq_best) : 0.f;
    } else if (pass == 1) {
      float Mq = -INFINITY, Mp = -INFINITY;
      for (int j = 0; j < nch; ++j) {
        const float* b = part + (int64_t)j * kDualFields * N + n;
        Mq = fmaxf(Mq, b[0]);
        Mp = fmaxf(Mp, b[2 * N]);
      }
      float Sq = 0.f, Sp = 0.f, A = 0.f, B = 0.f;
      for (int j = 0; j < nch; ++j) {
        const float* b = part + (int64_t)j * kDualFields * N + n;
        const float rq = exp2f(b[0] - Mq);
        const float rp = exp2f(b[2 * N] - Mp);
        Sq += b[N] * rq;
        B += b[5 * N] * rq;
        Sp += b[3 * N] * rp;
        A += b[4 * N] * rp;
      }
      const float Lq = (Mq + log2f(Sq)) * kLn2;
      const float Lp = (Mp + log2f(Sp)) * kLn2;
      // KL(p||q) = sum p (z_p - z_q) - L_p + L_q;  KL(q||p) = sum q (z_q - z_p) - L_q + L_p.
      const float kl = A / Sp - Lp + Lq;
      const float rkl = B / Sq - Lq + Lp;
      stats[gn] = Lq;
      stats[ldN + gn] = Lp;
      stats[2 * ldN + gn] = (kind == kRKL) ? rkl : kl;
      loss = valid ? ((kind == kRKL) ? rkl : kl) : 0.f;
    } else if (kind == kJSD) {
      float jp = 0.f, jq = 0.f;
      for (int j = 0; j < nch; ++j) {
        jp += part[(2 * (int64_t)j) * N + n];
        jq += part[(2 * (int64_t)j + 1) * N + n];
      }
      const float jsd = 0.5f * (jp + jq);
      stats[3 * ldN + gn] = jsd;
      stats[4 * ldN + gn] = 0.5f * jq;
      loss = valid ? jsd : 0.f;
    } else {
      float al = 0.f, S = 0.f;
      for (int j = 0; j < nch; ++j) {
        al += part[(2 * (int64_t)j) * N + n];
        S += part[(2 * (int64_t)j + 1) * N + n];
      }
      stats[3 * ldN + gn] = al;
      stats[4 * ldN + gn] = S;
      if (alpha_tok) alpha_tok[gn] = al;
      const float kl = stats[2 * ldN + gn];
      float l;
      if (kind == kTV) {
        l = 1.f - al;
      } else if (kind == kNLA) {
        l = -logf(fmaxf(al, 1e-30f));
      } else {
        const float lam = expf(-3.f * al);
        l = lam * kl + (1.f - lam) * (1.f - al);
      }
      loss = valid ? l : 0.f;
    }
    if (loss_tok) loss_tok[gn] = loss;
    lsum = static_cast<double>(loss);
    cnt = valid ? 1 : 0;
  }
  block_reduce_store(lsum, cnt, blk_sum + row0 / kCombineThreads, blk_cnt + row0 / kCombineThreads);
}

__global__ void __launch_bounds__(1024)
    finalize_kernel(const double* blk_sum, const long long* blk_cnt, int nblk, double* loss_sum,
                    int64_t* n_valid, float* loss_mean) {
  __shared__ double ss[32];
  __shared__ long long sc[32];
  double v = 0.0;
  long long c = 0;
  for (int i = threadIdx.x; i < nblk; i += blockDim.x) {
    v += blk_sum[i];
    c += blk_cnt[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v += __shfl_down_sync(0xffffffffu, v, o);
    c += __shfl_down_sync(0xffffffffu, c, o);
  }
  if ((threadIdx.x & 31) == 0) {
    ss[threadIdx.x >> 5] = v;
    sc[threadIdx.x >> 5] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    long long k = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
      t += ss[i];
      k += sc[i];
    }
    *loss_sum = t;
    *n_valid = static_cast<int64_t>(k);
    if (loss_mean) *loss_mean = k > 0 ? static_cast<float>(t / static_cast<double>(k)) : 0.f;
  }
}

__global__ void zero_f32_kernel(float* p, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = 0.f;
}

cudaError_t launch_combine(int kind, int pass, const float* part, int nch, const float* zy,
                           const int32_t* labels, int32_t ignore_index, int64_t N, int64_t V,
                           float* loss_tok, float* alpha_tok, float* stats, double* blk_sum,
                           long long* blk_cnt, int* status, cudaStream_t s, int64_t row0,
                           int64_t ldN) {
  if (ldN < 0) ldN = N;
  const int blocks = static_cast<int>((N + kCombineThreads - 1) / kCombineThreads);
  combine_kernel<<<blocks, kCombineThreads, 0, s>>>(kind, pass, part, nch, zy, labels,
                                                    ignore_index, N, V, loss_tok, alpha_tok,
                                                    stats, blk_sum, blk_cnt, status, row0, ldN);
  return cudaGetLastError();
}

cudaError_t launch_finalize(const double* blk_sum, const long long* blk_cnt, int nblk,
                            double* loss_sum, int64_t* n_valid, float* loss_mean,
                            cudaStream_t s) {
  finalize_kernel<<<1, 1024, 0, s>>>(blk_sum, blk_cnt, nblk, loss_sum, n_valid, loss_mean);
  return cudaGetLastError();
}

cudaError_t launch_zero_f32(float* p, int64_t n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int sms = sm_count() > 0 ? sm_count() : 148;
  zero_f32_kernel<<<sms * 4, 256, 0, s>>>(p, n);
  return cudaGetLastError();
}


// ----------------------------------------------------------------------------------------
// Weighted combinations: per-row merge of the union partials into the statistics and the
// per-term losses, the weighted total, and the fixed-order reductions.
// ----------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kCombineThreads)
    combo_combine_kernel(int pass, ComboW cw, const float* __restrict__ part, int nch,
                         const float* __restrict__ zy, const int32_t* __restrict__ labels,
                         int32_t ignore_index, int64_t N, int64_t V, float* stats,
                         float* term_tok, int* status) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kCombineThreads + threadIdx.x;
  if (n >= N) return;
  bool valid = true;
  if (labels) {
    const int32_t y = labels[n];
    valid = y != ignore_index;
    if (cw.w[kCE] != 0.f && valid && (y < 0 || y >= V)) {
      if (pass == 1) atomicOr(status, kFlagLabelRange);
      valid = false;
    }
  }
  if (pass == 1) {
    float Mq = -INFINITY, Mp = -INFINITY, best = -INFINITY, zq_best = 0.f;
    int idx = -1;
    for (int j = 0; j < nch; ++j) {
      const float* b = part + (int64_t)j * kUnionFields * N + n;
      Mq = fmaxf(Mq, b[0]);
      Mp = fmaxf(Mp, b[2 * N]);
      const float v = b[6 * N];
      const int k = __float_as_int(b[7 * N]);
      if (k >= 0 && (v > best || (v == best && k < idx))) {
        best = v;
        idx = k;
        zq_best = b[8 * N];
      }
    }
    float Sq = 0.f, Sp = 0.f, A = 0.f, B = 0.f;
    for (int j = 0; j < nch; ++j) {
      const float* b = part + (int64_t)j * kUnionFields * N + n;
      const float rq = exp2f(b[0] - Mq);
      const float rp = exp2f(b[2 * N] - Mp);
      Sq += b[N] * rq;
      B += b[5 * N] * rq;
      Sp += b[3 * N] * rp;
      A += b[4 * N] * rp;
    }
    const float Lq = (Mq + log2f(Sq)) * kLn2;
    const float Lp = (Mp + log2f(Sp)) * kLn2;
    const float kl = A / Sp - Lp + Lq;
    const float rkl = B / Sq - Lq + Lp;
    stats[n] = Lq;
    stats[N + n] = Lp;
    stats[2 * N + n] = kl;
    stats[3 * N + n] = rkl;
    stats[8 * N + n] = __int_as_float((valid && idx >= 0) ? idx : ignore_index);
    for (int k = 0; k < kNumKinds; ++k) term_tok[k * N + n] = 0.f;
    if (valid) {
      if (cw.w[kCE] != 0.f) term_tok[kCE * N + n] = Lq - zy[n];
      term_tok[kKL * N + n] = kl;
      term_tok[kRKL * N + n] = rkl;
      if (idx >= 0) term_tok[kCEArgmax * N + n] = Lq - zq_best;
    }
  } else {
    float al = 0.f, S = 0.f, jp = 0.f, jq = 0.f;
    for (int j = 0; j < nch; ++j) {
      const float* b = part + (int64_t)j * kPass2Fields * N + n;
      al += b[0];
      S += b[N];
      jp += b[2 * N];
      jq += b[3 * N];
    }
    const float jsd = 0.5f * (jp + jq);
    stats[4 * N + n] = al;
    stats[5 * N + n] = S;
    stats[6 * N + n] = jsd;
    stats[7 * N + n] = 0.5f * jq;
    if (valid) {
      const float kl = stats[2 * N + n];
      const float lam = expf(-3.f * al);
      term_tok[kTV * N + n] = 1.f - al;
      term_tok[kNLA * N + n] = -logf(fmaxf(al, 1e-30f));
      term_tok[kLK * N + n] = lam * kl + (1.f - lam) * (1.f - al);
      term_tok[kJSD * N + n] = jsd;
    }
  }
}

__global__ void __launch_bounds__(kCombineThreads)
    combo_total_kernel(ComboW cw, const float* __restrict__ term_tok,
                       const int32_t* __restrict__ labels, int32_t ignore_index, int64_t N,
                       int64_t V, float* loss_tok, float* term_out, double* blk_sums,
                       long long* blk_cnt) {
  constexpr int kW = kCombineThreads / 32;
  __shared__ double ss[kW][1 + kNumKinds];
  __shared__ long long sc[kW];
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kCombineThreads + threadIdx.x;
  double v[1 + kNumKinds];
  for (int k = 0; k <= kNumKinds; ++k) v[k] = 0.0;
  long long cnt = 0;
  if (n < N) {
    bool valid = true;
    if (labels) {
      const int32_t y = labels[n];
      valid = y != ignore_index;
      if (cw.w[kCE] != 0.f && valid && (y < 0 || y >= V)) valid = false;
    }
    float total = 0.f;
    for (int k = 0; k < kNumKinds; ++k) {
      const float t = valid ? term_tok[k * N + n] : 0.f;
      if (cw.w[k] != 0.f) total = fmaf(cw.w[k], t, total);
      if (term_out) term_out[k * N + n] = (cw.w[k] != 0.f) ? t : 0.f;
      v[1 + k] = (cw.w[k] != 0.f) ? static_cast<double>(t) : 0.0;
    }
    if (loss_tok) loss_tok[n] = total;
    v[0] = static_cast<double>(total);
    cnt = valid ? 1 : 0;
  }
  for (int k = 0; k <= kNumKinds; ++k) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[k] += __shfl_down_sync(0xffffffffu, v[k], o);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_down_sync(0xffffffffu, cnt, o);
  const int wi = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    for (int k = 0; k <= kNumKinds; ++k) ss[wi][k] = v[k];
    sc[wi] = cnt;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 0; k <= kNumKinds; ++k) {
      double t = 0.0;
      for (int i = 0; i < kW; ++i) t += ss[i][k];
      blk_sums[static_cast<int64_t>(blockIdx.x) * (1 + kNumKinds) + k] = t;
    }
    long long c = 0;
    for (int i = 0; i < kW; ++i) c += sc[i];
    blk_cnt[blockIdx.x] = c;
  }
}

__global__ void __launch_bounds__(256)
    combo_finalize_kernel(const double* blk_sums, const long long* blk_cnt, int nblk,
                          double* loss_sum, double* term_sum, int64_t* n_valid,
                          float* loss_mean) {
  __shared__ double ss[8][1 + kNumKinds];
  __shared__ long long sc[8];
  double v[1 + kNumKinds];
  for (int k = 0; k <= kNumKinds; ++k) v[k] = 0.0;
  long long c = 0;
  for (int i = threadIdx.x; i < nblk; i += blockDim.x) {
    for (int k = 0; k <= kNumKinds; ++k) v[k] += blk_sums[static_cast<int64_t>(i) * (1 + kNumKinds) + k];
    c += blk_cnt[i];
  }
  for (int k = 0; k <= kNumKinds; ++k) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[k] += __shfl_down_sync(0xffffffffu, v[k], o);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_down_sync(0xffffffffu, c, o);
  const int wi = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    for (int k = 0; k <= kNumKinds; ++k) ss[wi][k] = v[k];
    sc[wi] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t[1 + kNumKinds];
    long long k_valid = 0;
    for (int k = 0; k <= kNumKinds; ++k) {
      t[k] = 0.0;
      for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t[k] += ss[i][k];
    }
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) k_valid += sc[i];
    *loss_sum = t[0];
    if (term_sum)
      for (int k = 0; k < kNumKinds; ++k) term_sum[k] = t[1 + k];
    *n_valid = static_cast<int64_t>(k_valid);
    if (loss_mean)
      *loss_mean = k_valid > 0 ? static_cast<float>(t[0] / static_cast<double>(k_valid)) : 0.f;
  }
}

cudaError_t launch_combo_combine(int pass, const ComboW& cw, const float* part, int nch,
                                 const float* zy, const int32_t* labels, int32_t ignore_index,
                                 int64_t N, int64_t V, float* stats, float* term_tok,
                                 int* status, cudaStream_t s) {
  const int blocks = static_cast<int>((N + kCombineThreads - 1) / kCombineThreads);
  combo_combine_kernel<<<blocks, kCombineThreads, 0, s>>>(pass, cw, part, nch, zy, labels,
                                                          ignore_index, N, V, stats, term_tok,
                                                          status);
  return cudaGetLastError();
}

cudaError_t launch_combo_total(const ComboW& cw, const float* term_tok, const int32_t* labels,
                               int32_t ignore_index, int64_t N, int64_t V, float* loss_tok,
                               float* term_out, double* blk_sums, long long* blk_cnt,
                               cudaStream_t s) {
  const int blocks = static_cast<int>(std::max<int64_t>(1, (N + kCombineThreads - 1) / kCombineThreads));
  combo_total_kernel<<<blocks, kCombineThreads, 0, s>>>(cw, term_tok, labels, ignore_index, N, V,
                                                        loss_tok, term_out, blk_sums, blk_cnt);
  return cudaGetLastError();
}

cudaError_t launch_combo_finalize(const double* blk_sums, const long long* blk_cnt, int nblk,
                                  double* loss_sum, double* term_sum, int64_t* n_valid,
                                  float* loss_mean, cudaStream_t s) {
  combo_finalize_kernel<<<1, 256, 0, s>>>(blk_sums, blk_cnt, nblk, loss_sum, term_sum, n_valid,
                                          loss_mean);
  return cudaGetLastError();
}


// ----------------------------------------------------------------------------------------
// Fused forward + backward ("Backward pass": per token chunk, the logits, the loss and the
// gradients; the chunk's logits are kept, as on the page, instead of recomputed): kernels
// that read the chunk's stored fp32 logits.  Memory-bound, one CTA per row, float4 loads.
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ void block_sum2(float& a, float& b) {
  __shared__ float sa[32], sb[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_down_sync(0xffffffffu, a, o);
    b += __shfl_down_sync(0xffffffffu, b, o);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    sa[w] = a;
    sb[w] = b;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float ta = 0.f, tb = 0.f;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) {
      ta += sa[i];
      tb += sb[i];
    }
    a = ta;
    b = tb;
  }
}

__global__ void __launch_bounds__(1024)
    count_valid_kernel(const int32_t* __restrict__ labels, int32_t ignore_index, int64_t N,
                       int64_t V, int check_range, int64_t* n_valid) {
  __shared__ long long sc[32];
  long long c = 0;
  for (int64_t i = threadIdx.x; i < N; i += blockDim.x) {
    bool valid = true;
    if (labels) {
      const int32_t y = labels[i];
      valid = y != ignore_index && (!check_range || (y >= 0 && y < V));
    }
    c += valid ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_down_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) sc[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long t = 0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += sc[i];
    *n_valid = static_cast<int64_t>(t);
  }
}

// alpha = sum min(p, q) and S = sum_{q<p} q, or the JSD halves jp, jq, of one row.
__global__ void __launch_bounds__(256)
    logits_pass2_kernel(int kind, const float* __restrict__ lq, const float* __restrict__ lp,
                        int64_t ldl, const float* __restrict__ stats, int64_t row0, int64_t ldN,
                        int64_t rows, int64_t V, float* part) {
  const int64_t r = blockIdx.x;
  if (r >= rows) return;
  const int64_t gn = row0 + r;
  const float Lq = stats[gn], Lp = stats[ldN + gn];
  const float lq2 = Lq * kLog2e, lp2 = Lp * kLog2e;
  const float* rq = lq + r * ldl;
  const float* rp = lp + r * ldl;
  float a = 0.f, b = 0.f;
  for (int64_t c = static_cast<int64_t>(threadIdx.x) * 4; c < V; c += 4 * blockDim.x) {
    const float4 q4 = *reinterpret_cast<const float4*>(rq + c);
    const float4 p4 = *reinterpret_cast<const float4*>(rp + c);
    const float zq[4] = {q4.x, q4.y, q4.z, q4.w};
    const float zp[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (c + j >= V) break;
      const float qv = exp2f(fmaf(zq[j], kLog2e, -lq2));
      const float pv = exp2f(fmaf(zp[j], kLog2e, -lp2));
      if (kind == kJSD) {
        const float ms = pv + qv;
        if (ms > 0.f) {
          const float lm = log2f(0.5f * ms) * kLn2;
          a = fmaf(pv, (zp[j] - Lp) - lm, a);
          b = fmaf(qv, (zq[j] - Lq) - lm, b);
        }
      } else {
        a += fminf(pv, qv);
        b += (qv < pv) ? qv : 0.f;
      }
    }
  }
  block_sum2(a, b);
  if (threadIdx.x == 0) {
    part[r] = a;
    part[rows + r] = b;
  }
}

template <bool DUAL>
__global__ void __launch_bounds__(256)
    logits_dz_kernel(const DzParams p, const float* __restrict__ lq,
                     const float* __restrict__ lp, int64_t ldl) {
  // One block per row.  Each pass covers 32 * blockDim consecutive columns as 8 groups of
  // 4 per thread, the lanes of a warp on consecutive groups, so that every load reads and
  // every store writes one contiguous span per warp (512 and 256 bytes).
  const int64_t r = blockIdx.x;
  EpiDz<DUAL> e;
  e.unit_begin(p, 0, static_cast<int>(r));
  if (!e.row_ok) return;
  const float* rq = lq + r * ldl;
  const float* rp = DUAL ? lp + r * ldl : lq;
  __nv_bfloat16* out = p.dz + r * p.ldz;
  const int64_t span = 4 * static_cast<int64_t>(blockDim.x);
  for (int64_t base = 4 * static_cast<int64_t>(threadIdx.x); base < p.V; base += 8 * span) {
    float vq[32], vp[32];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int64_t c = base + k * span;
      if (c < p.V) {  // a float4 that starts below V lies within the row (ldl % 4 == 0)
        const float4 a = *reinterpret_cast<const float4*>(rq + c);
        vq[4 * k] = a.x, vq[4 * k + 1] = a.y, vq[4 * k + 2] = a.z, vq[4 * k + 3] = a.w;
        if (DUAL) {
          const float4 b = *reinterpret_cast<const float4*>(rp + c);
          vp[4 * k] = b.x, vp[4 * k + 1] = b.y, vp[4 * k + 2] = b.z, vp[4 * k + 3] = b.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) vq[4 * k + j] = vp[4 * k + j] = -INFINITY;
      }
    }
    if (DUAL) {
      // Elementwise: no column enters the divergences' formulas, except in choosing how
      // the target's 2^x is computed, which must match the GEMM epilogue's choice for the
      // same column: the FMA-pipe form for columns with ((c / 2) % 8) < the share.  This
      // thread's columns are 4 t + j + multiples of 16 (j < 4): their (c / 2) % 8 is
      // 2 (t % 4) or 2 (t % 4) + 1, on the same side of an even share, so the rule is one per
      // thread.
      static_assert(SLM_EXP2_FMA_DUAL % 2 == 0, "one rule per thread needs an even share");
      const int c16 = static_cast<int>((4 * threadIdx.x) & 15);
      e.apply(vq, vp, 0, (c16 >> 1) < SLM_EXP2_FMA_DUAL ? 1 : 0);
    } else {
      // CE: the same formula as the GEMM epilogue's, with each value's own column.
#pragma unroll
      for (int k = 0; k < 8; ++k)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int64_t c = base + k * span + j;
          const float qv = exp2f(fmaf(vq[4 * k + j], kLog2e, -e.lq2));
          vq[4 * k + j] = e.g * (qv - (c == e.lab ? 1.f : 0.f));
        }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int64_t c = base + k * span;
      if (c + 4 <= p.V) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(vq[4 * k], vq[4 * k + 1]);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(vq[4 * k + 2], vq[4 * k + 3]);
        uint2 w;
        w.x = *reinterpret_cast<const uint32_t*>(&lo);
        w.y = *reinterpret_cast<const uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(out + c) = w;
      } else {
        for (int j = 0; j < 4 && c + j < p.V; ++j) out[c + j] = __float2bfloat16_rn(vq[4 * k + j]);
      }
    }
  }
}

cudaError_t launch_count_valid(const int32_t* labels, int32_t ignore_index, int64_t N,
                               int64_t V, int check_range, int64_t* n_valid, cudaStream_t s) {
  count_valid_kernel<<<1, 1024, 0, s>>>(labels, ignore_index, N, V, check_range, n_valid);
  return cudaGetLastError();
}

cudaError_t launch_logits_pass2(int kind, const float* lq, const float* lp, int64_t ldl,
                                const float* stats, int64_t row0, int64_t ldN, int64_t rows,
                                int64_t V, float* part, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  logits_pass2_kernel<<<static_cast<unsigned>(rows), 256, 0, s>>>(kind, lq, lp, ldl, stats, row0,
                                                                  ldN, rows, V, part);
  return cudaGetLastError();
}

cudaError_t launch_logits_dz(const DzParams& p, const float* lq, const float* lp, int64_t ldl,
                             cudaStream_t s) {
  if (p.rows <= 0) return cudaSuccess;
  if (p.kind == kCE)
    logits_dz_kernel<false><<<static_cast<unsigned>(p.rows), 256, 0, s>>>(p, lq, lp, ldl);
  else
    logits_dz_kernel<true><<<static_cast<unsigned>(p.rows), 256, 0, s>>>(p, lq, lp, ldl);
  return cudaGetLastError();
}


// ----------------------------------------------------------------------------------------
// Alignment before chunking ("Correctness: alignment before chunking"): the label of
// position t for a head that predicts `shift` tokens ahead is tokens[t + shift], unless the
// target lies past the sequence, in another packed sequence, or under the loss mask.
// ----------------------------------------------------------------------------------------
__global__ void align_labels_kernel(const int32_t* __restrict__ tokens,
                                    const uint8_t* __restrict__ loss_mask,
                                    const int32_t* __restrict__ seq_ids, int64_t B, int64_t S,
                                    int32_t shift, int32_t ignore_index, int32_t* labels) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (n >= B * S) return;
  const int64_t b = n / S;
  const int64_t t = n - b * S;
  const int64_t u = t + shift;
  int32_t y = ignore_index;
  if (u < S) {
    const int64_t nu = b * S + u;
    const bool masked = loss_mask && loss_mask[nu] == 0;
    const bool crosses = seq_ids && seq_ids[nu] != seq_ids[n];
    if (!masked && !crosses) y = tokens[nu];
  }
  labels[n] = y;
}

__global__ void __launch_bounds__(kCombineThreads)
    flat_combine_kernel(const float* __restrict__ part, int nch, int64_t N, int64_t V,
                        float* flat) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kCombineThreads + threadIdx.x;
  if (n >= N) return;
  float M = -INFINITY;
  for (int j = 0; j < nch; ++j) M = fmaxf(M, part[(int64_t)j * kFlatFields * N + n]);
  float S = 0.f, S2 = 0.f;
  for (int j = 0; j < nch; ++j) {
    const float* b = part + (int64_t)j * kFlatFields * N + n;
    const float r = exp2f(b[0] - M);
    S += b[N] * r;
    S2 += b[2 * N] * (r * r);
  }
  // ||p||_2 = sqrt(S2) / S, so cos(p, uniform) = S / (sqrt(V) sqrt(S2)).
  flat[n] = S / (sqrtf(static_cast<float>(V)) * sqrtf(S2));
}

cudaError_t launch_align_labels(const int32_t* tokens, const uint8_t* loss_mask,
                                const int32_t* seq_ids, int64_t B, int64_t S, int32_t shift,
                                int32_t ignore_index, int32_t* labels, cudaStream_t s) {
  const int64_t n = B * S;
  if (n <= 0) return cudaSuccess;
  align_labels_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(
      tokens, loss_mask, seq_ids, B, S, shift, ignore_index, labels);
  return cudaGetLastError();
}

cudaError_t launch_flat_combine(const float* part, int nch, int64_t N, int64_t V, float* flat,
                                cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  flat_combine_kernel<<<static_cast<unsigned>((N + kCombineThreads - 1) / kCombineThreads),
                        kCombineThreads, 0, s>>>(part, nch, N, V, flat);
  return cudaGetLastError();
}

}  // namespace slm

namespace slm {
// Test hook: the FMA-pipe exponential and the MUFU one (exp2f) side by side.
__global__ void exp2_pair_kernel(const float* __restrict__ x, float* y_fma, float* y_mufu,
                                 int64_t n) {
  const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 a = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  const float2 f = exp2_fma2(a);
  y_fma[i] = f.x;
  y_mufu[i] = exp2f(a.x);
  if (i + 1 < n) {
    y_fma[i + 1] = f.y;
    y_mufu[i + 1] = exp2f(a.y);
  }
}

cudaError_t launch_exp2_pair(const float* x, float* y_fma, float* y_mufu, int64_t n,
                             cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t pairs = (n + 1) / 2;
  exp2_pair_kernel<<<static_cast<unsigned>((pairs + 255) / 256), 256, 0, s>>>(x, y_fma, y_mufu,
                                                                               n);
  return cudaGetLastError();
}
}  // namespace slm

// The persistent fused backward (one launch per chunk for the logits gradient, dH and dW).
#include "slm_bwd_fused.cuh"
