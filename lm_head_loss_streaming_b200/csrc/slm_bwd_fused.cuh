// slm_bwd_fused.cuh - the persistent fused backward of one token chunk ("Training
// speculative decoders: removing the logits and attention bottlenecks", "Backward pass":
// per chunk, recompute the logits, form their gradient, produce the chunk's hidden-state
// gradient and accumulate the LM-head gradient), as ONE launch instead of three.
//
// Included once, by slm_kernels.cu, after the epilogues and the pair launcher it reuses.
//
// The CTA pairs run three kinds of 2-SM tcgen05 GEMM units through one shared-memory ring
// (4 slots of 48 KB) and one 512-column TMEM allocation.  In claim order:
//   Z units  the logits-gradient tiles dZ = f(H W^T) (EpiDz / EpiDzCombo), in the
//            forward's raster order, in loose lockstep;
//   H units  dH = dZ W, 256 x 512 tiles, K = V;
//   W units  dW (+)= dZ^T H, 256 x 256 tiles double-buffered in TMEM, K = chunk rows.
// The leader CTA's producer claims the pair's next unit from a counter in global memory and
// hands it to every warp of both CTAs through a 4-deep queue in shared memory, so the pairs
// share the work dynamically (a pair that ends its dH tiles early takes more dW tiles).
// A dH tile of rows [256 m, +256) needs dZ rows [256 m, +256) over the whole vocabulary; a dW
// tile of vocabulary rows [256 v, +256) needs those dZ columns over every row of the chunk.
// So every epilogue warp, once the dZ stores of a Z unit have landed, adds 1 to the unit's
// M-tile counter and to its vocabulary-run counter; before loading anything of an H or W
// unit, the producer waits until the counter it needs is complete.  Every Z unit precedes
// every H and W unit in claim order, a Z unit waits for nothing (its lockstep wait gives up
// on its own), and a unit is only claimed by a running pair: so each counter a producer
// waits on is completed by running pairs, however many pairs are resident.  The wait is
// bounded all the same; if it runs out the kernel records kFlagTimeout and unwinds like
// every other bounded wait.
#pragma once

namespace slm {

constexpr int kFStages = 4;
constexpr uint32_t kFSlot = 48u * 1024u;  // one ring slot: the largest stage of the three kinds
constexpr int kFNwg = 2;                  // epilogue warpgroups per CTA
constexpr int kFThreads = 64 + 128 * kFNwg;
constexpr int kFQueue = 4;                // claimed units in flight between the warps
constexpr int kFStageBytesPerWarp = 4096;  // epilogue staging per warp (dZ and dW blocks)
// Readers of a queue slot, each arriving once on the leader's "empty" barrier: the leader's
// MMA warp and epilogue warps, the other CTA's producer and epilogue warps.
constexpr int kFQueueReaders = 1 + 4 * kFNwg + 1 + 4 * kFNwg;

struct FusedQueue {
  uint64_t full[kFQueue];   // per CTA: the slot holds a unit (arrived by the leader's claimer)
  uint64_t empty[kFQueue];  // leader only: every reader of both CTAs has read the slot
  int unit[kFQueue];        // claimed unit index, -1 = no more units
};

__device__ __forceinline__ int ld_acquire_s32(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add_s32(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Orders this thread's generic-proxy global accesses with its async-proxy (TMA) ones.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait on a barrier whose phase a remote CTA completes (all 32 lanes; the result is
// warp-uniform).
__device__ __forceinline__ bool wait_warp_cluster(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, const DevCtl& ctl) {
  const uint32_t a = smem_u32(bar);
  bool done = mbar_try_wait_cluster(a, parity);
  if (!done) {
    const long long t0 = clock64();
    while (true) {
      done = mbar_try_wait_cluster(a, parity);
      if (done || *abort) break;
      if (clock64() - t0 > ctl.timeout_cycles) {
        *abort = 1;
        atomicOr(ctl.status, kFlagTimeout);
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, done);
}

// The producer's wait for a dependency counter (warp-collective; lane 0 polls).  After it,
// the dZ tiles the counter covers are visible to this thread's TMA loads.
__device__ __forceinline__ bool wait_count(const int* ctr, int target, volatile int* abort,
                                           const DevCtl& ctl) {
  const int lane = threadIdx.x & 31;
  int ok = 1;
  if (lane == 0) {
    if (ld_acquire_s32(ctr) < target) {
      const long long t0 = clock64();
      while (ld_acquire_s32(ctr) < target) {
        if (*abort) {
          ok = 0;
          break;
        }
        if (clock64() - t0 > ctl.timeout_cycles) {
          *abort = 1;
          atomicOr(ctl.status, kFlagTimeout);
          ok = 0;
          break;
        }
        __nanosleep(256);
      }
    }
    fence_proxy_async_global();
  }
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Unit u of a num_m x num_n grid in raster groups of `group` M tiles: the groups in order,
// within a group the N tiles in order and the M tiles fastest.  Units claimed one after the
// other then share their N-tile operand, and the pairs running at one time read the
// operands of about `group` M tiles and 74 / `group` N tiles.
__device__ __forceinline__ void grouped_coords(int u, int num_m, int num_n, int group, int& mt,
                                               int& nt) {
  const int per_group = group * num_n;
  const int grp = u / per_group;
  const int r = u - grp * per_group;
  const int gm = min(group, num_m - grp * group);
  nt = r / gm;
  mt = grp * group + (r - nt * gm);
}

// Unit u of the claim order -> kind (0: Z, 1: H, 2: W) and its two coordinates: (M tile,
// vocabulary run) for Z, (M tile, N tile) for H and W.
__device__ __forceinline__ int fused_unit(const BwdFusedGeom& fg, int u, int& a, int& b) {
  const int uz = fg.gz.num_units;
  if (u < uz) {
    unit_coords(fg.gz, u, a, b);
    return 0;
  }
  u -= uz;
  const int uh = fg.num_mh * fg.num_nh;
  if (u < uh) {
    grouped_coords(u, fg.num_mh, fg.num_nh, fg.group_h, a, b);
    return 1;
  }
  grouped_coords(u - uh, fg.num_mw, fg.num_nw, fg.group_w, a, b);
  return 2;
}

template <bool DUAL, class EpiZ>
__global__ void __launch_bounds__(kFThreads, 1)
    bwd_fused_kernel(const __grid_constant__ CUtensorMap tHq,
                     const __grid_constant__ CUtensorMap tHp,
                     const __grid_constant__ CUtensorMap tWk,
                     const __grid_constant__ CUtensorMap tDzK,
                     const __grid_constant__ CUtensorMap tWmn,
                     const __grid_constant__ CUtensorMap tDzMn,
                     const __grid_constant__ CUtensorMap tHmn,
                     const __grid_constant__ BwdFusedGeom fg,
                     const __grid_constant__ DzParams pz, const DhParams ph, const DwParams pw,
                     const DevCtl ctl) {
  // Z units: the draft (and target) hidden states against W, both K-major.
  constexpr int kNumAZ = DUAL ? 2 : 1;
  constexpr int kSubZ = DUAL ? 1 : 2;
  constexpr int kTileZ = 256 * kSubZ;  // vocabulary columns per Z accumulator
  constexpr uint32_t kABytes = kBM * kBK * 2;      // 16 KB: 128 rows x 64 of K
  constexpr uint32_t kSliceBytes = 128 * kBK * 2;  // 16 KB: 128 columns x 64 of K
  constexpr uint32_t kStageZ = kNumAZ * kABytes + kSubZ * kSliceBytes;
  constexpr uint32_t kStageH = kABytes + 2 * kSliceBytes;
  constexpr uint32_t kStageW = kABytes + kSliceBytes;
  static_assert(kStageZ <= kFSlot && kStageH <= kFSlot && kStageW <= kFSlot, "ring slot");
  // Each stage's expected bytes are exactly the boxes its producer issues (bf16): Z: one
  // 64 x 128 box per operand and per 128-column W slice; H: one 64 x 128 dZ box and four
  // 64 x 64 W boxes; W: two 64 x 64 dZ boxes and two 64 x 64 H boxes.
  static_assert(kStageZ == (kNumAZ + kSubZ) * 64u * 128u * 2u, "Z stage bytes");
  static_assert(kStageH == 64u * 128u * 2u + 4u * 64u * 64u * 2u, "H stage bytes");
  static_assert(kStageW == 4u * 64u * 64u * 2u, "W stage bytes");
  constexpr uint32_t kIdescZ = idesc_bf16_f32(2 * kBM, 256, false, false);
  constexpr uint32_t kIdescH = idesc_bf16_f32(2 * kBM, 256, false, true);
  constexpr uint32_t kIdescW = idesc_bf16_f32(2 * kBM, 256, true, true);
  const GemmGeom& gz = fg.gz;
  const int total_units = gz.num_units + fg.num_mh * fg.num_nh + fg.num_mw * fg.num_nw;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  PairCtl<kFStages>* pc = reinterpret_cast<PairCtl<kFStages>*>(smem + kFStages * kFSlot);
  FusedQueue* fq = reinterpret_cast<FusedQueue*>(pc + 1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFStages; ++s) {
      mbar_init(&pc->full[s], 1);
      mbar_init(&pc->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&pc->tfull[b], 1);
      mbar_init(&pc->tempty[b], 2 * 4 * kFNwg);
    }
    mbar_init(&pc->fin, 1);
    for (int q = 0; q < kFQueue; ++q) {
      mbar_init(&fq->full[q], 1);
      mbar_init(&fq->empty[q], kFQueueReaders);
    }
    pc->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tHq);
    if (DUAL) tma_prefetch_desc(&tHp);
    tma_prefetch_desc(&tWk);
    tma_prefetch_desc(&tDzK);
    tma_prefetch_desc(&tWmn);
    tma_prefetch_desc(&tDzMn);
    tma_prefetch_desc(&tHmn);
  }
  if (warp == 1) {
    tmem_alloc_pair(&pc->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = pc->tmem_base;
  volatile int* abort = &pc->abort;

  // The next unit of this pair: the q-th slot of the queue.  Readers wait for the slot,
  // read it and release it on the leader; on abort they see -1.
  auto read_unit = [&](uint32_t q) -> int {
    const int slot = static_cast<int>(q % kFQueue);
    if (!wait_warp_cluster(&fq->full[slot], (q / kFQueue) & 1u, abort, ctl)) return -1;
    const int u = *reinterpret_cast<volatile int*>(&fq->unit[slot]);
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&fq->empty[slot]), 0));
    return u;
  };

  if (warp == 0) {
    // ------------------------------ TMA producer (both CTAs) ------------------------------
    uint32_t it = 0;
    bool ok = true;
    // Leader: claims the pair's next unit and publishes it to the queues of both CTAs.
    const uint32_t peer = rank ^ 1u;
    auto claim_unit = [&](uint32_t q) -> int {
      const int slot = static_cast<int>(q % kFQueue);
      if (!wait_warp_cluster(&fq->empty[slot], ((q / kFQueue) & 1u) ^ 1u, abort, ctl)) return -1;
      int u = -1;
      if (lane == 0) {
        u = atomicAdd(fg.claim, 1);
        if (u >= total_units) u = -1;
        fq->unit[slot] = u;
        st_shared_cluster_u32(mapa_shared(smem_u32(&fq->unit[slot]), peer),
                              static_cast<uint32_t>(u));
        mbar_arrive_cluster(mapa_shared(smem_u32(&fq->full[slot]), rank));
        mbar_arrive_cluster(mapa_shared(smem_u32(&fq->full[slot]), peer));
      }
      return __shfl_sync(0xffffffffu, u, 0);
    };
    // Acquires the next ring slot and announces its bytes (both CTAs') on the leader.
    auto acquire = [&](uint32_t stage_bytes) -> uint8_t* {
      const int s = it % kFStages;
      const uint32_t ph = (it / kFStages) & 1u;
      if (!wait_warp(&pc->empty[s], ph ^ 1u, abort, ctl)) return nullptr;
      if (lane == 0 && leader) mbar_arrive_expect_tx(&pc->full[s], 2 * stage_bytes);
      return smem + s * kFSlot;
    };
    const bool sync_pub =
        gz.epoch != 0 && leader && pair < kMaxSyncPairs && npairs <= kMaxSyncPairs;
    bool sync_on = sync_pub;
    bool sync_done = !sync_pub;
    uint32_t sync_step = 0;
    const int need_rows = gz.units_n * kFusedEpiWarps;
    const int need_runs = gz.num_m * kFusedEpiWarps;
    for (uint32_t q = 0; ok; ++q) {
      const int u = leader ? claim_unit(q) : read_unit(q);
      if (u < 0) break;
      int a, b;
      const int kind = fused_unit(fg, u, a, b);
      if (kind != 0 && !sync_done) {
        // Past the Z units: this pair holds nobody back in the lockstep any more.
        if (lane == 0)
          st_relaxed_u64(&g_pair_progress[pair],
                         (static_cast<unsigned long long>(gz.epoch) << 32) | 0xffffffffull);
        __syncwarp();
        sync_done = true;
      }
      if (kind == 0) {
        // Z unit (M tile a, vocabulary run b).
        const int mrow = a * 2 * kBM + static_cast<int>(rank) * kBM;
        const int n_end = min((b + 1) * gz.vc, gz.num_n);
        for (int nt = b * gz.vc; ok && nt < n_end; ++nt) {
          for (int kb = 0; kb < gz.k_blocks; ++kb, ++it) {
            if (sync_on && it % static_cast<uint32_t>(gz.sync_kb) == 0)
              sync_on = lockstep(gz, pair, npairs, ++sync_step, ctl);
            uint8_t* st = acquire(kStageZ);
            if (!st) {
              ok = false;
              break;
            }
            if (lane == 0) {
              uint64_t* bar = &pc->full[it % kFStages];
              const int k0 = kb * kBK;
              tma_load_2d_pair(st, &tHq, bar, k0, mrow);
              if (DUAL) tma_load_2d_pair(st + kABytes, &tHp, bar, k0, mrow);
#pragma unroll
              for (int sub = 0; sub < kSubZ; ++sub)
                tma_load_2d_pair(st + kNumAZ * kABytes + sub * kSliceBytes, &tWk, bar, k0,
                                 nt * kTileZ + sub * 256 + static_cast<int>(rank) * 128);
            }
            __syncwarp();
          }
        }
      } else if (kind == 1) {
        // H unit: dH[rows of M tile a, columns of N tile b] = dZ W (A = dZ K-major, B = W
        // read MN-major).
        if (gz.num_units > 0 && !wait_count(&fg.rows_done[a], need_rows, abort, ctl)) {
          ok = false;
          break;
        }
        const int mrow = a * 2 * kBM + static_cast<int>(rank) * kBM;
        for (int kb = 0; kb < fg.kb_h; ++kb, ++it) {
          uint8_t* st = acquire(kStageH);
          if (!st) {
            ok = false;
            break;
          }
          if (lane == 0) {
            uint64_t* bar = &pc->full[it % kFStages];
            const int k0 = kb * kBK;
            tma_load_2d_pair(st, &tDzK, bar, k0, mrow);
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
              const int ncol = b * 512 + sub * 256 + static_cast<int>(rank) * 128;
              uint8_t* bdst = st + kABytes + sub * kSliceBytes;
              tma_load_2d_pair(bdst, &tWmn, bar, ncol, k0);
              tma_load_2d_pair(bdst + 8192, &tWmn, bar, ncol + 64, k0);
            }
          }
          __syncwarp();
        }
      } else {
        // W unit: dW[vocabulary rows of tile a, columns of tile b] (+)= dZ^T H (both
        // operands MN-major: A from the dZ chunk, B from the chunk's hidden states).
        if (gz.num_units > 0) {
          const int run = ((a * 2 * kBM) / fg.bn_z) / gz.vc;
          if (!wait_count(&fg.runs_done[run], need_runs, abort, ctl)) {
            ok = false;
            break;
          }
        }
        const int mrow = a * 2 * kBM + static_cast<int>(rank) * kBM;
        const int ncol = b * 256 + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < fg.kb_w; ++kb, ++it) {
          uint8_t* st = acquire(kStageW);
          if (!st) {
            ok = false;
            break;
          }
          if (lane == 0) {
            uint64_t* bar = &pc->full[it % kFStages];
            const int k0 = kb * kBK;
            tma_load_2d_pair(st, &tDzMn, bar, mrow, k0);
            tma_load_2d_pair(st + 8192, &tDzMn, bar, mrow + 64, k0);
            tma_load_2d_pair(st + kABytes, &tHmn, bar, ncol, k0);
            tma_load_2d_pair(st + kABytes + 8192, &tHmn, bar, ncol + 64, k0);
          }
          __syncwarp();
        }
      }
    }
    if (!sync_done && lane == 0)
      st_relaxed_u64(&g_pair_progress[pair],
                     (static_cast<unsigned long long>(gz.epoch) << 32) | 0xffffffffull);
    __syncwarp();
    if (ok) {
      // Producer tail: the last stage releases (remote arrives from the leader's MMA warp)
      // land before this CTA exits.
      const uint32_t first = it > (uint32_t)kFStages ? it - kFStages : 0u;
      bool tail_ok = true;
      for (uint32_t i = first; tail_ok && i < it; ++i)
        tail_ok = wait_warp(&pc->empty[i % kFStages], (i / kFStages) & 1u, abort, ctl);
      if (!tail_ok)
        for (int i = 0; i < 100; ++i) __nanosleep(1000);
    } else if (leader) {
      // Aborting: the pair's copies in flight land before the final cluster barrier (the
      // full barriers count both CTAs' bytes).  Readers still waiting for a unit give up on
      // their own bounded waits.
      const uint32_t first = it > (uint32_t)kFStages ? it - kFStages : 0u;
      for (uint32_t i = first; i < it; ++i)
        wait_warp(&pc->full[i % kFStages], (i / kFStages) & 1u, abort, ctl, false);
    } else {
      for (int i = 0; i < 100; ++i) __nanosleep(1000);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (leader only) ------------------------------
    if (leader) {
      uint32_t it = 0;
      uint32_t acq0 = 0u, acq1 = 0u;  // times each TMEM buffer was taken
      uint32_t wt = 0;                // W tiles so far: they alternate between the buffers
      bool ok = true;
      // Takes TMEM buffer b (both halves for a 512-column tile) once the epilogue released it.
      auto take = [&](int b, bool wide) -> bool {
        if (wide || b == 0) {
          if (!wait_warp(&pc->tempty[0], (acq0 & 1u) ^ 1u, abort, ctl)) return false;
          ++acq0;
        }
        if (wide || b == 1) {
          if (!wait_warp(&pc->tempty[1], (acq1 & 1u) ^ 1u, abort, ctl)) return false;
          ++acq1;
        }
        tc_fence_after();
        return true;
      };
      // One tile: kb_n K blocks; `issue(addr, kb)` issues one stage's MMAs.
      auto run_tile = [&](int kb_n, int b, auto&& issue) -> bool {
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % kFStages;
          if (!wait_warp(&pc->full[s], (it / kFStages) & 1u, abort, ctl)) return false;
          tc_fence_after();
          if (lane == 0) {
            issue(smem_u32(smem + s * kFSlot), kb);
            umma_commit_pair_mc(&pc->empty[s], 0x3);
          }
          __syncwarp();
        }
        if (lane == 0) umma_commit_pair_mc(&pc->tfull[b], 0x3);
        __syncwarp();
        return true;
      };
      for (uint32_t q = 0; ok; ++q) {
        const int u = read_unit(q);
        if (u < 0) break;
        int a, b;
        const int kind = fused_unit(fg, u, a, b);
        if (kind == 0) {
          const int n_end = min((b + 1) * gz.vc, gz.num_n);
          for (int nt = b * gz.vc; ok && nt < n_end; ++nt) {
            ok = take(0, true) &&
                 run_tile(gz.k_blocks, 0, [&](uint32_t a_addr, int kb) {
                   const uint32_t b_addr = a_addr + kNumAZ * kABytes;
#pragma unroll
                   for (int kk = 0; kk < kBK / 16; ++kk)
#pragma unroll
                     for (int sub = 0; sub < kSubZ; ++sub) {
                       const uint64_t bd =
                           smem_desc_sw128(b_addr + sub * kSliceBytes + kk * 32, 16, 1024);
#pragma unroll
                       for (int x = 0; x < kNumAZ; ++x)
                         umma_bf16_pair(tmem + (x * kSubZ + sub) * 256,
                                        smem_desc_sw128(a_addr + x * kABytes + kk * 32, 16, 1024),
                                        bd, kIdescZ, (kb | kk) != 0 ? 1u : 0u);
                     }
                 });
          }
        } else if (kind == 1) {
          ok = take(0, true) &&
               run_tile(fg.kb_h, 0, [&](uint32_t a_addr, int kb) {
#pragma unroll
                 for (int kk = 0; kk < kBK / 16; ++kk) {
                   const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
#pragma unroll
                   for (int sub = 0; sub < 2; ++sub)
                     umma_bf16_pair(tmem + sub * 256, ad,
                                    smem_desc_sw128(
                                        a_addr + kABytes + sub * kSliceBytes + kk * 2048, 8192, 1024),
                                    kIdescH, (kb | kk) != 0 ? 1u : 0u);
                 }
               });
        } else {
          const int buf = static_cast<int>(wt & 1u);
          ++wt;
          ok = take(buf, false) &&
               run_tile(fg.kb_w, buf, [&](uint32_t a_addr, int kb) {
#pragma unroll
                 for (int kk = 0; kk < kBK / 16; ++kk)
                   umma_bf16_pair(tmem + buf * 256,
                                  smem_desc_sw128(a_addr + kk * 2048, 8192, 1024),
                                  smem_desc_sw128(a_addr + kABytes + kk * 2048, 8192, 1024),
                                  kIdescW, (kb | kk) != 0 ? 1u : 0u);
               });
        }
      }
      if (lane == 0) umma_commit_pair_mc(&pc->fin, 0x1);
      __syncwarp();
      wait_warp(&pc->fin, 0u, abort, ctl, false);
    }
  } else {
    // ------------------------------ epilogue (both CTAs) ------------------------------
    const int qw = warp & 3;  // a warp may only touch TMEM lanes [32 * (warp % 4), +32)
    const int wg = (warp - 2) >> 2;
    const int row = qw * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(qw * 32) << 16;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&pc->tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&pc->tempty[1]), 0);
    uint32_t got0 = 0u, got1 = 0u;  // times each tfull barrier was waited on
    uint32_t wt = 0;
    bool first_release = true;
    // Waits for TMEM buffer b's accumulator; returns false on abort.
    auto wait_acc = [&](int b) -> bool {
      uint32_t& got = b ? got1 : got0;
      if (!wait_warp(&pc->tfull[b], got & 1u, abort, ctl)) return false;
      ++got;
      tc_fence_after();
      return true;
    };
    // Releases buffer b (both for a 512-column tile) to the MMA issuer.
    auto release = [&](int b, bool wide) {
      tc_fence_before();
      __syncwarp();
      // Test hook (fault == 1): withhold the first release so that the MMA issuer's
      // bounded wait runs out and the kernel unwinds with a timeout.
      const bool withhold = ctl.fault == 1 && first_release;
      first_release = false;
      if (lane == 0 && !withhold) {
        if (wide || b == 0) mbar_arrive_cluster(tempty_leader0);
        if (wide || b == 1) mbar_arrive_cluster(tempty_leader1);
      }
    };
    // One staging buffer per epilogue warp, shared by the Z epilogue (dZ blocks on their way
    // to a TMA store) and the dW epilogue (its read-add-write blocks): a warp works on one
    // unit at a time.
    uint8_t* stage_base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(fq + 1) + 1023) & ~static_cast<uintptr_t>(1023));
    float* warp_stage = reinterpret_cast<float*>(stage_base + (warp - 2) * kFStageBytesPerWarp);
    EpiZ ez;
    if constexpr (EpiStageBytes<EpiZ>::value > 0) ez.stage = warp_stage;
    EpiDh eh;
    EpiDwStaged ew;
    ew.stage = warp_stage;
    bool ok = true;
    for (uint32_t q = 0; ok; ++q) {
      const int u = read_unit(q);
      if (u < 0) break;
      int a, b;
      const int kind = fused_unit(fg, u, a, b);
      const int row0 = a * 2 * kBM + static_cast<int>(rank) * kBM;
      if (kind == 0) {
        const int n_end = min((b + 1) * gz.vc, gz.num_n);
        ez.unit_begin(pz, row0, row);
        for (int nt = b * gz.vc; nt < n_end; ++nt) {
          if (!wait_acc(0)) {
            ok = false;
            break;
          }
          const int c0 = wg * (kTileZ / kFNwg);
          ez.template tile<kTileZ>(pz, tmem + lane_bits, row0, static_cast<int64_t>(nt) * kTileZ,
                                   c0, c0 + kTileZ / kFNwg, row);
          release(0, true);
        }
        if (!ok) break;
        ez.unit_end(pz, row0, 0, row);
        // This warp's dZ stores of the unit have landed: count the unit for its M tile and
        // its vocabulary run.
        if (lane == 0) bulk_wait_all();
        __threadfence();
        __syncwarp();
        if (lane == 0) {
          fence_proxy_async_global();
          red_release_add_s32(&fg.rows_done[a], 1);
          red_release_add_s32(&fg.runs_done[b], 1);
        }
      } else if (kind == 1) {
        if (!wait_acc(0)) {
          ok = false;
          break;
        }
        const int c0 = wg * 256;
        eh.tile<512>(ph, tmem + lane_bits, row0, static_cast<int64_t>(b) * 512, c0, c0 + 256,
                     row);
        release(0, true);
      } else {
        const int buf = static_cast<int>(wt & 1u);
        ++wt;
        if (!wait_acc(buf)) {
          ok = false;
          break;
        }
        const int c0 = wg * 128;
        ew.tile<256>(pw, tmem + lane_bits + buf * 256, row0, static_cast<int64_t>(b) * 256, c0,
                     c0 + 128, row);
        release(buf, false);
      }
    }
    if constexpr (EpiHasFinish<EpiZ>::value) ez.finish();
  }

  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

template <bool DUAL, class EpiZ>
static cudaError_t launch_bwd_fused_t(const CUtensorMap& tHq, const CUtensorMap& tHp,
                                      const CUtensorMap& tWk, const CUtensorMap& tDzK,
                                      const CUtensorMap& tWmn, const CUtensorMap& tDzMn,
                                      const CUtensorMap& tHmn, const BwdFusedGeom& fg_in,
                                      const DzParams& pz, const DhParams& ph,
                                      const DwParams& pw, const DevCtl& c, cudaStream_t s) {
  static_assert(EpiStageBytes<EpiZ>::value <= kFStageBytesPerWarp &&
                    EpiStageBytes<EpiDwStaged>::value <= kFStageBytesPerWarp,
                "epilogue staging per warp");
  constexpr size_t kSmem = 1024 + kFStages * static_cast<size_t>(kFSlot) +
                           sizeof(PairCtl<kFStages>) + sizeof(FusedQueue) + 1024 +
                           static_cast<size_t>(kFStageBytesPerWarp) * 4 * kFNwg;
  static_assert(kSmem <= 232448, "shared memory per CTA");
  auto kern = bwd_fused_kernel<DUAL, EpiZ>;
  cudaError_t e = cudaSuccess;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
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
  cfg.blockDim = dim3(kFThreads, 1, 1);
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
  const int units = fg_in.gz.num_units + fg_in.num_mh * fg_in.num_nh + fg_in.num_mw * fg_in.num_nw;
  const int pairs = std::max(1, std::min(units, max_clusters[dev]));
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  BwdFusedGeom fg = fg_in;
  fg.gz.epoch = 0;
  if (fg.gz.num_units > 0 && fg.gz.sync_kb > 0 && fg.gz.slack >= 0 && pairs > 1 &&
      pairs <= kMaxSyncPairs) {
    // A fresh tag per launch, from a range of its own.
    static std::atomic<uint32_t> next_epoch{1u << 30};
    uint32_t ep = next_epoch.fetch_add(1);
    if (ep == 0) ep = next_epoch.fetch_add(1);
    fg.gz.epoch = ep;
  }
  return cudaLaunchKernelEx(&cfg, kern, tHq, tHp, tWk, tDzK, tWmn, tDzMn, tHmn, fg, pz, ph, pw,
                            c);
}

cudaError_t launch_bwd_fused(int zkind, const CUtensorMap& tHq, const CUtensorMap& tHp,
                             const CUtensorMap& tWk, const CUtensorMap& tDzK,
                             const CUtensorMap& tWmn, const CUtensorMap& tDzMn,
                             const CUtensorMap& tHmn, const BwdFusedGeom& fg,
                             const DzParams& pz, const DhParams& ph, const DwParams& pw,
                             const DevCtl& c, cudaStream_t s) {
  if (zkind == 0)
    return launch_bwd_fused_t<false, EpiDz<false>>(tHq, tHp, tWk, tDzK, tWmn, tDzMn, tHmn, fg, pz,
                                                   ph, pw, c, s);
  if (zkind == 1)
    return launch_bwd_fused_t<true, EpiDz<true>>(tHq, tHp, tWk, tDzK, tWmn, tDzMn, tHmn, fg, pz,
                                                 ph, pw, c, s);
  return launch_bwd_fused_t<true, EpiDzCombo>(tHq, tHp, tWk, tDzK, tWmn, tDzMn, tHmn, fg, pz, ph,
                                              pw, c, s);
}

}  // namespace slm
