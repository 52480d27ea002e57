// slm_schedule.h - how the host lays the GEMMs' work out over the CTA pairs: tile and
// vocabulary-run sizes, raster groups and the loose-lockstep parameters.  Together with the
// kernels these decide the GEMMs' launch shape and memory traffic.  Included by
// slm_api.cu only.
#pragma once

#include <stdint.h>

#include <algorithm>

#include "../../include/slm.h"
#include "slm_internal.h"

namespace slm {
namespace {

#ifndef SLM_GROUP_PAIRS
#define SLM_GROUP_PAIRS 8
#endif
#ifndef SLM_MAX_RUNS
#define SLM_MAX_RUNS 32
#endif
// Loose lockstep of the GEMMs' CTA pairs (K blocks per progress step, steps of slack; 0 K
// blocks = off): V for the GEMMs over the vocabulary (forward, logits gradient, second
// pass), B for the dH and dW GEMMs.
// Raster groups of the persistent backward's dH and dW units (M tiles per group, M tile
// fastest).  Its pairs claim units one at a time and drift out of phase, so only units
// claimed close together share operands in L2; the groups put the units that share an
// operand next to each other.  The separate dH and dW launches start all pairs together
// and keep the plain row-major order.
#ifndef SLM_GROUP_B
#define SLM_GROUP_B 8
#endif
#ifndef SLM_SYNC_KB_V
#define SLM_SYNC_KB_V 16
#endif
#ifndef SLM_SYNC_SLACK_V
#define SLM_SYNC_SLACK_V 2
#endif
#ifndef SLM_SYNC_KB_B
#define SLM_SYNC_KB_B 0
#endif
#ifndef SLM_SYNC_SLACK_B
#define SLM_SYNC_SLACK_B 2
#endif
constexpr int kPairM = 2 * kBM;                // M rows of one 2-SM tile
constexpr int kGroupPairs = SLM_GROUP_PAIRS;   // pair M tiles per raster group
constexpr int kMaxRuns = SLM_MAX_RUNS;         // vocabulary runs per row, at most
constexpr int kGroupB = SLM_GROUP_B;           // M tiles per group of fused dH / dW units

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Kinds whose forward reads the target logits z_p (all but hard-label CE).
inline bool dual_kind(int k) { return k != SLM_CE; }

// M tiles per raster group of a grid of fused dH or dW units with num_n N tiles: half the
// group when a row of the grid is long (d >= 16384 for dH, >= 8192 for dW), where fewer M
// tiles per round keep each round's operand slices within L2 (measured at d = 16384:
// 1-2% faster than the full group; at d = 4096 the full group is 0.7% faster).
inline int group_b(int num_n) { return num_n >= 32 ? std::max(1, kGroupB / 2) : kGroupB; }

// Forward vocabulary schedule: tiles of `bn` columns, grouped into at most kMaxRuns runs per row
// (so the per-row partials stay O(N)), each run at least 2048 columns long.  Each run
// leaves kFwdPartsPerRun partial slots per row (one per epilogue warpgroup).
struct FwdSched {
  int bn, num_n, vc, units_n, slots, fields;
};

FwdSched fwd_sched(int kind, int64_t V) {
  FwdSched f;
  f.bn = dual_kind(kind) ? kTileDual : kTileCE;
  f.num_n = static_cast<int>(ceil_div(V, f.bn));
  const int min_vc = std::max(1, 2048 / f.bn);
  f.vc = std::max<int>(min_vc, static_cast<int>(ceil_div(f.num_n, kMaxRuns)));
  f.vc = std::min(f.vc, f.num_n);
  f.units_n = static_cast<int>(ceil_div(f.num_n, f.vc));
  f.slots = f.units_n * kFwdPartsPerRun;
  f.fields = kind == SLM_CE ? kCEFields : (kind == SLM_CE_ARGMAX_P ? kArgmaxFields : kDualFields);
  return f;
}

// Tile schedule of a GEMM with M tiles of `bm` rows (256: a 2-SM CTA pair).
GemmGeom geom(int64_t M, int64_t Nn, int64_t K, int bn, int vc, int group_m, int bm,
              int sync_kb, int slack) {
  GemmGeom g{};
  g.sync_kb = sync_kb;
  g.slack = slack;
  g.num_m = static_cast<int>(ceil_div(M, bm));
  g.num_n = static_cast<int>(ceil_div(Nn, bn));
  g.k_blocks = static_cast<int>(ceil_div(K, kBK));
  g.vc = std::max(1, std::min(vc, g.num_n));
  g.group_m = std::max(1, std::min(group_m, g.num_m));
  g.units_n = static_cast<int>(ceil_div(g.num_n, g.vc));
  g.num_units = g.num_m * g.units_n;
  return g;
}

}  // namespace
}  // namespace slm
