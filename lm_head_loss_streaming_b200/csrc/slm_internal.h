// slm_internal.h - types shared by the host orchestrator (slm_api.cu) and the kernels
// (slm_kernels.cu).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace slm {

// Tile shape of every GEMM: a 2-SM CTA pair computes 256 rows of the M operand (128 per
// CTA, one TMEM lane per row) with 64 bf16 of K per pipeline stage (one 128-byte swizzle
// row).  N tile widths (columns of one accumulator):
constexpr int kBM = 128;          // M rows per CTA
constexpr int kBK = 64;           // K per stage
constexpr int kTileCE = 512;      // CE forward / logits-gradient: one accumulator, 2 x 256-wide MMAs
constexpr int kTileDual = 256;    // target + draft: two accumulators of 256 columns
constexpr int kTileDh = 512;      // dH = dZ W
constexpr int kTileDw = 256;      // dW += dZ^T H (double-buffered)
// The forward epilogue runs as two warpgroups, each over half of the tile's columns, and
// each writes its own per-row partial statistics: partial slots per vocabulary run.
constexpr int kFwdPartsPerRun = 2;

// Device status word bits.
constexpr int kFlagLabelRange = 1;
constexpr int kFlagTimeout = 2;

enum LossKind : int { kCE = 0, kKL = 1, kTV = 2, kNLA = 3, kLK = 4, kRKL = 5, kJSD = 6,
                      kCEArgmax = 7 };

// Fields of the forward's per-row partial statistics (per vocabulary-run slot).
constexpr int kDualFields = 6;    // m_q, s_q, m_p, s_p, A (p-weighted z_p - z_q), B (q-weighted z_q - z_p)
constexpr int kArgmaxFields = 5;  // m_q, s_q, max z_p, its column, z_q at that column
constexpr int kCEFields = 2;      // m, s

// Weighted combinations: one weight per loss kind (0 = term absent).
constexpr int kNumKinds = 8;
constexpr int kUnionFields = 9;   // pass 1: the dual fields + max z_p, its column, z_q there
constexpr int kPass2Fields = 4;   // pass 2: alpha, S, jp, jq
constexpr int kComboStats = 9;    // L_q, L_p, KL, RKL, alpha, S, JSD, T, argmax target
struct ComboW {
  float w[kNumKinds];
};

// Persistent tile schedule.  Work units are (M tile, run of `vc` consecutive N tiles);
// units are ordered in groups of `group_m` M tiles: for each N run, every M tile of the
// group, so that CTAs running at the same time share the N-operand tiles in L2.
struct GemmGeom {
  int num_m;      // M tiles
  int num_n;      // N tiles
  int k_blocks;   // K blocks of kBK
  int vc;         // N tiles per unit
  int group_m;    // M tiles per raster group
  int units_n;    // ceil(num_n / vc)
  int num_units;  // num_m * units_n
  // Loose lockstep of the pairs (set at launch): every sync_kb K blocks a pair publishes its
  // progress under this launch's tag `epoch` and waits, briefly and boundedly, until no
  // started pair is more than `slack` such steps behind it.  epoch 0 = off.
  uint32_t epoch;
  int sync_kb;
  int slack;
  // CTA pairs to leave idle (so that a collective on another stream finds free SMs).
  int reserve_pairs;
};

struct DevCtl {
  int* status;               // device status word (in the workspace)
  long long timeout_cycles;  // bound of every pipeline wait
  int fault;                 // test hook: 1 = the epilogue withholds its first accumulator
                             // release; 2 = the pairs' lockstep waits give up at once
};

// Forward statistics (pass 1) and the alpha pass (pass 2).
struct FwdParams {
  const int32_t* labels;  // CE labels (required for CE)
  int32_t ignore_index;
  int64_t N, V;
  float* part;         // [units_n * kFwdPartsPerRun][fields][N]
  float* zy;           // [N] label logit (CE)
  const float* stats;  // pass 2: L_q, L_p
  int with_jsd;        // combination pass 2: accumulate the JSD halves too
  float* lq_out;       // fused path: store the fp32 draft logits here ([N][ldl]), or NULL
  float* lp_out;       // fused path: store the fp32 target logits here, or NULL
  int64_t ldl;         // leading dimension of the stored logits (V rounded up to 4)
  CUtensorMap lq_map;  // fused path: store maps of lq_out / lp_out as fp32 [N][V] (row
  CUtensorMap lp_map;  // stride ldl), box 32 x 32, 128-byte swizzle
};

// Logits-gradient tile (backward recompute + dZ epilogue).
struct DzParams {
  int kind;
  const int32_t* labels;
  int32_t ignore_index;
  int64_t row0, rows;  // token chunk [row0, row0 + rows)
  int64_t N, V;
  const float* stats;
  const float* grad_tok;
  const float* grad_scale;
  const int64_t* n_valid;
  __nv_bfloat16* dz;  // [rows][ldz]
  int64_t ldz;
  ComboW cw;          // weighted combination (EpiDzCombo only)
  CUtensorMap dz_map;  // dz as bf16 [rows][V] (row stride ldz), box 64 x 32, 128-byte
                       // swizzle: the store map of EpiDz
};

struct DhParams {
  __nv_bfloat16* dH;  // [N][d]
  int64_t row0, rows, d;
};

struct DwParams {
  float* dW;  // [V][d]
  int64_t V, d;
  int beta;  // 1: add to dW, 0: overwrite
};

// Persistent fused backward of one token chunk (bwd_fused_kernel): the logits-gradient
// units (Z), then the dH units (H) and the dW units (W) in one launch, claimed by the CTA
// pairs in that order from a counter.  Every epilogue warp counts the Z units it finished
// per M tile and per vocabulary run; a producer waits for the counts its next dH or dW unit
// needs.
constexpr int kFusedEpiWarps = 16;  // epilogue warps of a pair (2 CTAs x 2 warpgroups)
struct BwdFusedGeom {
  GemmGeom gz;           // Z units (M = chunk rows, N = V, K = d); gz.num_units = 0: none
  int bn_z;              // dZ tile width (vocabulary columns per Z tile)
  int num_mh, num_nh;    // H units: 256-row M tiles of the chunk x 512-column tiles of d
  int kb_h;              // H K blocks (over V)
  int num_mw, num_nw;    // W units: 256-row tiles of the vocabulary x 256-column tiles of d
  int kb_w;              // W K blocks (over the chunk's rows)
  int group_h, group_w;  // M tiles per raster group of the H and W units (M tile fastest)
  int* claim;            // next unit to claim (zero at launch)
  int* rows_done;        // [gz.num_m] finished Z units per M tile, x kFusedEpiWarps
  int* runs_done;        // [gz.units_n] finished Z units per vocabulary run, x kFusedEpiWarps
};

// Kernel launchers (slm_kernels.cu).  Each returns the launch's error status.
int sm_count();
cudaError_t launch_fwd_ce(const CUtensorMap& tH, const CUtensorMap& tW, const GemmGeom& g,
                          const FwdParams& p, const DevCtl& c, cudaStream_t s);
cudaError_t launch_fwd_dual(const CUtensorMap& tHq, const CUtensorMap& tHp, const CUtensorMap& tW,
                            const GemmGeom& g, const FwdParams& p, const DevCtl& c, bool rkl,
                            cudaStream_t s);
cudaError_t launch_fwd_argmax(const CUtensorMap& tHq, const CUtensorMap& tHp,
                              const CUtensorMap& tW, const GemmGeom& g, const FwdParams& p,
                              const DevCtl& c, cudaStream_t s);
cudaError_t launch_jsd(const CUtensorMap& tHq, const CUtensorMap& tHp, const CUtensorMap& tW,
                       const GemmGeom& g, const FwdParams& p, const DevCtl& c, cudaStream_t s);
cudaError_t launch_alpha(const CUtensorMap& tHq, const CUtensorMap& tHp, const CUtensorMap& tW,
                         const GemmGeom& g, const FwdParams& p, const DevCtl& c,
                         cudaStream_t s);
cudaError_t launch_dz_ce(const CUtensorMap& tH, const CUtensorMap& tW, const GemmGeom& g,
                         const DzParams& p, const DevCtl& c, cudaStream_t s);
cudaError_t launch_dz_dual(const CUtensorMap& tHq, const CUtensorMap& tHp, const CUtensorMap& tW,
                           const GemmGeom& g, const DzParams& p, const DevCtl& c,
                           cudaStream_t s);
cudaError_t launch_dh(const CUtensorMap& tDz, const CUtensorMap& tW, const GemmGeom& g,
                      const DhParams& p, const DevCtl& c, cudaStream_t s);
cudaError_t launch_dw(const CUtensorMap& tDzT, const CUtensorMap& tH, const GemmGeom& g,
                      const DwParams& p, const DevCtl& c, cudaStream_t s);
// The persistent fused backward of one chunk.  zkind: 0 = CE logits gradient (one
// operand), 1 = the divergences' (two operands), 2 = weighted combination; with
// fg.gz.num_units == 0 only phases H and W run (dZ already in the chunk buffer).  The
// launcher sets the lockstep tag of the Z units; the claim counter and the completion
// counters must be zero when the launch starts.
cudaError_t launch_bwd_fused(int zkind, const CUtensorMap& tHq, const CUtensorMap& tHp,
                             const CUtensorMap& tWk, const CUtensorMap& tDzK,
                             const CUtensorMap& tWmn, const CUtensorMap& tDzMn,
                             const CUtensorMap& tHmn, const BwdFusedGeom& fg,
                             const DzParams& pz, const DhParams& ph, const DwParams& pw,
                             const DevCtl& c, cudaStream_t s);

// Fused forward + backward over stored chunk logits.
// Valid rows (label != ignore_index; for CE also in [0, V)) -> *n_valid.
cudaError_t launch_count_valid(const int32_t* labels, int32_t ignore_index, int64_t N,
                               int64_t V, int check_range, int64_t* n_valid, cudaStream_t s);
// Second pass of the alpha losses / JSD from stored logits: one partial slot per row.
cudaError_t launch_logits_pass2(int kind, const float* lq, const float* lp, int64_t ldl,
                                const float* stats, int64_t row0, int64_t ldN, int64_t rows,
                                int64_t V, float* part, cudaStream_t s);
// Logits gradient of the rows [p.row0, p.row0 + p.rows) from stored logits.
cudaError_t launch_logits_dz(const DzParams& p, const float* lq, const float* lp, int64_t ldl,
                             cudaStream_t s);

// Test hook: the epilogues' FMA-pipe 2^x beside exp2f, elementwise.
cudaError_t launch_exp2_pair(const float* x, float* y_fma, float* y_mufu, int64_t n,
                             cudaStream_t s);

// Draft-head helpers.
constexpr int kFlatFields = 3;  // m, s, s2 = sum 2^(2 (z log2e - m))
cudaError_t launch_align_labels(const int32_t* tokens, const uint8_t* loss_mask,
                                const int32_t* seq_ids, int64_t B, int64_t S, int32_t shift,
                                int32_t ignore_index, int32_t* labels, cudaStream_t s);
cudaError_t launch_fwd_flat(const CUtensorMap& tHp, const CUtensorMap& tW, const GemmGeom& g,
                            const FwdParams& p, const DevCtl& c, cudaStream_t s);
cudaError_t launch_flat_combine(const float* part, int nch, int64_t N, int64_t V,
                                float* flat, cudaStream_t s);

// Weighted combinations.
cudaError_t launch_fwd_union(const CUtensorMap& tHq, const CUtensorMap& tHp,
                             const CUtensorMap& tW, const GemmGeom& g, const FwdParams& p,
                             const DevCtl& c, cudaStream_t s);
cudaError_t launch_pass2_union(const CUtensorMap& tHq, const CUtensorMap& tHp,
                               const CUtensorMap& tW, const GemmGeom& g, const FwdParams& p,
                               const DevCtl& c, cudaStream_t s);
cudaError_t launch_dz_combo(const CUtensorMap& tHq, const CUtensorMap& tHp,
                            const CUtensorMap& tW, const GemmGeom& g, const DzParams& p,
                            const DevCtl& c, cudaStream_t s);
// pass 1: stats 0-3 and 8, per-term losses of ce / kl / rkl / argmax; pass 2: stats 4-7 and
// the per-term losses of tv / nla / lk / jsd.  term_tok is [kNumKinds][N].
cudaError_t launch_combo_combine(int pass, const ComboW& cw, const float* part, int nch,
                                 const float* zy, const int32_t* labels, int32_t ignore_index,
                                 int64_t N, int64_t V, float* stats, float* term_tok,
                                 int* status, cudaStream_t s);
// Weighted per-token total, optional copy of the per-term losses, per-block sums of the
// total and of every term ([nblk][1 + kNumKinds] doubles) and valid counts.
cudaError_t launch_combo_total(const ComboW& cw, const float* term_tok, const int32_t* labels,
                               int32_t ignore_index, int64_t N, int64_t V, float* loss_tok,
                               float* term_out, double* blk_sums, long long* blk_cnt,
                               cudaStream_t s);
cudaError_t launch_combo_finalize(const double* blk_sums, const long long* blk_cnt, int nblk,
                                  double* loss_sum, double* term_sum, int64_t* n_valid,
                                  float* loss_mean, cudaStream_t s);

// Row combines and the deterministic loss reduction.
// N rows starting at row0 of a batch whose statistics have leading dimension ldN
// (-1: ldN = N); partials and label logits are indexed by the row within the launch.
cudaError_t launch_combine(int kind, int pass, const float* part, int nch, const float* zy,
                           const int32_t* labels, int32_t ignore_index, int64_t N, int64_t V,
                           float* loss_tok, float* alpha_tok, float* stats, double* blk_sum,
                           long long* blk_cnt, int* status, cudaStream_t s, int64_t row0 = 0,
                           int64_t ldN = -1);
cudaError_t launch_finalize(const double* blk_sum, const long long* blk_cnt, int nblk,
                            double* loss_sum, int64_t* n_valid, float* loss_mean,
                            cudaStream_t s);
cudaError_t launch_zero_f32(float* p, int64_t n, cudaStream_t s);

constexpr int kCombineThreads = 256;

}  // namespace slm
