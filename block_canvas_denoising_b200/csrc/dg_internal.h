// dg_internal.h -- kernel parameter blocks and launch helpers shared by the
// host entry points (dg_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dg.h"

namespace dg {

// Tile of the fused head+sampler kernel.  A CTA pair (cluster of 2, tcgen05
// cta_group::2) computes 256 canvas rows x 256 vocabulary columns per tile;
// each CTA stages 128 rows of h and 128 rows of E per 64-wide K block (one
// 128-byte swizzle row) and holds its 128 x 256 float32 half in TMEM.
constexpr int kPairM = 256;                       // rows per pair tile
constexpr int kBlockM = 128;                      // rows per CTA
constexpr int kBlockN = 256;                      // vocabulary columns per tile
constexpr int kHalfN = 128;                       // E rows staged per CTA
constexpr int kBlockK = 64;                       // bf16 K per stage: one 128-byte row
constexpr int kBlockKFp8 = 128;                   // E4M3 K per stage: one 128-byte row
constexpr int kEpiWarps = 16;                     // 4 column groups x 4 lane quarters
constexpr int kColGroups = kEpiWarps / 4;         // 64 columns each
// The MMA issuer is warp 0 and the TMA producer warp 1: the warp schedulers
// favour lower warps, and the single thread that feeds the tensor core must
// not wait behind the epilogue warps sharing its scheduler.  The epilogue
// warps 2..17 cover every (TMEM lane quarter = warp % 4, column group) pair.
constexpr int kMmaWarp = 0;
constexpr int kProducerWarp = 1;
constexpr int kEpiWarp0 = 2;
constexpr int kHeadThreads = (kEpiWarps + 2) * 32;
constexpr int kTileBytes = 128 * 128;             // 128 rows x 128 B, 128-byte swizzle
constexpr int kPartialFields = 7;                 // m2, S, T2, zmax, zarg, gkey, garg
// per-unit exchange of the column groups' partials inside a CTA
constexpr int kPartSmemBytes = kColGroups * kBlockM * kPartialFields * 4;
// best screening key seen so far by each column group, per row of the CTA
constexpr int kRecSmemBytes = kColGroups * kBlockM * 4;
// Largest Philox word of each group of 8 logits for the 32 rows of the MMA
// warp's lane quarter, one tile ahead, computed by the other epilogue warps:
// [2 buffers][32 rows][kBlockN / 8 groups].
constexpr int kWmaxSmemBytes = 2 * 32 * (kBlockN / 8) * 4;

// Pipeline of the two head variants.  bf16 embedder: a stage holds one h
// tile and one E tile of 64 K.  E4M3 embedder: a stage holds the two E4M3
// terms of h (h1, h2) and one tile of E codes, 128 K each.
template <bool kFp8>
struct HeadCfg {
  static constexpr int kStages = kFp8 ? 4 : 6;
  static constexpr int kBlockKElems = kFp8 ? kBlockKFp8 : kBlockK;
  static constexpr int kATiles = kFp8 ? 2 : 1;
  static constexpr int kStageBytes = (kATiles + 1) * kTileBytes;
  static constexpr int kSmemBytes =
      kStages * kStageBytes + 1024 + 256 + kPartSmemBytes + kRecSmemBytes + kWmaxSmemBytes;
};
static_assert(HeadCfg<false>::kSmemBytes <= 232448, "bf16 head exceeds 227 KB of shared memory");
static_assert(HeadCfg<true>::kSmemBytes <= 232448, "FP8 head exceeds 227 KB of shared memory");
constexpr uint64_t kDefaultWaitNs = 4000000000ull;

// Per-canvas step data, filled on the host.
struct CanvasParam {
  int32_t k;        // Philox counter step word: step index | block << 16
  float inv_tau;    // float32(1 / tau_k), tau_k in float64
  uint8_t has_prev;
  uint8_t active;
  uint8_t pad[2];
};

// Work split of the head: MT pair row tiles (256 rows, one canvas each) x NT
// vocabulary tiles, cut into units of consecutive vocabulary tiles of one
// row tile.  Unit u covers row tile u % MT and vocabulary tiles
// [q NT / Q, (q+1) NT / Q), q = u / MT; pair p runs units p, p + pairs, ...
// grid = 2 * pairs CTAs.  Row tile m is canvas HeadParams::mtile[m]: only
// the canvases a step updates are split (a frozen canvas costs no work).
struct HeadSplit {
  int MT, NT, KB, Q, units, pairs, grid;
};

struct HeadParams {
  int32_t R, d, V, B;
  int32_t v_off;         // vocabulary index of E's first row (vocabulary-sharded step), else 0
  HeadSplit split;
  uint32_t seed_lo, seed_hi;
  const float* e_scale;  // FP8: per-vocabulary-row scale, else null
  const float* row_inv;  // FP8: 2^-k_r, the inverse of h's per-row split scale, else null
  float* part;           // partial records, kPartialFields planes of [R][Q]
  uint32_t* err;         // device fault latch
  float* logits_out;     // optional raw logits [R, V]
  uint32_t* row_rec;     // [R] best screening key per row so far (ordered encoding, 0 = none)
  uint64_t wait_ns;
  uint32_t rk0[10], rk1[10];  // Philox round keys of the seed
  CanvasParam cp[DG_MAX_B];
  uint8_t mtile[DG_MAX_B];     // canvas of row tile m (m < split.MT)
  // Device-side loop: when set, the per-canvas data, the row tiles' canvases
  // and their number are read from device memory (written by the loop's
  // control kernel) instead of cp, mtile and split.MT.
  const CanvasParam* cp_dev;
  const uint8_t* mtile_dev;
  const int32_t* mt_dev;
  // Self-conditioning signal: when set, also write the block-scaled
  // probabilities ptilde[r, v] = bf16(2^(z c2 - pref[v / 64, r])) [R, V] and
  // the block references pref [V / 64, R].
  uint16_t* ptilde;
  float* pref;
};

struct MergeParams {
  int32_t R;             // rows of the whole batch (plane stride of the records)
  int32_t B;             // canvases this launch updates (canvas_of[0 .. B-1])
  int32_t V, P;
  int32_t S;             // shards: records of row r are shard s's [7][R][P] block, s < S
  const float* part;
  float* entropy;
  int32_t* sampled;
  int32_t* argmax;
  int32_t* canvas;
  int32_t* prev_argmax;
  uint8_t* accept;
  int32_t* stop;
  uint32_t* tickets;  // [B], self-resetting
  uint32_t* row_rec;  // [R] the head's per-row key records, cleared here for the next step
  uint32_t seed_lo, seed_hi;
  double entropy_bound;
  double stop_entropy;
  int32_t selection_rule;  // dg_selection
  int32_t top_k;
  CanvasParam cp[DG_MAX_B];
  uint8_t canvas_of[DG_MAX_B];  // canvas of block group g (32 CTAs per canvas)
  // Device-side loop: per-canvas data, the canvases to update and their
  // number from device memory; block groups past the number exit at once.
  const CanvasParam* cp_dev;
  const uint8_t* canvas_of_dev;
  const int32_t* n_dev;
  float2* rowstat;  // self-conditioning: per row (m2, 1 / S) of the merged softmax, or null
};

// kblock: K elements per stage (kBlockK, or kBlockKFp8 for the FP8 head);
// KB = ceil(d / kblock), the last stage's K tail read as zeros.  At most
// q_cap units per row tile (the records per row the workspace holds).
HeadSplit head_split(int R, int V, int d, int max_pairs, int kblock, int q_cap = 1 << 30);
int head_max_pairs(bool fp8);

// Device memory of the device-side loop (inside the caller's loop-state
// buffer): the per-canvas data of the step about to run, the canvases still
// running (canvas_of[0 .. *n_active - 1]) and their number.
struct LoopDevState {
  CanvasParam* cp;
  uint8_t* canvas_of;
  int32_t* n_active;
};

// Enqueue one step whose per-canvas data come from `loop` (device memory)
// with every canvas's work split prepared, as the device-side loop's graph
// body does; k_any is any valid step index (used for the host-side checks).
dg_status enqueue_loop_step(const dg_shape* shape, const dg_params* params, const void* h, const void* E,
                            const float* e_scale, int32_t k_any, int32_t* canvas, int32_t* prev_argmax,
                            uint8_t* accept, float* entropy, int32_t* sampled, int32_t* argmax, int32_t* stop,
                            void* workspace, size_t ws_bytes, const LoopDevState* loop, cudaStream_t stream);

// Workspace layout (byte offsets), see dg_workspace_size().
struct WsLayout {
  size_t err_off, tickets_off, rec_off, part_off, h1_off, h2_off, rinv_off, total;
  size_t zero_prefix;  // bytes from the start that must be zero before a step (latch, tickets, records)
  int P;
};
// FP8 embedder only: h1, h2 E4M3 [R, d] (the two terms of h's split) and
// rinv float [R] (2^-k_r).
WsLayout ws_layout(const dg_shape& s, int max_pairs);

// Text returned by dg_last_error_message() on this host thread.
void set_last_error_message(const char* msg);

// The argument checks of dg_denoise_step other than those of the workspace
// (shape, parameters, pointers, alignment, step range, device): DG_OK or
// the status dg_denoise_step would return, before anything is enqueued.
dg_status check_step_call(const dg_shape* shape, const dg_params* params, const void* h, const void* E,
                          const float* e_scale, const int32_t* step_idx, const uint8_t* has_prev,
                          int32_t* canvas, int32_t* prev_argmax, uint8_t* accept, float* entropy,
                          int32_t* sampled, int32_t* argmax, int32_t* stop);

// Synchronise `st`, read the 32-bit fault latch at `latch` (device), clear it
// if set, and map it to a status (DG_OK, DG_ERR_TIMEOUT, DG_ERR_VALUE,
// DG_ERR_CUDA).
dg_status read_and_clear_latch(void* latch, cudaStream_t st);

// bf16 head: tmA = h bf16 [R, d], tmB = E bf16 [V, d] (tmA2 unused).
// FP8 head:  tmA = h1, tmA2 = h2 (E4M3 [R, d]), tmB = E codes E4M3 [V, d].
// pdl: launch as a programmatic dependent of the preceding kernel (off
// inside graphs built by the device-side loop).
cudaError_t launch_head(bool fp8, const CUtensorMap& tmA, const CUtensorMap& tmA2, const CUtensorMap& tmB,
                        const HeadParams& p, cudaStream_t stream, bool pdl = true);
// Split each row r of h (bf16 [R, d], d a multiple of 8, 16-byte aligned)
// into E4M3 terms h1 + h2 = h * 2^k_r and write rinv[r] = 2^-k_r; latches
// kErrHiddenRange in *err if some h is not finite.
cudaError_t launch_hidden_split(const void* h, uint8_t* h1, uint8_t* h2, float* rinv, int R, int d,
                                uint32_t* err, cudaStream_t stream);
// pdl: launch as a programmatic dependent of the preceding kernel (the
// head); off inside graphs built by the device-side loop.
cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream, bool pdl = true);
// canvas[b * L + s] = (r V) >> 32, r = Philox word 0 of counter
// (0, s | 3 << 16, ctr_step, b): the uniform noise a block starts from.
cudaError_t launch_init_canvas(int32_t* canvas, int B, int L, int V, uint32_t ctr_step, uint32_t seed_lo,
                               uint32_t seed_hi, cudaStream_t stream);
// Self-conditioning signal (selfcond.cu): normalise the head's block-scaled
// probabilities P [R, V] (bf16, in place) with the merged row statistics,
// then signal = P . Et^T by split-K tcgen05 GEMM into `part` and a fixed-
// order reduction.  e_scale: the FP8 embedder's row scales (folded into P),
// else null.
cudaError_t launch_selfcond(const uint16_t* P, const uint16_t* Et, const float* pref, const float2* rowstat,
                            const float* e_scale, float* part, float* signal, int R, int d, int V, uint32_t* err,
                            cudaStream_t stream);
// K slices of the split-K GEMM and co-resident CTA pairs of it (per device).
int selfcond_slices(int R, int d, int V, int pairs);
int selfcond_gemm_pairs();
// Et[c, v] = E[v, c] as bf16 (E4M3 codes widen exactly); V, d multiples of 32.
cudaError_t launch_transpose(const void* E, bool fp8, uint16_t* Et, int V, int d, cudaStream_t stream);

// The argument checks shared by the entry points (shape; parameters).
dg_status check_shape_and_params(const dg_shape* shape, const dg_params* params);
cudaError_t launch_wait_selftest(uint32_t* err, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_gumbel_probe(const uint32_t* words, int n, float* g_exact, float* lg2e_approx,
                                cudaStream_t stream);

}  // namespace dg
