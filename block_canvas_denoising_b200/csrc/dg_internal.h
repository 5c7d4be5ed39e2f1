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
constexpr int kBlockK = 64;
constexpr int kStages = 6;
constexpr int kEpiWarps = 16;                     // 4 column groups x 4 lane quarters
constexpr int kColGroups = kEpiWarps / 4;         // 64 columns each
constexpr int kProducerWarp = kEpiWarps;          // warp 16
constexpr int kMmaWarp = kEpiWarps + 1;           // warp 17
constexpr int kHeadThreads = (kEpiWarps + 2) * 32;
constexpr int kAStageBytes = kBlockM * kBlockK * 2;
constexpr int kBStageBytes = kHalfN * kBlockK * 2;
constexpr int kPartialFields = 7;                 // m2, S, T2, zmax, zarg, gkey, garg
// per-unit exchange of the column groups' partials inside a CTA
constexpr int kPartSmemBytes = kColGroups * kBlockM * kPartialFields * 4;
constexpr int kHeadSmemBytes = kStages * (kAStageBytes + kBStageBytes) + 1024 + 256 + kPartSmemBytes;
constexpr uint64_t kDefaultWaitNs = 4000000000ull;

// Per-canvas step data, filled on the host.
struct CanvasParam {
  int32_t k;        // step index
  float inv_tau;    // float32(1 / tau_k), tau_k in float64
  uint8_t has_prev;
  uint8_t active;
  uint8_t pad[2];
};

// Work split of the head: MT pair row tiles (256 rows) x NT vocabulary
// tiles, cut into units of consecutive vocabulary tiles of one row tile.
// Unit u covers row tile u % MT and vocabulary tiles [q NT / Q, (q+1) NT / Q),
// q = u / MT; pair p runs units p, p + pairs, ...  grid = 2 * pairs CTAs.
struct HeadSplit {
  int MT, NT, KB, Q, units, pairs, grid;
};

struct HeadParams {
  int32_t R, d, V, B;
  HeadSplit split;
  uint32_t seed_lo, seed_hi;
  const float* e_scale;  // per-vocabulary-row scale (FP8) or null
  float* part;           // partial records, kPartialFields planes of [R][Q]
  uint32_t* err;         // device fault latch
  float* logits_out;     // optional raw logits [R, V]
  uint64_t wait_ns;
  uint32_t rk0[10], rk1[10];  // Philox round keys of the seed
  CanvasParam cp[DG_MAX_B];
};

struct MergeParams {
  int32_t R, B, V, P;
  const float* part;
  float* entropy;
  int32_t* sampled;
  int32_t* argmax;
  int32_t* canvas;
  int32_t* prev_argmax;
  uint8_t* accept;
  int32_t* stop;
  uint32_t* tickets;  // [B], self-resetting
  uint32_t seed_lo, seed_hi;
  double entropy_bound;
  double stop_entropy;
  CanvasParam cp[DG_MAX_B];
};

HeadSplit head_split(int R, int V, int d, int max_pairs);
int head_max_pairs();

// Workspace layout (byte offsets), see dg_workspace_size().
struct WsLayout {
  size_t err_off, tickets_off, part_off, total;
  int P;
};
WsLayout ws_layout(const dg_shape& s, int max_pairs);

// Text returned by dg_last_error_message() on this host thread.
void set_last_error_message(const char* msg);

cudaError_t launch_head(const CUtensorMap& tmA, const CUtensorMap& tmB, const HeadParams& p,
                        cudaStream_t stream);
cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream);
cudaError_t launch_wait_selftest(uint32_t* err, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_gumbel_probe(const uint32_t* words, int n, float* g_exact, float* lg2e_approx,
                                cudaStream_t stream);

}  // namespace dg
