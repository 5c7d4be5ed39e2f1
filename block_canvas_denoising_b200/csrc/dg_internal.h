// dg_internal.h -- kernel parameter blocks and launch helpers shared by the
// host entry points (dg_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dg.h"

namespace dg {

// Tile of the fused head+sampler kernel: 128 canvas rows x 256 vocabulary
// columns, K staged 64 bf16 (128 B, one swizzle row) at a time.
constexpr int kBlockM = 128;
constexpr int kBlockN = 256;
constexpr int kBlockK = 64;
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;                      // 2 column groups x 4 lane quarters
constexpr int kHeadThreads = 64 + kEpiWarps * 32; // producer, MMA, epilogue
constexpr int kAStageBytes = kBlockM * kBlockK * 2;
constexpr int kBStageBytes = kBlockN * kBlockK * 2;
constexpr int kHeadSmemBytes = kStages * (kAStageBytes + kBStageBytes) + 1024 + 256;
constexpr int kPartialFields = 7;                 // m2, S, T2, zmax, zarg, gkey, garg
constexpr uint64_t kDefaultWaitNs = 4000000000ull;

// Per-canvas step data, filled on the host.
struct CanvasParam {
  int32_t k;        // step index
  float inv_tau;    // float32(1 / tau_k), tau_k in float64
  uint8_t has_prev;
  uint8_t active;
  uint8_t pad[2];
};

// Work split of the head: MT row tiles x NT vocabulary tiles, cut into
// units of consecutive vocabulary tiles of one row tile.  Unit u covers row
// tile u % MT and vocabulary tiles [q NT / Q, (q+1) NT / Q), q = u / MT.
struct HeadSplit {
  int MT, NT, KB, Q, units, grid;
};

struct HeadParams {
  int32_t R, d, V, B;
  HeadSplit split;
  uint32_t seed_lo, seed_hi;
  const float* e_scale;  // per-vocabulary-row scale (FP8) or null
  float* part;           // partial records, kPartialFields planes of [2Q][R]
  uint32_t* err;         // device fault latch
  float* logits_out;     // optional raw logits [R, V]
  uint64_t wait_ns;
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

HeadSplit head_split(int R, int V, int d, int num_sms);

// Workspace layout (byte offsets), see dg_workspace_size().
struct WsLayout {
  size_t err_off, tickets_off, part_off, total;
  int P;
};
WsLayout ws_layout(const dg_shape& s, int num_sms);

cudaError_t launch_head(const CUtensorMap& tmA, const CUtensorMap& tmB, const HeadParams& p,
                        cudaStream_t stream);
cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream);
cudaError_t launch_wait_selftest(uint32_t* err, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_gumbel_probe(const uint32_t* words, int n, float* g_exact, float* lg2e_approx,
                                cudaStream_t stream);

}  // namespace dg
