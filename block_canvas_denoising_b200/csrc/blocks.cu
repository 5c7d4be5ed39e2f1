// blocks.cu -- block-by-block generation ("DiffusionGemma Technical Report",
// Figure 4: generation proceeds block after block; each 256-token block is
// denoised from noise until it settles, then encoded and appended to the
// context the next block is conditioned on).
//
// The model (encoder, KV cache, denoiser) is the caller's: it is reached
// through the hidden-state callback, which receives the blocks committed so
// far.  This file adds the noise canvas a block starts from (uniform over
// the vocabulary, Figure 3) and the driver that chains the adaptive loop over
// blocks, each block drawing its own random streams (the block index enters
// the Philox counter's step word).
#include <string.h>

#include "dg_device.cuh"
#include "dg_internal.h"

namespace dg {

__global__ void __launch_bounds__(256) init_canvas_kernel(int32_t* canvas, int n, int L, int V, uint32_t ctr_step,
                                                          uint32_t seed_lo, uint32_t seed_hi) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t b = static_cast<uint32_t>(i / L);
  const uint32_t s = static_cast<uint32_t>(i % L);
  uint32_t r[4];
  philox4x32_10(0u, s | (kPurposeInit << 16), ctr_step, b, seed_lo, seed_hi, r);
  canvas[i] = static_cast<int32_t>((static_cast<uint64_t>(r[0]) * static_cast<uint64_t>(V)) >> 32);
}

cudaError_t launch_init_canvas(int32_t* canvas, int B, int L, int V, uint32_t ctr_step, uint32_t seed_lo,
                               uint32_t seed_hi, cudaStream_t stream) {
  const int n = B * L;
  init_canvas_kernel<<<(n + 255) / 256, 256, 0, stream>>>(canvas, n, L, V, ctr_step, seed_lo, seed_hi);
  return cudaGetLastError();
}

namespace {

// Adapts the block callback to the loop's: the loop calls back with
// (k, canvas, h_out); the block, the committed prefix and the caller's
// context ride along here.
struct BlockCall {
  dg_block_hidden_fn fn;
  void* user;
  int32_t block;
  const int32_t* committed;
};

int block_trampoline(int32_t k, const int32_t* canvas, void* h_out, void* user, void* stream) {
  const BlockCall* c = static_cast<const BlockCall*>(user);
  return c->fn(c->block, k, canvas, c->committed, h_out, c->user, stream);
}

}  // namespace

}  // namespace dg

using namespace dg;

extern "C" dg_status dg_init_canvas(const dg_shape* shape, const dg_params* params, int32_t* canvas,
                                    void* stream) {
  const dg_status st = check_shape_and_params(shape, params);
  if (st != DG_OK) return st;
  if (canvas == nullptr) return DG_ERR_INVALID_ARG;
  const uint32_t ctr_step = static_cast<uint32_t>(params->block) << 16;  // k = 0 of the block
  if (launch_init_canvas(canvas, shape->B, shape->L, shape->V, ctr_step,
                         static_cast<uint32_t>(params->seed & 0xFFFFFFFFull),
                         static_cast<uint32_t>(params->seed >> 32), static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return DG_ERR_CUDA;
  return DG_OK;
}

extern "C" dg_status dg_generate_blocks(const dg_shape* shape, const dg_params* params, const void* E,
                                        const float* e_scale, int32_t n_blocks, dg_block_hidden_fn hidden_fn,
                                        void* user, void* h_buf, int32_t* blocks, int32_t* steps_taken,
                                        int32_t* canvas, int32_t* prev_argmax, uint8_t* accept, float* entropy,
                                        int32_t* sampled, int32_t* argmax, int32_t* stop, void* workspace,
                                        size_t ws_bytes, void* stream) {
  dg_status st = check_shape_and_params(shape, params);
  if (st != DG_OK) return st;
  if (n_blocks < 1 || hidden_fn == nullptr || blocks == nullptr || steps_taken == nullptr || canvas == nullptr)
    return DG_ERR_INVALID_ARG;
  if (static_cast<int64_t>(params->block) + n_blocks - 1 > 65535) return DG_ERR_INVALID_ARG;
  const int B = shape->B;
  const size_t rows = static_cast<size_t>(B) * shape->L;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t has_prev[DG_MAX_B];
  for (int32_t j = 0; j < n_blocks; ++j) {
    dg_params pj = *params;
    pj.block = params->block + j;
    if ((st = dg_init_canvas(shape, &pj, canvas, stream)) != DG_OK) return st;
    memset(has_prev, 0, sizeof(has_prev));
    BlockCall call{hidden_fn, user, j, j > 0 ? blocks : nullptr};
    st = dg_denoise_loop(shape, &pj, E, e_scale, block_trampoline, &call, 0, h_buf, canvas, prev_argmax,
                         has_prev, steps_taken + static_cast<size_t>(j) * B, accept, entropy, sampled, argmax,
                         stop, workspace, ws_bytes, stream);
    if (st != DG_OK) return st;
    // append: the committed block joins the context of the next ones
    if (cudaMemcpyAsync(blocks + static_cast<size_t>(j) * rows, canvas, sizeof(int32_t) * rows,
                        cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
      return DG_ERR_CUDA;
  }
  if (cudaStreamSynchronize(cs) != cudaSuccess) return DG_ERR_CUDA;
  return DG_OK;
}
