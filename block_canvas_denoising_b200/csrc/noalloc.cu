// noalloc.cu -- dg_denoise_step_noalloc: the denoising step for callers that
// cannot hand the library a workspace.
//
// Some callers cannot allocate device memory at the point where they run a
// step: a serving runtime that has carved up all of the GPU's memory for its
// own pools at start-up, or an embedding that is not allowed to call the CUDA
// allocator on its hot path (cudaMalloc and cudaFree can synchronise the
// device and stall unrelated work).  For them this entry point keeps its
// scratch -- the partial-record planes, the per-canvas tickets and the fault
// latch that dg_denoise_step otherwise takes from the caller's workspace --
// in a fixed array of this library's own device memory.
//
// The array is file-scope device memory of kNoAllocScratchBytes: every GPU
// that loads the library holds it until the process exits, whether or not
// this entry point is ever called.  Shapes whose scratch would not fit are
// rejected before anything is launched.
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "dg_internal.h"

namespace {

// 8 MiB: enough for B <= 4 canvases at d = 2816, V = 262,144 on a 148-SM
// B200 (a B = 1 step uses about 0.5 MiB), and for larger batches of smaller
// vocabularies.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the symbol's host-side name is not a device address).
dg_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DG_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[160];
      snprintf(msg, sizeof(msg), "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      dg::set_last_error_message(msg);
      return DG_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DG_OK;
}

}  // namespace

extern "C" dg_status dg_denoise_step_noalloc(const dg_shape* shape, const dg_params* params, const void* h,
                                             const void* E, const float* e_scale, const int32_t* step_idx,
                                             const uint8_t* has_prev, const uint8_t* active, int32_t* canvas,
                                             int32_t* prev_argmax, uint8_t* accept, float* entropy,
                                             int32_t* sampled, int32_t* argmax, int32_t* stop, void* stream) {
  // Every argument check runs before anything touches the shared array.
  dg_status st = dg::check_step_call(shape, params, h, E, e_scale, step_idx, has_prev, canvas, prev_argmax,
                                     accept, entropy, sampled, argmax, stop);
  if (st != DG_OK) return st;
  const size_t need = dg_workspace_size(shape);
  if (need == 0) {
    dg::set_last_error_message("dg_denoise_step_noalloc: the head kernel cannot run on this device");
    return DG_ERR_CUDA;
  }
  if (need > kNoAllocScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "dg_denoise_step_noalloc: this shape needs %zu bytes of scratch, the fixed array holds %zu",
             need, kNoAllocScratchBytes);
    dg::set_last_error_message(msg);
    return DG_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  if ((st = scratch_address(&ws)) != DG_OK) return st;
  // The array keeps the previous call's contents.  The per-canvas tickets
  // and the per-row key records must start at zero (everything after them
  // is written before it is read), so clear them on the caller's stream;
  // this does not allocate.  The fault latch in front of them is left as it
  // is: a fault of an earlier call stays there until dg_noalloc_status()
  // reads and clears it.
  const dg::WsLayout lay = dg::ws_layout(*shape, dg::head_max_pairs(shape->e_dtype == DG_E_FP8_E4M3));
  const cudaError_t e = cudaMemsetAsync(static_cast<unsigned char*>(ws) + lay.tickets_off, 0,
                                        lay.zero_prefix - lay.tickets_off, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    char msg[200];
    snprintf(msg, sizeof(msg), "dg_denoise_step_noalloc: clearing the scratch array: %s", cudaGetErrorString(e));
    dg::set_last_error_message(msg);
    return DG_ERR_CUDA;
  }
  return dg_denoise_step(shape, params, h, E, e_scale, step_idx, has_prev, active, canvas, prev_argmax, accept,
                         entropy, sampled, argmax, stop, ws, kNoAllocScratchBytes, stream);
}

extern "C" dg_status dg_noalloc_status(void* stream) {
  void* ws = nullptr;
  const dg_status st = scratch_address(&ws);
  if (st != DG_OK) return st;
  return dg::read_and_clear_latch(ws, static_cast<cudaStream_t>(stream));
}

extern "C" dg_status dg_noalloc_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
  void* ws = nullptr;
  const dg_status st = scratch_address(&ws);
  if (st != DG_OK) return st;
  if (dg::launch_wait_selftest(static_cast<uint32_t*>(ws), limit_ns, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return DG_ERR_CUDA;
  return dg_noalloc_status(stream);
}
