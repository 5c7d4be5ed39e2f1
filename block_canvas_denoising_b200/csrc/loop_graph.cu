// loop_graph.cu -- the adaptive loop run on the device.
//
// "DiffusionGemma" (Google AI for Developers), Recommended serving
// configuration: at most 48 denoising steps; stop early once the canvas-mean
// entropy is below 0.005 and two consecutive predictions agree.  The host
// loop (dg_denoise_loop) reads the stop flags back after every step.  Here
// the whole loop is one CUDA graph: a conditional (while) node whose body is
//   [the caller's hidden-state graph] -> head -> merge -> loop control,
// and the control kernel does what the host loop does between steps --
// commit and freeze the canvases that stopped (or reached the last step),
// advance k, prepare the next step's per-canvas data (step word, 1/tau in
// float64 exactly as the host computes it) and the list of canvases still
// running -- then sets the while condition.  Nothing returns to the host
// until every canvas is done.  The graph holds no per-call value, so it can
// be built once (dg_loop_graph_create) and run many times
// (dg_loop_graph_run): an init kernel writes the call's first step and
// previous-prediction flags into the loop state before each launch.
//
// Loop state (caller-owned device memory, dg_loop_state_bytes(B) bytes):
//   offset 0   int32 k, the step the body is about to run (the hidden-state
//              graph reads it), then int32 canvases still running, int32
//              steps run, int32 stop reason (0 running, 1 done, 2 fault),
//              int32 the call's first step
//   offset 256 CanvasParam[B], then uint8 canvas_of[B], uint8 has_prev[B],
//              uint8 active[B] (256-byte aligned each), int32 steps[B].
#include <string.h>

#include <mutex>
#include <new>

#include "dg_device.cuh"
#include "dg_internal.h"
#include "per_device.h"

namespace dg {

namespace {

struct LoopLayout {
  size_t cp, canvas_of, has_prev, active, steps, total;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

LoopLayout loop_layout(int B) {
  LoopLayout l;
  l.cp = 256;
  l.canvas_of = up256(l.cp + sizeof(CanvasParam) * static_cast<size_t>(B));
  l.has_prev = up256(l.canvas_of + static_cast<size_t>(B));
  l.active = up256(l.has_prev + static_cast<size_t>(B));
  l.steps = up256(l.active + static_cast<size_t>(B));
  l.total = up256(l.steps + sizeof(int32_t) * static_cast<size_t>(B));
  return l;
}

struct LoopHeader {
  int32_t k;
  int32_t n_active;
  int32_t iterations;
  int32_t reason;
  int32_t k_start;  // the call's first step (the graph itself holds no per-call value)
};

// Everything the init and control kernels need; passed by value.  The
// control kernel is captured into the graph, so it reads the per-call
// values (k_start, has_prev) from the loop state, which the init kernel
// writes before each launch.
struct LoopCtl {
  LoopHeader* hdr;
  CanvasParam* cp;
  uint8_t* canvas_of;
  uint8_t* has_prev;
  uint8_t* active;
  int32_t* steps;
  const int32_t* stop;
  const int32_t* sampled;
  int32_t* canvas;
  const uint32_t* err;
  int32_t B, L, N, k_start, block;
  double tau0, tau1;
  cudaGraphConditionalHandle handle;
  uint8_t has_prev_in[DG_MAX_B];
};

// 1 / tau_k in float64, rounded once to float32: the same operations, in
// the same order, as the host's schedule (explicitly rounded, no fused
// multiply-add).
DG_DEV float inv_tau_dev(const LoopCtl& c, int k) {
  double tau;
  if (c.N == 1) {
    tau = c.tau0;
  } else {
    const double span = __dmul_rn(__dsub_rn(c.tau0, c.tau1), static_cast<double>(k));
    tau = __dsub_rn(c.tau0, __ddiv_rn(span, static_cast<double>(c.N - 1)));
  }
  return __double2float_rn(__ddiv_rn(1.0, tau));
}

// Per-canvas data of step k for every canvas and the list of canvases still
// running (one CTA; every thread must call it).
DG_DEV void prepare_step(const LoopCtl& c, int k) {
  const int b = threadIdx.x;
  if (b < c.B) {
    CanvasParam p;
    p.k = static_cast<int32_t>(static_cast<uint32_t>(k) | (static_cast<uint32_t>(c.block) << 16));
    p.inv_tau = inv_tau_dev(c, k);
    p.has_prev = c.has_prev[b];
    p.active = c.active[b];
    p.pad[0] = p.pad[1] = 0;
    c.cp[b] = p;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = 0;
    for (int i = 0; i < c.B; ++i)
      if (c.active[i]) c.canvas_of[n++] = static_cast<uint8_t>(i);
    c.hdr->n_active = n;
  }
}

__global__ void __launch_bounds__(256) loop_init_kernel(const __grid_constant__ LoopCtl c) {
  const int b = threadIdx.x;
  if (b < c.B) {
    c.has_prev[b] = c.has_prev_in[b];
    c.active[b] = 1;
    c.steps[b] = 0;
  }
  if (b == 0) {
    c.hdr->k = c.k_start;
    c.hdr->k_start = c.k_start;
    c.hdr->iterations = 0;
    c.hdr->reason = 0;
  }
  __syncthreads();
  prepare_step(c, c.k_start);
}

__global__ void __launch_bounds__(256) loop_control_kernel(const __grid_constant__ LoopCtl c) {
  __shared__ uint8_t s_commit[DG_MAX_B];
  __shared__ int s_k, s_k0;
  if (threadIdx.x == 0) {
    s_k = c.hdr->k;
    s_k0 = c.hdr->k_start;
  }
  __syncthreads();
  const int k = s_k;
  const int b = threadIdx.x;
  if (b < c.B) {
    uint8_t commit = 0;
    if (c.active[b]) {
      c.has_prev[b] = 1;
      if (c.stop[b] != 0 || k == c.N - 1) {
        // stop (or the last step): the canvas takes this step's sampled
        // tokens and is frozen
        commit = 1;
        c.active[b] = 0;
        c.steps[b] = k - s_k0 + 1;
      }
    }
    s_commit[b] = commit;
  }
  __syncthreads();
  for (int i = 0; i < c.B; ++i) {
    if (!s_commit[i]) continue;
    const size_t base = static_cast<size_t>(i) * c.L;
    for (int s = threadIdx.x; s < c.L; s += blockDim.x) c.canvas[base + s] = c.sampled[base + s];
  }
  __syncthreads();
  const int kn = k + 1;
  if (threadIdx.x == 0) {
    c.hdr->k = kn;
    c.hdr->iterations += 1;
  }
  prepare_step(c, kn < c.N ? kn : c.N - 1);
  if (threadIdx.x == 0) {
    const bool fault = __ldcg(c.err) != 0u;
    const bool more = c.hdr->n_active > 0 && kn < c.N && !fault;
    c.hdr->reason = more ? 0 : (fault ? 2 : 1);
    cudaGraphSetConditional(c.handle, more ? 1u : 0u);
  }
}

// A private non-blocking stream per device to capture the loop body on
// (the caller's stream may be the legacy default stream, which cannot be
// captured).
bool capture_stream(cudaStream_t* out) {
  static PerDevice<cudaStream_t> streams;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  return streams.get(dev, [](cudaStream_t* s) { return cudaStreamCreateWithFlags(s, cudaStreamNonBlocking) == cudaSuccess; },
                     out);
}

std::mutex g_capture_mu;  // one capture on a device's private stream at a time

}  // namespace

}  // namespace dg

using namespace dg;

extern "C" size_t dg_loop_state_bytes(int32_t B) {
  if (B < 1 || B > DG_MAX_B) return 0;
  return loop_layout(B).total;
}

// The built loop behind a dg_loop_graph handle.
struct dg_loop_graph_s {
  LoopCtl c;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  int device = -1;
  void* workspace = nullptr;
  size_t ws_bytes = 0;
};

extern "C" dg_status dg_loop_graph_create(const dg_shape* shape, const dg_params* params, const void* E,
                                          const float* e_scale, void* hidden_graph, void* h_buf, int32_t* canvas,
                                          int32_t* prev_argmax, uint8_t* accept, float* entropy, int32_t* sampled,
                                          int32_t* argmax, int32_t* stop, void* loop_state, size_t state_bytes,
                                          void* workspace, size_t ws_bytes, dg_loop_graph* out) {
  if (out == nullptr) return DG_ERR_INVALID_ARG;
  *out = nullptr;
  dg_status st = check_shape_and_params(shape, params);
  if (st != DG_OK) return st;
  if (loop_state == nullptr || h_buf == nullptr || canvas == nullptr || workspace == nullptr)
    return DG_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(loop_state) & 255u) != 0) return DG_ERR_INVALID_ARG;
  const int B = shape->B;
  const LoopLayout lay = loop_layout(B);
  if (state_bytes < lay.total) return DG_ERR_WORKSPACE;
  // the head's per-device launch set-up happens here, outside the capture
  const size_t ws_need = dg_workspace_size(shape);
  if (ws_need == 0) return DG_ERR_NO_DEVICE;
  if (ws_bytes < ws_need) return DG_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_NO_DEVICE;
  uint8_t* base = static_cast<uint8_t*>(loop_state);

  LoopCtl c;
  memset(&c, 0, sizeof(c));
  c.hdr = reinterpret_cast<LoopHeader*>(base);
  c.cp = reinterpret_cast<CanvasParam*>(base + lay.cp);
  c.canvas_of = base + lay.canvas_of;
  c.has_prev = base + lay.has_prev;
  c.active = base + lay.active;
  c.steps = reinterpret_cast<int32_t*>(base + lay.steps);
  c.stop = stop;
  c.sampled = sampled;
  c.canvas = canvas;
  c.err = static_cast<const uint32_t*>(workspace);  // the fault latch heads the workspace
  c.B = B;
  c.L = shape->L;
  c.N = params->max_steps;
  c.block = params->block;
  c.tau0 = params->tau0;
  c.tau1 = params->tau1;
  LoopDevState devst{c.cp, c.canvas_of, &c.hdr->n_active};

  // ---- the graph: while (condition) { hidden graph; step; control }
  cudaStream_t cap;
  if (!capture_stream(&cap)) return DG_ERR_CUDA;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  cudaGraphConditionalHandle handle;
  {
    std::lock_guard<std::mutex> lock(g_capture_mu);
    if (cudaGraphCreate(&graph, 0) != cudaSuccess) return DG_ERR_CUDA;
    if (cudaGraphConditionalHandleCreate(&handle, graph, 1, cudaGraphCondAssignDefault) != cudaSuccess) {
      cudaGraphDestroy(graph);
      set_last_error_message("cudaGraphConditionalHandleCreate failed");
      return DG_ERR_CUDA;
    }
    c.handle = handle;
    cudaGraphNodeParams np = {};
    np.type = cudaGraphNodeTypeConditional;
    np.conditional.handle = handle;
    np.conditional.type = cudaGraphCondTypeWhile;
    np.conditional.size = 1;
    cudaGraphNode_t cond;
    if (cudaGraphAddNode(&cond, graph, nullptr, 0, &np) != cudaSuccess) {
      cudaGraphDestroy(graph);
      set_last_error_message("adding the conditional node failed");
      return DG_ERR_CUDA;
    }
    cudaGraph_t body = np.conditional.phGraph_out[0];
    cudaGraphNode_t child = nullptr;
    if (hidden_graph != nullptr &&
        cudaGraphAddChildGraphNode(&child, body, nullptr, 0, static_cast<cudaGraph_t>(hidden_graph)) !=
            cudaSuccess) {
      cudaGraphDestroy(graph);
      set_last_error_message("the hidden-state graph cannot be embedded in the loop body");
      return DG_ERR_INVALID_ARG;
    }
    if (cudaStreamBeginCaptureToGraph(cap, body, child ? &child : nullptr, nullptr, child ? 1 : 0,
                                      cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
      cudaGraphDestroy(graph);
      set_last_error_message("capture of the loop body failed to start");
      return DG_ERR_CUDA;
    }
    // the step's kernels read the per-canvas step words from the loop
    // state; the step index passed here only satisfies the range check
    st = enqueue_loop_step(shape, params, h_buf, E, e_scale, 0, canvas, prev_argmax, accept, entropy, sampled,
                           argmax, stop, workspace, ws_bytes, &devst, cap);
    if (st == DG_OK) {
      loop_control_kernel<<<1, 256, 0, cap>>>(c);
      if (cudaGetLastError() != cudaSuccess) st = DG_ERR_CUDA;
    }
    cudaGraph_t captured = nullptr;
    const cudaError_t ec = cudaStreamEndCapture(cap, &captured);
    if (st == DG_OK && ec != cudaSuccess) {
      set_last_error_message("capture of the loop body failed");
      st = DG_ERR_CUDA;
    }
    if (st == DG_OK && cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) {
      set_last_error_message("instantiating the loop graph failed");
      st = DG_ERR_CUDA;
    }
  }
  if (st != DG_OK) {
    if (exec != nullptr) cudaGraphExecDestroy(exec);
    cudaGraphDestroy(graph);
    return st;
  }
  dg_loop_graph g = new (std::nothrow) dg_loop_graph_s;
  if (g == nullptr) {
    cudaGraphExecDestroy(exec);
    cudaGraphDestroy(graph);
    return DG_ERR_CUDA;
  }
  g->c = c;
  g->graph = graph;
  g->exec = exec;
  g->device = dev;
  g->workspace = workspace;
  g->ws_bytes = ws_bytes;
  *out = g;
  return DG_OK;
}

extern "C" dg_status dg_loop_graph_run(dg_loop_graph g, int32_t k_start, uint8_t* has_prev, int32_t* steps_taken,
                                       void* stream) {
  if (g == nullptr || has_prev == nullptr || steps_taken == nullptr) return DG_ERR_INVALID_ARG;
  if (k_start < 0 || k_start >= g->c.N) return DG_ERR_RANGE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != g->device) {
    set_last_error_message("dg_loop_graph_run: the graph was built on another device");
    return DG_ERR_INVALID_ARG;
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  LoopCtl c = g->c;
  c.k_start = k_start;
  for (int b = 0; b < c.B; ++b) c.has_prev_in[b] = has_prev[b] ? 1 : 0;
  loop_init_kernel<<<1, 256, 0, cs>>>(c);
  if (cudaGetLastError() != cudaSuccess || cudaGraphLaunch(g->exec, cs) != cudaSuccess) {
    set_last_error_message("launching the loop graph failed");
    return DG_ERR_CUDA;
  }
  int32_t steps_h[DG_MAX_B];
  uint8_t hp_h[DG_MAX_B];
  if (cudaMemcpyAsync(steps_h, c.steps, sizeof(int32_t) * c.B, cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
      cudaMemcpyAsync(hp_h, c.has_prev, c.B, cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
      cudaStreamSynchronize(cs) != cudaSuccess) {
    set_last_error_message("reading the loop's results failed");
    return DG_ERR_CUDA;
  }
  for (int b = 0; b < c.B; ++b) {
    steps_taken[b] = steps_h[b];
    has_prev[b] = hp_h[b];
  }
  // a bounded wait that ran out (or a non-finite FP8 hidden state) stopped
  // the loop early: report it
  return dg_device_status(g->workspace, g->ws_bytes, stream);
}

extern "C" void dg_loop_graph_destroy(dg_loop_graph g) {
  if (g == nullptr) return;
  int cur = -1;
  const bool switch_dev = cudaGetDevice(&cur) == cudaSuccess && cur != g->device;
  if (switch_dev) cudaSetDevice(g->device);
  if (g->exec != nullptr) cudaGraphExecDestroy(g->exec);
  if (g->graph != nullptr) cudaGraphDestroy(g->graph);
  if (switch_dev) cudaSetDevice(cur);
  delete g;
}

extern "C" dg_status dg_denoise_loop_graph(const dg_shape* shape, const dg_params* params, const void* E,
                                           const float* e_scale, void* hidden_graph, int32_t k_start,
                                           void* h_buf, int32_t* canvas, int32_t* prev_argmax, uint8_t* has_prev,
                                           int32_t* steps_taken, uint8_t* accept, float* entropy,
                                           int32_t* sampled, int32_t* argmax, int32_t* stop, void* loop_state,
                                           size_t state_bytes, void* workspace, size_t ws_bytes, void* stream) {
  dg_status st = check_shape_and_params(shape, params);
  if (st != DG_OK) return st;
  if (has_prev == nullptr || steps_taken == nullptr) return DG_ERR_INVALID_ARG;
  if (k_start < 0 || k_start >= params->max_steps) return DG_ERR_RANGE;
  dg_loop_graph g = nullptr;
  st = dg_loop_graph_create(shape, params, E, e_scale, hidden_graph, h_buf, canvas, prev_argmax, accept, entropy,
                            sampled, argmax, stop, loop_state, state_bytes, workspace, ws_bytes, &g);
  if (st != DG_OK) return st;
  st = dg_loop_graph_run(g, k_start, has_prev, steps_taken, stream);
  dg_loop_graph_destroy(g);
  return st;
}
