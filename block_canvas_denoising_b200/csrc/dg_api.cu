// dg_api.cu -- host side of the C ABI declared in include/dg.h: argument
// checks, the temperature schedule, TMA descriptors, kernel launches and the
// adaptive loop.
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "dg_device.cuh"
#include "dg_internal.h"

namespace dg {

namespace {

constexpr size_t kAlign = 256;

thread_local char t_last_error[256] = "";

// Record a failed CUDA call's message for dg_last_error_message().
bool cuda_ok(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return true;
  snprintf(t_last_error, sizeof(t_last_error), "%s: %s (%d)", what, cudaGetErrorString(e),
           static_cast<int>(e));
  return false;
}

thread_local cudaEvent_t t_head_ev_start = nullptr;
thread_local cudaEvent_t t_head_ev_stop = nullptr;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Current device's SM count, or -1 when it is not an sm_100 part.
int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (major != 10) return -1;
  return sms;
}

dg_status check_shape(const dg_shape* s) {
  if (s == nullptr) return DG_ERR_INVALID_ARG;
  if (s->B < 1 || s->B > DG_MAX_B || s->L != 256 || s->d < kBlockK || s->d % kBlockK != 0 ||
      s->V < kBlockN || s->V % kBlockN != 0)
    return DG_ERR_UNSUPPORTED_SHAPE;
  if (s->e_dtype != DG_E_BF16 && s->e_dtype != DG_E_FP8_E4M3) return DG_ERR_UNSUPPORTED_SHAPE;
  return DG_OK;
}

bool finite_pos(double x) { return x > 0.0 && x < 1e300; }

dg_status check_params(const dg_params* p) {
  if (p == nullptr) return DG_ERR_INVALID_ARG;
  if (p->max_steps < 1 || !finite_pos(p->tau0) || !finite_pos(p->tau1)) return DG_ERR_INVALID_ARG;
  if (!(p->entropy_bound >= 0.0 && p->entropy_bound < 1e300)) return DG_ERR_INVALID_ARG;
  if (!(p->stop_entropy >= 0.0 && p->stop_entropy < 1e300)) return DG_ERR_INVALID_ARG;
  if (p->selection_rule < DG_SELECT_CUMSUM || p->selection_rule > DG_SELECT_TOPK) return DG_ERR_INVALID_ARG;
  if (p->selection_rule == DG_SELECT_TOPK && (p->top_k < 1 || p->top_k > 256)) return DG_ERR_INVALID_ARG;
  // the Philox counter's step word is k | block << 16
  if (p->max_steps > 65536 || p->block < 0 || p->block > 65535) return DG_ERR_INVALID_ARG;
  return DG_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Temperature of step k ([Docs] "DiffusionGemma", Recommended serving
// configuration, temperature schedule: linear from tau0 to tau1 over the N
// steps), in float64, and its float32 reciprocal.
float inv_tau_of(const dg_params& p, int k) {
  double tau;
  if (p.max_steps == 1) {
    tau = p.tau0;
  } else {
    const double span = (p.tau0 - p.tau1) * static_cast<double>(k);
    tau = p.tau0 - span / static_cast<double>(p.max_steps - 1);
  }
  return static_cast<float>(1.0 / tau);
}

// 2-D tensor map over a row-major [rows, inner] matrix with elements of
// `dtype` (`esize` bytes); box = box_inner x box_rows elements.
bool encode_2d(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t esize, CUtensorMapSwizzle swizzle,
               const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * esize};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

enum class StepMode { kFull, kHeadOnly, kMergeOnly };

struct StepArgs {
  const dg_shape* shape;
  const dg_params* params;
  const void* h;
  const void* E;
  const float* e_scale;
  const int32_t* step_idx;
  const uint8_t* has_prev;
  const uint8_t* active;
  int32_t* canvas;
  int32_t* prev_argmax;
  uint8_t* accept;
  float* entropy;
  int32_t* sampled;
  int32_t* argmax;
  int32_t* stop;
  float* logits;
  void* workspace;
  size_t ws_bytes;
  cudaStream_t stream;
  StepMode mode = StepMode::kFull;
  int32_t v_off = 0;              // head: vocabulary index of E's first row
  float* part_out = nullptr;      // head only: the records [7][R][P] go here
  const float* part_in = nullptr; // merge only: S shards' records [S][7][R][P]
  int32_t S = 1, P = 0;           // merge only
  const LoopDevState* loop = nullptr;  // device-side loop: per-canvas data from device memory
  uint16_t* ptilde = nullptr;          // self-conditioning: block-scaled probabilities [R, V]
  float* pref = nullptr;               // and their block references [R, V / 64]
  float2* rowstat = nullptr;           // and the merged (m2, 1 / S) per row
};

// Every check of a step's arguments except those of the workspace: shape,
// parameters, pointers and their alignment, step indices, the device.
dg_status check_step_inputs(const StepArgs& a) {
  dg_status st = check_shape(a.shape);
  if (st != DG_OK) return st;
  if ((st = check_params(a.params)) != DG_OK) return st;
  const dg_shape& s = *a.shape;
  const dg_params& pr = *a.params;
  const bool head = a.mode != StepMode::kMergeOnly;
  const bool merge = a.mode != StepMode::kHeadOnly;
  if (!a.step_idx) return DG_ERR_INVALID_ARG;
  if (head && (!a.h || !a.E || !aligned16(a.h) || !aligned16(a.E))) return DG_ERR_INVALID_ARG;
  if (merge && (!a.has_prev || !a.canvas || !a.prev_argmax || !a.accept || !a.entropy || !a.sampled ||
                !a.argmax || !a.stop))
    return DG_ERR_INVALID_ARG;
  const bool fp8 = s.e_dtype == DG_E_FP8_E4M3;
  // the per-row scale belongs to the FP8 embedder only
  if (head && (fp8 ? (a.e_scale == nullptr || !aligned16(a.e_scale)) : a.e_scale != nullptr))
    return DG_ERR_INVALID_ARG;
  if (a.logits != nullptr && !aligned16(a.logits)) return DG_ERR_INVALID_ARG;
  if (a.mode == StepMode::kHeadOnly && (a.part_out == nullptr || !aligned16(a.part_out) || a.v_off < 0 ||
                                        a.v_off % kBlockN != 0))
    return DG_ERR_INVALID_ARG;
  if (a.mode == StepMode::kMergeOnly && (a.part_in == nullptr || a.S < 1 || a.P < 1)) return DG_ERR_INVALID_ARG;
  for (int b = 0; b < s.B; ++b)
    if (a.step_idx[b] < 0 || a.step_idx[b] >= pr.max_steps) return DG_ERR_RANGE;
  if (device_sms() <= 0) return DG_ERR_NO_DEVICE;
  return DG_OK;
}

dg_status run_step(const StepArgs& a) {
  dg_status st = check_step_inputs(a);
  if (st != DG_OK) return st;
  if (!a.workspace || !aligned16(a.workspace)) return DG_ERR_INVALID_ARG;
  const dg_shape& s = *a.shape;
  const dg_params& pr = *a.params;
  const bool head = a.mode != StepMode::kMergeOnly;
  const bool merge = a.mode != StepMode::kHeadOnly;
  const bool fp8 = s.e_dtype == DG_E_FP8_E4M3;
  const int pairs = head_max_pairs(fp8);
  if (pairs <= 0) {
    snprintf(t_last_error, sizeof(t_last_error), "no CTA pair of the head kernel fits on this device");
    return DG_ERR_CUDA;
  }
  const WsLayout ws = ws_layout(s, pairs);
  if (a.ws_bytes < (head ? ws.total : ws.zero_prefix)) return DG_ERR_WORKSPACE;

  const int R = s.B * s.L;
  uint8_t* wsb = static_cast<uint8_t*>(a.workspace);
  uint32_t* row_rec = reinterpret_cast<uint32_t*>(wsb + ws.rec_off);

  CanvasParam cps[DG_MAX_B];
  memset(cps, 0, sizeof(cps));
  uint8_t upd[DG_MAX_B] = {};  // the canvases this call updates, in order
  int n_upd = 0;
  for (int b = 0; b < s.B; ++b) {
    // the kernels use k only as the Philox counter's step word
    cps[b].k = static_cast<int32_t>(static_cast<uint32_t>(a.step_idx[b]) | (static_cast<uint32_t>(pr.block) << 16));
    cps[b].inv_tau = inv_tau_of(pr, a.step_idx[b]);
    cps[b].has_prev = (merge && a.has_prev[b]) ? 1 : 0;
    cps[b].active = (a.active == nullptr || a.active[b]) ? 1 : 0;
    if (cps[b].active) upd[n_upd++] = static_cast<uint8_t>(b);
  }
  if (n_upd == 0) return DG_OK;  // every canvas frozen: nothing to do
  const uint32_t seed_lo = static_cast<uint32_t>(pr.seed & 0xFFFFFFFFull);
  const uint32_t seed_hi = static_cast<uint32_t>(pr.seed >> 32);
  float* part = reinterpret_cast<float*>(wsb + ws.part_off);
  int q_used = ws.P;  // records per row the head writes

  if (head) {
    // TMA boxes: one CTA's share of a stage, 128 rows x 128 bytes of K (the
    // 128-byte swizzle span); the kernel's expect-tx byte counts and shared-
    // memory slots are sized from the same constants.  K beyond d reads as 0.
    static_assert(kTileBytes == kBlockK * 2 * kBlockM && kTileBytes == kBlockKFp8 * 1 * kHalfN,
                  "TMA box / stage tile mismatch");
    CUtensorMap tmA, tmA2, tmB;
    if (fp8) {
      // h -> h1 + h2 (E4M3) with a power-of-two row scale, in the workspace
      uint8_t* h1 = wsb + ws.h1_off;
      uint8_t* h2 = wsb + ws.h2_off;
      if (!cuda_ok(launch_hidden_split(a.h, h1, h2, reinterpret_cast<float*>(wsb + ws.rinv_off), R, s.d,
                                       reinterpret_cast<uint32_t*>(wsb + ws.err_off), a.stream),
                   "hidden-state split launch"))
        return DG_ERR_CUDA;
      const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
      const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
      if (!encode_2d(&tmA, U8, 1, SW, h1, s.d, R, kBlockKFp8, kBlockM) ||
          !encode_2d(&tmA2, U8, 1, SW, h2, s.d, R, kBlockKFp8, kBlockM) ||
          !encode_2d(&tmB, U8, 1, SW, a.E, s.d, s.V, kBlockKFp8, kHalfN))
        return DG_ERR_CUDA;
    } else {
      const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
      const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
      if (!encode_2d(&tmA, BF, 2, SW, a.h, s.d, R, kBlockK, kBlockM) ||
          !encode_2d(&tmB, BF, 2, SW, a.E, s.d, s.V, kBlockK, kHalfN))
        return DG_ERR_CUDA;
      tmA2 = tmA;  // unused by the bf16 head
    }
    if (a.mode == StepMode::kHeadOnly) {
      // the per-row key records must start empty; without the merge of this
      // call nothing else clears them
      if (!cuda_ok(cudaMemsetAsync(row_rec, 0, sizeof(uint32_t) * static_cast<size_t>(R), a.stream),
                   "record clear"))
        return DG_ERR_CUDA;
      part = a.part_out;
    }

    HeadParams hp;
    memset(&hp, 0, sizeof(hp));
    hp.R = R;
    hp.d = s.d;
    hp.V = s.V;
    hp.B = s.B;
    hp.v_off = a.v_off;
    // only the updated canvases' row tiles are split into work units; at
    // most ws.P records per row (the workspace's planes)
    hp.split = head_split(n_upd * s.L, s.V, s.d, pairs, fp8 ? kBlockKFp8 : kBlockK, ws.P);
    memcpy(hp.mtile, upd, sizeof(upd));
    q_used = hp.split.Q;
    hp.seed_lo = seed_lo;
    hp.seed_hi = seed_hi;
    // Philox4x32-10 round keys: key + i * (0x9E3779B9, 0xBB67AE85), mod 2^32
    for (int i = 0; i < 10; ++i) {
      hp.rk0[i] = seed_lo + static_cast<uint32_t>(i) * 0x9E3779B9u;
      hp.rk1[i] = seed_hi + static_cast<uint32_t>(i) * 0xBB67AE85u;
    }
    hp.e_scale = a.e_scale;
    hp.row_inv = fp8 ? reinterpret_cast<const float*>(wsb + ws.rinv_off) : nullptr;
    hp.part = part;
    hp.err = reinterpret_cast<uint32_t*>(wsb + ws.err_off);
    hp.logits_out = a.logits;
    hp.row_rec = row_rec;
    hp.wait_ns = kDefaultWaitNs;
    memcpy(hp.cp, cps, sizeof(cps));

    hp.ptilde = a.ptilde;
    hp.pref = a.pref;
    if (a.loop != nullptr) {
      hp.cp_dev = a.loop->cp;
      hp.mtile_dev = a.loop->canvas_of;
      hp.mt_dev = a.loop->n_active;
    }
    const bool events = t_head_ev_start != nullptr && a.loop == nullptr;
    if (events && cudaEventRecord(t_head_ev_start, a.stream) != cudaSuccess) return DG_ERR_CUDA;
    if (!cuda_ok(launch_head(fp8, tmA, tmA2, tmB, hp, a.stream, a.loop == nullptr), "head kernel launch"))
      return DG_ERR_CUDA;
    if (events && cudaEventRecord(t_head_ev_stop, a.stream) != cudaSuccess) return DG_ERR_CUDA;
  }
  if (!merge) return DG_OK;

  MergeParams mp;
  memset(&mp, 0, sizeof(mp));
  mp.R = R;
  mp.B = n_upd;
  mp.V = s.V;
  mp.P = a.mode == StepMode::kMergeOnly ? a.P : q_used;
  mp.S = a.mode == StepMode::kMergeOnly ? a.S : 1;
  mp.part = a.mode == StepMode::kMergeOnly ? a.part_in : part;
  mp.entropy = a.entropy;
  mp.sampled = a.sampled;
  mp.argmax = a.argmax;
  mp.canvas = a.canvas;
  mp.prev_argmax = a.prev_argmax;
  mp.accept = a.accept;
  mp.stop = a.stop;
  mp.tickets = reinterpret_cast<uint32_t*>(wsb + ws.tickets_off);
  mp.row_rec = row_rec;
  mp.seed_lo = seed_lo;
  mp.seed_hi = seed_hi;
  mp.entropy_bound = pr.entropy_bound;
  mp.selection_rule = pr.selection_rule;
  mp.top_k = pr.top_k;
  mp.stop_entropy = pr.stop_entropy;
  memcpy(mp.cp, cps, sizeof(cps));
  memcpy(mp.canvas_of, upd, sizeof(upd));
  mp.rowstat = a.rowstat;
  if (a.loop != nullptr) {
    mp.cp_dev = a.loop->cp;
    mp.canvas_of_dev = a.loop->canvas_of;
    mp.n_dev = a.loop->n_active;
  }
  if (!cuda_ok(launch_merge(mp, a.stream, a.loop == nullptr), "merge kernel launch")) return DG_ERR_CUDA;
  return DG_OK;
}

}  // namespace

dg_status enqueue_loop_step(const dg_shape* shape, const dg_params* params, const void* h, const void* E,
                            const float* e_scale, int32_t k_any, int32_t* canvas, int32_t* prev_argmax,
                            uint8_t* accept, float* entropy, int32_t* sampled, int32_t* argmax, int32_t* stop,
                            void* workspace, size_t ws_bytes, const LoopDevState* loop, cudaStream_t stream) {
  int32_t ks[DG_MAX_B];
  uint8_t hp[DG_MAX_B];
  for (int b = 0; b < DG_MAX_B; ++b) {
    ks[b] = k_any;
    hp[b] = 0;
  }
  StepArgs a{shape,  params,  h,       E,      e_scale, ks,      hp,        nullptr,  canvas, prev_argmax,
             accept, entropy, sampled, argmax, stop,    nullptr, workspace, ws_bytes, stream};
  a.loop = loop;
  return run_step(a);
}

// Self-conditioning workspace: the step's workspace, then P [R, V] bf16,
// the block references [R, V / 64], the row statistics [R] float2 and the
// split-K partial sums [Sk, R, d] float32.
struct SelfcondLayout {
  size_t p_off, pref_off, stat_off, part_off, total;
};

SelfcondLayout selfcond_layout(const dg_shape& s, size_t step_ws, int gemm_pairs) {
  SelfcondLayout l;
  const size_t R = static_cast<size_t>(s.B) * s.L;
  l.p_off = align_up(step_ws);
  l.pref_off = align_up(l.p_off + R * s.V * 2);
  l.stat_off = align_up(l.pref_off + R * (s.V / 64) * 4);
  l.part_off = align_up(l.stat_off + R * 8);
  const int sk = selfcond_slices(static_cast<int>(R), s.d, s.V, gemm_pairs);
  l.total = align_up(l.part_off + static_cast<size_t>(sk) * R * s.d * 4);
  return l;
}

dg_status run_selfcond_step(const dg_shape* shape, const dg_params* params, const void* h, const void* E,
                            const float* e_scale, const void* E_t, const int32_t* step_idx,
                            const uint8_t* has_prev, int32_t* canvas, int32_t* prev_argmax, uint8_t* accept,
                            float* entropy, int32_t* sampled, int32_t* argmax, int32_t* stop, float* signal,
                            void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (E_t == nullptr || signal == nullptr || !aligned16(E_t) || !aligned16(signal)) return DG_ERR_INVALID_ARG;
  dg_status st = check_step_call(shape, params, h, E, e_scale, step_idx, has_prev, canvas, prev_argmax, accept,
                                 entropy, sampled, argmax, stop);
  if (st != DG_OK) return st;
  const size_t step_ws = dg_workspace_size(shape);
  const int gp = selfcond_gemm_pairs();
  if (step_ws == 0 || gp < 1) return DG_ERR_CUDA;
  const SelfcondLayout lay = selfcond_layout(*shape, step_ws, gp);
  if (workspace == nullptr || ws_bytes < lay.total) return DG_ERR_WORKSPACE;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  StepArgs a{shape,  params,  h,       E,      e_scale, step_idx, has_prev,  nullptr,  canvas, prev_argmax,
             accept, entropy, sampled, argmax, stop,    nullptr,  workspace, step_ws, stream};
  a.ptilde = reinterpret_cast<uint16_t*>(wsb + lay.p_off);
  a.pref = reinterpret_cast<float*>(wsb + lay.pref_off);
  a.rowstat = reinterpret_cast<float2*>(wsb + lay.stat_off);
  if ((st = run_step(a)) != DG_OK) return st;
  const int R = shape->B * shape->L;
  if (!cuda_ok(launch_selfcond(a.ptilde, static_cast<const uint16_t*>(E_t), a.pref, a.rowstat,
                               shape->e_dtype == DG_E_FP8_E4M3 ? e_scale : nullptr,
                               reinterpret_cast<float*>(wsb + lay.part_off), signal, R, shape->d, shape->V,
                               reinterpret_cast<uint32_t*>(wsb), stream),
               "self-conditioning launch"))
    return DG_ERR_CUDA;
  return DG_OK;
}

dg_status check_shape_and_params(const dg_shape* shape, const dg_params* params) {
  const dg_status st = check_shape(shape);
  return st != DG_OK ? st : check_params(params);
}

dg_status check_step_call(const dg_shape* shape, const dg_params* params, const void* h, const void* E,
                          const float* e_scale, const int32_t* step_idx, const uint8_t* has_prev,
                          int32_t* canvas, int32_t* prev_argmax, uint8_t* accept, float* entropy,
                          int32_t* sampled, int32_t* argmax, int32_t* stop) {
  StepArgs a{shape,   params,  h,      E,    e_scale, step_idx, has_prev, nullptr,  canvas, prev_argmax,
             accept,  entropy, sampled, argmax, stop,   nullptr,  nullptr,  0, nullptr};
  return check_step_inputs(a);
}

dg_status read_and_clear_latch(void* latch, cudaStream_t st) {
  uint32_t err = 0;
  if (!cuda_ok(cudaMemcpyAsync(&err, latch, sizeof(err), cudaMemcpyDeviceToHost, st), "fault latch read"))
    return DG_ERR_CUDA;
  if (!cuda_ok(cudaStreamSynchronize(st), "stream synchronise")) return DG_ERR_CUDA;
  if (err != 0) {
    if (!cuda_ok(cudaMemsetAsync(latch, 0, sizeof(err), st), "fault latch clear")) return DG_ERR_CUDA;
    if (!cuda_ok(cudaStreamSynchronize(st), "stream synchronise")) return DG_ERR_CUDA;
    if (err & ~kErrValueMask) {
      set_last_error_message("a device-side bounded wait ran out");
      return DG_ERR_TIMEOUT;
    }
    set_last_error_message((err & kErrHiddenRange) ? "FP8 head: a hidden-state value is not finite"
                                                   : "self-conditioning: logits span more than the "
                                                     "probability blocks' range");
    return DG_ERR_VALUE;
  }
  return DG_OK;
}

void set_last_error_message(const char* msg) {
  snprintf(t_last_error, sizeof(t_last_error), "%s", msg);
}

WsLayout ws_layout(const dg_shape& s, int max_pairs) {
  WsLayout w;
  const int R = s.B * s.L;
  const bool fp8 = s.e_dtype == DG_E_FP8_E4M3;
  const HeadSplit sp = head_split(R, s.V, s.d, max_pairs, fp8 ? kBlockKFp8 : kBlockK);
  w.P = sp.Q;
  w.err_off = 0;
  w.tickets_off = kAlign;
  w.rec_off = align_up(w.tickets_off + sizeof(uint32_t) * static_cast<size_t>(s.B));
  w.part_off = align_up(w.rec_off + sizeof(uint32_t) * static_cast<size_t>(R));
  w.zero_prefix = w.part_off;
  const size_t hsz = fp8 ? static_cast<size_t>(R) * s.d : 0;  // one E4M3 term of h
  w.h1_off = align_up(w.part_off + sizeof(float) * kPartialFields * static_cast<size_t>(w.P) * R);
  w.h2_off = align_up(w.h1_off + hsz);
  w.rinv_off = align_up(w.h2_off + hsz);
  w.total = align_up(w.rinv_off + (fp8 ? sizeof(float) * static_cast<size_t>(R) : 0));
  return w;
}

}  // namespace dg

using namespace dg;

extern "C" {

dg_params dg_default_params(void) {
  dg_params p;
  p.tau0 = 0.8;
  p.tau1 = 0.4;
  p.max_steps = 48;
  p.entropy_bound = 0.1;
  p.stop_entropy = 0.005;
  p.seed = 1234;
  p.selection_rule = DG_SELECT_CUMSUM;
  p.top_k = 1;
  p.block = 0;
  return p;
}

const char* dg_error_string(dg_status s) {
  switch (s) {
    case DG_OK: return "ok";
    case DG_ERR_INVALID_ARG: return "invalid argument";
    case DG_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case DG_ERR_WORKSPACE: return "workspace too small";
    case DG_ERR_RANGE: return "step index out of range";
    case DG_ERR_CUDA: return "CUDA runtime error";
    case DG_ERR_TIMEOUT: return "device-side wait timed out";
    case DG_ERR_CALLBACK: return "hidden-state callback failed";
    case DG_ERR_NO_DEVICE: return "no sm_100 device";
    case DG_ERR_VALUE: return "input value outside the supported range";
  }
  return "unknown status";
}

size_t dg_workspace_size(const dg_shape* shape) {
  if (check_shape(shape) != DG_OK) return 0;
  if (device_sms() <= 0) return 0;
  const int pairs = head_max_pairs(shape->e_dtype == DG_E_FP8_E4M3);
  if (pairs <= 0) return 0;
  return ws_layout(*shape, pairs).total;
}

dg_status dg_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  if (workspace == nullptr) return DG_ERR_INVALID_ARG;
  if (cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DG_ERR_CUDA;
  return DG_OK;
}

dg_status dg_denoise_step(const dg_shape* shape, const dg_params* params, const void* h, const void* E,
                          const float* e_scale, const int32_t* step_idx, const uint8_t* has_prev,
                          const uint8_t* active, int32_t* canvas, int32_t* prev_argmax, uint8_t* accept,
                          float* entropy, int32_t* sampled, int32_t* argmax, int32_t* stop,
                          void* workspace, size_t ws_bytes, void* stream) {
  StepArgs a{shape,   params,  h,      E,    e_scale, step_idx, has_prev, active,   canvas, prev_argmax,
             accept,  entropy, sampled, argmax, stop,   nullptr,  workspace, ws_bytes,
             static_cast<cudaStream_t>(stream)};
  return run_step(a);
}

dg_status dg_debug_logits(const dg_shape* shape, const dg_params* params, const void* h, const void* E,
                          const float* e_scale, const int32_t* step_idx, const uint8_t* has_prev,
                          const uint8_t* active, int32_t* canvas, int32_t* prev_argmax, uint8_t* accept,
                          float* entropy, int32_t* sampled, int32_t* argmax, int32_t* stop,
                          float* logits, void* workspace, size_t ws_bytes, void* stream) {
  if (logits == nullptr) return DG_ERR_INVALID_ARG;
  StepArgs a{shape,   params,  h,      E,    e_scale, step_idx, has_prev, active,   canvas, prev_argmax,
             accept,  entropy, sampled, argmax, stop,   logits,   workspace, ws_bytes,
             static_cast<cudaStream_t>(stream)};
  return run_step(a);
}

dg_status dg_device_status(void* workspace, size_t ws_bytes, void* stream) {
  if (workspace == nullptr || ws_bytes < kAlign) return DG_ERR_INVALID_ARG;
  return read_and_clear_latch(workspace, static_cast<cudaStream_t>(stream));
}

dg_status dg_denoise_loop(const dg_shape* shape, const dg_params* params, const void* E,
                          const float* e_scale, dg_hidden_fn hidden_fn, void* user, int32_t k_start,
                          void* h_buf, int32_t* canvas, int32_t* prev_argmax, uint8_t* has_prev,
                          int32_t* steps_taken, uint8_t* accept, float* entropy, int32_t* sampled,
                          int32_t* argmax, int32_t* stop, void* workspace, size_t ws_bytes,
                          void* stream) {
  dg_status st = check_shape(shape);
  if (st != DG_OK) return st;
  if ((st = check_params(params)) != DG_OK) return st;
  if (hidden_fn == nullptr || h_buf == nullptr || has_prev == nullptr || steps_taken == nullptr)
    return DG_ERR_INVALID_ARG;
  if (k_start < 0 || k_start >= params->max_steps) return DG_ERR_RANGE;
  const int B = shape->B, L = shape->L;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int32_t ks[DG_MAX_B];
  uint8_t act[DG_MAX_B];
  int32_t stop_h[DG_MAX_B];
  for (int b = 0; b < B; ++b) {
    act[b] = 1;
    steps_taken[b] = 0;
  }
  for (int k = k_start; k < params->max_steps; ++k) {
    if (hidden_fn(k, canvas, h_buf, user, stream) != 0) return DG_ERR_CALLBACK;
    for (int b = 0; b < B; ++b) ks[b] = k;
    st = dg_denoise_step(shape, params, h_buf, E, e_scale, ks, has_prev, act, canvas, prev_argmax, accept,
                         entropy, sampled, argmax, stop, workspace, ws_bytes, stream);
    if (st != DG_OK) return st;
    if (cudaMemcpyAsync(stop_h, stop, sizeof(int32_t) * B, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
      return DG_ERR_CUDA;
    if ((st = dg_device_status(workspace, ws_bytes, stream)) != DG_OK) return st;
    bool any = false;
    for (int b = 0; b < B; ++b) {
      if (!act[b]) continue;
      has_prev[b] = 1;
      if (stop_h[b] || k == params->max_steps - 1) {
        // commit: every slot takes this step's sampled token
        if (cudaMemcpyAsync(canvas + static_cast<size_t>(b) * L, sampled + static_cast<size_t>(b) * L,
                            sizeof(int32_t) * L, cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
          return DG_ERR_CUDA;
        act[b] = 0;
        steps_taken[b] = k - k_start + 1;
      } else {
        any = true;
      }
    }
    if (!any) break;
  }
  if (cudaStreamSynchronize(cs) != cudaSuccess) return DG_ERR_CUDA;
  return DG_OK;
}

int32_t dg_partials_count(const dg_shape* shard_shape) {
  if (check_shape(shard_shape) != DG_OK) return 0;
  if (device_sms() <= 0) return 0;
  const int pairs = head_max_pairs(shard_shape->e_dtype == DG_E_FP8_E4M3);
  if (pairs <= 0) return 0;
  return ws_layout(*shard_shape, pairs).P;
}

dg_status dg_head_partials(const dg_shape* shard_shape, const dg_params* params, int32_t v_offset,
                           const void* h, const void* E_shard, const float* e_scale_shard,
                           const int32_t* step_idx, float* partials, void* workspace, size_t ws_bytes,
                           void* stream) {
  StepArgs a{shard_shape, params, h, E_shard, e_scale_shard, step_idx, nullptr, nullptr, nullptr, nullptr,
             nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, workspace, ws_bytes,
             static_cast<cudaStream_t>(stream)};
  a.mode = StepMode::kHeadOnly;
  a.v_off = v_offset;
  a.part_out = partials;
  return run_step(a);
}

dg_status dg_merge_partials(const dg_shape* shape, const dg_params* params, const float* partials,
                            int32_t shards, int32_t count, const int32_t* step_idx, const uint8_t* has_prev,
                            const uint8_t* active, int32_t* canvas, int32_t* prev_argmax, uint8_t* accept,
                            float* entropy, int32_t* sampled, int32_t* argmax, int32_t* stop, void* workspace,
                            size_t ws_bytes, void* stream) {
  StepArgs a{shape,   params,  nullptr, nullptr, nullptr, step_idx, has_prev, active, canvas, prev_argmax,
             accept,  entropy, sampled, argmax,  stop,    nullptr,  workspace, ws_bytes,
             static_cast<cudaStream_t>(stream)};
  a.mode = StepMode::kMergeOnly;
  a.part_in = partials;
  a.S = shards;
  a.P = count;
  return run_step(a);
}

const char* dg_last_error_message(void) { return t_last_error; }

dg_status dg_set_head_events(void* ev_start, void* ev_stop) {
  if ((ev_start == nullptr) != (ev_stop == nullptr)) return DG_ERR_INVALID_ARG;
  t_head_ev_start = static_cast<cudaEvent_t>(ev_start);
  t_head_ev_stop = static_cast<cudaEvent_t>(ev_stop);
  return DG_OK;
}

dg_status dg_selftest_bounded_wait(uint64_t limit_ns, void* workspace, size_t ws_bytes, void* stream) {
  if (workspace == nullptr || ws_bytes < kAlign) return DG_ERR_INVALID_ARG;
  if (device_sms() <= 0) return DG_ERR_NO_DEVICE;
  if (launch_wait_selftest(static_cast<uint32_t*>(workspace), limit_ns, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return DG_ERR_CUDA;
  return dg_device_status(workspace, ws_bytes, stream);
}

size_t dg_selfcond_workspace_size(const dg_shape* shape) {
  const size_t step_ws = dg_workspace_size(shape);
  if (step_ws == 0) return 0;
  const int gp = selfcond_gemm_pairs();
  if (gp < 1) return 0;
  return selfcond_layout(*shape, step_ws, gp).total;
}

dg_status dg_embedder_transpose(const dg_shape* shape, const void* E, void* E_t, void* stream) {
  dg_status st = check_shape(shape);
  if (st != DG_OK) return st;
  if (E == nullptr || E_t == nullptr) return DG_ERR_INVALID_ARG;
  if (device_sms() <= 0) return DG_ERR_NO_DEVICE;
  if (!cuda_ok(launch_transpose(E, shape->e_dtype == DG_E_FP8_E4M3, static_cast<uint16_t*>(E_t), shape->V,
                                shape->d, static_cast<cudaStream_t>(stream)),
               "transpose launch"))
    return DG_ERR_CUDA;
  return DG_OK;
}

dg_status dg_denoise_step_selfcond(const dg_shape* shape, const dg_params* params, const void* h, const void* E,
                                   const float* e_scale, const void* E_t, const int32_t* step_idx,
                                   const uint8_t* has_prev, int32_t* canvas, int32_t* prev_argmax,
                                   uint8_t* accept, float* entropy, int32_t* sampled, int32_t* argmax,
                                   int32_t* stop, float* signal, void* workspace, size_t ws_bytes, void* stream) {
  return run_selfcond_step(shape, params, h, E, e_scale, E_t, step_idx, has_prev, canvas, prev_argmax, accept,
                           entropy, sampled, argmax, stop, signal, workspace, ws_bytes,
                           static_cast<cudaStream_t>(stream));
}

dg_status dg_debug_gumbel(const uint32_t* words, int32_t n, float* g_exact, float* lg2e_approx,
                          void* stream) {
  if (n < 0 || (n > 0 && (!words || !g_exact || !lg2e_approx))) return DG_ERR_INVALID_ARG;
  if (device_sms() <= 0) return DG_ERR_NO_DEVICE;
  if (launch_gumbel_probe(words, n, g_exact, lg2e_approx, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DG_ERR_CUDA;
  return DG_OK;
}

}  // extern "C"
