// merge_select.cu -- cross-tile merge of the head's partials, then the
// per-canvas entropy-bounded selection, renoise and stop test.
//
// Each CTA merges the partial records of 8 rows (a warp per row, fixed
// order), writes entropy / sampled / argmax of those rows and takes a ticket
// on its canvas; the CTA that takes the last ticket of a canvas runs the
// per-canvas step for all 256 slots:
//   * selection ([Docs] "DiffusionGemma", Recommended serving configuration,
//     token selection, entropy bound 0.1): slots ordered by (entropy, slot);
//     slot s is accepted when the running entropy sum up to and including s
//     is <= the bound, and the lowest-entropy slot always is (the default
//     rule); the variants accept when the sum over the slots before s is
//     <= the bound, or when s is among the top_k lowest;
//   * renoise (same row: unselected tokens fully renoised; [Report]
//     "DiffusionGemma Technical Report", Figure 3: uniform noise): token
//     (r V) >> 32 from Philox counter (0, slot | 1 << 16, k, b), lane 0;
//   * stop ([Docs] adaptive early stopping, threshold 0.005): the canvas
//     has a previous prediction, its mean entropy is below the threshold and
//     every slot's argmax equals the previous one.
#include <float.h>
#include <limits.h>

#include "dg_device.cuh"
#include "dg_internal.h"

namespace dg {

namespace {

constexpr int kRowsPerCta = 8;  // one warp per row

DG_DEV Partial partial_load(const float* part, size_t plane, size_t idx) {
  Partial a;
  a.m2 = __ldcg(part + 0 * plane + idx);
  a.Sp = __ldcg(part + 1 * plane + idx);
  a.T2 = __ldcg(part + 2 * plane + idx);
  a.zmax = __ldcg(part + 3 * plane + idx);
  a.zarg = __float_as_int(__ldcg(part + 4 * plane + idx));
  a.gkey = __ldcg(part + 5 * plane + idx);
  a.garg = __float_as_int(__ldcg(part + 6 * plane + idx));
  return a;
}

DG_DEV Partial partial_shfl_down(const Partial& a, int off) {
  Partial o;
  o.m2 = __shfl_down_sync(0xffffffffu, a.m2, off);
  o.Sp = __shfl_down_sync(0xffffffffu, a.Sp, off);
  o.T2 = __shfl_down_sync(0xffffffffu, a.T2, off);
  o.zmax = __shfl_down_sync(0xffffffffu, a.zmax, off);
  o.zarg = __shfl_down_sync(0xffffffffu, a.zarg, off);
  o.gkey = __shfl_down_sync(0xffffffffu, a.gkey, off);
  o.garg = __shfl_down_sync(0xffffffffu, a.garg, off);
  return o;
}

}  // namespace

__global__ void __launch_bounds__(256)
merge_select_kernel(const __grid_constant__ MergeParams p) {
  __shared__ unsigned long long s_key[256];
  __shared__ float s_h[256];
  __shared__ double s_red[8];
  __shared__ int s_last;

  const int t = threadIdx.x;
  const int warp = t >> 5;
  const int lane = t & 31;
  constexpr int kCtasPerCanvas = 256 / kRowsPerCta;
  const int grp = blockIdx.x / kCtasPerCanvas;
  int b;  // only the canvases this step updates
  if (p.canvas_of_dev != nullptr) {
    // device-side loop: the launch covers every canvas; the loop's control
    // kernel lists the ones still running
    if (grp >= __ldcg(p.n_dev)) return;
    b = __ldcg(p.canvas_of_dev + grp);
  } else {
    b = p.canvas_of[grp];
  }
  const int row = b * 256 + (blockIdx.x % kCtasPerCanvas) * kRowsPerCta + warp;
  const size_t plane = static_cast<size_t>(p.R) * p.P;

  // The next step's head may launch now (it waits for this grid before it
  // touches memory); then wait, as a programmatic dependent of the head,
  // until the partial records are complete and visible.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- merge the P partial records of this row: lane j takes j, j+32, ...;
  // then a fixed tree over the lanes (lane i absorbs lane i + off)
  Partial a;
  partial_init(a);
  const size_t shard_stride = static_cast<size_t>(kPartialFields) * plane;
  const int n_rec = p.S * p.P;
  // the first four records of each lane are loaded before any is merged
  // (one round trip to L2 instead of four: a B = 1 row has 74 records)
  {
    Partial r4[4];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int qq = lane + 32 * it;
      if (qq < n_rec) {
        const int s = qq / p.P, q = qq - s * p.P;
        r4[it] = partial_load(p.part + s * shard_stride, plane, static_cast<size_t>(row) * p.P + q);
      } else {
        partial_init(r4[it]);
      }
    }
#pragma unroll
    for (int it = 0; it < 4; ++it) partial_merge(a, r4[it]);
  }
  for (int qq = lane + 128; qq < n_rec; qq += 32) {
    const int s = qq / p.P, q = qq - s * p.P;
    partial_merge(a, partial_load(p.part + s * shard_stride, plane, static_cast<size_t>(row) * p.P + q));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const Partial o = partial_shfl_down(a, off);
    if (lane < off) partial_merge(a, o);
  }
  if (lane == 0) {
    p.row_rec[row] = 0u;  // the head's key record of this row starts empty next step
    // H = ln S - ln2 T2 / S with S = 1 + Sp, in float64 from the float32
    // record, clamped at 0 (the exact value is >= 0)
    const double sp = static_cast<double>(a.Sp);
    double H = log1p(sp) - 0.69314718055994530942 * static_cast<double>(a.T2) / (1.0 + sp);
    H = H > 0.0 ? H : 0.0;
    p.entropy[row] = static_cast<float>(H);
    if (p.rowstat != nullptr) p.rowstat[row] = make_float2(a.m2, static_cast<float>(1.0 / (1.0 + sp)));
    p.sampled[row] = a.garg;
    p.argmax[row] = a.zarg;
  }

  // ---- ticket: the last CTA of this canvas does the per-canvas step
  __threadfence();
  __syncthreads();
  if (t == 0) {
    const uint32_t prev = atomicAdd(&p.tickets[b], 1u);
    s_last = (prev == kCtasPerCanvas - 1) ? 1 : 0;
    if (s_last) p.tickets[b] = 0u;  // reset for the next step
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  CanvasParam cp;
  if (p.cp_dev != nullptr) {
    cp.k = __ldcg(&p.cp_dev[b].k);
    cp.has_prev = __ldcg(&p.cp_dev[b].has_prev);
  } else {
    cp = p.cp[b];
  }
  const int s = t;  // slot
  const int grow = b * 256 + s;
  const float H = __ldcg(p.entropy + grow);
  const int samp = __ldcg(p.sampled + grow);
  const int amax = __ldcg(p.argmax + grow);

  // ---- entropy-bounded selection: order by (H, slot); H >= 0 so its bits
  // order like the values
  const unsigned long long key =
      (static_cast<unsigned long long>(__float_as_uint(H)) << 32) | static_cast<unsigned>(s);
  s_key[s] = key;
  s_h[s] = H;
  __syncthreads();
  // Running sums over the slots ordered before this one (exclusive) or up
  // to and including it (inclusive): four independent float64 sums over
  // i = j mod 4, added in a fixed order.  The rank is the slot's position.
  double cs[4] = {0.0, 0.0, 0.0, 0.0};
  int rk[4] = {0, 0, 0, 0};
  const bool inclusive = p.selection_rule == DG_SELECT_CUMSUM;
#pragma unroll 4
  for (int i = 0; i < 256; i += 4) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const unsigned long long ki = s_key[i + j];
      const bool before = ki < key;
      if (before || (inclusive && ki == key)) cs[j] += static_cast<double>(s_h[i + j]);
      rk[j] += before ? 1 : 0;
    }
  }
  const double csum = (cs[0] + cs[1]) + (cs[2] + cs[3]);
  const int rank = (rk[0] + rk[1]) + (rk[2] + rk[3]);
  bool accepted;
  if (p.selection_rule == DG_SELECT_TOPK)
    accepted = rank < p.top_k;
  else  // CUMSUM: inclusive sum <= bound, at least one; MI: exclusive sum <= bound
    accepted = (csum <= p.entropy_bound) || (rank == 0);

  // ---- renoise
  int tok = samp;
  if (!accepted) {
    uint32_t r[4];
    philox4x32_10(0u, static_cast<uint32_t>(s) | (kPurposeRenoise << 16), static_cast<uint32_t>(cp.k),
                  static_cast<uint32_t>(b), p.seed_lo, p.seed_hi, r);
    tok = static_cast<int>((static_cast<uint64_t>(r[0]) * static_cast<uint64_t>(p.V)) >> 32);
  }

  // ---- stop: mean entropy (float64 sum in a fixed tree order) and agreement
  double hsum = static_cast<double>(H);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) hsum += __shfl_xor_sync(0xffffffffu, hsum, off);
  if ((t & 31) == 0) s_red[t >> 5] = hsum;
  const int prev = p.prev_argmax[grow];
  const int same = __syncthreads_and(prev == amax);
  double total = 0.0;
#pragma unroll
  for (int w = 0; w < 8; ++w) total += s_red[w];
  const double mean_h = total / 256.0;
  const bool stop = cp.has_prev && same && (mean_h < p.stop_entropy);

  p.accept[grow] = accepted ? 1 : 0;
  p.canvas[grow] = tok;
  p.prev_argmax[grow] = amax;
  if (t == 0) p.stop[b] = stop ? 1 : 0;
}

cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.B * (256 / kRowsPerCta), 1, 1);  // p.B: canvases updated
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  // programmatic dependent launch: the launch overlaps the head kernel's
  // tail; griddepcontrol.wait in the kernel orders the data
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, merge_select_kernel, p);
}

}  // namespace dg
