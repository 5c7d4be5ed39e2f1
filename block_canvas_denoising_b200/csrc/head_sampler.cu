// head_sampler.cu -- the fused tied-LM-head + sampler kernel for sm_100a.
//
// z = h . E^T ([Report] "DiffusionGemma Technical Report", Table 1: the
// 740M embedder over the 262k vocabulary is the output head) is computed
// tile by tile on the 5th-generation tensor cores and never leaves the SM:
// each 128 x 256 float32 accumulator tile lives in tensor memory (TMEM) and
// is reduced in place by the epilogue warps into per-row partials of
//   * the online softmax of x = z / tau_k in base 2: m2 = max x log2(e),
//     S = sum 2^(x log2 e - m2), T2 = sum (x log2 e - m2) 2^(...), carried
//     as Sp = S - 1 with the maximum's unit mass kept out of the sums -- the
//     entropy of the tempered distribution follows as ln S - ln2 T2 / S
//     ([Docs] "DiffusionGemma", Recommended serving configuration: entropy
//     drives token selection and adaptive stopping; temperature schedule);
//   * the argmax of z (the prediction compared across steps for stopping);
//   * the Gumbel-max draw argmax_v fl(fl(z_v / tau) + g32(u_v)) with u_v
//     from Philox4x32-10 counter (v >> 2, slot, k, b), lane v & 3.
//
// The kernel runs as CTA pairs (clusters of 2) on the tcgen05 cta_group::2
// path: the pair computes 256 rows x 256 vocabulary columns per tile, the
// leader CTA issuing 256x256xK MMAs over both CTAs' shared memory; each CTA
// holds its 128-row half of the tile in its own TMEM.
//
// Warp roles (576 threads, one CTA per SM, persistent):
//   warp 0       TMEM allocator; in the leader, the MMA issuer.
//   warp 1       TMA producer: this CTA's halves of the h and E tiles into a
//                shared-memory ring (completion on the leader's barrier).
//   warps 2..17  epilogue: warp w reads TMEM lane quarter w % 4 and 64-column
//                group (w - 2) / 4 of each tile; two accumulators alternate so
//                the epilogue of tile t overlaps the MMAs of tile t + 1.
//
// FP8 embedder (E4M3 codes q with a float32 scale s_v per vocabulary row):
// the codes go from HBM to the tensor cores untouched (kind::f8f6f4, half
// the bytes of bf16).  h is split once per step by a small kernel into two
// E4M3 terms with a power-of-two row scale, h[r] * 2^k_r = h1[r] + h2[r],
// and every K step issues the two MMAs h1 . q^T and h2 . q^T into the same
// accumulator -- at twice the bf16 rate, the same tensor time as one bf16
// MMA.  The epilogue forms z = (acc * s_v) * 2^-k_r.  The split is exact
// for every |h| >= 2^-9 max_k |h[r, k]| (8 significant bits in two 4-bit
// terms); below that its error is at most 2^-10 * 2^-k_r.
// ([Docs] "DiffusionGemma": the model is served with FP8 weights.)
#include <float.h>
#include <limits.h>

#include <cuda_bf16.h>

#include "dg_device.cuh"
#include "dg_internal.h"
#include "per_device.h"

namespace dg {

namespace {

// Row tiles this launch covers, and the per-canvas data: from device memory
// in the device-side loop's instance (kDev), else from the launch
// parameters (a separate instance keeps those reads out of the sampler's
// register budget).
template <bool kDev>
DG_DEV int row_tiles(const HeadParams& p) {
  if constexpr (kDev) return __ldcg(p.mt_dev);
  return p.split.MT;
}
template <bool kDev>
DG_DEV CanvasParam canvas_param(const HeadParams& p, int b) {
  if constexpr (kDev) {
    CanvasParam c;
    c.k = __ldcg(&p.cp_dev[b].k);
    c.inv_tau = __ldcg(&p.cp_dev[b].inv_tau);
    return c;
  }
  return p.cp[b];
}

// Unit u: row tile (canvas) m, vocabulary tiles [n0, n1), unit index q
// within the row tile; mt = row_tiles(p).
template <bool kDev>
DG_DEV void unit_range(const HeadParams& p, int mt, int u, int& m, int& n0, int& n1, int& q) {
  const HeadSplit& sp = p.split;
  q = u / mt;
  if constexpr (kDev)
    m = static_cast<int>(__ldcg(p.mtile_dev + (u - q * mt)));
  else
    m = p.mtile[u - q * mt];
  n0 = static_cast<int>((static_cast<int64_t>(q) * sp.NT) / sp.Q);
  n1 = static_cast<int>((static_cast<int64_t>(q + 1) * sp.NT) / sp.Q);
}

DG_DEV void latch_error(uint32_t* err, uint32_t code) { atomicOr(err, code); }

DG_DEV void gumbel_update(Partial& pt, float key, int v) {
  if (key > pt.gkey || (key == pt.gkey && v < pt.garg)) {
    pt.gkey = key;
    pt.garg = v;
  }
}

// The specified key of one element, kept out of line: it is needed rarely,
// and inlining it at every call site would bloat the epilogue's loop.
__device__ __noinline__ float key_exact_call(float z, float inv_tau, uint32_t w) {
  return key_exact(z, inv_tau, w);
}

DG_DEV void confirm_exact(Partial& pt, float z, float inv_tau, uint32_t w, int v) {
  gumbel_update(pt, key_exact_call(z, inv_tau, w), v);
}

// Streaming state of the Gumbel screen.  Every element gets a screening key
// ka within e of its specified key (kGumbelApproxErr plus roundings); keys
// are packed with the element's index in their 3 lowest bits, which moves
// them by at most 7 ulps.  Per group of 8 the largest two packed keys
// (K1g, K2g) are found branch-free; with eps above twice the combined error:
//   * K1g < K1a - eps: nothing in the group can beat the pending candidate;
//   * a near-tie (K2g >= K1g - eps inside the group, or |K1g - K1a| <= eps)
//     confirms exactly every group element within eps of K1g (rare);
//   * K1g > K1a + eps: the group's best becomes the pending candidate (the
//     old one is then certainly worse).
// The pending candidate is confirmed exactly at the end of each unit.
struct Screen {
  float K1a;       // packed screening key of the pending candidate (-inf if none)
  float z1;        // its logit
  uint32_t w1;     // its Philox word
  int v1;          // its vocabulary index
  float lim_eps;   // the group bound's limit: max(K1a, thr) less its margin
};

DG_DEV float screen_eps(float k) {
  return 2.0f * kGumbelApproxErr + (fabsf(k) + 64.0f) * 1.9073486328125e-06f;  // 2^-19
}

// The group bound's limit, formed when thr (per tile) or K1a changes.
DG_DEV void screen_limit(Screen& sc, float thr) {
  const float lim = fmaxf(sc.K1a, thr);
  sc.lim_eps = lim - 2.0f * screen_eps(lim);
}

DG_DEV void screen_reset(Screen& sc) { sc.K1a = -FLT_MAX; }

DG_DEV void screen_flush(Screen& sc, Partial& pt, float inv_tau) {
  if (sc.K1a > -FLT_MAX) confirm_exact(pt, sc.z1, inv_tau, sc.w1, sc.v1);
  screen_reset(sc);
}

DG_DEV void top2(float& a1, float& a2, float b1, float b2) {
  const float hi = fmaxf(a1, b1);
  a2 = fmaxf(fminf(a1, b1), fmaxf(a2, b2));
  a1 = hi;
}

// The Philox counter words of one slot, (slot | purpose << 16, k, b): with
// kHoist the first two rounds' slot-constant products formed once
// (philox_row), else the three words themselves (the FP8 instance, whose
// registers are tighter, draws with the plain rounds).
template <bool kHoist>
DG_DEV PhiloxRow slot_counter(uint32_t c1, uint32_t c2, uint32_t c3, const uint32_t (&rk0)[10],
                              const uint32_t (&rk1)[10]) {
  if constexpr (kHoist) return philox_row(c1, c2, c3, rk0, rk1);
  PhiloxRow r;
  r.x0r1 = c1;
  r.b1 = c2;
  r.e0 = c3;
  r.c1k = 0;
  r.d = 0;
  return r;
}

// The Philox words of the 8 consecutive vocabulary entries 4 cb .. 4 cb + 7
// of the slot whose counter words are `pr`.
template <bool kHoist>
DG_DEV void philox_words8(uint32_t cb, const PhiloxRow& pr, const uint32_t (&rk0)[10], const uint32_t (&rk1)[10],
                          uint32_t (&w)[8]) {
  uint32_t wa[4], wb[4];
  if constexpr (kHoist) {
    philox4x32_10_row(cb, pr, rk0, rk1, wa);
    philox4x32_10_row(cb + 1, pr, rk0, rk1, wb);
  } else {
    philox4x32_10_keys(cb, pr.x0r1, pr.b1, pr.e0, rk0, rk1, wa);
    philox4x32_10_keys(cb + 1, pr.x0r1, pr.b1, pr.e0, rk0, rk1, wb);
  }
#pragma unroll
  for (int l = 0; l < 4; ++l) {
    w[l] = wa[l];
    w[4 + l] = wb[l];
  }
}

// Eight consecutive logits of one row: z[0..7] are vocabulary v0 .. v0+7.
// thr: the best screening key any column group of this row has reached in
// the current unit (a lower bound on the row's winning key, up to eps).
// wm_pre: when have_wm (warp-uniform), the group's largest Philox word,
// computed beforehand by another warp; the words themselves are then drawn
// here only if the group passes its bound.
// Largest of three floats (finite inputs: the same value as two fmaxf).
DG_DEV float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Largest of a group's eight Philox words.
DG_DEV uint32_t max_word8(const uint32_t (&w)[8]) {
  return __vimax3_u32(__vimax3_u32(w[0], w[1], w[2]), __vimax3_u32(w[3], w[4], w[5]), max(w[6], w[7]));
}

// Two float32 lanes in one 64-bit register for the packed f32x2 arithmetic
// (each lane rounds exactly as the scalar instruction).
DG_DEV uint64_t pack2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
DG_DEV void unpack2(uint64_t v, float& a, float& b) { asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v)); }
DG_DEV uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
DG_DEV uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Online softmax partial of a group, base 2: every element below the running
// maximum adds e = 2^(z c2 - m2) to Sp and (z c2 - m2) e to T2, in two lanes
// (even and odd elements) folded at the end.  kSel: the group holds the
// running maximum, whose unit elements are left out; otherwise every element
// is below it and no test is needed.
template <bool kSel>
DG_DEV void softmax8(const float (&z)[8], float c2, Partial& pt) {
  const float nm = -pt.m2;
  const uint64_t c22 = pack2(c2, c2), nm2 = pack2(nm, nm);
  uint64_t s = pack2(0.f, 0.f), t = pack2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    const uint64_t dd = fma2(pack2(z[j], z[j + 1]), c22, nm2);
    float d0, d1;
    unpack2(dd, d0, d1);
    float e0 = ex2_approx(d0), e1 = ex2_approx(d1);
    if (kSel) {
      e0 = z[j] < pt.zmax ? e0 : 0.f;
      e1 = z[j + 1] < pt.zmax ? e1 : 0.f;
    }
    const uint64_t ee = pack2(e0, e1);
    s = add2(s, ee);
    t = fma2(dd, ee, t);
  }
  float s0, s1, t0, t1;
  unpack2(s, s0, s1);
  unpack2(t, t0, t1);
  pt.Sp += s0 + s1;
  pt.T2 += t0 + t1;
}

template <bool kHoist>
DG_DEV void process8(const float (&z)[8], int v0, float inv_tau, float c2, const PhiloxRow& pr,
                     const uint32_t (&rk0)[10], const uint32_t (&rk1)[10], float thr, bool have_wm,
                     uint32_t wm_pre, Partial& pt, Screen& sc) {
  // ---- group max; does the group hold the row's running maximum?  (c2 > 0,
  // so the maximum of z is the maximum of x; groups arrive in increasing v)
  const float gmax = fmax3(fmax3(z[0], z[1], z[2]), fmax3(z[3], z[4], z[5]), fmaxf(z[6], z[7]));
  if (gmax >= pt.zmax) {
    // elements equal to the maximum are units (exponent exactly 0): count
    // them, and find the first (the argmax, ties to the lower index)
    float neq = 0.f;
    int jj = 7;
#pragma unroll
    for (int j = 7; j >= 0; --j) {
      const bool eq = z[j] == gmax;
      neq += eq ? 1.f : 0.f;
      jj = eq ? j : jj;
    }
    if (gmax > pt.zmax) {
      // new maximum: the old total mass 1 + Sp joins the ordinary mass,
      // shifted by delta = m2_old - m2_new <= 0
      const float nm2 = gmax * c2;
      const float delta = pt.m2 - nm2;
      const float scl = ex2_approx(delta);
      const float tot = 1.0f + pt.Sp;
      pt.T2 = (pt.T2 + delta * tot) * scl;
      pt.Sp = fmaf(tot, scl, neq - 1.0f);
      pt.m2 = nm2;
      pt.zmax = gmax;
      pt.zarg = v0 + jj;
    } else {
      pt.Sp += neq;  // exact ties with the running maximum: more units
    }
    softmax8<true>(z, c2, pt);
  } else {
    softmax8<false>(z, c2, pt);
  }

  // ---- Gumbel-max screen (branch-free except for rare near-ties)
  // Group bound: g32 is nondecreasing in the Philox word and x = fl(z inv_tau)
  // in z, so no key of the group exceeds fl(fl(gmax inv_tau) + g32(max word)).
  // When even that bound is clearly below the best key already known for the
  // row, no element of the group can win or tie: skip it (first with the
  // largest possible noise, before any Philox work, then with the group's).
  // The margin covers the screen's error on both keys and the index packing.
  const float lim_eps = sc.lim_eps;
  const float x0max = __fmaf_rn(gmax, inv_tau, kGumbelC0);
  if (x0max + (kGumbelMaxNoise + 1e-3f - kGumbelC0) < lim_eps) return;
  const uint32_t cb = static_cast<uint32_t>(v0) >> 2;
  uint32_t w[8];
  if (have_wm) {
    if (__fmaf_rn(lg2_exp1_approx(wm_pre), -kLn2, x0max) < lim_eps) return;
    philox_words8<kHoist>(cb, pr, rk0, rk1, w);
  } else {
    philox_words8<kHoist>(cb, pr, rk0, rk1, w);
    const uint32_t wm = max_word8(w);
    if (__fmaf_rn(lg2_exp1_approx(wm), -kLn2, x0max) < lim_eps) return;
  }
  float kp[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float x0 = __fmaf_rn(z[j], inv_tau, kGumbelC0);
    const float ka = __fmaf_rn(lg2_exp1_approx(w[j]), -kLn2, x0);
    kp[j] = __int_as_float((__float_as_int(ka) & ~7) | j);
  }
  float a1 = fmaxf(kp[0], kp[1]), a2 = fminf(kp[0], kp[1]);
  float b1 = fmaxf(kp[2], kp[3]), b2 = fminf(kp[2], kp[3]);
  float c1 = fmaxf(kp[4], kp[5]), c2b = fminf(kp[4], kp[5]);
  float d1 = fmaxf(kp[6], kp[7]), d2 = fminf(kp[6], kp[7]);
  top2(a1, a2, b1, b2);
  top2(c1, c2b, d1, d2);
  top2(a1, a2, c1, c2b);
  const float K1g = a1, K2g = a2;
  const float eps = screen_eps(K1g);
  if (K1g >= sc.K1a - eps && (K2g >= K1g - eps || K1g <= sc.K1a + eps)) {
    const float lo = K1g - eps;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (kp[j] >= lo) confirm_exact(pt, z[j], inv_tau, w[j], v0 + j);
  }
  if (K1g > sc.K1a + eps) {
    const int j1 = __float_as_int(K1g) & 7;
    float zs = z[0];
    uint32_t ws = w[0];
#pragma unroll
    for (int j = 1; j < 8; ++j) {
      zs = (j == j1) ? z[j] : zs;
      ws = (j == j1) ? w[j] : ws;
    }
    sc.K1a = K1g;
    sc.z1 = zs;
    sc.w1 = ws;
    sc.v1 = v0 + j1;
    screen_limit(sc, thr);
  }
}

// Scales (FP8 embedder: z = (acc * s_v) * rinv, rinv = 2^-k_r), optional
// logits dump, then the group's reductions.
// Self-conditioning: the group's block-scaled probabilities
// bf16(2^(z c2 - ref)) for the 64-entry block it belongs to; the block's
// reference is set at its first group: the running maximum so far, or the
// group's own maximum when the unit has just started (values of later
// groups may exceed 1; a block whose values exceed 2^126 latches a fault).
// Only the self-conditioning instances (kProbs) contain it.
__device__ __forceinline__ float write_probabilities(float4 za, float4 zb, int v0, int row, float c2, const HeadParams& p,
                                                 float m2, float blk_ref) {
  const float z[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
  if ((v0 & 63) == 0) {
    const float g = fmaxf(fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3])), fmaxf(fmaxf(z[4], z[5]), fmaxf(z[6], z[7])));
    blk_ref = fmaxf(m2, g * c2);
    p.pref[static_cast<size_t>(v0 / 64) * p.R + row] = blk_ref;  // [V / 64][R]: coalesced over rows
  }
  uint32_t w[4];
  bool over = false;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float d0 = fmaf(z[2 * j], c2, -blk_ref), d1 = fmaf(z[2 * j + 1], c2, -blk_ref);
    over |= (d0 > 126.0f) || (d1 > 126.0f);
    const __nv_bfloat162 b = __floats2bfloat162_rn(ex2_approx(fminf(d0, 126.0f)), ex2_approx(fminf(d1, 126.0f)));
    w[j] = *reinterpret_cast<const uint32_t*>(&b);
  }
  if (over) atomicOr(p.err, kErrProbRange);
  *reinterpret_cast<uint4*>(p.ptilde + static_cast<size_t>(row) * p.V + v0) = make_uint4(w[0], w[1], w[2], w[3]);
  return blk_ref;
}

template <bool kFp8, bool kProbs>
DG_DEV void epi_group(const uint32_t* r, int v0, int row, float rinv, float inv_tau, float c2,
                      const PhiloxRow& pr, float thr, bool have_wm, uint32_t wm_pre, const HeadParams& p,
                      Partial& pt, Screen& sc, float& blk_ref) {
  float z[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) z[j] = __uint_as_float(r[j]);
  if (kFp8) {
    const float4* scp = reinterpret_cast<const float4*>(p.e_scale + v0);
    const float4 s0 = __ldg(scp), s1 = __ldg(scp + 1);
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) z[j] = __fmul_rn(__fmul_rn(z[j], sv[j]), rinv);
  }
  if (p.logits_out != nullptr) {
    float4* dst = reinterpret_cast<float4*>(p.logits_out + static_cast<size_t>(row) * p.V + v0);
    dst[0] = make_float4(z[0], z[1], z[2], z[3]);
    dst[1] = make_float4(z[4], z[5], z[6], z[7]);
  }
  if (kProbs)
    blk_ref = write_probabilities(make_float4(z[0], z[1], z[2], z[3]), make_float4(z[4], z[5], z[6], z[7]), v0, row,
                                  c2, p, pt.m2, blk_ref);
  // z, e_scale and the dump are indexed within this launch's rows of E; the
  // sampler (Philox counters, token indices) uses the global vocabulary index
  process8<!kFp8>(z, v0 + p.v_off, inv_tau, c2, pr, p.rk0, p.rk1, thr, have_wm, wm_pre, pt, sc);
}

// Named barrier over the epilogue warps only (barrier 1).
DG_DEV void epilogue_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
}

}  // namespace

// One CTA of 576 threads per SM: its 18 warps share the four schedulers'
// register files as 5 + 5 + 4 + 4 warps, so a thread may use at most 96
// registers (5 x 32 x 96 <= 16,384), which the launch bound enforces.
// kProbs: the self-conditioning instance, which also writes the block-scaled
// probabilities; kDev: the device-side loop's instance, which reads the
// per-canvas data from device memory (separate instances keep that code out
// of the plain sampler's register budget).
template <bool kFp8, bool kProbs, bool kDev>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kHeadThreads, 1)
head_sampler_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                    const __grid_constant__ CUtensorMap tmB, const __grid_constant__ HeadParams p) {
  using Cfg = HeadCfg<kFp8>;
  constexpr int kStages = Cfg::kStages;
  constexpr int kATiles = Cfg::kATiles;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // stage s: A tile(s) at sA + (s * kATiles + t) * kTileBytes, E tile at sB + s * kTileBytes
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kATiles * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kStages * kTileBytes);
  // barriers: full[S], empty[S], tfull[2], tempty[2], wfull[2], wempty[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 8);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // [column group][field][row of the CTA half]
  float* sPart = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);
  // [column group][row of the CTA half]: best screening key of the unit so far
  volatile float* sRec = sPart + kColGroups * kPartialFields * kBlockM;
  // [buffer][group of 8 columns][row of the MMA warp's lane quarter]
  uint32_t* sWmax = reinterpret_cast<uint32_t*>(sPart + kColGroups * kPartialFields * kBlockM + kColGroups * kBlockM);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader (issues the MMAs), 1 = peer
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const HeadSplit& sp = p.split;
  const int mt = row_tiles<kDev>(p);       // row tiles (canvases) of this launch
  const int units = mt * sp.Q;

  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[kStages + s]); };
  auto tfull_bar = [&](int a) { return smem_u32(&bars[2 * kStages + a]); };
  auto tempty_bar = [&](int a) { return smem_u32(&bars[2 * kStages + 2 + a]); };
  auto wfull_bar = [&](int b) { return smem_u32(&bars[2 * kStages + 4 + b]); };
  auto wempty_bar = [&](int b) { return smem_u32(&bars[2 * kStages + 6 + b]); };

  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmA);
    if (kFp8) prefetch_tensormap(&tmA2);
    prefetch_tensormap(&tmB);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);   // leader's producer arrival + both CTAs' bytes
      mbar_init(empty_bar(s), 1);  // one multicast commit per use
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);               // one multicast commit per tile
      mbar_init(tempty_bar(a), 2 * kEpiWarps);  // every epilogue warp of the pair
      mbar_init(wfull_bar(a), kEpiWarps - 4);   // the 12 word-helper warps
      mbar_init(wempty_bar(a), 4);              // the MMA quarter's 4 warps
    }
    *s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(smem_u32(tmem_slot), 2 * kBlockN);
    tmem_relinquish_pair();
  }
  if (threadIdx.x >= kEpiWarp0 * 32) sRec[threadIdx.x - kEpiWarp0 * 32] = -FLT_MAX;
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Launched as a programmatic dependent of the preceding kernel (the
  // previous step's merge, which clears the key records and reads the
  // partial records this launch overwrites): the set-up above overlaps its
  // tail; nothing here reads or writes global memory before it completes.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    // Each CTA loads its own halves: 128 rows of h (rows rank*128 of the
    // pair tile) and 128 rows of E (the rank-th half of the 256 vocabulary
    // columns).  All copies complete on the leader's full barrier.
    if (lane == 0) {
      const uint64_t pol_h = policy_evict_last();   // h is re-read by every tile
      const uint64_t pol_e = policy_evict_first();  // E streams through once
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = pair; u < units && ok; u += npairs) {
        int m, n0, n1, q;
        unit_range<kDev>(p, mt, u, m, n0, n1, q);
        for (int n = n0; n < n1 && ok; ++n) {
          for (int kb = 0; kb < sp.KB; ++kb) {
            if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, p.wait_ns)) {
              latch_error(p.err, kErrWaitTmaProducer);
              ok = false;
              break;
            }
            const uint32_t fb = full_bar(stage);
            if (rank == 0) mbar_arrive_expect_tx(fb, 2 * Cfg::kStageBytes);
            const uint32_t fb_leader = mapa_shared(fb, 0);
            const int kx = kb * Cfg::kBlockKElems;  // 128 B of K: 16-byte aligned
            const int hrow = m * kPairM + static_cast<int>(rank) * kBlockM;
            uint8_t* a0 = sA + stage * kATiles * kTileBytes;
            tma_load_2d_pair(smem_u32(a0), &tmA, fb_leader, kx, hrow, pol_h);
            if (kFp8) tma_load_2d_pair(smem_u32(a0 + kTileBytes), &tmA2, fb_leader, kx, hrow, pol_h);
            tma_load_2d_pair(smem_u32(sB + stage * kTileBytes), &tmB, fb_leader, kx,
                             n * kBlockN + static_cast<int>(rank) * kHalfN, pol_e);
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      // Tail: wait until the MMAs have released every stage, so no commit
      // arrival can land in this CTA's shared memory after it exits.
      for (int i = 0; i < kStages && ok; ++i) {
        if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, p.wait_ns)) {
          latch_error(p.err, kErrWaitTmaProducer);
          ok = false;
        }
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer (leader)
    // One thread feeds the tensor core while 4 epilogue warps share its
    // scheduler, so its loop is kept short: descriptors and barrier
    // addresses advance by constant 32-bit steps per stage.
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = kFp8 ? instr_desc_e4m3_f32(kPairM, kBlockN) : instr_desc_bf16_f32(kPairM, kBlockN);
      const uint64_t a_desc0 = smem_desc_k_sw128(smem_u32(sA));
      const uint64_t b_desc0 = smem_desc_k_sw128(smem_u32(sB));
      const uint32_t a_hi = static_cast<uint32_t>(a_desc0 >> 32), b_hi = static_cast<uint32_t>(b_desc0 >> 32);
      const uint32_t a_lo0 = static_cast<uint32_t>(a_desc0), b_lo0 = static_cast<uint32_t>(b_desc0);
      constexpr uint32_t kAStep = (kATiles * kTileBytes) >> 4;  // descriptor units of 16 B
      constexpr uint32_t kBStep = kTileBytes >> 4;
      const uint32_t full0 = full_bar(0), empty0 = empty_bar(0);
      uint32_t a_lo = a_lo0, b_lo = b_lo0, fb = full0, eb = empty0;
      int stage = 0;
      uint32_t phase = 0;
      int tile = 0;
      bool ok = true;
      for (int u = pair; u < units && ok; u += npairs) {
        int m, n0, n1, q;
        unit_range<kDev>(p, mt, u, m, n0, n1, q);
        for (int n = n0; n < n1 && ok; ++n, ++tile) {
          const int acc = tile & 1;
          const uint32_t acc_phase = (tile >> 1) & 1;
          if (!mbar_wait_bounded<true>(tempty_bar(acc), acc_phase ^ 1u, p.wait_ns)) {
            latch_error(p.err, kErrWaitMmaAcc);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBlockN);
          for (int kb = 0; kb < sp.KB; ++kb) {
            if (!mbar_wait_bounded(fb, phase, p.wait_ns)) {
              latch_error(p.err, kErrWaitMmaFull);
              ok = false;
              break;
            }
            tc_fence_after();
            // 32 B of K per instruction (16 bf16 or 32 E4M3): +2 in the
            // descriptor's 16-byte address field, inside the swizzled rows
#pragma unroll
            for (int k32 = 0; k32 < 4; ++k32) {
              const uint32_t acc_flag = (kb > 0 || k32 > 0) ? 1u : 0u;
              tc_mma_pair_lohi<kFp8>(d_tmem, a_lo + 2u * k32, a_hi, b_lo + 2u * k32, b_hi, idesc, acc_flag);
              if (kFp8)  // h2 . q^T: the second A tile of the stage
                tc_mma_pair_lohi<kFp8>(d_tmem, a_lo + (kTileBytes >> 4) + 2u * k32, a_hi, b_lo + 2u * k32, b_hi,
                                       idesc, 1u);
            }
            tc_commit_pair_mc(eb, 0x3);  // frees the stage in both CTAs
            a_lo += kAStep;
            b_lo += kBStep;
            fb += 8;
            eb += 8;
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1u;
              a_lo = a_lo0;
              b_lo = b_lo0;
              fb = full0;
              eb = empty0;
            }
          }
          if (ok) tc_commit_pair_mc(tfull_bar(acc), 0x3);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
    const int cg = (warp - kEpiWarp0) >> 2;     // 64-column group of the tile
    const int rloc = quarter * 32 + lane;
    // Integer multiplies next to the MMA issuer slow the tensor core, so the
    // Philox words that bound each group of 8 logits of the MMA warp's lane
    // quarter are drawn one tile ahead by the other 12 epilogue warps
    // (helpers) into sWmax; the MMA quarter's warps draw words themselves
    // only for the rare groups that pass their bound.
    constexpr int kMmaQuarter = kMmaWarp & 3;
    constexpr int kTileGroups = kBlockN / 8;  // 32 groups of 8 columns per tile
    const bool mma_quarter = quarter == kMmaQuarter;
    const int hidx = cg * 3 + (quarter > kMmaQuarter ? quarter - 1 : quarter);  // helpers: 0..11
    // Helpers: the largest Philox word of every group of tile t (row tile m_t,
    // vocabulary tile n_t) for the MMA quarter's 32 rows, into buffer t & 1.
    auto produce_words = [&](int t, int m_t, int n_t) -> bool {
      const int buf = t & 1;
      if (!mbar_wait_bounded(wempty_bar(buf), ((t >> 1) & 1) ^ 1u, p.wait_ns)) {
        latch_error(p.err, kErrWaitEpilogue);
        *s_abort = 1;
        return false;
      }
      uint32_t* dst = sWmax + buf * (kTileGroups * 32);
      for (int i = hidx * 32 + lane; i < kTileGroups * 32; i += (kEpiWarps - 4) * 32) {
        const int r = i & 31, g = i >> 5;
        const int hrow = m_t * kPairM + static_cast<int>(rank) * kBlockM + kMmaQuarter * 32 + r;
        const int hb = hrow >> 8;
        uint32_t w[8];
        const PhiloxRow pr = slot_counter<!kFp8>(static_cast<uint32_t>(hrow & 255) | (kPurposeGumbel << 16),
                                                 static_cast<uint32_t>(canvas_param<kDev>(p, hb).k),
                                                 static_cast<uint32_t>(hb), p.rk0, p.rk1);
        philox_words8<!kFp8>(static_cast<uint32_t>(p.v_off + n_t * kBlockN + g * 8) >> 2, pr, p.rk0, p.rk1, w);
        dst[g * 32 + r] = max_word8(w);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(wfull_bar(buf));
      return true;
    };
    // Every epilogue warp runs the same units and named barriers even after
    // a failed wait (it then skips the work), so the barriers cannot deadlock.
    int tile = 0;
    bool ok = true;
    if (!mma_quarter && pair < units) {
      int m, n0, n1, q;
      unit_range<kDev>(p, mt, pair, m, n0, n1, q);
      ok = produce_words(0, m, n0);
    }
    for (int u = pair; u < units; u += npairs) {
      int m, n0, n1, q;
      unit_range<kDev>(p, mt, u, m, n0, n1, q);
      const int row = m * kPairM + static_cast<int>(rank) * kBlockM + rloc;
      const int b = row >> 8;
      const int slot = row & 255;
      const CanvasParam cp = canvas_param<kDev>(p, b);
      const float inv_tau = cp.inv_tau;
      const float rinv = kFp8 ? __ldg(p.row_inv + row) : 1.0f;
      const float c2 = __fmul_rn(inv_tau, kLog2e);
      // Philox counter (v >> 2, slot | purpose << 16, k, b): the row's constants
      const PhiloxRow pr = slot_counter<!kFp8>(static_cast<uint32_t>(slot) | (kPurposeGumbel << 16),
                                               static_cast<uint32_t>(cp.k), static_cast<uint32_t>(b), p.rk0, p.rk1);
      Partial pt;
      partial_init(pt);
      Screen sc;
      screen_reset(sc);
      uint32_t grec = __ldcg(p.row_rec + row);
      float published = -FLT_MAX;
      for (int n = n0; n < n1; ++n, ++tile) {
        const int acc = tile & 1;
        const uint32_t acc_phase = (tile >> 1) & 1;
        if (ok && *s_abort) ok = false;
        if (!ok) continue;
        if (!mma_quarter) {
          // the words of the next tile (this unit's next, or the next unit's first)
          int mn = m, nn = n + 1;
          bool more = nn < n1;
          if (!more && u + npairs < units) {
            int n1n, qn;
            unit_range<kDev>(p, mt, u + npairs, mn, nn, n1n, qn);
            more = true;
          }
          if (more && !produce_words(tile + 1, mn, nn)) {
            ok = false;
            continue;
          }
        } else if (!mbar_wait_bounded(wfull_bar(tile & 1), (tile >> 1) & 1, p.wait_ns)) {
          latch_error(p.err, kErrWaitEpilogue);
          *s_abort = 1;
          ok = false;
          continue;
        }
        const uint32_t* wsrc = sWmax + (tile & 1) * (kTileGroups * 32) + cg * 8 * 32 + lane;
        if (!mbar_wait_bounded(tfull_bar(acc), acc_phase, p.wait_ns)) {
          latch_error(p.err, kErrWaitEpilogue);
          *s_abort = 1;
          ok = false;
          continue;
        }
        tc_fence_after();
        // 8 groups of 8 columns; the TMEM load of group g+1 is in flight
        // while group g is processed
        constexpr int kGroups = kBlockN / kColGroups / 8;
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                               static_cast<uint32_t>(acc * kBlockN + cg * (kBlockN / kColGroups));
        const int vbase = n * kBlockN + cg * (kBlockN / kColGroups);
        // best key this row has reached so far: in this CTA's column groups
        // (shared memory) and in every CTA (the global record, read one tile
        // ahead to hide its latency); stale values are lower, hence safe
        const float thr = fmaxf(fmaxf(fmaxf(sRec[0 * kBlockM + rloc], sRec[1 * kBlockM + rloc]),
                                      fmaxf(sRec[2 * kBlockM + rloc], sRec[3 * kBlockM + rloc])),
                                key_order_dec(grec));
        screen_limit(sc, thr);
        grec = __ldcg(p.row_rec + row);
        uint32_t ra[8], rb[8];
        float blk_ref = 0.f;  // self-conditioning: this tile's 64-entry block reference
        __syncwarp();
        tmem_load8_issue(tbase, ra);
        tmem_load8_wait(ra);
#pragma unroll 1
        for (int g = 0; g < kGroups; g += 2) {
          tmem_load8_issue(tbase + 8 * (g + 1), rb);
          epi_group<kFp8, kProbs>(ra, vbase + 8 * g, row, rinv, inv_tau, c2, pr, thr, mma_quarter,
                          mma_quarter ? wsrc[g * 32] : 0u, p, pt, sc, blk_ref);
          tmem_load8_wait(rb);
          if (g + 2 < kGroups) tmem_load8_issue(tbase + 8 * (g + 2), ra);
          epi_group<kFp8, kProbs>(rb, vbase + 8 * (g + 1), row, rinv, inv_tau, c2, pr, thr, mma_quarter,
                          mma_quarter ? wsrc[(g + 1) * 32] : 0u, p, pt, sc, blk_ref);
          tmem_load8_wait(ra);
          __syncwarp();
        }
        sRec[cg * kBlockM + rloc] = sc.K1a;
        if (sc.K1a > published) {
          atomicMax(p.row_rec + row, key_order_enc(sc.K1a));
          published = sc.K1a;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0)
            mbar_arrive(tempty_bar(acc));
          else
            mbar_arrive_remote(mapa_shared(tempty_bar(acc), 0));
          if (mma_quarter) mbar_arrive(wempty_bar(tile & 1));  // its words are consumed
        }
      }
      if (ok) screen_flush(sc, pt, inv_tau);
      // ---- merge the column groups' partials of each row in the CTA, then
      // write one record per (row, unit): planes of [R][Q]
      if (cg != 0) {
        float* d = sPart + (cg * kPartialFields) * kBlockM + rloc;
        d[0 * kBlockM] = pt.m2;
        d[1 * kBlockM] = pt.Sp;
        d[2 * kBlockM] = pt.T2;
        d[3 * kBlockM] = pt.zmax;
        d[4 * kBlockM] = __int_as_float(pt.zarg);
        d[5 * kBlockM] = pt.gkey;
        d[6 * kBlockM] = __int_as_float(pt.garg);
      }
      epilogue_sync();
      if (cg == 0 && ok) {
#pragma unroll 1
        for (int g2 = 1; g2 < kColGroups; ++g2) {
          const float* s2 = sPart + (g2 * kPartialFields) * kBlockM + rloc;
          Partial o;
          o.m2 = s2[0 * kBlockM];
          o.Sp = s2[1 * kBlockM];
          o.T2 = s2[2 * kBlockM];
          o.zmax = s2[3 * kBlockM];
          o.zarg = __float_as_int(s2[4 * kBlockM]);
          o.gkey = s2[5 * kBlockM];
          o.garg = __float_as_int(s2[6 * kBlockM]);
          partial_merge(pt, o);
        }
        const size_t plane = static_cast<size_t>(p.R) * sp.Q;
        const size_t idx = static_cast<size_t>(row) * sp.Q + q;
        float* part = p.part;
        part[0 * plane + idx] = pt.m2;
        part[1 * plane + idx] = pt.Sp;
        part[2 * plane + idx] = pt.T2;
        part[3 * plane + idx] = pt.zmax;
        part[4 * plane + idx] = __int_as_float(pt.zarg);
        part[5 * plane + idx] = pt.gkey;
        part[6 * plane + idx] = __int_as_float(pt.garg);
      }
      // the next unit may cover other rows: its records start afresh (no
      // epilogue warp reads them between the two barriers)
      sRec[cg * kBlockM + rloc] = -FLT_MAX;
      epilogue_sync();
    }
  }

  // Let the dependent merge kernel launch; it waits (griddepcontrol.wait)
  // for this grid's completion before reading the partial records.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // Both CTAs stay resident until the pair is done: the leader's MMAs read
  // the peer's shared memory and the peer arrives on the leader's barriers.
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, 2 * kBlockN);
  }
}

// Launch set-up of one head variant on the current device: allow its
// dynamic shared memory, then count the CTA pairs that fit at once.
template <bool kFp8, bool kProbs, bool kDev>
bool setup_on_current_device(int* pairs) {
  constexpr int kSmem = HeadCfg<kFp8>::kSmemBytes;
  if (cudaFuncSetAttribute(head_sampler_kernel<kFp8, kProbs, kDev>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
      cudaSuccess)
    return false;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kHeadThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, head_sampler_kernel<kFp8, kProbs, kDev>, &cfg) != cudaSuccess || n < 1)
    return false;
  *pairs = n;
  return true;
}

// Co-resident CTA pairs of a head variant on the current device (-1 if it
// cannot run there), set up once per device.
template <bool kFp8, bool kProbs, bool kDev>
int max_pairs_of() {
  static PerDevice<int> cache;
  int dev = -1, pairs = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (!cache.get(dev, [](int* v) { return setup_on_current_device<kFp8, kProbs, kDev>(v); }, &pairs)) return -1;
  return pairs;
}

// The sampler instances decide the work split; the self-conditioning
// instances must fit the same number of pairs (checked at launch).
int head_max_pairs(bool fp8) { return fp8 ? max_pairs_of<true, false, false>() : max_pairs_of<false, false, false>(); }

HeadSplit head_split(int R, int V, int d, int max_pairs, int kblock, int q_cap) {
  HeadSplit s;
  s.MT = R / kPairM;
  s.NT = V / kBlockN;
  s.KB = (d + kblock - 1) / kblock;
  const long long quads = static_cast<long long>(s.MT) * (s.NT / 4);
  const long long octs = static_cast<long long>(s.MT) * (s.NT / 8);
  const long long hexs = static_cast<long long>(s.MT) * (s.NT / 16);
  // The longest units that still give every pair at least 8: fewer unit ends
  // (each merges the column groups' records and meets two named barriers).
  // Measured at B = 32: units of 8 tiles 1.2 % faster than 4, 16 another 0.9 %.
  if (s.NT % 16 == 0 && hexs >= 8LL * max_pairs) {
    s.Q = s.NT / 16;
  } else if (s.NT % 8 == 0 && octs >= 8LL * max_pairs) {
    s.Q = s.NT / 8;
  } else if (s.NT % 4 == 0 && quads >= 8LL * max_pairs) {
    s.Q = s.NT / 4;  // units of 4 vocabulary tiles, many per pair
  } else {
    int q = max_pairs / s.MT;
    if (q < 1) q = 1;
    if (q > s.NT) q = s.NT;
    s.Q = q;  // about one unit per pair
  }
  if (s.Q > q_cap) s.Q = q_cap;
  s.units = s.MT * s.Q;
  s.pairs = s.units < max_pairs ? s.units : max_pairs;
  s.grid = 2 * s.pairs;
  return s;
}

cudaError_t launch_head(bool fp8, const CUtensorMap& tmA, const CUtensorMap& tmA2, const CUtensorMap& tmB,
                        const HeadParams& p, cudaStream_t stream, bool pdl) {
  const bool probs = p.ptilde != nullptr;
  const bool dev = p.cp_dev != nullptr;
  if (probs && dev) return cudaErrorInvalidValue;  // no instance writes the signal inside the device loop
  int fit;
  if (probs)
    fit = fp8 ? max_pairs_of<true, true, false>() : max_pairs_of<false, true, false>();
  else if (dev)
    fit = fp8 ? max_pairs_of<true, false, true>() : max_pairs_of<false, false, true>();
  else
    fit = head_max_pairs(fp8);
  if (fit < p.split.grid / 2) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.split.grid, 1, 1);
  cfg.blockDim = dim3(kHeadThreads, 1, 1);
  cfg.dynamicSmemBytes = fp8 ? HeadCfg<true>::kSmemBytes : HeadCfg<false>::kSmemBytes;
  cfg.stream = stream;
  // programmatic dependent launch: the set-up overlaps the preceding
  // kernel's tail; griddepcontrol.wait in the kernel orders the data
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (fp8) {
    if (probs) return cudaLaunchKernelEx(&cfg, head_sampler_kernel<true, true, false>, tmA, tmA2, tmB, p);
    if (dev) return cudaLaunchKernelEx(&cfg, head_sampler_kernel<true, false, true>, tmA, tmA2, tmB, p);
    return cudaLaunchKernelEx(&cfg, head_sampler_kernel<true, false, false>, tmA, tmA2, tmB, p);
  }
  if (probs) return cudaLaunchKernelEx(&cfg, head_sampler_kernel<false, true, false>, tmA, tmA2, tmB, p);
  if (dev) return cudaLaunchKernelEx(&cfg, head_sampler_kernel<false, false, true>, tmA, tmA2, tmB, p);
  return cudaLaunchKernelEx(&cfg, head_sampler_kernel<false, false, false>, tmA, tmA2, tmB, p);
}

}  // namespace dg
