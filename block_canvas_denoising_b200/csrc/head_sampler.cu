// head_sampler.cu -- the fused tied-LM-head + sampler kernel for sm_100a.
//
// z = h . E^T ([Report] "DiffusionGemma Technical Report", Table 1: the
// 740M embedder over the 262k vocabulary is the output head) is computed
// tile by tile on the 5th-generation tensor cores and never leaves the SM:
// each 128 x 256 float32 accumulator tile lives in tensor memory (TMEM) and
// is reduced in place by the epilogue warps into per-row partials of
//   * the online softmax of x = z / tau_k in base 2: m2 = max x log2(e),
//     S = sum 2^(x log2 e - m2), T2 = sum (x log2 e - m2) 2^(...)  -- the
//     entropy of the tempered distribution follows as ln S - ln2 T2 / S
//     ([Docs] "DiffusionGemma", Recommended serving configuration: entropy
//     drives token selection and adaptive stopping; temperature schedule);
//   * the argmax of z (the prediction compared across steps for stopping);
//   * the Gumbel-max draw argmax_v fl(fl(z_v / tau) + g32(u_v)) with u_v
//     from Philox4x32-10 counter (v >> 2, slot, k, b), lane v & 3.
//
// Warp roles (320 threads, one CTA per SM, persistent):
//   warp 0      TMA producer: h and E tiles -> 4-stage shared-memory ring.
//   warp 1      TMEM allocator and MMA issuer (tcgen05.mma, 128x256x16 bf16).
//   warps 2..9  epilogue: warp w reads TMEM lane quarter w % 4 and column
//               half (w - 2) / 4 of each tile; two accumulators alternate
//               so the epilogue of tile t overlaps the MMAs of tile t + 1.
#include <float.h>
#include <limits.h>

#include "dg_device.cuh"
#include "dg_internal.h"

namespace dg {

namespace {

struct Partial {
  float m2, S, T2;  // base-2 online softmax of x = z * inv_tau
  float zmax;       // argmax of z
  int zarg;
  float gkey;       // best specified Gumbel key so far
  int garg;
};

DG_DEV void unit_range(const HeadSplit& sp, int u, int& m, int& n0, int& n1, int& q) {
  q = u / sp.MT;
  m = u - q * sp.MT;
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

// One 32-column chunk of one row: z[0..31] are logits v0 .. v0+31.
DG_DEV void process_chunk(const float (&z)[32], int v0, float inv_tau, float c2, uint32_t ctr1,
                          uint32_t ctr2, uint32_t ctr3, uint32_t k0, uint32_t k1, Partial& pt) {
  // ---- argmax of z (ties to the lower index; chunks arrive in increasing v)
  float cmax = z[0];
#pragma unroll
  for (int j = 1; j < 32; ++j) cmax = fmaxf(cmax, z[j]);
  if (cmax > pt.zmax) {
    int jj = 0;
#pragma unroll
    for (int j = 31; j >= 0; --j) jj = (z[j] == cmax) ? j : jj;
    pt.zmax = cmax;
    pt.zarg = v0 + jj;
  }

  // ---- online softmax partial, base 2
  const float cm2 = cmax * c2;
  if (cm2 > pt.m2) {
    const float delta = pt.m2 - cm2;
    const float sc = ex2_approx(delta);
    pt.T2 = (pt.T2 + delta * pt.S) * sc;
    pt.S = pt.S * sc;
    pt.m2 = cm2;
  }
  {
    float s0 = 0.f, s1 = 0.f, t0 = 0.f, t1 = 0.f;
    const float nm = -pt.m2;
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const float d0 = fmaf(z[j], c2, nm);
      const float d1 = fmaf(z[j + 1], c2, nm);
      const float e0 = ex2_approx(d0);
      const float e1 = ex2_approx(d1);
      s0 += e0;
      s1 += e1;
      t0 = fmaf(d0, e0, t0);
      t1 = fmaf(d1, e1, t1);
    }
    pt.S += s0 + s1;
    pt.T2 += t0 + t1;
  }

  // ---- Gumbel-max: screen with the approximate key, confirm exactly
  const uint32_t cbase = static_cast<uint32_t>(v0) >> 2;
  float K1 = -FLT_MAX, K2 = -FLT_MAX, zK1 = 0.f;
  int j1 = 0;
#pragma unroll
  for (int q4 = 0; q4 < 8; ++q4) {
    uint32_t r[4];
    philox4x32_10(cbase + q4, ctr1, ctr2, ctr3, k0, k1, r);
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      const int j = 4 * q4 + l;
      const float x = __fmul_rn(z[j], inv_tau);
      const float ka = __fmaf_rn(lg2_exp1_approx(r[l]), -kLn2, x);
      const bool p = ka > K1;
      K2 = fmaxf(K2, p ? K1 : ka);
      zK1 = p ? z[j] : zK1;
      j1 = p ? j : j1;
      K1 = p ? ka : K1;
    }
  }
  // Any specified key differs from its approximate key by at most
  // kGumbelApproxErr plus the roundings of the two keys; eps is twice that
  // bound with room to spare.
  const float eps = 2.0f * kGumbelApproxErr + (fabsf(K1) + 64.0f) * 9.5367431640625e-07f;
  if (K1 >= pt.gkey - eps) {
    if (K2 >= K1 - eps) {
      // near-tie inside the chunk: confirm every element
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        uint32_t r[4];
        philox4x32_10(cbase + q4, ctr1, ctr2, ctr3, k0, k1, r);
#pragma unroll
        for (int l = 0; l < 4; ++l) gumbel_update(pt, key_exact(z[4 * q4 + l], inv_tau, r[l]), v0 + 4 * q4 + l);
      }
    } else {
      uint32_t r[4];
      philox4x32_10(cbase + (static_cast<uint32_t>(j1) >> 2), ctr1, ctr2, ctr3, k0, k1, r);
      const int l = j1 & 3;
      const uint32_t rw = (l == 0) ? r[0] : (l == 1) ? r[1] : (l == 2) ? r[2] : r[3];
      gumbel_update(pt, key_exact(zK1, inv_tau, rw), v0 + j1);
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(kHeadThreads, 1)
head_sampler_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ HeadParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kAStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kStages * kBStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const HeadSplit& sp = p.split;

  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[kStages + s]); };
  auto tfull_bar = [&](int a) { return smem_u32(&bars[2 * kStages + a]); };
  auto tempty_bar = [&](int a) { return smem_u32(&bars[2 * kStages + 2 + a]); };

  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), kEpiWarps);
    }
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 2 * kBlockN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_h = policy_evict_last();   // h is re-read by every unit
      const uint64_t pol_e = policy_evict_first();  // E streams through once
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < sp.units && ok; u += gridDim.x) {
        int m, n0, n1, q;
        unit_range(sp, u, m, n0, n1, q);
        for (int n = n0; n < n1 && ok; ++n) {
          for (int kb = 0; kb < sp.KB; ++kb) {
            if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, p.wait_ns)) {
              latch_error(p.err, kErrWaitTmaProducer);
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(full_bar(stage), kAStageBytes + kBStageBytes);
            tma_load_2d(smem_u32(sA + stage * kAStageBytes), &tmA, full_bar(stage), kb * kBlockK,
                        m * kBlockM, pol_h);
            tma_load_2d(smem_u32(sB + stage * kBStageBytes), &tmB, full_bar(stage), kb * kBlockK,
                        n * kBlockN, pol_e);
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc_bf16_f32(kBlockM, kBlockN);
      int stage = 0;
      uint32_t phase = 0;
      int tile = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < sp.units && ok; u += gridDim.x) {
        int m, n0, n1, q;
        unit_range(sp, u, m, n0, n1, q);
        for (int n = n0; n < n1 && ok; ++n, ++tile) {
          const int acc = tile & 1;
          const uint32_t acc_phase = (tile >> 1) & 1;
          if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, p.wait_ns)) {
            latch_error(p.err, kErrWaitMmaAcc);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBlockN);
          for (int kb = 0; kb < sp.KB; ++kb) {
            if (!mbar_wait_bounded(full_bar(stage), phase, p.wait_ns)) {
              latch_error(p.err, kErrWaitMmaFull);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t adesc = smem_desc_k_sw128(smem_u32(sA + stage * kAStageBytes));
            const uint64_t bdesc = smem_desc_k_sw128(smem_u32(sB + stage * kBStageBytes));
#pragma unroll
            for (int k16 = 0; k16 < kBlockK / 16; ++k16) {
              // advance 16 bf16 = 32 B along K inside the swizzled rows
              tc_mma_bf16(d_tmem, adesc + 2u * k16, bdesc + 2u * k16, idesc,
                          (kb > 0 || k16 > 0) ? 1u : 0u);
            }
            tc_commit(empty_bar(stage));
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (ok) tc_commit(tfull_bar(acc));
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int cg = ew >> 2;        // column half of the tile
    const uint32_t k0 = p.seed_lo, k1 = p.seed_hi;
    const int P = 2 * sp.Q;
    int tile = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < sp.units && ok; u += gridDim.x) {
      int m, n0, n1, q;
      unit_range(sp, u, m, n0, n1, q);
      const int row = m * kBlockM + quarter * 32 + lane;
      const int b = row >> 8;
      const int slot = row & 255;
      const CanvasParam cp = p.cp[b];
      const float inv_tau = cp.inv_tau;
      const float c2 = __fmul_rn(inv_tau, kLog2e);
      const uint32_t ctr1 = static_cast<uint32_t>(slot) | (kPurposeGumbel << 16);
      const uint32_t ctr2 = static_cast<uint32_t>(cp.k);
      const uint32_t ctr3 = static_cast<uint32_t>(b);
      Partial pt;
      pt.m2 = -1.0e30f;
      pt.S = 0.f;
      pt.T2 = 0.f;
      pt.zmax = -FLT_MAX;
      pt.zarg = INT_MAX;
      pt.gkey = -FLT_MAX;
      pt.garg = INT_MAX;
      for (int n = n0; n < n1; ++n, ++tile) {
        const int acc = tile & 1;
        const uint32_t acc_phase = (tile >> 1) & 1;
        if (!mbar_wait_bounded(tfull_bar(acc), acc_phase, p.wait_ns)) {
          latch_error(p.err, kErrWaitEpilogue);
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < kBlockN / 2 / 32; ++c) {
          const int col = acc * kBlockN + cg * (kBlockN / 2) + c * 32;
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + col;
          float z[32];
          __syncwarp();
          tmem_load_32cols(taddr, z);
          const int v0 = n * kBlockN + cg * (kBlockN / 2) + c * 32;
          if (p.e_scale != nullptr) {
            const float4* sc = reinterpret_cast<const float4*>(p.e_scale + v0);
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 s4 = __ldg(sc + j4);
              z[4 * j4 + 0] = __fmul_rn(z[4 * j4 + 0], s4.x);
              z[4 * j4 + 1] = __fmul_rn(z[4 * j4 + 1], s4.y);
              z[4 * j4 + 2] = __fmul_rn(z[4 * j4 + 2], s4.z);
              z[4 * j4 + 3] = __fmul_rn(z[4 * j4 + 3], s4.w);
            }
          }
          if (p.logits_out != nullptr) {
            float4* dst = reinterpret_cast<float4*>(p.logits_out + static_cast<size_t>(row) * p.V + v0);
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4)
              dst[j4] = make_float4(z[4 * j4], z[4 * j4 + 1], z[4 * j4 + 2], z[4 * j4 + 3]);
          }
          process_chunk(z, v0, inv_tau, c2, ctr1, ctr2, ctr3, k0, k1, pt);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(acc));
      }
      if (!ok) break;
      // one partial record per (row, unit, column half), planes of [P][R]
      const size_t plane = static_cast<size_t>(P) * p.R;
      const size_t idx = static_cast<size_t>(2 * q + cg) * p.R + row;
      float* part = p.part;
      part[0 * plane + idx] = pt.m2;
      part[1 * plane + idx] = pt.S;
      part[2 * plane + idx] = pt.T2;
      part[3 * plane + idx] = pt.zmax;
      part[4 * plane + idx] = __int_as_float(pt.zarg);
      part[5 * plane + idx] = pt.gkey;
      part[6 * plane + idx] = __int_as_float(pt.garg);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, 2 * kBlockN);
  }
}

HeadSplit head_split(int R, int V, int d, int num_sms) {
  HeadSplit s;
  s.MT = R / kBlockM;
  s.NT = V / kBlockN;
  s.KB = d / kBlockK;
  const long long quads = static_cast<long long>(s.MT) * (s.NT / 4);
  if (s.NT % 4 == 0 && quads >= 8LL * num_sms) {
    s.Q = s.NT / 4;  // units of 4 vocabulary tiles, many per CTA
  } else {
    int q = num_sms / s.MT;
    if (q < 1) q = 1;
    if (q > s.NT) q = s.NT;
    s.Q = q;  // about one unit per CTA
  }
  s.units = s.MT * s.Q;
  s.grid = s.units < num_sms ? s.units : num_sms;
  return s;
}

cudaError_t launch_head(const CUtensorMap& tmA, const CUtensorMap& tmB, const HeadParams& p,
                        cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(head_sampler_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kHeadSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  head_sampler_kernel<<<p.split.grid, kHeadThreads, kHeadSmemBytes, stream>>>(tmA, tmB, p);
  return cudaGetLastError();
}

}  // namespace dg
