// selfcond.cu -- the self-conditioning signal of a step on the device.
//
// "DiffusionGemma Technical Report", Table 1: the model carries a 7.8M-
// parameter MLP for self-conditioning (about d^2 at d = 2816: one d x d
// projection of a d-wide signal); the pages do not define the signal.
// Reading taken here: the signal of slot r is the embedding expected under
// the step's tempered distribution,
//     s[r] = sum_v p[r, v] E[v],   p[r] = softmax(z[r] / tau_k),
// a second contraction over the whole vocabulary against the embedder.
//
// At d = 2816 the output (B*256 x d float32) does not fit in tensor memory
// next to the logits, so the signal is formed in four passes:
//   1. the fused head (head_sampler.cu), asked for it, also writes block-
//      scaled probabilities: Pt[r, v] = bf16(2^(z c2 - ref)) for each block
//      of 64 vocabulary entries with its own reference ref[r, block] (the
//      running maximum when the block starts), ref to `pref` ([V / 64][R]);
//   2. normalise (here): P[r, v] = bf16(Pt[r, v] 2^(ref - m2_r) / S_r) in
//      place, with the row's final maximum m2_r and normaliser S_r from the
//      merge (and the FP8 embedder's row scale s_v folded in);
//   3. split-K GEMM (here, tcgen05 pairs): partial[q] = P[:, K_q] . Et[:, K_q]^T
//      over vocabulary slices K_q, with Et = E^T [d, V] bf16 made once per
//      embedder (dg_embedder_transpose), so both operands are K-major;
//   4. reduce (here): s = sum_q partial[q] in a fixed order.
// The normalisation stays a pass of its own (one read and one write of P).
// Folding it into the GEMM -- warps rescaling each landed A tile in shared
// memory before the MMA reads it -- adds a shared-memory read and write of
// every tile to the TMA write and the MMA read, which already use the SM's
// shared-memory bandwidth at the MMA rate; measured, that GEMM ran about
// three times longer than this pass and the plain GEMM together.
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <string.h>

#include "dg_device.cuh"
#include "dg_internal.h"
#include "per_device.h"

namespace dg {

namespace {

// ---------------------------------------------------------------------------
// split-K GEMM: C[m, n] = sum_k A[m, k] B[n, k], A = P [R, V], B = Et [d, V]
// ---------------------------------------------------------------------------
constexpr int kGemmStages = 6;
constexpr int kGemmEpiWarps = 8;                       // 4 lane quarters x 2 column halves
constexpr int kGemmThreads = (2 + kGemmEpiWarps) * 32;
constexpr int kGemmSmem = kGemmStages * 2 * kTileBytes + 1024 + 256;
static_assert(kGemmSmem <= 232448, "split-K GEMM exceeds 227 KB of shared memory");

struct GemmParams {
  int32_t R, d, V;
  int32_t MT, NT, KB, Sk;  // row tiles, d tiles, K stages, K slices
  int32_t units;           // MT * NT * Sk
  float* part;             // [Sk][R][d]
  uint32_t* err;
  uint64_t wait_ns;
};

// Unit u: d tile n (fastest, so pairs running at once share the P slice in
// L2), row tile m, K slice q covering stages [k0, k1).
DG_DEV void gemm_unit(const GemmParams& p, int u, int& m, int& n, int& q, int& k0, int& k1) {
  n = u % p.NT;
  const int rest = u / p.NT;
  m = rest % p.MT;
  q = rest / p.MT;
  k0 = static_cast<int>((static_cast<int64_t>(q) * p.KB) / p.Sk);
  k1 = static_cast<int>((static_cast<int64_t>(q + 1) * p.KB) / p.Sk);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
selfcond_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kGemmStages * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kGemmStages * kTileBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kGemmStages + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[kGemmStages + s]); };
  auto tfull_bar = [&](int a) { return smem_u32(&bars[2 * kGemmStages + a]); };
  auto tempty_bar = [&](int a) { return smem_u32(&bars[2 * kGemmStages + 2 + a]); };

  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * kGemmEpiWarps);
    }
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(smem_u32(tmem_slot), 2 * kBlockN);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 1) {
    // ---- producer: this CTA's 128 rows of P and 128 rows of Et per stage
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();   // slices are shared by the pairs running at once
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = pair; u < p.units && ok; u += npairs) {
        int m, n, q, k0, k1;
        gemm_unit(p, u, m, n, q, k0, k1);
        for (int kb = k0; kb < k1; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, p.wait_ns)) {
            atomicOr(p.err, kErrWaitTmaProducer);
            ok = false;
            break;
          }
          const uint32_t fb = full_bar(stage);
          if (rank == 0) mbar_arrive_expect_tx(fb, 4 * kTileBytes);
          const uint32_t fb_leader = mapa_shared(fb, 0);
          const int kx = kb * kBlockK;
          tma_load_2d_pair(smem_u32(sA + stage * kTileBytes), &tmA, fb_leader, kx,
                           m * kPairM + static_cast<int>(rank) * kBlockM, pol);
          tma_load_2d_pair(smem_u32(sB + stage * kTileBytes), &tmB, fb_leader, kx,
                           n * kBlockN + static_cast<int>(rank) * kHalfN, pol);
          if (++stage == kGemmStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      for (int i = 0; i < kGemmStages && ok; ++i) {  // every stage released before exit
        if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, p.wait_ns)) {
          atomicOr(p.err, kErrWaitTmaProducer);
          ok = false;
        }
        if (++stage == kGemmStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 0) {
    // ---- MMA issuer (leader)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = instr_desc_bf16_f32(kPairM, kBlockN);
      const uint64_t a0 = smem_desc_k_sw128(smem_u32(sA));
      const uint64_t b0 = smem_desc_k_sw128(smem_u32(sB));
      const uint32_t a_hi = static_cast<uint32_t>(a0 >> 32), b_hi = static_cast<uint32_t>(b0 >> 32);
      constexpr uint32_t kStep = kTileBytes >> 4;
      int stage = 0;
      uint32_t phase = 0;
      int tile = 0;
      bool ok = true;
      for (int u = pair; u < p.units && ok; u += npairs, ++tile) {
        int m, n, q, k0, k1;
        gemm_unit(p, u, m, n, q, k0, k1);
        const int acc = tile & 1;
        if (!mbar_wait_bounded<true>(tempty_bar(acc), ((tile >> 1) & 1) ^ 1u, p.wait_ns)) {
          atomicOr(p.err, kErrWaitMmaAcc);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBlockN);
        for (int kb = k0; kb < k1; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, p.wait_ns)) {
            atomicOr(p.err, kErrWaitMmaFull);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_lo = static_cast<uint32_t>(a0) + static_cast<uint32_t>(stage) * kStep;
          const uint32_t b_lo = static_cast<uint32_t>(b0) + static_cast<uint32_t>(stage) * kStep;
#pragma unroll
          for (int k32 = 0; k32 < 4; ++k32)
            tc_mma_pair_lohi<false>(d_tmem, a_lo + 2u * k32, a_hi, b_lo + 2u * k32, b_hi, idesc,
                                    (kb > k0 || k32 > 0) ? 1u : 0u);
          tc_commit_pair_mc(empty_bar(stage), 0x3);
          if (++stage == kGemmStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit_pair_mc(tfull_bar(acc), 0x3);
      }
    }
  } else {
    // ---- epilogue: lane quarter warp % 4, column half (warp - 2) / 4
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    int tile = 0;
    bool ok = true;
    for (int u = pair; u < p.units; u += npairs, ++tile) {
      int m, n, q, k0, k1;
      gemm_unit(p, u, m, n, q, k0, k1);
      const int acc = tile & 1;
      if (ok && !mbar_wait_bounded(tfull_bar(acc), (tile >> 1) & 1, p.wait_ns)) {
        atomicOr(p.err, kErrWaitEpilogue);
        ok = false;
      }
      if (!ok) continue;
      tc_fence_after();
      const int row = m * kPairM + static_cast<int>(rank) * kBlockM + quarter * 32 + lane;
      float* dst = p.part + (static_cast<size_t>(q) * p.R + row) * p.d;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * kBlockN + half * (kBlockN / 2));
#pragma unroll 1
      for (int c = 0; c < kBlockN / 2; c += 8) {
        uint32_t r[8];
        tmem_load8_issue(tbase + c, r);
        tmem_load8_wait(r);
        const int col = n * kBlockN + half * (kBlockN / 2) + c;
        if (col < p.d) {  // d is a multiple of 64: a group of 8 is all in or all out
          float4* o = reinterpret_cast<float4*>(dst + col);
          o[0] = make_float4(__uint_as_float(r[0]), __uint_as_float(r[1]), __uint_as_float(r[2]), __uint_as_float(r[3]));
          o[1] = make_float4(__uint_as_float(r[4]), __uint_as_float(r[5]), __uint_as_float(r[6]), __uint_as_float(r[7]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(tempty_bar(acc));
        else
          mbar_arrive_remote(mapa_shared(tempty_bar(acc), 0));
      }
    }
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, 2 * kBlockN);
  }
}

bool gemm_setup(int* pairs) {
  if (cudaFuncSetAttribute(selfcond_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem) !=
      cudaSuccess)
    return false;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = kGemmSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, selfcond_gemm_kernel, &cfg) != cudaSuccess || n < 1) return false;
  *pairs = n;
  return true;
}

// ---------------------------------------------------------------------------
// normalise the block-scaled probabilities in place
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) selfcond_normalize_kernel(uint4* __restrict__ pt, const float* __restrict__ pref,
                                                                 const float2* __restrict__ rowstat,
                                                                 const float* __restrict__ e_scale, int R, int V) {
  const int v8 = V / 8;
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<size_t>(R) * v8) return;
  const int r = static_cast<int>(i / v8);
  const int v0 = static_cast<int>(i - static_cast<size_t>(r) * v8) * 8;
  const float2 st = __ldg(rowstat + r);  // (m2, 1 / S)
  const float ref = __ldg(pref + static_cast<size_t>(v0 / 64) * R + r);  // pref is [V / 64][R]
  const float f = exp2f(ref - st.x) * st.y;
  uint4 w = pt[i];
  uint32_t* wp = &w.x;
  float sv[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) sv[j] = 1.0f;
  if (e_scale != nullptr) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(e_scale + v0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(e_scale + v0) + 1);
    sv[0] = a.x; sv[1] = a.y; sv[2] = a.z; sv[3] = a.w;
    sv[4] = b.x; sv[5] = b.y; sv[6] = b.z; sv[7] = b.w;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float lo = __uint_as_float(wp[j] << 16) * f * sv[2 * j];
    const float hi = __uint_as_float(wp[j] & 0xFFFF0000u) * f * sv[2 * j + 1];
    const __nv_bfloat162 o = __floats2bfloat162_rn(lo, hi);
    wp[j] = *reinterpret_cast<const uint32_t*>(&o);
  }
  pt[i] = w;
}

// ---------------------------------------------------------------------------
// s = sum over the K slices, in slice order
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) selfcond_reduce_kernel(const float4* __restrict__ part, float4* __restrict__ out,
                                                              size_t n4, int Sk) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  float4 a = __ldg(part + i);
  for (int q = 1; q < Sk; ++q) {
    const float4 b = __ldg(part + static_cast<size_t>(q) * n4 + i);
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
  }
  out[i] = a;
}

// ---------------------------------------------------------------------------
// Et[c, v] = E[v, c] (bf16; E4M3 codes widen to bf16 exactly), 32 x 32 tiles
// ---------------------------------------------------------------------------
template <bool kFp8>
__global__ void __launch_bounds__(256) transpose_kernel(const void* __restrict__ E, uint16_t* __restrict__ Et,
                                                        int V, int d) {
  __shared__ uint16_t tile[32][33];
  const int v0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  for (int j = ty; j < 32; j += 8) {
    const size_t idx = static_cast<size_t>(v0 + j) * d + c0 + tx;
    uint16_t b;
    if (kFp8) {
      const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<const __nv_fp8_storage_t*>(E)[idx], __NV_E4M3);
      const float f = __half2float(*reinterpret_cast<const __half*>(&hr));
      b = static_cast<uint16_t>(__float_as_uint(f) >> 16);  // exact: an E4M3 value has 4 significant bits
    } else {
      b = static_cast<const uint16_t*>(E)[idx];
    }
    tile[j][tx] = b;
  }
  __syncthreads();
  for (int j = ty; j < 32; j += 8) Et[static_cast<size_t>(c0 + j) * V + v0 + tx] = tile[tx][j];
}

bool encode_kmajor(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBlockK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int selfcond_gemm_pairs() {
  static PerDevice<int> cache;
  int dev = -1, pairs = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (!cache.get(dev, [](int* v) { return gemm_setup(v); }, &pairs)) return -1;
  return pairs;
}

int selfcond_slices(int R, int d, int V, int pairs) {
  const int MT = R / kPairM, NT = (d + kBlockN - 1) / kBlockN, KB = V / kBlockK;
  int sk = (4 * pairs) / (MT * NT);
  if (sk < 1) sk = 1;
  if (sk > KB) sk = KB;
  return sk;
}

cudaError_t launch_selfcond(const uint16_t* P, const uint16_t* Et, const float* pref, const float2* rowstat,
                            const float* e_scale, float* part, float* signal, int R, int d, int V, uint32_t* err,
                            cudaStream_t stream) {
  const int pairs = selfcond_gemm_pairs();
  if (pairs < 1) return cudaErrorInvalidConfiguration;
  // 2. normalise
  const size_t n8 = static_cast<size_t>(R) * (V / 8);
  selfcond_normalize_kernel<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<uint4*>(const_cast<uint16_t*>(P)), pref, rowstat, e_scale, R, V);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 3. split-K GEMM
  CUtensorMap tmA, tmB;
  if (!encode_kmajor(&tmA, P, V, R, kBlockM) || !encode_kmajor(&tmB, Et, V, d, kHalfN))
    return cudaErrorInvalidValue;
  GemmParams gp;
  memset(&gp, 0, sizeof(gp));
  gp.R = R;
  gp.d = d;
  gp.V = V;
  gp.MT = R / kPairM;
  gp.NT = (d + kBlockN - 1) / kBlockN;
  gp.KB = V / kBlockK;
  gp.Sk = selfcond_slices(R, d, V, pairs);
  gp.units = gp.MT * gp.NT * gp.Sk;
  gp.part = part;
  gp.err = err;
  gp.wait_ns = kDefaultWaitNs;
  const int grid = 2 * (gp.units < pairs ? gp.units : pairs);
  selfcond_gemm_kernel<<<grid, kGemmThreads, kGemmSmem, stream>>>(tmA, tmB, gp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 4. reduce
  const size_t n4 = static_cast<size_t>(R) * d / 4;
  selfcond_reduce_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(part), reinterpret_cast<float4*>(signal), n4, gp.Sk);
  return cudaGetLastError();
}

cudaError_t launch_transpose(const void* E, bool fp8, uint16_t* Et, int V, int d, cudaStream_t stream) {
  dim3 grid(V / 32, d / 32);
  if (fp8)
    transpose_kernel<true><<<grid, 256, 0, stream>>>(E, Et, V, d);
  else
    transpose_kernel<false><<<grid, 256, 0, stream>>>(E, Et, V, d);
  return cudaGetLastError();
}

}  // namespace dg
