// hidden_split.cu -- h (bf16) -> two E4M3 terms for the FP8-embedder head.
//
// The FP8 head multiplies E4M3 operands on the tensor cores
// (tcgen05 kind::f8f6f4).  To keep h at bf16 precision, each row r of h is
// scaled by a power of two 2^k_r, chosen as the largest with
// max_k |h[r, k]| * 2^k_r <= 448 (the largest E4M3 value), and split:
//   x  = h * 2^k_r                      (exact in float32)
//   h1 = E4M3(x), h2 = E4M3(x - h1)     (round to nearest even)
// A bf16 value has 8 significant bits; h1 keeps the leading 4 and the
// remainder x - h1 fits the 4 of h2, so h1 + h2 = x exactly whenever
// |x| >= 2^-2 (the remainder's last bit is then >= 2^-9, the smallest
// E4M3 step).  Below that the sum is within 2^-10 of x.  The head then
// forms z = (acc * s_v) * 2^-k_r; rinv[r] = 2^-k_r.  k_r is kept within
// [-126, 126].  A row holding a non-finite value latches kErrHiddenRange
// (reported as DG_ERR_VALUE) and leaves the step's results undefined.
#include <cuda_fp8.h>

#include "dg_device.cuh"
#include "dg_internal.h"

namespace dg {

namespace {

constexpr int kSplitWarps = 8;

// Power-of-two exponent k with amax * 2^k <= 448 < amax * 2^(k+1).
DG_DEV int split_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  const uint32_t bits = __float_as_uint(amax);
  const int e = static_cast<int>((bits >> 23) & 0xFF);
  if (e == 0) return 126;                                  // subnormal row maximum
  // amax = m * 2^(e-127), m in [1, 2); 448 = 1.75 * 2^8
  const uint32_t mant = bits & 0x7FFFFFu;
  int k = 8 - (e - 127);
  if (mant > 0x600000u) k -= 1;                            // m > 1.75
  return k < -126 ? -126 : (k > 126 ? 126 : k);
}

DG_DEV float pow2f(int k) { return __uint_as_float(static_cast<uint32_t>(k + 127) << 23); }

// Two float32 values -> their E4M3 codes and the codes of the remainders.
DG_DEV void split2(float a, float b, uint16_t& hi, uint16_t& lo) {
  const __nv_fp8x2_storage_t q1 = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __half2_raw r1 = __nv_cvt_fp8x2_to_halfraw2(q1, __NV_E4M3);
  const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&r1));
  const __nv_fp8x2_storage_t q2 =
      __nv_cvt_float2_to_fp8x2(make_float2(a - f1.x, b - f1.y), __NV_SATFINITE, __NV_E4M3);
  hi = q1;
  lo = q2;
}

__global__ void __launch_bounds__(kSplitWarps * 32) hidden_split_kernel(const uint4* __restrict__ h,
                                                                     uint2* __restrict__ h1, uint2* __restrict__ h2,
                                                                     float* __restrict__ rinv, int R, int d8,
                                                                     uint32_t* err) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kSplitWarps + (threadIdx.x >> 5);
  if (r >= R) return;
  const uint4* hr = h + static_cast<size_t>(r) * d8;
  float amax = 0.0f;
  bool bad = false;
  for (int i = lane; i < d8; i += 32) {
    const uint4 x = __ldg(hr + i);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
      bad |= !isfinite(lo) || !isfinite(hi);
      amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  bad = __any_sync(0xFFFFFFFFu, bad);
  const int k = bad ? 0 : split_exponent(amax);
  const float c = pow2f(k);
  if (lane == 0) {
    rinv[r] = pow2f(-k);
    if (bad) atomicOr(err, kErrHiddenRange);
  }
  uint2* o1 = h1 + static_cast<size_t>(r) * d8;
  uint2* o2 = h2 + static_cast<size_t>(r) * d8;
  for (int i = lane; i < d8; i += 32) {
    const uint4 x = __ldg(hr + i);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint16_t a[4], b[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16) * c, hi = __uint_as_float(w[j] & 0xFFFF0000u) * c;
      split2(lo, hi, a[j], b[j]);
    }
    o1[i] = make_uint2(static_cast<uint32_t>(a[0]) | (static_cast<uint32_t>(a[1]) << 16),
                       static_cast<uint32_t>(a[2]) | (static_cast<uint32_t>(a[3]) << 16));
    o2[i] = make_uint2(static_cast<uint32_t>(b[0]) | (static_cast<uint32_t>(b[1]) << 16),
                       static_cast<uint32_t>(b[2]) | (static_cast<uint32_t>(b[3]) << 16));
  }
}

}  // namespace

cudaError_t launch_hidden_split(const void* h, uint8_t* h1, uint8_t* h2, float* rinv, int R, int d,
                                uint32_t* err, cudaStream_t stream) {
  if (R <= 0 || d <= 0) return cudaSuccess;
  const int blocks = (R + kSplitWarps - 1) / kSplitWarps;
  hidden_split_kernel<<<blocks, kSplitWarps * 32, 0, stream>>>(static_cast<const uint4*>(h),
                                                              reinterpret_cast<uint2*>(h1),
                                                              reinterpret_cast<uint2*>(h2), rinv, R, d / 8, err);
  return cudaGetLastError();
}

}  // namespace dg
