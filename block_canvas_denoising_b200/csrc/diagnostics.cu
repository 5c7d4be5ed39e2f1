// diagnostics.cu -- two small kernels behind the diagnostic entry points:
//   * a self test of the bounded mbarrier wait: it waits on a barrier that
//     nobody arrives at and must give up after `limit_ns`, latching
//     kErrSelftest, with the context left usable;
//   * a probe of the Gumbel transforms on given Philox words: the specified
//     IEEE-only g32 and the approximate lg2(E / ln 2) the screening pass uses.
#include "dg_device.cuh"
#include "dg_internal.h"

namespace dg {

__global__ void wait_selftest_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbarrier_init();
    // phase 0 never completes: nobody arrives
    if (!mbar_wait_bounded(smem_u32(&bar), 0u, limit_ns)) atomicOr(err, kErrSelftest);
  }
}

__global__ void gumbel_probe_kernel(const uint32_t* words, int n, float* g_exact, float* lg2e) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t r = words[i];
  g_exact[i] = gumbel_exact(r);
  lg2e[i] = lg2_exp1_approx(r);
}

cudaError_t launch_wait_selftest(uint32_t* err, uint64_t limit_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_gumbel_probe(const uint32_t* words, int n, float* g_exact, float* lg2e_approx,
                                cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  gumbel_probe_kernel<<<(n + 255) / 256, 256, 0, stream>>>(words, n, g_exact, lg2e_approx);
  return cudaGetLastError();
}

}  // namespace dg
