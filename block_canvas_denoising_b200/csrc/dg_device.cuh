// dg_device.cuh -- device building blocks of the sm_100a denoising step:
// inline-PTX wrappers (mbarrier, TMA, tcgen05), Philox4x32-10, the
// IEEE-only float32 log that defines the sampler's Gumbel key, and the fast
// approximate key used to screen candidates.
#pragma once

#include <cuda.h>
#include <float.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define DG_DEV __device__ __forceinline__

namespace dg {

// ---------------------------------------------------------------------------
// status latch (shared with the host through the workspace)
// ---------------------------------------------------------------------------
enum : uint32_t {
  kErrWaitTmaProducer = 1u << 0,  // producer gave up waiting for a free stage
  kErrWaitMmaFull = 1u << 1,      // MMA issuer gave up waiting for a loaded stage
  kErrWaitMmaAcc = 1u << 2,       // MMA issuer gave up waiting for a drained accumulator
  kErrWaitEpilogue = 1u << 3,     // epilogue gave up waiting for a finished tile
  kErrSelftest = 1u << 4,         // the bounded-wait self test ran out (expected)
  kErrHiddenRange = 1u << 5,      // FP8 head: a hidden-state value is not finite
  kErrProbRange = 1u << 6,        // self-conditioning: a probability block outside its encoding's range
};
// Latched codes that report a value problem (DG_ERR_VALUE) rather than a
// bounded wait that ran out (DG_ERR_TIMEOUT).
constexpr uint32_t kErrValueMask = kErrHiddenRange | kErrProbRange;

// ---------------------------------------------------------------------------
// small PTX helpers
// ---------------------------------------------------------------------------
DG_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

DG_DEV uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

DG_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

DG_DEV void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

DG_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

DG_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

// Suspend-time hint of mbarrier.try_wait: a waiting warp sleeps until the
// phase completes or this many nanoseconds pass.  A long hint (measured:
// about 5 % fewer cycles per step than the default) keeps waiting warps
// from re-polling next to the MMA issuer.
constexpr uint32_t kTryWaitSuspendNs = 10000;

DG_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "n"(kTryWaitSuspendNs)
      : "memory");
  return ok != 0;
}

// The same test with acquire semantics at cluster scope: for barriers that
// the peer CTA's threads arrive on (release.cluster) after writing memory
// the waiter then reads.
DG_DEV bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "n"(kTryWaitSuspendNs)
      : "memory");
  return ok != 0;
}

// Wait for the phase of parity `parity` to complete, for at most `limit_ns`
// nanoseconds of %globaltimer.  Returns false if the limit ran out.
template <bool kClusterScope = false>
DG_DEV bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  auto test = [&]() {
    return kClusterScope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
  };
  if (test()) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (test()) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// 2-D tiled TMA load for a tcgen05 cta_group::2 pair: the copy lands in this
// CTA's shared memory and completes on `bar`, which may be the peer CTA's
// barrier (a shared::cluster address from mapa).  x is the inner
// (contiguous) coordinate in elements, y the row.
DG_DEV void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                             uint64_t cache_hint) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "l"(cache_hint)
      : "memory");
}

// ---------------------------------------------------------------------------
// clusters
// ---------------------------------------------------------------------------
DG_DEV uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
DG_DEV uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

DG_DEV void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier in another CTA of the cluster.
DG_DEV void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

DG_DEV void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// L2 cache-policy words for the TMA cache hint.
DG_DEV uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
DG_DEV uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor core, accumulators in tensor memory), in
// the pair form (cta_group::2): TMEM is allocated in both CTAs of the pair by
// one warp of each; the leader issues the MMA over both CTAs' operands.
// ---------------------------------------------------------------------------
DG_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
DG_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

DG_DEV void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
DG_DEV void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
DG_DEV void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Arrive once on the barrier at this shared-memory offset in every CTA of
// `cta_mask` when the pair MMAs issued so far by this thread have completed.
DG_DEV void tc_commit_pair_mc(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          bar),
      "h"(cta_mask)
      : "memory");
}

// D[tmem of both CTAs] (+)= A[smem of both] * B[smem of both]^T (M = 256
// over the pair, N split between the two CTAs' B tiles), f32 accumulate:
// kind::f16 with bf16 operands (K = 16 per instruction) or kind::f8f6f4
// with E4M3 operands (K = 32).  Each smem descriptor is given as its two
// 32-bit halves (the low half carries the start address, so stepping along
// K or to the next stage is one 32-bit add), for an issuing loop with as few
// instructions as possible.
template <bool kE4M3>
DG_DEV void tc_mma_pair_lohi(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo, uint32_t b_hi,
                             uint32_t idesc, uint32_t accumulate) {
  if (kE4M3) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "mov.b64 da, {%1, %2};\n\t"
        "mov.b64 db, {%3, %4};\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
        "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "mov.b64 da, {%1, %2};\n\t"
        "mov.b64 db, {%3, %4};\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
        "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// Shared-memory matrix descriptor of a K-major tile stored by TMA with the
// 128-byte swizzle: rows of 128 B, 8-row (1024 B) swizzle atoms stacked
// along M/N.  Fields: start address >> 4 [0,14), leading byte offset >> 4
// [16,30) (unused by swizzled K-major, set to 1), stride byte offset >> 4
// [32,46) = 1024 B between 8-row groups, descriptor version 1 at [46,48),
// base offset 0 (tiles are 1024-B aligned), swizzle mode 2 (128 B) at [61,64).
DG_DEV uint64_t smem_desc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor, kind::f16: f32 accumulator [4,6)=1, A bf16
// [7,10)=1, B bf16 [10,13)=1, both K-major (bits 15, 16 = 0), N>>3 at
// [17,23), M>>4 at [24,29).
__host__ __device__ constexpr uint32_t instr_desc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// kind::f8f6f4 with E4M3 A and B (format code 0 in [7,10) and [10,13)),
// f32 accumulator, both K-major.
__host__ __device__ constexpr uint32_t instr_desc_e4m3_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Issue a load of 8 consecutive f32 columns of this thread's TMEM lane.
DG_DEV void tmem_load8_issue(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
DG_DEV void tmem_load8_wait(uint32_t (&r)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7])
               :
               : "memory");
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of
// (x0,x1,x2,x3) -> (hi(M1 x2)^x1^k0, lo(M1 x2), hi(M0 x0)^x3^k1, lo(M0 x0))
// with the key bumped by the Weyl constants after each round.
// ---------------------------------------------------------------------------
DG_DEV void philox4x32_10(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3, uint32_t k0,
                          uint32_t k1, uint32_t (&out)[4]) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * x0;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * x2;
    const uint32_t y0 = static_cast<uint32_t>(p1 >> 32) ^ x1 ^ k0;
    const uint32_t y2 = static_cast<uint32_t>(p0 >> 32) ^ x3 ^ k1;
    x1 = static_cast<uint32_t>(p1);
    x3 = static_cast<uint32_t>(p0);
    x0 = y0;
    x2 = y2;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  out[0] = x0;
  out[1] = x1;
  out[2] = x2;
  out[3] = x3;
}

// Same, with the ten round keys (key + i * Weyl constants) precomputed in
// two arrays (kernel parameters).
DG_DEV void philox4x32_10_keys(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3,
                               const uint32_t (&k0)[10], const uint32_t (&k1)[10], uint32_t (&out)[4]) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * x0;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * x2;
    const uint32_t y0 = static_cast<uint32_t>(p1 >> 32) ^ x1 ^ k0[i];
    const uint32_t y2 = static_cast<uint32_t>(p0 >> 32) ^ x3 ^ k1[i];
    x1 = static_cast<uint32_t>(p1);
    x3 = static_cast<uint32_t>(p0);
    x0 = y0;
    x2 = y2;
  }
  out[0] = x0;
  out[1] = x1;
  out[2] = x2;
  out[3] = x3;
}

// Philox4x32-10 words of counter (x0, c1, c2, c3) for many x0 with c1..c3
// fixed (one canvas slot at one step): the first round's product M1 c2 and
// the second round's product M0 (hi(M1 c2) ^ c1 ^ k0) do not depend on x0,
// so they are formed once per slot.  The outputs are those of
// philox4x32_10_keys bit for bit.
struct PhiloxRow {
  uint32_t x0r1;  // word 0 after round 1:  hi(M1 c2) ^ c1 ^ k0[0]
  uint32_t b1;    // lo(M1 c2) ^ k0[1]: round 2 mixes it into word 0
  uint32_t e0;    // c3 ^ k1[0]: round 1 mixes it into word 2
  uint32_t c1k;   // hi(M0 x0r1) ^ k1[1]: round 2 mixes it into word 2
  uint32_t d;     // lo(M0 x0r1): word 3 after round 2
};

__host__ __device__ __forceinline__ PhiloxRow philox_row(uint32_t c1, uint32_t c2, uint32_t c3,
                                                         const uint32_t (&k0)[10], const uint32_t (&k1)[10]) {
  PhiloxRow r;
  const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c2;
  r.x0r1 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ k0[0];
  r.b1 = static_cast<uint32_t>(p1) ^ k0[1];
  r.e0 = c3 ^ k1[0];
  const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * r.x0r1;
  r.c1k = static_cast<uint32_t>(p0 >> 32) ^ k1[1];
  r.d = static_cast<uint32_t>(p0);
  return r;
}

__host__ __device__ __forceinline__ void philox4x32_10_row(uint32_t x0, const PhiloxRow& r,
                                                           const uint32_t (&k0)[10], const uint32_t (&k1)[10],
                                                           uint32_t (&out)[4]) {
  // round 1: only the product M0 x0 depends on x0
  const uint64_t q0 = static_cast<uint64_t>(0xD2511F53u) * x0;
  const uint32_t y2 = static_cast<uint32_t>(q0 >> 32) ^ r.e0;
  const uint32_t x3a = static_cast<uint32_t>(q0);
  // round 2: the product M0 x0r1 is the row's
  const uint64_t q1 = static_cast<uint64_t>(0xCD9E8D57u) * y2;
  uint32_t w0 = static_cast<uint32_t>(q1 >> 32) ^ r.b1;
  uint32_t w1 = static_cast<uint32_t>(q1);
  uint32_t w2 = r.c1k ^ x3a;
  uint32_t w3 = r.d;
#pragma unroll
  for (int i = 2; i < 10; ++i) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * w0;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * w2;
    const uint32_t y0 = static_cast<uint32_t>(p1 >> 32) ^ w1 ^ k0[i];
    const uint32_t y2b = static_cast<uint32_t>(p0 >> 32) ^ w3 ^ k1[i];
    w1 = static_cast<uint32_t>(p1);
    w3 = static_cast<uint32_t>(p0);
    w0 = y0;
    w2 = y2b;
  }
  out[0] = w0;
  out[1] = w1;
  out[2] = w2;
  out[3] = w3;
}

// ---------------------------------------------------------------------------
// Per-row partial of the fused head: base-2 online softmax of x = z / tau,
// argmax of z, best specified Gumbel key.
//
// The softmax part is kept relative to the running maximum: m2 = fl(zmax c2)
// (c2 = log2(e) / tau), every element other than the maximum contributes
// e = 2^d with d = z c2 - m2 (one rounding), and the maximum itself is the
// unit 2^0 -- it enters neither sum.  The record holds
//   Sp = S - 1 = (number of elements equal to zmax) - 1 + sum_{z < zmax} e,
//   T2 = sum_{z < zmax} d e,
// so the normaliser's excess over the unit is carried explicitly and keeps
// its relative precision however small it is (for a confident slot S - 1 is
// far below the float32 spacing of S = 1).  The entropy follows as
//   H = ln S - ln2 T2 / S = log1p(Sp) - ln2 T2 / (1 + Sp).
// An empty record is m2 = -1e30, Sp = -1 (S = 0), T2 = 0.
// ---------------------------------------------------------------------------
struct Partial {
  float m2, Sp, T2;
  float zmax;
  int zarg;
  float gkey;
  int garg;
};

DG_DEV void partial_init(Partial& a) {
  a.m2 = -1.0e30f;
  a.Sp = -1.f;
  a.T2 = 0.f;
  a.zmax = -3.402823466e38f;
  a.zarg = 0x7fffffff;
  a.gkey = -3.402823466e38f;
  a.garg = 0x7fffffff;
}

// Merge b into a.  Softmax: the record with the larger m2 keeps its unit;
// the other's whole mass 1 + Sp_l moves into the ordinary mass, shifted by
// dl = m2_l - m2_h <= 0:  Sp = Sp_h + (1 + Sp_l) 2^dl,
// T2 = T2_h + (T2_l + dl (1 + Sp_l)) 2^dl.  Argmax and Gumbel key: the
// larger value wins, ties to the lower vocabulary index.
DG_DEV void partial_merge(Partial& a, const Partial& b) {
  const bool bhi = b.m2 > a.m2;
  const float mh = bhi ? b.m2 : a.m2, ml = bhi ? a.m2 : b.m2;
  const float sph = bhi ? b.Sp : a.Sp, spl = bhi ? a.Sp : b.Sp;
  const float th = bhi ? b.T2 : a.T2, tl = bhi ? a.T2 : b.T2;
  const float dl = ml - mh;
  const float sl = exp2f(dl);
  const float tot_l = 1.0f + spl;
  a.T2 = th + (tl + dl * tot_l) * sl;
  a.Sp = fmaf(tot_l, sl, sph);
  a.m2 = mh;
  if (b.zmax > a.zmax || (b.zmax == a.zmax && b.zarg < a.zarg)) {
    a.zmax = b.zmax;
    a.zarg = b.zarg;
  }
  if (b.gkey > a.gkey || (b.gkey == a.gkey && b.garg < a.garg)) {
    a.gkey = b.gkey;
    a.garg = b.garg;
  }
}

// Stream purposes (high half of counter word 1).
constexpr uint32_t kPurposeGumbel = 0u;
constexpr uint32_t kPurposeRenoise = 1u;
constexpr uint32_t kPurposeInit = 3u;  // the noise canvas a block starts from

// ---------------------------------------------------------------------------
// The float32 key of the Gumbel-max draw, IEEE operations only.
//
// L(y): y = 2^e m, m in [1,2), halved (e+1) when m > sqrt(2); f = m - 1,
// s = f / (m + 1), z = s^2, ln m = 2s + s z (2/3 + z (2/5 + z (2/7 + z (2/9
// + z 2/11)))) (the atanh series of ln m = 2 atanh((m-1)/(m+1))), result
// e LN2_HI + (ln m + e LN2_LO) with LN2_HI = ln 2 truncated to 16 fraction
// bits.  Every constant is the float32 nearest to the stated rational.
// ---------------------------------------------------------------------------
DG_DEV float log_ieee(float y) {
  const float kC3 = __uint_as_float(0x3f2aaaabu);   // RN(2/3)
  const float kC5 = __uint_as_float(0x3ecccccdu);   // RN(2/5)
  const float kC7 = __uint_as_float(0x3e924925u);   // RN(2/7)
  const float kC9 = __uint_as_float(0x3e638e39u);   // RN(2/9)
  const float kC11 = __uint_as_float(0x3e3a2e8cu);  // RN(2/11)
  const float kLn2Hi = __uint_as_float(0x3f317200u);  // 45426 / 65536
  const float kLn2Lo = __uint_as_float(0x35bfbe8eu);  // RN(ln 2 - LN2_HI)
  const uint32_t b = __float_as_uint(y);
  int e = static_cast<int>((b >> 23) & 0xFFu) - 127;
  const uint32_t mant = b & 0x7FFFFFu;
  float m = __uint_as_float(mant | 0x3F800000u);
  if (mant > 0x3504F3u) {  // m > sqrt(2)
    m = __fmul_rn(m, 0.5f);
    e += 1;
  }
  const float f = __fsub_rn(m, 1.0f);
  const float s = __fdiv_rn(f, __fadd_rn(m, 1.0f));
  const float z = __fmul_rn(s, s);
  float r = __fmul_rn(z, kC11);
  r = __fadd_rn(kC9, r);
  r = __fmul_rn(z, r);
  r = __fadd_rn(kC7, r);
  r = __fmul_rn(z, r);
  r = __fadd_rn(kC5, r);
  r = __fmul_rn(z, r);
  r = __fadd_rn(kC3, r);
  r = __fmul_rn(z, r);
  const float lnm = __fadd_rn(__fadd_rn(s, s), __fmul_rn(s, r));
  const float ef = static_cast<float>(e);
  return __fadd_rn(__fmul_rn(ef, kLn2Hi), __fadd_rn(lnm, __fmul_rn(ef, kLn2Lo)));
}

// u = (2 (r >> 9) + 1) 2^-24, exact.
DG_DEV float uniform_from_word(uint32_t r) {
  return __fmul_rn(static_cast<float>(2u * (r >> 9) + 1u), 5.9604644775390625e-08f);
}

// g32(u) = -L(-L(u)): the Gumbel noise of the specified key.
DG_DEV float gumbel_exact(uint32_t r) {
  const float u = uniform_from_word(r);
  return -log_ieee(-log_ieee(u));
}

// The specified float32 key: fl(fl(z * inv_tau) + g32).
DG_DEV float key_exact(float z, float inv_tau, uint32_t r) {
  return __fadd_rn(__fmul_rn(z, inv_tau), gumbel_exact(r));
}

DG_DEV float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
DG_DEV float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Screening transform.  With E = -ln u (an Exp(1) variable) and
// E2 = E / ln 2 = -lg2 u, the Gumbel noise is g = -ln E = C0 - ln2 lg2(E2)
// with C0 = -ln(ln 2).  This returns an approximation of lg2(E2): for
// u > 15/16 (y = 1 - u < 1/16, where the hardware lg2 of u loses relative
// accuracy) E2 comes from -lg2(1 - y) = (y + y^2/2 + y^3/3 + y^4/4 + ...)/ln 2,
// otherwise from the hardware lg2.  Its distance from the specified g32 is
// measured over all 2^23 inputs by the GPU tests and bounded by
// kGumbelApproxErr.
DG_DEV float lg2_exp1_approx(uint32_t r) {
  const float one_plus = __uint_as_float((r >> 9) | 0x3F800000u);  // 1 + r23 2^-23
  const float u = __fsub_rn(one_plus, __uint_as_float(0x3f7fffffu));  // - (1 - 2^-24), exact
  const float y = __fsub_rn(1.0f, u);                                 // exact
  // -(y/ln2)(1 + y/2 + y^2/3 + y^3/4): coefficients -1/(k ln 2)
  float t = __fmaf_rn(y, -0.36067376022224085f, -0.48089834696298783f);
  t = __fmaf_rn(y, t, -0.72134752044448170f);
  t = __fmaf_rn(y, t, -1.44269504088896341f);
  const float neg_e2_series = __fmul_rn(y, t);
  const float neg_e2_log = lg2_approx(u);  // lg2 u = -E2
  const float neg_e2 = (y < 0.0625f) ? neg_e2_series : neg_e2_log;
  return lg2_approx(-neg_e2);
}

// C0 = -ln(ln 2): g = C0 - ln2 * lg2(E2).
constexpr float kGumbelC0 = 0.36651292058166432f;

// Order-preserving map of a (non-NaN) float onto uint32: a < b <=> enc(a) <
// enc(b); 0 is never produced and stands for "no key yet".
DG_DEV uint32_t key_order_enc(float k) {
  const uint32_t b = __float_as_uint(k);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
DG_DEV float key_order_dec(uint32_t e) {
  if (e == 0u) return -FLT_MAX;
  return __uint_as_float((e & 0x80000000u) ? (e & 0x7FFFFFFFu) : ~e);
}

// The largest specified noise, g32 at the largest u = 1 - 2^-24 (g32 is
// nondecreasing in the word; both facts are checked against the oracle over
// all 2^23 inputs).
constexpr float kGumbelMaxNoise = 16.635532f;

// |approx key - specified key| <= kGumbelApproxErr + rounding of the keys.
constexpr float kGumbelApproxErr = 1.0e-5f;
constexpr float kLn2 = 0.693147182464599609375f;
constexpr float kLog2e = 1.44269502162933349609375f;

}  // namespace dg
