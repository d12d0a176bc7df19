// Device helpers of the tensor-core decode kernels (absorbed and expanded
// forms): elected issue, bounded mbarrier waits, TMEM loads and stores,
// nibble-to-fp16 operand extraction, TMA / bulk loads with an L2 policy.
// Written from the PTX ISA's descriptions of these instructions.
#pragma once
#include <cuda.h>
#include <stdint.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace fsq {
namespace tc {

using namespace ptx;

// One lane of a converged warp (elect.sync)
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, e;\n\t}"
      : "=r"(e));
  return e != 0;
}
// A commit issued by one elected lane of a converged warp
__device__ __forceinline__ void tc_commit_elect(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

// Pooling operand values as fp16 subnormals, no bias: nibble J of both
// half-words left in place in mantissa bits 0..3 (value n 2^-24) or bits 4..7
// (value n 2^-20).  w holds, per half-word, the four nibbles of one token.
__device__ __forceinline__ void nib_sub4(uint32_t w, uint32_t &j0, uint32_t &j1, uint32_t &j2, uint32_t &j3) {
  const uint32_t ws = w >> 8;
  j0 = w & 0x000F000Fu;   // n 2^-24
  j1 = w & 0x00F000F0u;   // n 2^-20
  j2 = ws & 0x000F000Fu;  // n 2^-24
  j3 = ws & 0x00F000F0u;  // n 2^-20
}

// Physical K position of token r in the pooling operand (see the 16x256b store below).
__device__ __forceinline__ int kappa_of_token(int r) {
  return (r & ~15) | (((r >> 1) & 3) << 2) | (((r >> 3) & 1) << 1) | (r & 1);
}

// max(a, b, c) in one instruction (three-input max.f32, sm_100)
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the special-function unit (inputs <= 8 here; -inf gives 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 128-byte-swizzle layout of a TMA tile: 16-byte chunk c of row r sits at chunk c ^ (r % 8).
__device__ __forceinline__ int swz(int r, int chunk) { return r * 128 + ((chunk ^ (r & 7)) << 4); }

// L2 policy for the code stream, which every call reads once: evict it
// first, so that it does not push out of L2 the small operands each call
// re-reads (E, W_kv, the partials)
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// With several queries per cache row (virtual rows of one call) the CTAs of
// the row's queries read the same tiles at about the same time: keep them in
// L2 at normal priority so that each tile crosses HBM about once.
__device__ __forceinline__ uint64_t l2_evict_normal() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c0, int c1, int c2, uint64_t *bar,
                                            uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                              uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// 32-bit little-endian load from a 2-byte aligned shared address
__device__ __forceinline__ uint32_t lds_u32_a2(const uint8_t *p) {
  const uint16_t *h = reinterpret_cast<const uint16_t *>(p);
  return (uint32_t)h[0] | ((uint32_t)h[1] << 16);
}

// Bounded barrier wait.  mbarrier.try_wait with a suspend-time hint parks the
// warp in hardware until the phase completes (or the hint expires), so a
// waiting warp takes no issue slots from the working warps of its scheduler.
// Gives up after `limit_ns` or once *abort is set.
__device__ __forceinline__ bool bar_test(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(a), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool bar_try(uint32_t a, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(a), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
// Tests of two or three phases at once: the tests are independent, so their
// shared-memory round trips overlap (a completed hand-off costs one of them)
__device__ __forceinline__ bool bar_test2(uint32_t a0, uint32_t p0, uint32_t a1, uint32_t p1) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q, [%3], %4;\n\t"
      "and.pred p, p, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(a0), "r"(p0), "r"(a1), "r"(p1)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool bar_test3(uint32_t a0, uint32_t p0, uint32_t a1, uint32_t p1, uint32_t a2,
                                          uint32_t p2) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p, q, r;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q, [%3], %4;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 r, [%5], %6;\n\t"
      "and.pred p, p, q;\n\t"
      "and.pred p, p, r;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(a0), "r"(p0), "r"(a1), "r"(p1), "r"(a2), "r"(p2)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool wait_bar(uint64_t *b, uint32_t parity, volatile uint32_t *abort, uint64_t limit_ns) {
  const uint32_t a = smem_u32(b);
  if (bar_test(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (bar_try(a, parity, 1000u)) return true;
    if ((it & 7u) == 0u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) return false;
    }
  }
}
// Waits for two (three) phases: one combined test, then each in turn
__device__ __forceinline__ bool wait_bars(uint64_t *b0, uint32_t p0, uint64_t *b1, uint32_t p1,
                                          volatile uint32_t *abort, uint64_t limit_ns) {
  if (bar_test2(smem_u32(b0), p0, smem_u32(b1), p1)) return true;
  return wait_bar(b0, p0, abort, limit_ns) && wait_bar(b1, p1, abort, limit_ns);
}
__device__ __forceinline__ bool wait_bars(uint64_t *b0, uint32_t p0, uint64_t *b1, uint32_t p1, uint64_t *b2,
                                          uint32_t p2, volatile uint32_t *abort, uint64_t limit_ns) {
  if (bar_test3(smem_u32(b0), p0, smem_u32(b1), p1, smem_u32(b2), p2)) return true;
  return wait_bar(b0, p0, abort, limit_ns) && wait_bar(b1, p1, abort, limit_ns) && wait_bar(b2, p2, abort, limit_ns);
}

// Named barrier over `nthreads` threads that returns the OR of `pred` over them.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0u;
}

// Error path: wait (time-bounded, ignoring the abort flag) for an async copy
// already issued into this CTA's shared memory, so none lands after exit.
__device__ __forceinline__ void drain_bar(uint64_t *b, uint32_t parity, uint64_t limit_ns) {
  const uint32_t a = smem_u32(b);
  const uint64_t t0 = globaltimer_ns();
  while (!bar_test(a, parity)) {
    __nanosleep(100);
    if (globaltimer_ns() - t0 > limit_ns) return;
  }
}

__device__ __forceinline__ void tmem_st_16x256b_x4(uint32_t taddr, const uint32_t *r) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t *r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
template <int HQ>
__device__ __forceinline__ void tmem_ld_hq(uint32_t ta, uint32_t *r) {
  if constexpr (HQ == 16) tmem_ld16(ta, r);
  else tmem_ld8(ta, r);
}
template <int HQ>
__device__ __forceinline__ void tmem_st_hq(uint32_t ta, const uint32_t *r) {
  if constexpr (HQ == 16) tmem_st16(ta, r);
  else tmem_st8(ta, r);
}

template <int NQ>
__device__ __forceinline__ void tmem_ld_nq(uint32_t ta, uint32_t *r) {
  if constexpr (NQ == 32) tmem_ld32(ta, r);
  else tmem_ld16(ta, r);
}
template <int NQ>
__device__ __forceinline__ void tmem_st_nq(uint32_t ta, const uint32_t *r) {
  if constexpr (NQ == 32) tmem_st32(ta, r);
  else tmem_st16(ta, r);
}

}  // namespace tc
}  // namespace fsq
