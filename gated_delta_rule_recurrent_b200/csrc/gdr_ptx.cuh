// PTX helpers shared by the decode kernels: mbarriers with bounded waits,
// TMA and bulk copies, 4-byte cp.async, packed fp32 pairs (sm_100 f32x2),
// and the device-global error word that bounded waits report into.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_decode.cuh"

namespace gdr {

// Bits of the device error word: a consumer's wait for a ready tile; a wait on
// the producing side (a free stage, or landed copies to finalise); the final
// wait for copies still in flight.
constexpr unsigned kErrConsumerWait = 1u;
constexpr unsigned kErrProducerWait = 2u;
constexpr unsigned kErrDrainWait = 4u;

static __device__ unsigned int g_device_error = 0;

constexpr long long kWaitLimitCycles = 4000000000LL;  // ~2 s at 2 GHz

// Test builds only (-DGDR_TEST_HOOKS, never the shipped library): the limit of
// the abandonable waits below is a device variable the host can shorten, and
// the producer of every decode kernel can hold back one tile: it then starts
// no copy for that tile and never signals it ready, as if its copies never
// landed, and stops issuing. Its consumers' waits run out, with no copy in
// flight anywhere.
#ifdef GDR_TEST_HOOKS
static __device__ long long g_test_wait_limit = kWaitLimitCycles;
static __device__ int g_test_hold_tile = -1;
__device__ __forceinline__ long long abandonable_wait_limit() {
  return *reinterpret_cast<volatile long long*>(&g_test_wait_limit);
}
__device__ __forceinline__ bool test_hold_tile(int tile) {
  return tile == *reinterpret_cast<volatile int*>(&g_test_hold_tile);
}
#else
__device__ __forceinline__ constexpr long long abandonable_wait_limit() { return kWaitLimitCycles; }
__device__ __forceinline__ constexpr bool test_hold_tile(int) { return false; }
#endif

// Byte offset of (row i, 16-byte chunk holding column col) in a state tile
// loaded by TMA with the 128-byte swizzle as [col / 64][row][64 columns]:
// within each 128-byte row segment, chunk c sits at position c ^ (i % 8).
template <int DK>
__host__ __device__ __forceinline__ int swz_offset(int i, int col) {
  return ((((col >> 6) * DK + i)) << 7) + ((((col >> 3) & 7) ^ (i & 7)) << 4);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but the thread may stay suspended in the instruction for
// up to `hint_ns` nanoseconds while the phase is incomplete (it resumes as
// soon as the phase completes), so a waiting warp takes few issue slots.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar, uint32_t parity,
                                                      uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

constexpr uint32_t kWaitSuspendNs = 20000;

// Wait for the phase of parity `parity` to complete, for at most
// kWaitLimitCycles. Returns false when the budget ran out. Used for work that
// is already in flight and ends by itself: copies a CTA must see land before
// it exits, and tensor-core MMAs it issued.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_suspend(bar, parity, kWaitSuspendNs)) {
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
  return true;
}

// Failure protocol of the decode kernels. Each CTA keeps an abort word in
// shared memory (0 at start). A wait on another role's signal ("ready",
// "free") is abandonable: it returns false when its own budget runs out (it
// then ORs `err_bit` into the device error word and sets the abort word), or,
// once it has blocked for a while, when the abort word is set by any other wait
// of the CTA. Whoever sees a wait fail stops for good: a producer issues no more
// copies, a finaliser or sums warp signals no more tiles ready, a consumer
// commits no state and frees no more stages. Because nobody signals after a
// failure, no stage is refilled over a phase that never completed, so no wait
// can mistake an old phase for a new one; the tiles a CTA commits are exactly
// the ones whose inputs were seen to land. Copies already started are drained
// with mbar_wait_bounded before the CTA exits.
//
// The abort word is looked at only once a wait has lasted a quarter of its
// budget (never, on a normal call): a wait's loop then costs what a plain
// bounded wait costs, and a CTA still winds down within a budget of a failure.
__device__ __forceinline__ bool mbar_wait_abandonable(uint32_t bar, uint32_t parity,
                                                      volatile int* abort_word, unsigned err_bit) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long limit = abandonable_wait_limit();
  const long long t0 = clock64();
  while (!mbar_try_wait_suspend(bar, parity, kWaitSuspendNs)) {
    const long long dt = clock64() - t0;
    if (dt > (limit >> 2)) {
      if (*abort_word != 0) return false;
      if (dt > limit) {
        atomicOr(&g_device_error, err_bit);
        *abort_word = 1;
        return false;
      }
    }
  }
  return true;
}

// A producer's wait for a free stage: the loop of mbar_wait_bounded with the
// budget of the abandonable waits. It does not look at the abort word (a
// producer waits once per tile, and the extra load in its loop measured ~6 %
// on the multi-token tensor-core kernel); when the budget runs out it ORs
// `err_bit` into the device error word, sets the abort word and returns false.
__device__ __forceinline__ bool mbar_wait_free(uint32_t bar, uint32_t parity,
                                               volatile int* abort_word, unsigned err_bit) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long limit = abandonable_wait_limit();
  const long long t0 = clock64();
  while (!mbar_try_wait_suspend(bar, parity, kWaitSuspendNs)) {
    if (clock64() - t0 > limit) {
      atomicOr(&g_device_error, err_bit);
      *abort_word = 1;
      return false;
    }
  }
  return true;
}

// bar.sync over `count` threads that also ANDs a predicate across them: every
// participant gets true exactly when every participant passed true.
__device__ __forceinline__ bool named_barrier_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// 1-D bulk copy global -> shared; both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 4-byte asynchronous copy global -> shared (both 4-byte aligned).
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// Arrive on `bar` once every cp.async this thread has issued so far has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void flag_error(unsigned bit) { atomicOr(&g_device_error, bit); }

// The bf16 at `p` is fetched as the aligned 32-bit word that holds it (that
// word never leaves the page of `p`, so the wider read cannot fault).
__device__ __forceinline__ const void* word_of(const uint16_t* p) {
  return reinterpret_cast<const void*>(reinterpret_cast<uintptr_t>(p) & ~uintptr_t(3));
}
__device__ __forceinline__ float bf16_in_word(uint32_t w, const uint16_t* p) {
  return (reinterpret_cast<uintptr_t>(p) & 2) ? bf16_hi(w) : bf16_lo(w);
}

// Packed pairs of fp32 (sm_100 f32x2 instructions: one issue slot for two
// IEEE round-to-nearest operations, bit-identical to two scalar ones).
__device__ __forceinline__ unsigned long long pk(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 upk(unsigned long long v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Named barrier over `count` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_barrier(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

}  // namespace gdr
