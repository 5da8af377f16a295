// tcgen05 helpers for sm_100a: tensor-memory (TMEM) allocation, loads and stores,
// shared-memory matrix descriptors, the kind::f16 MMA (bf16 operands from
// shared memory, fp32 accumulator in TMEM) and its completion on an mbarrier,
// the fences between thread syncs and tensor-core work, and the TMA tile
// store with its bulk-group waits.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "gdr_ptx.cuh"

namespace gdr {

// ---------------------------------------------------------------- descriptors

// Layout field of a shared-memory matrix descriptor.
enum UmmaLayout : uint32_t {
  kUmmaInterleave = 0,  // no swizzle: 8 x 16-byte core matrices, 128 contiguous bytes each
  kUmmaSwizzle128 = 2,  // 128-byte swizzle, 1024-byte atoms of 8 rows x 128 bytes
};

// Shared-memory matrix descriptor, 64 bits:
//   bits  0-13  start address >> 4
//   bits 16-29  leading-dimension byte offset >> 4
//   bits 32-45  stride-dimension byte offset >> 4
//   bits 46-47  descriptor version (1 on sm_100)
//   bits 49-51  base offset (0: swizzle atoms are 1024-byte aligned)
//   bit  52     leading-offset mode (0: a byte offset)
//   bits 61-63  layout
// What the two offsets step over depends on the operand's major-ness and the
// layout:
//   K-major, no swizzle: LBO = between the two 8-element core matrices along
//     K of one instruction, SBO = between 8-row groups along M (or N);
//   M/N-major, no swizzle: LBO = between 8-row groups along K, SBO = between
//     8-element groups along M (or N);
//   M/N-major, 128-byte swizzle: LBO = between 64-element blocks along M (or
//     N), SBO = between 8-row groups along K.
__device__ __forceinline__ uint64_t umma_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              UmmaLayout layout) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
         (static_cast<uint64_t>(layout) << 61);
}

// Instruction descriptor of a kind::f16 MMA with bf16 A and B and an fp32
// accumulator, 32 bits:
//   bits  4-5   D format (1 = f32)
//   bits  7-9   A format (1 = bf16)
//   bits 10-12  B format (1 = bf16)
//   bit  15     A major (0 = K, 1 = M)
//   bit  16     B major (0 = K, 1 = N)
//   bits 17-22  N >> 3
//   bits 24-28  M >> 4
template <int M, int N, bool A_MN, bool B_MN>
__host__ __device__ constexpr uint32_t umma_idesc_bf16() {
  static_assert(M == 64 || M == 128, "M is 64 or 128 with one CTA");
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "N is a multiple of 16 in [16, 256]");
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(A_MN) << 15) |
         (static_cast<uint32_t>(B_MN) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------- MMA

// True in exactly one active lane of the warp (all lanes must execute it).
__device__ __forceinline__ bool elect_one() {
  uint32_t is_elected;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(is_elected));
  return is_elected != 0;
}

// The descriptor `desc` with its start address moved on by `bytes` (a
// multiple of 16 that keeps the address inside shared memory).
__host__ __device__ __forceinline__ uint64_t umma_desc_advance(uint64_t desc, uint32_t bytes) {
  return desc + static_cast<uint64_t>(bytes >> 4);
}

// D[M x N] (+)= A[M x 16] * B[N x 16]^T for one instruction (K = 16), issued
// by one thread; D in TMEM at `d_tmem` (lane 0, first column).
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(static_cast<uint32_t>(accumulate))
      : "memory");
}

// Arrive once on `bar` when every MMA this thread has issued so far is done.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                   "r"(bar)
               : "memory");
}

// ---------------------------------------------------------------- TMEM

// Allocate `ncols` columns (a power of two >= 32) for the CTA; one whole warp
// executes it, and the base address lands in shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Order tensor-core work against thread syncs: `before` ahead of a barrier
// that publishes finished TMEM reads, `after` behind a barrier that precedes
// TMEM reads or MMAs.
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane: the warp reads the
// 32 lanes that start at the lane field of `taddr` (32 * (warp % 4)).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane, written; the warp
// writes the 32 lanes that start at the lane field of `taddr`.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// Until this thread's TMEM stores are done (before an MMA or a thread sync
// that hands the columns on).
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- proxies, TMA store

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads, TMA stores).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, int x, int y, int z,
                                             uint32_t src) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
          map),
      "r"(x), "r"(y), "r"(z), "r"(src)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Until this thread's bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Until this thread's bulk stores are complete (written to global memory).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

}  // namespace gdr
