// Fifth-generation tensor-core (tcgen05) building blocks for sm_100a:
// tensor-memory allocation, shared-memory matrix descriptors, the MMA issue
// and commit, tensor-memory loads and the fences that order them against
// thread synchronisation.  Operands are staged in shared memory in the
// no-swizzle ("interleaved") canonical layouts: 8 rows x 16 bytes core
// matrices, 128 contiguous bytes each.
#pragma once

#include <stdint.h>

namespace wsvd {
namespace tc05 {

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor, no swizzle.  `lbo` and `sbo` are byte
// strides between core matrices:
//   K-major operand:  lbo = next 16-byte chunk along K, sbo = next 8-row group along M/N;
//   MN-major operand: lbo = next 8-row group along K,   sbo = next 8-element group along M/N.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);  // descriptor version 1, layout 0 (none)
}

// Swizzled variant: `layout` 2 = 128-byte, 4 = 64-byte, 6 = 32-byte swizzle
// (the patterns TMA writes with CU_TENSOR_MAP_SWIZZLE_128B / 64B / 32B; the
// atom -- 8 rows of the swizzle width -- must be aligned to its own size).
//   K-major:  rows of the swizzle width, sbo = next 8-row group (lbo unused);
//   MN-major: sbo = next 8-row group along K, lbo = next swizzle-width group along M/N.
__device__ __forceinline__ uint64_t smem_desc_sw(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return smem_desc(saddr, lbo, sbo) | ((uint64_t)layout << 61);
}

// Instruction descriptor of a dense MMA (cta_group::1).
//   cfmt: accumulator 1 = f32, 2 = s32; afmt / bfmt: kind::f16 0 = f16, kind::i8 1 = signed;
//   amaj / bmaj: 0 = K-major, 1 = MN-major.
__host__ __device__ constexpr uint32_t instr_desc(int cfmt, int afmt, int bfmt, int amaj, int bmaj, int M, int N) {
  return ((uint32_t)cfmt << 4) | ((uint32_t)afmt << 7) | ((uint32_t)bfmt << 10) | ((uint32_t)amaj << 15) |
         ((uint32_t)bmaj << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- tensor memory
// One full warp allocates `ncols` columns (a power of two >= 32) and writes
// the base address to shared memory; the permit is released right away so
// that other CTAs on the SM may allocate.
__device__ __forceinline__ void alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem))),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Generic-proxy shared-memory writes made visible to the tensor core's
// (async proxy) operand reads; each writing thread executes it before the
// synchronisation that hands the buffer to the MMA issuer.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- MMA
// D[tmem] (+)= A[smem] . B[smem]^T.
// Warp-level issue: every lane of a converged warp executes the call with the
// same operands and one elected lane (the lowest) issues the instruction.
// Issued this way an MMA costs what the tensor core needs for it; issued from
// a lone lane behind a divergent branch it costs about a hundred cycles
// whatever its shape (measured on B200).
__device__ __forceinline__ void mma_f16_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             bool accum) {
  asm volatile(
      "{\n\t.reg .pred e, p;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)accum)
      : "memory");
}
__device__ __forceinline__ void mma_i8_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            bool accum) {
  asm volatile(
      "{\n\t.reg .pred e, p;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)accum)
      : "memory");
}
// Arrives once on `bar` when every MMA the elected lane issued before has
// completed, their shared-memory reads included (the same lane: the lowest of
// a converged warp).
__device__ __forceinline__ void commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
      : "memory");
}

// ---------------------------------------------------------------- loads
// 8 consecutive 32-bit columns of this thread's lane (warp w may read lanes
// 32 (w % 4) .. 32 (w % 4) + 31; the lane is part of taddr).
__device__ __forceinline__ void ld8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr)
               : "memory");
}
// 32 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

}  // namespace tc05
}  // namespace wsvd
