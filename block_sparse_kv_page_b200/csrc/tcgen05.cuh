// 5th-generation tensor core (tcgen05) helpers for sm_100a: tensor-memory
// allocation, shared-memory operand descriptors, the MMA issued by one thread,
// its completion on an mbarrier, and accumulator loads from tensor memory.
//
// Operand layout used throughout: K-major tiles staged by TMA with
// SWIZZLE_128B, i.e. rows of 128 bytes (64 bf16 or 32 fp32 of the K axis), 8-row
// swizzle atoms of 1024 bytes, each K-chunk of 128 bytes a separate
// [rows][128 B] region whose base is 1024-byte aligned.  One MMA consumes 32
// bytes of K per row (16 bf16), so step k of chunk c starts at
// chunk_base(c) + 32 * (k % 4); the hardware applies the swizzle from the
// address bits, as TMA did when it wrote the tile.
#pragma once

#include "common.cuh"

namespace sa {
namespace tc {

// ---------------------------------------------------------------- tensor memory
// Allocate `ncols` columns (power of 2, 32..512) of tensor memory; the whole
// warp calls it; the TMEM address lands in shared memory at `slot`.
SA_DEV void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_addr(slot)),
               "r"(ncols)
               : "memory");
}
// Let other CTAs of the SM allocate (call once, after this CTA's allocation).
SA_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
// Free the allocation (whole warp; before the CTA exits).
SA_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols) : "memory");
}

SA_DEV void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
SA_DEV void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor: start address >> 4 in bits [0,14), leading
// byte offset >> 4 in [16,30) (unused for swizzled K-major tiles: 16 B),
// stride byte offset >> 4 in [32,46) (1024 B between 8-row atoms), version 1
// in [46,48), base offset 0 (atoms 1024-aligned), layout 2 = 128-byte swizzle
// in [61,64).
SA_DEV uint64_t smem_desc_sw128(const void* p) {
  const uint64_t a = (uint64_t)((smem_addr(p) & 0x3FFFFu) >> 4);
  return a | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, dense, fp32 accumulator (bits [4,6) = 1), both
// operands K-major; `fmt` = 1 for bf16 (kind::f16) in the A [7,10) and B
// [10,13) format fields; N >> 3 in [17,23), M >> 4 in
// [24,29).
__host__ __device__ constexpr uint32_t idesc_f32acc(uint32_t fmt, uint32_t M, uint32_t N) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}
constexpr uint32_t kFmtBF16 = 1;

// ---------------------------------------------------------------- MMA
// D[tmem] (+)= A[smem] . B[smem]^T, issued by a single thread.
SA_DEV void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, bool acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)acc)
      : "memory");
}
// D[tmem] (+)= A[tmem] . B[smem]^T: A (M = 128 rows) in tensor memory, row m in
// lane m, two bf16 of the K axis per 32-bit column (lower K index in the low
// half), so a K = 16 step starts 8 columns after the previous one.
SA_DEV void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, bool acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"((uint32_t)acc)
      : "memory");
}
// Arrive on `bar` once every tcgen05 operation this thread issued so far is done.
SA_DEV void commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   smem_addr(bar))
               : "memory");
}

// ---------------------------------------------------------------- accumulator loads
// 16 consecutive fp32 columns of this thread's TMEM lane (warp w of a
// warpgroup reads lanes 32 w .. 32 w + 31).  Complete after wait_ld().
SA_DEV void ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
SA_DEV void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
// Ties 16 registers filled by ld_32x32b_x16 to this point of the program:
// placed after wait_ld(), it keeps the compiler from moving their uses above
// the wait (the asm reads and "writes" them; it emits no instruction).
SA_DEV void reg_fence(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])::"memory");
}
// Store 16 consecutive fp32 columns of this thread's TMEM lane (same lane
// mapping as ld_32x32b_x16).  Complete after wait_st().
SA_DEV void st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
SA_DEV void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

}  // namespace tc
}  // namespace sa
