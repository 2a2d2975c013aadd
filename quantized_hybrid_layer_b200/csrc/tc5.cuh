// Fifth-generation tensor core (tcgen05) primitives for sm_100a: tensor-memory
// allocation, register <-> tensor-memory moves, the integer MMA with its A
// operand in tensor memory and its B operand in shared memory, and the
// completion / ordering instructions around them.
//
// Tensor memory (TMEM) is 128 lanes x 512 columns of 32 bits per SM.  An
// address is (lane << 16) | column.  A warp may only touch the 32 lanes of its
// quarter, 32 * (warp % 4) .. + 31.  For an M = 128 MMA, row m of A and of the
// accumulator D lives in lane m; A's K bytes are packed four to a column, D's
// N int32 results one to a column.
#pragma once

#include "common.cuh"

namespace qhl {

// ---- allocation (one full warp) --------------------------------------------
// Allocate `ncols` columns (a power of two >= 32); the base address is written
// to *slot (shared memory).  Blocks until that many columns are free on the SM.
QHL_DEV void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
QHL_DEV void tmem_dealloc(uint32_t base, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols) : "memory");
}

// ---- ordering of tensor-core work against thread synchronisation -----------
QHL_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
QHL_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---- registers -> TMEM (each thread its own lane, 8 consecutive columns) ----
QHL_DEV void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
// 32 consecutive columns of the thread's lane in one instruction.
QHL_DEV void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
QHL_DEV void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---- TMEM -> registers: 4 consecutive columns of the thread's lane ----------
QHL_DEV void tmem_ld4(uint32_t taddr, int (&v)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(taddr)
               : "memory");
}
QHL_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---- shared-memory matrix descriptor (K-major, no swizzle) ------------------
// The canonical layout: "core matrices" of 8 rows x 16 bytes stored as 128
// contiguous bytes (row r at 16 r); the core matrix holding the next 16 bytes
// of K sits `lbo` bytes further, the one holding the next 8 rows `sbo` bytes
// further.  Fields: start address >> 4 (bits 0-13), lbo >> 4 (16-29), sbo >> 4
// (32-45), descriptor version 1 (bits 46-47), swizzle mode 0 (bits 61-63).
QHL_DEV uint64_t smem_desc_kmajor(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// ---- instruction descriptor of kind::i8 ------------------------------------
// D int32 (bits 4-5 = 2), A unsigned / signed 8-bit (bits 7-9 = 0 / 1),
// B signed 8-bit (bits 10-12 = 1), both K-major, N >> 3 (bits 17-22),
// M >> 4 (bits 24-28).
__host__ __device__ constexpr uint32_t idesc_i8(bool a_signed, int m, int n) {
  return (2u << 4) | ((a_signed ? 1u : 0u) << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(m >> 4) << 24);
}

// D[tmem] (=|+=) A[tmem] * B[smem]^T, one M x N x 32 integer product issued by
// the calling thread (asynchronous: completion through tc_commit).
QHL_DEV void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// Arrive (once) on the mbarrier when every tcgen05 MMA this thread issued so
// far has completed.
QHL_DEV void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

}  // namespace qhl
