// Inline-PTX wrappers for the 5th-generation tensor cores of sm_100a (tcgen05):
// tensor-memory (TMEM) allocation, single-thread MMA issue with operands in
// shared memory, completion tracking on mbarriers, and TMEM -> register loads.
//
// Operand encodings follow the PTX ISA's tcgen05 matrix descriptors:
//   shared-memory descriptor (64 bit): start address >> 4 in bits 0-13,
//     leading-dimension byte offset >> 4 in bits 16-29, stride-dimension byte
//     offset >> 4 in bits 32-45, descriptor version 1 in bits 46-47, swizzle
//     mode in bits 61-63 (0 none, 2 = 128-byte swizzle);
//   instruction descriptor (32 bit) for kind::f16: D format (1 = f32) in bits
//     4-5, A and B formats (1 = bf16) in bits 7-9 and 10-12, A / B major-ness
//     (0 = K-major, 1 = MN-major) in bits 15 and 16, N >> 3 in bits 17-22,
//     M >> 4 in bits 24-28.
// Layouts used by the kernels (bf16 elements):
//   K-major, 128-byte swizzle: row r of a [rows][64] tile at r * 128 bytes,
//     16-byte chunk c stored at chunk c ^ (r % 8); 8-row groups 1024 bytes
//     apart (SBO); one MMA consumes 16 K-elements, the next K step starts 32
//     bytes further.  This is also what a TMA box of [16][64] bf16 with the
//     128-byte swizzle writes.
//   MN-major, 128-byte swizzle: the same tile read with rows as K and the 64
//     contiguous elements of a row as M or N (8-row K groups 1024 bytes apart).
//   K-major, no swizzle, K = 16: element (r, k) at (r % 8) * 16 + (k % 8) * 2 +
//     (k / 8) * 128 + (r / 8) * 256 bytes (core matrices of 8 rows x 16 bytes;
//     LBO = 128, SBO = 256).
// Accumulators: an M = 64 accumulator row m lives in TMEM lane
// (m % 16) + 32 * (m / 16); a warp may only touch the 32 lanes of its own
// quarter (warp id % 4).  tcgen05.ld 16x256b on a 16-lane group returns the
// mma.sync m16n8 C-fragment layout: thread (g = lane / 4, t = lane % 4) gets
// rows g and g + 8, columns 2t and 2t + 1 of each 8-column block.
#pragma once

#include <stdint.h>

namespace ttt {
namespace tc05 {

constexpr uint32_t kSwizzleNone = 0, kSwizzle128 = 2;

__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t swizzle) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)(swizzle & 7u) << 61);
}
// [rows][64] bf16 tile, K-major, 128-byte swizzle; k_step advances 16 elements
__device__ __forceinline__ uint64_t desc_k128(uint32_t saddr, int k_step) {
    return smem_desc(saddr + 32u * (uint32_t)k_step, 16, 1024, kSwizzle128);
}
// the same tile with its rows as K and its 64 columns as M or N
__device__ __forceinline__ uint64_t desc_mn128(uint32_t saddr) { return smem_desc(saddr, 2048, 1024, kSwizzle128); }
// [rows][16] bf16 tile, K-major, no swizzle (core-matrix layout above)
__device__ __forceinline__ uint64_t desc_k16(uint32_t saddr) { return smem_desc(saddr, 128, 256, kSwizzleNone); }

__host__ __device__ constexpr uint32_t kmajor16_offset(int row, int k) {
    return (uint32_t)((row & 7) * 16 + (k & 7) * 2 + (k >> 3) * 128 + (row >> 3) * 256);
}

// ---------------------------------------------------------------- TMEM allocation (one full warp)
__device__ __forceinline__ void tmem_alloc(uint32_t slot_saddr, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_saddr), "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

// ---------------------------------------------------------------- MMA (one thread)
// D[tmem] (+)= A[smem] * B[smem]; accumulate = 0 overwrites D
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// D[tmem] (+)= A[tmem] * B[smem]: A (K-major, bf16 pairs in 32-bit columns) read from tensor memory,
// in the accumulator's lane layout; column address a_tmem covers one K step of 16 elements (8 columns)
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// arrive once on the mbarrier when every tcgen05 operation this thread issued so far has completed
__device__ __forceinline__ void commit(uint32_t bar_saddr) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_saddr)
                 : "memory");
}

// ---------------------------------------------------------------- ordering
__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- TMEM -> registers (whole warp)
__device__ __forceinline__ void ld_16x256b_x1(uint32_t taddr, float (&v)[4]) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 4; i++) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void ld_16x256b_x2(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; i++) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void ld_16x256b_x8(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------- registers -> TMEM (whole warp)
// 16x128b: thread (g = lane / 4, t = lane % 4) writes rows g and g + 8 of a 16-lane group at column
// 4 r + t of repetition r: exactly the mma.sync m16n8k16 A-fragment registers (a0: row g, k pair 2t;
// a1: row g + 8; a2: row g, k pair 8 + 2t; a3: row g + 8) laid out as a K-major bf16 operand.
__device__ __forceinline__ void st_16x128b_x1(uint32_t taddr, uint32_t r0, uint32_t r1) {
    asm volatile("tcgen05.st.sync.aligned.16x128b.x1.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(r0), "r"(r1) : "memory");
}
__device__ __forceinline__ void st_16x128b_x2(uint32_t taddr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("tcgen05.st.sync.aligned.16x128b.x2.b32 [%0], {%1, %2, %3, %4};"
                 ::"r"(taddr), "r"(r0), "r"(r1), "r"(r2), "r"(r3) : "memory");
}
__device__ __forceinline__ void st_16x128b_x8(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__host__ __device__ constexpr uint32_t taddr_lane(uint32_t lane) { return lane << 16; }

}  // namespace tc05
}  // namespace ttt
