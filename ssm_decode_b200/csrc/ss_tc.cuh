// Fifth-generation tensor-core (tcgen05) building blocks for sm_100a: tensor
// memory (TMEM) allocation, tf32 MMAs whose operands are shared-memory matrix
// descriptors or (for A) a TMEM address, commits of MMA groups to mbarriers,
// TMEM loads and stores by warps, and the fences that order them against
// ordinary thread execution.  Only one CTA of a cluster (cta_group::1) and no
// multicast are used.
#pragma once
#include "ss_common.cuh"

namespace ss {
namespace tc {

// Shared-memory matrix descriptor: start address, leading and stride byte
// offsets (each in 16-byte units, 14 bits), the descriptor version of this
// architecture (1, bits 46-47) and the layout type (bits 61-63).  Two
// 128-byte-swizzled layouts are used, both made of column blocks of 32 fp32
// values (128-byte rows) whose swizzle atoms are 1024-byte aligned:
//   SW128 (type 2):     16-byte chunk c of row r stored at chunk c ^ (r % 8);
//                       K-major operands (rows are M / N indices holding 32
//                       consecutive K elements): stride offset = bytes between
//                       groups of 8 rows, leading offset unused (16); the start
//                       address moves 32 bytes per K step of 8 inside a row.
//   SW128_32B (type 1): 32-byte chunk c of row r stored at chunk c ^ (r % 4);
//                       the only layout the tensor core takes for MN-major
//                       tf32 operands (rows are K indices holding 32
//                       consecutive M / N elements): leading offset = bytes
//                       between 32-element M / N blocks, stride offset = bytes
//                       between groups of 4 rows (512 for adjacent rows).
constexpr uint32_t LAYOUT_SW128 = 2, LAYOUT_SW128_32B = 1;
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
           (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (uint64_t(layout) << 61);
}

// Instruction descriptor of a dense tf32 x tf32 -> fp32 MMA of shape M x N
// (K = 8 per instruction): D format fp32 (bits 4-5 = 1), A and B tf32
// (bits 7-9 and 10-12 = 2), A / B major (bits 15 / 16: 0 = K-major,
// 1 = MN-major), N / 8 in bits 17-22, M / 16 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
           (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Instruction descriptor of a dense bf16 x bf16 -> fp32 MMA (kind::f16, K = 16
// per instruction): A and B formats 1 (bf16) in bits 7-9 and 10-12, both
// K-major, N / 8 in bits 17-22, M / 16 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// D[tmem] (+)= A * B with both operands bf16 in shared memory.  One thread issues.
__device__ __forceinline__ void mma_ss_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]; acc = 0 overwrites D.  One thread issues.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]; A is K-major in TMEM (lane = row of A,
// one column per K element).  One thread issues.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// The mbarrier receives one arrival once every MMA this thread issued before
// has completed (their results are then in TMEM and their smem reads done).
__device__ __forceinline__ void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Whole warp: allocate `ncols` TMEM columns (a power of two >= 32); the base
// address is written to *dst (shared memory).
__device__ __forceinline__ void alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// Shared-memory writes of this thread become visible to the async proxy
// (tensor-core operand reads, bulk tensor stores) after a later barrier.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

// TMEM address of (lane, column).
__device__ __forceinline__ uint32_t taddr(uint32_t base, uint32_t lane, uint32_t col) {
    return base + (lane << 16) + col;
}

// Warp-wide 32x32b TMEM accesses: lane i of the warp reads / writes TMEM lane
// (32 * (warp % 4) + i), `N` consecutive 32-bit columns starting at the
// address's column.  The address's lane field must be that quarter's first lane.
__device__ __forceinline__ void ld16(uint32_t a, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(a)
        : "memory");
}
__device__ __forceinline__ void st16(uint32_t a, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(a),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// Byte offsets of element (row, col) in a buffer of column blocks of 32 fp32
// values: block col / 32 holds `rows` rows of 128 bytes.
//   sw128_off:  16-byte chunk c of row r at chunk c ^ (r % 8) (SW128);
//   sw32b_off:  32-byte chunk c of row r at chunk c ^ (r % 4) (SW128_32B, also
//               what a bulk tensor copy with CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
//               writes for a box of 32 fp32 columns).
__host__ __device__ constexpr uint32_t sw128_off(int rows, int row, int col) {
    return uint32_t((col >> 5) * (rows * 128) + row * 128 + ((((col & 31) >> 2) ^ (row & 7)) << 4) + ((col & 3) << 2));
}
// The same 16-byte-chunk swizzle for bf16 elements: column blocks of 64 values.
__host__ __device__ constexpr uint32_t sw128h_off(int rows, int row, int col) {
    return uint32_t((col >> 6) * (rows * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + ((col & 7) << 1));
}
__host__ __device__ constexpr uint32_t sw32b_off(int rows, int row, int col) {
    return uint32_t((col >> 5) * (rows * 128) + row * 128 + ((((col & 31) >> 3) ^ (row & 3)) << 5) + ((col & 7) << 2));
}

}  // namespace tc
}  // namespace ss
