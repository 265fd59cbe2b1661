// Tensor-core building blocks shared by the flush kernels: split-precision
// tf32 warp MMAs, 2-D TMA tensor loads of the state with the 128-byte
// swizzle, and the host-side tensor-map encoding.
#pragma once
#include <cuda.h>   // CUtensorMap and its enums; the encoder is fetched from the driver at run time

#include "ss_common.cuh"

namespace ss {

// x = hi + lo with hi = x truncated to tf32 (the low 13 mantissa bits
// cleared) and lo = x - hi, exact in fp32; the MMA keeps lo's top bits, so
// hi*b + lo*b is within 2^-20 |x b| of x*b.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = __float_as_uint(x) & 0xffffe000u;
    lo = __float_as_uint(x - __uint_as_float(hi));
}
// The same, kept where it is written: splitting the 64 accumulators of the
// read-out once, ahead of its loop over basis tiles, would need 128 more
// registers.
__device__ __forceinline__ void split_tf32_here(float x, uint32_t& hi, uint32_t& lo) {
    asm volatile("and.b32 %0, %1, 0xffffe000;\n" : "=r"(hi) : "r"(__float_as_uint(x)));
    lo = __float_as_uint(x - __uint_as_float(hi));
}

// Tiled tensor copy of a 2-D box (x = column, y = row) into shared memory,
// completing on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// D += A B for one m16n8k8 tile (tf32 inputs, fp32 accumulators).
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The state tile arrives as dv/32 boxes of dk rows x 32 floats (128 bytes)
// with the 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8).
// Byte offset of element (row, col):
template <int K>
__device__ __forceinline__ int tile_off(int row, int col) {
    const int cc = col & 31;
    return (col >> 5) * (K * 128) + row * 128 + ((((cc >> 2) ^ (row & 7)) << 4) | ((cc & 3) << 2));
}

// Tensor map of the state viewed as (B*H*dk) rows of dv floats, boxes of
// dk rows x 32 floats, 128-byte swizzle of 16-byte chunks, or of 32-byte
// chunks with atom32 (host; cached per buffer and swizzle).
cudaError_t state_tensor_map(const float* state, long long rows, int K, int V, CUtensorMap* out,
                             bool atom32 = false);

// Issue (one thread) the dv/32 swizzled boxes of head u's state tile.
template <int K, int V>
__device__ __forceinline__ void issue_state_tile(const CUtensorMap* map, long long u, unsigned char* dst, uint64_t* bar) {
    mbar_expect_tx(bar, K * V * 4);
#pragma unroll
    for (int bx = 0; bx < V / 32; ++bx) tma_load_2d(dst + bx * K * 128, map, 32 * bx, int(u * K), bar);
}

}  // namespace ss
