// chunk_mma.cuh -- warp-level bf16 tensor-core helpers (ldmatrix + mma.sync
// m16n8k16, fp32 accumulate) for the chunk-parallel kernel.
//
// Fragment conventions (per warp, lane = threadIdx.x & 31):
//   A 16x16 (row-major):  a[0] rows 0-7  k 0-7,  a[1] rows 8-15 k 0-7,
//                         a[2] rows 0-7  k 8-15, a[3] rows 8-15 k 8-15.
//   B 16x8:               b0 k 0-7, b1 k 8-15 (column n = lane / 4).
//   C 16x8 fp32:          c[0], c[1] at (lane/4, 2*(lane%4) + {0,1}),
//                         c[2], c[3] at (lane/4 + 8, same columns).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace falcon {

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A tile (m0..m0+15, k0..k0+15) from row-major storage [M][ld].
__device__ __forceinline__ void load_a_rm(uint32_t (&a)[4], const bf16 *base, int ld, int m0, int k0,
                                          int lane) {
    ldsm_x4(a, base + (m0 + (lane & 15)) * ld + k0 + ((lane >> 4) << 3));
}

// A tile (m0.., k0..) from storage [K][ld] holding A transposed (M contiguous).
__device__ __forceinline__ void load_a_km(uint32_t (&a)[4], const bf16 *base, int ld, int m0, int k0,
                                          int lane) {
    const int mi = lane >> 3, r = lane & 7;
    ldsm_x4_t(a, base + (k0 + ((mi >> 1) << 3) + r) * ld + m0 + ((mi & 1) << 3));
}

// Two B tiles (n0..n0+7 and n0+8..n0+15, k0..k0+15) from storage [N][ld]
// (K contiguous). b = {b0(n0), b1(n0), b0(n0+8), b1(n0+8)}.
__device__ __forceinline__ void load_b_nk(uint32_t (&b)[4], const bf16 *base, int ld, int n0, int k0,
                                          int lane) {
    ldsm_x4(b, base + (n0 + (lane & 7) + ((lane >> 4) << 3)) * ld + k0 + (((lane >> 3) & 1) << 3));
}

// Two B tiles from storage [K][ld] (N contiguous).
__device__ __forceinline__ void load_b_kn(uint32_t (&b)[4], const bf16 *base, int ld, int n0, int k0,
                                          int lane) {
    const int mi = lane >> 3, r = lane & 7;
    ldsm_x4_t(b, base + (k0 + ((mi & 1) << 3) + r) * ld + n0 + ((mi >> 1) << 3));
}

}  // namespace falcon
