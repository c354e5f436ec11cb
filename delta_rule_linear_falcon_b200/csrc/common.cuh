// common.cuh -- small device helpers shared by the libfalcon kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace falcon {

// Error word codes a kernel may set (read and cleared by falcon_check_device_errors).
enum : int { kDevErrNone = 0, kDevErrGeometry = 1, kDevErrTimeout = 2 };

// Element access for the two I/O dtypes. Values are widened to fp32.
template <typename IO> struct Io;

// ld/st convert at the access. cvt and zero serve code that keeps loaded values in the input
// type until it needs them (a prefetch queue), so that no instruction waits on those loads early.
template <> struct Io<float> {
    static __device__ __forceinline__ float ld(const float *p, size_t i) { return p[i]; }
    static __device__ __forceinline__ float cvt(float x) { return x; }
    static __device__ __forceinline__ float zero() { return 0.f; }
    static __device__ __forceinline__ void st(float *p, size_t i, float x) { p[i] = x; }
    // 8 consecutive elements starting at i (i multiple of 8, 16-byte aligned rows)
    static __device__ __forceinline__ void ld8(const float *p, size_t i, float (&x)[8]) {
        const float4 a = *reinterpret_cast<const float4 *>(p + i);
        const float4 b = *reinterpret_cast<const float4 *>(p + i + 4);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
    static __device__ __forceinline__ void st2(float *p, size_t i, float a, float b) {
        *reinterpret_cast<float2 *>(p + i) = make_float2(a, b);
    }
};

template <> struct Io<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16 *p, size_t i) {
        return __bfloat162float(p[i]);
    }
    static __device__ __forceinline__ float cvt(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 zero() { return __float2bfloat16(0.f); }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, size_t i, float x) {
        p[i] = __float2bfloat16_rn(x);
    }
    static __device__ __forceinline__ void ld8(const __nv_bfloat16 *p, size_t i, float (&x)[8]) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p + i);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(h[j]);
            x[2 * j] = f.x;
            x[2 * j + 1] = f.y;
        }
    }
    static __device__ __forceinline__ void st2(__nv_bfloat16 *p, size_t i, float a, float b) {
        *reinterpret_cast<__nv_bfloat162 *>(p + i) = __floats2bfloat162_rn(a, b);
    }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Normalised step size beta = eta / (norm_sum + eps); a zero denominator
// (zero key and eps = 0) means no write.
__device__ __forceinline__ float step_size(float eta, float norm_sum, float eps) {
    const float den = norm_sum + eps;
    return den > 0.f ? eta / den : 0.f;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ void set_error(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}

}  // namespace falcon
