// decode.cu -- falcon_decode_step: one token of the recurrence for every
// (sequence, head), with the fp32 state read and written in place.
//
// For one head, with x = k_prev (the prefix-aligned key, "Fast Weight
// Attention for Continual Learning", authors' abstract; x = k for the same-step
// association of Kaczmarz Linear Attention) and y = v:
//   beta = eta / (||x||^2 + eps)
//   r_i  = S_i . x,   s_i = S_i . q          (one pass over row i of S)
//   Falcon-1:  u_i = beta (y_i - alpha r_i)   Falcon-1A:  u_i = beta y_i
//   o_i  = alpha s_i + u_i (x . q)           (read after write)
//   S_i <- alpha S_i + u_i x                 (written back in the same pass)
//   k_prev <- k
// The state dominates the traffic (2 * dv * dk * 4 bytes per head), so the
// kernel is bound by HBM bandwidth: each warp streams 16 whole rows (coalesced
// 128-bit loads for dk = 128), reduces the 32 partial dot products of those
// rows with a transpose-reduce (31 shuffles) and writes the rows back.
#include "common.cuh"
#include "launch.h"

namespace falcon {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kRowsPerWarp = 16;  // 16 rows x {S.x, S.q} = 32 partial sums

template <int VPL> struct Vec;
template <> struct Vec<1> {
    static __device__ __forceinline__ void ld(const float *p, float (&x)[1]) { x[0] = __ldcs(p); }
    static __device__ __forceinline__ void st(float *p, const float (&x)[1]) { __stcs(p, x[0]); }
};
template <> struct Vec<2> {
    static __device__ __forceinline__ void ld(const float *p, float (&x)[2]) {
        const float2 a = __ldcs(reinterpret_cast<const float2 *>(p));
        x[0] = a.x; x[1] = a.y;
    }
    static __device__ __forceinline__ void st(float *p, const float (&x)[2]) {
        __stcs(reinterpret_cast<float2 *>(p), make_float2(x[0], x[1]));
    }
};
template <> struct Vec<4> {
    static __device__ __forceinline__ void ld(const float *p, float (&x)[4]) {
        const float4 a = __ldcs(reinterpret_cast<const float4 *>(p));
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    }
    static __device__ __forceinline__ void st(float *p, const float (&x)[4]) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
    }
};

// 32 per-lane partial sums in, lane l returns the warp-wide total of value l.
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
    for (int off = 16, n = 16; off >= 1; off >>= 1, n >>= 1) {
        const bool hi = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < n; ++i) {
            const float send = hi ? v[i] : v[i + n];
            const float keep = hi ? v[i + n] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0];
}

template <int DK, typename IO, bool REGRESSION>
__global__ void __launch_bounds__(kDecThreads, 2)
decode_kernel(DecodeParams p) {
    constexpr int VPL = DK / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long nh = blockIdx.x;
    const int dv = p.dv;
    float *S = p.S + nh * (size_t)dv * DK;
    IO *kp = reinterpret_cast<IO *>(p.k_prev) + nh * (size_t)DK;
    const IO *qh = reinterpret_cast<const IO *>(p.q) + nh * (size_t)DK;
    const IO *kh = reinterpret_cast<const IO *>(p.k) + nh * (size_t)DK;
    const IO *vh = reinterpret_cast<const IO *>(p.v) + nh * (size_t)dv;
    IO *oh = reinterpret_cast<IO *>(p.o) + nh * (size_t)dv;

    float x[VPL], qv[VPL];
    const IO *xs = p.same_step ? kh : kp;   // same-step association: the current key
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        x[j] = Io<IO>::ld(xs, lane * VPL + j);
        qv[j] = Io<IO>::ld(qh, lane * VPL + j);
    }
    float xx = 0.f, xq = 0.f;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        xx += x[j] * x[j];
        xq += x[j] * qv[j];
    }
    xx = warp_sum(xx);
    xq = warp_sum(xq);
    const float a = p.alpha[nh];
    const float beta = step_size(p.eta[nh], xx, p.eps);

    __syncthreads();  // every warp holds x = k_prev before it is replaced
    if (warp == 0) {
#pragma unroll
        for (int j = 0; j < VPL; ++j) kp[lane * VPL + j] = kh[lane * VPL + j];
    }

    for (int base = warp * kRowsPerWarp; base < dv; base += kDecWarps * kRowsPerWarp) {
        float s[kRowsPerWarp][VPL];
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            if (base + i < dv) Vec<VPL>::ld(S + (size_t)(base + i) * DK + lane * VPL, s[i]);
            else {
#pragma unroll
                for (int j = 0; j < VPL; ++j) s[i][j] = 0.f;
            }
        }
        float part[32];
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            float r = 0.f, sq = 0.f;
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                r += s[i][j] * x[j];
                sq += s[i][j] * qv[j];
            }
            part[2 * i] = r;
            part[2 * i + 1] = sq;
        }
        const float tot = transpose_reduce32(part, lane);       // lane 2i: S_i.x, lane 2i+1: S_i.q
        const float other = __shfl_xor_sync(0xffffffffu, tot, 1);
        const int row = base + (lane >> 1);
        float u = 0.f;
        if ((lane & 1) == 0 && row < dv) {
            const float y = Io<IO>::ld(vh, row);
            u = REGRESSION ? beta * (y - a * tot) : beta * y;
            Io<IO>::st(oh, row, a * other + u * xq);
        }
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const float ui = __shfl_sync(0xffffffffu, u, 2 * i);
            if (base + i < dv) {
#pragma unroll
                for (int j = 0; j < VPL; ++j) s[i][j] = a * s[i][j] + ui * x[j];
                Vec<VPL>::st(S + (size_t)(base + i) * DK + lane * VPL, s[i]);
            }
        }
    }
}

template <int DK, typename IO>
static cudaError_t launch_dec_t(const DecodeParams &p, cudaStream_t s) {
    const long grid = (long)p.N * p.H;
    if (grid == 0) return cudaSuccess;
    if (p.regression) decode_kernel<DK, IO, true><<<(unsigned)grid, kDecThreads, 0, s>>>(p);
    else decode_kernel<DK, IO, false><<<(unsigned)grid, kDecThreads, 0, s>>>(p);
    return cudaGetLastError();
}

template <typename IO>
static cudaError_t launch_dec_io(const DecodeParams &p, cudaStream_t s) {
    switch (p.dk) {
        case 32: return launch_dec_t<32, IO>(p, s);
        case 64: return launch_dec_t<64, IO>(p, s);
        case 128: return launch_dec_t<128, IO>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode(const DecodeParams &p, cudaStream_t s) {
    return p.io_bf16 ? launch_dec_io<__nv_bfloat16>(p, s) : launch_dec_io<float>(p, s);
}

}  // namespace falcon
