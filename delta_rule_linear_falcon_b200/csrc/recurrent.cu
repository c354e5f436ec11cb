// recurrent.cu -- falcon_fwd_recurrent: the literal per-token recurrence with an
// fp32 state (the recurrent form of "Fast Weight Attention for Continual
// Learning": authors' abstract; ai.info overview, Methodology in Plain English).
//
// One CTA per (b, h). Thread i owns row i of S (d_v rows of d_k fp32 in shared
// memory, padded stride so that the row-per-thread walk is bank-conflict
// free). Keys and values of the last w pairs live in a ring in shared memory.
// Per step t (0-based, pair j = t - m for window slot m):
//   Sbar = alpha_t S
//   beta = eta_t / (sum_m ||x_{t-m}||^2 + eps)
//   regression:     S_i = Sbar_i - beta sum_m (Sbar_i . x_{t-m} - y_{t-m,i}) x_{t-m}
//   inner product:  S_i = Sbar_i + beta sum_m y_{t-m,i} x_{t-m}
//   o_{t,i} = S_i . q_t                       (read after write)
#include "common.cuh"
#include "launch.h"

namespace falcon {

constexpr int kRecThreads = 128;

template <typename IO, bool REGRESSION>
__global__ void __launch_bounds__(kRecThreads)
recurrent_kernel(RecParams p) {
    extern __shared__ float smem[];
    const int dk = p.dk, dv = p.dv, W = p.window;
    const int ldS = dk + 1;
    float *sS = smem;                        // dv x ldS
    float *sX = sS + (size_t)dv * ldS;       // W x dk  key ring
    float *sY = sX + (size_t)W * dk;         // W x dv  value ring
    float *sN = sY + (size_t)W * dv;         // W       squared key norms
    float *sQ = sN + W;                      // dk      current query
    float *sBeta = sQ + dk;                  // 1

    const int tid = threadIdx.x;
    const long bh = blockIdx.x;
    const int T = p.T;
    const IO *q = reinterpret_cast<const IO *>(p.q) + bh * (size_t)T * dk;
    const IO *k = reinterpret_cast<const IO *>(p.k) + bh * (size_t)T * dk;
    const IO *v = reinterpret_cast<const IO *>(p.v) + bh * (size_t)T * dv;
    const IO *kp = p.k_prev ? reinterpret_cast<const IO *>(p.k_prev) + bh * (size_t)dk : nullptr;
    const float *alpha = p.alpha + bh * (size_t)T;
    const float *eta = p.eta + bh * (size_t)T;
    IO *o = reinterpret_cast<IO *>(p.o) + bh * (size_t)T * dv;

    for (int idx = tid; idx < dv * dk; idx += kRecThreads) {
        const int i = idx / dk, c = idx % dk;
        sS[i * ldS + c] = p.S0 ? p.S0[bh * (size_t)dv * dk + idx] : 0.f;
    }
    for (int idx = tid; idx < W * (dk + dv + 1); idx += kRecThreads) sX[idx] = 0.f;  // ring + norms
    __syncthreads();

    for (int t = 0; t < T; ++t) {
        const int slot = t % W;
        // (A) stage pair t = (x_t, y_t) and the query
        for (int c = tid; c < dk; c += kRecThreads) {
            float x;
            if (t >= 1) x = Io<IO>::ld(k, (size_t)(t - 1) * dk + c);
            else x = kp ? Io<IO>::ld(kp, c) : 0.f;
            sX[slot * dk + c] = x;
            sQ[c] = Io<IO>::ld(q, (size_t)t * dk + c);
        }
        for (int i = tid; i < dv; i += kRecThreads) sY[slot * dv + i] = Io<IO>::ld(v, (size_t)t * dv + i);
        __syncthreads();
        // (B) squared norm of x_t and the step size over the window
        if (tid < 32) {
            float s = 0.f;
            for (int c = tid; c < dk; c += 32) s += sX[slot * dk + c] * sX[slot * dk + c];
            s = warp_sum(s);
            if (tid == 0) {
                sN[slot] = s;
                const int nw = t + 1 < W ? t + 1 : W;
                float ns = 0.f;
                for (int m = 0; m < nw; ++m) ns += sN[(t - m) % W];
                sBeta[0] = step_size(eta[t], ns, p.eps);
            }
        }
        __syncthreads();
        // (C) row updates and the read after the write
        const float a = alpha[t];
        const float beta = sBeta[0];
        const int nw = t + 1 < W ? t + 1 : W;
        for (int i = tid; i < dv; i += kRecThreads) {
            float *Si = sS + i * ldS;
            float coef[64];
            if (REGRESSION) {
                for (int m = 0; m < nw; ++m) {
                    const float *x = sX + ((t - m) % W) * dk;
                    float r = 0.f;
                    for (int c = 0; c < dk; ++c) r += Si[c] * x[c];
                    coef[m] = beta * (a * r - sY[((t - m) % W) * dv + i]);  // beta (Sbar x - y)
                }
            } else {
                for (int m = 0; m < nw; ++m) coef[m] = -beta * sY[((t - m) % W) * dv + i];
            }
            float out = 0.f;
            for (int c = 0; c < dk; ++c) {
                float s = a * Si[c];
                for (int m = 0; m < nw; ++m) s -= coef[m] * sX[((t - m) % W) * dk + c];
                Si[c] = s;
                out += s * sQ[c];
            }
            Io<IO>::st(o, (size_t)t * dv + i, out);
        }
        __syncthreads();
    }

    if (p.S_out)
        for (int idx = tid; idx < dv * dk; idx += kRecThreads)
            p.S_out[bh * (size_t)dv * dk + idx] = sS[(idx / dk) * ldS + idx % dk];
    if (p.k_last) {
        IO *kl = reinterpret_cast<IO *>(p.k_last) + bh * (size_t)dk;
        for (int c = tid; c < dk; c += kRecThreads) {
            float x = 0.f;
            if (T >= 1) x = Io<IO>::ld(k, (size_t)(T - 1) * dk + c);
            else if (kp) x = Io<IO>::ld(kp, c);
            Io<IO>::st(kl, c, x);
        }
    }
}

size_t recurrent_smem_bytes(int dk, int dv, int window) {
    return sizeof(float) * ((size_t)dv * (dk + 1) + (size_t)window * (dk + dv + 1) + dk + 1);
}

template <typename IO, bool REG>
static cudaError_t launch_rec(const RecParams &p, cudaStream_t s) {
    const size_t smem = recurrent_smem_bytes(p.dk, p.dv, p.window);
    auto kern = recurrent_kernel<IO, REG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long grid = (long)p.B * p.H;
    if (grid == 0) return cudaSuccess;
    kern<<<(unsigned)grid, kRecThreads, smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_recurrent(const RecParams &p, cudaStream_t s) {
    const bool reg = p.regression;
    if (p.io_bf16) return reg ? launch_rec<__nv_bfloat16, true>(p, s) : launch_rec<__nv_bfloat16, false>(p, s);
    return reg ? launch_rec<float, true>(p, s) : launch_rec<float, false>(p, s);
}

}  // namespace falcon
