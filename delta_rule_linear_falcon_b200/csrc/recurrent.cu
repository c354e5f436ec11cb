// recurrent.cu -- falcon_fwd_recurrent: the literal per-token recurrence with an
// fp32 state (the recurrent form of "Fast Weight Attention for Continual
// Learning": authors' abstract; ai.info overview, Methodology in Plain English).
//
// One CTA per (b, h). Thread i owns row i of S in registers (d_k padded to
// DKMAX); keys and values of the last w pairs live in a ring in shared memory.
// The inputs of step t+1 are loaded into registers while step t computes, so
// the per-step latency is two barriers and the row arithmetic.
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
constexpr int kRecMaxWindow = 64;

template <typename IO, bool REGRESSION, int DKMAX>
__global__ void __launch_bounds__(kRecThreads)
recurrent_kernel(RecParams p) {
    extern __shared__ float smem[];
    const int dk = p.dk, dv = p.dv, W = p.window;
    float *sX = smem;                   // W x DKMAX key ring (zero padded)
    float *sY = sX + (size_t)W * DKMAX; // W x dv   value ring
    float *sQ = sY + (size_t)W * dv;    // 2 x DKMAX queries (double buffered)

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

    for (int idx = tid; idx < W * (DKMAX + dv) + 2 * DKMAX; idx += kRecThreads) smem[idx] = 0.f;

    const bool has_row = tid < dv;
    float S[DKMAX];
#pragma unroll
    for (int c = 0; c < DKMAX; ++c)
        S[c] = (has_row && p.S0 && c < dk) ? p.S0[(bh * (size_t)dv + tid) * dk + c] : 0.f;

    // registers holding the inputs of the step about to be staged
    auto load_x = [&](int t) -> float {   // key half of pair t, coordinate tid
        if (tid >= dk) return 0.f;
        if (p.same_step) return Io<IO>::ld(k, (size_t)t * dk + tid);
        if (t >= 1) return Io<IO>::ld(k, (size_t)(t - 1) * dk + tid);
        return kp ? Io<IO>::ld(kp, tid) : 0.f;
    };
    float xr = 0.f, qr = 0.f, yr = 0.f, ar = 1.f, er = 0.f;
    if (T > 0) {
        xr = load_x(0);
        qr = tid < dk ? Io<IO>::ld(q, tid) : 0.f;
        yr = has_row ? Io<IO>::ld(v, tid) : 0.f;
        ar = alpha[0];
        er = eta[0];
    }
    __syncthreads();

    int slot = 0;
    for (int t = 0; t < T; ++t) {
        // (A) stage pair t and q_t, then start loading step t+1
        if (tid < dk) {
            sX[slot * DKMAX + tid] = xr;
            sQ[(t & 1) * DKMAX + tid] = qr;
        }
        if (has_row) sY[slot * dv + tid] = yr;
        const float a = ar, e = er;
        if (t + 1 < T) {
            xr = load_x(t + 1);
            qr = tid < dk ? Io<IO>::ld(q, (size_t)(t + 1) * dk + tid) : 0.f;
            yr = has_row ? Io<IO>::ld(v, (size_t)(t + 1) * dv + tid) : 0.f;
            ar = alpha[t + 1];
            er = eta[t + 1];
        }
        __syncthreads();

        // (B) window step size (every thread computes it from the ring)
        const int nw = t + 1 < W ? t + 1 : W;
        float ns = 0.f;
        {
            int sl = slot;
            for (int m = 0; m < nw; ++m) {
                const float *x = sX + sl * DKMAX;
#pragma unroll 8
                for (int c = 0; c < DKMAX; ++c) ns += x[c] * x[c];
                sl = sl == 0 ? W - 1 : sl - 1;
            }
        }
        const float beta = step_size(e, ns, p.eps);

        // (C) row update and the read after the write
        if (has_row) {
#pragma unroll
            for (int c = 0; c < DKMAX; ++c) S[c] *= a;  // Sbar
            if (W == 1) {
                const float *x = sX;  // slot 0
                float r = 0.f;
#pragma unroll
                for (int c = 0; c < DKMAX; ++c) r += S[c] * x[c];
                const float coef = REGRESSION ? beta * (r - sY[tid]) : -beta * sY[tid];
#pragma unroll
                for (int c = 0; c < DKMAX; ++c) S[c] -= coef * x[c];
            } else {
                float coef[kRecMaxWindow];
                int sl = slot;
                for (int m = 0; m < nw; ++m) {
                    const float *x = sX + sl * DKMAX;
                    if (REGRESSION) {
                        float r = 0.f;
#pragma unroll
                        for (int c = 0; c < DKMAX; ++c) r += S[c] * x[c];
                        coef[m] = beta * (r - sY[sl * dv + tid]);
                    } else {
                        coef[m] = -beta * sY[sl * dv + tid];
                    }
                    sl = sl == 0 ? W - 1 : sl - 1;
                }
                sl = slot;
                for (int m = 0; m < nw; ++m) {
                    const float *x = sX + sl * DKMAX;
                    const float cm = coef[m];
#pragma unroll
                    for (int c = 0; c < DKMAX; ++c) S[c] -= cm * x[c];
                    sl = sl == 0 ? W - 1 : sl - 1;
                }
            }
            const float *qq = sQ + (t & 1) * DKMAX;
            float out = 0.f;
#pragma unroll
            for (int c = 0; c < DKMAX; ++c) out += S[c] * qq[c];
            Io<IO>::st(o, (size_t)t * dv + tid, out);
        }
        slot = slot + 1 == W ? 0 : slot + 1;
        __syncthreads();
    }

    if (p.S_out && has_row) {
        float *So = p.S_out + (bh * (size_t)dv + tid) * dk;
#pragma unroll
        for (int c = 0; c < DKMAX; ++c)
            if (c < dk) So[c] = S[c];
    }
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

static int dk_max(int dk) { return dk <= 32 ? 32 : (dk <= 64 ? 64 : 128); }

size_t recurrent_smem_bytes(int dk, int dv, int window) {
    const int D = dk_max(dk);
    return sizeof(float) * ((size_t)window * (D + dv) + 2 * D);
}

template <typename IO, bool REG, int DKMAX>
static cudaError_t launch_rec(const RecParams &p, cudaStream_t s) {
    const size_t smem = recurrent_smem_bytes(p.dk, p.dv, p.window);
    auto kern = recurrent_kernel<IO, REG, DKMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long grid = (long)p.B * p.H;
    if (grid == 0) return cudaSuccess;
    kern<<<(unsigned)grid, kRecThreads, smem, s>>>(p);
    return cudaGetLastError();
}

template <typename IO, bool REG>
static cudaError_t launch_rec_dk(const RecParams &p, cudaStream_t s) {
    switch (dk_max(p.dk)) {
        case 32: return launch_rec<IO, REG, 32>(p, s);
        case 64: return launch_rec<IO, REG, 64>(p, s);
        default: return launch_rec<IO, REG, 128>(p, s);
    }
}

cudaError_t launch_recurrent(const RecParams &p, cudaStream_t s) {
    if (p.dk > 128 || p.dv > kRecThreads || p.window > kRecMaxWindow || p.window < 1) return cudaErrorInvalidValue;
    const bool reg = p.regression;
    if (p.io_bf16) return reg ? launch_rec_dk<__nv_bfloat16, true>(p, s) : launch_rec_dk<__nv_bfloat16, false>(p, s);
    return reg ? launch_rec_dk<float, true>(p, s) : launch_rec_dk<float, false>(p, s);
}

}  // namespace falcon
