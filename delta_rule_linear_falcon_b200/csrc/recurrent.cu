// recurrent.cu -- falcon_fwd_recurrent: the literal per-token recurrence with an
// fp32 state (the recurrent form of "Fast Weight Attention for Continual
// Learning": authors' abstract; ai.info overview, Methodology in Plain English).
//
// One CTA per (b, h). Thread i owns row i of S in registers (d_k padded to
// DKMAX); keys and values of the last w pairs live in a ring of w + 1 slots in
// shared memory, so a single barrier per step separates writing a slot from its
// last read. The inputs of step t + A are loaded into registers while step t
// computes (a register queue A = 3..8 steps deep, held in the input type and
// converted only when the step stages them, so that no instruction waits on a load
// before that step), which keeps global-load latency off the per-step path. The
// squared norm of each pair is reduced once, when the pair is staged (one partial
// per warp), and the window sum reads those partials. The rows are kept as
// S = sigma S' with one scale sigma per head: the decay multiplies sigma, and the
// update, in units of sigma, is one fused multiply-add per entry,
//   S' <- S' - (coef / sigma) x,   coef as below with Sbar . x = sigma (S' . x);
// sigma is folded back into the rows whenever it leaves [2^-60, 2^60] (a zero decay
// included).
// Window 1 has an instantiation of its own, without the window loops; with 128 key
// columns the row takes 128 registers, and both of these keep the rest of the kernel in
// registers too (the state row spilled before, and a step took two to three times as long).
// Per step t (0-based, pair j = t - m for window slot m):
//   Sbar = alpha_t S
//   beta = eta_t / (sum_m ||x_{t-m}||^2 + eps)
//   regression:     S_i = Sbar_i - beta sum_m (Sbar_i . x_{t-m} - y_{t-m,i}) x_{t-m}
//   inner product:  S_i = Sbar_i + beta sum_m y_{t-m,i} x_{t-m}
//   o_{t,i} = S_i . q_t                       (read after write)
// Falcon-2 / 2A (window 1): thread c also keeps the running energy n_c of key coordinate c,
// n_c <- alpha_t n_c + x_c^2, and stages the write key direction z_c = x_c / (n_c + eps) beside
// the key; the pair's norm partial is x . z, so beta = eta / (x^T D x + eps) and the row update is
//   Falcon-2:  S_i = Sbar_i - beta (Sbar_i . x - y_i) z      Falcon-2A: S_i = Sbar_i + beta y_i z
#include "common.cuh"
#include "launch.h"

namespace falcon {

constexpr int kRecThreads = 128;
constexpr int kRecWarps = kRecThreads / 32;
constexpr int kRecMaxWindow = 64;
// Steps of inputs in flight ahead of the one being computed: fewer for wide rows, whose
// longer steps cover the load latency sooner and whose state row takes more registers.
template <int DKMAX> __host__ __device__ constexpr int ahead() { return DKMAX >= 128 ? 3 : (DKMAX >= 64 ? 6 : 8); }

// Dot product of a register row with a shared-memory vector, four independent partial sums.
template <int DKMAX>
__device__ __forceinline__ float row_dot(const float (&S)[DKMAX], const float *x) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int c = 0; c < DKMAX; c += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(x + c);
        a0 = fmaf(S[c], v.x, a0);
        a1 = fmaf(S[c + 1], v.y, a1);
        a2 = fmaf(S[c + 2], v.z, a2);
        a3 = fmaf(S[c + 3], v.w, a3);
    }
    return (a0 + a1) + (a2 + a3);
}

// ONE: the window is one pair (compiled without the window loops, whose per-pair coefficients
// would otherwise take registers from the state row).
template <typename IO, bool REGRESSION, int DKMAX, bool PERCOL, bool ONE>
__global__ void __launch_bounds__(kRecThreads)
recurrent_kernel(RecParams p) {
    extern __shared__ __align__(16) float smem[];
    const int dk = p.dk, dv = p.dv, W = ONE ? 1 : p.window, RS = W + 1;
    float *sX = smem;                        // RS x DKMAX key ring (zero padded)
    float *sY = sX + (size_t)RS * DKMAX;     // RS x DVP value ring
    const int DVP = (dv + 3) & ~3;
    float *sQ = sY + (size_t)RS * DVP;       // 2 x DKMAX queries (double buffered)
    float *sN = sQ + 2 * DKMAX;              // RS x kRecWarps partial squared norms of the pairs
    float *sZ = sN + RS * kRecWarps;         // RS x DKMAX write-key directions (a copy of the key for
                                             // the other rules, so that the update and the dot product
                                             // read different arrays: when they read one, the compiler
                                             // keeps the dot product's loads for the update, 128 more
                                             // live registers beside the row)
    constexpr int kAhead = ahead<DKMAX>();

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long bh = blockIdx.x;
    const int T = p.T;
    const IO *q = reinterpret_cast<const IO *>(p.q) + bh * (size_t)T * dk;
    const IO *k = reinterpret_cast<const IO *>(p.k) + bh * (size_t)T * dk;
    const IO *v = reinterpret_cast<const IO *>(p.v) + bh * (size_t)T * dv;
    const IO *kp = p.k_prev ? reinterpret_cast<const IO *>(p.k_prev) + bh * (size_t)dk : nullptr;
    const float *alpha = p.alpha + bh * (size_t)T;
    const float *eta = p.eta + bh * (size_t)T;
    IO *o = reinterpret_cast<IO *>(p.o) + bh * (size_t)T * dv;

    for (int idx = tid; idx < RS * (DKMAX + DVP + kRecWarps) + 2 * DKMAX + RS * DKMAX; idx += kRecThreads)
        smem[idx] = 0.f;
    // running energy of key coordinate tid (per-column rules)
    float ncol = (PERCOL && p.n0 && tid < dk) ? p.n0[bh * (size_t)dk + tid] : 0.f;

    const bool has_row = tid < dv;
    float sigma = 1.f;                      // S = sigma S' (S' is the register row)
    float S[DKMAX];
#pragma unroll
    for (int c = 0; c < DKMAX; ++c)
        S[c] = (has_row && p.S0 && c < dk) ? p.S0[(bh * (size_t)dv + tid) * dk + c] : 0.f;

    const IO z0 = Io<IO>::zero();
    auto load_x = [&](int t) -> IO {   // key half of pair t, coordinate tid
        if (tid >= dk) return z0;
        if (p.same_step) return k[(size_t)t * dk + tid];
        if (t >= 1) return k[(size_t)(t - 1) * dk + tid];
        return kp ? kp[tid] : z0;
    };
    // register queue: inputs of steps t .. t + kAhead - 1, slot t % kAhead, in the input type
    IO xr[kAhead], qr[kAhead], yr[kAhead];
    float ar[kAhead], er[kAhead];
    auto fetch = [&](int t, IO &x, IO &qq, IO &y, float &a, float &e) {
        if (t < T) {
            x = load_x(t);
            qq = tid < dk ? q[(size_t)t * dk + tid] : z0;
            y = has_row ? v[(size_t)t * dv + tid] : z0;
            a = alpha[t];
            e = eta[t];
        }
    };
#pragma unroll
    for (int i = 0; i < kAhead; ++i) {
        xr[i] = z0; qr[i] = z0; yr[i] = z0; ar[i] = 1.f; er[i] = 0.f;
        fetch(i, xr[i], qr[i], yr[i], ar[i], er[i]);
    }
    __syncthreads();

    int slot = 0;
    for (int t0 = 0; t0 < T; t0 += kAhead) {
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int t = t0 + i;
            if (t >= T) break;
            // (A) stage pair t and q_t with the pair's squared-norm partial, refill the queue slot
            const float xi = Io<IO>::cvt(xr[i]);
            {
                float x2 = xi * xi;
                if (PERCOL) {   // x . z with z = D x: the D-weighted squared norm
                    ncol = ar[i] * ncol + x2;
                    const float den = ncol + p.eps;
                    const float z = (tid < dk && den > 0.f) ? xi / den : 0.f;
                    if (tid < dk) sZ[slot * DKMAX + tid] = z;   // entries dk.. stay zero
                    x2 = z * xi;
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) x2 += __shfl_xor_sync(0xffffffffu, x2, off);
                if (lane == 0) sN[slot * kRecWarps + warp] = x2;
            }
            if (tid < dk) {
                sX[slot * DKMAX + tid] = xi;
                if (!PERCOL && ONE) sZ[slot * DKMAX + tid] = xi;
                sQ[(t & 1) * DKMAX + tid] = Io<IO>::cvt(qr[i]);
            }
            if (has_row) sY[slot * DVP + tid] = Io<IO>::cvt(yr[i]);
            const float a = ar[i], e = er[i];
            fetch(t + kAhead, xr[i], qr[i], yr[i], ar[i], er[i]);
            __syncthreads();

            // (B) window step size from the staged partial norms
            const int nw = t + 1 < W ? t + 1 : W;
            float ns = 0.f;
            {
                int sl = slot;
                for (int m = 0; m < nw; ++m) {
#pragma unroll
                    for (int w = 0; w < kRecWarps; ++w) ns += sN[sl * kRecWarps + w];
                    sl = sl == 0 ? RS - 1 : sl - 1;
                }
            }
            const float beta = step_size(e, ns, p.eps);

            // (C) row update and the read after the write
            // Sbar = (a sigma) S'; the block-uniform scale is folded into the rows if it would leave range
            float sc = a * sigma;
            if (!(sc >= 0x1p-60f && sc <= 0x1p60f)) {
#pragma unroll
                for (int c = 0; c < DKMAX; ++c) S[c] *= sc;
                sc = 1.f;
            }
            sigma = sc;
            const float inv = 1.f / sc;
            if (has_row) {
                if (ONE || W == 1) {
                    const float *x = sX + slot * DKMAX;
                    const float *zw = sZ + slot * DKMAX;   // write-key direction
                    const float y = sY[slot * DVP + tid] * inv;
                    const float coef = REGRESSION ? beta * (row_dot<DKMAX>(S, x) - y) : -beta * y;   // / sigma
#pragma unroll
                    for (int c = 0; c < DKMAX; c += 4) {
                        const float4 xv = *reinterpret_cast<const float4 *>(zw + c);
                        S[c] -= coef * xv.x;
                        S[c + 1] -= coef * xv.y;
                        S[c + 2] -= coef * xv.z;
                        S[c + 3] -= coef * xv.w;
                    }
                } else {
                    float coef[kRecMaxWindow];
                    int sl = slot;
                    for (int m = 0; m < nw; ++m) {
                        const float y = sY[sl * DVP + tid] * inv;
                        coef[m] = REGRESSION ? beta * (row_dot<DKMAX>(S, sX + sl * DKMAX) - y) : -beta * y;
                        sl = sl == 0 ? RS - 1 : sl - 1;
                    }
                    sl = slot;
                    for (int m = 0; m < nw; ++m) {
                        const float *x = sX + sl * DKMAX;
                        const float cm = coef[m];
#pragma unroll
                        for (int c = 0; c < DKMAX; ++c) S[c] -= cm * x[c];
                        sl = sl == 0 ? RS - 1 : sl - 1;
                    }
                }
                Io<IO>::st(o, (size_t)t * dv + tid, sigma * row_dot<DKMAX>(S, sQ + (t & 1) * DKMAX));
            }
            slot = slot + 1 == RS ? 0 : slot + 1;
        }
    }

    if (PERCOL && p.n_out && tid < dk) p.n_out[bh * (size_t)dk + tid] = ncol;
    if (p.S_out && has_row) {
        float *So = p.S_out + (bh * (size_t)dv + tid) * dk;
#pragma unroll
        for (int c = 0; c < DKMAX; ++c)
            if (c < dk) So[c] = sigma * S[c];
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
    const size_t rs = (size_t)window + 1, dvp = (size_t)((dv + 3) & ~3);
    return sizeof(float) * (rs * (D + dvp + kRecWarps) + 2 * D + rs * D);   // + write-key ring
}

template <typename IO, bool REG, int DKMAX>
static cudaError_t launch_rec(const RecParams &p, cudaStream_t s) {
    const size_t smem = recurrent_smem_bytes(p.dk, p.dv, p.window);
    auto kern = p.per_column      ? recurrent_kernel<IO, REG, DKMAX, true, true>
                : p.window == 1 ? recurrent_kernel<IO, REG, DKMAX, false, true>
                                : recurrent_kernel<IO, REG, DKMAX, false, false>;
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
    if (p.per_column && p.window != 1) return cudaErrorInvalidValue;
    const bool reg = p.regression;
    if (p.io_bf16) return reg ? launch_rec_dk<__nv_bfloat16, true>(p, s) : launch_rec_dk<__nv_bfloat16, false>(p, s);
    return reg ? launch_rec_dk<float, true>(p, s) : launch_rec_dk<float, false>(p, s);
}

}  // namespace falcon
