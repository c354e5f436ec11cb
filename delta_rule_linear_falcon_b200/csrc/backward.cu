// backward.cu -- falcon_bwd_recurrent: gradients of the recurrent form (reverse mode
// through the per-token recurrence of "Fast Weight Attention for Continual Learning",
// authors' abstract; the pages give the forward rules only, so these are their
// derivatives) for Falcon-1/1A/3/3A, with the same-step flag, an initial state and a
// cached key. fp32 state and fp32 arithmetic; q, k, v in the I/O dtype, every gradient
// in fp32.
//
// The rows of S evolve independently given the keys, so each (b, h) is split into slices of
// 8 value rows, one CTA of 128 threads each; every sum over value rows that the backward forms
// (dq, dx, dbeta, dalpha) feeds only an output gradient, so each slice adds its part to the
// zeroed outputs with atomics. With U = dL/dS after step t (starting from dS_T),
// step t (0-based, pairs j = t - m of window slot m, Sbar = alpha_t S_{t-1}) gives
//   U += dO_t q_t^T,                       dq_t = S_t^T dO_t
//   regression (r_m = Sbar x_m - y_m, S_t = Sbar - beta sum_m r_m x_m^T):
//     dbeta = -sum_m r_m^T U x_m,   dr_m = -beta U x_m,   dy_m = -dr_m
//     dx_m  = -beta U^T r_m + Sbar^T dr_m,   dSbar = U + sum_m dr_m x_m^T
//   inner product (S_t = Sbar + beta sum_m y_m x_m^T):
//     dbeta = sum_m y_m^T U x_m,   dy_m = beta U x_m,   dx_m = beta U^T y_m,   dSbar = U
//   beta = eta_t / (N + eps), N = sum_m ||x_m||^2 (no gradient through it when N + eps = 0):
//     deta_t = dbeta / (N + eps),   dx_m += -2 dbeta beta / (N + eps) x_m
//   dalpha_t = <dSbar, S_{t-1}>,   U <- alpha_t dSbar
// and dx_m, dy_m are scattered to the key and value rows of pair j (x_j = k_{j-1}, k_prev
// for j = 0, or k_j with the same-step flag); dS0 is the last U.
//
// The states are not kept: a first forward pass stores S at the start of every segment of
// C steps in the workspace, and the reverse sweep re-runs each segment forward from its
// checkpoint into a buffer of C + 1 states before walking it backwards. The slice's rows of U
// and of the two states a step needs (before and after it) sit in shared memory. Row products
// (U x, Sbar x, the state update) take sixteen threads per value row i, each every sixteenth
// column, reduced with four shuffles; the row stride is 16 more than a multiple of 32 floats, so
// the 32 threads of a warp (2 rows x 16 column phases) hit 32 different banks. Column products
// (S^T dO, U^T r, Sbar^T dr) take one thread per key column over the slice's rows.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace falcon {

namespace {

constexpr int kBwdRows = 8;                     // value rows per CTA (a slice of a head)
constexpr int kBwdThreads = 128;                // row products: kRowThr threads per row (all 128 threads);
                                                // column products: one thread per key column (d_k <= 128)
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kRowThr = kBwdThreads / kBwdRows; // threads per value row in the row products (16)
static_assert(32 % kRowThr == 0 && kRowThr % 4 == 0, "a warp holds whole rows; rows stay 16-byte aligned");
static_assert(kBwdRows % 2 == 0, "the column products take the rows in pairs");
constexpr int kBwdMaxWindow = 8;                // pairs per step the register prefetch holds

struct BwdSmem {
    int LD, dk, w;
    // offsets in floats; row vectors hold the kBwdRows rows of the slice
    size_t oU, oP, oA, oX, oY, oQ, oG, oUx, oR, oDr, oRed, total;
};

__host__ __device__ inline BwdSmem bwd_smem(int dk, int w) {
    BwdSmem s;
    // row stride = kRowThr mod 32 floats: the rows of a warp's row products (kRowThr threads each)
    // and a column phase fall on distinct banks
    s.LD = ((dk + 31) / 32) * 32 + kRowThr; s.dk = dk; s.w = w;
    constexpr int R = kBwdRows;
    const size_t mat = (size_t)R * s.LD;
    s.oU = 0; s.oP = mat; s.oA = 2 * mat;
    s.oX = 3 * mat;
    s.oY = s.oX + (size_t)w * dk;
    s.oQ = s.oY + (size_t)w * R;
    s.oG = s.oQ + dk;
    s.oUx = s.oG + R;
    s.oR = s.oUx + (size_t)w * R;
    s.oDr = s.oR + (size_t)w * R;
    s.oRed = s.oDr + (size_t)w * R;
    s.total = s.oRed + 2 * kBwdWarps + 4;
    return s;
}

// Sum over the CTA; every thread gets the result. Two barriers.
__device__ __forceinline__ float block_sum(float x, float *red) {
    x = warp_sum(x);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();                 // earlier readers of red are done
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kBwdWarps; ++i) s += red[i];
    return s;
}

// Sum over the kRowThr threads of a value row (lanes kRowThr i ..); all of them get it.
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
    for (int o = 1; o < kRowThr; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <typename IO>
struct BwdCtx {
    const BwdParams &p;
    const IO *q, *k, *v, *kp;
    const float *al, *et;
    int T, dk, dv, w;
    bool same;
    // element c of the key row of pair j, in the input type (0 for j < 0, or for the first pair
    // without k_prev)
    __device__ IO key_raw(long j, int c) const {
        if (j < 0) return Io<IO>::zero();
        if (same) return k[(size_t)j * dk + c];
        if (j >= 1) return k[(size_t)(j - 1) * dk + c];
        return kp ? kp[c] : Io<IO>::zero();
    }
};

template <typename IO, bool REG>
__global__ void __launch_bounds__(kBwdThreads)
bwd_recurrent_kernel(BwdParams p) {
    extern __shared__ __align__(16) float smem[];
    const int dk = p.dk, dv = p.dv, w = p.window, T = p.T, C = p.seg;
    const BwdSmem L = bwd_smem(dk, w);
    const int LD = L.LD;
    constexpr int RS = kBwdRows;                    // row stride of the slice's row vectors
    float *sU = smem + L.oU, *sP = smem + L.oP, *sA = smem + L.oA;
    float *sX = smem + L.oX, *sY = smem + L.oY, *sQ = smem + L.oQ, *sG = smem + L.oG;
    float *sUx = smem + L.oUx, *sR = smem + L.oR, *sDr = smem + L.oDr, *sRed = smem + L.oRed;
    const int tid = threadIdx.x;
    const int nsl = (dv + kBwdRows - 1) / kBwdRows;
    const size_t bh = blockIdx.x / nsl;
    const int sl = blockIdx.x % nsl, r0 = sl * kBwdRows, R = min(kBwdRows, dv - r0);   // the slice's rows
    const int ri = tid / kRowThr, rq = tid % kRowThr;   // row products: slice row ri, columns rq, rq + kRowThr, ..
    const bool rok = ri < R;
    const int cc = tid;                             // column products: key column cc over the slice's rows
    const size_t DD = (size_t)dv * dk;              // a head's state in the caller's arrays
    const size_t DS = (size_t)kBwdRows * dk;        // a slice's state in the workspace
    // Shared memory starts at zero: rows R .. kBwdRows - 1 of every row array then stay zero (each
    // writer of a row is guarded by its row), so the column products run over all kBwdRows rows.
    for (int i = tid; i < (int)L.total; i += kBwdThreads) smem[i] = 0.f;
    __syncthreads();

    BwdCtx<IO> ctx{p,
                   reinterpret_cast<const IO *>(p.q) + bh * T * dk,
                   reinterpret_cast<const IO *>(p.k) + bh * T * dk,
                   reinterpret_cast<const IO *>(p.v) + bh * T * dv,
                   p.k_prev ? reinterpret_cast<const IO *>(p.k_prev) + bh * dk : nullptr,
                   p.alpha + bh * T, p.eta + bh * T, T, dk, dv, w, p.same_step};
    const IO *q = ctx.q;
    const float *dO = p.dO + bh * T * dv;
    // every gradient array starts at zero (the launch clears them): value rows belong to one
    // slice, the rest take each slice's part by atomic adds
    float *gq = p.dq + bh * T * dk, *gk = p.dk_out + bh * T * dk, *gv = p.dv_out + bh * T * dv;
    float *gal = p.dalpha + bh * T, *get = p.deta + bh * T;
    float *gkp = (p.dk_prev && p.k_prev) ? p.dk_prev + bh * dk : nullptr;
    const int nseg = (T + C - 1) / C;
    float *ckpt = p.ws + ((size_t)bh * nsl + sl) * (size_t)(nseg + C + 1) * DS;   // nseg checkpoints,
    float *buf = ckpt + (size_t)nseg * DS;                                         // then C + 1 states

    // dense dv x dk (global) <-> padded rows (shared): a warp per row, lanes along it
    const int warp = tid >> 5, lane = tid & 31;
    auto store_state = [&](float *dst, const float *src) {
        for (int i = warp; i < R; i += kBwdWarps)
            for (int c = lane; c < dk; c += 32) dst[(size_t)i * dk + c] = src[i * LD + c];
    };
    auto load_state = [&](float *dst, const float *src) {
        for (int i = warp; i < R; i += kBwdWarps)
            for (int c = lane; c < dk; c += 32) dst[i * LD + c] = src ? src[(size_t)i * dk + c] : 0.f;
    };
    // The states the kernel keeps in its workspace (16-byte aligned, d_k a multiple of 4) move as
    // 16-byte words, with a batch of loads in flight per thread before any is stored: one memory
    // latency per state rather than one per row.
    const bool vec = (dk & 3) == 0;
    const int q4 = dk >> 2, n4 = R * q4;
    constexpr int kBatch = 4;
    auto load_ws_state = [&](float *dst, const float *src) {
        if (!vec) {
            load_state(dst, src);
            return;
        }
        for (int base = tid; base < n4; base += kBwdThreads * kBatch) {
            float4 r[kBatch];
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int e = base + b * kBwdThreads;
                if (e < n4) r[b] = reinterpret_cast<const float4 *>(src)[e];
            }
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int e = base + b * kBwdThreads;
                if (e < n4) {
                    const int i = e / q4, c4 = e - i * q4;
                    *reinterpret_cast<float4 *>(dst + i * LD + 4 * c4) = r[b];
                }
            }
        }
    };
    auto store_ws_state = [&](float *dst, const float *src) {
        if (!vec) {
            store_state(dst, src);
            return;
        }
        for (int e = tid; e < n4; e += kBwdThreads) {
            const int i = e / q4, c4 = e - i * q4;
            reinterpret_cast<float4 *>(dst)[e] = *reinterpret_cast<const float4 *>(src + i * LD + 4 * c4);
        }
    };
    // The inputs of a step, loaded one step ahead into registers (thread tid < dk holds key and
    // query element tid, tid < R value and dO element r0 + tid of the slice's rows), so that their
    // memory latency overlaps the step before instead of sitting on the chain of steps.
    // one step's inputs, the bf16 ones kept in the input type until commit converts them
    struct StepIn {
        float a, e, g;
        IO q, x[kBwdMaxWindow], y[kBwdMaxWindow];
    };
    auto fetch = [&](long t, StepIn &in, bool qg) {
        const IO z = Io<IO>::zero();
        in.a = 1.f; in.e = 0.f; in.q = z; in.g = 0.f;
#pragma unroll
        for (int m = 0; m < kBwdMaxWindow; ++m) in.x[m] = in.y[m] = z;
        if (t < 0 || t >= T) return;
        in.a = ctx.al[t];
        in.e = ctx.et[t];
        if (qg) {
            if (tid < dk) in.q = q[(size_t)t * dk + tid];
            if (tid < R) in.g = dO[(size_t)t * dv + r0 + tid];
        }
#pragma unroll
        for (int m = 0; m < kBwdMaxWindow; ++m) {
            if (m < w) {
                const long j = t - m;
                if (tid < dk) in.x[m] = ctx.key_raw(j, tid);
                if (tid < R && j >= 0) in.y[m] = ctx.v[(size_t)j * dv + r0 + tid];
            }
        }
    };
    auto commit = [&](const StepIn &in, bool qg) {   // into sX, sY (and sQ, sG)
#pragma unroll
        for (int m = 0; m < kBwdMaxWindow; ++m) {
            if (m < w) {
                if (tid < dk) sX[(size_t)m * dk + tid] = Io<IO>::cvt(in.x[m]);
                if (tid < R) sY[m * RS + tid] = Io<IO>::cvt(in.y[m]);
            }
        }
        if (qg) {
            if (tid < dk) sQ[tid] = Io<IO>::cvt(in.q);
            if (tid < R) sG[tid] = in.g;
        }
    };
    // beta of a step from the staged keys (every thread gets it) and its denominator
    auto step_beta = [&](float eta_t, float &beta, float &den) {
        float part = 0.f;
        for (int e = tid; e < w * dk; e += kBwdThreads) part += sX[e] * sX[e];
        const float n = block_sum(part, sRed);
        den = n + p.eps;
        beta = den > 0.f ? eta_t / den : 0.f;
    };
    // one forward step on the state in sP (padded rows), in place
    auto forward_step = [&](const StepIn &in) {
        __syncthreads();                   // sX / sY and sP are free
        commit(in, false);
        __syncthreads();
        float beta, den;
        step_beta(in.e, beta, den);
        const float a = in.a;
        float *Si = sP + (size_t)(rok ? ri : 0) * LD;
        if (rok)
#pragma unroll 4
            for (int c = rq; c < dk; c += kRowThr) Si[c] *= a;
        if (REG) {
            // residuals at the decayed state first (every window pair), then the update
            for (int m = 0; m < w; ++m) {
                const float *x = sX + (size_t)m * dk;
                float r = 0.f;
                if (rok)
#pragma unroll 4
                    for (int c = rq; c < dk; c += kRowThr) r = fmaf(Si[c], x[c], r);
                r = row_sum(r);
                if (rok && rq == 0) sR[m * RS + ri] = r - sY[m * RS + ri];
            }
            __syncwarp();
            if (rok)
                for (int m = 0; m < w; ++m) {
                    const float *x = sX + (size_t)m * dk;
                    const float br = beta * sR[m * RS + ri];
#pragma unroll 4
                    for (int c = rq; c < dk; c += kRowThr) Si[c] = fmaf(-br, x[c], Si[c]);
                }
        } else if (rok) {
            for (int m = 0; m < w; ++m) {
                const float *x = sX + (size_t)m * dk;
                const float by = beta * sY[m * RS + ri];
#pragma unroll 4
                for (int c = rq; c < dk; c += kRowThr) Si[c] = fmaf(by, x[c], Si[c]);
            }
        }
    };

    // ---- pass 1: checkpoints S_{s C}, s = 0 .. nseg-1
    load_state(sP, p.S0 ? p.S0 + bh * DD + (size_t)r0 * dk : nullptr);
    StepIn cur, nxt;
    fetch(0, cur, false);
    for (int s = 0; s < nseg; ++s) {
        __syncthreads();
        store_ws_state(ckpt + (size_t)s * DS, sP);
        if (s + 1 == nseg) break;
        for (long t = (long)s * C; t < (long)(s + 1) * C; ++t) {
            fetch(t + 1, nxt, false);
            forward_step(cur);
            cur = nxt;
        }
    }

    // ---- reverse sweep, segment by segment
    load_state(sU, p.dS_T ? p.dS_T + bh * DD + (size_t)r0 * dk : nullptr);
    for (int s = nseg - 1; s >= 0; --s) {
        const long t0 = (long)s * C, t1 = min((long)T, t0 + C);
        __syncthreads();
        load_ws_state(sP, ckpt + (size_t)s * DS);
        __syncthreads();
        store_ws_state(buf, sP);
        fetch(t0, cur, false);
        for (long t = t0; t < t1; ++t) {
            fetch(t + 1 < t1 ? t + 1 : -1, nxt, false);
            forward_step(cur);
            __syncthreads();
            store_ws_state(buf + (size_t)(t - t0 + 1) * DS, sP);
            cur = nxt;
        }
        // sA = state after the last step of the segment
        __syncthreads();
        load_ws_state(sA, buf + (size_t)(t1 - t0) * DS);
        fetch(t1 - 1, cur, true);
        for (long t = t1 - 1; t >= t0; --t) {
            fetch(t - 1 >= t0 ? t - 1 : -1, nxt, true);
            __syncthreads();
            load_ws_state(sP, buf + (size_t)(t - t0) * DS);   // state before step t
            commit(cur, true);
            __syncthreads();
            float beta, den;
            step_beta(cur.e, beta, den);
            const float a = cur.a;
            // rows: U += dO q^T; U x_m; residuals r_m at the decayed state
            float part = 0.f;
            {
                float *Ui = sU + (size_t)(rok ? ri : 0) * LD;
                const float *Pi = sP + (size_t)(rok ? ri : 0) * LD;
                if (rok) {
                    const float g = sG[ri];
#pragma unroll 4
                    for (int c = rq; c < dk; c += kRowThr) Ui[c] = fmaf(g, sQ[c], Ui[c]);
                }
                for (int m = 0; m < w; ++m) {
                    const float *x = sX + (size_t)m * dk;
                    float ux = 0.f, sx = 0.f;
                    if (rok)
#pragma unroll 4
                        for (int c = rq; c < dk; c += kRowThr) {
                            ux = fmaf(Ui[c], x[c], ux);
                            sx = fmaf(Pi[c], x[c], sx);
                        }
                    ux = row_sum(ux);
                    sx = row_sum(sx);
                    if (rok && rq == 0) {
                        sUx[m * RS + ri] = ux;
                        if (REG) {
                            const float r = a * sx - sY[m * RS + ri];
                            sR[m * RS + ri] = r;
                            part -= r * ux;
                        } else {
                            part += sY[m * RS + ri] * ux;
                        }
                    }
                }
            }
            const float dbeta = block_sum(part, sRed);   // this slice's part
            const bool has_den = den > 0.f;
            const float dN = has_den ? -dbeta * beta / den : 0.f;
            if (tid == 0 && has_den) atomicAdd(get + t, dbeta / den);
            // rows: dr_m, dy_m (scattered to the value row of pair j)
            if (rok)
                for (int m = rq; m < w; m += kRowThr) {
                    const float ux = sUx[m * RS + ri];
                    if (REG) sDr[m * RS + ri] = -beta * ux;
                    const long j = t - m;
                    // dy = -dr (regression) = beta U x; with one pair per step a value row has one term
                    if (j >= 0) {
                        float *gvj = gv + (size_t)j * dv + r0 + ri;
                        if (w == 1) *gvj = beta * ux;
                        else *gvj += beta * ux;
                    }
                }
            __syncthreads();
            // columns: dq_t = S_t^T dO_t; dx_m (scattered to the key row of pair j): this slice's rows
            if (cc < dk) {
                float acc0 = 0.f, acc1 = 0.f;   // two chains over the slice's rows (zero beyond R)
#pragma unroll
                for (int i = 0; i < kBwdRows; i += 2) {
                    acc0 = fmaf(sA[i * LD + cc], sG[i], acc0);
                    acc1 = fmaf(sA[(i + 1) * LD + cc], sG[i + 1], acc1);
                }
                atomicAdd(gq + (size_t)t * dk + cc, acc0 + acc1);
                for (int m = 0; m < w; ++m) {
                    float dx;
                    if (REG) {   // -beta U^T r + alpha S^T dr, each sum its own chain
                        const float *r = sR + m * RS, *dr = sDr + m * RS;
                        float ur = 0.f, pd = 0.f;
#pragma unroll
                        for (int i = 0; i < kBwdRows; ++i) {
                            ur = fmaf(sU[i * LD + cc], r[i], ur);
                            pd = fmaf(sP[i * LD + cc], dr[i], pd);
                        }
                        dx = fmaf(-beta, ur, a * pd);
                    } else {
                        const float *y = sY + m * RS;
                        float u0 = 0.f, u1 = 0.f;
#pragma unroll
                        for (int i = 0; i < kBwdRows; i += 2) {
                            u0 = fmaf(sU[i * LD + cc], y[i], u0);
                            u1 = fmaf(sU[(i + 1) * LD + cc], y[i + 1], u1);
                        }
                        dx = beta * (u0 + u1);
                    }
                    dx = fmaf(2.f * dN, sX[(size_t)m * dk + cc], dx);
                    const long j = t - m;
                    if (j < 0) continue;
                    float *dst = ctx.same ? gk + (size_t)j * dk + cc
                                          : (j >= 1 ? gk + (size_t)(j - 1) * dk + cc : gkp ? gkp + cc : nullptr);
                    if (dst) atomicAdd(dst, dx);
                }
            }
            __syncthreads();
            // rows: dSbar = U + sum_m dr_m x_m^T; dalpha = <dSbar, S_{t-1}>; U <- alpha dSbar
            part = 0.f;
            if (rok) {
                float *Ui = sU + (size_t)ri * LD;
                const float *Pi = sP + (size_t)ri * LD;
#pragma unroll 4
                for (int c = rq; c < dk; c += kRowThr) {
                    float d = Ui[c];
                    if (REG)
                        for (int m = 0; m < w; ++m) d = fmaf(sDr[m * RS + ri], sX[(size_t)m * dk + c], d);
                    part = fmaf(d, Pi[c], part);
                    Ui[c] = a * d;
                }
            }
            const float dal = block_sum(part, sRed);   // this slice's part
            if (tid == 0) atomicAdd(gal + t, dal);
            // the state before step t is the state after step t - 1
            float *tmp = sA; sA = sP; sP = tmp;
            cur = nxt;
        }
    }
    __syncthreads();
    if (p.dS0) store_state(p.dS0 + bh * DD + (size_t)r0 * dk, sU);
}

}  // namespace

size_t bwd_workspace_bytes(int B, int H, int T, int dk, int dv, int *seg_out) {
    int C = (int)ceil(sqrt((double)(T > 0 ? T : 1)));
    if (C < 1) C = 1;
    const long long nseg = (T + C - 1) / C;
    if (seg_out) *seg_out = C;
    const long long nsl = (dv + kBwdRows - 1) / kBwdRows;   // slices of kBwdRows value rows per head
    return (size_t)B * H * nsl * (size_t)(nseg + C + 1) * kBwdRows * dk * sizeof(float);
}

size_t bwd_smem_bytes(int dk, int dv, int w) {
    (void)dv;   // the shared buffers hold one slice of kBwdRows value rows
    return bwd_smem(dk, w).total * sizeof(float);
}

cudaError_t launch_bwd_recurrent(const BwdParams &p, cudaStream_t s) {
    const size_t smem = bwd_smem_bytes(p.dk, p.dv, p.window);
    // the slices add their parts of dq, dk, dv's w > 1 terms, dalpha, deta and dk_prev: all start at zero
    const size_t BH = (size_t)p.B * p.H, T = (size_t)p.T;
    cudaError_t e0;
    if ((e0 = cudaMemsetAsync(p.dq, 0, BH * T * p.dk * sizeof(float), s)) != cudaSuccess) return e0;
    if ((e0 = cudaMemsetAsync(p.dk_out, 0, BH * T * p.dk * sizeof(float), s)) != cudaSuccess) return e0;
    if ((e0 = cudaMemsetAsync(p.dv_out, 0, BH * T * p.dv * sizeof(float), s)) != cudaSuccess) return e0;
    if ((e0 = cudaMemsetAsync(p.dalpha, 0, BH * T * sizeof(float), s)) != cudaSuccess) return e0;
    if ((e0 = cudaMemsetAsync(p.deta, 0, BH * T * sizeof(float), s)) != cudaSuccess) return e0;
    if (p.dk_prev && p.k_prev &&
        (e0 = cudaMemsetAsync(p.dk_prev, 0, BH * p.dk * sizeof(float), s)) != cudaSuccess)
        return e0;
    const long long nsl = (p.dv + kBwdRows - 1) / kBwdRows;
    auto pick = [&](auto kern) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)((long long)p.B * p.H * nsl), kBwdThreads, smem, s>>>(p);
        return cudaGetLastError();
    };
    if (p.io_bf16)
        return p.regression ? pick(bwd_recurrent_kernel<__nv_bfloat16, true>)
                            : pick(bwd_recurrent_kernel<__nv_bfloat16, false>);
    return p.regression ? pick(bwd_recurrent_kernel<float, true>) : pick(bwd_recurrent_kernel<float, false>);
}

}  // namespace falcon
