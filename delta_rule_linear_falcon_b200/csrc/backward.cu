// backward.cu -- falcon_bwd_recurrent: gradients of the recurrent form (reverse mode
// through the per-token recurrence of "Fast Weight Attention for Continual Learning",
// authors' abstract; the pages give the forward rules only, so these are their
// derivatives) for Falcon-1/1A/3/3A, with the same-step flag, an initial state and a
// cached key. fp32 state and fp32 arithmetic; q, k, v in the I/O dtype, every gradient
// in fp32.
//
// One CTA of 512 threads per (b, h). With U = dL/dS after step t (starting from dS_T),
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
// checkpoint into a buffer of C + 1 states before walking it backwards. U and the two
// states a step needs (before and after it) sit in shared memory. Row products (U x, Sbar x,
// the state update) take four threads per value row i, each every fourth column, reduced
// with two shuffles; the row stride is 4 more than a multiple of 32 floats, so the 32 threads
// of a warp (8 rows x 4 column phases) hit 32 different banks. Column products (S^T dO,
// U^T r, Sbar^T dr) take one thread per key column c in each of four row groups, reduced
// through shared memory.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace falcon {

namespace {

constexpr int kBwdThreads = 512;
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kRowGroups = kBwdThreads / 128;   // column products: four row groups of 128 columns
constexpr int kBwdMaxWindow = 8;                // pairs per step the register prefetch holds

struct BwdSmem {
    int LD, dk, dv, w;
    // offsets in floats
    size_t oU, oP, oA, oX, oY, oQ, oG, oUx, oR, oDr, oPart, oRed, total;
};

__host__ __device__ inline BwdSmem bwd_smem(int dk, int dv, int w) {
    BwdSmem s;
    s.LD = ((dk + 27) / 32) * 32 + 4; s.dk = dk; s.dv = dv; s.w = w;
    const size_t mat = (size_t)dv * s.LD;
    s.oU = 0; s.oP = mat; s.oA = 2 * mat;
    s.oX = 3 * mat;
    s.oY = s.oX + (size_t)w * dk;
    s.oQ = s.oY + (size_t)w * dv;
    s.oG = s.oQ + dk;
    s.oUx = s.oG + dv;
    s.oR = s.oUx + (size_t)w * dv;
    s.oDr = s.oR + (size_t)w * dv;
    s.oPart = s.oDr + (size_t)w * dv;                 // kRowGroups x (1 + w) x dk partial column sums
    s.oRed = s.oPart + (size_t)kRowGroups * (1 + w) * dk;
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

// Sum over the four threads of a value row (lanes 4i .. 4i + 3); all four get it.
__device__ __forceinline__ float quad_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    return x;
}

template <typename IO>
struct BwdCtx {
    const BwdParams &p;
    const IO *q, *k, *v, *kp;
    const float *al, *et;
    int T, dk, dv, w;
    bool same;
    // key row of pair j into dst (dk floats): k_{j-1}, k_prev for j = 0 (or 0), k_j with the flag
    __device__ void pair_key(float *dst, long j) const {
        const int tid = threadIdx.x;
        const IO *src = nullptr;
        size_t base = 0;
        if (j >= 0) {
            if (same) { src = k; base = (size_t)j * dk; }
            else if (j >= 1) { src = k; base = (size_t)(j - 1) * dk; }
            else if (kp) { src = kp; base = 0; }
        }
        for (int c = tid; c < dk; c += kBwdThreads) dst[c] = src ? Io<IO>::ld(src, base + c) : 0.f;
    }
    // element c of the key row of pair j (0 for j < 0, or for the first pair without k_prev)
    __device__ float key_elem(long j, int c) const {
        if (j < 0) return 0.f;
        if (same) return Io<IO>::ld(k, (size_t)j * dk + c);
        if (j >= 1) return Io<IO>::ld(k, (size_t)(j - 1) * dk + c);
        return kp ? Io<IO>::ld(kp, c) : 0.f;
    }
    // stage the w pairs of step t (keys, values) into shared memory
    __device__ void stage_pairs(float *sX, float *sY, long t) const {
        const int tid = threadIdx.x;
        for (int m = 0; m < w; ++m) {
            pair_key(sX + (size_t)m * dk, t - m);
            const long j = t - m;
            for (int i = tid; i < dv; i += kBwdThreads)
                sY[(size_t)m * dv + i] = j >= 0 ? Io<IO>::ld(v, (size_t)j * dv + i) : 0.f;
        }
    }
};

template <typename IO, bool REG>
__global__ void __launch_bounds__(kBwdThreads)
bwd_recurrent_kernel(BwdParams p) {
    extern __shared__ __align__(16) float smem[];
    const int dk = p.dk, dv = p.dv, w = p.window, T = p.T, C = p.seg;
    const BwdSmem L = bwd_smem(dk, dv, w);
    const int LD = L.LD;
    float *sU = smem + L.oU, *sP = smem + L.oP, *sA = smem + L.oA;
    float *sX = smem + L.oX, *sY = smem + L.oY, *sQ = smem + L.oQ, *sG = smem + L.oG;
    float *sUx = smem + L.oUx, *sR = smem + L.oR, *sDr = smem + L.oDr, *sRed = smem + L.oRed;
    float *sPart = smem + L.oPart;
    const int tid = threadIdx.x;
    const int ri = tid >> 2, rq = tid & 3;          // row products: value row ri, columns rq, rq + 4, ..
    const bool rok = ri < dv;
    const int cc = tid & 127, rg = tid >> 7;        // column products: key column cc, rows rg, rg + 4, ..
    const size_t bh = blockIdx.x;
    const size_t DD = (size_t)dv * dk;

    BwdCtx<IO> ctx{p,
                   reinterpret_cast<const IO *>(p.q) + bh * T * dk,
                   reinterpret_cast<const IO *>(p.k) + bh * T * dk,
                   reinterpret_cast<const IO *>(p.v) + bh * T * dv,
                   p.k_prev ? reinterpret_cast<const IO *>(p.k_prev) + bh * dk : nullptr,
                   p.alpha + bh * T, p.eta + bh * T, T, dk, dv, w, p.same_step};
    const IO *q = ctx.q;
    const float *dO = p.dO + bh * T * dv;
    float *gq = p.dq + bh * T * dk, *gk = p.dk_out + bh * T * dk, *gv = p.dv_out + bh * T * dv;
    float *gal = p.dalpha + bh * T, *get = p.deta + bh * T;
    float *gkp = (p.dk_prev && p.k_prev) ? p.dk_prev + bh * dk : nullptr;
    const int nseg = (T + C - 1) / C;
    float *ckpt = p.ws + bh * (size_t)(nseg + C + 1) * DD;   // nseg checkpoints, then C + 1 states
    float *buf = ckpt + (size_t)nseg * DD;

    // the key and value gradients accumulate over the w steps that read a pair
    for (size_t e = tid; e < (size_t)T * dk; e += kBwdThreads) gk[e] = 0.f;
    for (size_t e = tid; e < (size_t)T * dv; e += kBwdThreads) gv[e] = 0.f;
    if (gkp)
        for (int c = tid; c < dk; c += kBwdThreads) gkp[c] = 0.f;

    // dense dv x dk (global) <-> padded rows (shared): a warp per row, lanes along it
    const int warp = tid >> 5, lane = tid & 31;
    auto store_state = [&](float *dst, const float *src) {
        for (int i = warp; i < dv; i += kBwdWarps)
            for (int c = lane; c < dk; c += 32) dst[(size_t)i * dk + c] = src[i * LD + c];
    };
    auto load_state = [&](float *dst, const float *src) {
        for (int i = warp; i < dv; i += kBwdWarps)
            for (int c = lane; c < dk; c += 32) dst[i * LD + c] = src ? src[(size_t)i * dk + c] : 0.f;
    };
    // The states the kernel keeps in its workspace (16-byte aligned, d_k a multiple of 4) move as
    // 16-byte words, with a batch of loads in flight per thread before any is stored: one memory
    // latency per state rather than one per row.
    const bool vec = (dk & 3) == 0;
    const int q4 = dk >> 2, n4 = dv * q4;
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
    // query element tid, tid < dv value and dO element tid; d_k, d_v <= 128 < 512 threads), so
    // that their memory latency overlaps the step before instead of sitting on the chain of steps.
    struct StepIn {
        float a, e, q, g, x[kBwdMaxWindow], y[kBwdMaxWindow];
    };
    auto fetch = [&](long t, StepIn &in, bool qg) {
        in.a = 1.f; in.e = 0.f; in.q = 0.f; in.g = 0.f;
#pragma unroll
        for (int m = 0; m < kBwdMaxWindow; ++m) in.x[m] = in.y[m] = 0.f;
        if (t < 0 || t >= T) return;
        in.a = ctx.al[t];
        in.e = ctx.et[t];
        if (qg) {
            if (tid < dk) in.q = Io<IO>::ld(q, (size_t)t * dk + tid);
            if (tid < dv) in.g = dO[(size_t)t * dv + tid];
        }
#pragma unroll
        for (int m = 0; m < kBwdMaxWindow; ++m) {
            if (m < w) {
                const long j = t - m;
                if (tid < dk) in.x[m] = ctx.key_elem(j, tid);
                if (tid < dv && j >= 0) in.y[m] = Io<IO>::ld(ctx.v, (size_t)j * dv + tid);
            }
        }
    };
    auto commit = [&](const StepIn &in, bool qg) {   // into sX, sY (and sQ, sG)
#pragma unroll
        for (int m = 0; m < kBwdMaxWindow; ++m) {
            if (m < w) {
                if (tid < dk) sX[(size_t)m * dk + tid] = in.x[m];
                if (tid < dv) sY[(size_t)m * dv + tid] = in.y[m];
            }
        }
        if (qg) {
            if (tid < dk) sQ[tid] = in.q;
            if (tid < dv) sG[tid] = in.g;
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
            for (int c = rq; c < dk; c += 4) Si[c] *= a;
        if (REG) {
            // residuals at the decayed state first (every window pair), then the update
            for (int m = 0; m < w; ++m) {
                const float *x = sX + (size_t)m * dk;
                float r = 0.f;
                if (rok)
                    for (int c = rq; c < dk; c += 4) r = fmaf(Si[c], x[c], r);
                r = quad_sum(r);
                if (rok && rq == 0) sR[(size_t)m * dv + ri] = r - sY[(size_t)m * dv + ri];
            }
            __syncwarp();
            if (rok)
                for (int m = 0; m < w; ++m) {
                    const float *x = sX + (size_t)m * dk;
                    const float br = beta * sR[(size_t)m * dv + ri];
                    for (int c = rq; c < dk; c += 4) Si[c] = fmaf(-br, x[c], Si[c]);
                }
        } else if (rok) {
            for (int m = 0; m < w; ++m) {
                const float *x = sX + (size_t)m * dk;
                const float by = beta * sY[(size_t)m * dv + ri];
                for (int c = rq; c < dk; c += 4) Si[c] = fmaf(by, x[c], Si[c]);
            }
        }
    };

    // ---- pass 1: checkpoints S_{s C}, s = 0 .. nseg-1
    load_state(sP, p.S0 ? p.S0 + bh * DD : nullptr);
    StepIn cur, nxt;
    fetch(0, cur, false);
    for (int s = 0; s < nseg; ++s) {
        __syncthreads();
        store_ws_state(ckpt + (size_t)s * DD, sP);
        if (s + 1 == nseg) break;
        for (long t = (long)s * C; t < (long)(s + 1) * C; ++t) {
            fetch(t + 1, nxt, false);
            forward_step(cur);
            cur = nxt;
        }
    }

    // ---- reverse sweep, segment by segment
    load_state(sU, p.dS_T ? p.dS_T + bh * DD : nullptr);
    for (int s = nseg - 1; s >= 0; --s) {
        const long t0 = (long)s * C, t1 = min((long)T, t0 + C);
        __syncthreads();
        load_ws_state(sP, ckpt + (size_t)s * DD);
        __syncthreads();
        store_ws_state(buf, sP);
        fetch(t0, cur, false);
        for (long t = t0; t < t1; ++t) {
            fetch(t + 1 < t1 ? t + 1 : -1, nxt, false);
            forward_step(cur);
            __syncthreads();
            store_ws_state(buf + (size_t)(t - t0 + 1) * DD, sP);
            cur = nxt;
        }
        // sA = state after the last step of the segment
        __syncthreads();
        load_ws_state(sA, buf + (size_t)(t1 - t0) * DD);
        fetch(t1 - 1, cur, true);
        for (long t = t1 - 1; t >= t0; --t) {
            fetch(t - 1 >= t0 ? t - 1 : -1, nxt, true);
            __syncthreads();
            load_ws_state(sP, buf + (size_t)(t - t0) * DD);   // state before step t
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
                    for (int c = rq; c < dk; c += 4) Ui[c] = fmaf(g, sQ[c], Ui[c]);
                }
                for (int m = 0; m < w; ++m) {
                    const float *x = sX + (size_t)m * dk;
                    float ux = 0.f, sx = 0.f;
                    if (rok)
                        for (int c = rq; c < dk; c += 4) {
                            ux = fmaf(Ui[c], x[c], ux);
                            sx = fmaf(Pi[c], x[c], sx);
                        }
                    ux = quad_sum(ux);
                    sx = quad_sum(sx);
                    if (rok && rq == 0) {
                        sUx[(size_t)m * dv + ri] = ux;
                        if (REG) {
                            const float r = a * sx - sY[(size_t)m * dv + ri];
                            sR[(size_t)m * dv + ri] = r;
                            part -= r * ux;
                        } else {
                            part += sY[(size_t)m * dv + ri] * ux;
                        }
                    }
                }
            }
            const float dbeta = block_sum(part, sRed);
            const bool has_den = den > 0.f;
            const float dN = has_den ? -dbeta * beta / den : 0.f;
            if (tid == 0) get[t] = has_den ? dbeta / den : 0.f;
            // rows: dr_m, dy_m (scattered to the value row of pair j)
            if (rok)
                for (int m = rq; m < w; m += 4) {
                    const float ux = sUx[(size_t)m * dv + ri];
                    if (REG) sDr[(size_t)m * dv + ri] = -beta * ux;
                    const long j = t - m;
                    // dy = -dr (regression) = beta U x; with one pair per step a value row has one term
                    if (j >= 0) {
                        if (w == 1) gv[(size_t)j * dv + ri] = beta * ux;
                        else gv[(size_t)j * dv + ri] += beta * ux;
                    }
                }
            __syncthreads();
            // columns: dq_t = S_t^T dO_t; dx_m (scattered to the key row of pair j)
            if (cc < dk) {   // partial sums over the rows of this thread's group
                float acc = 0.f;
                for (int i = rg; i < dv; i += kRowGroups) acc = fmaf(sA[(size_t)i * LD + cc], sG[i], acc);
                sPart[(size_t)rg * (1 + w) * dk + cc] = acc;
                for (int m = 0; m < w; ++m) {
                    float dx = 0.f;
                    if (REG) {
                        const float *r = sR + (size_t)m * dv, *dr = sDr + (size_t)m * dv;
                        for (int i = rg; i < dv; i += kRowGroups) {
                            dx = fmaf(-beta * sU[(size_t)i * LD + cc], r[i], dx);
                            dx = fmaf(a * sP[(size_t)i * LD + cc], dr[i], dx);
                        }
                    } else {
                        const float *y = sY + (size_t)m * dv;
                        for (int i = rg; i < dv; i += kRowGroups) dx = fmaf(beta * sU[(size_t)i * LD + cc], y[i], dx);
                    }
                    sPart[((size_t)rg * (1 + w) + 1 + m) * dk + cc] = dx;
                }
            }
            __syncthreads();
            for (int e = tid; e < (1 + w) * dk; e += kBwdThreads) {   // e = slot * dk + c
                const int slot = e / dk, c = e - slot * dk;
                float v = 0.f;
#pragma unroll
                for (int g = 0; g < kRowGroups; ++g) v += sPart[(size_t)g * (1 + w) * dk + e];
                if (slot == 0) {
                    gq[(size_t)t * dk + c] = v;
                    continue;
                }
                const int m = slot - 1;
                const float dx = fmaf(2.f * dN, sX[(size_t)m * dk + c], v);
                const long j = t - m;
                if (j < 0) continue;
                // with one pair per step a key row has one term (no read of the zero it starts from)
                float *dst = ctx.same ? gk + (size_t)j * dk + c
                                      : (j >= 1 ? gk + (size_t)(j - 1) * dk + c : gkp ? gkp + c : nullptr);
                if (!dst) continue;
                if (w == 1) *dst = dx;
                else *dst += dx;
            }
            __syncthreads();
            // rows: dSbar = U + sum_m dr_m x_m^T; dalpha = <dSbar, S_{t-1}>; U <- alpha dSbar
            part = 0.f;
            if (rok) {
                float *Ui = sU + (size_t)ri * LD;
                const float *Pi = sP + (size_t)ri * LD;
                for (int c = rq; c < dk; c += 4) {
                    float d = Ui[c];
                    if (REG)
                        for (int m = 0; m < w; ++m) d = fmaf(sDr[(size_t)m * dv + ri], sX[(size_t)m * dk + c], d);
                    part = fmaf(d, Pi[c], part);
                    Ui[c] = a * d;
                }
            }
            const float dal = block_sum(part, sRed);
            if (tid == 0) gal[t] = dal;
            // the state before step t is the state after step t - 1
            float *tmp = sA; sA = sP; sP = tmp;
            cur = nxt;
        }
    }
    __syncthreads();
    if (p.dS0) store_state(p.dS0 + bh * DD, sU);
}

}  // namespace

size_t bwd_workspace_bytes(int B, int H, int T, int dk, int dv, int *seg_out) {
    int C = (int)ceil(sqrt((double)(T > 0 ? T : 1)));
    if (C < 1) C = 1;
    const long long nseg = (T + C - 1) / C;
    if (seg_out) *seg_out = C;
    return (size_t)B * H * (size_t)(nseg + C + 1) * dv * dk * sizeof(float);
}

size_t bwd_smem_bytes(int dk, int dv, int w) { return bwd_smem(dk, dv, w).total * sizeof(float); }

cudaError_t launch_bwd_recurrent(const BwdParams &p, cudaStream_t s) {
    const size_t smem = bwd_smem_bytes(p.dk, p.dv, p.window);
    auto pick = [&](auto kern) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)((long long)p.B * p.H), kBwdThreads, smem, s>>>(p);
        return cudaGetLastError();
    };
    if (p.io_bf16)
        return p.regression ? pick(bwd_recurrent_kernel<__nv_bfloat16, true>)
                            : pick(bwd_recurrent_kernel<__nv_bfloat16, false>);
    return p.regression ? pick(bwd_recurrent_kernel<float, true>) : pick(bwd_recurrent_kernel<float, false>);
}

}  // namespace falcon
