// chunk_kernel.cuh -- chunk-parallel forward pass of the Falcon rules, with the
// positive-decay renormalisation the authors' abstract of "Fast Weight
// Attention for Continual Learning" names for its parallel forms.
//
// One CTA owns one (b, h) and a slice of DVS value rows of the state, and
// walks the sequence block by block; the fp32 state stays on chip for the
// whole sequence, so q, k, v, alpha, eta are read once and o is written once.
// Rows of the state are independent given the keys, so value slices of one
// head run in separate CTAs with no communication.
//
// A block holds CT tokens and E = CT * w pseudo-value rows; row e = s*w + m
// carries pair j = t0 + s - m (key x_j = k_{j-1}, value y_j = v_j) and the
// step size / decay of token s. With g_s the block-local cumulative log2 decay
// and S_c the state entering the block:
//   (prep)   beta_s = eta_s / (sum_m ||x_{s*w+m}||^2 + eps);  g_s = cumsum log2 alpha
//   (local)  L[e][e'] = beta_s 2^(g_s - g_s') (x_e . x_e')   for s' < s
//            P[i][e'] = 2^(g_i - g_s') (q_i . x_e')           for s' <= i  (read after write)
//            T = (I + L)^-1                                   (regression family only)
//   (prop)   R = diag(beta) (Y - diag(2^g) X S_c^T)
//            U = T R            (inner-product family: U = diag(beta) Y)
//            O = diag(2^g) Q S_c^T + P U
//            S_{c+1} = 2^(g_last) S_c + U'^T X,   U' = diag(2^(g_last - g_s)) U
// Every exponent above is <= 0 (positive-decay renormalisation): no factor is
// ever a quotient of cumulative products, so long sequences cannot underflow
// or overflow the decay.
//
// The state is kept transposed (S^T, d_k x DVS) in mma accumulator
// registers of warps 0..DK/16-1 and mirrored in shared memory as bf16 for the
// products that read it. Products use bf16 operands with fp32 accumulation;
// the solve of T runs in fp32.
#pragma once

#include "chunk_mma.cuh"
#include "common.cuh"
#include "launch.h"

namespace falcon {

constexpr int kChunkThreads = 256;
constexpr int kRowsTile = 64;  // pseudo-value rows per block (E <= 64)

template <int DK, int DVS>
struct ChunkSmem {
    static constexpr int ET = kRowsTile;
    static constexpr int LDX = DK + 8;    // bf16 row strides padded by 16 bytes
    static constexpr int LDY = DVS + 8;
    static constexpr int LDE = ET + 8;
    static constexpr int LDF = ET + 1;    // fp32 solve buffers
    static constexpr size_t oX = 0;
    static constexpr size_t oQ = oX + sizeof(bf16) * ET * LDX;
    static constexpr size_t oY = oQ + sizeof(bf16) * ET * LDX;
    static constexpr size_t oS = oY + sizeof(bf16) * ET * LDY;
    static constexpr size_t oT = oS + sizeof(bf16) * DK * LDY;
    static constexpr size_t oP = oT + sizeof(bf16) * ET * LDE;
    static constexpr size_t oR = oP + sizeof(bf16) * ET * LDE;
    static constexpr size_t oU = oR + sizeof(bf16) * ET * LDY;
    static constexpr size_t oU2 = oU + sizeof(bf16) * ET * LDY;
    static constexpr size_t oL = oU2 + sizeof(bf16) * ET * LDY;
    static constexpr size_t oTf = oL + sizeof(float) * ET * LDF;
    static constexpr size_t oM = oTf + sizeof(float) * ET * LDF;
    static constexpr size_t oNrm = oM + sizeof(float) * 3 * 256;
    static constexpr size_t oG2 = oNrm + sizeof(float) * ET;
    static constexpr size_t oBeta = oG2 + sizeof(float) * ET;
    static constexpr size_t oStep = oBeta + sizeof(float) * ET;
    static constexpr size_t oScal = oStep + sizeof(int) * ET;
    static constexpr size_t bytes = oScal + 16;
};

template <int DK, int DVS, bool REG, typename IO>
__global__ void __launch_bounds__(kChunkThreads, 1)
chunk_fwd_kernel(ChunkParams p) {
    using L = ChunkSmem<DK, DVS>;
    constexpr int ET = L::ET, LDX = L::LDX, LDY = L::LDY, LDE = L::LDE, LDF = L::LDF;
    constexpr int NT = DVS / 8;          // n-tiles across the value slice
    constexpr int S_WARPS = DK / 16;     // warps holding a 16-row tile of S^T
    constexpr int CPR = DK / 8;          // 16-byte chunks per key row
    constexpr int CPRY = DVS / 8;        // 16-byte chunks per value-slice row
    static_assert(DK % 16 == 0 && DK <= 128 && DVS % 16 == 0 && DVS <= 128, "tile shape");

    extern __shared__ __align__(16) unsigned char smem[];
    bf16 *sX = reinterpret_cast<bf16 *>(smem + L::oX);
    bf16 *sQ = reinterpret_cast<bf16 *>(smem + L::oQ);
    bf16 *sY = reinterpret_cast<bf16 *>(smem + L::oY);
    bf16 *sS = reinterpret_cast<bf16 *>(smem + L::oS);
    bf16 *sT = reinterpret_cast<bf16 *>(smem + L::oT);
    bf16 *sP = reinterpret_cast<bf16 *>(smem + L::oP);
    bf16 *sR = reinterpret_cast<bf16 *>(smem + L::oR);
    bf16 *sU = reinterpret_cast<bf16 *>(smem + L::oU);
    bf16 *sU2 = reinterpret_cast<bf16 *>(smem + L::oU2);
    float *sL = reinterpret_cast<float *>(smem + L::oL);
    float *sTf = reinterpret_cast<float *>(smem + L::oTf);
    float *sM = reinterpret_cast<float *>(smem + L::oM);
    float *sNrm = reinterpret_cast<float *>(smem + L::oNrm);
    float *sG2 = reinterpret_cast<float *>(smem + L::oG2);
    float *sBeta = reinterpret_cast<float *>(smem + L::oBeta);
    int *sStep = reinterpret_cast<int *>(smem + L::oStep);
    float *sScal = reinterpret_cast<float *>(smem + L::oScal);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nsplit = p.dv / DVS;
    const long bh = blockIdx.x / nsplit;
    const int dv0 = (blockIdx.x % nsplit) * DVS;
    const int T = p.T, dv = p.dv, W = p.window, CT = p.tok_per_blk, E = CT * W;
    if (E > ET || E < 1 || dv % DVS != 0) {  // host guarantees this; refuse rather than overrun
        if (tid == 0) set_error(p.err, kDevErrGeometry);
        return;
    }

    const IO *q = reinterpret_cast<const IO *>(p.q) + bh * (size_t)T * DK;
    const IO *k = reinterpret_cast<const IO *>(p.k) + bh * (size_t)T * DK;
    const IO *v = reinterpret_cast<const IO *>(p.v) + bh * (size_t)T * dv;
    const IO *kp = p.k_prev ? reinterpret_cast<const IO *>(p.k_prev) + bh * (size_t)DK : nullptr;
    const float *alpha = p.alpha + bh * (size_t)T;
    const float *eta = p.eta + bh * (size_t)T;
    IO *o = reinterpret_cast<IO *>(p.o) + bh * (size_t)T * dv;

    // ---- once per CTA: row -> step map, zero upper blocks of T, initial state
    for (int e = tid; e < ET; e += kChunkThreads) sStep[e] = e < E ? e / W : CT - 1;
    for (int idx = tid; idx < ET * LDF; idx += kChunkThreads) sTf[idx] = 0.f;

    float accS[NT][4];
    const int sr = 16 * warp + (lane >> 2);  // S^T rows (key coordinates) of this thread
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int c = 8 * nt + 2 * (lane & 3);  // value coordinate within the slice
#pragma unroll
        for (int h = 0; h < 4; ++h) accS[nt][h] = 0.f;
        if (warp < S_WARPS && p.S0) {
            const float *S0 = p.S0 + bh * (size_t)dv * DK;
            accS[nt][0] = S0[(size_t)(dv0 + c) * DK + sr];
            accS[nt][1] = S0[(size_t)(dv0 + c + 1) * DK + sr];
            accS[nt][2] = S0[(size_t)(dv0 + c) * DK + sr + 8];
            accS[nt][3] = S0[(size_t)(dv0 + c + 1) * DK + sr + 8];
        }
        if (warp < S_WARPS) {
            *reinterpret_cast<uint32_t *>(sS + sr * LDY + c) = pack_bf16x2(accS[nt][0], accS[nt][1]);
            *reinterpret_cast<uint32_t *>(sS + (sr + 8) * LDY + c) = pack_bf16x2(accS[nt][2], accS[nt][3]);
        }
    }
    __syncthreads();

    float accO[NT][4];
    for (int t0 = 0; t0 < T; t0 += CT) {
        const int nval = min(CT, T - t0);

        // ---- (1) stage the block: expanded keys X, queries Q, values Y; key norms
        for (int idx = tid; idx < ET * CPR; idx += kChunkThreads) {
            const int e = idx / CPR, ch = idx % CPR;
            float x8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) x8[j] = 0.f;
            if (e < E) {
                const int s = e / W, m = e % W;
                const long j = (long)t0 + s - m;
                if (s < nval) {
                    if (p.same_step) {                  // pair j holds k_j
                        if (j >= 0) Io<IO>::ld8(k, (size_t)j * DK + ch * 8, x8);
                    } else if (j >= 1) Io<IO>::ld8(k, (size_t)(j - 1) * DK + ch * 8, x8);
                    else if (j == 0 && kp) Io<IO>::ld8(kp, (size_t)ch * 8, x8);
                }
            }
            float nrm = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) nrm += x8[j] * x8[j];
#pragma unroll
            for (int off = CPR / 2; off >= 1; off >>= 1) nrm += __shfl_xor_sync(0xffffffffu, nrm, off);
            if (ch == 0) sNrm[e] = nrm;
            uint4 pk;
            pk.x = pack_bf16x2(x8[0], x8[1]); pk.y = pack_bf16x2(x8[2], x8[3]);
            pk.z = pack_bf16x2(x8[4], x8[5]); pk.w = pack_bf16x2(x8[6], x8[7]);
            *reinterpret_cast<uint4 *>(sX + e * LDX + ch * 8) = pk;

            float q8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) q8[j] = 0.f;
            if (e < nval) Io<IO>::ld8(q, (size_t)(t0 + e) * DK + ch * 8, q8);
            pk.x = pack_bf16x2(q8[0], q8[1]); pk.y = pack_bf16x2(q8[2], q8[3]);
            pk.z = pack_bf16x2(q8[4], q8[5]); pk.w = pack_bf16x2(q8[6], q8[7]);
            *reinterpret_cast<uint4 *>(sQ + e * LDX + ch * 8) = pk;
        }
        for (int idx = tid; idx < ET * CPRY; idx += kChunkThreads) {
            const int e = idx / CPRY, ch = idx % CPRY;
            float y8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) y8[j] = 0.f;
            if (e < E) {
                const int s = e / W, m = e % W;
                const long j = (long)t0 + s - m;
                if (s < nval && j >= 0) Io<IO>::ld8(v, (size_t)j * dv + dv0 + ch * 8, y8);
            }
            uint4 pk;
            pk.x = pack_bf16x2(y8[0], y8[1]); pk.y = pack_bf16x2(y8[2], y8[3]);
            pk.z = pack_bf16x2(y8[4], y8[5]); pk.w = pack_bf16x2(y8[6], y8[7]);
            *reinterpret_cast<uint4 *>(sY + e * LDY + ch * 8) = pk;
        }
        __syncthreads();

        // ---- (2) prep: step sizes and block-local cumulative log2 decay (warp 0)
        if (warp == 0) {
            float la[2], bt[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int s = lane + 32 * hh;
                const bool valid = s < nval;
                la[hh] = valid ? log2f(alpha[t0 + s]) : 0.f;
                float ns = 0.f;
                if (valid)
                    for (int m = 0; m < W; ++m) ns += sNrm[s * W + m];
                bt[hh] = valid ? step_size(eta[t0 + s], ns, p.eps) : 0.f;
            }
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y0 = __shfl_up_sync(0xffffffffu, la[0], off);
                const float y1 = __shfl_up_sync(0xffffffffu, la[1], off);
                if (lane >= off) { la[0] += y0; la[1] += y1; }
            }
            la[1] += __shfl_sync(0xffffffffu, la[0], 31);
            sG2[lane] = la[0];
            sG2[lane + 32] = la[1];
            sBeta[lane] = bt[0];
            sBeta[lane + 32] = bt[1];
            __syncwarp();
            if (lane == 0) sScal[0] = sG2[nval - 1];
        }
        __syncthreads();
        const float gl = sScal[0];

        // ---- (3) decay-weighted key Gram (L) and query-key tile (P)
        if (warp >= 4 || REG) {
            const bf16 *Asrc = warp < 4 ? sX : sQ;
            const int m0 = 16 * (warp & 3);
            float acc[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h = 0; h < 4; ++h) acc[nt][h] = 0.f;
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                uint32_t a[4];
                load_a_rm(a, Asrc, LDX, m0, 16 * kk, lane);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b[4];
                    load_b_nk(b, sX, LDX, 16 * np, 16 * kk, lane);
                    mma_bf16_16816(acc[2 * np], a, b[0], b[1]);
                    mma_bf16_16816(acc[2 * np + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int row = m0 + (lane >> 2) + 8 * h;
                    const int col = 8 * nt + 2 * (lane & 3);
                    if (warp < 4) {
                        const int se = sStep[row];
                        const float bg = sBeta[se], ge = sG2[se];
#pragma unroll
                        for (int c2 = 0; c2 < 2; ++c2) {
                            const int sc = sStep[col + c2];
                            sL[row * LDF + col + c2] =
                                sc < se ? bg * exp2f(ge - sG2[sc]) * acc[nt][2 * h + c2] : 0.f;
                        }
                    } else {
                        const float gi = sG2[row];
                        const int s0 = sStep[col], s1 = sStep[col + 1];
                        const float p0 = s0 <= row ? exp2f(gi - sG2[s0]) * acc[nt][2 * h] : 0.f;
                        const float p1 = s1 <= row ? exp2f(gi - sG2[s1]) * acc[nt][2 * h + 1] : 0.f;
                        *reinterpret_cast<uint32_t *>(sP + row * LDE + col) = pack_bf16x2(p0, p1);
                    }
                }
        }
        __syncthreads();

        // ---- (4) T = (I + L)^-1 in fp32, by 16x16 blocks (regression family)
        if (REG) {
            if (tid < 64) {  // diagonal blocks: one thread per column
                const int b = tid >> 4, j = tid & 15;
                const float *Lb = sL + (16 * b) * LDF + 16 * b;
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < i; ++m) acc += Lb[i * LDF + m] * x[m];
                    x[i] = i < j ? 0.f : (i == j ? 1.f : -acc);
                }
                float *Tb = sTf + (16 * b) * LDF + 16 * b;
#pragma unroll
                for (int i = 0; i < 16; ++i) Tb[i * LDF + j] = x[i];
            }
            __syncthreads();
            for (int d = 1; d < 4; ++d) {  // block sub-diagonals, nearest first
                const int nb = 4 - d;
                for (int idx = tid; idx < nb * 256; idx += kChunkThreads) {
                    const int bj = idx >> 8, bi = bj + d, r = (idx >> 4) & 15, c = idx & 15;
                    const float *Lrow = sL + (16 * bi + r) * LDF;
                    float acc = 0.f;
                    for (int m = 16 * bj; m < 16 * bi; ++m) acc += Lrow[m] * sTf[m * LDF + 16 * bj + c];
                    sM[idx] = acc;
                }
                __syncthreads();
                for (int idx = tid; idx < nb * 256; idx += kChunkThreads) {
                    const int bj = idx >> 8, bi = bj + d, r = (idx >> 4) & 15, c = idx & 15;
                    const float *Trow = sTf + (16 * bi + r) * LDF + 16 * bi;
                    const float *Mb = sM + (bj << 8);
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < 16; ++m) acc += Trow[m] * Mb[m * 16 + c];
                    sTf[(16 * bi + r) * LDF + 16 * bj + c] = -acc;
                }
                __syncthreads();
            }
            for (int idx = tid; idx < ET * ET / 2; idx += kChunkThreads) {
                const int r = idx / (ET / 2), c = 2 * (idx % (ET / 2));
                *reinterpret_cast<uint32_t *>(sT + r * LDE + c) =
                    pack_bf16x2(sTf[r * LDF + c], sTf[r * LDF + c + 1]);
            }
        }

        // ---- (5) residuals against the carried state, and the state's share of O
        {
            const bf16 *Asrc = warp < 4 ? sX : sQ;
            const int m0 = 16 * (warp & 3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int h = 0; h < 4; ++h) accO[nt][h] = 0.f;
            if (warp >= 4 || REG) {
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    uint32_t a[4];
                    load_a_rm(a, Asrc, LDX, m0, 16 * kk, lane);
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        uint32_t b[4];
                        load_b_kn(b, sS, LDY, 16 * np, 16 * kk, lane);
                        mma_bf16_16816(accO[2 * np], a, b[0], b[1]);
                        mma_bf16_16816(accO[2 * np + 1], a, b[2], b[3]);
                    }
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int row = m0 + (lane >> 2) + 8 * h;
                    const int col = 8 * nt + 2 * (lane & 3);
                    if (warp < 4) {
                        const int s = sStep[row];
                        const float bs = sBeta[s];
                        const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sY + row * LDY + col));
                        if (REG) {
                            const float gs = exp2f(sG2[s]);
                            *reinterpret_cast<uint32_t *>(sR + row * LDY + col) =
                                pack_bf16x2(bs * (y.x - gs * accO[nt][2 * h]), bs * (y.y - gs * accO[nt][2 * h + 1]));
                        } else {
                            const float f = exp2f(gl - sG2[s]);
                            const float u0 = bs * y.x, u1 = bs * y.y;
                            *reinterpret_cast<uint32_t *>(sU + row * LDY + col) = pack_bf16x2(u0, u1);
                            *reinterpret_cast<uint32_t *>(sU2 + row * LDY + col) = pack_bf16x2(f * u0, f * u1);
                        }
                    } else {
                        const float gi = exp2f(sG2[row]);
                        accO[nt][2 * h] *= gi;
                        accO[nt][2 * h + 1] *= gi;
                    }
                }
        }
        __syncthreads();

        // ---- (6) U = T R and its decayed copy for the state update (regression family)
        if (REG) {
            if (warp < 4) {  // accO is dead in warps 0-3 after (5): reuse it for U
                const int m0 = 16 * warp;
                float (&acc)[NT][4] = accO;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int h = 0; h < 4; ++h) acc[nt][h] = 0.f;
#pragma unroll
                for (int kk = 0; kk < ET / 16; ++kk) {
                    uint32_t a[4];
                    load_a_rm(a, sT, LDE, m0, 16 * kk, lane);
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        uint32_t b[4];
                        load_b_kn(b, sR, LDY, 16 * np, 16 * kk, lane);
                        mma_bf16_16816(acc[2 * np], a, b[0], b[1]);
                        mma_bf16_16816(acc[2 * np + 1], a, b[2], b[3]);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int row = m0 + (lane >> 2) + 8 * h;
                        const int col = 8 * nt + 2 * (lane & 3);
                        const float f = exp2f(gl - sG2[sStep[row]]);
                        const float u0 = acc[nt][2 * h], u1 = acc[nt][2 * h + 1];
                        *reinterpret_cast<uint32_t *>(sU + row * LDY + col) = pack_bf16x2(u0, u1);
                        *reinterpret_cast<uint32_t *>(sU2 + row * LDY + col) = pack_bf16x2(f * u0, f * u1);
                    }
            }
            __syncthreads();
        }

        // ---- (7a) O = diag(2^g) Q S^T + P U, written out
        if (warp >= 4) {
            const int m0 = 16 * (warp - 4);
#pragma unroll
            for (int kk = 0; kk < ET / 16; ++kk) {
                uint32_t a[4];
                load_a_rm(a, sP, LDE, m0, 16 * kk, lane);
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    uint32_t b[4];
                    load_b_kn(b, sU, LDY, 16 * np, 16 * kk, lane);
                    mma_bf16_16816(accO[2 * np], a, b[0], b[1]);
                    mma_bf16_16816(accO[2 * np + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int i = m0 + (lane >> 2) + 8 * h;
                    const int col = 8 * nt + 2 * (lane & 3);
                    if (i < nval)
                        Io<IO>::st2(o, (size_t)(t0 + i) * dv + dv0 + col, accO[nt][2 * h], accO[nt][2 * h + 1]);
                }
        }
        // ---- (7b) S^T <- 2^(g_last) S^T + X^T U'
        if (warp < S_WARPS) {
            const float dl = exp2f(gl);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int h = 0; h < 4; ++h) accS[nt][h] *= dl;
#pragma unroll
            for (int kk = 0; kk < ET / 16; ++kk) {
                uint32_t a[4];
                load_a_km(a, sX, LDX, 16 * warp, 16 * kk, lane);
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    uint32_t b[4];
                    load_b_kn(b, sU2, LDY, 16 * np, 16 * kk, lane);
                    mma_bf16_16816(accS[2 * np], a, b[0], b[1]);
                    mma_bf16_16816(accS[2 * np + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int c = 8 * nt + 2 * (lane & 3);
                *reinterpret_cast<uint32_t *>(sS + sr * LDY + c) = pack_bf16x2(accS[nt][0], accS[nt][1]);
                *reinterpret_cast<uint32_t *>(sS + (sr + 8) * LDY + c) = pack_bf16x2(accS[nt][2], accS[nt][3]);
            }
        }
        __syncthreads();
    }

    // ---- final state and the continuation key
    if (p.S_out && warp < S_WARPS) {
        float *So = p.S_out + bh * (size_t)dv * DK;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int c = 8 * nt + 2 * (lane & 3);
            So[(size_t)(dv0 + c) * DK + sr] = accS[nt][0];
            So[(size_t)(dv0 + c + 1) * DK + sr] = accS[nt][1];
            So[(size_t)(dv0 + c) * DK + sr + 8] = accS[nt][2];
            So[(size_t)(dv0 + c + 1) * DK + sr + 8] = accS[nt][3];
        }
    }
    if (p.k_last && dv0 == 0) {
        IO *kl = reinterpret_cast<IO *>(p.k_last) + bh * (size_t)DK;
        for (int c = tid; c < DK; c += kChunkThreads) {
            float x = 0.f;
            if (T >= 1) x = Io<IO>::ld(k, (size_t)(T - 1) * DK + c);
            else if (kp) x = Io<IO>::ld(kp, c);
            Io<IO>::st(kl, c, x);
        }
    }
}

template <int DK, int DVS, bool REG, typename IO>
cudaError_t launch_chunk_t(const ChunkParams &p, cudaStream_t s) {
    using L = ChunkSmem<DK, DVS>;
    auto kern = chunk_fwd_kernel<DK, DVS, REG, IO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
    if (e != cudaSuccess) return e;
    const long grid = (long)p.B * p.H * (p.dv / DVS);
    if (grid == 0) return cudaSuccess;
    kern<<<(unsigned)grid, kChunkThreads, L::bytes, s>>>(p);
    return cudaGetLastError();
}

template <int DK, int DVS>
cudaError_t launch_chunk_dk_dvs(const ChunkParams &p, cudaStream_t s) {
    if (!p.io_bf16) return cudaErrorInvalidValue;  // the entry point admits bf16 I/O only
    return p.regression ? launch_chunk_t<DK, DVS, true, __nv_bfloat16>(p, s)
                        : launch_chunk_t<DK, DVS, false, __nv_bfloat16>(p, s);
}

// Per-DK dispatchers, one translation unit each (compile in parallel).
cudaError_t launch_chunk_dk32(const ChunkParams &p, int dvs, cudaStream_t s);
cudaError_t launch_chunk_dk64(const ChunkParams &p, int dvs, cudaStream_t s);
cudaError_t launch_chunk_dk128(const ChunkParams &p, int dvs, cudaStream_t s);

#define FALCON_CHUNK_DK_DISPATCH(DKV)                                                   \
    cudaError_t launch_chunk_dk##DKV(const ChunkParams &p, int dvs, cudaStream_t s) {    \
        switch (dvs) {                                                                  \
            case 16: return launch_chunk_dk_dvs<DKV, 16>(p, s);                          \
            case 32: return launch_chunk_dk_dvs<DKV, 32>(p, s);                          \
            case 64: return launch_chunk_dk_dvs<DKV, 64>(p, s);                          \
            case 128: return launch_chunk_dk_dvs<DKV, 128>(p, s);                        \
            default: return cudaErrorInvalidValue;                                      \
        }                                                                               \
    }

}  // namespace falcon
