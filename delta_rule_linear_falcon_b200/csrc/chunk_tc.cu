// chunk_tc.cu -- chunk-parallel forward pass on the 5th-generation tensor cores
// (tcgen05, TMEM accumulators, TMA-staged bf16 tiles) for d_k = d_v = 128,
// bf16 I/O and one pair per step (Falcon-1, Falcon-1A). This is the
// chunk-parallel form with positive-decay renormalisation of "Fast Weight
// Attention for Continual Learning" (authors' abstract); the block algebra is
// the one documented in chunk_kernel.cuh.
//
// One CTA of 256 threads per (b, h) walks the sequence in blocks of 64 tokens.
// Every product is an M = 128 tcgen05 MMA with the value index d_v on the
// TMEM lanes (thread t of warp w owns lane 32*(w%4) + lane, half w/4 of the
// columns):
//   (a) [X;Q] X^T        -> G (lanes 0-63) and P (lanes 64-127), 64 columns
//   (b) S [X;Q]^T        -> S X^T and S Q^T, 128 columns
//   (d) U^T = R^T T^T    (R = diag(beta)(Y - diag(2^g) X S^T), T = (I+L)^-1)
//   (e) O_p^T = U^T P~^T
//   (f) dS = U'^T X      (X read as an MN-major operand; U' = diag(2^(g_last-g)) U)
// The fp32 state lives in registers (64 values per thread); its bf16 copy in
// shared memory is the A operand of (b). TMA brings the next block's X (keys
// shifted by one token: x_t = k_{t-1}; the row before the sequence start and
// rows past its end are zero-filled by the tensor map), Q and V while the
// current block computes; O leaves through a TMA store.
// Every wait is bounded: on expiry the CTA records a timeout in the device
// error word and unwinds.
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
#include "tc_common.cuh"

namespace falcon {

namespace {

constexpr int kThreads = 256;
constexpr int kBlk = 64;                 // tokens (= pseudo-value rows) per block
constexpr long long kWaitBudget = 1ll << 31;  // SM clocks (about 1 s)

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t kStageBytes = 49152;        // [X;Q] 2 atoms x 128 rows (32 KB) + V 2 atoms x 64 rows (16 KB)
constexpr uint32_t oStage = 0;                 // 2 stages
constexpr uint32_t oS = 2 * kStageBytes;       // S bf16: 2 atoms x 128 rows
constexpr uint32_t oRT = oS + 32768;           // R^T, then U^T: 1 atom x 128 rows
constexpr uint32_t oU2 = oRT + 16384;          // U'^T: 1 atom x 128 rows (the solve's W scratch aliases nothing here)
constexpr uint32_t oT = oU2 + 16384;           // T bf16: 1 atom x 64 rows
constexpr uint32_t oP = oT + 8192;             // P~ bf16: 1 atom x 64 rows
constexpr uint32_t oL = oP + 8192;             // L fp32 64 x 65; reused as the O staging tile (16 KB)
constexpr uint32_t oTf = oL + 17408;           // T fp32 64 x 65
constexpr uint32_t oScal = oTf + 16640;        // beta[64], g2[64], norms[64], misc
constexpr uint32_t oBar = oScal + 1024;        // mbarriers + TMEM slot + abort flag
constexpr uint32_t kSmemBytes = oBar + 128 + 1024;  // + alignment slack
constexpr int LDF = 65;

// TMEM columns
constexpr uint32_t cGP = 0, cSX = 64, cSQ = 128, cUT = 192, cOT = 256, cDS = 320, kTmemCols = 512;

constexpr uint32_t kIdescN64 = tc::idesc_bf16(128, 64, 0, 0);
constexpr uint32_t kIdescN128 = tc::idesc_bf16(128, 128, 0, 0);
constexpr uint32_t kIdescN128Bmn = tc::idesc_bf16(128, 128, 0, 1);

__device__ __forceinline__ void st_chunk(uint8_t *base, uint32_t off, const float *v8) {
    uint4 pk;
    pk.x = pack_bf16x2(v8[0], v8[1]);
    pk.y = pack_bf16x2(v8[2], v8[3]);
    pk.z = pack_bf16x2(v8[4], v8[5]);
    pk.w = pack_bf16x2(v8[6], v8[7]);
    *reinterpret_cast<uint4 *>(base + off) = pk;
}

// T = (I + L)^-1 for a strictly lower-triangular 64 x 64 fp32 L (row stride LDF), in 16 x 16 blocks:
//  - diagonal blocks by right-looking forward substitution, one thread per column;
//  - W_im = -T_ii L_im for every block below the diagonal (overwrites L_im);
//  - T_ij = sum_{m=j}^{i-1} W_im T_mj, one block diagonal at a time.
// Entries above the block diagonal of Tf must be zero on entry.
__device__ __forceinline__ void solve_unit_lower(float *sL, float *sTf, int tid) {
    if (tid < 64) {
        const int b = tid >> 4, j = tid & 15;
        const float *Lb = sL + (16 * b) * LDF + 16 * b;
        float x[16], acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            x[m] = m < j ? 0.f : (m == j ? 1.f : -acc[m]);
#pragma unroll
            for (int i = m + 1; i < 16; ++i) acc[i] += Lb[i * LDF + m] * x[m];
        }
        float *Tb = sTf + (16 * b) * LDF + 16 * b;
#pragma unroll
        for (int i = 0; i < 16; ++i) Tb[i * LDF + j] = x[i];
    }
    __syncthreads();
    // W_im = -T_ii L_im for the 6 blocks (i, m), i > m; computed into registers, then stored over L_im.
    {
        float w[6];
        int pos[6];
        int n = 0;
#pragma unroll
        for (int blk = 0; blk < 6; ++blk) {
            const int i = blk < 1 ? 1 : (blk < 3 ? 2 : 3);
            const int m = blk < 1 ? 0 : (blk < 3 ? blk - 1 : blk - 3);
            const int r = tid >> 4, c = tid & 15;
            const float *Ti = sTf + (16 * i + r) * LDF + 16 * i;
            const float *Lim = sL + (16 * i) * LDF + 16 * m + c;
            float s = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k) s += Ti[k] * Lim[k * LDF];
            w[n] = -s;
            pos[n] = (16 * i + r) * LDF + 16 * m + c;
            ++n;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 6; ++k) sL[pos[k]] = w[k];
    }
    __syncthreads();
    // block diagonals d = 1, 2, 3
#pragma unroll
    for (int d = 1; d < 4; ++d) {
        for (int idx = tid; idx < (4 - d) * 256; idx += kThreads) {
            const int j = idx >> 8, i = j + d, r = (idx >> 4) & 15, c = idx & 15;
            const float *Wrow = sL + (16 * i + r) * LDF;
            float s = 0.f;
            for (int m = j; m < i; ++m) {
                const float *Tm = sTf + (16 * m) * LDF + 16 * j + c;
                const float *Wm = Wrow + 16 * m;
#pragma unroll
                for (int k = 0; k < 16; ++k) s += Wm[k] * Tm[k * LDF];
            }
            sTf[(16 * i + r) * LDF + 16 * j + c] = s;
        }
        __syncthreads();
    }
}

}  // namespace

template <bool REG>
__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                ChunkParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sS = sm + oS;
    uint8_t *sRT = sm + oRT;
    uint8_t *sU2 = sm + oU2;
    uint8_t *sT = sm + oT;
    uint8_t *sP = sm + oP;
    float *sL = reinterpret_cast<float *>(sm + oL);
    float *sTf = reinterpret_cast<float *>(sm + oTf);
    float *sBeta = reinterpret_cast<float *>(sm + oScal);
    float *sG2 = sBeta + 64;
    float *sNrm = sG2 + 64;
    float *sMisc = sNrm + 64;  // [0] = g_last
    uint64_t *bar_full = reinterpret_cast<uint64_t *>(sm + oBar);  // [2]
    uint64_t *bar_a = bar_full + 2;
    uint64_t *bar_b = bar_full + 3;
    uint64_t *bar_d = bar_full + 4;
    uint64_t *bar_ef = bar_full + 5;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_full + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, hf = warp >> 2;           // TMEM lane quarter, column half
    const int row = 32 * qd + lane;                    // TMEM lane = value row d_v (or G/P row)
    const int bh = blockIdx.x;
    const int T = p.T;
    const int nblk = (T + kBlk - 1) / kBlk;
    constexpr int D = 128;

    if (tid == 0) {
        tc::mbar_init(&bar_full[0], 1);
        tc::mbar_init(&bar_full[1], 1);
        tc::mbar_init(bar_a, 1);
        tc::mbar_init(bar_b, 1);
        tc::mbar_init(bar_d, 1);
        tc::mbar_init(bar_ef, 1);
        *abort_flag = 0;
        tc::mbar_fence_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tslot, kTmemCols);
        tc::tmem_relinquish();
    }
    for (int idx = tid; idx < 64 * LDF; idx += kThreads) sTf[idx] = 0.f;

    // initial state: thread owns S[row][64*hf .. 64*hf+63]
    float S[64];
    {
        const float *S0 = p.S0 ? p.S0 + ((size_t)bh * D + row) * D + 64 * hf : nullptr;
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
            float4 v = S0 ? *reinterpret_cast<const float4 *>(S0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = v.x; S[j + 1] = v.y; S[j + 2] = v.z; S[j + 3] = v.w;
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) st_chunk(sS + hf * 16384, tc::sw128_chunk(row, ch), S + 8 * ch);
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tslot;
    const uint32_t tl = tbase + ((uint32_t)(32 * qd) << 16);  // this warp's lane quarter

    auto issue_loads = [&](int c) {
        uint8_t *stg = sm + oStage + (c & 1) * kStageBytes;
        const int t0 = c * kBlk;
        tc::mbar_arrive_expect_tx(&bar_full[c & 1], kStageBytes);
        tc::tma_load_3d(stg + 0, &tmK, 0, t0 - 1, bh, &bar_full[c & 1]);      // X, atom 0
        tc::tma_load_3d(stg + 16384, &tmK, 64, t0 - 1, bh, &bar_full[c & 1]); // X, atom 1
        tc::tma_load_3d(stg + 8192, &tmQ, 0, t0, bh, &bar_full[c & 1]);       // Q, atom 0 (rows 64..127)
        tc::tma_load_3d(stg + 24576, &tmQ, 64, t0, bh, &bar_full[c & 1]);     // Q, atom 1
        tc::tma_load_3d(stg + 32768, &tmV, 0, t0, bh, &bar_full[c & 1]);      // V, dv 0..63
        tc::tma_load_3d(stg + 40960, &tmV, 64, t0, bh, &bar_full[c & 1]);     // V, dv 64..127
    };
    if (tid == 0 && nblk > 0) issue_loads(0);

    int pending_load = nblk > 0 ? 0 : -1;  // block whose loads may still be in flight
    bool ok = true;
    for (int c = 0; c < nblk; ++c) {
        const int t0 = c * kBlk;
        const int nval = min(kBlk, T - t0);
        const uint32_t par = c & 1;
        uint8_t *stg = sm + oStage + (c & 1) * kStageBytes;
        const uint32_t aXQ = tc::smem_u32(stg);

        // ---- P0: this block's tiles; prefetch the next block; free the O staging tile
        ok = tc::mbar_wait(&bar_full[c & 1], (c >> 1) & 1, abort_flag, kWaitBudget);
        if (__syncthreads_or(!ok)) break;
        pending_load = -1;
        if (tid == 0) {
            tc::tma_store_wait_read0();
            if (c + 1 < nblk) {
                issue_loads(c + 1);
                pending_load = c + 1;
            }
        }
        if (c == 0 && p.k_prev && tid < 16) {  // x_1 = k_prev: row 0 of X (row 0 is unswizzled)
            const uint4 v = *reinterpret_cast<const uint4 *>(
                reinterpret_cast<const __nv_bfloat16 *>(p.k_prev) + (size_t)bh * D + tid * 8);
            *reinterpret_cast<uint4 *>(stg + (tid >> 3) * 16384 + (tid & 7) * 16) = v;
            tc::fence_proxy_async();
        }
        __syncthreads();

        // ---- P1: key norms (4 threads per row), then step sizes and cumulative log2 decay
        {
            const int e = tid >> 2, part = tid & 3;
            const uint8_t *rowp = stg + (part >> 1) * 16384;
            float nrm = 0.f;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const uint4 u = *reinterpret_cast<const uint4 *>(rowp + tc::sw128_chunk(e, 4 * (part & 1) + cc));
                const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 f = __bfloat1622float2(h2[k]);
                    nrm += f.x * f.x + f.y * f.y;
                }
            }
            nrm += __shfl_xor_sync(0xffffffffu, nrm, 1);
            nrm += __shfl_xor_sync(0xffffffffu, nrm, 2);
            if (part == 0) sNrm[e] = nrm;
        }
        __syncthreads();
        if (warp == 0) {
            const float *alpha = p.alpha + (size_t)bh * T + t0;
            const float *eta = p.eta + (size_t)bh * T + t0;
            float la[2], bt[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int s = lane + 32 * hh;
                const bool valid = s < nval;
                la[hh] = valid ? log2f(alpha[s]) : 0.f;
                bt[hh] = valid ? step_size(eta[s], sNrm[s], p.eps) : 0.f;
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
            if (lane == 0) sMisc[0] = sG2[nval - 1];
        }
        __syncthreads();

        // ---- P2: issue (a) and (b); both overlap the local epilogue and the solve
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t aS = tc::smem_u32(sS);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t ko = (ks >> 2) * 16384 + (ks & 3) * 32;
                tc::mma_bf16(tbase + cGP, tc::sdesc(aXQ + ko, 16, 1024), tc::sdesc(aXQ + ko, 16, 1024),
                             kIdescN64, ks > 0);
            }
            tc::mma_commit(bar_a);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t ko = (ks >> 2) * 16384 + (ks & 3) * 32;
                tc::mma_bf16(tbase + cSX, tc::sdesc(aS + ko, 16, 1024), tc::sdesc(aXQ + ko, 16, 1024),
                             kIdescN128, ks > 0);
            }
            tc::mma_commit(bar_b);
        }
        const float gl = sMisc[0];

        // ---- P3: L (fp32) from G, P~ (bf16) from P
        ok = tc::mbar_wait(bar_a, par, abort_flag, kWaitBudget);
        if (__syncthreads_or(!ok)) break;
        tc::fence_after_sync();
        {
            float v[32];
            tc::tmem_ld32(tl + cGP + 32 * hf, v);
            if (qd < 2) {
                if (REG) {
                    const int e = row;
                    const float be = sBeta[e], ge = sG2[e];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int e2 = 32 * hf + j;
                        sL[e * LDF + e2] = e2 < e ? be * exp2f(ge - sG2[e2]) * v[j] : 0.f;
                    }
                }
            } else {
                const int i = row - 64;
                const float gi = sG2[i];
                float pv[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int e2 = 32 * hf + j;
                    pv[j] = e2 <= i ? exp2f(gi - sG2[e2]) * v[j] : 0.f;
                }
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) st_chunk(sP, tc::sw128_chunk(i, 4 * hf + cc), pv + 8 * cc);
            }
        }
        tc::fence_proxy_async();
        __syncthreads();

        // ---- P4: T = (I + L)^-1 (regression family)
        if (REG) {
            solve_unit_lower(sL, sTf, tid);
            {
                const int r = tid >> 2, ch0 = 2 * (tid & 3);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
                    st_chunk(sT, tc::sw128_chunk(r, ch0 + cc), sTf + r * LDF + 8 * (ch0 + cc));
            }
            tc::fence_proxy_async();
        }

        // ---- P5: residuals R^T = diag(beta)(Y - diag(2^g) X S^T) (or U^T directly)
        ok = tc::mbar_wait(bar_b, par, abort_flag, kWaitBudget);
        if (__syncthreads_or(!ok)) break;
        tc::fence_after_sync();
        {
            float v[32];
            tc::tmem_ld32(tl + cSX + 32 * hf, v);
            const uint8_t *Vt = stg + 32768 + (row >> 6) * 8192;
            const int dcol = row & 63;
            float r[32], r2[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int e = 32 * hf + j;
                const float y = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(
                    Vt + tc::sw128_chunk(e, dcol >> 3) + (dcol & 7) * 2));
                const float be = sBeta[e];
                if (REG) {
                    r[j] = be * (y - exp2f(sG2[e]) * v[j]);
                } else {
                    r[j] = be * y;
                    r2[j] = exp2f(gl - sG2[e]) * r[j];
                }
            }
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) st_chunk(sRT, tc::sw128_chunk(row, 4 * hf + cc), r + 8 * cc);
            if (!REG) {
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) st_chunk(sU2, tc::sw128_chunk(row, 4 * hf + cc), r2 + 8 * cc);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();

        // ---- P6: U^T = R^T T^T and its decayed copy (regression family)
        if (REG) {
            if (tid == 0) {
                tc::fence_after_sync();
                const uint32_t aR = tc::smem_u32(sRT), aT = tc::smem_u32(sT);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tbase + cUT, tc::sdesc(aR + ks * 32, 16, 1024), tc::sdesc(aT + ks * 32, 16, 1024),
                                 kIdescN64, ks > 0);
                tc::mma_commit(bar_d);
            }
            ok = tc::mbar_wait(bar_d, par, abort_flag, kWaitBudget);
            if (__syncthreads_or(!ok)) break;
            tc::fence_after_sync();
            {
                float v[32], u2[32];
                tc::tmem_ld32(tl + cUT + 32 * hf, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) u2[j] = exp2f(gl - sG2[32 * hf + j]) * v[j];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    st_chunk(sRT, tc::sw128_chunk(row, 4 * hf + cc), v + 8 * cc);
                    st_chunk(sU2, tc::sw128_chunk(row, 4 * hf + cc), u2 + 8 * cc);
                }
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncthreads();
        }

        // ---- P7: (e) O_p^T = U^T P~^T and (f) dS = U'^T X
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t aU = tc::smem_u32(sRT), aP = tc::smem_u32(sP), aU2 = tc::smem_u32(sU2);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_bf16(tbase + cOT, tc::sdesc(aU + ks * 32, 16, 1024), tc::sdesc(aP + ks * 32, 16, 1024),
                             kIdescN64, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_bf16(tbase + cDS, tc::sdesc(aU2 + ks * 32, 16, 1024),
                             tc::sdesc(aXQ + ks * 2048, 16384, 1024), kIdescN128Bmn, ks > 0);
            tc::mma_commit(bar_ef);
        }
        ok = tc::mbar_wait(bar_ef, par, abort_flag, kWaitBudget);
        if (__syncthreads_or(!ok)) break;
        tc::fence_after_sync();

        // ---- P8: O = diag(2^g) Q S^T + P~ U (staged, TMA store) and S <- 2^g_last S + dS
        {
            float a[32], b[32];
            tc::tmem_ld32(tl + cSQ + 32 * hf, a);
            tc::tmem_ld32(tl + cOT + 32 * hf, b);
            __nv_bfloat16 *stO = reinterpret_cast<__nv_bfloat16 *>(sL) + (row >> 6) * 4096 + (row & 63);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int i = 32 * hf + j;
                stO[i * 64] = __float2bfloat16_rn(exp2f(sG2[i]) * a[j] + b[j]);
            }
            const float dl = exp2f(gl);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                tc::tmem_ld32(tl + cDS + 64 * hf + 32 * hh, a);
#pragma unroll
                for (int j = 0; j < 32; ++j) S[32 * hh + j] = dl * S[32 * hh + j] + a[j];
            }
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_chunk(sS + hf * 16384, tc::sw128_chunk(row, ch), S + 8 * ch);
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            tc::tma_store_3d(&tmO, sL, 0, t0, bh);
            tc::tma_store_3d(&tmO, reinterpret_cast<uint8_t *>(sL) + 8192, 64, t0, bh);
            tc::tma_store_commit();
        }
    }

    // ---- unwind: loads still in flight, stores, final state, TMEM
    if (!ok) {
        if (tid == 0) set_error(p.err, kDevErrTimeout);
        if (tid == 0 && pending_load >= 0) {
            const volatile int no_abort = 0;
            tc::mbar_wait(&bar_full[pending_load & 1], (pending_load >> 1) & 1, &no_abort, kWaitBudget);
        }
    }
    if (tid == 0) tc::tma_store_wait0();
    if (ok && p.S_out) {
        float *So = p.S_out + ((size_t)bh * D + row) * D + 64 * hf;
#pragma unroll
        for (int j = 0; j < 64; j += 4) *reinterpret_cast<float4 *>(So + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    if (ok && p.k_last && tid < 16) {
        const __nv_bfloat16 *src = nullptr;
        if (T >= 1) src = reinterpret_cast<const __nv_bfloat16 *>(p.k) + ((size_t)bh * T + (T - 1)) * D;
        else if (p.k_prev) src = reinterpret_cast<const __nv_bfloat16 *>(p.k_prev) + (size_t)bh * D;
        const uint4 v = src ? *reinterpret_cast<const uint4 *>(src + tid * 8) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.k_last) + (size_t)bh * D + tid * 8) = v;
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------------ host side

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 3-D view (128 columns, T rows, B*H heads) of a (B,H,T,128) bf16 tensor, 64 x 64 boxes.
bool make_map(CUtensorMap *m, const void *base, int T, long long BH, bool swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)T * 128 * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool chunk_tc_supported(const ChunkParams &p) {
    return p.dk == 128 && p.dv == 128 && p.io_bf16 && p.window == 1 && p.tok_per_blk == kBlk && p.T >= 1 &&
           encode_fn() != nullptr;
}

cudaError_t launch_chunk_tc(const ChunkParams &p, cudaStream_t s) {
    const long long BH = (long long)p.B * p.H;
    CUtensorMap mK, mQ, mV, mO;
    if (!make_map(&mK, p.k, p.T, BH, true) || !make_map(&mQ, p.q, p.T, BH, true) ||
        !make_map(&mV, p.v, p.T, BH, true) || !make_map(&mO, p.o, p.T, BH, false))
        return cudaErrorInvalidValue;
    auto kern = p.regression ? chunk_tc_kernel<true> : chunk_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)BH, kThreads, kSmemBytes, s>>>(mK, mQ, mV, mO, p);
    return cudaGetLastError();
}

}  // namespace falcon
