// chunk_ws.cu -- warp-specialised chunk-parallel forward pass on tcgen05 for
// d_k = d_v = 128, bf16 I/O, one pair per step (Falcon-1, Falcon-1A), 64-token
// blocks. The block algebra is the chunk-parallel form with positive-decay
// renormalisation of "Fast Weight Attention for Continual Learning" (authors'
// abstract), written out in chunk_kernel.cuh.
//
// One CTA of 512 threads per (b, h). The state-independent work of block c+1
// (Gram tiles, triangular solve) runs while the state-dependent chain of block
// c runs, on separate warps that hand work over through mbarriers:
//   warp 0      TMA producer: [X;Q] and V of each block (2 stages)
//   warp 1      MMA issuer: (a) [X;Q]X^T -> G,P   (b) S X^T -> SX, S Q~^T -> O
//                           (d) U^T = R^T T^T   (e) O += U^T P~^T   (f) dS = U^T X~
//               issued as soon as their inputs are ready (critical chain first)
//   warps 2-3   helpers: x_1 patch, key norms, step sizes, cumulative log2 decay
//               and its tables; Q~ = diag(2^g) Q after (a); X~ = diag(2^(g_last-g)) X
//               after (b), so the state update needs no extra scaled copy
//   warps 4-7   local: L = diag(beta)(Gamma o G) (fp32), P~ = Gamma o P (bf16),
//               T = (I + L)^-1 (fp32, tensor-core tf32 block products)
//   warps 8-15  chain: R^T = diag(beta)(Y - diag(2^g) SX)^T, U^T to bf16, the fp32
//               state S <- 2^g_last S + dS (in registers) and its bf16 copy, O out
// Every decay factor is 2^(g_i - g_j) with i >= j (never a quotient of
// cumulative products). Every wait is bounded; a timeout is recorded in the
// device error word and all roles unwind.
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
#include "tc_common.cuh"

namespace falcon {

namespace {

constexpr int kThreads = 512;
constexpr int kBlk = 64;
constexpr long long kWaitBudget = 1ll << 31;  // SM clocks, about 1 s
constexpr int LDF = 68;                       // fp32 solve buffers: 16-byte rows, conflict-free A fragments

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t kStage = 49152;                 // [X;Q] 2 atoms x 128 rows + V 2 atoms x 64 rows
constexpr uint32_t oStage = 0;                     // 2 stages
constexpr uint32_t oS = 2 * kStage;                // S bf16: 2 atoms x 128 rows (A of (b))
constexpr uint32_t oRT = oS + 32768;               // R^T then U^T: 1 atom x 128 rows
constexpr uint32_t oT = oRT + 16384;               // T bf16 x 2 slots (B of (d))
constexpr uint32_t oP = oT + 16384;                // P~ bf16 x 2 slots (B of (e))
constexpr uint32_t oL = oP + 16384;                // L / W fp32 64 x LDF
constexpr uint32_t oTf = oL + 64 * LDF * 4;        // T fp32 64 x LDF
constexpr uint32_t oScal = oTf + 64 * LDF * 4;     // 3 slots x {beta, gam, f, g2}[64] + g_last[3] + misc
constexpr uint32_t oBar = oScal + 3 * 1024 + 64;
constexpr uint32_t kSmem = oBar + 64 * 8 + 1024;
static_assert(kSmem <= 232448, "shared memory");

// TMEM columns
constexpr uint32_t cGP = 0, cSX = 64, cO = 128 /* + 64 * slot */, cUT = 256, cDS = 320, kTmemCols = 512;

constexpr uint32_t kIdN64 = tc::idesc_bf16(128, 64, 0, 0);
constexpr uint32_t kIdN128Bmn = tc::idesc_bf16(128, 128, 0, 1);

// barrier indices
enum {
    B_FULL = 0,        // [2] TMA -> helpers
    B_SFREE = 2,       // [2] (f) done -> producer
    B_XQ = 4,          // helpers -> MMA (a)
    B_ADONE = 5,       // (a) done -> helpers, local
    B_GPFREE = 6,      // local read G/P -> MMA (a) of the next block
    B_SCAL = 7,        // [3] helpers -> local, chain (scalar slot c % 3)
    B_QSC = 10,        // Q~ ready -> MMA (b)
    B_BDONE = 11,      // (b) done -> helpers, chain
    B_XSC = 12,        // X~ ready -> MMA (f)
    B_RT = 13,         // R^T ready -> MMA (d)
    B_TRDY = 14,       // [2] T ready -> MMA (d)
    B_PRDY = 16,       // [2] P~ ready -> MMA (e)
    B_DDONE = 18,      // (d) done -> chain
    B_TFREE = 19,      // [2] (d) done -> local (T slot free)
    B_URDY = 21,       // U^T ready -> MMA (e),(f)
    B_EFDONE = 22,     // (e),(f) done -> chain
    B_PFREE = 23,      // [2] (e) done -> local (P~ slot free)
    B_SRDY = 25,       // S bf16 ready -> MMA (b)
    B_OFREE = 26,      // [2] O slot read -> MMA (b)
    B_FINAL = 28,      // MMA drain at exit
    B_COUNT = 29
};

__device__ __forceinline__ void named_bar(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void st_chunk8(uint8_t *base, uint32_t off, const float *v8) {
    uint4 pk;
    pk.x = pack_bf16x2(v8[0], v8[1]);
    pk.y = pack_bf16x2(v8[2], v8[3]);
    pk.z = pack_bf16x2(v8[4], v8[5]);
    pk.w = pack_bf16x2(v8[6], v8[7]);
    *reinterpret_cast<uint4 *>(base + off) = pk;
}

// Scale the 16 chunks (128 bf16) of row `r` of a two-atom, 128-row-per-atom tile by `s`.
__device__ __forceinline__ void scale_row(uint8_t *tile, int r, float s) {
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            uint4 *pp = reinterpret_cast<uint4 *>(tile + a * 16384 + tc::sw128_chunk(r, ch));
            uint4 u = *pp;
            __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 f = __bfloat1622float2(h[k]);
                h[k] = __floats2bfloat162_rn(f.x * s, f.y * s);
            }
            *pp = u;
        }
}

// ---- tf32 warp MMA for the 16 x 16 blocks of the triangular solve
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// acc (16 x 16, two 16x8 n-tiles) += A (16 x 16, row stride LDF) * B (16 x 16, row stride LDF)
__device__ __forceinline__ void mma16_acc(float (&acc)[2][4], const float *A, const float *B, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = to_tf32(A[g * LDF + 8 * ks + t]);
        const uint32_t a1 = to_tf32(A[(g + 8) * LDF + 8 * ks + t]);
        const uint32_t a2 = to_tf32(A[g * LDF + 8 * ks + t + 4]);
        const uint32_t a3 = to_tf32(A[(g + 8) * LDF + 8 * ks + t + 4]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = to_tf32(B[(8 * ks + t) * LDF + 8 * nt + g]);
            const uint32_t b1 = to_tf32(B[(8 * ks + t + 4) * LDF + 8 * nt + g]);
            mma_tf32(acc[nt], a0, a1, a2, a3, b0, b1);
        }
    }
}

__device__ __forceinline__ void store16(float *C, const float (&acc)[2][4], int lane, float sign) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        C[g * LDF + 8 * nt + 2 * t] = sign * acc[nt][0];
        C[g * LDF + 8 * nt + 2 * t + 1] = sign * acc[nt][1];
        C[(g + 8) * LDF + 8 * nt + 2 * t] = sign * acc[nt][2];
        C[(g + 8) * LDF + 8 * nt + 2 * t + 1] = sign * acc[nt][3];
    }
}

// T = (I + L)^-1 for strictly lower L (64 x 64 fp32) by 16 x 16 blocks, run by the
// 128 threads of the local warpgroup (named barrier 2):
//   diagonal blocks by forward substitution (one thread per column);
//   W_im = -T_ii L_im (stored over L_im); T_ij = sum_{m=j}^{i-1} W_im T_mj per block diagonal.
// Entries above the block diagonal of Tf are zero on entry and stay zero.
__device__ __forceinline__ void solve_local(float *sL, float *sTf, int lt, int lw, int lane) {
    if (lt < 64) {
        const int b = lt >> 4, j = lt & 15;
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
    named_bar(2, 128);
    // W blocks (i, m): (1,0) (2,0) (2,1) (3,0) (3,1) (3,2); warp lw takes blocks lw and lw + 4
    float wacc[2][2][4];
    int nw = 0;
    int wi[2], wm[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int blk = lw + 4 * k;
        if (blk < 6) {
            const int i = blk < 1 ? 1 : (blk < 3 ? 2 : 3);
            const int m = blk < 1 ? 0 : (blk < 3 ? blk - 1 : blk - 3);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 4; ++h) wacc[k][nt][h] = 0.f;
            mma16_acc(wacc[k], sTf + (16 * i) * LDF + 16 * i, sL + (16 * i) * LDF + 16 * m, lane);
            wi[k] = i;
            wm[k] = m;
            nw = k + 1;
        }
    }
    named_bar(2, 128);
#pragma unroll
    for (int k = 0; k < 2; ++k)
        if (k < nw) store16(sL + (16 * wi[k]) * LDF + 16 * wm[k], wacc[k], lane, -1.f);
    named_bar(2, 128);
#pragma unroll
    for (int d = 1; d < 4; ++d) {
        const int j = lw;          // block column; warp lw computes T_{j+d, j}
        const int i = j + d;
        if (i < 4) {
            float acc[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 4; ++h) acc[nt][h] = 0.f;
            for (int m = j; m < i; ++m)
                mma16_acc(acc, sL + (16 * i) * LDF + 16 * m, sTf + (16 * m) * LDF + 16 * j, lane);
            store16(sTf + (16 * i) * LDF + 16 * j, acc, lane, 1.f);
        }
        named_bar(2, 128);
    }
}

}  // namespace

template <bool REG>
__global__ void __launch_bounds__(kThreads, 1)
chunk_ws_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                const __grid_constant__ CUtensorMap tmV, ChunkParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sS = sm + oS;
    uint8_t *sRT = sm + oRT;
    float *sL = reinterpret_cast<float *>(sm + oL);
    float *sTf = reinterpret_cast<float *>(sm + oTf);
    // Scalars of block c live in slot c % 3 (beta[64] gam[64] f[64] g2[64]); three slots, because the
    // helpers prepare block c+1 while the chain may still read block c-1.
    float *sScal = reinterpret_cast<float *>(sm + oScal);
    float *sGL = sScal + 768;                              // g_last per slot
    float *sMisc = sScal + 772;                            // helper scan carry
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + oBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int T = p.T;
    const int nblk = (T + kBlk - 1) / kBlk;
    constexpr int D = 128;

    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) tc::mbar_init(&bars[i], 1);
        *abort_flag = 0;
        tc::mbar_fence_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tslot, kTmemCols);
        tc::tmem_relinquish();
    }
    for (int idx = tid; idx < 64 * LDF; idx += kThreads) sTf[idx] = 0.f;
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tslot;

    // Leader-polled bounded wait, made uniform across a role with its named barrier.
    auto role_wait = [&](uint64_t *bar, uint32_t parity, bool leader, int bar_id, int nthr) -> bool {
        if (leader && !tc::mbar_wait(bar, parity, abort_flag, kWaitBudget)) *abort_flag = 1;
        named_bar(bar_id, nthr);
        return *abort_flag == 0;
    };

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            for (int c = 0; c < nblk; ++c) {
                const int s = c & 1;
                if (c >= 2 && !tc::mbar_wait(&bars[B_SFREE + s], ((c >> 1) + 1) & 1, abort_flag, kWaitBudget)) {
                    *abort_flag = 1;
                    break;
                }
                uint8_t *stg = sm + oStage + s * kStage;
                const int t0 = c * kBlk;
                uint64_t *fb = &bars[B_FULL + s];
                tc::mbar_arrive_expect_tx(fb, kStage);
                tc::tma_load_3d(stg + 0, &tmK, 0, t0 - 1, bh, fb);
                tc::tma_load_3d(stg + 16384, &tmK, 64, t0 - 1, bh, fb);
                tc::tma_load_3d(stg + 8192, &tmQ, 0, t0, bh, fb);
                tc::tma_load_3d(stg + 24576, &tmQ, 64, t0, bh, fb);
                tc::tma_load_3d(stg + 32768, &tmV, 0, t0, bh, fb);
                tc::tma_load_3d(stg + 40960, &tmV, 64, t0, bh, fb);
            }
            // drain: every armed stage must have landed before the CTA can exit
            const volatile int no_abort = 0;
            for (int c = nblk - 2 < 0 ? 0 : nblk - 2; c < nblk; ++c)
                tc::mbar_wait(&bars[B_FULL + (c & 1)], (c >> 1) & 1, &no_abort, kWaitBudget);
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            const uint32_t aS = tc::smem_u32(sS), aRT = tc::smem_u32(sRT);
            int na = 0, nb = 0, nd = 0, nef = 0;
            long long idle_since = clock64();
            while (nef < nblk && !*abort_flag) {
                bool prog = false;
                // (e) + (f)
                if (nef < (REG ? nd : nb)) {
                    const int c = nef, s = c & 1;
                    if (tc::mbar_try_wait(&bars[B_URDY], c & 1) &&
                        tc::mbar_try_wait(&bars[B_PRDY + s], (c >> 1) & 1) &&
                        tc::mbar_try_wait(&bars[B_XSC], c & 1)) {
                        tc::fence_after_sync();
                        const uint32_t aX = tc::smem_u32(sm + oStage + s * kStage);
                        const uint32_t aP = tc::smem_u32(sm + oP + s * 8192);
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            tc::mma_bf16(tbase + cO + 64 * s, tc::sdesc(aRT + ks * 32, 16, 1024),
                                         tc::sdesc(aP + ks * 32, 16, 1024), kIdN64, 1);
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            tc::mma_bf16(tbase + cDS, tc::sdesc(aRT + ks * 32, 16, 1024),
                                         tc::sdesc(aX + ks * 2048, 16384, 1024), kIdN128Bmn, ks > 0);
                        tc::mma_commit(&bars[B_EFDONE]);
                        tc::mma_commit(&bars[B_PFREE + s]);
                        tc::mma_commit(&bars[B_SFREE + s]);
                        ++nef;
                        prog = true;
                    }
                }
                // (d)
                if (REG && nd < nb) {
                    const int c = nd, s = c & 1;
                    if (tc::mbar_try_wait(&bars[B_RT], c & 1) && tc::mbar_try_wait(&bars[B_TRDY + s], (c >> 1) & 1)) {
                        tc::fence_after_sync();
                        const uint32_t aT = tc::smem_u32(sm + oT + s * 8192);
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            tc::mma_bf16(tbase + cUT, tc::sdesc(aRT + ks * 32, 16, 1024),
                                         tc::sdesc(aT + ks * 32, 16, 1024), kIdN64, ks > 0);
                        tc::mma_commit(&bars[B_DDONE]);
                        tc::mma_commit(&bars[B_TFREE + s]);
                        ++nd;
                        prog = true;
                    }
                }
                // (b)
                if (nb < na) {
                    const int c = nb, s = c & 1;
                    if (tc::mbar_try_wait(&bars[B_QSC], c & 1) && tc::mbar_try_wait(&bars[B_SRDY], c & 1) &&
                        (c < 2 || tc::mbar_try_wait(&bars[B_OFREE + s], ((c >> 1) + 1) & 1))) {
                        tc::fence_after_sync();
                        const uint32_t aX = tc::smem_u32(sm + oStage + s * kStage);
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks) {
                            const uint32_t ko = (ks >> 2) * 16384 + (ks & 3) * 32;
                            tc::mma_bf16(tbase + cSX, tc::sdesc(aS + ko, 16, 1024), tc::sdesc(aX + ko, 16, 1024),
                                         kIdN64, ks > 0);
                        }
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks) {
                            const uint32_t ko = (ks >> 2) * 16384 + (ks & 3) * 32;
                            tc::mma_bf16(tbase + cO + 64 * s, tc::sdesc(aS + ko, 16, 1024),
                                         tc::sdesc(aX + 8192 + ko, 16, 1024), kIdN64, ks > 0);
                        }
                        tc::mma_commit(&bars[B_BDONE]);
                        ++nb;
                        prog = true;
                    }
                }
                // (a)
                if (na < nblk) {
                    const int c = na, s = c & 1;
                    if (tc::mbar_try_wait(&bars[B_XQ], c & 1) &&
                        (c < 1 || tc::mbar_try_wait(&bars[B_GPFREE], (c - 1) & 1))) {
                        tc::fence_after_sync();
                        const uint32_t aX = tc::smem_u32(sm + oStage + s * kStage);
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks) {
                            const uint32_t ko = (ks >> 2) * 16384 + (ks & 3) * 32;
                            tc::mma_bf16(tbase + cGP, tc::sdesc(aX + ko, 16, 1024), tc::sdesc(aX + ko, 16, 1024),
                                         kIdN64, ks > 0);
                        }
                        tc::mma_commit(&bars[B_ADONE]);
                        ++na;
                        prog = true;
                    }
                }
                if (prog) {
                    idle_since = clock64();
                } else if (clock64() - idle_since > kWaitBudget) {
                    *abort_flag = 1;
                }
            }
            // drain every MMA issued so far
            tc::mma_commit(&bars[B_FINAL]);
            const volatile int no_abort = 0;
            tc::mbar_wait(&bars[B_FINAL], 0, &no_abort, kWaitBudget);
        }
    } else if (warp < 4) {
        // ================================================================ helpers (64 threads)
        const int ht = tid - 64;           // row / token index 0..63
        const bool leader = ht == 0;
        const float *alpha_h = p.alpha + (size_t)bh * T, *eta_h = p.eta + (size_t)bh * T;
        float ga = 1.f, ge = 0.f;          // gates of the block prep() handles next
        auto load_gates = [&](int c) {
            const int t = c * kBlk + ht;
            ga = t < T ? alpha_h[t] : 1.f;
            ge = t < T ? eta_h[t] : 0.f;
        };
        auto prep = [&](int c) -> bool {   // block c: x_1 patch, norms, step sizes, decay tables
            const int s = c & 1, u = c % 3;
            uint8_t *stg = sm + oStage + s * kStage;
            if (!role_wait(&bars[B_FULL + s], (c >> 1) & 1, leader, 1, 64)) return false;
            const int t0 = c * kBlk, nval = min(kBlk, T - t0);
            if (c == 0 && p.k_prev && ht < 16) {
                const uint4 v = *reinterpret_cast<const uint4 *>(
                    reinterpret_cast<const __nv_bfloat16 *>(p.k_prev) + (size_t)bh * D + ht * 8);
                *reinterpret_cast<uint4 *>(stg + (ht >> 3) * 16384 + (ht & 7) * 16) = v;
                tc::fence_proxy_async();
            }
            named_bar(1, 64);
            float nrm = 0.f;
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(stg + a * 16384 + tc::sw128_chunk(ht, ch));
                    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 f = __bfloat1622float2(h2[k]);
                        nrm += f.x * f.x + f.y * f.y;
                    }
                }
            const bool valid = ht < nval;
            float la = valid ? log2f(ga) : 0.f;
            const float bt = valid ? step_size(ge, nrm, p.eps) : 0.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, la, off);
                if (lane >= off) la += y;
            }
            if (ht == 31) sMisc[0] = la;
            named_bar(1, 64);
            if (ht >= 32) la += sMisc[0];
            float *sc = sScal + u * 256;
            sc[ht] = bt;
            sc[128 + ht] = 0.f;  // placeholder, f filled below
            sc[192 + ht] = la;
            sc[64 + ht] = exp2f(la);
            named_bar(1, 64);
            const float gl = sc[192 + nval - 1];
            sc[128 + ht] = exp2f(gl - la);
            if (leader) sGL[u] = gl;
            named_bar(1, 64);
            if (leader) {
                mbar_arrive(&bars[B_SCAL + u]);
                mbar_arrive(&bars[B_XQ]);
            }
            return true;
        };
        if (nblk > 0) load_gates(0);
        bool ok = nblk > 0 ? prep(0) : true;
        for (int c = 0; c < nblk && ok; ++c) {
            const int s = c & 1;
            if (c + 1 < nblk) load_gates(c + 1);  // in flight while block c's Q is scaled
            uint8_t *stg = sm + oStage + s * kStage;
            const float *sc = sScal + (c % 3) * 256;
            // Q~ = diag(2^g) Q once (a) no longer needs Q
            if (!(ok = role_wait(&bars[B_ADONE], c & 1, leader, 1, 64))) break;
            scale_row(stg, 64 + ht, sc[64 + ht]);
            tc::fence_proxy_async();
            named_bar(1, 64);
            if (leader) mbar_arrive(&bars[B_QSC]);
            // next block's prep overlaps this block's chain
            if (c + 1 < nblk && !(ok = prep(c + 1))) break;
            // X~ = diag(2^(g_last - g)) X once (b) no longer needs X
            if (!(ok = role_wait(&bars[B_BDONE], c & 1, leader, 1, 64))) break;
            scale_row(stg, ht, sc[128 + ht]);
            tc::fence_proxy_async();
            named_bar(1, 64);
            if (leader) mbar_arrive(&bars[B_XSC]);
        }
    } else if (warp < 8) {
        // ================================================================ local (128 threads)
        const int lt = tid - 128, lw = warp - 4;
        const int r = 32 * lw + lane;      // TMEM lane: G row (r < 64) or P row r - 64
        const bool leader = lt == 0;
        const uint32_t tl = tbase + ((uint32_t)(32 * lw) << 16);
        for (int c = 0; c < nblk; ++c) {
            const int s = c & 1;
            if (!role_wait(&bars[B_ADONE], c & 1, leader, 2, 128)) break;
            if (!role_wait(&bars[B_SCAL + c % 3], (c / 3) & 1, leader, 2, 128)) break;
            tc::fence_after_sync();
            float v[64];
            {
                float h0[32], h1[32];
                tc::tmem_ld32(tl + cGP, h0);
                tc::tmem_ld32(tl + cGP + 32, h1);
#pragma unroll
                for (int j = 0; j < 32; ++j) { v[j] = h0[j]; v[32 + j] = h1[j]; }
            }
            tc::fence_before_sync();
            named_bar(2, 128);
            if (leader) mbar_arrive(&bars[B_GPFREE]);
            const float *sc = sScal + (c % 3) * 256;
            if (r < 64) {
                if (REG) {
                    const float be = sc[r], ge = sc[192 + r];
                    float *Lr = sL + r * LDF;
#pragma unroll
                    for (int j0 = 0; j0 < 64; j0 += 4) {
                        float4 w;
                        w.x = j0 + 0 < r ? be * exp2f(ge - sc[192 + j0 + 0]) * v[j0 + 0] : 0.f;
                        w.y = j0 + 1 < r ? be * exp2f(ge - sc[192 + j0 + 1]) * v[j0 + 1] : 0.f;
                        w.z = j0 + 2 < r ? be * exp2f(ge - sc[192 + j0 + 2]) * v[j0 + 2] : 0.f;
                        w.w = j0 + 3 < r ? be * exp2f(ge - sc[192 + j0 + 3]) * v[j0 + 3] : 0.f;
                        *reinterpret_cast<float4 *>(Lr + j0) = w;
                    }
                }
            } else {
                const int i = r - 64;
                // the P~ slot is free once (e) of block c-2 is done
                bool okp = c < 2 || tc::mbar_wait(&bars[B_PFREE + s], ((c >> 1) + 1) & 1, abort_flag, kWaitBudget);
                if (!okp) *abort_flag = 1;
                const float gi = sc[192 + i];
                uint8_t *sP = sm + oP + s * 8192;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    float pv[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int j = 8 * ch + k;
                        pv[k] = j <= i ? exp2f(gi - sc[192 + j]) * v[j] : 0.f;
                    }
                    st_chunk8(sP, tc::sw128_chunk(i, ch), pv);
                }
                tc::fence_proxy_async();
            }
            named_bar(2, 128);
            if (*abort_flag) break;
            if (leader) mbar_arrive(&bars[B_PRDY + s]);
            if (REG) {
                solve_local(sL, sTf, lt, lw, lane);
                if (c >= 2 && !role_wait(&bars[B_TFREE + s], ((c >> 1) + 1) & 1, leader, 2, 128)) break;
                uint8_t *sT = sm + oT + s * 8192;
                const int rr = lt >> 1, ch0 = 4 * (lt & 1);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const float4 x0 = *reinterpret_cast<const float4 *>(sTf + rr * LDF + 8 * (ch0 + cc));
                    const float4 x1 = *reinterpret_cast<const float4 *>(sTf + rr * LDF + 8 * (ch0 + cc) + 4);
                    const float t8[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    st_chunk8(sT, tc::sw128_chunk(rr, ch0 + cc), t8);
                }
                tc::fence_proxy_async();
                named_bar(2, 128);
                if (leader) mbar_arrive(&bars[B_TRDY + s]);
            }
        }
    } else {
        // ================================================================ chain (256 threads)
        const int ct = tid - 256;
        const int qd = warp & 3, hf = (warp - 8) >> 2;
        const int row = 32 * qd + lane;    // TMEM lane = value row
        const bool leader = ct == 0;
        const uint32_t tl = tbase + ((uint32_t)(32 * qd) << 16);
        float S[64];
        {
            const float *S0 = p.S0 ? p.S0 + ((size_t)bh * D + row) * D + 64 * hf : nullptr;
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
                const float4 x = S0 ? *reinterpret_cast<const float4 *>(S0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
            }
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_chunk8(sS + hf * 16384, tc::sw128_chunk(row, ch), S + 8 * ch);
            tc::fence_proxy_async();
            named_bar(3, 256);
            if (leader) mbar_arrive(&bars[B_SRDY]);
        }
        bool ok = true;
        for (int c = 0; c < nblk; ++c) {
            const int s = c & 1, t0 = c * kBlk, nval = min(kBlk, T - t0);
            if (!(ok = role_wait(&bars[B_BDONE], c & 1, leader, 3, 256))) break;
            if (!(ok = role_wait(&bars[B_SCAL + c % 3], (c / 3) & 1, leader, 3, 256))) break;
            tc::fence_after_sync();
            const float *sc = sScal + (c % 3) * 256;
            const float gl = sGL[c % 3];
            // R^T (or U^T) from S X^T and the values
            {
                float v[32], rv[32];
                tc::tmem_ld32(tl + cSX + 32 * hf, v);
                const uint8_t *Vt = sm + oStage + s * kStage + 32768 + (row >> 6) * 8192;
                const int dc = row & 63;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int e = 32 * hf + j;
                    const float y = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(
                        Vt + (e >> 3) * 1024 + (e & 7) * 128 + ((((dc >> 3) ^ (e & 7))) << 4) + (dc & 7) * 2));
                    rv[j] = REG ? sc[e] * (y - sc[64 + e] * v[j]) : sc[e] * y;
                }
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) st_chunk8(sRT, tc::sw128_chunk(row, 4 * hf + cc), rv + 8 * cc);
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            named_bar(3, 256);
            if (leader) mbar_arrive(&bars[REG ? B_RT : B_URDY]);
            if (REG) {
                if (!(ok = role_wait(&bars[B_DDONE], c & 1, leader, 3, 256))) break;
                tc::fence_after_sync();
                float v[32];
                tc::tmem_ld32(tl + cUT + 32 * hf, v);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) st_chunk8(sRT, tc::sw128_chunk(row, 4 * hf + cc), v + 8 * cc);
                tc::fence_proxy_async();
                tc::fence_before_sync();
                named_bar(3, 256);
                if (leader) mbar_arrive(&bars[B_URDY]);
            }
            // state update: S <- 2^g_last S + dS, then its bf16 copy for (b) of the next block
            if (!(ok = role_wait(&bars[B_EFDONE], c & 1, leader, 3, 256))) break;
            tc::fence_after_sync();
            {
                const float dl = exp2f(gl);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    tc::tmem_ld32(tl + cDS + 64 * hf + 32 * hh, v);
#pragma unroll
                    for (int j = 0; j < 32; ++j) S[32 * hh + j] = dl * S[32 * hh + j] + v[j];
                }
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) st_chunk8(sS + hf * 16384, tc::sw128_chunk(row, ch), S + 8 * ch);
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            named_bar(3, 256);
            if (leader) mbar_arrive(&bars[B_SRDY]);
            // outputs of this block (off the critical chain)
            {
                float v[32];
                tc::tmem_ld32(tl + cO + 64 * s + 32 * hf, v);
                __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(p.o) + ((size_t)bh * T + t0) * D + row;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int i = 32 * hf + j;
                    if (i < nval) o[(size_t)i * D] = __float2bfloat16_rn(v[j]);
                }
            }
            tc::fence_before_sync();
            named_bar(3, 256);
            if (leader) mbar_arrive(&bars[B_OFREE + s]);
        }
        if (ok && !*abort_flag) {
            if (p.S_out) {
                float *So = p.S_out + ((size_t)bh * D + row) * D + 64 * hf;
#pragma unroll
                for (int j = 0; j < 64; j += 4)
                    *reinterpret_cast<float4 *>(So + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
            }
            if (p.k_last && ct < 16) {
                const __nv_bfloat16 *src = nullptr;
                if (T >= 1) src = reinterpret_cast<const __nv_bfloat16 *>(p.k) + ((size_t)bh * T + (T - 1)) * D;
                else if (p.k_prev) src = reinterpret_cast<const __nv_bfloat16 *>(p.k_prev) + (size_t)bh * D;
                const uint4 x = src ? *reinterpret_cast<const uint4 *>(src + ct * 8) : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.k_last) + (size_t)bh * D + ct * 8) = x;
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && *abort_flag) set_error(p.err, kDevErrTimeout);
    if (warp == 0) tc::tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------------ host side

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_ws() {
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

// (128 columns, T rows, B*H heads) bf16 view with 64 x 64 boxes, 128-byte swizzle.
bool map_tile(CUtensorMap *m, const void *base, int T, long long BH) {
    cuuint64_t dims[3] = {128, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)T * 128 * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return encode_fn_ws()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool chunk_ws_supported(const ChunkParams &p) {
    return p.dk == 128 && p.dv == 128 && p.io_bf16 && p.window == 1 && p.tok_per_blk == kBlk && p.T >= 1 &&
           encode_fn_ws() != nullptr;
}

cudaError_t launch_chunk_ws(const ChunkParams &p, cudaStream_t s) {
    const long long BH = (long long)p.B * p.H;
    CUtensorMap mK, mQ, mV;
    if (!map_tile(&mK, p.k, p.T, BH) || !map_tile(&mQ, p.q, p.T, BH) || !map_tile(&mV, p.v, p.T, BH))
        return cudaErrorInvalidValue;
    auto kern = p.regression ? chunk_ws_kernel<true> : chunk_ws_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)BH, kThreads, kSmem, s>>>(mK, mQ, mV, p);
    return cudaGetLastError();
}

}  // namespace falcon
