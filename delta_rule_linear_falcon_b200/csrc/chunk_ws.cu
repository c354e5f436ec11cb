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
//   warp 1      MMA issuer: (a) [X;Q]X^T -> G,P   (b) S [X;Q~]^T -> [SX | O] (N = 128),
//                           (y) V^T I -> Y^T (the tensor core transposes the values;
//                               issued right after (e),(f) of the previous block)
//                           (d) U^T = R^T T'^T  (e) O += U^T P~^T   (f) dS = U^T X~
//               issued as soon as their inputs are ready (critical chain first)
//   warps 2-3   helpers: x_1 patch, key norms, step sizes, cumulative log2 decay
//               and its tables; Q~ = diag(2^g) Q after (a); P~ = Gamma o P from TMEM
//               lanes 64-127 (their quarters)
//   warps 4-7   local: L = diag(beta)(Gamma o G) (fp32) from TMEM lanes 0-63,
//               T = (I + L)^-1 (fp32, tensor-core tf32 block products), stored as
//               T' = T diag(beta) so the residual needs no step size
//   warps 8-15  chain: R^T = (Y - diag(2^g) SX)^T; X~ = diag(2^(g_last-g)) X in place while
//               (d) runs, so the state update needs no extra scaled copy; U^T to bf16; the fp32
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
constexpr uint32_t oBar = oScal + 4 * 1024;        // 3 slots + 3 column-factor tables + g_last + misc
constexpr uint32_t oI = oBar + 1024;               // 64 x 64 bf16 identity (B of (y)), 1024-aligned
constexpr uint32_t kSmem = oI + 8192 + 1024;
static_assert(kSmem <= 232448, "shared memory");

// TMEM columns
// GP | [SX_0 | O_0] | [SX_1 | O_1] | Y^T, later U^T (same columns) | dS
constexpr uint32_t cGP = 0, cSXO = 64 /* + 128 * slot */, cUT = 320, cY = 320, cDS = 384, kTmemCols = 512;

constexpr uint32_t kIdN64 = tc::idesc_bf16(128, 64, 0, 0);
constexpr uint32_t kIdN128 = tc::idesc_bf16(128, 128, 0, 0);
constexpr uint32_t kIdN128Bmn = tc::idesc_bf16(128, 128, 0, 1);
constexpr uint32_t kIdN64Amn = tc::idesc_bf16(128, 64, 1, 0);

// barrier indices
enum {
    B_FULL = 0,        // [2] TMA -> helpers
    B_SFREE = 2,       // [2] (f) done -> producer
    B_XQ = 4,          // helpers -> MMA (a)
    B_ADONE = 5,       // (a) done -> helpers, local
    B_GPFREE = 6,      // local read G and helpers read P (2 arrivals) -> MMA (a) of the next block
    B_SCAL = 7,        // [3] helpers -> local, chain (scalar slot c % 3)
    B_QSC = 10,        // Q~ ready -> MMA (b)
    B_BDONE = 11,      // (b) done -> helpers, chain
    B_XSC = 12,        // (unused)
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
#pragma unroll 1
    for (int q = 0; q < 16; ++q) {
        const int a = q >> 3, ch = q & 7;
        {
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
    if (lt < 64) {  // column j of the inverse of diagonal block b, left-looking, rows of L as float4
        const int b = lt >> 4, j = lt & 15;
        const float *Lb = sL + (16 * b) * LDF + 16 * b;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float l[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float4 w = *reinterpret_cast<const float4 *>(Lb + i * LDF + 4 * q4);
                l[4 * q4] = w.x; l[4 * q4 + 1] = w.y; l[4 * q4 + 2] = w.z; l[4 * q4 + 3] = w.w;
            }
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int m = 0; m < i; ++m) {
                if (m & 1) a1 += l[m] * x[m];
                else a0 += l[m] * x[m];
            }
            x[i] = i < j ? 0.f : (i == j ? 1.f : -(a0 + a1));
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
    float *sGL = sScal + 960;                              // g_last per slot (after 3 x cf[64])
    float *sMisc = sScal + 964;                            // helper scan carry
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + oBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int T = p.T;
    const int nblk = (T + kBlk - 1) / kBlk;
    constexpr int D = 128;

    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) tc::mbar_init(&bars[i], i == B_GPFREE ? 2 : 1);
        *abort_flag = 0;
        tc::mbar_fence_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tslot, kTmemCols);
        tc::tmem_relinquish();
    }
    for (int idx = tid; idx < 64 * LDF; idx += kThreads) sTf[idx] = 0.f;
    for (int idx = tid; idx < 64 * 8; idx += kThreads) {  // identity, row e has a 1 at column e
        const int e = idx >> 3, ch = idx & 7;
        float v8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v8[k] = (8 * ch + k == e) ? 1.f : 0.f;
        st_chunk8(sm + oI, tc::sw128_chunk(e, ch), v8);
    }
    tc::fence_proxy_async();
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
            // Descriptors are built once; a K step only moves the 14-bit start-address field
            // (address >> 4), which stays below 2^14 for every operand here, so a plain add is exact.
            const uint64_t dS = tc::sdesc(tc::smem_u32(sS), 16, 1024);
            const uint64_t dRT = tc::sdesc(tc::smem_u32(sRT), 16, 1024);
            const uint64_t dI = tc::sdesc(tc::smem_u32(sm + oI), 16, 1024);
            uint64_t dX[2], dXmn[2], dV[2], dT[2], dP[2];
#pragma unroll
            for (int st = 0; st < 2; ++st) {
                const uint32_t a = tc::smem_u32(sm + oStage + st * kStage);
                dX[st] = tc::sdesc(a, 16, 1024);            // [X;Q] K-major (also X as N=64 / N=128 B)
                dXmn[st] = tc::sdesc(a, 16384, 1024);       // X as an MN-major B (dk atoms 16 KB apart)
                dV[st] = tc::sdesc(a + 32768, 8192, 1024);  // V as an MN-major A (dv atoms 8 KB apart)
                dT[st] = tc::sdesc(tc::smem_u32(sm + oT + st * 8192), 16, 1024);
                dP[st] = tc::sdesc(tc::smem_u32(sm + oP + st * 8192), 16, 1024);
            }
            auto kmaj = [](int ks) -> uint64_t { return (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4); };
            auto wait = [&](int b, uint32_t parity) -> bool {
                if (!tc::mbar_wait(&bars[b], parity, abort_flag, kWaitBudget)) {
                    *abort_flag = 1;
                    return false;
                }
                return true;
            };
            // (a): [X;Q] X^T -> G (lanes 0-63), P (lanes 64-127)
            auto issue_a = [&](int c) {
                const uint64_t d = dX[c & 1];
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) tc::mma_bf16(tbase + cGP, d + kmaj(ks), d + kmaj(ks), kIdN64, ks > 0);
                tc::mma_commit(&bars[B_ADONE]);
            };
            // (y): Y^T = V^T I (V read as an MN-major A operand of the stage tile)
            auto issue_y = [&](int c) {
                const uint64_t d = dV[c & 1];
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tbase + cY, d + (uint64_t)(ks * 128), dI + (uint64_t)(ks * 2), kIdN64Amn, ks > 0);
            };
            // Program order per block c (each wait parks this thread until its inputs are ready):
            //   (b)_c, then (a)_{c+1} (runs while the chain forms R_c), (d)_c, (e)(f)_c, then (y)_{c+1}
            //   (its columns are free once U^T_c has been read, which (e)(f)_c's inputs imply).
            bool ok = nblk > 0 && wait(B_XQ, 0);
            if (ok) {
                issue_a(0);
                issue_y(0);
            }
            for (int c = 0; c < nblk && ok; ++c) {
                const int s = c & 1;
                // (b): S [X; Q~]^T in one N = 128 pass -> [SX | O] of slot s
                if (!(ok = wait(B_QSC, c & 1) && wait(B_SRDY, c & 1) &&
                           (c < 2 || wait(B_OFREE + s, ((c >> 1) + 1) & 1))))
                    break;
                tc::fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc::mma_bf16(tbase + cSXO + 128 * s, dS + kmaj(ks), dX[s] + kmaj(ks), kIdN128, ks > 0);
                tc::mma_commit(&bars[B_BDONE]);
                // (a) of the next block
                if (c + 1 < nblk) {
                    if (!(ok = wait(B_XQ, (c + 1) & 1) && wait(B_GPFREE, c & 1))) break;
                    tc::fence_after_sync();
                    issue_a(c + 1);
                }
                // (d): U^T = R^T T'^T
                if (REG) {
                    if (!(ok = wait(B_RT, c & 1) && wait(B_TRDY + s, (c >> 1) & 1))) break;
                    tc::fence_after_sync();
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        tc::mma_bf16(tbase + cUT, dRT + (uint64_t)(ks * 2), dT[s] + (uint64_t)(ks * 2), kIdN64, ks > 0);
                    tc::mma_commit(&bars[B_DDONE]);
                    tc::mma_commit(&bars[B_TFREE + s]);
                }
                // (e) O += U^T P~^T and (f) dS = U^T X~
                if (!(ok = wait(B_URDY, c & 1) && wait(B_PRDY + s, (c >> 1) & 1))) break;
                tc::fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tbase + cSXO + 128 * s + 64, dRT + (uint64_t)(ks * 2), dP[s] + (uint64_t)(ks * 2),
                                 kIdN64, 1);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tbase + cDS, dRT + (uint64_t)(ks * 2), dXmn[s] + (uint64_t)(ks * 128), kIdN128Bmn,
                                 ks > 0);
                tc::mma_commit(&bars[B_EFDONE]);
                tc::mma_commit(&bars[B_PFREE + s]);
                tc::mma_commit(&bars[B_SFREE + s]);
                // (y) of the next block (its tiles landed before xq_ready of that block)
                if (c + 1 < nblk) issue_y(c + 1);
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
            sScal[3 * 256 + 64 * u + ht] = exp2f(sc[192 + (ht | 15)] - la);
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
            if (!(ok = role_wait(&bars[B_ADONE], c & 1, leader, 1, 64))) break;
            // P of query row i = ht from TMEM lanes 64..127 (this pair of warps' quarters), released at once
            tc::fence_after_sync();
            float v[64];
            {
                const uint32_t tl = tbase + ((uint32_t)(64 + 32 * (warp - 2)) << 16);
                float h0[32], h1[32];
                tc::tmem_ld32(tl + cGP, h0);
                tc::tmem_ld32(tl + cGP + 32, h1);
#pragma unroll
                for (int j = 0; j < 32; ++j) { v[j] = h0[j]; v[32 + j] = h1[j]; }
            }
            tc::fence_before_sync();
            // Q~ = diag(2^g) Q once (a) no longer needs Q
            scale_row(stg, 64 + ht, sc[64 + ht]);
            tc::fence_proxy_async();
            named_bar(1, 64);
            if (leader) {
                mbar_arrive(&bars[B_GPFREE]);
                mbar_arrive(&bars[B_QSC]);
            }
            // next block's prep overlaps this block's chain (and unblocks (a) of the next block)
            if (c + 1 < nblk && !(ok = prep(c + 1))) break;
            // P~ = Gamma o P into P~ slot s, once (e) of block c-2 has released it
            if (c >= 2 && !(ok = role_wait(&bars[B_PFREE + s], ((c >> 1) + 1) & 1, leader, 1, 64))) break;
            {
                const float *g2 = sc + 192, *cf = sScal + 3 * 256 + 64 * (c % 3);
                const int i = ht, rb = i >> 4;
                const float gri = g2[i];
                float fac[4], gd[16];
#pragma unroll
                for (int jb = 0; jb < 4; ++jb) {
                    const float f = exp2f(fminf(gri - g2[16 * jb + 15], 0.f));
                    fac[jb] = jb < rb ? f : 0.f;
                }
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int j = 16 * rb + k;
                    const float f = exp2f(fminf(gri - g2[j], 0.f));
                    gd[k] = j <= i ? f : 0.f;
                }
                uint8_t *sP = sm + oP + s * 8192;
#pragma unroll
                for (int jb = 0; jb < 4; ++jb) {
                    const bool below = jb < rb, diag = jb == rb;
                    float pv[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const int j = 16 * jb + k;
                        const float gm = below ? fac[jb] * cf[j] : (diag ? gd[k] : 0.f);
                        pv[k] = gm * v[j];
                    }
                    st_chunk8(sP, tc::sw128_chunk(i, 2 * jb), pv);
                    st_chunk8(sP, tc::sw128_chunk(i, 2 * jb + 1), pv + 8);
                }
                tc::fence_proxy_async();
                named_bar(1, 64);
                if (leader) mbar_arrive(&bars[B_PRDY + s]);
            }
        }
    } else if (warp < 8) {
        // ================================================================ local (128 threads)
        const int lt = tid - 128, lw = warp - 4;
        const int r = 32 * lw + lane;      // TMEM lane: G row for lw < 2 (P rows belong to the helpers)
        const bool leader = lt == 0;
        const uint32_t tl = tbase + ((uint32_t)(32 * lw) << 16);
        for (int c = 0; c < nblk; ++c) {
            const int s = c & 1;
            if (!role_wait(&bars[B_ADONE], c & 1, leader, 2, 128)) break;
            if (!role_wait(&bars[B_SCAL + c % 3], (c / 3) & 1, leader, 2, 128)) break;
            tc::fence_after_sync();
            const float *sc = sScal + (c % 3) * 256;
            if (lw < 2) {                                   // G rows r = 0..63 -> L (regression family)
                float v[64];
                {
                    float h0[32], h1[32];
                    tc::tmem_ld32(tl + cGP, h0);
                    tc::tmem_ld32(tl + cGP + 32, h1);
#pragma unroll
                    for (int j = 0; j < 32; ++j) { v[j] = h0[j]; v[32 + j] = h1[j]; }
                }
                tc::fence_before_sync();
                if (REG) {
                    // Decay factors 2^(g_r - g_j), j < r: below the 16x16 diagonal blocks they factor
                    // through the last index of column block jb, 2^(g_r - g_{16jb+15}) * cf[j] with
                    // cf[j] = 2^(g_{16jb+15} - g_j) (a helper table), both in (0, 1]; inside the
                    // diagonal block they are formed directly. Selects only, no divergent branches.
                    const float *g2 = sc + 192, *cf = sScal + 3 * 256 + 64 * (c % 3);
                    const int rb = r >> 4;
                    const float gri = g2[r], be = sc[r];
                    float fac[4], gd[16];
#pragma unroll
                    for (int jb = 0; jb < 4; ++jb) {
                        const float f = exp2f(fminf(gri - g2[16 * jb + 15], 0.f));
                        fac[jb] = jb < rb ? be * f : 0.f;
                    }
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const int j = 16 * rb + k;
                        const float f = exp2f(fminf(gri - g2[j], 0.f));
                        gd[k] = j < r ? be * f : 0.f;
                    }
                    float *Lr = sL + r * LDF;
#pragma unroll
                    for (int j0 = 0; j0 < 64; j0 += 4) {
                        float w4[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int j = j0 + k, jb = j >> 4;
                            const float gm = jb < rb ? fac[jb] * cf[j] : (jb == rb ? gd[j & 15] : 0.f);
                            w4[k] = gm * v[j];
                        }
                        *reinterpret_cast<float4 *>(Lr + j0) = make_float4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
            named_bar(2, 128);
            if (leader) mbar_arrive(&bars[B_GPFREE]);
            if (*abort_flag) break;
            if (REG) {
                solve_local(sL, sTf, lt, lw, lane);
                if (c >= 2 && !role_wait(&bars[B_TFREE + s], ((c >> 1) + 1) & 1, leader, 2, 128)) break;
                uint8_t *sT = sm + oT + s * 8192;
                const int rr = lt >> 1, ch0 = 4 * (lt & 1);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const float4 x0 = *reinterpret_cast<const float4 *>(sTf + rr * LDF + 8 * (ch0 + cc));
                    const float4 x1 = *reinterpret_cast<const float4 *>(sTf + rr * LDF + 8 * (ch0 + cc) + 4);
                    const float *bcol = sScal + (c % 3) * 256 + 8 * (ch0 + cc);  // beta of columns
                    const float t8[8] = {x0.x * bcol[0], x0.y * bcol[1], x0.z * bcol[2], x0.w * bcol[3],
                                         x1.x * bcol[4], x1.y * bcol[5], x1.z * bcol[6], x1.w * bcol[7]};
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
            // R^T = Y^T - SX diag(2^g) (regression) or U^T = Y^T diag(beta) (inner product),
            // 16 columns at a time, both operands from TMEM
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float y[16], v[16], rv[16];
                const int e0 = 32 * hf + 16 * hh;
                tc::tmem_ld16(tl + cY + e0, y);
                if (REG) tc::tmem_ld16(tl + cSXO + 128 * s + e0, v);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    rv[j] = REG ? y[j] - sc[64 + e0 + j] * v[j] : sc[e0 + j] * y[j];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
                    st_chunk8(sRT, tc::sw128_chunk(row, 4 * hf + 2 * hh + cc), rv + 8 * cc);
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            named_bar(3, 256);
            if (REG && leader) mbar_arrive(&bars[B_RT]);
            // X~ = diag(2^(g_last - g)) X in place (X is no longer needed unscaled once (b) is done),
            // so that (f) forms sum_e 2^(g_last - g_e) u_e x_e^T directly; done while (d) runs.
            {
                const int xr = ct >> 2, part = ct & 3;
                uint8_t *xt = sm + oStage + s * kStage + (part >> 1) * 16384;
                const float f = sc[128 + xr];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint4 *pp = reinterpret_cast<uint4 *>(xt + tc::sw128_chunk(xr, 4 * (part & 1) + k));
                    uint4 u = *pp;
                    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        const float2 x2 = __bfloat1622float2(h[q2]);
                        h[q2] = __floats2bfloat162_rn(x2.x * f, x2.y * f);
                    }
                    *pp = u;
                }
            }
            if (!REG) {
                tc::fence_proxy_async();
                named_bar(3, 256);
                if (leader) mbar_arrive(&bars[B_URDY]);
            }
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
                tc::tmem_ld32(tl + cSXO + 128 * s + 64 + 32 * hf, v);
                // lane pairs (2k, 2k+1) hold neighbouring value rows: the even lane stores the pair for
                // even tokens, the odd lane for odd tokens, as 4-byte bf16x2 stores
                const bool odd = lane & 1;
                __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(p.o) + ((size_t)bh * T + t0) * D + (row & ~1);
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float mine = odd ? v[j + 1] : v[j];
                    const float give = odd ? v[j] : v[j + 1];
                    const float other = __shfl_xor_sync(0xffffffffu, give, 1);
                    const int i = 32 * hf + j + (odd ? 1 : 0);
                    const float lo = odd ? other : mine, hi = odd ? mine : other;
                    if (i < nval)
                        *reinterpret_cast<uint32_t *>(o + (size_t)i * D) = pack_bf16x2(lo, hi);
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
