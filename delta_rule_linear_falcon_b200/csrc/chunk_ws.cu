// chunk_ws.cu -- warp-specialised chunk-parallel forward pass on tcgen05 for
// d_k = d_v = 128, bf16 I/O, blocks of 64 pseudo-value rows: 64 tokens of one pair
// each (Falcon-1, Falcon-1A), or 64 / w tokens of w pairs each (Falcon-3, Falcon-3A
// with a window of w = 2 or 4; see "Windowed rules" below). The block algebra is the
// chunk-parallel form with positive-decay
// renormalisation of "Fast Weight Attention for Continual Learning" (authors'
// abstract), written out in chunk_kernel.cuh, regrouped so that the state
// recurrence crosses only two tensor-core steps per block. With g the block-local
// cumulative log2 decay, beta the step sizes, T = (I + L)^-1 and
//   T' = T diag(beta),  T_f = diag(2^(g_last - g)) T',  A = T_f^T X,  B' = P~ T'
// (all independent of the state), one block is
//   R'^T = Y^T - (S X^T) diag(2^g)                          (regression; Y^T for inner product)
//   O^T  = (S Q^T) diag(2^g) + R'^T B'^T,   S <- 2^g_last S + R'^T A.
// For the inner-product rule T = I, so T_f and T' are diagonal and no solve runs.
// The regression rules never form R'^T: with Z~ = (S X^T) diag(2^g) the products split into
//   dS = Y^T A + (-Z~) A,   R'^T B'^T = Y^T B'^T + (-Z~) B'^T,
// where the Y^T terms read the value tile straight from shared memory (an MN-major A operand)
// and only -Z~ passes through the chain warps (fp32 -> bf16 in tensor memory).
//
// One CTA of 512 threads per (b, h); the state-independent work of later blocks
// runs on other warps while the state chain of block c runs:
//   warp 0      TMA producer: [X;Q] of each block into a 3-slot ring (the solve runs two
//               blocks ahead), V into a 2-slot ring
//   warp 1      inner-product rules: the MMA issuer of the chain ((b), E, dS below);
//               regression rules: streams V into its ring as the chain frees the slots
//   MMAs (one elected thread issues each group):
//                 (a)  [X;Q] X^T -> G (lanes 0-63), P (lanes 64-127)                (warp 0)
//                 (A)  A^T = X^T T_f   and  (B')  B' = [P~; *] T'        (state independent, warp 0)
//                 (b)  [S X^T | S Q^T] with S (bf16) read from tensor memory
//                 Y^T A, then (f') dS += -Z~ A;  Y^T B'^T, then (e') += -Z~ B'^T
//                 with -Z~ (bf16) from tensor memory          (regression rules: chain warp 8)
//               The chain warps issue their own groups right after the named barrier that ends
//               their tensor-memory writes, so only MMA completions cross an mbarrier.
//   warps 2-3   helpers: x_1 patch, cumulative log2 decay and its tables; P~ = Gamma o P
//               from TMEM lanes 64-127; T_f and T' in bf16 from the solved T
//   warps 4-7   local: step sizes from the key norms on the diagonal of G,
//               L = diag(beta)(Gamma o G) (fp32) from TMEM lanes 0-63,
//               T = (I + L)^-1 (fp32, tensor-core tf32 block products)
//   warps 8-15  chain: A^T, B' from TMEM to shared memory; -Z~ (bf16 into TMEM); the fp32
//               state S <- 2^g_last S + dS (in registers) and its bf16 copy in TMEM;
//               O = 2^g o (Q S^T) + B' R' out
// Every decay factor is 2^(g_i - g_j) with i >= j (never a quotient of
// cumulative products). Every wait is bounded; a timeout is recorded in the
// device error word and all roles unwind.
//
// Windowed rules (W = w pairs per step, TB = 64 / W tokens per block). Row r of a block
// holds pair j = t0 + s - m of token s = r % TB, m = r / TB (m-major order), so X and Y
// arrive as W boxes of TB consecutive key / value rows (key rows t0 - m - 1, value rows
// t0 - m; rows before the sequence read as zero, and zero rows are no-ops). A row takes the
// decay and the step size of its token: beta_s = eta_s / (sum_m ||x_(m,s)||^2 + eps), the sum
// over the W diagonal entries of G of that token. L couples a row only to rows of strictly
// earlier tokens (all residuals of one step are taken at the same decayed state), so it is
// strictly lower triangular in token-major order u = s * W + m: the local warps permute G
// into that order for the solve and permute T back to m-major order for the MMAs. P~ masks
// by token (a query reads the pairs of its own and earlier tokens); only the TB query rows
// are loaded and only TB outputs are written per block.
//
// Two-pass path (regression rules, given a workspace of 16 KB per block and head). The solve
// does not depend on the state, so chunk_local_kernel runs it for every block of every head
// at once and writes T_f and T' (bf16, in the order the tensor cores read them) to the
// workspace. The chain kernel then runs with PRE set: the feed warp brings each block's tiles
// into a two-slot ring with one bulk copy, the helpers only prepare the decays and P~, and the
// local warps, with no solve left, store the outputs of each block instead of the chain.
#include <cuda.h>

#include "chunk_mma.cuh"
#include "common.cuh"
#include "launch.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace falcon {

namespace {

constexpr int kThreads = 512;
constexpr int kBlk = 64;
constexpr long long kDrainBudget = kDefaultWaitBudget;  // waits for own loads / MMAs in flight at exit
constexpr int LDF = 68;                       // fp32 solve buffers: 16-byte rows, conflict-free A fragments
constexpr int kChainWarps = 8;

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t kXQ = 32768;                    // [X;Q]: 2 atoms (d 0-63, 64-127) x 128 rows (X 0-63, Q 64-127)
constexpr uint32_t kVst = 16384;                   // V: 2 atoms (v 0-63, 64-127) x 64 rows
constexpr uint32_t oXQ = 0;                        // 3 slots
constexpr uint32_t oV = oXQ + 3 * kXQ;             // 2 slots
constexpr uint32_t oTF = oV + 2 * kVst;            // T_f bf16, 64 x 64 row-major (MN-major B of (A))
constexpr uint32_t oTP = oTF + 8192;               // T' bf16 (MN-major B of (B'))
constexpr uint32_t oPB = oTP + 8192;               // rows 0-63 P~ (A of (B')), rows 64-127 B' (B of (e'))
constexpr uint32_t oA = oPB + 16384;               // A^T bf16, 128 rows (d) x 64 (i) (B of (f'))
constexpr uint32_t oL = oA + 16384;                // L / W fp32 64 x LDF
constexpr uint32_t oTf = oL + 64 * LDF * 4;        // T fp32 64 x LDF
constexpr uint32_t oScal = oTf + 64 * LDF * 4;     // 4 slots x {beta, 2^g, 2^(g_last-g), g}[64], 4 x cf[64], g_last[4], misc, norms[64]
constexpr uint32_t oBar = oScal + 4096 + 1024 + 512;
constexpr uint32_t kSmem = oBar + 512 + 1024;
static_assert(kSmem <= 232448, "shared memory");

// TMEM columns
// GP | slot 0 | slot 1 | A^T, B' | S (bf16) then -Z~ (bf16)
// Slot c & 1 holds [S X^T | S Q^T] of block c from (b); once the chain has read S X^T, (e') puts
// R'^T B'^T in its place. Regression rules: dS of block c takes the AB columns once the chain has
// copied A^T and B' of the block out of them, and frees them for (A), (B') of the next block when
// the state update has read it, so the outputs of block c-1 can be read out of the other slot while
// (b) and (A), (B') run. Inner-product rules: dS of block c takes all of the other slot, free
// between the chain's read of the outputs of block c-1 and (b) of block c+1.
constexpr uint32_t cGP = 0, cSXO = 64 /* + 128 * slot */, cAB = 320, cSR = 448, kTmemCols = 512;

constexpr uint32_t kIdN64 = tc::idesc_bf16(128, 64, 0, 0);
constexpr uint32_t kIdN128 = tc::idesc_bf16(128, 128, 0, 0);
constexpr uint32_t kIdAT = tc::idesc_bf16(128, 64, 1, 1);   // X^T (MN-major A) x T_f (MN-major B)
constexpr uint32_t kIdBP = tc::idesc_bf16(128, 64, 0, 1);   // P~ (K-major A) x T' (MN-major B)
constexpr uint32_t kIdVP = tc::idesc_bf16(128, 64, 1, 0);   // (diag(beta) Y)^T (MN-major A) x P~ (K-major B)
constexpr uint32_t kIdVX = tc::idesc_bf16(128, 128, 1, 1);  // (diag(w) Y)^T (MN-major A) x X (MN-major B)
constexpr uint32_t kIdVA = tc::idesc_bf16(128, 128, 1, 0);  // Y^T (MN-major A) x A (K-major B, the A^T tile)

// barrier indices (arrival count 1 unless noted)
enum {
    B_FULLXQ = 0,      // [3] TMA [X;Q] landed -> helpers
    B_XQFREE = 3,      // [3] (a), (A) done (feed warp) and (b) done (chain MMA warp): 2 arrivals -> producer
    B_FULLV = 6,       // [2] TMA V landed -> MMAs (regression), local warps (inner product)
    B_VFREE = 8,       // [2] the MMAs that read V are done -> producer
    B_XQRDY = 10,      // [3] helpers prepared the block -> MMA (a)
    B_ADONE = 13,      // (a) done -> helpers, local
    B_GPFREE = 14,     // G read (local warps 4, 5) and P read (helpers): 3 arrivals -> MMA (a) of the next block
    B_SCAL = 15,       // [4] decay scalars of slot c % 4 ready -> local, chain
    B_SCALFREE = 19,   // [4] chain done with scalar slot, outputs stored (8 warps) -> helpers
    B_EDONE = 23,      // (e') done (it still reads -Z~ from TMEM) -> chain (before S overwrites it), outputs
    B_SOLVED = 24,     // T of the block solved (fp32, local) -> helpers (T tiles)
    B_TREAD = 25,      // helpers read T of the block -> local (the next solve may overwrite it)
    B_PRDY = 26,       // P~ ready -> MMA (B')
    B_TRDY = 27,       // T_f, T' (and the step sizes) ready -> MMA (A), (B')
    B_ABDONE = 28,     // (A), (B') done -> chain, local (T tiles free), helpers (P~ tile free)
    B_EARDY = 29,      // the AB columns are free again (8 warps): regression rules after dS is read, inner
                       // product after the outputs are read -> (A), (B') / dS of the next block
    B_BDONE = 30,      // (b) done -> chain
    B_RT = 31,         // -Z~ in TMEM (8 warps) -> MMA (e'), (f')
    B_EFDONE = 32,     // (f') done: dS in TMEM -> chain
    B_FINAL0 = 33,     // drain of the feed warp's MMAs at exit
    B_SRDY = 34,       // S bf16 in TMEM, dS read, O of the previous block read (8 warps) -> MMA (b)
    B_FINAL = 35,      // drain of the chain MMA warp's MMAs at exit
    B_SQDONE = 36,     // S Q^T done (it reads the bf16 state that -Z~ replaces) -> chain
    B_FULLT = 37,      // [2] two-pass path: the block's T_f, T' tiles landed -> MMA (A), (B')
    B_TFREE = 39,      // [2] two-pass path: (A), (B') that read the tile slot are done -> tile loads
    B_OUTFREE = 41,    // [2] two-pass path: outputs of the slot's block read (4 output warps) -> (b)
    B_EDONES = 43,     // [2] two-pass path: (e') of the slot's block done -> chain, output warps (one
                       // barrier per slot, so that a slow output warp never sees a later phase)
    B_COUNT = 45
};

__device__ __forceinline__ void named_bar(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Named barrier that also ORs a predicate over its participants: every thread gets the same answer.
__device__ __forceinline__ bool named_bar_or(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %3, 0;\n\tbar.red.or.pred p, %1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(r)
        : "r"(id), "r"(n), "r"((uint32_t)pred)
        : "memory");
    return r != 0;
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

// v[OFF + lane] of a register array, by a five-level select tree on the lane's bits
template <int OFF>
__device__ __forceinline__ float pick_lane(const float (&v)[64], int lane) {
    float t16[16], t8[8], t4[4], t2[2];
#pragma unroll
    for (int k = 0; k < 16; ++k) t16[k] = (lane & 16) ? v[OFF + 16 + k] : v[OFF + k];
#pragma unroll
    for (int k = 0; k < 8; ++k) t8[k] = (lane & 8) ? t16[8 + k] : t16[k];
#pragma unroll
    for (int k = 0; k < 4; ++k) t4[k] = (lane & 4) ? t8[4 + k] : t8[k];
#pragma unroll
    for (int k = 0; k < 2; ++k) t2[k] = (lane & 2) ? t4[2 + k] : t4[k];
    return (lane & 1) ? t2[1] : t2[0];
}

// O^T of block c (TMEM slot c & 1: S Q^T scaled by 2^g per token, plus R'^T B'^T) to global memory
// for value row `row` (TMEM lane base tl) and the query tokens 32 hf .. 32 hf + 31 of the block's TB:
// for each token a warp stores the bf16 outputs of its 32 consecutive value rows, 64 contiguous bytes
// per store instruction. dg2 holds 2^g of the block's tokens.
template <int TB>
__device__ __forceinline__ void store_out_rows(void *out, int bh, int T, int c, int row, uint32_t tl, int hf,
                                               const float *dg2) {
    constexpr int D = 128;
    const int t0 = c * TB, nval = min(TB, T - t0);
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(out) + ((size_t)bh * T + t0) * D + row;
#pragma unroll 1
    for (int h = 0; h < 4; ++h) {          // 8 tokens at a time
        const int i0 = 32 * hf + 8 * h;
        if (i0 >= TB) break;               // a block has TB query tokens
        // the scales first, so that their shared-memory latency overlaps the TMEM loads
        const float4 da = *reinterpret_cast<const float4 *>(dg2 + i0);
        const float4 db = *reinterpret_cast<const float4 *>(dg2 + i0 + 4);
        const float dg[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
        float v[8], w[8];
        tc::tmem_ld8x2(tl + cSXO + 128 * (c & 1) + 64 + i0, tl + cSXO + 128 * (c & 1) + i0, v, w);
        __nv_bfloat16 *oi = o + (size_t)i0 * D;
        if (i0 + 8 <= nval) {              // whole group (every group but the sequence's last)
#pragma unroll
            for (int j = 0; j < 8; ++j) oi[j * D] = __float2bfloat16_rn(dg[j] * v[j] + w[j]);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (i0 + j < nval) oi[j * D] = __float2bfloat16_rn(dg[j] * v[j] + w[j]);
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
//   diagonal blocks T_ii by forward substitution (one thread per column, one warp per block);
//   W_im = -T_ii L_im, stored over L_im by the warp that formed it;
//   T_ij = sum_{m=j}^{i-1} W_im T_mj, with the terms spread so that the longest chain of
//   dependent 16 x 16 products after W is three:
//     round A: T_10, T_21, T_32 and W_20 T_00;  round B: T_20, T_31 and W_30 T_00 + W_31 T_10;
//     round C: T_30.
// Entries above the block diagonal of Tf are zero on entry and stay zero.
// PACKED (a throughput-bound caller): the diagonal blocks go to two warps, 16 lanes per block.
template <bool PACKED = false>
__device__ __forceinline__ void solve_local(float *sL, float *sTf, int lt, int lw, int lane) {
    if (PACKED ? lw < 2 : lane < 16) {  // column j of the inverse of diagonal block b, left-looking, rows of L as float4
        const int b = PACKED ? 2 * lw + (lane >> 4) : lw, j = lane & 15;
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
    auto Lb = [&](int i, int m) { return sL + (16 * i) * LDF + 16 * m; };    // L_im, then W_im
    auto Tb = [&](int i, int m) { return sTf + (16 * i) * LDF + 16 * m; };
    auto zero = [](float (&acc)[2][4]) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 4; ++h) acc[nt][h] = 0.f;
    };
    // W blocks (i, m): (1,0) (2,0) (2,1) (3,0) (3,1) (3,2); warp lw takes blocks lw and lw + 4
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int blk = lw + 4 * k;
        if (blk < 6) {
            const int i = blk < 1 ? 1 : (blk < 3 ? 2 : 3);
            const int m = blk < 1 ? 0 : (blk < 3 ? blk - 1 : blk - 3);
            float acc[2][4];
            zero(acc);
            mma16_acc(acc, Tb(i, i), Lb(i, m), lane);
            __syncwarp();
            store16(Lb(i, m), acc, lane, -1.f);
        }
    }
    named_bar(2, 128);
    float part[2][4];
    zero(part);
    if (lw < 3) {          // round A: T_{lw+1, lw} = W_{lw+1, lw} T_{lw, lw}
        float acc[2][4];
        zero(acc);
        mma16_acc(acc, Lb(lw + 1, lw), Tb(lw, lw), lane);
        store16(Tb(lw + 1, lw), acc, lane, 1.f);
    } else {
        mma16_acc(part, Lb(2, 0), Tb(0, 0), lane);   // W_20 T_00, finished in round B
    }
    named_bar(2, 128);
    if (lw == 0) {         // round B
        mma16_acc(part, Lb(3, 0), Tb(0, 0), lane);   // W_30 T_00 + W_31 T_10, finished in round C
        mma16_acc(part, Lb(3, 1), Tb(1, 0), lane);
    } else if (lw == 1) {
        float acc[2][4];
        zero(acc);
        mma16_acc(acc, Lb(3, 1), Tb(1, 1), lane);
        mma16_acc(acc, Lb(3, 2), Tb(2, 1), lane);
        store16(Tb(3, 1), acc, lane, 1.f);
    } else if (lw == 3) {
        mma16_acc(part, Lb(2, 1), Tb(1, 0), lane);
        store16(Tb(2, 0), part, lane, 1.f);
    }
    named_bar(2, 128);
    if (lw == 0) {         // round C
        mma16_acc(part, Lb(3, 2), Tb(2, 0), lane);
        store16(Tb(3, 0), part, lane, 1.f);
    }
    named_bar(2, 128);
}

// ---- two-pass path of the regression rules, pass 1 (chunk_local_kernel)
constexpr int kLocThreads = 128;
constexpr int kLocCtasPerSm = 4;
constexpr uint32_t kTileBytes = 16384;              // T_f then T', bf16 64 x 64 each, 128-byte swizzled
constexpr uint32_t oLX = 0;                         // keys: 2 swizzled atoms of 64 rows
constexpr uint32_t oLT = 16384;                     // T fp32 64 x LDF
constexpr uint32_t oLL = oLT + 64 * LDF * 4;        // L / W fp32 64 x LDF, then the output tiles
constexpr uint32_t oLS = oLL + 64 * LDF * 4;        // beta[64], g[64], 2^(g_last - g)[64], cf[64], carry[36], barriers, TMEM slot
constexpr uint32_t kLocSmem = oLS + 4 * 256 + 36 * 4 + 32 + 1024;   // + alignment of the base to 1024 bytes

// One bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) into shared memory,
// completing on the mbarrier's transaction count.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(tc::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(tc::smem_u32(src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_addr(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

}  // namespace

// Pass 1 of the two-pass path of the regression rules. The chunk-local step depends only on a
// block's keys and gates, so it runs for every block at once before any state chain starts.
// Persistent CTAs of 128 threads walk the (head, block) items; per item they form G = X X^T on the
// tensor cores (tcgen05, fp32 accumulation in 64 TMEM columns), the step sizes from its diagonal and
// L = diag(beta)(Gamma o G) from the rows in registers (warps 0-1, which own TMEM lanes 0-63),
// T = (I + L)^-1 (solve_local), and write T_f = diag(2^(g_last - g)) T diag(beta) and
// T' = T diag(beta) as two bf16 tiles in the 128-byte swizzled order the tensor cores read, 16 KB
// per item at tiles + (head * nblk + block) * 16 KB. The arithmetic is the one the single-kernel
// path does on its local and helper warps, including the windowed layout (W pairs per step: rows in
// m-major order, L and T in token-major order, the tiles permuted back). The keys of the next item
// are loaded by TMA (128-byte
// swizzled; rows before or past the sequence read as zero) as soon as G of the current item is
// done, and the tiles leave by a bulk copy that is only waited for before their buffer is written
// again, so the loads and stores of one item overlap the arithmetic of the next.
template <int W>
__global__ void __launch_bounds__(kLocThreads, kLocCtasPerSm)
chunk_local_kernel(const __grid_constant__ CUtensorMap tmK, const ChunkParams p, const int nblk) {
    constexpr int TB = kBlk / W;   // tokens per block
    extern __shared__ __align__(1024) uint8_t lsm_raw[];
    uint8_t *lsm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(lsm_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sX = lsm + oLX;
    float *sT = reinterpret_cast<float *>(lsm + oLT);
    float *sL = reinterpret_cast<float *>(lsm + oLL);
    uint8_t *sOut = lsm + oLL;
    float *sBeta = reinterpret_cast<float *>(lsm + oLS);
    float *sG = sBeta + 64, *sFr = sBeta + 128, *sCF = sBeta + 192, *sCarry = sBeta + 256;
    float *sNrm = sCF;   // windowed rules: squared key norms of the rows (the cf table is W = 1 only)
    uint64_t *bar_k = reinterpret_cast<uint64_t *>(sBeta + 292), *bar_m = bar_k + 1;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_k + 2);

    const int lt = threadIdx.x, lw = lt >> 5, lane = lt & 31;
    const int T = p.T;
    const int kshift = p.same_step ? 0 : 1;
    constexpr int D = 128;
    const int items = p.B * p.H * nblk;   // below 2^31 (the host checks the workspace size)
    const volatile int no_abort = 0;
    // K-major [X] descriptor (128-byte swizzle, 8-row groups 1024 bytes apart); a K step of 16 moves
    // 32 bytes inside an atom of 64 columns, the second atom is 8 KB further. With M = 128 the A
    // operand's rows 64-127 run past the keys into the T buffer: their products land in TMEM lanes
    // 64-127, which nothing reads.
    const uint64_t dX = tc::sdesc(tc::smem_u32(sX), 16, 1024);
    auto kstep = [](int ks) -> uint64_t { return (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) >> 4); };
    constexpr uint32_t kIdG = tc::idesc_bf16(128, 64, 0, 0);

    // thread 0: TMA of item it's keys; rows m TB .. hold the pairs t0 - m .., i.e. key rows
    // t0 - m - kshift (W boxes of TB rows per 64-column atom)
    auto load_keys = [&](int it) {
        const int bh = it / nblk, c = it - bh * nblk;
        tc::mbar_arrive_expect_tx(bar_k, 16384);
#pragma unroll
        for (int m = 0; m < W; ++m) {
            tc::tma_load_3d(sX + m * TB * 128, &tmK, 0, c * TB - m - kshift, bh, bar_k);
            tc::tma_load_3d(sX + 8192 + m * TB * 128, &tmK, 64, c * TB - m - kshift, bh, bar_k);
        }
    };
    // gates of an item for the threads of rows 0..63: those of the row's token r % TB (alpha, eta;
    // 1 and 0 past the sequence)
    auto load_gates = [&](int it, float &a, float &e) {
        a = 1.f;
        e = 0.f;
        if (lt < 64 && it < items) {
            const int bh = it / nblk, t = (it - bh * nblk) * TB + lt % TB;
            if (t < T) {
                a = p.alpha[(size_t)bh * T + t];
                e = p.eta[(size_t)bh * T + t];
            }
        }
    };

    int it = blockIdx.x;
    if (lt == 0) {
        tc::mbar_init(bar_k, 1);
        tc::mbar_init(bar_m, 1);
        tc::mbar_fence_init();
        if (it < items) load_keys(it);
    }
    if (lw == 0) {
        tc::tmem_alloc(tslot, 64);
        tc::tmem_relinquish();
    }
    float ga, ge;
    load_gates(it, ga, ge);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tslot;
    if constexpr (W > 1) {
        // T starts at zero once: in token-major order the solve writes only the blocks on and below
        // the diagonal, and the permuted tiles read every entry
        for (int idx = lt; idx < 64 * LDF / 4; idx += kLocThreads)
            reinterpret_cast<float4 *>(sT)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (uint32_t k = 0; it < items; ++k, it += gridDim.x) {
        const int bh = it / nblk, c = it - bh * nblk;
        const int t0 = c * TB, nval = min(TB, T - t0);
        const int nx = it + gridDim.x;
        // cumulative log2 decay of the block's tokens (tokens past the sequence add nothing); for
        // W > 1 the TB <= 32 tokens are scanned by warp 0
        float la = 0.f;
        if (W == 1 ? lt < 64 : lt < 32) {
            la = (lt < TB && lt < nval) ? log2f(ga) : 0.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, la, off);
                if (lane >= off) la += y;
            }
            if (lt == 31) sCarry[0] = la;
        }
        const float ge_c = ge;
        load_gates(nx, ga, ge);   // the next item's gates, in flight during this one
        const bool landed = tc::mbar_wait(bar_k, k & 1, &no_abort, kDefaultWaitBudget);
        if (landed && c == 0 && kshift == 1 && p.k_prev && lt < 16 * W) {
            // pair 0 = (k_prev, v_0) sits in row m TB + m for every m < W: its key is the cached key
            const int m = lt >> 4, ch = lt & 15;
            const uint4 v = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(p.k_prev) +
                                                              (size_t)bh * D + ch * 8);
            *reinterpret_cast<uint4 *>(sX + (ch >> 3) * 8192 + tc::sw128_chunk(m * TB + m, ch & 7)) = v;
            tc::fence_proxy_async();   // the tensor cores read it
        }
        if (lt == 0) tc::tma_store_wait_read0();   // the previous item's tiles have left the L buffer
        tc::fence_before_sync();
        if (__syncthreads_or(!landed)) {
            if (lt == 0) set_error(p.err, kDevErrTimeout);
            break;
        }
        tc::fence_after_sync();
        if constexpr (W == 1) {
            if (lt >= 32 && lt < 64) la += sCarry[0];
            if (lt < 64) sG[lt] = la;
        } else {
            if (lt < TB) sCarry[1 + lt] = la;   // token decays g_s in sCarry[1 + s]
        }
        if (lw == 0) {   // G = X X^T -> TMEM columns 0-63, lanes 0-63
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) tc::mma_bf16_elect(tbase, dX + kstep(ks), dX + kstep(ks), kIdG, ks > 0);
            tc::mma_commit_elect(bar_m);
        }
        __syncthreads();
        if (lt < 64) {   // decay tables
            if constexpr (W == 1) {
                const float gl = sG[nval - 1];
                sFr[lt] = exp2f(gl - la);
                sCF[lt] = exp2f(sG[lt | 15] - la);
            } else {   // every row takes its token's decay
                const float g = sCarry[1 + lt % TB], gl = sCarry[nval];
                sG[lt] = g;
                sFr[lt] = exp2f(gl - g);
            }
        }
        const bool mok = tc::mbar_wait(bar_m, k & 1, &no_abort, kDefaultWaitBudget);
        if (lt == 0 && mok && nx < items) load_keys(nx);   // G has read the keys: the next item's may land
        if (__syncthreads_or(!mok)) {
            if (lt == 0) set_error(p.err, kDevErrTimeout);
            break;
        }
        tc::fence_after_sync();
        if (lw < 2) {   // G row r = lt from TMEM: step size, then L = diag(beta)(Gamma o G) row r
            const int r = lt, rb = r >> 4;
            float v[64];
            {
                float h0[32], h1[32];
                const uint32_t tl = tbase + ((uint32_t)(32 * lw) << 16);
                tc::tmem_ld32(tl, h0);
                tc::tmem_ld32(tl + 32, h1);
#pragma unroll
                for (int j = 0; j < 32; ++j) { v[j] = h0[j]; v[32 + j] = h1[j]; }
            }
            // ||x_r||^2 is the diagonal entry G[r][r] = v[32 lw + lane] (a warp-uniform branch on lw
            // keeps v in registers)
            float nrm = lw == 0 ? pick_lane<0>(v, lane) : pick_lane<32>(v, lane);
            if constexpr (W > 1) {   // the token's window: rows m TB + r % TB, m < W
                sNrm[r] = nrm;
                named_bar(3, 64);
                nrm = 0.f;
#pragma unroll
                for (int m = 0; m < W; ++m) nrm += sNrm[m * TB + r % TB];
            }
            const float be = r % TB < nval ? step_size(ge_c, nrm, p.eps) : 0.f;
            sBeta[r] = be;
          if constexpr (W > 1) {
            // row u = s W + m of L in token-major order (s = r % TB, m = r / TB) couples to the rows of
            // earlier tokens s' < s only: L[u][s' W + m'] = beta 2^(g_s - g_s') G[r][m' TB + s']
            const int rs = r % TB;
            const float gri = sG[r];
            float gd[TB];
#pragma unroll
            for (int sp = 0; sp < TB; ++sp) gd[sp] = sp < rs ? be * exp2f(fminf(gri - sG[sp], 0.f)) : 0.f;
            float *Lr = sL + (rs * W + r / TB) * LDF;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                float w4[4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int up = 4 * q + kk, sp = up / W, mp = up % W;
                    w4[kk] = gd[sp] * v[mp * TB + sp];
                }
                *reinterpret_cast<float4 *>(Lr + 4 * q) = make_float4(w4[0], w4[1], w4[2], w4[3]);
            }
          } else {
            // decay factors 2^(g_r - g_j), j < r: below the 16 x 16 diagonal blocks through the last
            // index of column block jb (2^(g_r - g_{16jb+15}) cf[j]), directly inside them; entries on
            // and above the diagonal are left as they come (the solve reads the strictly lower part)
            const float gri = sG[r];
            float gd[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 g4 = *reinterpret_cast<const float4 *>(sG + 16 * rb + 4 * q);
                gd[4 * q] = be * exp2f(fminf(gri - g4.x, 0.f));
                gd[4 * q + 1] = be * exp2f(fminf(gri - g4.y, 0.f));
                gd[4 * q + 2] = be * exp2f(fminf(gri - g4.z, 0.f));
                gd[4 * q + 3] = be * exp2f(fminf(gri - g4.w, 0.f));
            }
            float *Lr = sL + r * LDF;
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) {   // the solve reads no block above the row's diagonal one
                if (jb > rb) break;
                const float fac = be * exp2f(fminf(gri - sG[16 * jb + 15], 0.f));
                const bool below = jb < rb;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int j = 16 * jb + 4 * q;
                    const float4 c4 = *reinterpret_cast<const float4 *>(sCF + j);
                    const float w0 = below ? fac * c4.x : gd[4 * q];
                    const float w1 = below ? fac * c4.y : gd[4 * q + 1];
                    const float w2 = below ? fac * c4.z : gd[4 * q + 2];
                    const float w3 = below ? fac * c4.w : gd[4 * q + 3];
                    *reinterpret_cast<float4 *>(Lr + j) =
                        make_float4(w0 * v[j], w1 * v[j + 1], w2 * v[j + 2], w3 * v[j + 3]);
                }
            }
          }
        }
        tc::fence_before_sync();
        __syncthreads();
        // T = (I + L)^-1; its blocks above the diagonal are never written and never read (the tiles
        // below take only the chunks on and below the diagonal)
        solve_local<true>(sL, sT, lt, lw, lane);   // ends with a barrier of all 128 threads
        {   // thread (row rr, half h) writes columns 32 h .. 32 h + 31 of both tiles (m-major order):
            // T' = T diag(beta) and T_f = 2^(g_last - g) T'; for W = 1 the chunks above the diagonal
            // are zero, for W > 1 T is read in token-major order (row rr is token-major row
            // (rr % TB) W + rr / TB; the eight columns j0.. of a chunk share m' = j0 / TB and take
            // tokens j0 % TB + k, a stride of W)
            // for W > 1 a warp's 16 rows are taken from all W slots m (rr = m TB + s), so that their
            // token-major rows s W + m fall on different banks
            const int ix = lt >> 1, h = lt & 1;
            const int rr = W == 1 ? ix : (ix % W) * TB + ix / W;
            const float fr = sFr[rr];
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const int cc = 4 * h + k4, j0 = 8 * cc;
                float t8[8], f8[8];
                if (W > 1 || j0 <= rr) {
                    if constexpr (W == 1) {
                        const float4 x0 = *reinterpret_cast<const float4 *>(sT + rr * LDF + j0);
                        const float4 x1 = *reinterpret_cast<const float4 *>(sT + rr * LDF + j0 + 4);
                        t8[0] = x0.x; t8[1] = x0.y; t8[2] = x0.z; t8[3] = x0.w;
                        t8[4] = x1.x; t8[5] = x1.y; t8[6] = x1.z; t8[7] = x1.w;
                    } else {
                        const float *Trow = sT + ((rr % TB) * W + rr / TB) * LDF + (j0 % TB) * W + j0 / TB;
#pragma unroll
                        for (int q = 0; q < 8; ++q) t8[q] = Trow[q * W];
                    }
                    const float4 b0 = *reinterpret_cast<const float4 *>(sBeta + j0);
                    const float4 b1 = *reinterpret_cast<const float4 *>(sBeta + j0 + 4);
                    t8[0] *= b0.x; t8[1] *= b0.y; t8[2] *= b0.z; t8[3] *= b0.w;
                    t8[4] *= b1.x; t8[5] *= b1.y; t8[6] *= b1.z; t8[7] *= b1.w;
#pragma unroll
                    for (int q = 0; q < 8; ++q) f8[q] = fr * t8[q];
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) t8[q] = f8[q] = 0.f;
                }
                st_chunk8(sOut, tc::sw128_chunk(rr, cc), f8);
                st_chunk8(sOut + 8192, tc::sw128_chunk(rr, cc), t8);
            }
        }
        tc::fence_proxy_async();
        __syncthreads();
        if (lt == 0) {
            bulk_store(reinterpret_cast<uint8_t *>(p.tiles) + (size_t)it * kTileBytes, sOut, kTileBytes);
            tc::tma_store_commit();
        }
    }
    if (lt == 0) tc::tma_store_wait_read0();   // shared memory stays until the last copy has read it
    tc::fence_before_sync();
    __syncthreads();
    if (lw == 0) tc::tmem_dealloc(tbase, 64);
}

// PRE (regression rules): T_f and T' of every block were written by chunk_local_kernel; the feed
// warp brings them into a 2-slot ring with one bulk copy per block, and neither the local warps nor
// the helpers form them.
template <bool REG, int W, bool PRE>
__global__ void __launch_bounds__(kThreads, 1)
chunk_ws_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                const __grid_constant__ CUtensorMap tmV, ChunkParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sTF = sm + oTF, *sTP = sm + oTP, *sPB = sm + oPB, *sA = sm + oA;
    float *sL = reinterpret_cast<float *>(sm + oL);
    float *sTf = reinterpret_cast<float *>(sm + oTf);
    // Scalars of block c live in slot c % 4: beta[64] 2^g[64] 2^(g_last-g)[64] g[64]; the helpers
    // prepare two blocks ahead of the chain, which still reads the slot of its own block.
    float *sScal = reinterpret_cast<float *>(sm + oScal);
    float *sCF = sScal + 1024;                             // 4 x cf[64]
    float *sGL = sScal + 1280;                             // g_last per slot
    float *sMisc = sScal + 1284;                           // helper scan carry; token decays (windowed rules)
    float *sNrm = sScal + 1344;                            // squared key norms of the rows (windowed rules)
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + oBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int T = p.T;
    constexpr int TB = kBlk / W;          // tokens per block
    static_assert(W == 1 || W == 2 || W == 4, "window");
    const int nblk = (T + TB - 1) / TB;
    constexpr int D = 128;

    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) {
            const bool chain_arrivals = (i >= B_SCALFREE && i < B_SCALFREE + 4) || i == B_EARDY || i == B_RT ||
                                        i == B_SRDY;
            const bool two = i >= B_XQFREE && i < B_XQFREE + 3;
            const bool scal = i >= B_SCALFREE && i < B_SCALFREE + 4;
            const bool outw = i == B_OUTFREE || i == B_OUTFREE + 1;
            // two-pass path: the chain and the four output warps both read a scalar slot
            const uint32_t n = (PRE && scal) ? kChainWarps + 4
                               : chain_arrivals ? kChainWarps
                               : outw ? 4 : (i == B_GPFREE ? (PRE ? 1 : 3) : (two ? 2 : 1));
            tc::mbar_init(&bars[i], n);
        }
        *abort_flag = 0;
        tc::mbar_fence_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tslot, kTmemCols);
        tc::tmem_relinquish();
    }
    for (int idx = tid; idx < 64 * LDF; idx += kThreads) sTf[idx] = 0.f;
    if constexpr (W > 1) {  // query rows TB..63 of every [X;Q] slot: never loaded, kept zero
        for (int idx = tid; idx < 3 * 2 * (64 - TB) * 8; idx += kThreads) {
            const int ch = idx & 7, row = TB + (idx >> 3) % (64 - TB), at = (idx >> 3) / (64 - TB);
            *reinterpret_cast<uint4 *>(sm + oXQ + (at >> 1) * kXQ + (at & 1) * 16384 + 8192 + row * 128 + ch * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        tc::fence_proxy_async();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tslot;

    // Leader-polled bounded wait; the outcome is made uniform across the role by its named barrier.
    auto role_wait = [&](uint64_t *bar, uint32_t parity, bool leader, int bar_id, int nthr) -> bool {
        bool failed = false;
        if (leader && !tc::mbar_wait(bar, parity, abort_flag, p.wait_budget)) {
            *abort_flag = 1;
            failed = true;
        }
        return !named_bar_or(bar_id, nthr, failed);
    };
    // Lane-0-polled bounded wait, uniform across the warp.
    auto warp_wait = [&](uint64_t *bar, uint32_t parity) -> bool {
        int ok = 1;
        if (lane == 0 && !tc::mbar_wait(bar, parity, abort_flag, p.wait_budget)) {
            *abort_flag = 1;
            ok = 0;
        }
        return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };
    // Per-warp arrival on a barrier that counts the chain's warps (after this warp's TMEM traffic).
    auto warp_arrive = [&](uint64_t *bar) {
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar);
    };

    // Shared-memory descriptors (built once; a K step only moves the 14-bit start-address field,
    // address >> 4, which stays below 2^14 for every operand here, so a plain add is exact). Slot u
    // of the [X;Q] ring is kXQ bytes further: its descriptors are the slot-0 ones plus u * kXQ / 16,
    // kept arithmetic so that they stay warp-uniform.
    const uint64_t dXQ0 = tc::sdesc(tc::smem_u32(sm + oXQ), 16, 1024);      // [X;Q] K-major: (a), (b)
    auto slot_off = [](int u) -> uint64_t { return (uint64_t)(u * (kXQ >> 4)); };
    auto kmaj = [](int ks) -> uint64_t { return (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4); };
    // Whole-warp bounded wait of an issuing warp: every lane polls, the outcome is warp-uniform.
    auto wait_all = [&](int b, uint32_t parity) -> bool {
        const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars[b], parity, abort_flag, p.wait_budget));
        if (!ok) *abort_flag = 1;
        return ok;
    };

    // V of block j (regression rules: loaded by the chain MMA warp, which sees the chain free a slot)
    auto load_v = [&](int jv) {
        if (lane == 0) {
            uint8_t *dst = sm + oV + (jv & 1) * kVst;
            uint64_t *fb = &bars[B_FULLV + (jv & 1)];
            const int t0 = jv * TB;
            tc::mbar_arrive_expect_tx(fb, kVst);
#pragma unroll
            for (int m = 0; m < W; ++m) {  // value rows t0 - m ..
                tc::tma_load_3d(dst + m * TB * 128, &tmV, 0, t0 - m, bh, fb);
                tc::tma_load_3d(dst + 8192 + m * TB * 128, &tmV, 64, t0 - m, bh, fb);
            }
        }
        __syncwarp();
    };

    if (warp == 0) {
        // ================================================================ feed: TMA loads and the
        // state-independent MMAs (a), (A), (B'), issued by the whole warp (one elected lane issues).
        // Iteration j loads [X;Q] of block j and V of block j-1, then issues (a) of block j-1 and
        // (A), (B') of block j-2, each as soon as its inputs are ready. None of these waits on a later
        // iteration's work, and the chain only needs what earlier iterations issued, so the order
        // cannot deadlock; it keeps the Gram products and the solve of later blocks off the chain.
        const uint64_t dXmn0 = tc::sdesc(tc::smem_u32(sm + oXQ), 16384, 1024);  // X as an MN-major A
        const uint64_t dTF = tc::sdesc(tc::smem_u32(sTF), 8192, 1024);          // MN-major B, one N atom
        const uint64_t dTP = tc::sdesc(tc::smem_u32(sTP), 8192, 1024);
        // two-pass path: tile slot 1 in the fp32 L / T buffers, which no solve uses then
        const uint64_t dTF1 = tc::sdesc(tc::smem_u32(sm + oL), 8192, 1024);
        const uint64_t dTP1 = tc::sdesc(tc::smem_u32(sm + oL + 8192), 8192, 1024);
        const uint64_t dPB = tc::sdesc(tc::smem_u32(sPB), 16, 1024);            // [P~; B'] K-major
        const int kshift = p.same_step ? 0 : 1;   // prefix-aligned key rows of block j start at t0 - 1
        int kx = 0, kv = 0, kt = 0;
        bool ok = true;
        for (int j = 0; j <= nblk + 1 && ok; ++j) {
            // (a) first: it only needs its own slot (loaded in the previous iteration), so a slot that is
            // still busy for a later load never holds back the Gram product of the block the solve wants next
            const int ja = j - 1;   // (a) [X;Q] X^T -> G, P once the helpers prepared the block and the
            if (ja >= 0 && ja < nblk) {  // G/P columns were read for the block before
                if (!(ok = wait_all(B_XQRDY + ja % 3, (ja / 3) & 1) && (ja == 0 || wait_all(B_GPFREE, (ja - 1) & 1))))
                    break;
                tc::fence_after_sync();
                const uint64_t d = dXQ0 + slot_off(ja % 3);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) tc::mma_bf16_elect(tbase + cGP, d + kmaj(ks), d + kmaj(ks), kIdN64, ks > 0);
                tc::mma_commit_elect(&bars[B_ADONE]);
                if (!REG) tc::mma_commit_elect(&bars[B_XQFREE + ja % 3]);   // one of the slot's two arrivals
            }
            const int jt = j - 1;   // two-pass path: the tiles of block j-1, one iteration before (A), (B')
            if (PRE && jt >= 0 && jt < nblk) {
                if (jt >= 2 && !(ok = wait_all(B_TFREE + (jt & 1), ((jt >> 1) - 1) & 1))) break;
                if (lane == 0) {
                    uint64_t *fb = &bars[B_FULLT + (jt & 1)];
                    tc::mbar_arrive_expect_tx(fb, kTileBytes);
                    bulk_load(sm + ((jt & 1) ? oL : oTF),
                              reinterpret_cast<const uint8_t *>(p.tiles) + ((size_t)bh * nblk + jt) * kTileBytes,
                              kTileBytes, fb);
                }
                __syncwarp();
                kt = jt + 1;
            }
            if (j < nblk) {
                if (j == p.dbg_stall_block) break;  // test hook: this block is never loaded
                if (j >= 3 && !(ok = wait_all(B_XQFREE + j % 3, ((j / 3) - 1) & 1))) break;
                if (lane == 0) {
                    uint8_t *dst = sm + oXQ + (j % 3) * kXQ;
                    uint64_t *fb = &bars[B_FULLXQ + j % 3];
                    const int t0 = j * TB;
                    tc::mbar_arrive_expect_tx(fb, 16384 + TB * 256);
#pragma unroll
                    for (int m = 0; m < W; ++m) {  // rows m*TB.. hold the pairs t0 - m ..: key rows t0 - m - kshift
                        tc::tma_load_3d(dst + m * TB * 128, &tmK, 0, t0 - m - kshift, bh, fb);
                        tc::tma_load_3d(dst + 16384 + m * TB * 128, &tmK, 64, t0 - m - kshift, bh, fb);
                    }
                    tc::tma_load_3d(dst + 8192, &tmQ, 0, t0, bh, fb);
                    tc::tma_load_3d(dst + 16384 + 8192, &tmQ, 64, t0, bh, fb);
                }
                __syncwarp();
                kx = j + 1;
            }
            const int jv = j - 1;   // inner-product rules: V of block j-1 (the local warps scale it in place)
            if (!REG && jv >= 0 && jv < nblk) {
                if (jv >= 2 && !(ok = wait_all(B_VFREE + (jv & 1), ((jv >> 1) - 1) & 1))) break;
                load_v(jv);
                kv = jv + 1;
            }
            const int jb = j - 2;   // (A) A^T = X^T T_f and (B') B' = P~ T' into the AB columns, free once
            if (REG && jb >= 0 && jb < nblk) {  // the chain copied A^T, B' of the block before
                if (!(ok = (PRE ? wait_all(B_FULLT + (jb & 1), (jb >> 1) & 1) : wait_all(B_TRDY, jb & 1)) &&
                           wait_all(B_PRDY, jb & 1) && (jb == 0 || wait_all(B_EARDY, (jb - 1) & 1))))
                    break;
                tc::fence_after_sync();
                const int u = jb % 3;
                const bool t1 = PRE && (jb & 1);
                const uint64_t dtf = t1 ? dTF1 : dTF, dtp = t1 ? dTP1 : dTP;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_elect(tbase + cAB, dXmn0 + slot_off(u) + (uint64_t)(ks * 128), dtf + (uint64_t)(ks * 128), kIdAT, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_elect(tbase + cAB + 64, dPB + (uint64_t)(ks * 2), dtp + (uint64_t)(ks * 128), kIdBP, ks > 0);
                tc::mma_commit_elect(&bars[B_ABDONE]);
                tc::mma_commit_elect(&bars[B_XQFREE + u]);   // (a), (A) of the slot are done (one of two arrivals)
                if (PRE) tc::mma_commit_elect(&bars[B_TFREE + (jb & 1)]);
            }
        }
        if (!ok) *abort_flag = 1;
        // drain: every MMA this warp issued has completed, every armed load has landed
        tc::mma_commit_elect(&bars[B_FINAL0]);
        const volatile int no_abort = 0;
        tc::mbar_wait(&bars[B_FINAL0], 0, &no_abort, kDrainBudget);
        if (lane == 0) {
            for (int c = kx - 3 < 0 ? 0 : kx - 3; c < kx; ++c)
                tc::mbar_wait(&bars[B_FULLXQ + c % 3], (c / 3) & 1, &no_abort, kDrainBudget);
            for (int c = kv - 2 < 0 ? 0 : kv - 2; c < kv; ++c)
                tc::mbar_wait(&bars[B_FULLV + (c & 1)], (c >> 1) & 1, &no_abort, kDrainBudget);
            for (int c = kt - 2 < 0 ? 0 : kt - 2; c < kt; ++c)
                tc::mbar_wait(&bars[B_FULLT + (c & 1)], (c >> 1) & 1, &no_abort, kDrainBudget);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================================================================ chain MMAs (whole warp, elected lane issues)
        const uint64_t dBp = tc::sdesc(tc::smem_u32(sPB + 8192), 16, 1024);
        const uint64_t dAt = tc::sdesc(tc::smem_u32(sA), 16, 1024);
        bool ok = true;
        if (!REG) {
            // Inner-product rules: no solve, so the block's writes do not depend on the state.
            //   O   = diag(2^g) Q S^T + P~ diag(beta) Y     (E = (diag(beta) Y)^T P~^T, transposed)
            //   dS  = (diag(w) Y)^T X,   w = beta 2^(g_last - g),   S <- 2^g_last S + dS
            // The scaled value tiles (diag(beta) Y in place in the V slot, diag(w) Y in the T tile region)
            // are the MN-major A operands, read straight from shared memory; X is the MN-major B of dS and
            // P~ the K-major B of E. Slots alternate: dS of block c lands in the slot that held the outputs
            // of block c-1, [E | S Q^T] of block c in the one dS of block c-1 was read from.
            const uint64_t dPB = tc::sdesc(tc::smem_u32(sPB), 16, 1024);              // P~ rows 0-63, K-major B
            const uint64_t dVw = tc::sdesc(tc::smem_u32(sTF), 8192, 1024);            // diag(w) Y, MN-major A
            const uint64_t dXmnB = tc::sdesc(tc::smem_u32(sm + oXQ), 16384, 1024);   // X as an MN-major B
            for (int c = 0; c < nblk && ok; ++c) {
                const int s = c & 1, u = c % 3;
                const uint64_t dVb = tc::sdesc(tc::smem_u32(sm + oV + s * kVst), 8192, 1024);  // diag(beta) Y
                if (!(ok = wait_all(B_SRDY, c & 1) && wait_all(B_TRDY, c & 1) && wait_all(B_PRDY, c & 1))) break;
                tc::fence_after_sync();
                const uint64_t dQ = dXQ0 + slot_off(u) + (8192 >> 4);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)   // S Q^T -> columns 64-127 of slot s
                    tc::mma_bf16_ts_elect(tbase + cSXO + 128 * s + 64, tbase + cSR + 8 * ks, dQ + kmaj(ks), kIdN64, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // E -> columns 0-63 of slot s
                    tc::mma_bf16_elect(tbase + cSXO + 128 * s, dVb + (uint64_t)(ks * 128), dPB + (uint64_t)(ks * 2), kIdVP, ks > 0);
                tc::mma_commit_elect(&bars[B_BDONE]);              // outputs of block c ready
                // dS into slot s^1 once the outputs of block c-1 have been read out of it
                if (c >= 1 && !(ok = wait_all(B_EARDY, (c - 1) & 1))) break;
                tc::fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_elect(tbase + cSXO + 128 * (s ^ 1), dVw + (uint64_t)(ks * 128),
                                       dXmnB + slot_off(u) + (uint64_t)(ks * 128), kIdVX, ks > 0);
                tc::mma_commit_elect(&bars[B_EFDONE]);
                tc::mma_commit_elect(&bars[B_XQFREE + u]);   // the other arrival of the slot
                tc::mma_commit_elect(&bars[B_VFREE + s]);    // diag(beta) Y read: the V slot may refill
                tc::mma_commit_elect(&bars[B_ABDONE]);       // diag(w) Y read: the tile may be rewritten
            }
        }
        int kvr = 0;   // regression rules: V loads armed by this warp
        if (REG) {
            // (with the test hook, nothing at or after the stalled block is loaded, so that the armed loads
            // are exactly blocks 0 .. kvr-1)
            for (; kvr < 2 && kvr < nblk && (p.dbg_stall_block < 0 || kvr < p.dbg_stall_block); ++kvr) load_v(kvr);
        }
        // Regression rules: this warp only streams V; the chain warps issue their own MMAs and free a
        // V slot once the products that read it are done.
        for (int c = 0; c + 2 < nblk && ok && REG; ++c) {
            if (p.dbg_stall_block >= 0 && c + 2 >= p.dbg_stall_block) break;
            if (!(ok = wait_all(B_VFREE + (c & 1), (c >> 1) & 1))) break;
            load_v(c + 2);
            kvr = c + 3;
        }
        if (!ok) *abort_flag = 1;
        // drain every MMA issued by this warp and every V load it armed
        const volatile int no_abort = 0;
        if (!REG) {
            tc::mma_commit_elect(&bars[B_FINAL]);
            tc::mbar_wait(&bars[B_FINAL], 0, &no_abort, kDrainBudget);
        }
        if (lane == 0)
            for (int c = kvr - 2 < 0 ? 0 : kvr - 2; c < kvr; ++c)
                tc::mbar_wait(&bars[B_FULLV + (c & 1)], (c >> 1) & 1, &no_abort, kDrainBudget);
        __syncwarp();
    } else if (warp < 4) {
        // ================================================================ helpers (64 threads)
        const int ht = tid - 64;           // row / token index 0..63
        const bool leader = ht == 0;
        const float *alpha_h = p.alpha + (size_t)bh * T;
        float ga = 1.f;                    // decay gate of the block prep() handles next
        auto load_gates = [&](int c) {
            const int t = c * TB + ht;
            ga = (ht < TB && t < T) ? alpha_h[t] : 1.f;
        };
        auto prep = [&](int c) -> bool {   // block c: x_1 patch, decay tables
            const int u3 = c % 3, u4 = c % 4;
            uint8_t *xq = sm + oXQ + u3 * kXQ;
            if (c >= 4 && !role_wait(&bars[B_SCALFREE + u4], ((c >> 2) - 1) & 1, leader, 1, 64)) return false;
            if (!role_wait(&bars[B_FULLXQ + u3], (c / 3) & 1, leader, 1, 64)) return false;
            const int t0 = c * TB, nval = min(TB, T - t0);
            if (c == 0 && p.k_prev && !p.same_step && ht < 16 * W) {
                // pair 0 = (k_prev, v_0) sits in row m * TB + m of block 0 for every m < W
                const int m = ht >> 4, chunk = ht & 15;
                const uint4 v = *reinterpret_cast<const uint4 *>(
                    reinterpret_cast<const __nv_bfloat16 *>(p.k_prev) + (size_t)bh * D + chunk * 8);
                *reinterpret_cast<uint4 *>(xq + (chunk >> 3) * 16384 + tc::sw128_chunk(m * TB + m, chunk & 7)) = v;
                tc::fence_proxy_async();
            }
            const bool valid = ht < nval;
            float la = valid ? log2f(ga) : 0.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, la, off);
                if (lane >= off) la += y;
            }
            float *sc = sScal + u4 * 256;
            float gl;
            if (W == 1) {
                if (ht == 31) sMisc[0] = la;
                named_bar(1, 64);
                if (ht >= 32) la += sMisc[0];
                sc[64 + ht] = exp2f(la);
                sc[192 + ht] = la;
                named_bar(1, 64);
                gl = sc[192 + nval - 1];
                sc[128 + ht] = exp2f(gl - la);
                sCF[64 * u4 + ht] = exp2f(sc[192 + (ht | 15)] - la);
            } else {
                // TB <= 32 tokens: one warp's scan gives the token decays; every row takes its token's
                if (ht < TB) sMisc[1 + ht] = la;
                named_bar(1, 64);
                const float g = sMisc[1 + ht % TB];
                gl = sMisc[nval];
                sc[64 + ht] = exp2f(g);
                sc[192 + ht] = g;
                sc[128 + ht] = exp2f(gl - g);
            }
            if (leader) sGL[u4] = gl;
            named_bar(1, 64);
            if (leader) {
                mbar_arrive(&bars[B_SCAL + u4]);
                mbar_arrive(&bars[B_XQRDY + u3]);
            }
            return true;
        };
        bool ok = true;
        if (nblk > 0) {
            load_gates(0);
            ok = prep(0);
        }
        if (ok && nblk > 1) {
            load_gates(1);
            ok = prep(1);
        }
        for (int c = 0; c < nblk && ok; ++c) {
            if (c + 2 < nblk) load_gates(c + 2);  // in flight while block c is handled
            const float *sc = sScal + (c % 4) * 256;
            if (!(ok = role_wait(&bars[B_ADONE], c & 1, leader, 1, 64))) break;
            // P of query row i = ht from TMEM lanes 64..127 (this pair of warps' quarters)
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
            named_bar(1, 64);
            if (leader) mbar_arrive(&bars[B_GPFREE]);
            // P~ = Gamma o P (inclusive), packed to bf16 while (B') of the previous block still reads the tile
            uint32_t pk[32];
            if (W > 1) {
                // query token i = ht < TB reads the rows of tokens s' <= i (inclusive); rows of one token
                // share its decay 2^(g_i - g_s'); rows i >= TB of P are zero (their query rows are)
                const float *g2 = sc + 192;
                const int i = ht;
                const float gri = g2[i];
                float fac[TB];
#pragma unroll
                for (int sp = 0; sp < TB; ++sp) fac[sp] = sp <= i ? exp2f(fminf(gri - g2[sp], 0.f)) : 0.f;
#pragma unroll
                for (int j = 0; j < 64; j += 2) pk[j >> 1] = pack_bf16x2(fac[j % TB] * v[j], fac[(j + 1) % TB] * v[j + 1]);
            } else {
                const float *g2 = sc + 192, *cf = sCF + 64 * (c % 4);
                const int i = ht, rb = i >> 4;
                const float gri = g2[i];
                float gd[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 g4 = *reinterpret_cast<const float4 *>(g2 + 16 * rb + 4 * q);
                    const int j = 16 * rb + 4 * q;
                    gd[4 * q] = j <= i ? exp2f(fminf(gri - g4.x, 0.f)) : 0.f;
                    gd[4 * q + 1] = j + 1 <= i ? exp2f(fminf(gri - g4.y, 0.f)) : 0.f;
                    gd[4 * q + 2] = j + 2 <= i ? exp2f(fminf(gri - g4.z, 0.f)) : 0.f;
                    gd[4 * q + 3] = j + 3 <= i ? exp2f(fminf(gri - g4.w, 0.f)) : 0.f;
                }
#pragma unroll
                for (int jb = 0; jb < 4; ++jb) {
                    const float fac = jb < rb ? exp2f(fminf(gri - g2[16 * jb + 15], 0.f)) : 0.f;
                    const bool diag = jb == rb;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int j = 16 * jb + 4 * q;
                        const float4 c4 = *reinterpret_cast<const float4 *>(cf + j);
                        const float w0 = diag ? gd[4 * q] : fac * c4.x, w1 = diag ? gd[4 * q + 1] : fac * c4.y;
                        const float w2 = diag ? gd[4 * q + 2] : fac * c4.z, w3 = diag ? gd[4 * q + 3] : fac * c4.w;
                        pk[j >> 1] = pack_bf16x2(w0 * v[j], w1 * v[j + 1]);
                        pk[(j >> 1) + 1] = pack_bf16x2(w2 * v[j + 2], w3 * v[j + 3]);
                    }
                }
            }
            // the tile is free once the products of block c-1 that read P~ are done: (B') for the
            // regression rules, E for the inner-product rules
            if (c >= 1 && !(ok = role_wait(&bars[REG ? B_ABDONE : B_BDONE], (c - 1) & 1, leader, 1, 64))) break;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4 *>(sPB + tc::sw128_chunk(ht, ch)) =
                    make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
            tc::fence_proxy_async();
            named_bar(1, 64);
            if (leader) mbar_arrive(&bars[B_PRDY]);
            if (REG && !PRE) {
                // T_f = diag(2^(g_last - g)) T diag(beta) and T' = T diag(beta) (bf16, m-major order) from
                // the solved T; the tiles are free since (A), (B') of block c-1 are done (waited above)
                if (!(ok = role_wait(&bars[B_SOLVED], c & 1, leader, 1, 64))) break;
                const int rr = ht;
                const float fr = sc[128 + rr];
              if constexpr (W > 1) {
                // T' row rr into registers (all reads before any store, so that their latencies overlap)
                float tp[64];
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const int j0 = 8 * cc;
                    {
                        // T is in token-major order: row (rr % TB) W + rr / TB; the eight m-major columns
                        // j0.. share m' = j0 / TB and take tokens j0 % TB + k, i.e. a stride of W
                        const float *Trow = sTf + ((rr % TB) * W + rr / TB) * LDF + (j0 % TB) * W + j0 / TB;
#pragma unroll
                        for (int k = 0; k < 8; ++k) tp[j0 + k] = Trow[k * W];
                    }
                    const float4 b0 = *reinterpret_cast<const float4 *>(sc + j0);     // beta of the columns
                    const float4 b1 = *reinterpret_cast<const float4 *>(sc + j0 + 4);
                    tp[j0] *= b0.x; tp[j0 + 1] *= b0.y; tp[j0 + 2] *= b0.z; tp[j0 + 3] *= b0.w;
                    tp[j0 + 4] *= b1.x; tp[j0 + 5] *= b1.y; tp[j0 + 6] *= b1.z; tp[j0 + 7] *= b1.w;
                }
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    float f8[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) f8[k] = fr * tp[8 * cc + k];
                    st_chunk8(sTP, tc::sw128_chunk(rr, cc), tp + 8 * cc);
                    st_chunk8(sTF, tc::sw128_chunk(rr, cc), f8);
                }
              } else {
#pragma unroll 2
                for (int cc = 0; cc < 8; ++cc) {
                    const int j0 = 8 * cc;
                    float t8[8], f8[8];
                    {
                        const float4 x0 = *reinterpret_cast<const float4 *>(sTf + rr * LDF + j0);
                        const float4 x1 = *reinterpret_cast<const float4 *>(sTf + rr * LDF + j0 + 4);
                        t8[0] = x0.x; t8[1] = x0.y; t8[2] = x0.z; t8[3] = x0.w;
                        t8[4] = x1.x; t8[5] = x1.y; t8[6] = x1.z; t8[7] = x1.w;
                    }
                    const float4 b0 = *reinterpret_cast<const float4 *>(sc + j0);     // beta of the columns
                    const float4 b1 = *reinterpret_cast<const float4 *>(sc + j0 + 4);
                    const float bc[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        t8[k] *= bc[k];
                        f8[k] = fr * t8[k];
                    }
                    st_chunk8(sTP, tc::sw128_chunk(rr, cc), t8);
                    st_chunk8(sTF, tc::sw128_chunk(rr, cc), f8);
                }
              }
                tc::fence_proxy_async();
                named_bar(1, 64);
                if (leader) {
                    mbar_arrive(&bars[B_TREAD]);
                    mbar_arrive(&bars[B_TRDY]);
                }
            }
            // the block after next: its slot frees once (b) of block c-1 is done
            if (c + 2 < nblk && !(ok = prep(c + 2))) break;
        }
    } else if (warp < 8 && PRE) {
        // ================================================================ outputs (two-pass path)
        // The local warps have no solve to run; they store the outputs of each block once (e') is done,
        // which takes that work off the chain. Warp 4 + q reads TMEM lanes 32 q .. 32 q + 31.
        const int qd = warp & 3, row = 32 * qd + lane;
        const uint32_t tl = tbase + ((uint32_t)(32 * qd) << 16);
        for (int c = 0; c < nblk; ++c) {
            if (!warp_wait(&bars[B_EDONES + (c & 1)], (c >> 1) & 1)) break;
            tc::fence_after_sync();
            store_out_rows<TB>(p.o, bh, T, c, row, tl, 0, sScal + (c % 4) * 256 + 64);
            store_out_rows<TB>(p.o, bh, T, c, row, tl, 1, sScal + (c % 4) * 256 + 64);
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_OUTFREE + (c & 1)]);   // (b) of block c + 2 may take the slot
                mbar_arrive(&bars[B_SCALFREE + c % 4]);
            }
        }
    } else if (warp < 8) {
        // ================================================================ local (128 threads)
        const int lt = tid - 128, lw = warp - 4;
        const int r = 32 * lw + lane;      // TMEM lane: G row for lw < 2 (P rows belong to the helpers)
        const bool leader = lt == 0;
        const uint32_t tl = tbase + ((uint32_t)(32 * lw) << 16);
        const float *eta_h = p.eta + (size_t)bh * T;
        const int rs = r % TB;             // token of row r (rows of one token share its step size)
        float ge = (lw < 2 && rs < T) ? eta_h[rs] : 0.f;  // step-size gate of row r's token, one block ahead
        for (int c = 0; c < nblk && !PRE; ++c) {   // (the two-pass path has no work for these warps)
            const int u4 = c % 4;
            // (a) of the block follows the helpers' readiness of it, which follows its decay scalars:
            // ADONE alone says both
            if (!role_wait(&bars[B_ADONE], c & 1, leader, 2, 128)) break;
            tc::fence_after_sync();
            float *sc = sScal + u4 * 256;
            if (lw < 2) {                                   // G rows r = 0..63: step sizes, then L
                const float *g2 = sc + 192, *cf = sCF + 64 * u4;
                const int rb = r >> 4;
                float v[64];
                {
                    float h0[32], h1[32];
                    tc::tmem_ld32(tl + cGP, h0);
                    tc::tmem_ld32(tl + cGP + 32, h1);
#pragma unroll
                    for (int j = 0; j < 32; ++j) { v[j] = h0[j]; v[32 + j] = h1[j]; }
                }
                // G is in registers: its columns may take (a) of the next block
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_GPFREE]);
                // ||x_r||^2 is the diagonal entry G[r][r] = v[32 lw + lane] (a warp-uniform branch on lw
                // keeps v in registers)
                float nrm = lw == 0 ? pick_lane<0>(v, lane) : pick_lane<32>(v, lane);
                if (W > 1) {   // the token's window: rows m * TB + rs, m < W
                    sNrm[r] = nrm;
                    named_bar(3, 64);
                    nrm = 0.f;
#pragma unroll
                    for (int m = 0; m < W; ++m) nrm += sNrm[m * TB + rs];
                }
                const bool valid = c * TB + rs < T;
                const float be = valid ? step_size(ge, nrm, p.eps) : 0.f;
                sc[r] = be;
                const int tn = (c + 1) * TB + rs;
                ge = tn < T ? eta_h[tn] : 0.f;
              if (REG && W > 1) {
                // row u = rs * W + m of L in token-major order couples to the rows of earlier tokens
                // s' < rs only: L[u][s' W + m'] = beta 2^(g_rs - g_s') G[r][m' TB + s'], zero otherwise
                // (the rows of one token form the identity block of I + L)
                const float *g2 = sc + 192;
                const float gri = g2[r];
                float gd[TB];
#pragma unroll
                for (int sp = 0; sp < TB; ++sp) gd[sp] = sp < rs ? be * exp2f(fminf(gri - g2[sp], 0.f)) : 0.f;
                float *Lr = sL + (rs * W + r / TB) * LDF;
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    float w4[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int up = 4 * q + k, sp = up / W, mp = up % W;
                        w4[k] = gd[sp] * v[mp * TB + sp];
                    }
                    *reinterpret_cast<float4 *>(Lr + 4 * q) = make_float4(w4[0], w4[1], w4[2], w4[3]);
                }
              } else if (REG) {
                // Decay factors 2^(g_r - g_j), j < r: below the 16x16 diagonal blocks they factor
                // through the last index of column block jb, 2^(g_r - g_{16jb+15}) * cf[j] with
                // cf[j] = 2^(g_{16jb+15} - g_j) (a helper table), both in (0, 1]; inside the
                // diagonal block they are formed directly. The solve reads only the strictly lower
                // part, so entries on and above the diagonal are left as they come (finite, <= |G|).
                const float gri = g2[r];
                float gd[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 g4 = *reinterpret_cast<const float4 *>(g2 + 16 * rb + 4 * q);
                    gd[4 * q] = be * exp2f(fminf(gri - g4.x, 0.f));
                    gd[4 * q + 1] = be * exp2f(fminf(gri - g4.y, 0.f));
                    gd[4 * q + 2] = be * exp2f(fminf(gri - g4.z, 0.f));
                    gd[4 * q + 3] = be * exp2f(fminf(gri - g4.w, 0.f));
                }
                float *Lr = sL + r * LDF;
#pragma unroll
                for (int jb = 0; jb < 4; ++jb) {
                    const float fac = be * exp2f(fminf(gri - g2[16 * jb + 15], 0.f));
                    const bool below = jb < rb;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int j = 16 * jb + 4 * q;
                        const float4 c4 = *reinterpret_cast<const float4 *>(cf + j);
                        const float w0 = below ? fac * c4.x : gd[4 * q];
                        const float w1 = below ? fac * c4.y : gd[4 * q + 1];
                        const float w2 = below ? fac * c4.z : gd[4 * q + 2];
                        const float w3 = below ? fac * c4.w : gd[4 * q + 3];
                        *reinterpret_cast<float4 *>(Lr + j) =
                            make_float4(w0 * v[j], w1 * v[j + 1], w2 * v[j + 2], w3 * v[j + 3]);
                    }
                }
              }
            }
            named_bar(2, 128);
            if (!REG) {
                // The scaled value tiles of block c (inner-product rules): diag(beta) Y in place in its V
                // slot and diag(w) Y, w = beta 2^(g_last - g), into the T tile region, once V has landed and
                // the products of block c-1 no longer read the region. Thread (row rr, atom at) scales the
                // 64 values of its row in that atom; scaling does not care where the swizzle put them.
                if (!role_wait(&bars[B_FULLV + (c & 1)], (c >> 1) & 1, leader, 2, 128)) break;
                if (c >= 1 && !role_wait(&bars[B_ABDONE], (c - 1) & 1, leader, 2, 128)) break;
                const int rr = lt >> 1, at = lt & 1;
                const float bb = sc[rr], ww = bb * sc[128 + rr];
                const uint32_t line = at * 8192 + (rr >> 3) * 1024 + (rr & 7) * 128;
                uint8_t *vrow = sm + oV + (c & 1) * kVst + line;
                uint8_t *wrow = sTF + line;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const int cc = ch ^ (rr & 7);      // rows of a group start on different banks
                    const uint4 x = *reinterpret_cast<const uint4 *>(vrow + 16 * cc);
                    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
                    uint32_t bs[4], ws[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xs[k]));
                        bs[k] = pack_bf16x2(bb * f.x, bb * f.y);
                        ws[k] = pack_bf16x2(ww * f.x, ww * f.y);
                    }
                    *reinterpret_cast<uint4 *>(vrow + 16 * cc) = make_uint4(bs[0], bs[1], bs[2], bs[3]);
                    *reinterpret_cast<uint4 *>(wrow + 16 * cc) = make_uint4(ws[0], ws[1], ws[2], ws[3]);
                }
                tc::fence_proxy_async();
                named_bar(2, 128);
                if (leader) mbar_arrive(&bars[B_TRDY]);
                continue;
            }
            // the previous block's T has been read into its bf16 tiles before this solve overwrites it
            if (c >= 1 && !role_wait(&bars[B_TREAD], (c - 1) & 1, leader, 2, 128)) break;
            solve_local(sL, sTf, lt, lw, lane);   // ends with the local warps' barrier
            if (leader) mbar_arrive(&bars[B_SOLVED]);
        }
    } else {
        // ================================================================ chain (256 threads)
        const int ct = tid - 256;
        const int qd = warp & 3, hf = (warp - 8) >> 2;
        const int row = 32 * qd + lane;    // TMEM lane = value row (and key row d of A^T)
        const uint32_t tl = tbase + ((uint32_t)(32 * qd) << 16);
        float S[64];                       // fp32 state, row `row`, columns 64 hf ..
        auto store_S = [&]() {             // bf16 pairs of this thread's 64 columns -> TMEM A operand
            uint32_t pk[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) pk[j] = pack_bf16x2(S[2 * j], S[2 * j + 1]);
            tc::tmem_st32(tl + cSR + 32 * hf, pk);
        };
        auto store_out = [&](int c) {
            store_out_rows<TB>(p.o, bh, T, c, row, tl, hf, sScal + (c % 4) * 256 + 64);
        };
        {
            const float *S0 = p.S0 ? p.S0 + ((size_t)bh * D + row) * D + 64 * hf : nullptr;
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
                const float4 x = S0 ? *reinterpret_cast<const float4 *>(S0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
            }
            store_S();
            if (!REG) warp_arrive(&bars[B_SRDY]);
            else tc::fence_before_sync();
        }
        bool ok = true;
        for (int c = 0; c < nblk && !REG; ++c) {
            // Inner-product rules: the state update is the whole chain; the outputs of the block are
            // read out of the other slot afterwards, which frees it for dS of the next block.
            const int s = c & 1, u4 = c % 4;
            if (!(ok = warp_wait(&bars[B_EFDONE], c & 1))) break;
            tc::fence_after_sync();
            {
                const float dl = exp2f(sGL[u4]);
                const uint32_t cds = cSXO + 128 * (s ^ 1) + 64 * hf;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    tc::tmem_ld32(tl + cds + 32 * hh, v);
#pragma unroll
                    for (int j = 0; j < 32; ++j) S[32 * hh + j] = dl * S[32 * hh + j] + v[j];
                }
            }
            store_S();
            warp_arrive(&bars[B_SRDY]);
            store_out(c);
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_EARDY]);            // slot s read: dS of block c+1 may take it
                mbar_arrive(&bars[B_SCALFREE + u4]);
            }
        }
        // Regression rules: the chain warps issue the state chain's MMAs themselves (warp 8, one elected
        // lane), right after the named barrier that says their own TMEM writes are done; only the
        // completions of MMAs are mbarrier handoffs. Every wait is taken by one thread for all 256 and
        // its outcome shared through the barrier, so that a timeout unwinds all chain warps together.
        const bool issuer = warp == 8;
        auto chain_wait = [&](int b, uint32_t parity) -> bool {
            const bool r = role_wait(&bars[b], parity, ct == 32, 4, 256);   // polled by a warp that does not issue
            tc::fence_after_sync();
            return r;
        };
        const uint64_t dAtC = tc::sdesc(tc::smem_u32(sA), 16, 1024);          // A^T, K-major B of dS
        const uint64_t dBpC = tc::sdesc(tc::smem_u32(sPB + 8192), 16, 1024);  // B', K-major B of E
        // Two-pass path: the output warps store the outputs, so the chain only runs the state chain.
        // (b) is one group of N = 128 ([X;Q] as the B operand), and A^T, B' are copied out first:
        // their (A), (B') ran during the previous block's state update.
        for (int c = 0; c < nblk && REG && PRE; ++c) {
            const int s = c & 1, u = c % 3, u4 = c % 4;
            {   // the block's [X;Q] slot is ready, and the outputs of block c-2 have left slot s
                bool failed = false;
                if (ct == 32) {
                    failed = !tc::mbar_wait(&bars[B_XQRDY + u], (c / 3) & 1, abort_flag, p.wait_budget) ||
                             (c >= 2 && !tc::mbar_wait(&bars[B_OUTFREE + s], ((c >> 1) - 1) & 1, abort_flag,
                                                       p.wait_budget));
                    if (failed) *abort_flag = 1;
                }
                if (!(ok = !named_bar_or(4, 256, failed))) break;
                tc::fence_after_sync();
            }
            if (issuer) {
                const uint64_t dXQ = dXQ0 + slot_off(u);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc::mma_bf16_ts_elect(tbase + cSXO + 128 * s, tbase + cSR + 8 * ks, dXQ + kmaj(ks), kIdN128, ks > 0);
                tc::mma_commit_elect(&bars[B_BDONE]);
                tc::mma_commit_elect(&bars[B_XQFREE + u]);   // (b) of the slot is done (the other arrival)
            }
            if (!(ok = chain_wait(B_ABDONE, c & 1))) break;
            {
                float v[32];
                tc::tmem_ld32(tl + cAB + 32 * hf, v);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) st_chunk8(sA, tc::sw128_chunk(row, 4 * hf + cc), v + 8 * cc);
                if (qd < 2) {
                    tc::tmem_ld32(tl + cAB + 64 + 32 * hf, v);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        st_chunk8(sPB + 8192, tc::sw128_chunk(row, 4 * hf + cc), v + 8 * cc);
                }
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            if (!(ok = chain_wait(B_FULLV + s, (c >> 1) & 1))) break;
            const uint64_t dY = tc::sdesc(tc::smem_u32(sm + oV + s * kVst), 8192, 1024);   // Y^T, MN-major A
            if (issuer) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_elect(tbase + cAB, dY + (uint64_t)(ks * 128), dAtC + (uint64_t)(ks * 2), kIdVA, ks > 0);
            }
            // -Z~ = -(S X^T) diag(2^g) in place of the bf16 state, which (b) has finished reading
            if (!(ok = chain_wait(B_BDONE, c & 1))) break;
            {
                const float *dg = sScal + u4 * 256 + 64 + 32 * hf;
                uint32_t pk[16];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float x[16];
                    tc::tmem_ld16(tl + cSXO + 128 * s + 32 * hf + 16 * hh, x);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 d4 = *reinterpret_cast<const float4 *>(dg + 16 * hh + 4 * q4);
                        pk[8 * hh + 2 * q4] = pack_bf16x2(-d4.x * x[4 * q4], -d4.y * x[4 * q4 + 1]);
                        pk[8 * hh + 2 * q4 + 1] = pack_bf16x2(-d4.z * x[4 * q4 + 2], -d4.w * x[4 * q4 + 3]);
                    }
                }
                tc::tmem_st16(tl + cSR + 16 * hf, pk);
            }
            tc::fence_before_sync();
            if ((ok = !named_bar_or(4, 256, false)) && issuer) {
                tc::fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_ts_elect(tbase + cAB, tbase + cSR + 8 * ks, dAtC + (uint64_t)(ks * 2), kIdN128, true);
                tc::mma_commit_elect(&bars[B_EFDONE]);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_elect(tbase + cSXO + 128 * s, dY + (uint64_t)(ks * 128), dBpC + (uint64_t)(ks * 2), kIdVP, ks > 0);
                tc::mma_commit_elect(&bars[B_VFREE + s]);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_ts_elect(tbase + cSXO + 128 * s, tbase + cSR + 8 * ks, dBpC + (uint64_t)(ks * 2), kIdN64, true);
                tc::mma_commit_elect(&bars[B_EDONES + s]);
            }
            if (!ok) break;
            if (!(ok = chain_wait(B_EFDONE, c & 1))) break;
            {
                const float dl = exp2f(sGL[u4]);
                const uint32_t cds = cAB + 64 * hf;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    tc::tmem_ld32(tl + cds + 32 * hh, v);
#pragma unroll
                    for (int j = 0; j < 32; ++j) S[32 * hh + j] = dl * S[32 * hh + j] + v[j];
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_EARDY]);          // dS read: the AB columns may take (A), (B') of the next block
                mbar_arrive(&bars[B_SCALFREE + u4]);  // the chain's reads of the scalar slot are done
            }
            if (!(ok = chain_wait(B_EDONES + s, (c >> 1) & 1))) break;
            store_S();
            tc::fence_before_sync();
        }
        for (int c = 0; c < nblk && REG && !PRE; ++c) {
            const int s = c & 1, u = c % 3, u4 = c % 4;
            // (b) Z = S X^T then S Q^T -> slot s, S (bf16) from TMEM: the block's [X;Q] slot is ready (and
            // so are its decay scalars), and every chain thread's bf16 state is in TMEM (barrier).
            if (!(ok = chain_wait(B_XQRDY + u, (c / 3) & 1))) break;
            if (issuer) {
                const uint64_t dX = dXQ0 + slot_off(u), dQ = dX + (8192 >> 4);   // X rows 0-63, Q rows 64-127
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc::mma_bf16_ts_elect(tbase + cSXO + 128 * s, tbase + cSR + 8 * ks, dX + kmaj(ks), kIdN64, ks > 0);
                tc::mma_commit_elect(&bars[B_BDONE]);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc::mma_bf16_ts_elect(tbase + cSXO + 128 * s + 64, tbase + cSR + 8 * ks, dQ + kmaj(ks), kIdN64, ks > 0);
                tc::mma_commit_elect(&bars[B_SQDONE]);
                tc::mma_commit_elect(&bars[B_XQFREE + u]);   // (b) of the slot is done (the other arrival)
            }
            // outputs of the previous block while (b) and (A), (B') run: their slot takes (b) of the
            // next block
            if (c >= 1) {
                store_out(c - 1);
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_SCALFREE + (c - 1) % 4]);
            }
            // A^T (rows d, columns i) and B' (rows i < 64) from TMEM to their shared-memory tiles
            if (!(ok = chain_wait(B_ABDONE, c & 1))) break;
            {
                float v[32];
                tc::tmem_ld32(tl + cAB + 32 * hf, v);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) st_chunk8(sA, tc::sw128_chunk(row, 4 * hf + cc), v + 8 * cc);
                if (qd < 2) {
                    tc::tmem_ld32(tl + cAB + 64 + 32 * hf, v);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        st_chunk8(sPB + 8192, tc::sw128_chunk(row, 4 * hf + cc), v + 8 * cc);
                }
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            // Y^T A, the state-independent half of dS, into the AB columns once V has landed (the
            // barrier also says that A^T and B' have been read out of those columns)
            if (!(ok = chain_wait(B_FULLV + s, (c >> 1) & 1))) break;
            const uint64_t dY = tc::sdesc(tc::smem_u32(sm + oV + s * kVst), 8192, 1024);   // Y^T, MN-major A
            if (issuer) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_elect(tbase + cAB, dY + (uint64_t)(ks * 128), dAtC + (uint64_t)(ks * 2), kIdVA, ks > 0);
            }
            // -Z~ = -(S X^T) diag(2^g), bf16 into TMEM: with dS = Y^T A - Z~ A and E = Y^T B'^T - Z~ B'^T the
            // values themselves only enter through the tensor cores. It replaces the bf16 state, which
            // S Q^T may still be reading.
            if (!(ok = chain_wait(B_BDONE, c & 1))) break;
            {
                const float *dg = sScal + u4 * 256 + 64 + 32 * hf;   // 2^g of this thread's 32 rows
                uint32_t pk[16];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {   // 16 rows at a time (the state stays in registers)
                    float x[16];
                    tc::tmem_ld16(tl + cSXO + 128 * s + 32 * hf + 16 * hh, x);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 d4 = *reinterpret_cast<const float4 *>(dg + 16 * hh + 4 * q4);
                        pk[8 * hh + 2 * q4] = pack_bf16x2(-d4.x * x[4 * q4], -d4.y * x[4 * q4 + 1]);
                        pk[8 * hh + 2 * q4 + 1] = pack_bf16x2(-d4.z * x[4 * q4 + 2], -d4.w * x[4 * q4 + 3]);
                    }
                }
                if (!(ok = chain_wait(B_SQDONE, c & 1))) break;
                tc::tmem_st16(tl + cSR + 16 * hf, pk);
            }
            tc::fence_before_sync();
            // (f') dS += -Z~ A (the state update waits for it), then (e') Y^T B'^T - Z~ B'^T over S X^T in
            // slot s (the outputs wait for it); -Z~ (bf16) from TMEM
            if ((ok = !named_bar_or(4, 256, false)) && issuer) {
                tc::fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_ts_elect(tbase + cAB, tbase + cSR + 8 * ks, dAtC + (uint64_t)(ks * 2), kIdN128, true);
                tc::mma_commit_elect(&bars[B_EFDONE]);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_elect(tbase + cSXO + 128 * s, dY + (uint64_t)(ks * 128), dBpC + (uint64_t)(ks * 2), kIdVP, ks > 0);
                tc::mma_commit_elect(&bars[B_VFREE + s]);    // Y read: the V slot may refill
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_ts_elect(tbase + cSXO + 128 * s, tbase + cSR + 8 * ks, dBpC + (uint64_t)(ks * 2), kIdN64, true);
                tc::mma_commit_elect(&bars[B_EDONE]);
            }
            // state update: S <- 2^g_last S + dS, then its bf16 copy for (b) of the next block
            if (!(ok = chain_wait(B_EFDONE, c & 1))) break;
            {
                const float dl = exp2f(sGL[u4]);
                const uint32_t cds = cAB + 64 * hf;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    tc::tmem_ld32(tl + cds + 32 * hh, v);
#pragma unroll
                    for (int j = 0; j < 32; ++j) S[32 * hh + j] = dl * S[32 * hh + j] + v[j];
                }
            }
            warp_arrive(&bars[B_EARDY]);    // dS read: the AB columns may take (A), (B') of the next block
            // (e') still reads -Z~ from the columns the bf16 state takes
            if (!(ok = chain_wait(B_EDONE, c & 1))) break;
            store_S();
            tc::fence_before_sync();
        }
        if (REG && issuer) {
            // drain every MMA this warp issued (after a timeout some may still be in flight)
            tc::mma_commit_elect(&bars[B_FINAL]);
            const volatile int no_abort = 0;
            tc::mbar_wait(&bars[B_FINAL], 0, &no_abort, kDrainBudget);
            __syncwarp();
        }
        if (REG && !PRE && ok && nblk > 0 && !*abort_flag) {
            store_out(nblk - 1);
            tc::fence_before_sync();
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

bool chunk_ws_supported(const ChunkParams &p) {
    const bool w_ok = p.window == 1 || p.window == 2 || p.window == 4;
    return p.dk == 128 && p.dv == 128 && p.io_bf16 && w_ok && p.tok_per_blk * p.window == kBlk && p.T >= 1 &&
           encode_tiled_fn() != nullptr;
}

namespace {

template <int W>
cudaError_t launch_chunk_ws_w(const ChunkParams &p, cudaStream_t s) {
    const long long BH = (long long)p.B * p.H;
    constexpr int TB = kBlk / W;  // boxes of TB rows: the W shifted copies of a block's keys and values
    CUtensorMap mK, mQ, mV;
    if (!map_head_rows(&mK, p.k, p.T, BH, TB) || !map_head_rows(&mQ, p.q, p.T, BH, TB) ||
        !map_head_rows(&mV, p.v, p.T, BH, TB))
        return cudaErrorInvalidValue;
    const bool two_pass = p.tiles != nullptr && chunk_tile_bytes(p) > 0;
    cudaError_t e;
    auto kern = p.regression ? chunk_ws_kernel<true, W, false> : chunk_ws_kernel<false, W, false>;
    if (two_pass) {
        {
            const int nblk = (p.T + TB - 1) / TB;
            e = cudaFuncSetAttribute(chunk_local_kernel<W>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kLocSmem);
            if (e != cudaSuccess) return e;
            int dev = 0, sms = 0;
            if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
            if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
            const long long items = BH * nblk, slots = (long long)sms * kLocCtasPerSm;   // items < 2^31
            chunk_local_kernel<W><<<(unsigned)(items < slots ? items : slots), kLocThreads, kLocSmem, s>>>(mK, p, nblk);
            kern = chunk_ws_kernel<true, W, true>;
        }
    }
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)BH, kThreads, kSmem, s>>>(mK, mQ, mV, p);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_tile_bytes(const ChunkParams &p) {
    if (!p.regression || !chunk_ws_supported(p)) return 0;
    const int tb = kBlk / p.window;   // tokens per block
    const long long blocks = (long long)p.B * p.H * ((p.T + tb - 1) / tb);
    if (blocks <= 0 || blocks > (1LL << 30)) return 0;
    return (size_t)blocks * kTileBytes;
}

cudaError_t launch_chunk_ws(const ChunkParams &p, cudaStream_t s) {
    switch (p.window) {
        case 1: return launch_chunk_ws_w<1>(p, s);
        case 2: return launch_chunk_ws_w<2>(p, s);
        case 4: return launch_chunk_ws_w<4>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace falcon
