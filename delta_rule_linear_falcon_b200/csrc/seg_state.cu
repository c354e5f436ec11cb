// seg_state.cu -- sequence split of the chunk-parallel forward pass for the
// inner-product rule (Falcon-1A), for problems with fewer heads than SMs.
//
// The inner-product write S_t = alpha_t S_{t-1} + beta_t y_t x_t^T ("Fast Weight
// Attention for Continual Learning", authors' abstract: the additive variant of the
// write) has a scalar state transition, so over any run of tokens
//   S(after the run) = 2^(G_end) S(before the run) + D,
//   D = sum_t 2^(G_end - G_t) beta_t y_t x_t^T,
// with G_t the cumulative log2 decay of the run through token t; D does not depend on
// the state. A head of T tokens is cut into nseg segments of L tokens (whole 64-token
// blocks), and three launches on one stream give the same result as one pass:
//   1. seg_piece_kernel: D and G_end of every piece (a run of whole blocks inside a
//      segment) in parallel, as one tcgen05 product per piece,
//        D = (diag(w) Y)^T X,  w_t = beta_t 2^(G_end - G_t),  K = the piece's tokens;
//   2. seg_scan_kernel: the state at each segment start by the recurrence above over the
//      pieces, the final state, the key cached before each segment and the last key;
//   3. the chunk kernel on the segments viewed as heads of L tokens: the (B, H, T, d)
//      tensors are contiguous, so segment s of head h is head h * nseg + s of a
//      (B, H * nseg, L, d) view, started from its own state and cached key.
// Every decay factor is 2^a with a <= 0 (positive-decay renormalisation).
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace falcon {

namespace {

constexpr int kPThreads = 192;                 // warp 0 TMA, warp 1 MMA, warps 2-5 step sizes and drain
constexpr int kPBlk = 64;                      // tokens per pipeline stage (one block)
constexpr int kMaxPieceBlocks = 32;            // a piece holds at most 2048 tokens
constexpr int kMinSegBlocks = 8;               // a segment holds at least 8 blocks
constexpr int kStages = 3;
constexpr uint32_t kStage = 32768;             // X: 2 atoms (d 0-63, 64-127) x 64 rows, then Y the same
constexpr uint32_t oG = kStages * kStage;      // cumulative log2 decay of the piece, one float per token
constexpr uint32_t oRed = oG + kMaxPieceBlocks * kPBlk * 4;
constexpr uint32_t oPBar = oRed + 64;
enum : int { P_FULL = 0, P_SCALED = kStages, P_EMPTY = 2 * kStages, P_DONE = 3 * kStages, P_COUNT };
constexpr uint32_t kPSmem = oPBar + P_COUNT * 8 + 16 + 1024;   // + TMEM slot and abort flag, alignment slack
constexpr uint32_t kPCols = 128;
constexpr long long kPDrainBudget = kDefaultWaitBudget;       // waits for own loads / MMAs in flight at exit
constexpr uint32_t kIdD = tc::idesc_bf16(128, 128, 1, 1);     // (diag(w) Y)^T (MN-major A) x X (MN-major B)
constexpr size_t kStateBytes = 128 * 128 * sizeof(float);

struct PieceParams {
    int T;         // tokens per head
    int piece;     // tokens per piece
    int pneed;     // pieces per head computed by this launch
    int ptot;      // pieces per head in the workspace
    bool same_step;
    const void *k_prev;
    const float *alpha, *eta;
    float eps;
    float *D, *a;  // per piece: the state increment (d_v x d_k) and the log2 decay of the piece
    int *err;
    long long wait_budget;  // bounded waits give up after this many SM clocks
    int dbg_stall_block;    // test hook: the producer stops loading at this block (-1: never)
};

struct ScanParams {
    int nseg, pps, ptot, L, T;
    const void *k, *k_prev;
    const float *S0, *D, *a;
    float *Sinit, *S_out;
    void *kp, *k_last;
};

__device__ __forceinline__ void mbar_arrive_cta(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void scaler_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Barrier of the four scaling warps that also ORs a predicate over them.
__device__ __forceinline__ bool scaler_sync_or(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float sumsq_bf16x2(uint32_t u, float acc) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
    return fmaf(f.y, f.y, fmaf(f.x, f.x, acc));
}

__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t u, float w) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
    return pack_bf16x2(f.x * w, f.y * w);
}

// One CTA per (head, piece). The pairs of a 64-token block arrive by TMA in the 128-byte
// swizzled layout (token rows, d columns in two 64-column atoms); the scaling warps form
// ||x_t||^2 and w_t and scale the value rows in place (a row's line holds all 64 of its
// elements of an atom in some order, so neither needs the swizzle), then the MMA warp adds
// the block's four K = 16 steps into the 128 x 128 fp32 accumulator in tensor memory.
__global__ void __launch_bounds__(kPThreads, 2)
seg_piece_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, PieceParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *sG = reinterpret_cast<float *>(sm + oG);
    float *sRed = reinterpret_cast<float *>(sm + oRed);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + oPBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + P_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
    constexpr int D = 128;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x / p.pneed, piece = blockIdx.x % p.pneed;
    const int t0 = piece * p.piece, nst = p.piece / kPBlk;
    const size_t out = (size_t)head * p.ptot + piece;

    if (tid == 0) {
        for (int i = 0; i < P_COUNT; ++i) tc::mbar_init(&bars[i], (i >= P_SCALED && i < P_EMPTY) ? 4 : 1);
        *abort_flag = 0;
        tc::mbar_fence_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tslot, kPCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tslot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer: X (prefix-aligned keys) and Y per block
        if (lane == 0) {
            const int kshift = p.same_step ? 0 : 1;
            int armed = 0;
            for (int i = 0; i < nst && !*abort_flag; ++i) {
                if (i == p.dbg_stall_block) break;  // test hook: this block is never loaded
                const int s = i % kStages;
                if (i >= kStages &&
                    !tc::mbar_wait(&bars[P_EMPTY + s], ((i / kStages) - 1) & 1, abort_flag, p.wait_budget)) {
                    *abort_flag = 1;
                    break;
                }
                uint8_t *dst = sm + s * kStage;
                uint64_t *fb = &bars[P_FULL + s];
                const int t = t0 + i * kPBlk;
                tc::mbar_arrive_expect_tx(fb, kStage);
                tc::tma_load_3d(dst, &tmK, 0, t - kshift, head, fb);
                tc::tma_load_3d(dst + 8192, &tmK, 64, t - kshift, head, fb);
                tc::tma_load_3d(dst + 16384, &tmV, 0, t, head, fb);
                tc::tma_load_3d(dst + 24576, &tmV, 64, t, head, fb);
                armed = i + 1;
            }
            // every armed load must have landed before the CTA can exit
            const volatile int no_abort = 0;
            for (int i = armed - kStages < 0 ? 0 : armed - kStages; i < armed; ++i)
                tc::mbar_wait(&bars[P_FULL + i % kStages], (i / kStages) & 1, &no_abort, kPDrainBudget);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (whole warp, elected lane issues)
        const uint64_t dX = tc::sdesc(tc::smem_u32(sm), 8192, 1024);           // X: MN-major B, N = d_k
        const uint64_t dY = tc::sdesc(tc::smem_u32(sm + 16384), 8192, 1024);   // diag(w) Y: MN-major A, M = d_v
        bool ok = true;
        for (int i = 0; i < nst; ++i) {
            const int s = i % kStages;
            ok = __all_sync(0xffffffffu,
                            tc::mbar_wait(&bars[P_SCALED + s], (i / kStages) & 1, abort_flag, p.wait_budget));
            if (!ok) break;
            tc::fence_after_sync();
            const uint64_t so = (uint64_t)(s * (kStage >> 4));
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_bf16_elect(tbase, dY + so + (uint64_t)(ks * 128), dX + so + (uint64_t)(ks * 128), kIdD,
                                   (i | ks) != 0);
            tc::mma_commit_elect(&bars[P_EMPTY + s]);
        }
        if (!ok) *abort_flag = 1;
        tc::mma_commit_elect(&bars[P_DONE]);
        const volatile int no_abort = 0;
        tc::mbar_wait(&bars[P_DONE], 0, &no_abort, kPDrainBudget);
        __syncwarp();
    } else {
        // ------------------------------------------------ scaling warps (128 threads), then the drain
        const int st = tid - 64, sw = warp - 2;
        const bool leader = st == 0;
        const size_t hb = (size_t)head * p.T + t0;
        const float *alpha_h = p.alpha + hb, *eta_h = p.eta + hb;
        // G over the piece: each thread a run of m tokens, then an exclusive scan of the run totals
        const int m = (p.piece + 127) >> 7;
        float run = 0.f;
        for (int j = 0; j < m; ++j) {
            const int t = st * m + j;
            if (t < p.piece) {
                run += log2f(alpha_h[t]);
                sG[t] = run;
            }
        }
        float inc = run;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += y;
        }
        if (lane == 31) sRed[sw] = inc;
        scaler_sync();
        float base = inc - run;
        for (int w = 0; w < sw; ++w) base += sRed[w];
        for (int j = 0; j < m; ++j) {
            const int t = st * m + j;
            if (t < p.piece) sG[t] += base;
        }
        scaler_sync();
        const float gend = sG[p.piece - 1];
        if (leader) p.a[out] = gend;

        // two threads per token: thread `half` owns the token's line in atom `half`
        const int tok = st >> 1, half = st & 1;
        const uint32_t roff = (tok >> 3) * 1024 + (tok & 7) * 128;
        float e_next = eta_h[tok];
        bool ok = true;
        for (int i = 0; i < nst; ++i) {
            const int s = i % kStages;
            bool failed = false;
            if (leader && !tc::mbar_wait(&bars[P_FULL + s], (i / kStages) & 1, abort_flag, p.wait_budget)) {
                *abort_flag = 1;
                failed = true;
            }
            if (scaler_sync_or(failed)) {
                ok = false;
                break;
            }
            uint8_t *xa = sm + s * kStage + half * 8192;
            uint8_t *ya = xa + 16384;
            if (i == 0 && t0 == 0 && tok == 0 && p.k_prev && !p.same_step) {
                // x of the first token is the key cached before the sequence (row 0 is not permuted)
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    reinterpret_cast<const __nv_bfloat16 *>(p.k_prev) + (size_t)head * D + 64 * half);
#pragma unroll
                for (int c = 0; c < 8; ++c) reinterpret_cast<uint4 *>(xa)[c] = src[c];
            }
            const float e = e_next;
            if (i + 1 < nst) e_next = eta_h[(i + 1) * kPBlk + tok];
            // chunk c ^ (tok % 8) at step c: the eight rows of a 1024-byte group start their walk
            // on eight different 16-byte positions, so a warp's loads spread over all 32 banks
            const uint4 *xr = reinterpret_cast<const uint4 *>(xa + roff);
            float nrm = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 u = xr[c ^ (tok & 7)];
                nrm = sumsq_bf16x2(u.x, nrm);
                nrm = sumsq_bf16x2(u.y, nrm);
                nrm = sumsq_bf16x2(u.z, nrm);
                nrm = sumsq_bf16x2(u.w, nrm);
            }
            nrm += __shfl_xor_sync(0xffffffffu, nrm, 1);
            const float w = step_size(e, nrm, p.eps) * exp2f(fminf(gend - sG[i * kPBlk + tok], 0.f));
            uint4 *yr = reinterpret_cast<uint4 *>(ya + roff);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 u = yr[c ^ (tok & 7)];
                u.x = scale_bf16x2(u.x, w);
                u.y = scale_bf16x2(u.y, w);
                u.z = scale_bf16x2(u.z, w);
                u.w = scale_bf16x2(u.w, w);
                yr[c ^ (tok & 7)] = u;
            }
            tc::fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(&bars[P_SCALED + s]);
        }
        if (ok) {
            bool failed = false;
            if (leader && !tc::mbar_wait(&bars[P_DONE], 0, abort_flag, p.wait_budget)) {
                *abort_flag = 1;
                failed = true;
            }
            ok = !scaler_sync_or(failed);
        }
        if (ok) {
            // TMEM lane = d_v row, column = d_k: warp w reads lanes 32 (w % 4) ..
            tc::fence_after_sync();
            const int qd = warp & 3, row = 32 * qd + lane;
            const uint32_t ta = tbase + ((uint32_t)(32 * qd) << 16);
            float *Dr = p.D + (out * D + row) * D;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float v[32];
                tc::tmem_ld32(ta + 32 * cb, v);
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(Dr + 32 * cb + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && *abort_flag) set_error(p.err, kDevErrTimeout);
    if (warp == 1) tc::tmem_dealloc(tbase, kPCols);
}

// grid (16, heads) x 256 threads: each thread carries 4 consecutive entries of one head's
// 128 x 128 state through the pieces in order; the increments of four pieces are loaded
// before they are applied, so their loads overlap.
__global__ void __launch_bounds__(256) seg_scan_kernel(ScanParams p) {
    constexpr int E = 128 * 128;
    const int head = blockIdx.y;
    const int e = (blockIdx.x * 256 + threadIdx.x) * 4;
    float4 S = p.S0 ? *reinterpret_cast<const float4 *>(p.S0 + (size_t)head * E + e) : make_float4(0.f, 0.f, 0.f, 0.f);
    // pieces read: all of them when the final state is wanted, else all but the last segment's
    const int np = (p.S_out ? p.nseg : p.nseg - 1) * p.pps;
    const size_t pbase = (size_t)head * p.ptot;
    for (int pc0 = 0; pc0 < np; pc0 += 4) {
        float4 d[4];
        float f[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (pc0 + u < np) {
                d[u] = *reinterpret_cast<const float4 *>(p.D + (pbase + pc0 + u) * E + e);
                f[u] = exp2f(fminf(p.a[pbase + pc0 + u], 0.f));
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int pc = pc0 + u;
            if (pc < np) {
                if (pc % p.pps == 0)   // first piece of segment pc / pps: its starting state
                    *reinterpret_cast<float4 *>(p.Sinit + ((size_t)head * p.nseg + pc / p.pps) * E + e) = S;
                S = make_float4(fmaf(f[u], S.x, d[u].x), fmaf(f[u], S.y, d[u].y), fmaf(f[u], S.z, d[u].z),
                                fmaf(f[u], S.w, d[u].w));
            }
        }
    }
    if (p.S_out)
        *reinterpret_cast<float4 *>(p.S_out + (size_t)head * E + e) = S;
    else   // the last segment's pieces were not read: S is its starting state
        *reinterpret_cast<float4 *>(p.Sinit + ((size_t)head * p.nseg + p.nseg - 1) * E + e) = S;
    if (blockIdx.x == 0) {
        // key rows are 128 bf16 = 16 x 16 bytes: thread (r, c) copies chunk c of rows r, r + 16, ..
        const int c = threadIdx.x & 15, r = threadIdx.x >> 4;
        const uint4 *k = reinterpret_cast<const uint4 *>(p.k);
        if (p.kp) {
            for (int sg = r; sg < p.nseg; sg += 16) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (sg > 0)
                    v = k[((size_t)head * p.T + (size_t)sg * p.L - 1) * 16 + c];
                else if (p.k_prev)
                    v = reinterpret_cast<const uint4 *>(p.k_prev)[(size_t)head * 16 + c];
                reinterpret_cast<uint4 *>(p.kp)[((size_t)head * p.nseg + sg) * 16 + c] = v;
            }
        }
        if (p.k_last && r == 0)
            reinterpret_cast<uint4 *>(p.k_last)[(size_t)head * 16 + c] = k[((size_t)head * p.T + p.T - 1) * 16 + c];
    }
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace: D per piece | log2 decay per piece | state at each segment start | cached key per segment.
struct SegLayout {
    size_t oD, oA, oS, oK, bytes;
};

SegLayout seg_layout(long long heads, int nseg, int ptot) {
    SegLayout l;
    l.oD = 0;
    l.oA = up256((size_t)heads * ptot * kStateBytes);
    l.oS = l.oA + up256((size_t)heads * ptot * sizeof(float));
    l.oK = l.oS + (size_t)heads * nseg * kStateBytes;
    l.bytes = l.oK + up256((size_t)heads * nseg * 128 * 2);
    return l;
}

}  // namespace

SegPlan seg_plan(const ChunkParams &p, int num_sms) {
    SegPlan s;
    // one pair per step only: the state pass writes each token's own pair (a window would need the
    // pairs of the tokens before a piece as well)
    if (p.regression || p.window != 1 || !chunk_ws_supported(p) || p.T % kPBlk != 0) return s;
    const long long heads = (long long)p.B * p.H;
    const int nblk = p.T / kPBlk;
    int best = 1;
    for (int n = 2; n <= nblk / kMinSegBlocks; ++n)
        if (nblk % n == 0 && heads * n <= num_sms) best = n;
    if (best < 2) return s;
    s.nseg = best;
    s.L = p.T / best;
    const int bps = s.L / kPBlk;
    int pb = 1;
    for (int d = 1; d <= bps && d <= kMaxPieceBlocks; ++d)
        if (bps % d == 0) pb = d;
    s.piece = pb * kPBlk;
    s.bytes = seg_layout(heads, s.nseg, p.T / s.piece).bytes;
    return s;
}

cudaError_t launch_chunk_seg(const ChunkParams &p, const SegPlan &pl, void *workspace, cudaStream_t stream) {
    const long long heads = (long long)p.B * p.H;
    const int ptot = p.T / pl.piece;               // pieces per head
    const int pps = pl.L / pl.piece;               // pieces per segment
    const int pneed = p.S_out ? ptot : ptot - pps; // the last segment's pieces only feed the final state
    const SegLayout l = seg_layout(heads, pl.nseg, ptot);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *D = reinterpret_cast<float *>(ws + l.oD);
    float *a = reinterpret_cast<float *>(ws + l.oA);
    float *Sinit = reinterpret_cast<float *>(ws + l.oS);
    void *kp = ws + l.oK;

    CUtensorMap mK, mV;
    if (!map_head_rows(&mK, p.k, p.T, heads, 64) || !map_head_rows(&mV, p.v, p.T, heads, 64))
        return cudaErrorInvalidValue;
    PieceParams pp{};
    pp.T = p.T; pp.piece = pl.piece; pp.pneed = pneed; pp.ptot = ptot;
    pp.same_step = p.same_step; pp.k_prev = p.k_prev;
    pp.alpha = p.alpha; pp.eta = p.eta; pp.eps = p.eps;
    pp.D = D; pp.a = a; pp.err = p.err;
    pp.wait_budget = p.wait_budget; pp.dbg_stall_block = p.dbg_stall_block;
    cudaError_t e = cudaFuncSetAttribute(seg_piece_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPSmem);
    if (e != cudaSuccess) return e;
    seg_piece_kernel<<<(unsigned)(heads * pneed), kPThreads, kPSmem, stream>>>(mK, mV, pp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    ScanParams sp{};
    sp.nseg = pl.nseg; sp.pps = pps; sp.ptot = ptot; sp.L = pl.L; sp.T = p.T;
    sp.k = p.k; sp.k_prev = p.k_prev; sp.S0 = p.S0; sp.D = D; sp.a = a;
    sp.Sinit = Sinit; sp.S_out = p.S_out; sp.kp = p.same_step ? nullptr : kp; sp.k_last = p.k_last;
    seg_scan_kernel<<<dim3(16, (unsigned)heads), 256, 0, stream>>>(sp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    ChunkParams c = p;
    c.H = p.H * pl.nseg;
    c.T = pl.L;
    c.S0 = Sinit;
    c.k_prev = p.same_step ? nullptr : kp;
    c.S_out = nullptr;
    c.k_last = nullptr;
    return launch_chunk_ws(c, stream);
}

}  // namespace falcon
