// launch.h -- internal launch interface between the C ABI shell (api.cu) and
// the kernel translation units. Not installed; callers use include/falcon.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace falcon {

struct RecParams {
    int B, H, T, dk, dv, window;  // window = 1 for Falcon-1/1A
    bool regression, io_bf16;
    bool same_step;               // pair (k_t, v_t) instead of (k_{t-1}, v_t)
    bool per_column;              // Falcon-2/2A: write key z = eta D x / (x^T D x + eps)
    const float *n0;              // (B,H,dk) running column energies, or NULL (Falcon-2/2A)
    float *n_out;
    const void *q, *k, *v, *k_prev;
    const float *alpha, *eta, *S0;
    float eps;
    void *o, *k_last;
    float *S_out;
    int *err;
};

struct BwdParams {
    int B, H, T, dk, dv, window;  // window = 1 for Falcon-1/1A
    int seg;                      // steps per checkpointed segment
    bool regression, io_bf16, same_step;
    const void *q, *k, *v, *k_prev;
    const float *alpha, *eta, *S0;
    float eps;
    const float *dO, *dS_T;
    float *dq, *dk_out, *dv_out, *dalpha, *deta, *dS0, *dk_prev;
    float *ws;                    // per head: checkpoints, then one segment of states
};

struct DecodeParams {
    int N, H, dk, dv;
    bool regression, io_bf16;
    bool same_step;  // x = k instead of the cached k_prev
    float *S;
    void *k_prev;
    const void *q, *k, *v;
    const float *alpha, *eta;
    float eps;
    void *o;
    int *err;
};

struct ChunkParams {
    int B, H, T, dk, dv;
    int window;      // pairs per step (1 for Falcon-1/1A)
    int tok_per_blk; // tokens per block; rows per block = tok_per_blk * window <= 64
    bool regression, io_bf16;
    bool same_step;  // pair (k_t, v_t) instead of (k_{t-1}, v_t)
    const void *q, *k, *v, *k_prev;
    const float *alpha, *eta, *S0;
    float eps;
    void *o, *k_last;
    float *S_out;
    int *err;
    // Regression rules on the warp-specialised kernel: when set, a first launch writes the solved
    // T_f and T' tiles of every block here (chunk_tile_bytes) and the chain kernel reads them instead
    // of solving each block itself.
    void *tiles;
    // Bounded waits of the tensor-core kernels give up after wait_budget SM clocks. A test hook
    // (falcon_debug_stall_next_call) shortens it and makes the TMA producers stop loading at
    // block dbg_stall_block, so that the timeout path runs without faulting or hanging the GPU;
    // -1 = no stall.
    long long wait_budget;
    int dbg_stall_block;
};

constexpr long long kDefaultWaitBudget = 1ll << 31;  // SM clocks, about 1 s

size_t recurrent_smem_bytes(int dk, int dv, int window);
cudaError_t launch_recurrent(const RecParams &p, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams &p, cudaStream_t s);
size_t bwd_workspace_bytes(int B, int H, int T, int dk, int dv, int *seg_out);
size_t bwd_smem_bytes(int dk, int dv, int window);
cudaError_t launch_bwd_recurrent(const BwdParams &p, cudaStream_t s);
cudaError_t launch_chunk(const ChunkParams &p, int num_sms, cudaStream_t s);
// Warp-specialised tcgen05 / TMA kernel: d_k = d_v = 128, bf16 I/O, one pair per step, 64-token blocks.
bool chunk_ws_supported(const ChunkParams &p);
cudaError_t launch_chunk_ws(const ChunkParams &p, cudaStream_t s);
// Workspace of the two-pass path of the regression rules (0 where it does not apply).
size_t chunk_tile_bytes(const ChunkParams &p);

// Sequence split of the inner-product rule (seg_state.cu): the segments of each head run
// as heads of their own, started from states that a parallel pass and a scan provide.
struct SegPlan {
    int nseg = 1;       // segments per head (1: no split)
    int L = 0;          // tokens per segment, whole 64-token blocks
    int piece = 0;      // tokens per piece of the state pass; divides L
    size_t bytes = 0;   // device workspace the split needs
};
SegPlan seg_plan(const ChunkParams &p, int num_sms);
cudaError_t launch_chunk_seg(const ChunkParams &p, const SegPlan &plan, void *workspace, cudaStream_t s);

}  // namespace falcon
