// api.cu -- the C ABI of libfalcon (declared in include/falcon.h): host-side
// argument checks, kernel selection and status codes. No allocation happens
// here; every buffer belongs to the caller.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/falcon.h"
#include "common.cuh"
#include "launch.h"

namespace falcon {

// Device error word shared by all kernels of the library (per device).
__device__ int g_dev_error = 0;

namespace {

// One-shot stall armed by falcon_debug_stall_next_call for the next chunk call of this thread.
struct DebugStall {
    bool armed = false;
    int block = -1;
    long long budget = kDefaultWaitBudget;
};
thread_local DebugStall g_stall;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int *g_err_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

// Resolves, once per device, the device address of the error word and the SM
// count. Returns false when the current device cannot be queried.
bool device_info(int **err, int *sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_err_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_dev_error) != cudaSuccess) return false;
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
        g_err_ptr[dev] = static_cast<int *>(ptr);
        g_num_sms[dev] = n;
    }
    *err = g_err_ptr[dev];
    *sms = g_num_sms[dev];
    return true;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int base_rule(int r) { return r & ~FALCON_SAME_STEP; }
bool same_step(int r) { return (r & FALCON_SAME_STEP) != 0; }
bool rule_valid(int r) { return base_rule(r) >= FALCON_RULE_1 && base_rule(r) <= FALCON_RULE_2A; }
bool is_regression(int r) {
    return base_rule(r) == FALCON_RULE_1 || base_rule(r) == FALCON_RULE_3 || base_rule(r) == FALCON_RULE_2;
}
bool is_per_column(int r) { return base_rule(r) == FALCON_RULE_2 || base_rule(r) == FALCON_RULE_2A; }
bool is_windowed(int r) { return base_rule(r) == FALCON_RULE_3 || base_rule(r) == FALCON_RULE_3A; }

// Checks shared by the two sequence entry points.
falcon_status_t check_seq_args(const falcon_args_t *a) {
    if (!a) return FALCON_ERR_INVALID_ARG;
    if (!rule_valid(a->rule)) return FALCON_ERR_INVALID_ARG;
    if (a->io_dtype != FALCON_F32 && a->io_dtype != FALCON_BF16) return FALCON_ERR_INVALID_ARG;
    if (a->B < 0 || a->H < 0 || a->T < 0 || a->dk <= 0 || a->dv <= 0) return FALCON_ERR_INVALID_ARG;
    if (!(a->eps >= 0.f) || !isfinite(a->eps)) return FALCON_ERR_INVALID_ARG;
    if (is_windowed(a->rule) && a->window < 1) return FALCON_ERR_INVALID_ARG;
    const long long bh = (long long)a->B * a->H;
    if (bh > 0x7fffffffLL) return FALCON_ERR_UNSUPPORTED;
    const long long elems = bh * (long long)a->T * (a->dk > a->dv ? a->dk : a->dv);
    if (elems > (1LL << 50)) return FALCON_ERR_UNSUPPORTED;
    if (bh * a->T > 0) {
        if (!a->q || !a->k || !a->v || !a->alpha || !a->eta || !a->o) return FALCON_ERR_INVALID_ARG;
        if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->o))
            return FALCON_ERR_INVALID_ARG;
        if (!aligned4(a->alpha) || !aligned4(a->eta)) return FALCON_ERR_INVALID_ARG;
    }
    if (a->S0 && !aligned16(a->S0)) return FALCON_ERR_INVALID_ARG;
    if (a->S_out && !aligned16(a->S_out)) return FALCON_ERR_INVALID_ARG;
    if (a->k_prev && !aligned16(a->k_prev)) return FALCON_ERR_INVALID_ARG;
    if (a->k_last && !aligned16(a->k_last)) return FALCON_ERR_INVALID_ARG;
    if (is_per_column(a->rule) && ((a->n0 && !aligned4(a->n0)) || (a->n_out && !aligned4(a->n_out))))
        return FALCON_ERR_INVALID_ARG;
    return FALCON_OK;
}

bool dim_supported_chunk(int d) { return d == 32 || d == 64 || d == 128; }

// Value-slice width per CTA: the widest slice that still gives about one CTA
// per SM; narrower slices add CTAs (parallelism) at the cost of repeating the
// key-side work of each block once per slice.
int pick_value_slice(long long bh, int dv, int num_sms) {
    const int cand[4] = {128, 64, 32, 16};
    int best = 16;
    for (int i = 0; i < 4; ++i) {
        const int dvs = cand[i];
        if (dvs > dv || dv % dvs) continue;
        if (bh * (dv / dvs) * 4 >= (long long)num_sms * 3) return dvs;
        best = dvs;
    }
    return best;
}

// Launch parameters of the chunk-parallel pass from checked arguments.
ChunkParams chunk_params(const falcon_args_t *a) {
    ChunkParams p{};
    p.B = a->B; p.H = a->H; p.T = a->T; p.dk = a->dk; p.dv = a->dv;
    p.window = is_windowed(a->rule) ? a->window : 1;
    p.tok_per_blk = a->chunk / p.window;
    p.regression = is_regression(a->rule);
    p.same_step = same_step(a->rule);
    p.io_bf16 = a->io_dtype == FALCON_BF16;
    p.q = a->q; p.k = a->k; p.v = a->v; p.k_prev = a->k_prev;
    p.alpha = a->alpha; p.eta = a->eta; p.S0 = a->S0; p.eps = a->eps;
    p.o = a->o; p.k_last = a->k_last; p.S_out = a->S_out;
    p.wait_budget = kDefaultWaitBudget;
    p.dbg_stall_block = -1;
    return p;
}

}  // namespace

cudaError_t launch_chunk_dk32(const ChunkParams &p, int dvs, cudaStream_t s);
cudaError_t launch_chunk_dk64(const ChunkParams &p, int dvs, cudaStream_t s);
cudaError_t launch_chunk_dk128(const ChunkParams &p, int dvs, cudaStream_t s);

cudaError_t launch_chunk(const ChunkParams &p, int num_sms, cudaStream_t s) {
    if (chunk_ws_supported(p)) return launch_chunk_ws(p, s);
    const int dvs = pick_value_slice((long long)p.B * p.H, p.dv, num_sms);
    switch (p.dk) {
        case 32: return launch_chunk_dk32(p, dvs, s);
        case 64: return launch_chunk_dk64(p, dvs, s);
        case 128: return launch_chunk_dk128(p, dvs, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace falcon

using namespace falcon;

extern "C" {

size_t falcon_workspace_size(const falcon_args_t *a) {
    if (!a || check_seq_args(a) != FALCON_OK) return 0;
    if (is_per_column(a->rule)) return 0;
    if (a->io_dtype != FALCON_BF16) return 0;
    if (!dim_supported_chunk(a->dk) || !dim_supported_chunk(a->dv)) return 0;
    if (a->chunk != 16 && a->chunk != 32 && a->chunk != 64) return 0;
    if ((long long)a->B * a->H == 0) return 0;
    ChunkParams p = chunk_params(a);
    int sms = 0;
    if (!device_info(&p.err, &sms)) return 0;
    const size_t seg = seg_plan(p, sms).bytes;
    return seg ? seg : chunk_tile_bytes(p);
}

falcon_status_t falcon_fwd_chunk(const falcon_args_t *a, void *workspace, size_t workspace_bytes,
                                 falcon_stream_t stream) {
    falcon_status_t st = check_seq_args(a);
    if (st != FALCON_OK) return st;
    // The chunk form's products take bf16 tensor-core operands; fp32 inputs would be held to a
    // bf16 error bound, so fp32-accurate work goes through falcon_fwd_recurrent instead.
    if (a->io_dtype != FALCON_BF16) return FALCON_ERR_UNSUPPORTED;
    if (is_per_column(a->rule)) return FALCON_ERR_UNSUPPORTED;   // Falcon-2/2A: falcon_fwd_recurrent
    if (!dim_supported_chunk(a->dk) || !dim_supported_chunk(a->dv)) return FALCON_ERR_UNSUPPORTED;
    if (a->chunk != 16 && a->chunk != 32 && a->chunk != 64) return FALCON_ERR_UNSUPPORTED;
    const int w = is_windowed(a->rule) ? a->window : 1;
    if (w > a->chunk) return FALCON_ERR_UNSUPPORTED;
    if ((long long)a->B * a->H == 0) return FALCON_OK;

    ChunkParams p = chunk_params(a);
    if (g_stall.armed) {
        p.dbg_stall_block = g_stall.block;
        p.wait_budget = g_stall.budget;
        g_stall = DebugStall{};
    }
    int sms = 0;
    if (!device_info(&p.err, &sms)) return FALCON_ERR_CUDA;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const SegPlan plan = seg_plan(p, sms);
    if (plan.nseg > 1) {
        if (!workspace || workspace_bytes < plan.bytes) return FALCON_ERR_WORKSPACE;
        if (!aligned16(workspace)) return FALCON_ERR_INVALID_ARG;
        return launch_chunk_seg(p, plan, workspace, s) == cudaSuccess ? FALCON_OK : FALCON_ERR_CUDA;
    }
    // Regression rules: the two-pass path when the workspace holds every block's T tiles, the
    // single-kernel path otherwise (NULL or a smaller workspace is not an error here).
    const size_t tile_bytes = chunk_tile_bytes(p);
    if (tile_bytes > 0 && workspace && workspace_bytes >= tile_bytes) {
        if (!aligned16(workspace)) return FALCON_ERR_INVALID_ARG;
        p.tiles = workspace;
    }
    return launch_chunk(p, sms, s) == cudaSuccess ? FALCON_OK : FALCON_ERR_CUDA;
}

falcon_status_t falcon_fwd_recurrent(const falcon_args_t *a, falcon_stream_t stream) {
    falcon_status_t st = check_seq_args(a);
    if (st != FALCON_OK) return st;
    if (a->dk > 128 || a->dv > 128) return FALCON_ERR_UNSUPPORTED;
    const int w = is_windowed(a->rule) ? a->window : 1;
    if (w > 64) return FALCON_ERR_UNSUPPORTED;
    if ((long long)a->B * a->H == 0) return FALCON_OK;

    RecParams p{};
    p.B = a->B; p.H = a->H; p.T = a->T; p.dk = a->dk; p.dv = a->dv; p.window = w;
    p.regression = is_regression(a->rule);
    p.same_step = same_step(a->rule);
    p.per_column = is_per_column(a->rule);
    p.io_bf16 = a->io_dtype == FALCON_BF16;
    p.q = a->q; p.k = a->k; p.v = a->v; p.k_prev = a->k_prev;
    p.alpha = a->alpha; p.eta = a->eta; p.S0 = a->S0; p.eps = a->eps;
    p.o = a->o; p.k_last = a->k_last; p.S_out = a->S_out;
    p.n0 = p.per_column ? a->n0 : nullptr;
    p.n_out = p.per_column ? a->n_out : nullptr;
    int sms = 0;
    if (!device_info(&p.err, &sms)) return FALCON_ERR_CUDA;
    return launch_recurrent(p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? FALCON_OK
                                                                                     : FALCON_ERR_CUDA;
}

namespace {

// The forward arguments of a backward call (its outputs may be absent) and the backward limits.
falcon_status_t check_bwd_args(const falcon_args_t *a) {
    if (!a) return FALCON_ERR_INVALID_ARG;
    falcon_args_t b = *a;
    if (!b.o) b.o = const_cast<void *>(b.q);   // o is not read by the backward pass (only checked)
    b.S_out = nullptr;
    b.k_last = nullptr;
    falcon_status_t st = check_seq_args(&b);
    if (st != FALCON_OK) return st;
    if (is_per_column(a->rule)) return FALCON_ERR_UNSUPPORTED;
    if (a->dk > 128 || a->dv > 128) return FALCON_ERR_UNSUPPORTED;
    const int w = is_windowed(a->rule) ? a->window : 1;
    if (w > 8) return FALCON_ERR_UNSUPPORTED;   // the step inputs held in registers
    if (bwd_smem_bytes(a->dk, a->dv, w) > 232448) return FALCON_ERR_UNSUPPORTED;
    return FALCON_OK;
}

}  // namespace

size_t falcon_bwd_workspace_size(const falcon_args_t *a) {
    if (check_bwd_args(a) != FALCON_OK) return 0;
    if ((long long)a->B * a->H * a->T == 0) return 0;
    return bwd_workspace_bytes(a->B, a->H, a->T, a->dk, a->dv, nullptr);
}

falcon_status_t falcon_bwd_recurrent(const falcon_args_t *a, const falcon_grads_t *g, void *workspace,
                                     size_t workspace_bytes, falcon_stream_t stream) {
    falcon_status_t st = check_bwd_args(a);
    if (st != FALCON_OK) return st;
    if (!g) return FALCON_ERR_INVALID_ARG;
    const long long bh = (long long)a->B * a->H;
    if (bh * a->T == 0) return FALCON_OK;
    if (!g->dO || !g->dq || !g->dk || !g->dv || !g->dalpha || !g->deta) return FALCON_ERR_INVALID_ARG;
    const void *ptrs[] = {g->dO, g->dS_T, g->dq, g->dk, g->dv, g->dalpha, g->deta, g->dS0, g->dk_prev};
    for (const void *q : ptrs)
        if (q && !aligned4(q)) return FALCON_ERR_INVALID_ARG;
    int seg = 1;
    const size_t need = bwd_workspace_bytes(a->B, a->H, a->T, a->dk, a->dv, &seg);
    if (!workspace || workspace_bytes < need) return FALCON_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FALCON_ERR_INVALID_ARG;

    BwdParams p{};
    p.B = a->B; p.H = a->H; p.T = a->T; p.dk = a->dk; p.dv = a->dv;
    p.window = is_windowed(a->rule) ? a->window : 1;
    p.seg = seg;
    p.regression = is_regression(a->rule);
    p.io_bf16 = a->io_dtype == FALCON_BF16;
    p.same_step = same_step(a->rule);
    p.q = a->q; p.k = a->k; p.v = a->v; p.k_prev = a->k_prev;
    p.alpha = a->alpha; p.eta = a->eta; p.S0 = a->S0; p.eps = a->eps;
    p.dO = g->dO; p.dS_T = g->dS_T;
    p.dq = g->dq; p.dk_out = g->dk; p.dv_out = g->dv; p.dalpha = g->dalpha; p.deta = g->deta;
    p.dS0 = g->dS0; p.dk_prev = g->dk_prev;
    p.ws = static_cast<float *>(workspace);
    int *err = nullptr;
    int sms = 0;
    if (!device_info(&err, &sms)) return FALCON_ERR_CUDA;
    return launch_bwd_recurrent(p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? FALCON_OK
                                                                                         : FALCON_ERR_CUDA;
}

falcon_status_t falcon_decode_step(int rule, int io_dtype, int N, int H, int dk, int dv, float *S,
                                   void *k_prev, const void *q, const void *k, const void *v,
                                   const float *alpha, const float *eta, float eps, void *o,
                                   falcon_stream_t stream) {
    if (!rule_valid(rule)) return FALCON_ERR_INVALID_ARG;
    if (io_dtype != FALCON_F32 && io_dtype != FALCON_BF16) return FALCON_ERR_INVALID_ARG;
    if (N < 0 || H < 0 || dk <= 0 || dv <= 0) return FALCON_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !isfinite(eps)) return FALCON_ERR_INVALID_ARG;
    if (is_windowed(rule) || is_per_column(rule)) return FALCON_ERR_UNSUPPORTED;
    if (dk != 32 && dk != 64 && dk != 128) return FALCON_ERR_UNSUPPORTED;
    if (dv > 256) return FALCON_ERR_UNSUPPORTED;
    const long long nh = (long long)N * H;
    if (nh > 0x7fffffffLL) return FALCON_ERR_UNSUPPORTED;
    if (nh == 0) return FALCON_OK;
    if (!S || !k_prev || !q || !k || !v || !alpha || !eta || !o) return FALCON_ERR_INVALID_ARG;
    if (!aligned16(S) || !aligned16(k_prev) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
        !aligned16(o) || !aligned4(alpha) || !aligned4(eta))
        return FALCON_ERR_INVALID_ARG;

    DecodeParams p{};
    p.N = N; p.H = H; p.dk = dk; p.dv = dv;
    p.regression = is_regression(rule);
    p.same_step = same_step(rule);
    p.io_bf16 = io_dtype == FALCON_BF16;
    p.S = S; p.k_prev = k_prev; p.q = q; p.k = k; p.v = v;
    p.alpha = alpha; p.eta = eta; p.eps = eps; p.o = o;
    int sms = 0;
    if (!device_info(&p.err, &sms)) return FALCON_ERR_CUDA;
    return launch_decode(p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? FALCON_OK
                                                                                  : FALCON_ERR_CUDA;
}

const char *falcon_status_string(falcon_status_t s) {
    switch (s) {
        case FALCON_OK: return "ok";
        case FALCON_ERR_INVALID_ARG: return "invalid argument";
        case FALCON_ERR_UNSUPPORTED: return "unsupported shape or option";
        case FALCON_ERR_WORKSPACE: return "workspace too small";
        case FALCON_ERR_CUDA: return "CUDA error";
        case FALCON_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

falcon_status_t falcon_check_device_errors(falcon_stream_t stream) {
    int *err = nullptr;
    int sms = 0;
    if (!device_info(&err, &sms)) return FALCON_ERR_CUDA;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return FALCON_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FALCON_ERR_CUDA;
    if (h != 0) {
        const int zero = 0;
        if (cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return FALCON_ERR_CUDA;
    }
    if (h == kDevErrTimeout) return FALCON_ERR_TIMEOUT;
    if (h != 0) return FALCON_ERR_INVALID_ARG;
    return FALCON_OK;
}

falcon_status_t falcon_debug_stall_next_call(int block, long long wait_budget_cycles) {
    if (block < 0 || wait_budget_cycles < 10000 || wait_budget_cycles > kDefaultWaitBudget)
        return FALCON_ERR_INVALID_ARG;
    g_stall.armed = true;
    g_stall.block = block;
    g_stall.budget = wait_budget_cycles;
    return FALCON_OK;
}

int falcon_version(void) { return 100; }

}  // extern "C"
