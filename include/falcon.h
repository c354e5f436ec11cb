/*
 * falcon.h -- C ABI of libfalcon, the forward pass of the Falcon fast-weight
 * memory on NVIDIA B200 (sm_100a).
 *
 * The method ("Fast Weight Attention for Continual Learning", authors'
 * abstract): every head keeps a state S of d_v x d_k numbers. At step t the
 * state is written with the prefix-aligned pair (x_t, y_t) = (phi(k_{t-1}), v_t)
 * by a gated, normalised first-order update, and it is read after the write:
 * o_t = S_t q_t. phi is the identity here.
 *
 *   Falcon-1  (scalar NLMS, squared-error regression):
 *       Sbar = alpha_t S_{t-1};  beta_t = eta_t / (||x_t||^2 + eps)
 *       S_t  = Sbar - beta_t (Sbar x_t - y_t) x_t^T
 *   Falcon-3  (sliding-window mini-batch over the last w pairs, one step):
 *       beta_t = eta_t / (sum_{j in W_t} ||x_j||^2 + eps)
 *       S_t  = Sbar - beta_t sum_{j in W_t} (Sbar x_j - y_j) x_j^T
 *   Falcon-1A / Falcon-3A (negative inner-product objective):
 *       S_t  = Sbar + beta_t sum_{j in W_t} y_j x_j^T
 *   Falcon-2 / Falcon-2A (the per-column extension; a reading of the pages, which
 *   name it without equations): column c of S keeps the running energy of its key
 *   coordinate, n_{t,c} = alpha_t n_{t-1,c} + x_{t,c}^2, and the step is the NLMS
 *   step in the metric D = diag(1 / (n_c + eps)):
 *       z_t = eta_t D x_t / (x_t^T D x_t + eps)
 *       Falcon-2:  S_t = Sbar - (Sbar x_t - y_t) z_t^T     Falcon-2A: S_t = Sbar + y_t z_t^T
 * The step size is the Kaczmarz/NLMS one (Kaczmarz Linear Attention abstract,
 * thelatestinai.com page "Fast Weight Attention for Continual Learning").
 * W_t = {max(1, t-w+1) .. t} (1-based). x_1 = k_prev when a cache is given,
 * else 0 (no write at the first step). A pair whose denominator
 * ||x||^2 + eps is 0 writes nothing (beta = 0). alpha in (0, 1] and eta >= 0
 * are preconditions; they are not checked per element.
 *
 * Conventions shared by every entry point:
 *  - All tensors are dense, row-major, contiguous, in DEVICE memory owned by
 *    the caller. The library never allocates, frees or synchronises (except
 *    falcon_check_device_errors, which synchronises the given stream).
 *  - q, k: (B,H,T,d_k); v, o: (B,H,T,d_v); alpha, eta: (B,H,T) fp32;
 *    S0, S_out: (B,H,d_v,d_k) fp32 with S[i][c] the weight from key
 *    coordinate c to value coordinate i; k_prev, k_last: (B,H,d_k).
 *    q, k, v, o, k_prev and k_last share io_dtype (fp32 or bf16).
 *  - Every pointer must be 16-byte aligned except alpha and eta (4 bytes).
 *  - Calls are asynchronous on `stream` (0 = the legacy default stream).
 *    Shape, pointer, alignment and dtype checks run on the host before any
 *    launch; a failed check launches nothing and returns
 *    FALCON_ERR_INVALID_ARG or FALCON_ERR_UNSUPPORTED.
 *  - A launch failure returns FALCON_ERR_CUDA (the CUDA error is left for
 *    cudaGetLastError to report).
 *  - No exception crosses this boundary.
 */
#ifndef FALCON_H_
#define FALCON_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FALCON_API __attribute__((visibility("default")))
#else
#define FALCON_API
#endif

/* Same underlying type as cudaStream_t. */
typedef struct CUstream_st *falcon_stream_t;

typedef enum {
    FALCON_OK = 0,
    FALCON_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, bad enum   */
    FALCON_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement      */
    FALCON_ERR_WORKSPACE = 3,   /* workspace smaller than falcon_workspace_size()    */
    FALCON_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed              */
    FALCON_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up                */
} falcon_status_t;

typedef enum {
    FALCON_RULE_1 = 1,  /* Falcon-1: scalar NLMS                                  */
    FALCON_RULE_1A = 2, /* Falcon-1A: normalised additive (inner-product) write   */
    FALCON_RULE_3 = 3,  /* Falcon-3: sliding-window mini-batch (window w)         */
    FALCON_RULE_3A = 4, /* Falcon-3A: windowed inner-product write (window w)     */
    FALCON_RULE_2 = 5,  /* Falcon-2: per-column normalised NLMS (see below)       */
    FALCON_RULE_2A = 6  /* Falcon-2A: its inner-product counterpart               */
} falcon_rule_t;

/*
 * Flag OR-ed into a rule value (the `rule` field, or the `rule` argument of
 * falcon_decode_step): write the same-step pair (k_t, v_t) at step t, the
 * association of Kaczmarz Linear Attention (thelatestinai.com page of "Fast Weight
 * Attention for Continual Learning", KLA abstract), instead of the prefix-aligned
 * pair (k_{t-1}, v_t) of the authors' abstract. k_prev is then not used as a key
 * (k_last is still the last key, and the decode step still stores k into k_prev).
 */
#define FALCON_SAME_STEP 0x100

typedef enum { FALCON_F32 = 0, FALCON_BF16 = 1 } falcon_dtype_t;

/* Arguments of the two sequence entry points. Integer fields hold the enums
 * above. */
typedef struct {
    int rule;           /* falcon_rule_t, optionally | FALCON_SAME_STEP               */
    int io_dtype;       /* falcon_dtype_t of q, k, v, k_prev, k_last and o            */
    int B, H, T;        /* batch, heads, tokens (T >= 0)                              */
    int dk, dv;         /* key/query and value widths                                 */
    const void *q;      /* (B,H,T,dk)                                                 */
    const void *k;      /* (B,H,T,dk)                                                 */
    const void *v;      /* (B,H,T,dv)                                                 */
    const float *alpha; /* (B,H,T) decay gate, preconditions 0 < alpha <= 1           */
    const float *eta;   /* (B,H,T) step gate, precondition eta >= 0                   */
    float eps;          /* >= 0, added to the (window) squared key norm                */
    int window;         /* Falcon-3/3A window w >= 1; ignored by Falcon-1/1A           */
    int chunk;          /* chunk-parallel block: 16, 32 or 64 pseudo-value rows        */
    const float *S0;    /* (B,H,dv,dk) initial state, or NULL for zero                 */
    const void *k_prev; /* (B,H,dk) key cached before this segment, or NULL (x_1 = 0);
                           not read with FALCON_SAME_STEP                              */
    void *o;            /* (B,H,T,dv) output, written                                  */
    float *S_out;       /* (B,H,dv,dk) final state, or NULL                            */
    void *k_last;       /* (B,H,dk) last key (the cache for a continuation), or NULL   */
    const float *n0;    /* Falcon-2/2A: (B,H,dk) running column energies to start from,
                           or NULL for zero; ignored by the other rules                */
    float *n_out;       /* Falcon-2/2A: (B,H,dk) running column energies after the
                           sequence (part of the continuation cache), or NULL          */
} falcon_args_t;

/*
 * Bytes of device workspace falcon_fwd_chunk uses for these arguments on the
 * current device (0 when it uses none). Returns 0 for invalid arguments as
 * well; the call itself reports those. Nonzero in two cases, both described at
 * falcon_fwd_chunk:
 *   - the sequence split of the inner-product rules, which needs it: about
 *     (B*H*T/piece + B*H*nseg) * dv*dk*4 bytes, a few tens of MB for 16 heads of
 *     32768 tokens;
 *   - the two-pass path of the regression rules (Falcon-1, and Falcon-3 at
 *     window 1, 2 or 4, on the dk = dv = 128 bf16 kernel), which is optional:
 *     16 KB per block of 64 / window tokens per head, B*H*ceil(T*window/64)*16384
 *     bytes (134 MB for 128 heads of 4096 tokens at window 1); given less, or
 *     NULL, those rules run in one kernel instead.
 * The caller allocates it (16-byte aligned) and owns it; the call only uses it
 * while its kernels run on `stream`.
 */
FALCON_API size_t falcon_workspace_size(const falcon_args_t *args);

/*
 * falcon_fwd_chunk -- chunk-parallel forward pass with positive-decay
 * renormalisation (authors' abstract of "Fast Weight Attention for Continual
 * Learning"; ai.info overview, section Methodology in Plain English, which
 * describes the blocked form).
 *
 * Per block of pseudo-value rows the kernel forms the decay-weighted key Gram
 * and query-key tiles, solves the unit lower-triangular system of the block
 * (Falcon-1/3), applies it to the residuals against the state carried in from
 * the previous block, writes the block's outputs and passes the fp32 state on.
 * Decay factors are only ever formed as exp(g_i - g_j) with i >= j on a
 * block-local cumulative log decay, so each lies in (0, 1].
 *
 * Supported: Falcon-1/1A/3/3A (Falcon-2/2A return UNSUPPORTED here: they run on
 * falcon_fwd_recurrent); io_dtype FALCON_BF16 only; dk, dv in {32, 64, 128}; chunk in
 * {16, 32, 64}; Falcon-3/3A need 1 <= window <= chunk and process
 * floor(chunk / window) tokens per block. Tensor-core products take the bf16
 * inputs as operands with fp32 accumulation and an fp32 state. FALCON_F32
 * inputs return FALCON_ERR_UNSUPPORTED: bf16 operands could not hold them to an
 * fp32 error bound, so fp32-accurate work goes through falcon_fwd_recurrent.
 *
 * Sequence split (inner-product write, window 1, dk = dv = 128, bf16, chunk 64,
 * T a multiple of 64, and room for nseg >= 2 segments of at least 8 blocks each
 * with B*H*nseg <= the SM count; the largest such nseg dividing T/64 is taken):
 * the additive write has a scalar
 * state transition, so each head is cut into nseg segments of whole blocks;
 * one parallel pass forms every piece's state increment
 * sum_t 2^(G_end - G_t) beta_t y_t x_t^T and its decay, a scan gives the state
 * at each segment start, and the segments then run as heads of their own.
 * The result is the same up to rounding; falcon_workspace_size() says when
 * this path is taken and how much workspace it needs.
 *
 * Two-pass path (regression write, window 1, 2 or 4, dk = dv = 128, bf16, chunk
 * 64, when the workspace holds falcon_workspace_size() bytes): the chunk-local step
 * of a block (its Gram matrix, step sizes, L and T = (I + L)^-1) depends only on
 * the block's keys and gates, so a first launch solves every block of every
 * head at once and leaves its two bf16 T tiles in the workspace; the second
 * launch runs the state recurrence over the blocks and reads them. Both paths
 * do the same arithmetic; with less workspace, or NULL, the single kernel runs.
 *
 * `workspace` may be NULL when falcon_workspace_size() is 0.
 * Errors: INVALID_ARG (also a workspace not 16-byte aligned), UNSUPPORTED,
 * WORKSPACE (NULL or smaller than falcon_workspace_size() where the sequence
 * split needs it), CUDA.
 */
FALCON_API falcon_status_t falcon_fwd_chunk(const falcon_args_t *args, void *workspace,
                                 size_t workspace_bytes, falcon_stream_t stream);

/* Size of the fixed scratch array behind falcon_fwd_chunk_noalloc: 32 MiB. */
#define FALCON_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * falcon_fwd_chunk_noalloc -- falcon_fwd_chunk without a caller-provided
 * workspace, for callers that cannot allocate device memory where they run
 * the forward pass: a plugin that receives raw device pointers from a host
 * runtime with no allocator to offer, a serving loop in which a cudaMalloc
 * (which may synchronise the device) is not acceptable, or a process whose
 * device memory is owned by a pool it does not control. The paper has no
 * counterpart; this is a deployment convenience of this library.
 *
 * Arguments, results and errors are those of falcon_fwd_chunk. Where that call
 * uses workspace (falcon_workspace_size() > 0), this one uses a fixed array of
 * FALCON_NOALLOC_SCRATCH_BYTES in the library's device image instead; every
 * GPU that uses the library holds that array until the process exits. A
 * sequence split that needs more is rejected before anything runs with
 * FALCON_ERR_WORKSPACE (use falcon_fwd_chunk with your own workspace then);
 * the regression rules' two-pass path runs when its tiles fit in the array and
 * their single-kernel path otherwise. The call allocates and frees nothing.
 *
 * The array is reserved on a device no later than the first call there (with
 * lazy module loading, the CUDA default, that first call loads it; with eager
 * loading it is reserved when the library loads). The first call on each device
 * resolves the array's device address (with that device current) and keeps it;
 * make that first call before any stream capture. The kept address does not
 * survive cudaDeviceReset: do not use this entry point on a device after
 * resetting it in the same process. All calls share the one array per device: calls whose kernels can
 * overlap on the GPU (different streams without an ordering between them,
 * several host threads) race on it and give wrong results, so order them, for
 * example on one stream. Nothing in the array needs clearing between calls:
 * each call writes every byte it later reads.
 */
FALCON_API falcon_status_t falcon_fwd_chunk_noalloc(const falcon_args_t *args, falcon_stream_t stream);

/*
 * falcon_fwd_recurrent -- recurrent form (authors' abstract; ai.info overview,
 * section Methodology in Plain English): the literal per-token recurrence
 * with an fp32 state and fp32 arithmetic. One CTA per (b, h) walks t = 1..T.
 * Supported: 1 <= dk, dv <= 128; window <= 64 for Falcon-3/3A; `chunk` is
 * ignored. This is the entry point for Falcon-2/2A (with n0 / n_out).
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
FALCON_API falcon_status_t falcon_fwd_recurrent(const falcon_args_t *args, falcon_stream_t stream);

/*
 * falcon_bwd_recurrent -- gradients of the recurrent form for a loss L, given the
 * upstream gradients of the outputs and of the final state. The pages define the
 * forward rules only (authors' abstract); these are their derivatives, taken step by
 * step backwards through the same per-token recurrence (reverse mode):
 *   U = dL/dS_t (U = dS_T after the last step), then for t = T..1:
 *   U += dO_t q_t^T;  dq_t = S_t^T dO_t;
 *   Falcon-1/3 (r_j = Sbar x_j - y_j):  dbeta = -sum_j r_j^T U x_j;
 *     dy_j = beta U x_j;  dx_j = -beta U^T r_j - beta Sbar^T U x_j;  dSbar = U - beta sum_j U x_j x_j^T
 *   Falcon-1A/3A:  dbeta = sum_j y_j^T U x_j;  dy_j = beta U x_j;  dx_j = beta U^T y_j;  dSbar = U
 *   deta_t = dbeta / (N_t + eps);  dx_j += -2 dbeta beta / (N_t + eps) x_j  (N_t the pairs' squared norms;
 *   nothing flows through beta when N_t + eps = 0);  dalpha_t = <dSbar, S_{t-1}>;  U <- alpha_t dSbar.
 * dx of pair j goes to the key row it was read from (k_{j-1}; k_prev for the first pair, or k_j with
 * FALCON_SAME_STEP), dy to v_j, and dS0 is the final U.
 *
 * `args` is the forward call's (q, k, v, alpha, eta, eps, window, S0, k_prev, rule with the
 * flag); its outputs o, S_out, k_last and chunk are ignored. `grads` (every array fp32, dense,
 * device memory; 4-byte alignment):
 *   dO (B,H,T,dv) required; dS_T (B,H,dv,dk) or NULL (zero);
 *   dq, dk (B,H,T,dk), dv (B,H,T,dv), dalpha, deta (B,H,T) written;
 *   dS0 (B,H,dv,dk) written when not NULL; dk_prev (B,H,dk) written when not NULL and
 *   args->k_prev is given.
 * Workspace: falcon_bwd_workspace_size(args) bytes, 16-byte aligned (the states at the
 * start of every segment of about sqrt(T) steps and one segment of recomputed states,
 * fp32, per slice of 8 value rows of a head). fp32 state and arithmetic; one CTA of 128
 * threads per slice of 8 value rows of a (b, h): the rows of S evolve independently, and the
 * slices add their parts of dq, dk, dalpha, deta and dk_prev to the outputs with atomic adds
 * (so those sums are taken in no fixed order, and their last bits can differ between runs);
 * dv and dS0 rows are each written by one slice.
 * Supported: Falcon-1, 1A, 3, 3A (with or without FALCON_SAME_STEP); 1 <= dk, dv <= 128;
 * windows of up to 8 pairs. Falcon-2/2A return
 * UNSUPPORTED.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
typedef struct {
    const float *dO;
    const float *dS_T;
    float *dq, *dk, *dv;
    float *dalpha, *deta;
    float *dS0;
    float *dk_prev;
} falcon_grads_t;

FALCON_API size_t falcon_bwd_workspace_size(const falcon_args_t *args);
FALCON_API falcon_status_t falcon_bwd_recurrent(const falcon_args_t *args, const falcon_grads_t *grads,
                                                void *workspace, size_t workspace_bytes,
                                                falcon_stream_t stream);

/*
 * falcon_decode_step -- one token of the recurrence for N independent
 * sequences x H heads, in place: the recurrent form applied to a single step,
 * the incremental state update that the ai.info overview of "Fast Weight
 * Attention for Continual Learning" lists for streaming inference (section
 * Why This Matters).
 *
 *   x = k_prev (x = k with FALCON_SAME_STEP); beta = eta / (||x||^2 + eps); Sbar = alpha S
 *   Falcon-1:  S <- Sbar - beta (Sbar x - v) x^T     Falcon-1A: S <- Sbar + beta v x^T
 *   o = S q;   k_prev <- k
 *
 * S (N,H,dv,dk) fp32 and k_prev (N,H,dk) io_dtype are read and written in
 * place; q, k (N,H,dk), v (N,H,dv) io_dtype; alpha, eta (N,H) fp32;
 * o (N,H,dv) io_dtype is written. The buffers of one call must not overlap.
 * Supported: rule Falcon-1 or Falcon-1A (Falcon-3/3A need a window of past
 * pairs and Falcon-2/2A their column energies: both return UNSUPPORTED); dk in
 * {32, 64, 128}; 1 <= dv <= 256.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
FALCON_API falcon_status_t falcon_decode_step(int rule, int io_dtype, int N, int H, int dk, int dv,
                                   float *S, void *k_prev, const void *q, const void *k,
                                   const void *v, const float *alpha, const float *eta,
                                   float eps, void *o, falcon_stream_t stream);

/* Static, NUL-terminated description of a status code (never NULL). */
FALCON_API const char *falcon_status_string(falcon_status_t status);

/*
 * Synchronises `stream`, then reads and clears the library's device error
 * word (set by a kernel that detected an inconsistent launch, or by a bounded
 * wait that gave up). Returns FALCON_OK, FALCON_ERR_TIMEOUT, FALCON_ERR_CUDA
 * (a CUDA error surfaced while synchronising) or FALCON_ERR_INVALID_ARG
 * (a kernel rejected its launch geometry).
 */
FALCON_API falcon_status_t falcon_check_device_errors(falcon_stream_t stream);

/*
 * falcon_debug_stall_next_call -- test hook for the failure path; not for production use.
 * Arms a one-shot stall for the next falcon_fwd_chunk (or falcon_fwd_chunk_noalloc) call
 * made from this host thread: the TMA producer of every tensor-core kernel of that call
 * stops loading at block `block` (0-based 64-row block of each head or segment), and every
 * bounded device-side wait of the call gives up after `wait_budget_cycles` SM clocks
 * instead of about 2^31. A consumer's wait then runs out: the kernel records
 * FALCON_ERR_TIMEOUT in the device error word, waits for its own loads in flight (no load
 * is left pending, none was started for the stalled block), frees its tensor memory and
 * returns, so the context stays usable; falcon_check_device_errors() reports the timeout,
 * the call's outputs are undefined, and the following call runs normally. Calls that run
 * no tensor-core kernel, or that have fewer blocks than `block`, ignore the stall (it is
 * consumed all the same). The kernels' waits are bounded whether or not the hook is used;
 * the hook only lets a test reach that code without faulting or hanging a GPU (the pages
 * have no counterpart).
 * Errors: INVALID_ARG for block < 0 or a budget outside [10^4, 2^31].
 */
FALCON_API falcon_status_t falcon_debug_stall_next_call(int block, long long wait_budget_cycles);

/* Library version, major * 10000 + minor * 100 + patch. */
FALCON_API int falcon_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FALCON_H_ */
