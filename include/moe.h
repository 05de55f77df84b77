/*
 * moe.h -- C ABI of libmoe.so, the forward pass of a dropless
 * Mixture-of-Experts layer on one NVIDIA B200 (sm_100a).
 *
 * Symbols follow the course module "Mixture of Experts: routing, sorted
 * dispatch, Switch aux loss, aux-free bias" (sec. 2 symbol table): N tokens,
 * E experts, k experts per token, d_model, d_ff, router W_g, selection bias
 * b_e.  Its sec. 4 interface (topk_ids, dispatch, combine,
 * load_balance_loss, MoE.route / forward / update_bias) maps onto the entry
 * points below.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.  Every tensor pointer is DEVICE memory owned by the caller.  The
 *   library allocates nothing, frees nothing and never synchronises the
 *   host; all work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *   default stream).  Scratch comes from the caller's workspace `ws` of
 *   `ws_bytes` bytes, at least moe_workspace_size(cfg) and 256-byte aligned.
 * Layouts.  Row-major, contiguous:
 *   x         [N, d_model]            dtype
 *   W_g       [E, d_model]            dtype      (z_n = W_g x_n)
 *   W1, W3    [E, d_ff, d_model]      dtype      (row f of W1[e]: hidden unit f)
 *   W2        [E, d_model, d_ff]      dtype      (row c of W2[e]: output c)
 *   b1        [E, d_ff], b2 [E, d_model]  dtype  (optional)
 *   b_e       [E]                     float32
 *   topk_ids  [N, k] int32, topk_w [N, k] float32, probs [N, E] float32
 *   x_sorted, y_sorted [N*k, d_model] dtype
 *   perm, inv_perm [N*k] int32; offsets [E+1] int32; counts [E] int32
 *   Weights are stored output-feature-major (the nn.Linear convention), so
 *   both GEMM operands are contiguous along the reduction dimension.
 * dtype.  MOE_F32 (all fp32) or MOE_BF16 (x, weights, biases, outputs bf16;
 *   router, softmax, gates and every accumulation in fp32).
 * Errors.  Arguments are validated before anything is enqueued; a bad
 *   argument returns MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED /
 *   MOE_ERR_WORKSPACE and launches nothing.  A CUDA launch error returns
 *   MOE_ERR_CUDA (moe_last_error() gives the CUDA message).  Errors found on
 *   the device (an expert id outside [0, E), a device wait that ran out) are
 *   written to the caller's optional `dev_status` int32 word: the first
 *   error code is kept (the word must be 0 before the call; moe_forward
 *   clears it itself).  The library never traps.
 * Limits.  1 <= k <= min(E, 16); E <= 256; d_model and d_ff multiples of 8;
 *   N*k < 2^31; every pointer 16-byte aligned.
 * Threading.  Host-side state is limited to caches filled on first use and
 *   guarded by mutexes: per-device attributes (SM count, shared-memory
 *   opt-ins, occupancy), the driver entry points, and the device address of
 *   moe_dispatch_noalloc's scratch array.  Calls on different streams may run
 *   concurrently with separate workspaces.  The one piece of global DEVICE
 *   state is that scratch array: moe_dispatch_noalloc calls share it (see
 *   there); every other entry point touches only the caller's memory.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef struct CUstream_st *moe_stream_t; /* same type as cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_CUDA = 3,
    MOE_ERR_WORKSPACE = 4,
    MOE_ERR_TIMEOUT = 5,
    MOE_ERR_BAD_EXPERT_ID = 6
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Router table of the course module (sec. 2.1). */
typedef enum {
    MOE_ROUTER_SOFTMAX_TOPK = 0, /* top k of p = softmax(z); w = p, renormalised if norm_topk */
    MOE_ROUTER_TOPK_SOFTMAX = 1, /* top k of z; w = softmax over the chosen logits */
    MOE_ROUTER_SIGMOID = 2       /* top k of sigmoid(z) + b_e; w = sigmoid(z), renormalised if norm_topk */
} moe_router;

typedef enum {
    MOE_ACT_GELU = 0,  /* h = gelu_erf(W1 x + b1); y = W2 h + b2     ("nano-moe" MLP) */
    MOE_ACT_SWIGLU = 1 /* h = silu(W1 x) * (W3 x); y = W2 h (+ b2)   (gated MLP, act="silu") */
} moe_act;

typedef struct {
    int64_t N;            /* tokens (every leading axis flattened) */
    int32_t d_model;
    int32_t d_ff;         /* hidden width of one expert */
    int32_t E;            /* routed experts */
    int32_t k;            /* experts per token */
    int32_t router;       /* moe_router */
    int32_t norm_topk;    /* 1: renormalise the chosen weights to sum to 1 */
    float routed_scaling; /* every weight is multiplied by it (1.0 = off) */
    int32_t act;          /* moe_act */
    int32_t dtype;        /* moe_dtype */
    int32_t d_ff_shared;  /* hidden width of the shared expert; 0 = none */
} moe_config;

/*
 * Weights of the shared expert, the FFN every token passes through besides
 * its k routed experts (course module sec. 2.1: y_n = sum_{e in T_n}
 * w_{n,e} Expert_e(x_n) + Shared(x_n); S shared experts of width f are one
 * FFN of width S f; RustingBrain chapter "Mixture of Experts", sec. 15.4).
 * It has the routed experts' activation and dtype and width cfg->d_ff_shared
 * (Fs): W1 and W3 [Fs, d_model], W2 [d_model, Fs], row-major; b1 [Fs]
 * (GELU only) and b2 [d_model] may be NULL, W3 is SwiGLU only.  Its output
 * carries no gate weight and no routed_scaling.  Device pointers, 16-byte
 * aligned, owned by the caller.
 */
typedef struct {
    const void *W1;
    const void *b1;
    const void *W3;
    const void *W2;
    const void *b2;
} moe_shared_expert;

/* Stage boundaries recorded by moe_forward when stage_events is given. */
#define MOE_STAGE_ROUTE 0    /* router GEMM + scores + top-k + gates */
#define MOE_STAGE_DISPATCH 1 /* counts/offsets/loss/bias rule, scatter, row gather */
#define MOE_STAGE_GEMM1 2    /* x_sorted -> h (first expert GEMM + activation) */
#define MOE_STAGE_GEMM2 3    /* h -> y_sorted (second expert GEMM + bias), then the shared expert's FFN */
#define MOE_STAGE_COMBINE 4  /* weighted sum back in token order */
#define MOE_NUM_STAGES 5

/* Human-readable name of a status code (static string). */
MOE_API const char *moe_status_string(moe_status s);

/* Last CUDA error message seen by a failing call on this host thread. */
MOE_API const char *moe_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
MOE_API int32_t moe_version(void);

/*
 * Bytes of workspace that every entry point below accepts for `cfg` (the
 * largest need, that of moe_forward): per-chunk histograms and partial
 * probability sums, router partial logits, offsets, the GEMM tile tables,
 * perm / inv_perm, x_sorted, the hidden activations h [N*k, d_ff] (or
 * [N, d_ff_shared] if larger), y_sorted and the shared expert's output.
 * Returns 0 for an invalid cfg.
 */
MOE_API size_t moe_workspace_size(const moe_config *cfg);

/*
 * Router: course module sec. 2 (z_n = W_g x_n, p_n = softmax(z_n)) and the
 * sec. 2.1 router table, "ties go to the lowest id"; the sec. 4 topk_ids and
 * MoE.route.  For each token writes the k chosen expert ids, largest
 * selection score first (ties: lowest id), and their weights (times
 * routed_scaling).  b_e (sigmoid router only, may be NULL) enters the
 * selection score only, never the weights (sec. 2.5).  probs [N, E] (may be
 * NULL) receives softmax(z_n) for every router.  bf16 with E <= 32 runs as
 * one streaming kernel (each CTA reads the rows of x of its 32 tokens once,
 * the products on warp-level tensor-core MMAs, the selection fused); bf16
 * with E > 32 keeps the logits (partial sums over d when the reduction is
 * split) in the workspace between the tcgen05 logits kernel and the
 * selection kernel; fp32 runs one CUDA-core kernel.
 */
MOE_API moe_status moe_route(const moe_config *cfg, const void *x, const void *W_g,
                     const float *b_e, int32_t *topk_ids, float *topk_w,
                     float *probs, void *ws, size_t ws_bytes,
                     moe_stream_t stream);

/*
 * Sorted dispatch: course module sec. 2.2 and the sec. 4 dispatch.
 * Assignments a = n*k + j are stably sorted by expert id: perm[i] is the
 * assignment at sorted position i, inv_perm[perm[i]] = i,
 * x_sorted[i] = x[perm[i] / k], counts[e] = assignments to e,
 * offsets[e] = start of expert e's slice (offsets[0] = 0, offsets[E] = N*k).
 * perm, x and x_sorted may be NULL (then that output is skipped).  An
 * expert id outside [0, E) sets MOE_ERR_BAD_EXPERT_ID in dev_status; that
 * assignment is left out of counts and offsets, gets inv_perm = -1 and no
 * row, and every valid assignment keeps its stable position.
 */
MOE_API moe_status moe_dispatch(const moe_config *cfg, const void *x,
                        const int32_t *topk_ids, void *x_sorted, int32_t *perm,
                        int32_t *inv_perm, int32_t *offsets, int32_t *counts,
                        int32_t *dev_status, void *ws, size_t ws_bytes,
                        moe_stream_t stream);

/* Largest ceil(N / 32) * E that moe_dispatch_noalloc accepts (int32 slots of
 * its built-in scratch, 2 MiB): e.g. N <= 65536 tokens with E = 256. */
#define MOE_NOALLOC_DISPATCH_MAX_SLOTS (1 << 19)

/*
 * moe_dispatch without a workspace.  The pages have no counterpart of this
 * entry point; it exists for callers that cannot hand the library any scratch
 * memory: code that runs under a device-memory budget fixed before it starts
 * (a serving process that plans every buffer up front, or a plugin called by
 * a framework that owns the allocator) may not call cudaMalloc at all -- it
 * would break the owner's accounting and can stall the whole device -- and
 * has no spare buffer of moe_workspace_size bytes to pass in.
 *
 * Same arguments, outputs and errors as moe_dispatch, minus ws / ws_bytes.
 * The per-chunk scratch lives in a device array inside libmoe.so
 * (MOE_NOALLOC_DISPATCH_MAX_SLOTS int32, held by every GPU that loads the
 * library until the process exits); a larger problem returns
 * MOE_ERR_WORKSPACE and enqueues nothing.  Nothing is allocated, here or
 * later.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it with the
 * id of the device's context: make that first call before any stream
 * capture.  A call that finds a different context current (after
 * cudaDeviceReset) looks the address up again; so does every call made from
 * a thread on which no context is current yet.  Every call uses the same
 * array, so calls whose work overlaps on the GPU (e.g. on two streams) race:
 * order them.  Each call overwrites all the scratch it later reads, so
 * earlier contents never matter.
 */
MOE_API moe_status moe_dispatch_noalloc(const moe_config *cfg, const void *x,
                                const int32_t *topk_ids, void *x_sorted,
                                int32_t *perm, int32_t *inv_perm,
                                int32_t *offsets, int32_t *counts,
                                int32_t *dev_status, moe_stream_t stream);

/*
 * Expert FFNs over the ragged slices: course module sec. 2.2 ("each expert
 * runs once on its slice"), experts as in moe_act.  Rows
 * offsets[e] .. offsets[e+1]-1 of x_sorted go through expert e and land in
 * the same rows of y_sorted.  b1 (GELU only), W3 (SwiGLU only) and b2 may be
 * NULL where the activation does not use them.  offsets is read on the
 * device (no host synchronisation).
 */
MOE_API moe_status moe_expert_ffn(const moe_config *cfg, const void *x_sorted,
                          const int32_t *offsets, const void *W1,
                          const void *b1, const void *W3, const void *W2,
                          const void *b2, void *y_sorted, int32_t *dev_status,
                          void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Combine: course module sec. 2.2 and the sec. 4 combine:
 * y_n = sum_{j<k} topk_w[n, j] * y_sorted[inv_perm[n*k + j]], summed in slot
 * order with fp32 accumulation.  Needs no workspace.
 */
MOE_API moe_status moe_combine(const moe_config *cfg, const void *y_sorted,
                       const float *topk_w, const int32_t *inv_perm, void *y,
                       moe_stream_t stream);

/*
 * Shared expert over all N tokens (see moe_shared_expert):
 * y_shared[n] = Shared(x[n]), [N, d_model] in cfg->dtype, on the same
 * grouped-GEMM kernels as the routed experts (one slice of N rows).  Needs
 * cfg->d_ff_shared > 0; the hidden activations live in the workspace.
 */
MOE_API moe_status moe_shared_ffn(const moe_config *cfg, const void *x,
                          const moe_shared_expert *shared, void *y_shared,
                          int32_t *dev_status, void *ws, size_t ws_bytes,
                          moe_stream_t stream);

/*
 * moe_combine plus the shared expert's output: y_n = sum_{j<k} topk_w[n, j]
 * * y_sorted[inv_perm[n*k + j]] + y_shared[n] (course module sec. 2.1), with
 * the shared row added after the routed sum, in fp32.  y_shared NULL gives
 * moe_combine.  Needs no workspace.
 */
MOE_API moe_status moe_combine_shared(const moe_config *cfg, const void *y_sorted,
                              const float *topk_w, const int32_t *inv_perm,
                              const void *y_shared, void *y,
                              moe_stream_t stream);

/*
 * Router z-loss ("nano-moe", "Router z-loss"; RustingBrain chapter sec. 15.3
 * "The z-loss"): z = (1/N) sum_n (log sum_e exp z_{n,e})^2 over the router
 * logits z_n = W_g x_n, written as float to the device scalar z_loss_out
 * (per-token terms in fp32, summed in fp64 in a fixed order; 0 for N = 0).
 * The raw value: the loss coefficient is the caller's.  Recomputes the
 * routing into the workspace; moe_forward_ex returns the same value from its
 * own routing pass at almost no cost.
 */
MOE_API moe_status moe_router_z_loss(const moe_config *cfg, const void *x,
                             const void *W_g, float *z_loss_out,
                             int32_t *dev_status, void *ws, size_t ws_bytes,
                             moe_stream_t stream);

/*
 * Switch load-balance loss: course module sec. 2.3 and the sec. 4
 * load_balance_loss:  L = E * sum_e f_e P_e with f_e = (assignments to e)/N
 * and P_e = mean_n probs[n, e]; written as float to the device scalar
 * aux_out (reduced in fp64).  counts_out [E] (may be NULL) receives the
 * assignment counts.  If gamma > 0 and b_e_inout is given, also applies one
 * step of the sec. 2.5 sign rule b_e += gamma * sign(N*k/E - count_e)
 * (MoE.update_bias).
 */
MOE_API moe_status moe_aux_loss(const moe_config *cfg, const float *probs,
                        const int32_t *topk_ids, float *aux_out,
                        int32_t *counts_out, float gamma, float *b_e_inout,
                        int32_t *dev_status, void *ws, size_t ws_bytes,
                        moe_stream_t stream);

/*
 * The whole layer forward (course module sec. 4 MoE.forward; the shared
 * expert and the z-loss are in moe_forward_ex): route -> dispatch -> expert FFNs -> combine, plus the Switch loss
 * (aux_out, may be NULL) and the assignment counts (counts, may be NULL; the
 * sec. 4 expert_load).  If gamma > 0 and b_e_inout is given (sigmoid
 * router), b_e is used for this forward's selection and then moved by one
 * sign-rule step (sec. 2.5), after the selection.  topk_ids / topk_w (may be
 * NULL) receive the routing.  dev_status (may be NULL) is cleared at the
 * start.  stage_events (may be NULL) is an array of MOE_NUM_STAGES + 1
 * cudaEvent_t handles recorded on `stream` at the stage boundaries
 * (MOE_STAGE_*), for timing.  Enqueues only: no host synchronisation.
 */
MOE_API moe_status moe_forward(const moe_config *cfg, const void *x, const void *W_g,
                       float *b_e_inout, float gamma, const void *W1,
                       const void *b1, const void *W3, const void *W2,
                       const void *b2, void *y, int32_t *topk_ids,
                       float *topk_w, int32_t *counts, float *aux_out,
                       int32_t *dev_status, void *ws, size_t ws_bytes,
                       void *const *stage_events, moe_stream_t stream);

/*
 * moe_forward with the shared expert and the router z-loss (course module
 * sec. 2.1; "nano-moe", "Router z-loss").  shared (NULL iff
 * cfg->d_ff_shared == 0) adds Shared(x_n) to every output row after the
 * routed sum; z_loss_out (may be NULL) receives the router z-loss as in
 * moe_router_z_loss, taken from this forward's routing pass.  Every other
 * argument is that of moe_forward, which is this call with shared and
 * z_loss_out NULL (and rejects cfg->d_ff_shared > 0).
 */
MOE_API moe_status moe_forward_ex(const moe_config *cfg, const void *x, const void *W_g,
                          float *b_e_inout, float gamma, const void *W1,
                          const void *b1, const void *W3, const void *W2,
                          const void *b2, const moe_shared_expert *shared,
                          void *y, int32_t *topk_ids, float *topk_w,
                          int32_t *counts, float *aux_out, float *z_loss_out,
                          int32_t *dev_status, void *ws, size_t ws_bytes,
                          void *const *stage_events, moe_stream_t stream);

/*
 * The forward of one data-parallel rank (course module sec. 2.3 and 2.5: the
 * Switch loss and the sign rule are defined over the whole batch, which a
 * data-parallel layer splits across ranks).  Runs the layer like
 * moe_forward_ex on this call's N tokens and, instead of the local loss,
 * returns the two partials the whole-batch loss is made of:
 *   counts   [E] int32   assignments to each expert (required),
 *   psum_out [E] float64 sum over this call's tokens of p_{n,e} = softmax(z_n)
 *                        (required, 8-byte aligned; summed in fp64 in a fixed
 *                        order).
 * Summed over the ranks (an all-reduce of each; sums of integers and of the
 * rank totals), they go to moe_aux_from_partials.  b_e (sigmoid router, may
 * be NULL) selects only and is not moved here: its sign-rule step needs the
 * whole batch's load.  Every other argument is that of moe_forward_ex.
 */
MOE_API moe_status moe_forward_partials(const moe_config *cfg, const void *x, const void *W_g,
                                        const float *b_e, const void *W1, const void *b1,
                                        const void *W3, const void *W2, const void *b2,
                                        const moe_shared_expert *shared, void *y,
                                        int32_t *topk_ids, float *topk_w, int32_t *counts,
                                        double *psum_out, float *z_loss_out, int32_t *dev_status,
                                        void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The whole batch's Switch loss and sign-rule step from partials summed over
 * forwards (course module sec. 2.3, sec. 2.5): with counts [E] int32 and
 * psum [E] float64 (8-byte aligned) the sums over every rank's
 * moe_forward_partials, N = sum_e counts[e] / k (each token makes exactly k
 * assignments) and
 *   aux_out   = E sum_e counts[e] psum[e] / N^2   (float; 0 when N = 0),
 *   b_e_inout += gamma sign(N k - E counts[e])    (if gamma > 0 and given).
 * Either output may be NULL, not both.  Device pointers; one small kernel on
 * `stream`, reduced in fp64 in a fixed order, so ranks that pass the same
 * sums get the same bits.  Limits as moe_config (E <= 256, k <= min(E, 16)).
 */
MOE_API moe_status moe_aux_from_partials(int32_t E, int32_t k, const int32_t *counts,
                                         const double *psum, float *aux_out, float gamma,
                                         float *b_e_inout, moe_stream_t stream);

/*
 * Gradients written by moe_backward: fp32, row-major, caller-owned device
 * memory, 16-byte aligned (else MOE_ERR_INVALID_ARG), each overwritten (not
 * accumulated).  Shapes as the parameters:
 * dx [N, d_model], dW_g [E, d_model], dW1 / dW3 [E, d_ff, d_model],
 * db1 [E, d_ff], dW2 [E, d_model, d_ff], db2 [E, d_model]; the shared
 * expert's dWs1 / dWs3 [d_ff_shared, d_model], dbs1 [d_ff_shared],
 * dWs2 [d_model, d_ff_shared], dbs2 [d_model].  A gradient whose parameter
 * is absent (dW3 for GELU, db1 without b1, ...) is ignored and may be NULL;
 * dx, dW_g, dW1, dW2 (and dW3 for SwiGLU, dWs1 / dWs2 (/ dWs3) with a shared
 * expert) are required.
 */
typedef struct {
    float *dx;
    float *dW_g;
    float *dW1;
    float *db1;
    float *dW3;
    float *dW2;
    float *db2;
    float *dWs1;
    float *dbs1;
    float *dWs3;
    float *dWs2;
    float *dbs2;
} moe_grads;

/* Workspace bytes moe_backward needs for cfg (0 for an invalid cfg). */
MOE_API size_t moe_backward_workspace_size(const moe_config *cfg);

/*
 * Backward of the layer for an upstream gradient dy [N, d_model] (layer
 * dtype): the gradients of
 *   loss = <dy, y> + aux_coef * L_aux + z_coef * L_z
 * with y, L_aux (Switch loss, course module sec. 2.3) and L_z (router
 * z-loss, "nano-moe") as moe_forward_ex computes them from the same inputs.
 * b_e must be the selection bias the forward selected with (before its
 * sign-rule step).  The expert choice and f_e = count_e / N are piecewise
 * constant and carry no gradient (course module sec. 2.4); the bias selects
 * only.  Per token: the
 * gate of expert e gets <dy_n, Expert_e(x_n)>, the expert the output
 * gradient w dy_n, the shared expert dy_n; the Switch loss reaches the
 * router through dL_aux / dp_{n,e} = E f_e / N (course module sec. 2.3),
 * the z-loss through 2 lse(z_n) p_n / N.  The routing and the
 * expert pre-activations are recomputed (same kernels as the forward, so the
 * same expert choice); all products accumulate in fp32.  bf16: the expert
 * products run on the tensor cores, with the intermediate gradients (da,
 * du, w h) rounded to bf16 as operands; fp32: on the CUDA cores throughout.
 * Workspace: moe_backward_workspace_size(cfg) bytes (the recomputed
 * activations and the intermediate gradients; weights and activations are
 * read in place by the tensor-core products).  Enqueues only.
 */
MOE_API moe_status moe_backward(const moe_config *cfg, const void *x, const void *W_g,
                        const float *b_e, const void *W1, const void *b1,
                        const void *W3, const void *W2, const void *b2,
                        const moe_shared_expert *shared, const void *dy,
                        float aux_coef, float z_coef, const moe_grads *grads,
                        int32_t *dev_status, void *ws, size_t ws_bytes,
                        moe_stream_t stream);

/*
 * Row permutation, the regrouping step of expert parallelism (course module
 * "Going further": experts on different GPUs, tokens moved by all-to-all;
 * the rows one rank receives arrive grouped by sending rank and are
 * regrouped by expert): dst[dst_row[i]] = src[i] for i < rows, rows of d
 * elements of `dtype`.  dst_row should be a permutation of 0..rows-1; an
 * entry outside that range is skipped (that source row is not copied).
 * src, dst: device, 16-byte aligned, not overlapping; d > 0 and a multiple
 * of 8; rows < 2^31.  Enqueues only.
 */
MOE_API moe_status moe_permute_rows(int32_t dtype, const void *src, const int32_t *dst_row,
                                    void *dst, int64_t rows, int32_t d, moe_stream_t stream);

/*
 * Failure-detection check (the pages have no counterpart): launches one CTA
 * that waits on an mbarrier nothing ever arrives at, through the same
 * bounded wait every tcgen05 kernel of the library uses.  After the wait
 * limit (2 s of %globaltimer) the kernel writes MOE_ERR_TIMEOUT to
 * *dev_status (cleared first) and returns; the context stays usable.
 * Enqueues only: synchronise the stream, then read *dev_status.
 */
MOE_API moe_status moe_selftest_wait_timeout(int32_t *dev_status, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
