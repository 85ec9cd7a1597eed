/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) forward pass of a Qwen-family sparse MoE FFN
 * block: router, expert-contiguous permutation, SwiGLU experts and the weighted combine.
 *
 * The operation ("27. Mixture of experts", inference.shantanugoel.com):
 *   section "The router":  logits = W_r x; softmax over all E experts in FP32; keep the k
 *                          largest with their indices, ties broken by index; with
 *                          norm_topk_prob, divide the kept weights by their sum;
 *                          y = sum_{i in top-k} w_i expert_i(x).
 *   section "Dispatch":    experts stacked as gate_up [E, 2I, D] (gate rows first) and
 *                          down [E, D, I]; expert(x) = down(silu(gate x) * up x); grouped
 *                          dispatch sorts the N*k assignments by expert (stable) so each
 *                          expert's rows are contiguous.
 *   section "The shared expert": optionally y += sigmoid(w_s . x) * shared(x).
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major and contiguous,
 *    16-byte aligned.  bf16 tensors are passed as their 16-bit patterns (moe_bf16).
 *  - The library allocates no memory and never synchronises the host on these calls: all
 *    work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream).
 *    Scratch comes from the caller's workspace `ws` of `ws_bytes` bytes, sized with
 *    moe_workspace_size().  The workspace must not be used by two calls that can run at the
 *    same time.
 *  - Arguments are validated before anything is enqueued; an invalid call returns an error
 *    status and enqueues nothing.  There is no CPU fallback: a call that cannot run on the
 *    GPU fails with MOE_ERR_CUDA.
 *  - Inputs must be finite; NaN or Inf inputs give undefined outputs (never a fault).
 *  - Precision: router logits, softmax, routing weights and every accumulation are FP32;
 *    the SwiGLU intermediate h = silu(g) * u is rounded to bf16 (the down projection's MMA
 *    operand type); the k weighted expert outputs are summed in FP32 and the block output
 *    is rounded once to bf16 (round to nearest even).  opts->out_f32 returns that FP32 sum
 *    before its rounding.
 *  - Supported shapes: 1 <= E <= 512, 1 <= k <= min(E, 16), D and I (and I_s) multiples of
 *    128, T >= 1, T * (k + 1) < 2^31.  Other shapes return MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16;                /* raw bfloat16 bits */
typedef struct CUstream_st *moe_stream_t; /* identical to cudaStream_t */
typedef struct CUevent_st *moe_event_t;   /* identical to cudaEvent_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,    /* null / misaligned pointer, T < 1, bad struct */
    MOE_ERR_UNSUPPORTED = 2,    /* shape outside the supported set above */
    MOE_ERR_WORKSPACE = 3,      /* ws_bytes smaller than moe_workspace_size() */
    MOE_ERR_CUDA = 4,           /* a CUDA call failed (no GPU, launch error, ...) */
    MOE_ERR_DEVICE_TIMEOUT = 5  /* a kernel gave up a bounded wait (see moe_get_device_status) */
} moe_status;

/* Problem shape.  No field has a default: every one must be set.
 *   T  tokens, D hidden size, E routed experts, k experts per token, I expert width;
 *   norm_topk_prob  1 = renormalise the k kept weights to sum to 1, 0 = keep softmax values;
 *   tile_m  row padding of each expert segment in moe_permute (1 = none; 1..256).  The
 *           forward pass does not use it. */
typedef struct {
    int T, D, E, k, I;
    int norm_topk_prob;
    int tile_m;
} moe_dims;

/* Which expert path moe_forward_ex takes. */
enum {
    MOE_PATH_AUTO = 0,    /* the library's choice: MOE_PATH_DECODE where it applies, else
                             MOE_PATH_GROUPED (moe_forward_path tells which) */
    MOE_PATH_GROUPED = 1, /* permute + tcgen05 grouped GEMMs, TMA-fed, TMEM accumulators */
    MOE_PATH_DECODE = 2   /* the whole block in one kernel for one token (T = 1, D <= 2048,
                             and two blocks of ceil(D / SMs) down rows of I fit in an SM's
                             shared memory beside its buffers), bf16 or FP8 experts: one
                             block per SM, all resident at once (a call needs the whole GPU;
                             other work running on it delays the call, up to the wait limit,
                             after which it reports MOE_ERR_DEVICE_TIMEOUT).  Not with a
                             shared expert, expert_counts_out, slot_row_out or
                             MOE_DIAG_UNSIGNALLED_HANDOFF; asking for it then returns
                             MOE_ERR_UNSUPPORTED */
};

/* Diagnostics of moe_forward_ex (moe_opts.diag); 0 in normal use. */
enum {
    /* The down GEMM's per-expert hand-off wait (used when T*k <= 32*E) watches a completion
     * counter that nothing increments, so each such wait runs until its limit
     * (moe_opts.wait_limit_us) and the kernels wind down.  The output is then undefined and
     * moe_get_device_status reports MOE_ERR_DEVICE_TIMEOUT; the device stays usable.  For
     * testing the watchdog.  Shapes that do not use the hand-off return MOE_ERR_UNSUPPORTED. */
    MOE_DIAG_UNSIGNALLED_HANDOFF = 1,
    /* The decode kernel's grid-wide barrier waits for one block more than the grid has, so it
     * runs until its limit (moe_opts.wait_limit_us); the output is then undefined and
     * moe_get_device_status reports MOE_ERR_DEVICE_TIMEOUT; the device stays usable.  For
     * testing the watchdog of MOE_PATH_DECODE; where that path does not apply,
     * MOE_ERR_UNSUPPORTED. */
    MOE_DIAG_DECODE_BARRIER = 2
};

/* Options of moe_forward_ex.  Zero-initialise and set what is needed. */
typedef struct {
    const float *router_bias;        /* [E] FP32 added to the logits before the softmax, or NULL */
    const moe_bf16 *shared_gate_up;  /* [2*I_s, D] shared expert (gate rows first), or NULL */
    const moe_bf16 *shared_down;     /* [D, I_s]; required with shared_gate_up */
    const moe_bf16 *shared_gate;     /* [D] w_s: y += sigmoid(w_s . x) * shared(x); NULL = ungated */
    int I_s;                         /* shared expert width (multiple of 128) */
    const moe_bf16 *residual;        /* [T, D]: out = residual + block(x), or NULL */
    float *logits_out;               /* [T, E] FP32 router logits (bias included), or NULL */
    int32_t *topk_idx_out;           /* [T, k] selected experts, slot order, or NULL */
    float *topk_w_out;               /* [T, k] FP32 routing weights, or NULL */
    int path;                        /* MOE_PATH_* */
    moe_event_t *stage_events;       /* if n_stage_events == 6: recorded on `stream` at the start,
                                        after routing, after the permutation, after gate_up,
                                        after down and after the combine (as external events,
                                        so they become graph nodes under stream capture) */
    int n_stage_events;
    float *out_f32;                  /* [T, D] FP32 block output before its rounding to bf16
                                        (residual and shared expert included), or NULL */
    int32_t *expert_counts_out;      /* [E] assignments routed to each expert (the per-expert
                                        load), or NULL */
    int32_t *slot_row_out;           /* [T, k] row of assignment (t, j) in the expert-sorted
                                        order: the slot_row of moe_permute with tile_m = 1,
                                        or NULL */
    unsigned wait_limit_us;          /* limit of every bounded device wait in microseconds;
                                        0 = the default of 2 s */
    int diag;                        /* MOE_DIAG_* or 0 */
    /* FP8 weight-only experts.  When W_gate_up_fp8 is set, the routed experts' weights are
     * read from W_gate_up_fp8 [E, 2I, D] and W_down_fp8 [E, D, I] (one E4M3 byte per weight,
     * as written by moe_quantize_fp8_rows) with one FP32 scale per weight row,
     * gate_up_scale [E * 2I] and down_scale [E * D]; weight (e, r, c) = scale[e, r] *
     * value(q[e, r, c]).  The bf16 W_gate_up and W_down arguments are then not read and may
     * be NULL.  Tokens stay bf16; the weights are widened exactly (to bf16 in shared memory on
     * the grouped path, to FP32 in registers on the one-token kernel) and the row scale is
     * applied to the FP32 sums.  Supported at decode shapes (T*k <= 32*E) without a shared
     * expert; otherwise MOE_ERR_UNSUPPORTED. */
    const uint8_t *W_gate_up_fp8;    /* [E, 2I, D] E4M3, or NULL (bf16 weights) */
    const float *gate_up_scale;      /* [E * 2I] FP32 */
    const uint8_t *W_down_fp8;       /* [E, D, I] E4M3 */
    const float *down_scale;         /* [E * D] FP32 */
} moe_opts;

/* Per-row FP8 quantisation of a bf16 matrix W [rows, cols] (rows of the expert weight
 * tensors: pass W_gate_up as E*2I rows of D, W_down as E*D rows of I).  No format is fixed
 * by the pages; this is the plainest per-row (per output channel) E4M3 scheme:
 *   amax[r]  = max_c |W[r, c]|;
 *   scale[r] = amax[r] / 448 in FP32 (round to nearest even), or 1 when amax[r] == 0;
 *   q[r, c]  = E4M3 (OCP "e4m3fn": bias 7, max 448, no infinities) of the FP32 quotient
 *              W[r, c] / scale[r], rounded to nearest even and saturated to +-448.
 * Bitwise deterministic.  W [rows, cols] bf16, q [rows, cols] bytes, scale [rows] FP32; cols
 * a multiple of 16 and all pointers 16-byte aligned.  Enqueued on `stream`. */
moe_status moe_quantize_fp8_rows(const moe_bf16 *W, int64_t rows, int cols, uint8_t *q, float *scale,
                                 moe_stream_t stream);

/* The Switch balance loss of the router ("Qwen3-VL and Mixture of Experts", the fixes for
 * expert collapse, "An auxiliary balance loss"; the Qwen3-VL MoE walk-through,
 * "load_balancing_loss_func") and its gradient with respect to the router logits:
 *   p[t]   = softmax(logits[t]) in FP32;  P_e = (1/T) sum_t p[t, e];
 *   f_e    = (1/T) * number of (t, j) with topk_idx[t, j] == e  (entries outside [0, E) are
 *            not counted);
 *   loss   = alpha * E * sum_e f_e P_e;
 *   dlogits[t, e] = alpha * E / T * p[t, e] * (f_e - sum_i f_i p[t, i])  (f held fixed: the
 *            selection is not differentiable).
 * logits [T, E] FP32 (as moe_route returns them, bias included when one was given), topk_idx
 * [T, k] int32, loss: one FP32 value in device memory, dlogits [T, E] FP32 or NULL (loss only).
 * Workspace of moe_aux_loss_workspace_size(T, E) bytes, 256-byte aligned.  All sums run in a
 * fixed order: bitwise reproducible.  1 <= E <= 512, 1 <= k <= min(E, 16); enqueued on
 * `stream`. */
size_t moe_aux_loss_workspace_size(int T, int E);
moe_status moe_aux_loss(const float *logits, const int32_t *topk_idx, int T, int E, int k, float alpha,
                        float *loss, float *dlogits, void *ws, size_t ws_bytes, moe_stream_t stream);

/* The backward pass of the routed block for a given routing ("Qwen3-VL and Mixture of
 * Experts", "How the router and experts learn", "What gets trained": a token's gradient
 * reaches only the experts it chose, and the router learns through the gate weights; the
 * selection is held fixed).  For the loss sum_t dy[t] . y[t], y the block's output with the
 * routing topk_idx (normally the forward's), the gradients with respect to:
 *   dx [T, D]            the input x (+ dy when residual = 1, i.e. y = x + block(x));
 *   dW_r [E, D]          the router weights;      dbias [E] the router bias (or NULL);
 *   dW_gate_up [E,2I,D]  and dW_down [E, D, I]    (zero for experts no token chose);
 *   dlogits [T, E]       the router logits (or NULL);  dw [T, k] the routing weights (or NULL).
 * Per token and slot j (expert e, weight w_j, s = sigmoid(g), h = g s u):
 *   z = W_down[e]^T dy,  dw_j = h . z,  dh = w_j z,  dg = dh u s (1 + g (1 - s)),  du = dh g s;
 *   dp_j = (dw_j - sum_m dw_m w_m) / sum_m p_m (norm_topk_prob) or dw_j;
 *   dlogits = p (dp - sum_j p_j dp_j) + dlogits_add (e.g. moe_aux_loss's gradient; or NULL).
 * x, W_r, W_gate_up, W_down as for moe_forward; bias [E] FP32 or NULL (as given to the
 * forward); dy [T, D] bf16; topk_idx [T, k] int32 (entries outside [0, E) are skipped and
 * recorded in the device error word, which moe_get_device_status reads from ws).  Outputs are
 * FP32 and fully overwritten.  The router logits and g, u are recomputed; h, dg, du, w dy and
 * dlogits are rounded to bf16 once as GEMM operands; all sums run in a fixed order (bitwise
 * reproducible).  No shared expert.  Shapes as for moe_forward (dims->tile_m is ignored);
 * 16-byte aligned bf16/FP32 matrices, workspace of moe_backward_workspace_size(dims) bytes,
 * 256-byte aligned.  Enqueued on `stream`; allocates and synchronises nothing, so a call can
 * be captured in a CUDA graph once the same shape has run eagerly (the first call of a shape
 * sets kernel attributes). */
size_t moe_backward_workspace_size(const moe_dims *dims);
moe_status moe_backward(const moe_bf16 *x, const moe_bf16 *W_r, const float *bias,
                        const moe_bf16 *W_gate_up, const moe_bf16 *W_down, const moe_bf16 *dy,
                        const int32_t *topk_idx, const float *dlogits_add, int residual,
                        const moe_dims *dims, float *dx, float *dW_r, float *dbias,
                        float *dW_gate_up, float *dW_down, float *dlogits, float *dw, void *ws,
                        size_t ws_bytes, moe_stream_t stream);

/* Bytes of workspace that moe_route, moe_permute and moe_forward(_ex) need for `dims`
 * (and `opts`, which may be NULL).  Returns 0 for invalid or unsupported arguments. */
size_t moe_workspace_size(const moe_dims *dims, const moe_opts *opts);

/* Router ("27. Mixture of experts", section "The router"):
 *   logits[t, e] = sum_d x[t, d] W_r[e, d] (FP32 accumulate) (+ bias[e]);
 *   topk_idx[t, j] = expert of rank j by FP32 logit, equal logits -> lower index;
 *   topk_w[t, j] = softmax(logits[t])[idx] in FP32, divided by the sum of the k kept values
 *                  when dims->norm_topk_prob.
 * x [T, D] bf16, W_r [E, D] bf16 (nn.Linear layout), bias [E] FP32 or NULL,
 * logits [T, E] FP32 or NULL (then the workspace holds them), topk_idx [T, k] int32,
 * topk_w [T, k] FP32.
 * Summation order: D is summed in FP32 in slices added in slice order -- for T <= 64 in 8
 * equal slices, above in up to 8 slices whose number is fixed by (T, E, D).  Results are
 * bitwise reproducible; a token's logits do not depend on the other tokens within one of
 * those two regimes. */
moe_status moe_route(const moe_bf16 *x, const moe_bf16 *W_r, const float *bias,
                     const moe_dims *dims, float *logits, int32_t *topk_idx, float *topk_w,
                     void *ws, size_t ws_bytes, moe_stream_t stream);

/* Stable expert-contiguous permutation ("27. Mixture of experts", section "Dispatch",
 * grouped dispatch; counting sort over a = t*k + j):
 *   counts[e]  = number of assignments to expert e                       [E] int32
 *   offsets[0] = 0, offsets[e+1] = offsets[e] + ceil(counts[e]/tile_m)*tile_m   [E+1]
 *   rows offsets[e] .. offsets[e]+counts[e]-1 hold expert e's assignments in increasing a;
 *   row_token[r] = token of row r, -1 on padding rows                    [cap] int32
 *   slot_row[a]  = row of assignment a                                   [T*k] int32
 *   row_weight[r] = topk_w of row r (0 on padding), written when both are non-NULL [cap]
 *   x_perm[r, :] = x[row_token[r], :] (zeros on padding rows), written when x and x_perm
 *                  are non-NULL                                          [cap, D] bf16
 * cap must be >= T*k + E*(tile_m - 1).  topk_idx values outside [0, E) are skipped and
 * recorded in the device error word; moe_get_device_status then returns
 * MOE_ERR_INVALID_ARG. */
moe_status moe_permute(const int32_t *topk_idx, const float *topk_w, const moe_bf16 *x,
                       const moe_dims *dims, int32_t *counts, int32_t *offsets,
                       int32_t *row_token, int32_t *slot_row, float *row_weight,
                       moe_bf16 *x_perm, int cap, void *ws, size_t ws_bytes,
                       moe_stream_t stream);

/* The whole block: out[t] = sum_j w[t,j] * expert_{idx[t,j]}(x[t]).
 * x [T, D] bf16, W_r [E, D] bf16, W_gate_up [E, 2I, D] bf16 (gate rows 0..I-1, up rows
 * I..2I-1), W_down [E, D, I] bf16, out [T, D] bf16 (fully overwritten; must not alias x).
 * The k weighted outputs are summed in slot order in FP32 and rounded once to bf16.
 * Wider shapes run their expert GEMMs on pairs of SMs (thread-block clusters); setting the
 * environment variable MOE_B200_NO_PAIRS selects single-SM tiles instead (same results up to
 * FP32 summation order).
 * Results are bitwise reproducible for the same inputs.  At decode shapes (T*k <= 32*E) the
 * expert GEMMs may split the K sums of their last items into slices (added in slice order),
 * and how many depends on the batch's work, so a token's output can differ in the last bits
 * between batches (its routing does not, see moe_route).  For T = 1 the decode kernel
 * (MOE_PATH_DECODE) computes every dot product in a fixed order that does not depend on the
 * GPU's SM count. */
moe_status moe_forward(const moe_bf16 *x, const moe_bf16 *W_r, const moe_bf16 *W_gate_up,
                       const moe_bf16 *W_down, const moe_dims *dims, moe_bf16 *out, void *ws,
                       size_t ws_bytes, moe_stream_t stream);

/* moe_forward with options (router bias, gated shared expert, residual, routing outputs,
 * path choice, stage events).  out may alias opts->residual but not x.  On MOE_PATH_DECODE
 * the stage events after routing .. after the combine are all recorded after its one
 * kernel. */
moe_status moe_forward_ex(const moe_bf16 *x, const moe_bf16 *W_r, const moe_bf16 *W_gate_up,
                          const moe_bf16 *W_down, const moe_dims *dims, const moe_opts *opts,
                          moe_bf16 *out, void *ws, size_t ws_bytes, moe_stream_t stream);

/* The path (MOE_PATH_DECODE or MOE_PATH_GROUPED) that moe_forward_ex takes for these
 * arguments, in *path_out; the status moe_forward_ex would return for an invalid or
 * unsupported request, or MOE_ERR_CUDA without a device (the choice depends on the device's
 * SM count).  Enqueues nothing. */
moe_status moe_forward_path(const moe_dims *dims, const moe_opts *opts, int *path_out);

/* moe_forward for callers that cannot allocate device memory: plugin hosts that give a
 * kernel only its input and output buffers, and runtimes that forbid device allocation once
 * they have started (their memory is planned up front).  The pages have no counterpart:
 * this is a deployment variant of moe_forward, same arguments minus the workspace, same
 * results.
 * Scratch: a 64 MiB array in the library's own device memory (a file-scope device
 * variable), held by every GPU that loads this part of the library until the process
 * exits.  Calls whose moe_workspace_size(dims, NULL) exceeds 64 MiB return
 * MOE_ERR_WORKSPACE before enqueuing anything (the decode shapes fit: D=2048, E=128, k=8,
 * I=768 up to T=256).  Nothing is allocated or freed.
 * The first call on a device looks up the array's device address (once per device); make
 * that first call before any stream capture.  All calls on a device share the array and it
 * keeps the last call's contents; each call clears what must start at zero.  Calls that can
 * overlap on the GPU (other streams, unordered host threads) race on the array.
 * Its device error word (bounded waits, bad indices) is read with
 * moe_get_device_status_noalloc. */
moe_status moe_forward_noalloc(const moe_bf16 *x, const moe_bf16 *W_r, const moe_bf16 *W_gate_up,
                               const moe_bf16 *W_down, const moe_dims *dims, moe_bf16 *out,
                               moe_stream_t stream);

/* moe_get_device_status for moe_forward_noalloc, whose workspace the caller never sees:
 * synchronises `stream` and reports the device error word that the last
 * moe_forward_noalloc call on the current device left in the library's array (MOE_OK
 * before the first call).  The pages have no counterpart. */
moe_status moe_get_device_status_noalloc(moe_stream_t stream);

/* Synchronises `stream` and reports the device error word that the last call using `ws`
 * left: MOE_OK, MOE_ERR_DEVICE_TIMEOUT (a bounded wait expired), MOE_ERR_INVALID_ARG (an
 * expert index outside [0, E) reached moe_permute) or MOE_ERR_CUDA. */
moe_status moe_get_device_status(const void *ws, moe_stream_t stream);

/* Static, human-readable name of a status. */
const char *moe_status_string(moe_status s);

/* The CUDA runtime error code (a cudaError_t value) of the most recent CUDA call that made a
 * call of this library on the calling host thread return MOE_ERR_CUDA; 0 if there was none.
 * For diagnostics only: it is not reset by successful calls. */
int moe_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
