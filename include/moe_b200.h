/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) sparse Mixture-of-Experts FFN
 * forward library (libmoe_b200.so).
 *
 * The layer (per token x_t, t < T):
 *   logits  = W_g x_t (+ logit_offset)                 one score per expert
 *   p       = softmax(logits)
 *   chosen  = the K experts with the largest selection score
 *             (logit; or p + b with a selection bias b)
 *   w_k     = p[chosen_k] / sum_k' p[chosen_k']        renormalised gates
 *   dispatch: each expert serves at most `cap` (t,k) pairs, earlier tokens
 *             first; the rest are dropped
 *   y_t     = sum_s SharedExpert_s(x_t) + sum_{kept k} w_k Expert_{chosen_k}(x_t)
 *   Expert(x) = W_down (SiLU(W_gate x) * (W_up x))
 * plus the Switch statistics f_e, P_e and alpha * E * sum_e f_e P_e.
 * The residual add is the caller's.
 *
 * Sources (page title, section / equation):
 *   "Zen MoDE: Mixture of Distilled Experts Architecture": §3.1 Router
 *     Architecture (eq. router_standard, TopK(softmax(W_r x), K)); §5.2 Auxiliary
 *     Load Balancing Loss (eq. L_balance, f_e, P_e, alpha = 0.01); §5.3 Adaptive
 *     Capacity Factors (capacity_e = C * batch * seq / N_E).
 *   "Zen-Max: Maximum Capability via Mixture-of-Experts Architecture": §2.2
 *     Fine-Grained Expert Architecture (eq. Expert_i, SwiGLU; shared experts added
 *     to the routed outputs); §2.3 Auxiliary-Loss-Free Load Balancing
 *     (s_ij = softmax(x_i W_g)_j + b_j).
 *   "Scaling with experts" (jeff-ong.com): "The gating network" (the k best
 *     gates kept and rescaled to add up to 1; output = gate-weighted sum of the
 *     chosen experts); "A balance penalty"; "A budget" (per-expert capacity;
 *     a dropped assignment is not processed by its expert); "A shared expert".
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, row-major, densely packed, owned
 *     by the caller.  The library never allocates or frees device memory
 *     (except moe_ipc_malloc / moe_ipc_free, which exist to do so for buffers
 *     other processes map) and keeps no state between calls; scratch space is
 *     the caller's workspace `ws` of `ws_bytes` bytes (size from
 *     moe_workspace_size; 256-byte aligned).
 *   - Every call only enqueues work on `stream` and returns; nothing
 *     synchronises with the host (except moe_read_device_status).
 *   - Activations and weights are BF16 (MOE_DTYPE_BF16) or FP32 (MOE_DTYPE_F32);
 *     router logits, gate weights, offsets, biases and statistics are FP32.
 *     BF16 math: BF16 operands, FP32 accumulation, one rounding per stored
 *     intermediate (expert hidden activations, expert outputs, layer output).
 *   - Weight storage ("linear [out, in]" rows):
 *       w_gate [E, d]; w13 [E, 2F, d] (rows 0..F-1 gate proj, F..2F-1 up proj);
 *       w2 [E, d, F]; shared: w13 [N_s, 2F, d], w2 [N_s, d, F].
 *   - Alignment: every pointer 16-byte aligned; d_model and d_ff multiples of 8.
 *   - Return value: MOE_OK (0) or a negative moe_status.  Arguments are checked
 *     on the host before anything is enqueued; a rejected call enqueues nothing.
 *     Kernels that find bad data (an expert index outside [0, E)) or give up a
 *     bounded wait do not trap: they skip the access and set a bit in the
 *     device status word at the start of `ws` (see moe_read_device_status).
 *   - Thread safety: calls are independent; concurrent calls need distinct
 *     workspaces.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 2

typedef struct CUstream_st* moe_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,  /* bad shape, NULL pointer, misalignment, K > E, ... */
    MOE_ERR_UNSUPPORTED = -2,  /* valid problem this build does not handle (e.g. E > 256) */
    MOE_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed */
    MOE_ERR_DEVICE_CHECK = -4, /* a kernel reported bad data (see moe_read_device_status) */
    MOE_ERR_WORKSPACE = -5     /* ws too small or misaligned */
} moe_status;

typedef enum moe_dtype { MOE_DTYPE_BF16 = 0, MOE_DTYPE_F32 = 1 } moe_dtype;

/* moe_problem_t.flags */
#define MOE_FLAG_LOGITS_GIVEN 0x1u /* moe_route / moe_layer_forward read the logits
                                      instead of computing them from x and w_gate */
#define MOE_FLAG_BIAS_LOGIT 0x2u   /* selection bias added to the logit, not to p */
#define MOE_FLAG_EXTENDED_STATS 0x4u /* stats has 2E+7 entries: after the 2E+1 balance
                                        entries, the router z-loss and utilisation
                                        statistics (see moe_route) */
#define MOE_FLAG_EXPERT_CAPACITY 0x8u /* per-expert capacities from a device array
                                         (moe_weights_t.expert_capacity, or the
                                         argument of moe_dispatch_capacity) instead
                                         of the uniform ceil(C*T*K/E); the row
                                         bound moe_max_rows becomes T*K */
#define MOE_FLAG_SAVE_GU 0x10u /* training (BF16): moe_layer_forward also keeps the
                                  experts' gate and up projections in its
                                  workspace (larger: moe_workspace_size), so that
                                  moe_layer_backward does not recompute them */

/* Device status bits (moe_read_device_status). */
#define MOE_DEV_BAD_EXPERT 0x1     /* an expert index outside [0, E) was skipped */
#define MOE_DEV_WAIT_TIMEOUT 0x2   /* a pipeline wait gave up; results invalid */

/* The problem, in the pages' terms: T = batch * seq tokens of width d_model;
 * E routed experts ("N_E"), top_k ("K"), n_shared always-on experts, each
 * expert a SwiGLU of inner width d_ff; capacity factor C; alpha of the
 * balance loss.  Limits of this build: 1 <= top_k <= min(E, 32); E <= 256;
 * 1 <= T < 2^31 / max(E, top_k). */
typedef struct moe_problem {
    int64_t T;
    int32_t d_model;
    int32_t n_experts;
    int32_t top_k;
    int32_t n_shared;
    int32_t d_ff;
    float capacity_factor; /* <= 0: no capacity limit; else cap = ceil(C*T*K/E) */
    int32_t dtype;         /* moe_dtype */
    uint32_t flags;        /* MOE_FLAG_* */
    float alpha;           /* balance-loss coefficient, e.g. 0.01 */
} moe_problem_t;

/* Weights of one layer (device pointers, layouts above). */
typedef struct moe_weights {
    const void* w_gate;        /* [E, d]; unused with MOE_FLAG_LOGITS_GIVEN */
    const float* logit_offset; /* [E] additive logit offset, or NULL */
    const float* sel_bias;     /* [E] selection-only bias, or NULL */
    const void* w13;           /* [E, 2F, d] */
    const void* w2;            /* [E, d, F] */
    const void* w13_shared;    /* [N_s, 2F, d], NULL iff n_shared == 0 */
    const void* w2_shared;     /* [N_s, d, F],  NULL iff n_shared == 0 */
    const int32_t* expert_capacity; /* [E] with MOE_FLAG_EXPERT_CAPACITY (expert e
                                       keeps at most expert_capacity[e] pairs; a
                                       negative entry: no limit), else ignored */
} moe_weights_t;

/* Optional routing outputs of moe_layer_forward (device pointers; each may be
 * NULL, in which case the array lives in the workspace).  `logits` is an INPUT
 * when MOE_FLAG_LOGITS_GIVEN is set (then it must not be NULL). */
typedef struct moe_routing {
    float* logits;     /* [T, E] */
    int32_t* topk_idx; /* [T, K] */
    float* topk_w;     /* [T, K] */
    int32_t* counts;   /* [E]   assignments per expert before the capacity cut */
    int32_t* kept;     /* [E]   min(counts, cap) */
    int32_t* seg_off;  /* [E+1] exclusive prefix sum of kept */
    int32_t* slot_of;  /* [T, K] row of (t,k) in the expert-grouped arrays, or -1 if dropped */
    int32_t* perm;     /* [moe_max_rows] perm[slot] = t*K + k for slot < seg_off[E] */
} moe_routing_t;

/* ABI version of the loaded library (MOE_ABI_VERSION). */
int moe_abi_version(void);

/* Human-readable name of a moe_status value (static string). */
const char* moe_status_string(int code);

/* Per-expert capacity of `p`: ceil(C * T * K / E) computed in float64 as
 * (C * (T*K)) / E, or -1 when capacity_factor <= 0 (no limit).
 * Zen MoDE §5.3 capacity_e, scaled by K for top-K routing.  Pure host
 * function; returns -2 for a NULL or invalid problem. */
int64_t moe_capacity(const moe_problem_t* p);

/* Upper bound on kept (t,k) rows: min(T*K, E*cap) (T*K without a limit).
 * Rows of perm / x_perm / y_perm.  Returns -2 for an invalid problem. */
int64_t moe_max_rows(const moe_problem_t* p);

/* Workspace bytes every entry point below needs for problem `p` (one size for
 * all of them).  Pure host function. */
int moe_workspace_size(const moe_problem_t* p, size_t* bytes);

/* Zero the device status word at the start of `ws` (async on stream). */
int moe_reset_device_status(void* ws, moe_stream_t stream);

/* Synchronise `stream`, then copy the device status word into *bits.
 * Returns MOE_ERR_DEVICE_CHECK if any bit is set, MOE_OK otherwise. */
int moe_read_device_status(const void* ws, moe_stream_t stream, uint32_t* bits);

/* Router.  Zen MoDE §3.1 eq. router_standard; Zen-Max §2.3 (selection bias);
 * "Scaling with experts", The gating network / A balance penalty.
 *   x            [T, d]  activations (ignored with MOE_FLAG_LOGITS_GIVEN)
 *   w_gate       [E, d]  (ignored with MOE_FLAG_LOGITS_GIVEN)
 *   logit_offset [E] or NULL: added to every token's logits
 *   sel_bias     [E] or NULL: added to the selection score only
 *                (to p, or to the logit with MOE_FLAG_BIAS_LOGIT)
 *   logits       [T, E] fp32: output, or input with MOE_FLAG_LOGITS_GIVEN
 *                (then already including any offset; logit_offset is ignored)
 *   topk_idx     [T, K] out: chosen experts, best first; equal scores go to
 *                the lower index.  Without a bias the score is the fp32 logit;
 *                with a bias it is computed in float64.
 *   topk_w       [T, K] out: renormalised gate weights (sum to 1 per token)
 *   stats        [2E+1] out or NULL: f_e = counts_e / (T*K) (before the
 *                capacity cut), P_e = mean_t p[t,e], loss = alpha*E*sum f_e P_e.
 *                With MOE_FLAG_EXTENDED_STATS, [2E+7]: then
 *                [2E+1] router z-loss (1/T) sum_t (log sum_e exp l[t,e])^2
 *                       (Zen-Max §3.2; the coefficient is the caller's),
 *                [2E+2] entropy in bits of the load shares counts_e / (T*K),
 *                [2E+3] coefficient of variation of counts (population std / mean),
 *                [2E+4] drop rate sum(counts - kept) / (T*K), kept = min(counts, cap),
 *                [2E+5] number of experts with load below 50% of the mean,
 *                [2E+6] number above 200% of the mean
 *                (Zen MoDE §6.2, table tab:utilization).
 *                moe_route knows only the uniform capacity: MOE_FLAG_EXTENDED_STATS
 *                together with MOE_FLAG_EXPERT_CAPACITY is MOE_ERR_INVALID_ARG here
 *                (moe_layer_forward reports them for the per-expert capacities). */
int moe_route(const moe_problem_t* p, const void* x, const void* w_gate,
              const float* logit_offset, const float* sel_bias, float* logits,
              int32_t* topk_idx, float* topk_w, float* stats,
              void* ws, size_t ws_bytes, moe_stream_t stream);

/* Capacity-limited dispatch: group the (t,k) pairs by expert and gather rows.
 * "Scaling with experts", A budget; Zen MoDE §5.3.
 *   topk_idx [T, K] in (an index outside [0, E) is skipped and flagged)
 *   x        [T, d] in
 *   counts [E], kept [E], seg_off [E+1], slot_of [T, K], perm [moe_max_rows] out
 *            (definitions in moe_routing_t; rank of (t,k) within its expert =
 *            number of earlier tokens that chose the same expert; kept iff
 *            rank < cap; slot = seg_off[e] + rank; perm entries past
 *            seg_off[E] are left untouched)
 *   x_perm   [moe_max_rows, d] out: x_perm[slot] = x[perm[slot] / K] for
 *            slot < seg_off[E]; later rows untouched.  May be NULL (no gather).
 * With MOE_FLAG_EXPERT_CAPACITY use moe_dispatch_capacity (here: MOE_ERR_INVALID_ARG). */
int moe_dispatch(const moe_problem_t* p, const int32_t* topk_idx, const void* x,
                 int32_t* counts, int32_t* kept, int32_t* seg_off,
                 int32_t* slot_of, int32_t* perm, void* x_perm,
                 void* ws, size_t ws_bytes, moe_stream_t stream);

/* Expert SwiGLU FFNs (Zen-Max §2.2 eq. Expert_i).
 * mode MOE_FFN_ROUTED: x_rows [n_rows, d] grouped by expert; rows
 *   seg_off[e] .. seg_off[e+1]-1 go through expert e (w13 [E,2F,d],
 *   w2 [E,d,F]); y_rows [n_rows, d]; rows >= seg_off[E] untouched.
 *   n_rows is the allocated row count (>= seg_off[E], <= moe_max_rows).
 * mode MOE_FFN_SHARED: every row goes through all n_shared experts
 *   (w13 [N_s,2F,d], w2 [N_s,d,F]) and the outputs are summed, unweighted
 *   ("Scaling with experts", A shared expert); seg_off is ignored;
 *   1 <= n_rows <= T. */
#define MOE_FFN_ROUTED 0
#define MOE_FFN_SHARED 1
int moe_expert_ffn(const moe_problem_t* p, int32_t mode, const void* x_rows, int64_t n_rows,
                   const int32_t* seg_off, const void* w13, const void* w2, void* y_rows,
                   void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_expert_ffn (ROUTED) over n_segments row segments instead of E: rows
 * [seg_off[s], seg_off[s+1]) go through expert s % E.  This is the layout of
 * the expert-parallel receive buffer, where every source rank's rows for the
 * local experts arrive as one block (segments source-major, experts in order
 * within each source), so a single message per peer needs no regrouping.
 *   seg_off [n_segments + 1] int32 device, non-decreasing, seg_off[0] = 0,
 *           seg_off[n_segments] <= n_rows <= moe_max_rows(p);
 *   1 <= n_segments <= 256 (else MOE_ERR_UNSUPPORTED).
 * With more segments than experts the rows are first copied into expert order
 * in the workspace (each expert's rows one group, so its tiles are full and
 * its weights stream once per tile column) and the outputs copied back to the
 * segment order of x_rows; the result is that of computing segment by segment.
 * Everything else (weights [E, ...], y_rows, workspace, errors) as
 * moe_expert_ffn; FP32 problems use the CUDA-core path with the same rule.
 * The pages state expert parallelism ("Scaling with experts", What you still
 * pay for); this layout of its receive buffer is this library's. */
int moe_expert_ffn_segments(const moe_problem_t* p, const void* x_rows, int64_t n_rows,
                            const int32_t* seg_off, int32_t n_segments, const void* w13, const void* w2,
                            void* y_rows, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Gate-weighted combine back to token order ("Scaling with experts", The
 * gating network: y = g1 E1(x) + g2 E2(x); A budget: dropped pairs add 0).
 *   y[t] = y_shared[t] + sum_{k: slot_of[t,k] >= 0} topk_w[t,k] * y_perm[slot_of[t,k]]
 * summed in fp32 in that order (shared first, then k ascending), rounded once.
 *   y_perm [*, d]; slot_of [T, K]; topk_w [T, K]; y_shared [T, d] or NULL
 *   (required iff n_shared > 0); y [T, d] out. */
int moe_combine(const moe_problem_t* p, const void* y_perm, const int32_t* slot_of,
                const float* topk_w, const void* y_shared, void* y,
                void* ws, size_t ws_bytes, moe_stream_t stream);

/* The whole layer: route -> dispatch -> routed experts -> shared experts ->
 * combine, plus statistics, enqueued on one stream with no host sync.
 *   x [T, d] in; w weights; y [T, d] out;
 *   routing: optional outputs (NULL or any subset; logits is an input with
 *   MOE_FLAG_LOGITS_GIVEN); stats [2E+1] ([2E+7] with MOE_FLAG_EXTENDED_STATS)
 *   or NULL (as moe_route).
 * Resets the device status word first. */
int moe_layer_forward(const moe_problem_t* p, const void* x, const moe_weights_t* w,
                      void* y, const moe_routing_t* routing, float* stats,
                      void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_dispatch for callers that cannot give the library device memory for
 * scratch: a program whose device-memory budget is fixed up front (all of it
 * owned by its own pool or planner), or a host without a caching allocator,
 * for which a cudaMalloc / cudaFree around each call would synchronise the
 * device.  Same inputs, outputs and results as moe_dispatch, without ws: the
 * scratch (per-chunk histogram and chunk bases) lives in a 1 MiB array of
 * device memory that the library declares, which every GPU that loads the
 * library holds until the process exits.  Limit: 2 * ceil(T/256) * E <= 262144
 * (e.g. T <= 131072 at E = 256, T <= 524288 at E = 64); larger problems return
 * MOE_ERR_UNSUPPORTED and enqueue nothing.  All calls on a GPU share the array:
 * calls whose work overlaps on the GPU race, so serialise them.  The first call
 * on a device looks the array's address up (device current), and so does the
 * first call after the device's context was reset (cudaDeviceReset); make
 * such a call before any stream capture.  Expert indices outside [0, E) are skipped (slot -1) but
 * not reported (there is no status word).  MOE_FLAG_EXPERT_CAPACITY is not
 * accepted here (MOE_ERR_INVALID_ARG).  The pages have no counterpart of
 * this entry point. */
int moe_dispatch_noalloc(const moe_problem_t* p, const int32_t* topk_idx, const void* x,
                         int32_t* counts, int32_t* kept, int32_t* seg_off,
                         int32_t* slot_of, int32_t* perm, void* x_perm, moe_stream_t stream);

/* moe_dispatch with one capacity per expert (Zen MoDE §5.3: capacity_e may
 * differ per expert).  Requires MOE_FLAG_EXPERT_CAPACITY in p (the workspace
 * and moe_max_rows are then sized for T*K rows).
 *   expert_capacity [E] int32 in: expert e keeps the first expert_capacity[e]
 *            of its pairs in token order (negative: no limit); kept[e] =
 *            min(counts[e], expert_capacity[e]).
 * Everything else as moe_dispatch. */
int moe_dispatch_capacity(const moe_problem_t* p, const int32_t* topk_idx, const int32_t* expert_capacity,
                          const void* x, int32_t* counts, int32_t* kept, int32_t* seg_off,
                          int32_t* slot_of, int32_t* perm, void* x_perm,
                          void* ws, size_t ws_bytes, moe_stream_t stream);

/* Load-balancing update after a step, from that step's pre-capacity counts
 * [E] (moe_routing_t.counts).  One kernel, no workspace; either part may be
 * skipped by passing NULL for its output.
 *
 * Selection bias (Zen-Max §2.3 Auxiliary-Loss-Free Load Balancing: after each
 * step an overloaded expert's bias is lowered and an underloaded one's raised;
 * the page fixes neither the load measure nor the step).  Load = counts[e],
 * target = T*K/E, in float64 and rounded once into the float32 bias:
 *   MOE_BIAS_UPDATE_SIGN:         sel_bias[e] += bias_rate * sign(target - load)
 *   MOE_BIAS_UPDATE_PROPORTIONAL: sel_bias[e] += bias_rate * (target - load) / target
 *
 * Adaptive capacity (Zen MoDE §5.3 Adaptive Capacity Factors,
 * C_e = C_base + gamma * (fbar_e - 1/N_E)): count_hist is a ring of hist_len
 * rows of E int32 that this call owns between calls; `step` (0, 1, 2, ...
 * counted by the caller) selects row step % hist_len, where counts are
 * stored.  fbar_e = mean of counts[e] / (T*K) over the min(step+1, hist_len)
 * rows written so far; then
 *   expert_capacity[e] = clamp(ceil(C_e * T*K / E), 0, T)     (float64)
 * for the next step's MOE_FLAG_EXPERT_CAPACITY dispatch.  c_base > 0.
 *
 * Pointers are device pointers (16-byte aligned); sel_bias and
 * expert_capacity are updated in place / written.  Errors: MOE_ERR_INVALID_ARG
 * for NULL counts, both outputs NULL, a non-finite rate / c_base / gamma,
 * c_base <= 0, hist_len < 1, step < 0, an unknown bias_mode, or
 * expert_capacity without count_hist. */
#define MOE_BIAS_UPDATE_SIGN 0
#define MOE_BIAS_UPDATE_PROPORTIONAL 1
int moe_balance_update(const moe_problem_t* p, const int32_t* counts,
                       float* sel_bias, float bias_rate, int32_t bias_mode,
                       int32_t* count_hist, int32_t hist_len, int64_t step,
                       float c_base, float gamma, int32_t* expert_capacity,
                       moe_stream_t stream);

/* Gradients of the layer (device pointers, caller-owned).  FP32 weight
 * gradients in the weights' layouts; each optional one may be NULL. */
typedef struct moe_grads {
    void* dx;            /* [T, d] activations dtype, or NULL */
    float* dw13;         /* [E, 2F, d] (required) */
    float* dw2;          /* [E, d, F] (required) */
    float* dw13_shared;  /* [N_s, 2F, d], NULL iff n_shared == 0 */
    float* dw2_shared;   /* [N_s, d, F],  NULL iff n_shared == 0 */
    float* dw_gate;      /* [E, d] or NULL; must be NULL with MOE_FLAG_LOGITS_GIVEN */
    float* d_offset;     /* [E] or NULL (gradient of logit_offset) */
    float* d_logits;     /* [T, E] or NULL (gradient of the router logits) */
} moe_grads_t;

/* Scratch needed by moe_layer_backward (bytes).  Pure host function. */
int moe_backward_workspace_size(const moe_problem_t* p, size_t* bytes);

/* Backward of moe_layer_forward, for training.  Scaling with experts, "The
 * gating network" (the gate-weighted sum; gradients reach an expert only
 * through the tokens it processed), "A balance penalty"; Zen-Max §2.2
 * (Expert_i), §3.2 (router z-loss).  The routing of the forward is held fixed:
 * the choice of experts and the capacity cut carry no gradient, nor does the
 * selection bias.
 *   x, w     the forward's inputs (unchanged since)
 *   routing  the forward's routing (any NULL member is read from fwd_ws, where
 *            the forward then kept it)
 *   fwd_ws   the forward's workspace, untouched since that call (it holds the
 *            expert inputs, hidden activations and outputs the backward reads)
 *   dy       [T, d] dJ/dy; d_loss, d_zloss: dJ/d(balance loss), dJ/d(z-loss)
 *   grads    outputs (see moe_grads_t); the weight gradients are overwritten
 *   ws       moe_backward_workspace_size bytes, 256-byte aligned
 * Computes in BF16 with FP32 accumulation, like the forward: intermediate
 * gradients (dO, dh -> dg/du, dx rows, the logit gradient fed to the tensor
 * cores) are rounded to BF16, weight gradients accumulate in FP32 in TMEM.
 * The gate and up projections are read from fwd_ws when the forward ran with
 * MOE_FLAG_SAVE_GU (same flags here), else recomputed from the forward's
 * expert inputs.  FP32 problems return MOE_ERR_UNSUPPORTED. */
int moe_layer_backward(const moe_problem_t* p, const void* x, const moe_weights_t* w,
                       const moe_routing_t* routing, const void* fwd_ws, size_t fwd_ws_bytes,
                       const void* dy, float d_loss, float d_zloss, const moe_grads_t* grads,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* Stage boundaries recorded by moe_layer_forward_profiled. */
#define MOE_EV_START 0   /* before the router */
#define MOE_EV_ROUTED 1  /* after gate logits, selection and statistics */
#define MOE_EV_DISPATCHED 2 /* after histogram, scan, rank and gather */
#define MOE_EV_UP 3      /* after the routed up/gate projection with SwiGLU (and the
                            shared experts' one when they share its launch) */
#define MOE_EV_DOWN 4    /* after the routed down projection (and the shared one, ditto) */
#define MOE_EV_SHARED 5  /* after the shared experts (at MOE_EV_DOWN when they ran in
                            the routed launches) */
#define MOE_EV_END 6     /* after the combine */
#define MOE_NUM_EVENTS 7

/* moe_layer_forward, instrumented: additionally records events[i]
 * (cudaEvent_t handles the caller created on the stream's device; NULL
 * entries are skipped) on `stream` at the MOE_EV_* boundaries, so that the
 * time between two events is the time of that stage's kernels.  Stages that
 * do not run for this problem record their event at the same point as the
 * previous one.  With BF16, shared experts and the same expert-GEMM tile
 * shape for the routed and the shared experts, the shared experts run inside
 * the routed up and down launches (their tiles interleaved with the routed
 * ones), so MOE_EV_UP and MOE_EV_DOWN cover both and the shared stage is
 * empty.  *n_kernels (if not NULL) receives the number of kernels the call
 * enqueued.  Same arguments, results and errors as moe_layer_forward. */
int moe_layer_forward_profiled(const moe_problem_t* p, const void* x, const moe_weights_t* w,
                               void* y, const moe_routing_t* routing, float* stats,
                               void* ws, size_t ws_bytes, moe_stream_t stream,
                               void* const* events, int32_t* n_kernels);

/* Stages whose kernels moe_layer_forward_clocked times on the device. */
#define MOE_CLOCK_ROUTE 0    /* gate logits, selection, chunk statistics (the fused router) */
#define MOE_CLOCK_DISPATCH 1 /* scan, capacity, ranks, slots (histogram on moe_dispatch) */
#define MOE_CLOCK_GATHER 2   /* x rows into expert order */
#define MOE_CLOCK_UP 3       /* routed up/gate projection + SwiGLU (and the shared experts'
                                when they share its launch) */
#define MOE_CLOCK_DOWN 4     /* routed down projection (ditto) */
#define MOE_CLOCK_SHARED 5   /* the shared experts' own launches, when they run separately */
#define MOE_CLOCK_COMBINE 6  /* gate-weighted combine */
#define MOE_NUM_CLOCKS 7

/* moe_layer_forward, timed on the device: every BF16 kernel of a stage
 * stamps the global timer (ns) into clocks[2s] and clocks[2s + 1], so that
 * after the forward completes
 *     start_s = ~clocks[2s]   (bitwise complement: the earliest start)
 *     end_s   =  clocks[2s + 1] (the latest end)
 * span the stage's kernels from the first CTA that could read its inputs to
 * the last CTA's end, without the launch gaps an event pair would include.
 *   clocks: DEVICE array of 2 * MOE_NUM_CLOCKS uint64, 8-byte aligned, filled
 *           with zeros by the caller before the call (every stamp is an atomic
 *           max); a stage that did not run, or whose kernels do not stamp
 *           (the FP32 expert GEMMs and gate logits), leaves its pair at zero.
 * Kernel work and results are those of moe_layer_forward; each CTA adds two
 * atomics.  Same arguments and errors, plus MOE_ERR_INVALID_ARG for clocks.
 * This is measurement support, not a step of the pages' method. */
int moe_layer_forward_clocked(const moe_problem_t* p, const void* x, const moe_weights_t* w,
                              void* y, const moe_routing_t* routing, float* stats,
                              void* ws, size_t ws_bytes, moe_stream_t stream, uint64_t* clocks);

/* Expert-parallel exchange plan.  "Scaling with experts", What you still pay
 * for (experts partitioned over devices: a token travels to the device that
 * holds its expert, the output travels back); Zen MoDE §7.2 Communication
 * Overhead (all-to-all between the expert devices).
 *
 * HOST function: every pointer here is a HOST pointer; it enqueues nothing,
 * needs no device and may be called from any thread.
 *
 * n_ranks G >= 1 devices, rank in [0, G); n_experts E with E % G == 0; rank q
 * holds the global experts [q*E_l, (q+1)*E_l), E_l = E/G.  Each rank routes
 * and dispatches its own T tokens with the full router (moe_route +
 * moe_dispatch, the global E), so its kept rows for global expert e are
 * x_perm[seg_off[e] .. seg_off[e+1]).
 *   seg_off_all   [G, E+1] in: row s = rank s's seg_off (each starts at 0 and
 *                 never decreases)
 *   send          [G, 3] out: chunk q = {peer q, first row in this rank's
 *                 x_perm (and, on the way back, y_perm), rows}: the rows of
 *                 the experts peer q holds are contiguous in x_perm, from
 *                 seg_off[q E_l] to seg_off[(q+1) E_l]
 *   recv          [G, 3] out: chunk s = {peer s, first row in the local
 *                 buffer, rows}: source s's block, blocks in rank order
 *   local_seg_off [G * E_l + 1] out: segment s*E_l + el = the rows of local
 *                 expert el from source s, [local_seg_off[i], local_seg_off[i+1])
 *                 -- ready for moe_expert_ffn_segments with n_segments = G E_l
 *                 and the rank's E_l expert weights (segment i uses expert
 *                 i % E_l)
 * Forward: send chunk q of x_perm to peer q, receive chunk s into the local
 * buffer; back: send local chunk s of the expert outputs to s, receive chunk q
 * into y_perm.  One message each way per pair of ranks.  Chunks with 0 rows
 * may be skipped by both sides.
 * Errors: MOE_ERR_INVALID_ARG for NULL pointers, G < 1, rank out of range,
 * E % G != 0, offsets not starting at 0 or decreasing, more than INT32_MAX
 * local rows. */
int moe_ep_plan(int32_t n_ranks, int32_t rank, int32_t n_experts, const int32_t* seg_off_all,
                int32_t* send, int32_t* recv, int32_t* local_seg_off);

/* Expert-parallel exchange over peer memory (the rows and the outputs cross
 * between devices inside the kernels, as loads and stores to peer memory;
 * no copy and no collective on the data path).  Same sources and the same
 * expert placement as moe_ep_plan: rank q of G holds the global experts
 * [q E_l, (q+1) E_l), E_l = E / G; every rank routes and ranks its own T
 * tokens (moe_route, then moe_dispatch with x_perm = NULL).
 *
 * A rank's receive buffer (and its output buffer, row for row) is
 * expert-major: local expert el's rows from source rank 0, then from source 1,
 * ... -- the grouped expert GEMM's order.  Slot j of rank r for global expert
 * e lies at row j + delta_r[e] of the buffers of rank e / E_l.
 *
 * moe_ep_peer_plan (one small kernel on `stream`; no host synchronisation):
 *   seg_off_all   [G, E+1] int32 device in: row s = rank s's seg_off (the
 *                 all-gathered segment offsets; each starts at 0, never
 *                 decreases)
 *   delta         [E] int64 device out: delta_r[e] for rank `rank`
 *   local_seg_off [E_l + 1] int32 device out: the groups of rank `rank`'s
 *                 receive buffer (local expert el: rows [local_seg_off[el],
 *                 local_seg_off[el+1])), ready for moe_expert_ffn (ROUTED) of a
 *                 problem with E_l experts and those weights.
 *   Errors: MOE_ERR_INVALID_ARG for NULL pointers, G < 1, rank out of range,
 *   E > 256 or E % G != 0. */
int moe_ep_peer_plan(int32_t n_ranks, int32_t rank, int32_t n_experts, const int32_t* seg_off_all,
                     int64_t* delta, int32_t* local_seg_off, moe_stream_t stream);

/* moe_ep_scatter: the dispatch's row gather, each kept row written straight
 * into the receive buffer of the rank that holds its expert:
 *   for every slot j < seg_off[E] of this rank, expert e of that slot:
 *     recv_bufs[e / E_l][(j + delta[e]) * d ...] = x[(perm[j] / K) * d ...]
 *   x          [T, d] device in (16-byte aligned); perm, seg_off from this
 *              rank's moe_dispatch; delta [E] int64 device from moe_ep_peer_plan
 *   recv_bufs  [G] device array of device pointers: rank q's receive buffer
 *              (peer memory mapped into this process for q != rank, e.g. by
 *              moe_ipc_open), each [rows q receives, d]
 * The receiving rank may read its buffer once every rank's scatter has
 * completed (the caller orders that, e.g. with a barrier on the stream).
 * Errors: the problem's checks (as moe_dispatch); MOE_ERR_INVALID_ARG for
 * NULL pointers, an x not 16-byte aligned, n_ranks < 1 or E % n_ranks != 0;
 * MOE_ERR_CUDA for a failed launch. */
int moe_ep_scatter(const moe_problem_t* p, int32_t n_ranks, const void* x, const int32_t* perm,
                   const int32_t* seg_off, void* const* recv_bufs, const int64_t* delta,
                   moe_stream_t stream);

/* moe_ep_combine: moe_combine with each kept pair's expert output read from
 * the rank that computed it:
 *   y[t] = y_shared[t] + sum_{k: slot_of[t,k] >= 0} topk_w[t,k] *
 *          out_bufs[e / E_l][(slot_of[t,k] + delta[e]) * d ...],  e = topk_idx[t,k]
 * in moe_combine's order and rounding (shared first, then k ascending, FP32
 * sums, one rounding).  out_bufs [G] device array of device pointers (rank
 * q's output buffer, row for row its receive buffer); y_shared as in
 * moe_combine (NULL iff n_shared == 0); y [T, d] out.  Every rank's expert
 * GEMM must have completed before the call's kernel starts.
 * Errors: the problem's checks; MOE_ERR_INVALID_ARG for NULL pointers, y or
 * y_shared not 16-byte aligned, y_shared given iff n_shared == 0, n_ranks < 1
 * or E % n_ranks != 0; MOE_ERR_CUDA for a failed launch. */
int moe_ep_combine(const moe_problem_t* p, int32_t n_ranks, const void* const* out_bufs,
                   const int64_t* delta, const int32_t* topk_idx, const int32_t* slot_of,
                   const float* topk_w, const void* y_shared, void* y, moe_stream_t stream);

/* Buffers another process can map (CUDA IPC), for the receive and output
 * buffers of moe_ep_scatter / moe_ep_combine across processes:
 *   moe_ipc_malloc  a whole device allocation of `bytes` (so a peer that opens
 *                   its handle maps it at offset 0); free with moe_ipc_free
 *   moe_ipc_handle  its handle, MOE_IPC_HANDLE_BYTES bytes, into `handle` (host)
 *   moe_ipc_open    maps a handle from another process (peer access enabled
 *                   lazily); unmap with moe_ipc_close
 * Errors: MOE_ERR_INVALID_ARG for NULL pointers or 0 bytes; MOE_ERR_CUDA. */
#define MOE_IPC_HANDLE_BYTES 64
int moe_ipc_malloc(size_t bytes, void** ptr);
int moe_ipc_free(void* ptr);
int moe_ipc_handle(const void* ptr, void* handle);
int moe_ipc_open(const void* handle, void** ptr);
int moe_ipc_close(void* ptr);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
