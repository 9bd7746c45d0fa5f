/*
 * moe.h -- C ABI of libmoe.so: the forward pass of a top-k routed
 * mixture-of-experts (MoE) SwiGLU FFN layer on an NVIDIA B200 (sm_100a).
 *
 * The layer (one token row x of width d):
 *
 *   l_e    = x . W_router[e]                       e = 0..E-1, bias-free
 *   s_e    = softmax(l)_e  or  sigmoid(l_e)        score function
 *   ids    = the k experts with the largest keys, best first; the key is
 *            s_e + b_e with a balance bias b, else s_e (which the library
 *            ranks through l_e: both score functions are increasing in it);
 *            equal keys go to the lower expert index
 *   g_j    = s_{ids_j}, divided by sum_j s_{ids_j} when norm_topk is set
 *   y      = sum_j g_j * W_down[ids_j] (silu(W_gate[ids_j] x) * (W_up[ids_j] x))
 *          + sigmoid(w_s . x) * S_down (silu(S_gate x) * (S_up x))  (shared
 *            expert, only when h_shared > 0)
 *   silu(u) = u * sigmoid(u)
 *
 * Sources: "Tutorial 11: Mixture of Experts (MoE)" -- section 2 "The Router"
 * (route_topk: logits, softmax over all experts, top-k, gather of the kept
 * scores, optional renormalisation), section 3 "Expert Computation" (group
 * rows by expert, grouped expert linears, unsort and weighted sum), section 4
 * "The Complete MoE Layer" (weight shapes); "Small MoE Architecture, in depth"
 * -- section "A small MoE layer in PyTorch" (sigmoid scores, a balance bias
 * that only steers the selection, SwiGLU experts, shared expert added to every
 * token) and the paragraph on auxiliary-loss-free balancing after it;
 * "Mixture-of-Experts -- more capacity per byte of weight", section "What's
 * wired today" (the Switch load-balancing term).  The sigmoid gate on the
 * shared expert and the tie rule are this library's readings where the pages
 * are silent.
 *
 * Conventions for every entry point:
 *  - Tensors are row-major and contiguous, in DEVICE memory owned by the
 *    caller, on the current CUDA device.  The library allocates nothing,
 *    frees nothing and never synchronises the stream; all work is enqueued
 *    on `stream` (a cudaStream_t; NULL is the legacy default stream).
 *  - Element type of x, weights, act and y: bf16 (MOE_BF16) or fp32
 *    (MOE_F32), as cfg->dtype says.  Scores, gates and accumulators are
 *    fp32; ids and permutations are int32.
 *  - Arguments are validated on the host before anything is launched; an
 *    invalid call returns an error and enqueues nothing.  MOE_ERR_CUDA means
 *    a launch failed (cudaGetLastError); the stream may hold earlier work.
 *  - Errors found on the device (an out-of-range expert id handed to
 *    moe_permute, a bounded wait that ran out) set a device flag that
 *    moe_device_status() reads.
 *  - Limits: 1 <= k <= min(E, MOE_MAX_TOPK), 1 <= E <= MOE_MAX_EXPERTS,
 *    d, h and h_shared multiples of 8, T * k < 2^31, T * max(d, h) < 2^40.
 *    Valid shapes outside the limits return MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_MAX_EXPERTS 512
#define MOE_MAX_TOPK 16

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,    /* null pointer, negative size, k outside [1, E], bad enum */
    MOE_ERR_UNSUPPORTED = 2,    /* a valid shape outside the limits above */
    MOE_ERR_WORKSPACE = 3,      /* workspace pointer null or smaller than required */
    MOE_ERR_CUDA = 4,           /* a CUDA call or kernel launch failed */
    MOE_ERR_DEVICE_TIMEOUT = 5, /* a kernel's bounded wait ran out (from moe_device_status) */
    MOE_ERR_DEVICE_INPUT = 6    /* a kernel met an invalid device input (from moe_device_status) */
} moe_status;

typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score_fn;
typedef enum { MOE_BF16 = 0, MOE_F32 = 1 } moe_dtype;
/* How the k expert outputs of a token are summed ("Tutorial 11", section 3,
 * Step 3: unsort, then the gate-weighted sum over the k experts).
 *   MOE_COMBINE_ADD: each expert row is added into an fp32 accumulator by
 *       vector reductions as its tile finishes; the order of the additions
 *       varies from run to run, so y may differ in the last bits.
 *   MOE_COMBINE_ORDERED: each gate-weighted expert row is stored in its own
 *       fp32 slot row (T*k*d floats of workspace), and a final pass adds the
 *       slots of a token in slot order j = 0..k-1, then the shared expert:
 *       y is bit-identical from run to run.  Costs one more write and read
 *       of T*k*d floats.  Applies to the forward combine only (moe_backward
 *       still accumulates dx by reductions). */
typedef enum { MOE_COMBINE_ADD = 0, MOE_COMBINE_ORDERED = 1 } moe_combine_mode;

/* Layer shape and options.  All fields are plain integers so the struct has
 * one layout in every language binding. */
typedef struct {
    int64_t T;         /* tokens (rows of x and y); 0 is allowed and does nothing */
    int32_t d;         /* model width */
    int32_t E;         /* routed experts */
    int32_t h;         /* hidden width of each routed expert */
    int32_t k;         /* experts per token */
    int32_t norm_topk; /* nonzero: divide the k gates by their sum */
    int32_t score;     /* moe_score_fn */
    int32_t h_shared;  /* hidden width of the always-on shared expert; 0 = none */
    int32_t dtype;     /* moe_dtype of x, the weights, act and y */
    int32_t combine;   /* moe_combine_mode; 0 (MOE_COMBINE_ADD) by default */
} moe_config;

/* Device pointers into a moe_forward workspace (see moe_workspace_layout).
 * Pointers of absent parts are NULL. */
typedef struct {
    int32_t *ids;         /* [T, k]  selected experts, best first */
    float *gates;         /* [T, k]  gate of each selected expert */
    float *shared_gate;   /* [T]     sigmoid(w_s . x); NULL without a shared expert */
    int32_t *counts;      /* [E]     assignments per expert */
    int32_t *offsets;     /* [E + 1] exclusive prefix sum of counts */
    int32_t *sorted_rows; /* [T*k]   assignments r = t*k + j grouped by expert, stable */
    int32_t *inv_rows;    /* [T*k]   inverse permutation: inv_rows[sorted_rows[i]] = i */
    void *act;            /* [T*k, h] silu(gate)*up rows in grouped order (dtype) */
    void *act_shared;     /* [T, h_shared] shared-expert activations; NULL if absent */
    float *y_acc;         /* [T, d]  fp32 accumulator (scratch: undefined after the
                             call); NULL when dtype is MOE_F32 */
    float *y_slots;       /* [T*k, d] fp32 gate-weighted expert rows by assignment
                             r = t*k + j (MOE_COMBINE_ORDERED only; else NULL) */
} moe_workspace_views;

/* Options of the routing step for training; every field is optional (NULL
 * turns it off) and so is the struct (opts == NULL turns all off).  Both
 * pointers are device memory owned by the caller.
 *   balance_bias [E] fp32: added to the scores only to choose the top k; the
 *       gates still come from the unbiased scores ("Small MoE Architecture,
 *       in depth", SmallMoE.forward and the auxiliary-loss-free balancing
 *       paragraph after it).  Update it after a step with moe_update_bias.
 *   score_mean [E] fp32, out: P_e = (1/T) sum_t s_e(t), the mean over the T
 *       tokens of each expert's score (the whole score row, before
 *       selection): the router statistic of the Switch load-balancing term
 *       (moe_balance_loss).  Added in a fixed order, so repeated calls give
 *       identical bits. */
typedef struct {
    const float *balance_bias;
    float *score_mean;
} moe_route_opts;

/* Human-readable name of a status code (static storage; never NULL). */
const char *moe_status_string(moe_status status);

/* Checks a configuration against the rules and limits above (host only). */
moe_status moe_validate(const moe_config *cfg);

/* Bytes of device workspace that moe_forward needs for cfg (host only).
 * The same workspace also serves moe_combine. */
moe_status moe_workspace_size(const moe_config *cfg, size_t *bytes);

/* Carves a workspace of ws_bytes bytes at device address ws into the named
 * parts that moe_forward fills (host only; nothing is read or written on the
 * device).  ws must be 256-byte aligned. */
moe_status moe_workspace_layout(const moe_config *cfg, void *ws, size_t ws_bytes,
                                moe_workspace_views *views);

/* Router: logits, scores, top-k selection and gates for all T tokens.
 *   opts     routing options (balance bias, score statistic), or NULL
 *   x        [T, d]        dtype
 *   w_router [E, d]        dtype
 *   w_shared_gate [d]      dtype, or NULL (then shared_gate must be NULL)
 *   ids      [T, k] int32  out: selected experts, best first
 *   gates    [T, k] fp32   out
 *   probs    [T, E] fp32   out, optional (NULL): every expert's score s_e
 *   shared_gate [T] fp32   out, optional: sigmoid(w_s . x)
 *   ws, ws_bytes: device scratch of at least moe_route_workspace_size(cfg)
 *            bytes, 256-byte aligned
 * "Tutorial 11", section 2 (route_topk); "Small MoE Architecture, in depth",
 * forward of SmallMoE (sigmoid scores, balance bias, gates from the raw
 * scores). */
moe_status moe_route(const moe_config *cfg, const moe_route_opts *opts, const void *x,
                     const void *w_router, const void *w_shared_gate, int32_t *ids, float *gates,
                     float *probs, float *shared_gate, void *ws, size_t ws_bytes, void *stream);

/* Bytes of scratch that moe_route needs for cfg (host only). */
moe_status moe_route_workspace_size(const moe_config *cfg, size_t *bytes);

/* Balance-bias update after a training step ("Small MoE Architecture, in
 * depth", SmallMoE.forward in training, and the auxiliary-loss-free balancing
 * paragraph after it): with load_e = counts[e] and mean = sum(counts) / E,
 *   bias[e] += lr * sign(mean - load_e)
 * so an expert above the mean load loses lr, one below it gains lr and one at
 * the mean keeps its bias (the comparison is exact, in integers).
 *   counts [E] int32 (from moe_permute, or the workspace after moe_forward);
 *   bias   [E] fp32, updated in place (fp32 add, round to nearest).
 *   lr must be finite, else MOE_ERR_INVALID_ARG. */
moe_status moe_update_bias(const moe_config *cfg, const int32_t *counts, float lr, float *bias,
                           void *stream);

/* The Switch load-balancing term ("Mixture-of-Experts -- more capacity per
 * byte of weight", "What's wired today"):
 *   loss = alpha * E * sum_e f_e * P_e,   f_e = counts[e] / T
 * (f_e: the fraction of the T tokens dispatched to expert e; P_e: the mean
 * score from moe_route_opts.score_mean).  fp32; the sum over experts is a
 * fixed tree, so repeated calls give identical bits.
 *   counts [E] int32; score_mean [E] fp32; frac [E] fp32 out (f_e) or NULL;
 *   loss [1] fp32 out.  T = 0 gives f = 0 and loss = 0.  alpha must be
 *   finite, else MOE_ERR_INVALID_ARG. */
moe_status moe_balance_loss(const moe_config *cfg, const int32_t *counts, const float *score_mean,
                            float alpha, float *frac, float *loss, void *stream);

/* Grouping: counts, offsets and the stable permutation of the T*k
 * assignments by expert, and its inverse.
 *   ids         [T, k] int32 in [0, E)   (an id outside sets MOE_ERR_DEVICE_INPUT on
 *                                          the device flag, publishes empty experts
 *                                          and leaves sorted_rows/inv_rows unwritten)
 *   counts      [E] int32 out;  offsets [E + 1] int32 out (offsets[0] = 0)
 *   sorted_rows [T*k] int32 out: for each expert in turn, its assignments
 *               r = t*k + j in increasing r
 *   inv_rows    [T*k] int32 out: inv_rows[sorted_rows[i]] = i
 *   ws, ws_bytes: device scratch of at least moe_permute_workspace_size(cfg)
 *               bytes, 16-byte aligned, overlapping no other argument
 * "Tutorial 11", section 3, Step 1 (argsort of the flattened ids; the unsort
 * index of Step 3 is inv_rows). */
moe_status moe_permute(const moe_config *cfg, const int32_t *ids, int32_t *counts,
                       int32_t *offsets, int32_t *sorted_rows, int32_t *inv_rows, void *ws,
                       size_t ws_bytes, void *stream);

/* Bytes of scratch that moe_permute needs for cfg (host only). */
moe_status moe_permute_workspace_size(const moe_config *cfg, size_t *bytes);

/* Grouped gate/up projection with the SwiGLU product fused:
 *   act[i, :] = silu(W_gate[e] x_t) * (W_up[e] x_t)   for grouped row i of
 *   expert e, where t = sorted_rows[i] / k.
 *   x [T, d]; w_gate, w_up [E, h, d]; offsets [E + 1]; sorted_rows [T*k];
 *   act [T*k, h] out (dtype), grouped order.  Rows of x are read in place by
 *   index: no copy of x or of any weight is made.
 * "Tutorial 11", section 3, Step 2 (grouped_expert_linear for gate and up,
 * silu(gate) * up); the expert of "Small MoE Architecture, in depth". */
moe_status moe_grouped_swiglu(const moe_config *cfg, const void *x, const void *w_gate,
                              const void *w_up, const int32_t *offsets,
                              const int32_t *sorted_rows, void *act, void *stream);

/* Grouped down projection fused with the gate-weighted combine:
 *   y[t, :] = sum over the k assignments r = t*k + j of gates[r] * W_down[e] act[inv(r), :]
 *   act [T*k, h] (dtype, grouped order); w_down [E, d, h]; offsets [E + 1];
 *   sorted_rows [T*k]; gates [T, k] fp32; y [T, d] out (dtype, overwritten).
 *   ws / ws_bytes: with MOE_COMBINE_ADD, for MOE_BF16 an fp32 accumulator
 *   of T*d floats is needed, for MOE_F32 ws may be NULL, and the summation
 *   order over the k experts is not fixed; with MOE_COMBINE_ORDERED, T*k*d
 *   floats of slot rows are needed (either dtype) and the k rows of a token
 *   are added in slot order.  Any workspace of moe_workspace_size bytes works.
 * "Tutorial 11", section 3, Steps 2-3 (grouped down linear, unsort, weighted
 * sum over the k experts). */
moe_status moe_combine(const moe_config *cfg, const void *act, const void *w_down,
                       const int32_t *offsets, const int32_t *sorted_rows, const float *gates,
                       void *y, void *ws, size_t ws_bytes, void *stream);

/* moe_combine without a workspace, for callers that cannot allocate device
 * memory (for example a plugin inside an engine that pre-plans all device
 * memory, or code under a fixed memory budget).  The pages have no
 * counterpart: this is an interface choice of this library.
 *   Same arguments and result as moe_combine, minus ws / ws_bytes.  For
 *   MOE_BF16 the fp32 accumulator is a static device array of
 *   MOE_NOALLOC_MAX_ACC_FLOATS floats (16 MiB) that every GPU loading the
 *   library holds until exit; T * d above that limit returns
 *   MOE_ERR_WORKSPACE and enqueues nothing.  With MOE_COMBINE_ORDERED the
 *   same array holds the T*k*d floats of slot rows (either dtype), and the
 *   limit applies to T*k*d.  The call allocates nothing and
 *   calls no allocating routine.
 *   The first call on a device looks up the array's device address (a
 *   one-time, per-device set-up with that device current).  With CUDA's lazy
 *   module loading (the default) that look-up is also when the driver loads
 *   this part of the library onto the device and backs the array with device
 *   memory, so the first call may allocate: make it at start-up, outside any
 *   region that must not allocate and before any stream capture.  Later
 *   calls allocate nothing.  All calls share the array, whose contents are
 *   undefined between calls: each call clears the part it uses, and calls
 *   that overlap on the GPU (unordered streams) race on it. */
#define MOE_NOALLOC_MAX_ACC_FLOATS (4u << 20)
moe_status moe_combine_noalloc(const moe_config *cfg, const void *act, const void *w_down,
                               const int32_t *offsets, const int32_t *sorted_rows, const float *gates,
                               void *y, void *stream);

/* The whole layer: route, group, grouped SwiGLU, down projection and combine,
 * plus the shared expert when cfg->h_shared > 0.
 *   opts: routing options (balance bias, score statistic) or NULL;
 *   x [T, d]; w_router [E, d]; w_gate, w_up [E, h, d]; w_down [E, d, h];
 *   sh_gate, sh_up [h_shared, d], sh_down [d, h_shared], w_shared_gate [d]
 *   (all four NULL when h_shared == 0); y [T, d] out (dtype).
 *   ws: device workspace of at least moe_workspace_size(cfg) bytes, 256-byte
 *   aligned; afterwards it holds the routing results (moe_workspace_layout).
 * "Tutorial 11", section 4 (Moe.__call__); "Small MoE Architecture, in
 * depth", SmallMoE.forward (shared expert). */
moe_status moe_forward(const moe_config *cfg, const moe_route_opts *opts, const void *x,
                       const void *w_router, const void *w_gate, const void *w_up, const void *w_down,
                       const void *sh_gate, const void *sh_up, const void *sh_down,
                       const void *w_shared_gate, void *y, void *ws, size_t ws_bytes,
                       void *stream);

/* moe_forward for inputs and outputs in host memory: x_host [T, d] is copied
 * in and y_host [T, d] out by the call, in n = min(chunks, T, 256) pieces of
 * consecutive tokens.  With n >= 3 the first and last pieces hold half as
 * many tokens as the others (their copies are the ones no layer hides):
 * piece i is tokens [T c_i / (2n - 2), T c_(i+1) / (2n - 2)) with c_0 = 0,
 * c_i = 2i - 1 for 0 < i < n, c_n = 2n - 2 (integer division); with n <= 2,
 * tokens [T i / n, T (i + 1) / n).  Piece i's layer (moe_forward on its tokens,
 * without routing options) runs on `stream` once its rows are on the device,
 * and its y goes back on `copy_stream` while later pieces compute, so the
 * copies overlap the layer; each token's result is that of moe_forward on
 * its piece (the layer treats tokens independently; only the split of the
 * router's reductions can differ with the token count).  All copies to the
 * device are issued first.  More pieces hide more of the copies but re-read
 * the expert weights once per piece.
 *   x_host, y_host: page-locked host memory (pageable memory works, but its
 *   copies do not overlap); weights as for moe_forward, on the device.
 *   chunks >= 1 (more than T acts as T, more than 256 as 256); copy_stream: a
 *   second stream, or NULL to issue the copies on `stream` (no overlap).
 *   ws: device workspace of at least moe_forward_host_workspace_size(cfg,
 *   chunks) bytes, 256-byte aligned (the device copies of x and y, then the
 *   layer's workspace for the largest piece).
 * The call returns once everything is queued; when `stream` reaches the
 * point of the call's end, y_host is complete (the copy stream's last copy
 * is made a dependency of `stream`).  Events are created and destroyed by
 * the call; no device memory is allocated.  Overlapping calls that share ws
 * race on it. */
moe_status moe_forward_host_workspace_size(const moe_config *cfg, int32_t chunks, size_t *bytes);
moe_status moe_forward_host(const moe_config *cfg, const void *x_host, const void *w_router,
                            const void *w_gate, const void *w_up, const void *w_down,
                            const void *sh_gate, const void *sh_up, const void *sh_down,
                            const void *w_shared_gate, void *y_host, int32_t chunks, void *ws,
                            size_t ws_bytes, void *stream, void *copy_stream);

/* ---- training: the forward pass that keeps what the backward needs, and the
 * backward pass.  bf16 layers only (MOE_F32 returns MOE_ERR_UNSUPPORTED).
 * The pages train this layer ("Small models, sparse experts", "Dispatch
 * decides everything" quotes training tokens/s; "Small MoE Architecture, in
 * depth", SmallMoE) but print no backward: the gradient here is the chain rule
 * through the forward's steps.  The top-k selection (and the balance bias)
 * passes no gradient. */

/* Bytes of the workspace of one training step (moe_forward_train followed by
 * moe_backward on the same workspace; host only). */
moe_status moe_train_workspace_size(const moe_config *cfg, size_t *bytes);

/* moe_forward for training: the same arguments and output, plus it keeps in
 * ws what moe_backward needs (every token's score row and each grouped row's
 * pre-activations W_gate x and W_up x, in bf16).  It always takes the
 * tensor-core path.  ws: at least moe_train_workspace_size(cfg) bytes,
 * 256-byte aligned; pass it unchanged to moe_backward. */
moe_status moe_forward_train(const moe_config *cfg, const moe_route_opts *opts, const void *x,
                             const void *w_router, const void *w_gate, const void *w_up,
                             const void *w_down, const void *sh_gate, const void *sh_up,
                             const void *sh_down, const void *w_shared_gate, void *y, void *ws,
                             size_t ws_bytes, void *stream);

/* Gradients of the layer, given dy = dL/dy [T, d] (bf16), after
 * moe_forward_train with the same inputs on the same workspace ws:
 *   dx [T, d] bf16;  dw_router [E, d] fp32;  dw_gate, dw_up [E, h, d] bf16;
 *   dw_down [E, d, h] bf16;  with a shared expert dsh_gate, dsh_up [h_s, d]
 *   and dsh_down [d, h_s] bf16 and dw_shared_gate [d] fp32 (else NULL).
 * Every output is overwritten (an expert that received no rows gets a zero
 * gradient).  Accumulation is fp32; the routed rows' gradients reach the
 * weights in grouped order, dx through fp32 additions in token order (their
 * order over the k experts is not fixed).  ws also serves as the backward's
 * scratch, so it no longer holds the forward's activations afterwards. */
moe_status moe_backward(const moe_config *cfg, const void *x, const void *w_router,
                        const void *w_gate, const void *w_up, const void *w_down,
                        const void *sh_gate, const void *sh_up, const void *sh_down,
                        const void *w_shared_gate, const void *dy, void *ws, size_t ws_bytes,
                        void *dx, float *dw_router, void *dw_gate, void *dw_up, void *dw_down,
                        void *dsh_gate, void *dsh_up, void *dsh_down, float *dw_shared_gate,
                        void *stream);

/* ---- 4-bit routed experts ("Small MoE Architecture, in depth": "Worked
 * example: the batch-1 budget on a device" -- 4-bit weights, about half a
 * byte per parameter, so a decode step reads a quarter of the bf16 bytes --
 * and "Running experts that do not fit: offloading and quantisation" --
 * routed experts quantised, shared expert and router kept at higher
 * precision).  The pages fix no format; this library's: a weight matrix
 * [rows, cols] (cols a multiple of 64) is cut into groups of 64 consecutive
 * elements of a row; scale s = max|w| / 7 (fp32); code = round(w / s) in
 * [-7, 7], ties to even, both decided in fp32; stored as the nibble code + 8,
 * two per byte, the even element in the low nibble.  The value represented
 * is (nibble - 8) * s. */

/* Quantises w [rows, cols] (device, dtype MOE_BF16 or MOE_F32, cols a
 * multiple of 64, else MOE_ERR_UNSUPPORTED) into q [rows, cols / 2] bytes and
 * scales [rows, cols / 64] fp32 (device, caller-owned; w and q 16-byte
 * aligned).  For a layer: W_gate and W_up as [E * h, d], W_down as [E * d, h]. */
moe_status moe_quantize_q4(const void *w, int32_t dtype, int64_t rows, int32_t cols, uint8_t *q,
                           float *scales, void *stream);

/* moe_forward with 4-bit routed experts (q_* / s_* from moe_quantize_q4 of
 * W_gate, W_up [E * h, d] and W_down [E * d, h]); x, the router and the shared
 * expert stay bf16.  Served by the small-batch kernels, which stream the
 * chosen experts' 4-bit rows once: T * k <= moe_decode_max_rows(), bf16, d and
 * h multiples of 64 (else MOE_ERR_UNSUPPORTED).  ws: moe_workspace_size(cfg)
 * bytes.  The result is the layer evaluated on the represented weights. */
moe_status moe_forward_q4(const moe_config *cfg, const moe_route_opts *opts, const void *x,
                          const void *w_router, const uint8_t *q_gate, const float *s_gate,
                          const uint8_t *q_up, const float *s_up, const uint8_t *q_down,
                          const float *s_down, const void *sh_gate, const void *sh_up,
                          const void *sh_down, const void *w_shared_gate, void *y, void *ws,
                          size_t ws_bytes, void *stream);

/* Largest T*k that moe_forward serves with the CUDA-core small-batch kernels
 * (one warp per weight row, weights streamed once); larger batches use the
 * tensor-core grouped GEMM. */
int32_t moe_decode_max_rows(void);

/* Stages of moe_forward, in launch order. */
typedef enum {
    MOE_STAGE_ROUTE = 0,
    MOE_STAGE_PERMUTE = 1,
    MOE_STAGE_GATE_UP = 2,
    MOE_STAGE_SHARED_GATE_UP = 3,
    MOE_STAGE_DOWN = 4,
    MOE_STAGE_SHARED_DOWN = 5,
    MOE_STAGE_FINALIZE = 6,
    MOE_STAGE_COUNT = 7
} moe_stage;

/* Profiling hook for the calling host thread.  With events != NULL (n must be
 * MOE_STAGE_COUNT + 1 cudaEvent_t handles, created by the caller), every later
 * moe_forward (or moe_forward_q4) call on this thread records events[0] on its stream before its
 * first launch and events[i + 1] after stage i; a stage that does not run
 * records an empty interval.  events == NULL turns the hook off.  Host only. */
moe_status moe_profile_events(void *const *events, int32_t n);

/* NVTX ranges for the calling host thread: with on != 0, every later
 * moe_forward (or moe_forward_q4) call on this thread opens an NVTX range
 * named "moe <stage>" around the launches of each stage, so a profiler that
 * records NVTX shows which host calls issued which kernels.  on == 0 turns
 * them off (the default).  Host only; never fails. */
moe_status moe_profile_nvtx(int32_t on);

/* Number of kernels this library has launched in this process (all threads). */
int64_t moe_launch_count(void);

/* Synchronises `stream`, then reads and clears the current device's error
 * flag: MOE_ERR_DEVICE_TIMEOUT or MOE_ERR_DEVICE_INPUT if a kernel set it
 * since the last call, MOE_OK otherwise, MOE_ERR_CUDA if the stream itself
 * reports an error.  Blocking; meant for tests and debugging. */
moe_status moe_device_status(void *stream);

/* Self-test of the device failure path (the pages have no counterpart; it
 * exists so the timeout path can be exercised without faulting a GPU).
 * Enqueues on `stream` one kernel whose mbarrier wait can never complete,
 * through the same bounded wait the tensor-core kernels use, with a limit of
 * limit_ms milliseconds (1..10000).  When it runs out the kernel raises the
 * device flag and returns: the next moe_device_status() reports
 * MOE_ERR_DEVICE_TIMEOUT, and the context and stream stay usable.
 * Returns MOE_ERR_INVALID_ARG for a limit outside the range, MOE_ERR_CUDA if
 * the launch failed, MOE_OK otherwise. */
moe_status moe_selftest_wait_timeout(uint32_t limit_ms, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
