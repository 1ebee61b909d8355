/*
 * moe.h -- C ABI of libmoe: the forward pass of one Mixture-of-Experts layer
 * on one NVIDIA B200 (sm_100a).
 *
 * The layer is the one stated in the cookbook notebook "Mixture-of-experts
 * and expert parallelism" (llm-systems-cookbook, 05_serving/09):
 *
 *   router   (section "Top-k router")          logits = x W_r^T, gates =
 *            softmax(logits), the k largest gates and their experts; the
 *            weights are the raw probabilities (not renormalised).
 *   dispatch (sections "Capacity factor" and "Dispatch and gather")
 *            per-expert counts of the T*k assignments, the slot budget
 *            int(T*k/E*cf), and the grouping of tokens by expert.
 *   experts  (section "Dispatch and gather")    y = fc2(gelu(fc1(x))) with
 *            biased Linear layers and the exact erf GELU.
 *   combine  (section "Dispatch and gather")    out[t] = sum over t's kept
 *            assignments of gate * expert output; 0 when none is kept.
 *   stats    (sections "Capacity factor", "Switch Transformer auxiliary
 *            loss")  imbalance, drop rate and L_aux = E * sum_e f_e p_e.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every tensor is contiguous, row-major, in DEVICE memory owned by the
 *   caller.  The library never frees or keeps a caller pointer after the
 *   call returns.  Tensor base pointers must be 16-byte aligned.
 * - dtype is MOE_F32 (float) or MOE_BF16 (bfloat16 bits in uint16).  It is
 *   the type of x, the router and expert weights and biases, the grouped
 *   activations and the output.  Indices are int32; gates, probability sums
 *   and statistics are float.  Accumulation is always fp32.
 * - Sizes: T >= 0 tokens (T == 0 returns MOE_OK and launches nothing),
 *   1 <= E <= MOE_MAX_EXPERTS experts, 1 <= k <= min(E, MOE_MAX_TOPK),
 *   d and ff positive multiples of 8, T*k < 2^31.
 * - Layouts: x [T,d]; w_router [E,d]; logit_bias [E] float; w1 [E,ff,d];
 *   b1 [E,ff]; w2 [E,d,ff]; b2 [E,d]  (nn.Linear's [out,in] weight layout,
 *   experts stacked on the leading axis).  Assignment a = t*k + j is token
 *   t's j-th choice (j = 0 is the largest gate).
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *   legacy default stream) and never synchronises the host, except
 *   moe_get_error, moe_timing_read, moe_ffn_clock_enable / _read and the
 *   pipeline calls (each says so).  The layer calls are CUDA-graph
 *   capturable.
 * - Errors: argument and shape errors are returned synchronously, before
 *   anything is launched (MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED,
 *   MOE_ERR_WORKSPACE).  A failed launch returns MOE_ERR_CUDA.  Errors that
 *   only the device can see (an expert index outside [0,E) given to
 *   moe_dispatch, a pipeline wait that ran out of time) are recorded in a
 *   per-device error word and reported by moe_get_error; the affected
 *   outputs are then unspecified but every kernel still terminates.
 * - No C++ exception crosses this interface.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define MOE_OK               0
#define MOE_ERR_INVALID_ARG  1  /* null pointer, bad size, k > E, misaligned pointer */
#define MOE_ERR_UNSUPPORTED  2  /* dtype, d or ff not a multiple of 8, E or k above the limits */
#define MOE_ERR_WORKSPACE    3  /* workspace missing or smaller than the size query returns */
#define MOE_ERR_CUDA         4  /* a CUDA runtime call or kernel launch failed */
#define MOE_ERR_BAD_ROUTING  5  /* device: an expert index outside [0, E) */
#define MOE_ERR_TIMEOUT      6  /* device: a bounded pipeline wait gave up */

/* ---- dtypes ------------------------------------------------------------ */
#define MOE_F32   0
#define MOE_BF16  1

#define MOE_MAX_EXPERTS 256
#define MOE_MAX_TOPK    8
#define MOE_MAX_SHARED  8   /* shared always-on experts (moe_forward_ex) */

/* Layer statistics, written to DEVICE memory by moe_forward / moe_layer_stats.
 * Definitions (notebook sections "Capacity factor" and "Switch Transformer
 * auxiliary loss"), with counts taken before any capacity drop:
 *   aux_loss  = E * sum_e (counts_e / T) * (prob_sum_e / T)
 *   imbalance = max_e counts_e / (T*k/E)
 *   drop_rate = dropped / (T*k)
 * With overflow rerouting (moe_forward_ex), rows_kept, dropped and
 * drop_rate count the assignments served after rerouting.              */
typedef struct moe_stats {
    float   aux_loss;
    float   imbalance;
    float   drop_rate;
    int32_t rows_kept;   /* R = sum_e min(counts_e, capacity) */
    int32_t max_count;   /* max_e counts_e */
    int32_t dropped;     /* T*k - R */
    int32_t rerouted;    /* assignments served by a fallback expert (moe_forward_ex
                            with overflow rerouting; 0 otherwise) */
} moe_stats;

/* Human-readable name of a status code (static storage). */
MOE_API const char* moe_status_string(int status);

/* ABI version of this header: major*10000 + minor*100 + patch. */
MOE_API int moe_version(void);

/* Slot budget per expert, int(T*k/E*cf) computed in double (notebook section
 * "Capacity factor"; int() truncates).  cf <= 0 means no limit: returns -1.
 * Returns -1 also for invalid sizes (T < 0, k < 1, E < 1). */
MOE_API int moe_capacity(int T, int k, int E, double cf);

/* Bytes of workspace moe_forward needs for these sizes (0 for invalid
 * arguments).  The workspace holds the routing, the dispatch arrays and the
 * grouped activations xp [T*k,d], h [T*k,ff] and yp [T*k,d]. */
MOE_API size_t moe_workspace_size(int T, int d, int ff, int E, int k, int dtype);

/* Bytes of scratch moe_dispatch needs (per-block expert histograms). */
MOE_API size_t moe_dispatch_workspace_size(int T, int k, int E);

/* Byte offset of one of moe_forward's intermediate arrays inside its
 * workspace, for inspection and testing (the layout may change between
 * versions; query it, do not hard-code it).  `which` is one of the
 * MOE_WS_* values; returns (size_t)-1 for invalid arguments.  After
 * moe_forward completes: topk_idx/topk_gate [T,k] (when the caller passed no
 * output for them), counts [E], offsets [E+1], perm [R], slot_of [T*k],
 * row_gate [R], xp [R,d], h [R,ff]; yp [R,d] only when k > 1. */
#define MOE_WS_TOPK_IDX  0
#define MOE_WS_TOPK_GATE 1
#define MOE_WS_COUNTS    2
#define MOE_WS_OFFSETS   3
#define MOE_WS_PERM      4
#define MOE_WS_SLOT_OF   5
#define MOE_WS_ROW_GATE  6
#define MOE_WS_XP        7
#define MOE_WS_H         8
#define MOE_WS_YP        9
#define MOE_WS_FALLBACK_IDX  10  /* [T,F] moe_forward_ex with F > 0 rerouting rounds */
#define MOE_WS_FALLBACK_GATE 11  /* [T,F] */
MOE_API size_t moe_workspace_offset(int T, int d, int ff, int E, int k, int dtype, int which);

/* ---- step 1: router (notebook section "Top-k router") ------------------
 * logits[t,e] = sum_i x[t,i] w_router[e,i] (+ logit_bias[e]) accumulated in
 * fp32; g = softmax over e in fp32; the k experts with the largest logits,
 * in descending order, an exact tie going to the lower expert index.
 *   x          [T,d] dtype           w_router [E,d] dtype
 *   logit_bias [E] float or NULL     (added to the logits)
 *   topk_idx   [T,k] int32 (out)     topk_gate [T,k] float (out): g at those experts
 *   prob_sum   [E] float or NULL (out): sum over tokens of g[t,e]; it is
 *              overwritten (zeroed on the stream first).
 * Supports E <= MOE_MAX_EXPERTS, k <= MOE_MAX_TOPK. */
MOE_API int moe_router_topk(const void* x, const void* w_router, const float* logit_bias,
                    int T, int d, int E, int k, int dtype,
                    int32_t* topk_idx, float* topk_gate, float* prob_sum,
                    void* stream);

/* ---- step 2: dispatch (notebook sections "Capacity factor", "Dispatch and
 * gather") -----------------------------------------------------------------
 * counts[e]  = #{a : topk_idx[a] == e}                       (before drops)
 * kept_e     = counts[e] if capacity < 0, else min(counts[e], capacity)
 * offsets    = exclusive prefix sum of kept; offsets[E] = R rows kept
 * Expert e keeps its first kept_e assignments in token order; they occupy
 * grouped rows offsets[e] .. offsets[e+1]-1 in that order:
 *   perm[row]   = a of the assignment in that row            (rows < R)
 *   slot_of[a]  = its row, or -1 if the assignment was dropped
 *   drop_mask[a]= 1 if dropped, else 0
 *   row_gate[row] = topk_gate[perm[row]]     (if topk_gate and row_gate are given)
 *   xp[row,:]   = x[perm[row] / k, :]        (if x and xp are given)
 * Every output is produced exactly (integer work, bit-reproducible, no
 * dependence on thread timing).  perm, row_gate and xp are sized for T*k
 * rows; rows >= R are left untouched.
 *   ws/ws_bytes: scratch of at least moe_dispatch_workspace_size(T,k,E).
 * An index outside [0,E) is dropped and raises MOE_ERR_BAD_ROUTING in the
 * device error word. */
MOE_API int moe_dispatch(const int32_t* topk_idx, const float* topk_gate,
                 int T, int k, int E, int capacity,
                 int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* slot_of,
                 uint8_t* drop_mask, float* row_gate,
                 const void* x, void* xp, int d, int dtype,
                 void* ws, size_t ws_bytes, void* stream);

/* ---- dispatch without a workspace -------------------------------------
 * The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory: for example a serving runtime whose
 * allocator has reserved the whole device up front and hands out no extra
 * buffers, or a latency-critical path that must not call cudaMalloc (which
 * can synchronise the device) and has no workspace to pass.
 *
 * Same semantics, arguments and results as moe_dispatch, minus ws/ws_bytes.
 * Its scratch is a fixed array inside the library (1 MiB per GPU, held by
 * every GPU that loads the library until the process exits), so it
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * Limit: T*k <= MOE_NOALLOC_MAX_ASSIGNMENTS; larger calls return
 * MOE_ERR_WORKSPACE (and print why to stderr) before launching anything.
 * The first call on a device looks up the array's device address for that
 * device (cudaGetSymbolAddress, with that device current); make that first
 * call before any stream capture.  The address is kept with the CUDA
 * context it belongs to: after a device reset (cudaDeviceReset) or a
 * re-created primary context, the next call on that device sees a new
 * context and looks the address up again, so that call too belongs before
 * any capture.  All calls share the one array and it
 * keeps the last call's contents (every entry a call reads is written
 * earlier in that call, so nothing needs clearing): calls whose executions
 * overlap on the GPU, on different streams or host threads, race on it and
 * must be serialised by the caller. */
#define MOE_NOALLOC_MAX_ASSIGNMENTS (1 << 20)
MOE_API int moe_dispatch_noalloc(const int32_t* topk_idx, const float* topk_gate,
                                 int T, int k, int E, int capacity,
                                 int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* slot_of,
                                 uint8_t* drop_mask, float* row_gate,
                                 const void* x, void* xp, int d, int dtype, void* stream);

/* ---- step 3: grouped expert FFN (notebook section "Dispatch and gather")
 * For each expert e and each row r in offsets[e] .. offsets[e+1]-1:
 *   h[r,:]  = gelu(xp[r,:] W1_e^T + b1_e)          (exact erf GELU)
 *   yp[r,:] = g_r * (h[r,:] W2_e^T + b2_e),  g_r = row_gate[r] or 1 if NULL
 * offsets is read on the device (no host synchronisation); max_rows is the
 * number of rows xp, h and yp are allocated for (>= offsets[E], normally
 * T*k).  h is caller-provided scratch [max_rows, ff].  bf16 runs on the
 * tcgen05 tensor cores with fp32 accumulation in tensor memory; h and yp are
 * rounded to bf16.  f32 runs on the tensor cores as three-pass TF32 (each
 * operand split into a TF32 part and its fp32 remainder; fp32-level error). */
MOE_API int moe_grouped_ffn(const void* xp, const int32_t* offsets, int max_rows,
                    int E, int d, int ff,
                    const void* w1, const void* b1, const void* w2, const void* b2,
                    const float* row_gate, void* h, void* yp, int dtype,
                    void* stream);

/* ---- step 4: combine (notebook section "Dispatch and gather") ----------
 * out[t,:] = sum_{j<k, slot_of[t*k+j] >= 0} w_tj * yp[slot_of[t*k+j], :]
 * with w_tj = topk_gate[t*k+j], or 1 when topk_gate is NULL (gate already
 * applied by moe_grouped_ffn).  Summed in fp32 in slot order j; a token
 * whose every assignment was dropped gets 0.  out is [T,d] dtype. */
MOE_API int moe_combine(const void* yp, const int32_t* slot_of, const float* topk_gate,
                int T, int k, int d, int dtype, void* out, void* stream);

/* ---- statistics (notebook sections "Capacity factor", "Switch
 * Transformer auxiliary loss") ---------------------------------------------
 * From counts [E], offsets [E+1] (moe_dispatch) and prob_sum [E]
 * (moe_router_topk), writes one moe_stats to DEVICE memory. */
MOE_API int moe_layer_stats(const int32_t* counts, const int32_t* offsets, const float* prob_sum,
                    int T, int k, int E, moe_stats* stats, void* stream);

/* ---- the whole layer ---------------------------------------------------
 * Router -> dispatch -> grouped FFN -> combine (-> stats), all on `stream`,
 * no host synchronisation.  capacity < 0 means no limit (see moe_capacity).
 *   out           [T,d] dtype (out)
 *   stats         one moe_stats in device memory, or NULL
 *   topk_idx_out  [T,k] int32 or NULL: the routing, if the caller wants it
 *   topk_gate_out [T,k] float or NULL
 *   ws/ws_bytes   workspace of at least moe_workspace_size(T,d,ff,E,k,dtype)
 *                 bytes, 256-byte aligned. */
MOE_API int moe_forward(const void* x, const void* w_router, const float* logit_bias,
                const void* w1, const void* b1, const void* w2, const void* b2,
                int T, int d, int ff, int E, int k, int capacity, int dtype,
                void* out, moe_stats* stats,
                int32_t* topk_idx_out, float* topk_gate_out,
                void* ws, size_t ws_bytes, void* stream);

/* ---- extensions: shared experts and overflow rerouting ------------------
 *
 * Shared always-on experts (notebook section "Exercises", item 3): experts
 * that every token passes through beside its routed ones (the DeepSeek-V2
 * arrangement the exercise names).  S in [0, MOE_MAX_SHARED] shared experts
 * of the routed experts' form and shapes, in dtype:
 *   w1s [S,ff,d], b1s [S,ff], w2s [S,d,ff], b2s [S,d]
 *   shared_s(x) = fc2_s(gelu(fc1_s(x)))          (exact erf GELU)
 * Their outputs are added with weight 1 (no gate) to every token, also to
 * tokens whose routed assignments were all dropped.  Routing, dispatch,
 * capacity and the statistics concern the routed experts only.
 * Limits: T*(k+S) < 2^31.  S > MOE_MAX_SHARED returns MOE_ERR_UNSUPPORTED.
 *
 * Overflow rerouting (the blog "MoE Parallelism for Inference", section
 * "Common Bottlenecks", item 1: rejected tokens sent to less busy experts;
 * the cookbook notebook, section "What": overflow dropped or sent to a
 * fallback path).  With F >= 1 rounds and a capacity >= 0, the router also
 * ranks each token's next F experts (its fallbacks, by logit, ties to the
 * lower index).  After the plain dispatch, in round r = 1..F every token
 * that still has a dropped assignment offers its first dropped slot j to
 * its r-th fallback expert c; c accepts offers in token order while it
 * holds fewer than `capacity` rows.  An accepted slot is served by c with
 * gate softmax(logits)[c].  Expert e's grouped rows: its own kept
 * assignments in token order, then those it accepted in round 1 (token
 * order), round 2, ...  A token never uses one expert twice.  Needs
 * k + F <= min(E, MOE_MAX_TOPK); F = 0 (or capacity < 0) is the plain
 * dispatch.  Integer work: exact and independent of thread timing. */

/* Workspace of moe_forward_ex (S = F = 0: moe_workspace_size); 0 if the
 * sizes are invalid. */
MOE_API size_t moe_forward_ex_workspace_size(int T, int d, int ff, int E, int k, int S, int F, int dtype);

/* Byte offset of one moe_forward_ex intermediate (MOE_WS_*) in its
 * workspace.  With S > 0 the h and yp regions hold T*k routed rows, then
 * S*T shared rows (shared expert s, token t at row T*k + s*T + t). */
MOE_API size_t moe_forward_ex_workspace_offset(int T, int d, int ff, int E, int k, int S, int F, int dtype,
                                               int which);

/* The whole layer with shared experts and overflow rerouting:
 *   out[t,:] = sum over t's served slots j of g_tj * expert_{e_tj}(x[t,:])
 *              + sum_{s<S} shared_s(x[t,:])
 * where e_tj / g_tj are the slot's own expert and gate, or its fallback
 * expert and that expert's gate when rerouting served it.  S = 0 and
 * reroute_rounds = 0 is exactly moe_forward.  The shared experts run as S
 * extra row groups (T rows each) inside the same two grouped-FFN launches as
 * the routed experts; the combine adds their rows in fp32 after the routed
 * slots.  Rerouting adds 2 * F small launches to the dispatch.  stats, when
 * given, also reports `rerouted`.  ws: moe_forward_ex_workspace_size(T, d,
 * ff, E, k, S, reroute_rounds, dtype) bytes, 256-byte aligned.  Other
 * arguments as moe_forward. */
MOE_API int moe_forward_ex(const void* x, const void* w_router, const float* logit_bias,
                   const void* w1, const void* b1, const void* w2, const void* b2,
                   int S, const void* w1s, const void* b1s, const void* w2s, const void* b2s,
                   int reroute_rounds,
                   int T, int d, int ff, int E, int k, int capacity, int dtype,
                   void* out, moe_stats* stats,
                   int32_t* topk_idx_out, float* topk_gate_out,
                   void* ws, size_t ws_bytes, void* stream);

/* Step form of overflow rerouting: moe_dispatch with F rounds.
 *   ranked_idx [T, k+F] int32: each token's experts in router order (the
 *     first k are its assignments, the rest its fallbacks; distinct per
 *     row), e.g. moe_router_topk called with k+F;
 *   ranked_gate [T, k+F] float or NULL: their gates.
 * Outputs as moe_dispatch, for the assignments a = t*k + j: counts are the
 * own choices before any drop, offsets / perm / slot_of / drop_mask the
 * final grouped rows, row_gate[row] the gate of the expert that serves the
 * row (so combine with topk_gate = NULL after a gated grouped FFN).
 *   ws/ws_bytes: moe_dispatch_reroute_workspace_size(T, k, F, E) bytes,
 *   256-byte aligned.
 * An own choice outside [0,E) is dropped and raises MOE_ERR_BAD_ROUTING in
 * the device error word; a fallback outside [0,E) is never offered. */
MOE_API size_t moe_dispatch_reroute_workspace_size(int T, int k, int F, int E);
MOE_API int moe_dispatch_reroute(const int32_t* ranked_idx, const float* ranked_gate,
                         int T, int k, int F, int E, int capacity,
                         int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* slot_of,
                         uint8_t* drop_mask, float* row_gate,
                         const void* x, void* xp, int d, int dtype,
                         void* ws, size_t ws_bytes, void* stream);

/* Step form of the shared experts: ys[s*T + t, :] = shared_s(x[t, :]) for
 * s < S, t < T.  h is caller scratch [S*T, ff]; ys is [S*T, d]; both dtype.
 * Same kernels (tensor cores for bf16) as moe_grouped_ffn. */
MOE_API int moe_shared_ffn(const void* x, int T, int d, int ff, int S,
                   const void* w1s, const void* b1s, const void* w2s, const void* b2s,
                   void* h, void* ys, int dtype, void* stream);

/* moe_combine plus the shared experts' rows:
 *   out[t,:] = (moe_combine's value) + sum_{s<S} ys[s*T + t, :]
 * summed in fp32, routed slots first.  ys may be NULL when S == 0. */
MOE_API int moe_combine_shared(const void* yp, const int32_t* slot_of, const float* topk_gate,
                       const void* ys, int S, int T, int k, int d, int dtype, void* out, void* stream);

/* ---- end-to-end pipeline from host memory --------------------------------
 * A pipeline runs the layer (moe_forward_ex) on a sequence of token batches
 * that live in host memory: per step, the batch is copied host -> device,
 * the layer runs, and the output is copied device -> host.  The two copies
 * and the layer run on three streams the pipeline owns, over `depth` lanes
 * (one device input, output and workspace each), so the input copy of
 * step i+1 and the output copy of step i-1 overlap the layer of step i
 * (PCIe is full duplex).  With MOE_PIPELINE_GRAPHS each lane's layer call
 * is captured once into a CUDA graph at creation and replayed per step.
 * The host loop is native: a step costs about ten CUDA runtime calls.
 *
 * moe_pipeline_create:
 *   layer parameters, S, reroute_rounds, T, d, ff, E, k, capacity, dtype:
 *     as moe_forward_ex (device pointers, caller-owned, kept by the
 *     pipeline: they must stay valid and unchanged until destroy);
 *   depth: lanes, 1 <= depth <= MOE_PIPELINE_MAX_DEPTH;
 *   x_dev[depth], out_dev[depth]: device buffers [T, d] of dtype;
 *   ws[depth]: device workspaces of ws_bytes each, ws_bytes >=
 *     moe_forward_ex_workspace_size(T, d, ff, E, k, S, reroute_rounds,
 *     dtype), 256-byte aligned.  All caller-owned; creation zeroes the
 *     input buffers and runs the layer once per lane (warm-up).
 *   flags: 0 or MOE_PIPELINE_GRAPHS;
 *   out: receives the handle.
 * Errors: MOE_ERR_INVALID_ARG / MOE_ERR_WORKSPACE before any CUDA call,
 * moe_forward_ex's own argument errors from the warm-up, MOE_ERR_CUDA.
 *
 * moe_pipeline_run: steps i = 0..n-1 read x_host[i] (T*d elements of dtype)
 * and write out_host[i]; returns once every output is in host memory.
 * Host buffers should be pinned (page-locked) for the copies to overlap;
 * pageable memory gives the same results, with staged copies.  Entries may
 * repeat (the same buffer in several steps).  elapsed_ms (may be NULL)
 * receives the device time from before the first copy to after the last.
 * Not to be called concurrently on one pipeline.
 *
 * moe_pipeline_destroy: waits for the pipeline's streams and frees its
 * streams, events and graphs (not the caller's buffers); NULL is a no-op. */
#define MOE_PIPELINE_GRAPHS     1
#define MOE_PIPELINE_MAX_DEPTH  8
typedef struct moe_pipeline moe_pipeline;
MOE_API int moe_pipeline_create(const void* w_router, const float* logit_bias,
                        const void* w1, const void* b1, const void* w2, const void* b2,
                        int S, const void* w1s, const void* b1s, const void* w2s, const void* b2s,
                        int reroute_rounds, int T, int d, int ff, int E, int k, int capacity, int dtype,
                        int depth, void* const* x_dev, void* const* out_dev, void* const* ws, size_t ws_bytes,
                        int flags, moe_pipeline** out);
MOE_API int moe_pipeline_run(moe_pipeline* p, const void* const* x_host, void* const* out_host, int n,
                     float* elapsed_ms);
MOE_API int moe_pipeline_destroy(moe_pipeline* p);

/* ---- errors, counters, timing -------------------------------------------
 * moe_get_error: synchronises `stream`, then reads and clears the current
 * device's error word.  Returns MOE_OK, MOE_ERR_BAD_ROUTING,
 * MOE_ERR_TIMEOUT, or MOE_ERR_CUDA if the synchronisation itself failed. */
MOE_API int moe_get_error(void* stream);

/* Device GELU forms, for testing: y[i] = GELU(x[i]) (x, y device float[n]).
 * variant 0: 0.5 x (1 + erff(x / sqrt 2)), the fp32 path's form;
 * variant 1: the same with erf by Abramowitz & Stegun eq. 7.1.26 (|error|
 * <= 1.5e-7);
 * variant 2: variant 1 evaluated two values at a time with the paired fp32
 * instructions, the bf16 tensor-core epilogue's form (bit for bit variant
 * 1).  Any other variant: MOE_ERR_INVALID_ARG. */
MOE_API int moe_debug_gelu(const float* x, float* y, int n, int variant, void* stream);

/* Failure-path check: launches one kernel whose bounded wait on a barrier
 * that nothing completes gives up after limit_ns (0 < limit_ns <= 2 s, the
 * limit of the layer's own pipeline waits) and records MOE_ERR_TIMEOUT in
 * the device error word, exactly as a stalled pipeline wait would; the
 * context stays usable.  Read the status with moe_get_error. */
MOE_API int moe_debug_wait_timeout(int64_t limit_ns, void* stream);

/* Number of kernels this library has launched in this process. */
MOE_API uint64_t moe_launch_count(void);

/* Kernel identifiers for moe_timing_read. */
#define MOE_KERNEL_ROUTER   0
#define MOE_KERNEL_COUNT    1
#define MOE_KERNEL_SCAN     2
#define MOE_KERNEL_PERMUTE  3
#define MOE_KERNEL_GATHER   4
#define MOE_KERNEL_FFN1     5
#define MOE_KERNEL_FFN2     6
#define MOE_KERNEL_COMBINE  7
#define MOE_KERNEL_STATS    8
#define MOE_KERNEL_REROUTE  9   /* rerouting rounds (mark + scan kernels) */
#define MOE_NUM_KERNELS     10

/* moe_timing_enable(1): from now on every kernel launch is bracketed by
 * two CUDA events on its stream (events come from a pool created here, not
 * per call).  moe_timing_enable(0) stops recording.  Not thread-safe
 * against concurrent launches from several host threads. */
MOE_API int moe_timing_enable(int enable);

/* Synchronises on the recorded events and returns, per kernel identifier,
 * the summed device time in milliseconds and the number of launches since
 * the last read; then clears the record.  Arrays have MOE_NUM_KERNELS
 * entries; either may be NULL. */
MOE_API int moe_timing_read(double* ms_per_kernel, int64_t* launches_per_kernel);

/* SM clock of the grouped-FFN launches.  The power cap can hold the SM
 * clock well below its maximum within a millisecond, faster than an
 * outside clock sampler (nvidia-smi) follows it, so a tensor-bound launch
 * is read against the clock it actually ran at.  moe_ffn_clock_enable(1)
 * clears the record and makes every later fc1 / fc2 launch of the grouped
 * FFN note, in thread 0 of each CTA, the SM cycle counter and the global
 * nanosecond timer when the CTA starts its tiles and when it is done;
 * moe_ffn_clock_enable(0) stops that.  Both synchronise the device.
 * moe_ffn_clock_read synchronises and writes, for the most recent fc1 (index
 * 0) and fc2 (index 1) launch, the median over its CTAs of cycles per
 * microsecond (sm_mhz[2], MHz) and the time from the first CTA's start to
 * the last one's end (span_us[2]); 0 where no launch was recorded.  Either
 * array may be NULL.  Device-side cost: one load per CTA of each FFN
 * launch, and four stores per CTA while on. */
MOE_API int moe_ffn_clock_enable(int enable);
MOE_API int moe_ffn_clock_read(double* sm_mhz, double* span_us);

/* Profiler annotations (the blog "MoE Parallelism for Inference", section
 * on profiling: look at the router step and the expert passes separately).
 * When on, every entry point that enqueues GPU work opens an NVTX range
 * named after itself ("moe_forward", "moe_dispatch", ...), and every kernel
 * launch inside it a nested range "moe.kernel.<step>" (router, count, scan,
 * permute, gather, ffn1, ffn2, combine, stats, reroute), so that a timeline
 * from Nsight Systems, or from torch.profiler recording NVTX, shows the
 * steps apart.  The ranges mark host time: when the launches were issued.
 * Off by default; on when the environment variable MOE_NVTX is "1" at the
 * library's first check, or after moe_trace_enable(1).  With no profiler
 * attached a range costs next to nothing; off, one atomic load.
 * moe_trace_enable returns the previous setting (0 or 1) and never fails;
 * moe_trace_enabled returns the current one.  Host only: no GPU needed. */
MOE_API int moe_trace_enable(int enable);
MOE_API int moe_trace_enabled(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
