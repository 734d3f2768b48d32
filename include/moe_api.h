/*
 * moe_api.h -- C ABI of libmoe_b200.so: the forward pass of one top-k Mixture-of-Experts
 * SwiGLU FFN layer on one NVIDIA B200 (sm_100a).
 *
 * The layer (page "MoE", llm.rainlin.net, sections 2-4):
 *   r_t      = x_t W_r^T (+ b)                         router logits, fp32 accumulate
 *   p_t      = Softmax(r_t)                            fp32
 *   I_t      = TopK(p_t, K)
 *   alpha_te = p_te / sum_{j in I_t} p_tj              renormalised routing weights
 *   E_e(x)   = W_down^e (SiLU(W_gate^e x) (.) W_up^e x)
 *   y_t      = sum_{e in I_t} alpha_te E_e(x_t) + sigma(w_s^T x_t) E_s(x_t)
 * The shared expert term is optional.  moe_layer_forward can also add the decoder
 * layer's residual h (h_out = h + y, "MoE", section 4) before its single bf16 rounding.
 *
 * Conventions that hold for every entry point:
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise.  The caller
 *     allocates and owns every buffer, including the workspace; the library never
 *     allocates, frees or synchronises.  All work is enqueued on `stream` (a
 *     cudaStream_t passed as void*; NULL is the legacy default stream) and returns
 *     before it completes.
 *   - bf16 tensors are raw bf16 bit patterns (moe_bf16), row-major and contiguous.
 *     Matrix base pointers must be 16-byte aligned (MOE_ERR_ALIGN otherwise).
 *   - Arguments are checked on the host before anything is launched; a negative
 *     status means nothing was enqueued.  MOE_ERR_CUDA means a launch failed.
 *   - Device-side problems (an inconsistent routing table, a wait that ran out of its
 *     time budget) are recorded in a status word inside the workspace; read it with
 *     moe_read_device_status().
 *   - Supported shapes: 1 <= E <= 512, 1 <= K <= min(E, 16), D and f multiples of 128,
 *     128 <= D <= 8192, 128 <= f <= 8192, f_s = 0 or a multiple of 128 up to 8192,
 *     T >= 0 and T*K < 2^31.  Others return MOE_ERR_UNSUPPORTED.
 *   - Calls that share a workspace must not overlap on the GPU (same stream, or
 *     ordered by events).
 *   - The library keeps per-process host caches (TMA tensor maps by base address and
 *     shape, the kernels' shared-memory limits per device) so that a call does little host
 *     work; calls after a cudaDeviceReset are not supported.
 */
#ifndef MOE_API_H
#define MOE_API_H

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

typedef uint16_t moe_bf16; /* bf16 bit pattern */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_ARG = -1,         /* null pointer, negative size, inconsistent arguments */
    MOE_ERR_UNSUPPORTED = -2, /* shape outside the supported set */
    MOE_ERR_ALIGN = -3,       /* a matrix pointer is not 16-byte aligned */
    MOE_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed */
    MOE_ERR_TIMEOUT = -5,     /* device status only: a device wait ran out of its budget */
    MOE_ERR_WORKSPACE = -6,   /* workspace pointer null or smaller than required */
    MOE_ERR_DEVICE = -7       /* device status only: inconsistent routing table seen */
} moe_status;

/* Flags of moe_layer_params.flags and moe_route_ex. */
#define MOE_FLAG_DETERMINISTIC 1u /* combine by a fixed-order gather instead of fp32 atomics */
#define MOE_FLAG_BF16_WEIGHTS 2u  /* round the routing weights to bf16 ("MoE", section 2:
                                     the renormalised scores return to the model dtype) */

/* Router score functions. */
#define MOE_SCORE_SOFTMAX 0 /* p = softmax(r) over all experts ("MoE", section 2) */
#define MOE_SCORE_SIGMOID 1 /* s_e = sigma(r_e) per expert ("1.6 混合专家（MoE）", section 2) */

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
MOE_API int moe_version(void);

/*
 * Bytes of device workspace that moe_layer_forward needs for this shape (it also covers
 * moe_route and moe_grouped_swiglu with the same or smaller sizes).  f_s = 0 when there
 * is no shared expert.  Returns 0 for unsupported shapes.  The workspace must be 256-byte
 * aligned; its contents need no initialisation.
 */
MOE_API size_t moe_workspace_size(int T, int D, int E, int K, int f, int f_s);

/*
 * Router: logits, fp32 softmax, TopK and renormalisation ("MoE", section 2, router
 * equations; "1.6 混合专家（MoE）", section 2, renormalisation worked example).
 *   x            [T, D] bf16 tokens
 *   w_router     [E, D] bf16 router weight W_r (no bias)
 *   logit_bias   [E] fp32 added to the logits before the softmax, or NULL
 *   w_shared_gate[D] bf16 shared-expert gate vector w_s, or NULL
 * Outputs (device, caller-owned):
 *   topk_idx     [T, K] int32 selected experts, by descending probability; ties go to
 *                the lower expert index
 *   topk_w       [T, K] fp32 renormalised weights alpha (sum to 1 per token)
 *   expert_counts[E] int32 rows routed to each expert (overwritten, not accumulated)
 *   shared_gate  [T] fp32 sigma(w_s . x_t); required iff w_shared_gate != NULL
 * The logits are accumulated in fp32 and never rounded to bf16.  Since the softmax is
 * monotone and its denominator cancels in the renormalisation, the selection is made on
 * the logits and alpha_k = exp(r_k - r_max) / sum_{j in I} exp(r_j - r_max).
 * workspace: at least moe_workspace_size(T, D, E, K, 128, 0) bytes.
 */
MOE_API int moe_route(const moe_bf16* x, const moe_bf16* w_router, const float* logit_bias,
              const moe_bf16* w_shared_gate, int T, int D, int E, int K,
              int32_t* topk_idx, float* topk_w, int32_t* expert_counts, float* shared_gate,
              void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_route with the router variants of "1.6 混合专家（MoE）", sections 2-3:
 *   score_mode   MOE_SCORE_SOFTMAX (as moe_route) or MOE_SCORE_SIGMOID (s_e = sigma(r_e))
 *   select_bias  [E] fp32 added to the scores for the TopK selection only (the DeepSeek-V3
 *                bias method: the weights normalise the raw scores), or NULL
 *   flags        MOE_FLAG_BF16_WEIGHTS to round the weights to bf16
 * The weights are alpha_k = score_k / sum_{j in I} score_j; the selection keys are
 * score + select_bias.  Other arguments, outputs and errors as moe_route.
 */
MOE_API int moe_route_ex(const moe_bf16* x, const moe_bf16* w_router, const float* logit_bias,
                         const moe_bf16* w_shared_gate, int T, int D, int E, int K,
                         int score_mode, const float* select_bias, unsigned flags,
                         int32_t* topk_idx, float* topk_w, int32_t* expert_counts,
                         float* shared_gate, void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_route_noalloc: the router step of moe_route (same outputs, same argument rules)
 * for callers that cannot allocate device memory: code hosted by a framework that owns
 * every device allocation and hands its plugins no allocator, or latency-critical code
 * that cannot afford the device-wide synchronisation of cudaMalloc/cudaFree.  The source
 * pages have no counterpart to this entry point; it exists only for such callers.
 *   - It always runs the CUDA-core router kernel.  moe_route runs that same kernel except
 *     for T >= 256 with E a multiple of 128, where it takes the logits from the tensor
 *     cores; there the two sum the logits in different orders, so they agree within the
 *     router's parity tolerances (identical experts except on near-tie tokens, weights
 *     within 1e-3), not bit for bit.
 *   - No workspace argument.  The router's scratch (fp32 logits [T, E+1] and one ticket
 *     per 8 tokens) lives in a 1 MiB array that the library declares in device memory;
 *     every GPU that loads the library holds that 1 MiB until the process exits.
 *   - Limit: 256-byte-rounded 4*T*(E+1) bytes plus 4*ceil(T/8) bytes must fit in 1 MiB
 *     (for example T <= 1019 at E = 256, T <= 2030 at E = 128); larger calls return
 *     MOE_ERR_UNSUPPORTED before anything is enqueued.
 *   - The first call on a device looks up the array's device address (once per device,
 *     with that device current) and keeps it for the life of the process; make that first
 *     call before any stream capture.  Calls after a cudaDeviceReset of that device are
 *     not supported (the array may then live at another address).
 *   - There is no workspace, hence no device status word: nothing is recorded for
 *     moe_read_device_status (the router kernel has no device-side error to report).
 *   - Every call on a device shares the one array and it keeps the last call's contents:
 *     the call clears the tickets itself, but calls whose work overlaps on the GPU (other
 *     streams, other host threads) race on the array and must be serialised by the caller.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
MOE_API int moe_route_noalloc(const moe_bf16* x, const moe_bf16* w_router,
                              const float* logit_bias, const moe_bf16* w_shared_gate,
                              int T, int D, int E, int K, int32_t* topk_idx, float* topk_w,
                              int32_t* expert_counts, float* shared_gate, void* stream);

/*
 * Permutation: group the T*K (token, slot) pairs by expert ("MoE", section 3.2: each
 * routed expert gathers the tokens routed to it).  Row order inside a group is by
 * ascending token (stable).
 *   topk_idx [T, K] int32, topk_w [T, K] fp32 (NULL: sorted_w not written),
 *   expert_counts [E] int32 (as written by moe_route)
 * Outputs:
 *   expert_offsets [E+1] int32: rows of expert e are [offsets[e], offsets[e+1]);
 *                  offsets[E] = T*K
 *   sorted_token   [T*K] int32 token of each row
 *   sorted_w       [T*K] fp32 routing weight of each row (ignored if topk_w is NULL)
 *   slot_to_row    [T*K] int32 row of pair t*K+k (the inverse map)
 * workspace: NULL, or at least moe_workspace_size(T, 128, E, K, 128, 0) bytes (any layer
 * workspace for the same T, E, K qualifies) with its first 256 bytes zero before the
 * first call: it holds the device status word and the per-chunk expert histograms that
 * let many CTAs place T*K > 4096 entries; with NULL one CTA walks every entry.
 * Counts that disagree with topk_idx set MOE_ERR_DEVICE in the device status word of
 * `workspace` when it is not NULL; rows they would push out of the arrays are not written.
 */
MOE_API int moe_permute(const int32_t* topk_idx, const float* topk_w, const int32_t* expert_counts,
                int T, int E, int K, int32_t* expert_offsets, int32_t* sorted_token,
                float* sorted_w, int32_t* slot_to_row, void* workspace, void* stream);

/*
 * moe_permute with an expert capacity ("1.6 混合专家（MoE）", section 三, expert capacity and
 * token dropping): capacity >= 0 keeps only the first `capacity` entries of each expert in
 * ascending token order (see moe_expert_capacity); capacity < 0 is moe_permute.  Then
 *   expert_offsets[e+1] - expert_offsets[e] = min(counts[e], capacity),
 *   expert_offsets[E] = the kept total (<= T*K);
 *   slot_to_row[t*K+k] = -1 for a dropped pair;
 *   sorted_token / sorted_w rows from expert_offsets[E] to T*K are filled with token 0 and
 *   weight 0 (they belong to no group).
 * Other arguments, outputs and errors as moe_permute (expert_counts stay the full counts).
 */
MOE_API int moe_permute_ex(const int32_t* topk_idx, const float* topk_w,
                           const int32_t* expert_counts, int T, int E, int K, long long capacity,
                           int32_t* expert_offsets, int32_t* sorted_token, float* sorted_w,
                           int32_t* slot_to_row, void* workspace, void* stream);

/*
 * Grouped SwiGLU experts ("MoE", section 3 expert equation and section 3.2 expert loop):
 * for every group e and every row r in [offsets[e], offsets[e+1]) with token
 * t = sorted_token[r]:
 *   h_r = SiLU(W_gate^e x_t) (.) (W_up^e x_t)            bf16, fp32 accumulate
 *   v_r = W_down^e h_r                                    fp32 accumulate
 * and then, with w_r = sorted_w[r] (1 when sorted_w is NULL):
 *   out_acc[t, :] += w_r * v_r     (fp32 atomics; out_acc is NOT cleared), and/or
 *   y_sorted[r, :] = w_r * v_r     (fp32 [rows, D], one row per (token, expert) pair)
 * At least one of out_acc / y_sorted must be non-NULL.
 *   x            [T, D] bf16
 *   sorted_token [rows] int32, or NULL for the identity (row r is token r, rows <= T)
 *   expert_offsets [E+1] int32 on the device; offsets[E] = rows
 *   w_gate_up    [E, 2f, D] bf16: rows [0,f) gate, [f,2f) up of each expert
 *   w_down       [E, D, f] bf16
 * `rows` is the number of sorted rows (T*K for routed experts; T for a dense expert
 * given as E = 1, identity tokens and offsets {0, T}).
 * The token rows are gathered from x inside the gate_up kernel (no permuted copy).
 * workspace: at least 256 + 2*rows*f bytes rounded up to 256 (holds h); for example
 * moe_workspace_size(T, D, E, K, f, 0) with K = rows / T rounded up.
 */
MOE_API int moe_grouped_swiglu(const moe_bf16* x, const int32_t* sorted_token,
                       const int32_t* expert_offsets, const float* sorted_w,
                       const moe_bf16* w_gate_up, const moe_bf16* w_down,
                       int T, int rows, int D, int E, int f,
                       float* y_sorted, float* out_acc,
                       void* workspace, size_t ws_bytes, void* stream);

/*
 * Combine back to token order ("MoE", section 4 aggregation; the expert loop's weighted
 * index_add):
 *   out[t, :] = bf16( acc[t, :] + sum_k w_tk * y_sorted[slot_to_row[t*K+k], :]
 *                     + shared_gate[t] * shared_out[t, :] )
 * Every term is optional: out_acc (fp32 [T, D]) NULL -> acc = 0; y_sorted (fp32 [T*K, D])
 * NULL -> no routed sum; topk_w NULL -> w = 1 (y_sorted already weighted); shared_out
 * (bf16 [T, D]) NULL -> no shared term.  The k-sum runs in slot order (deterministic);
 * a pair with slot_to_row = -1 (dropped by an expert capacity, moe_permute_ex) adds nothing.
 */
MOE_API int moe_combine(const float* out_acc, const float* y_sorted, const int32_t* slot_to_row,
                const float* topk_w, const moe_bf16* shared_out, const float* shared_gate,
                int T, int D, int K, moe_bf16* out, void* stream);

/* Every input of one layer call. */
typedef struct moe_layer_params {
    const moe_bf16* x;                /* [T, D] */
    const moe_bf16* w_router;         /* [E, D] */
    const float* logit_bias;          /* [E] or NULL */
    const moe_bf16* w_gate_up;        /* [E, 2f, D] */
    const moe_bf16* w_down;           /* [E, D, f] */
    const moe_bf16* w_shared_gate;    /* [D] or NULL (no shared expert) */
    const moe_bf16* w_shared_gate_up; /* [2 f_s, D] or NULL */
    const moe_bf16* w_shared_down;    /* [D, f_s] or NULL */
    int T, D, E, K, f, f_s;           /* f_s = 0: no shared expert */
    unsigned flags;                   /* MOE_FLAG_* */
    int32_t* topk_idx_out;            /* optional [T, K] copy of the routing, or NULL */
    float* topk_w_out;                /* optional [T, K], or NULL */
    int32_t* expert_counts_out;       /* optional [E], or NULL */
    void* const* step_events;         /* optional: MOE_NUM_STEP_EVENTS cudaEvent_t handles */
    int score_mode;                   /* MOE_SCORE_SOFTMAX (0) or MOE_SCORE_SIGMOID */
    const float* select_bias;         /* [E] selection-only bias, or NULL (see moe_route_ex) */
    const moe_bf16* residual;         /* [T, D] decoder residual h: out = h + y, or NULL */
    /* Expert capacity ("1.6 混合专家（MoE）", section 三, expert capacity and token
     * dropping): capacity_factor > 0 limits every expert to
     * C = moe_expert_capacity(T, K, E, capacity_factor, min_capacity) of its assignments,
     * the first C in ascending token order; the others are dropped and add nothing (the
     * kept weights are not renormalised; a token whose every assignment is dropped gets
     * y = 0, i.e. out = residual).  0: no capacity (dropless, the default). */
    float capacity_factor;
    int min_capacity;                 /* lower bound on C (0: none) */
} moe_layer_params;

/*
 * Expert parallelism ("1.6 混合专家（MoE）", expert parallelism; "Qwen3.8-Flash-Next 架构笔记 ·
 * 04 / FFN & MOE", system costs): the E experts are spread over G devices, rank r holding
 * experts [r*El, (r+1)*El) with El = E / G.  Every rank routes and permutes its own tokens
 * (moe_route, moe_permute); the rows bound for rank d are then the contiguous range
 * [offsets[d*El], offsets[(d+1)*El]) of its expert-sorted order, so dispatch is one
 * all-to-all of the rows gathered into that order (moe_ep_dispatch_rows), with the
 * per-expert counts of those ranges exchanged first ([G, El] int32, counts[d*El + e] to
 * rank d).  The receiving rank groups what it received by expert (moe_ep_recv_layout), runs
 * moe_grouped_swiglu on its El experts gathering the received rows through recv_row
 * (sorted_token = recv_row, expert_offsets = recv_offsets, unweighted, y_sorted output),
 * puts the outputs back into receive order (moe_ep_return_rows) and sends them back with
 * the reverse all-to-all; each source then has its rows' expert outputs in its own sorted
 * order and sums them with moe_combine (y_sorted, slot_to_row, topk_w).  The exchanges
 * themselves are the caller's (NCCL all-to-all over NVLink between one process per GPU).
 */

/* x_sorted[r] = x[sorted_token[r]] for r < rows: the token rows in expert-sorted order,
 * ready to send ([rows, D] bf16, D a multiple of 8).  */
MOE_API int moe_ep_dispatch_rows(const moe_bf16* x, const int32_t* sorted_token, int rows, int D,
                                 moe_bf16* x_sorted, void* stream);

/*
 * Receive side of the dispatch: recv_counts [G, El] (device) holds the rows source s sent for
 * local expert e; the receive buffer holds n = sum(recv_counts) rows, source by source,
 * each source's rows in expert order.  Writes recv_offsets [El+1] (rows of local expert e
 * are [recv_offsets[e], recv_offsets[e+1]) of the expert-major order) and recv_row [n]
 * (expert-major row j reads receive-buffer row recv_row[j]; within an expert, sources in
 * rank order).  G * El <= 512.  workspace: NULL or a layer workspace whose status word
 * records MOE_ERR_DEVICE when the counts do not add up to n -- every group is then empty and
 * recv_row is not written.
 */
MOE_API int moe_ep_recv_layout(const int32_t* recv_counts, int G, int El, int n,
                               int32_t* recv_offsets, int32_t* recv_row, void* workspace,
                               void* stream);

/* y_ret[recv_row[j], :] = y[j, :] for j < n: expert outputs (fp32 [n, D], expert-major, as
 * moe_grouped_swiglu wrote them) back into receive-buffer order for the return all-to-all;
 * D a multiple of 4; a recv_row entry outside [0, n) is skipped. */
MOE_API int moe_ep_return_rows(const float* y, const int32_t* recv_row, int n, int D,
                               float* y_ret, void* stream);

/*
 * The expert capacity the layer applies: max(min_capacity, ceil(capacity_factor * T * K / E))
 * assignments per expert -- the batch's T*K (token, expert) assignments spread over E
 * experts, times the capacity factor (for top-1 routing this is the pages' tokens / experts
 * x capacity_factor).  Computed in double precision.  Returns -1 for capacity_factor <= 0
 * (no capacity) or bad sizes.
 */
MOE_API long long moe_expert_capacity(int T, int K, int E, float capacity_factor,
                                      int min_capacity);

/*
 * Step boundaries at which moe_layer_forward records p->step_events[i] on its stream when
 * step_events is not NULL (events created by the caller; used to time each kernel of the
 * layer; a NULL entry is skipped).  Steps absent from a call (no shared expert) get a
 * zero-length interval.  An event recorded between two kernels stops the second from
 * starting early (programmatic dependent launch), so record only the boundaries needed.
 */
enum {
    MOE_EV_START = 0,    /* before the workspace clear */
    MOE_EV_ROUTER,       /* router (one kernel, or GEMM + selection for T >= 256) */
    MOE_EV_PERMUTE,      /* permutation kernel */
    MOE_EV_GATE_UP,      /* grouped gate_up GEMM + SwiGLU (gathers the token rows) */
    MOE_EV_DOWN,         /* grouped down GEMM + weighted scatter-add */
    MOE_EV_SHARED,       /* shared expert (gate_up and down) */
    MOE_EV_COMBINE,      /* combine to the bf16 output */
    MOE_EV_END,
    MOE_NUM_STEP_EVENTS
};

/*
 * The whole layer: route, permute, grouped SwiGLU (routed experts and, when present, the
 * shared expert scaled by sigma(w_s . x)), combine to out [T, D] bf16 -- plus the residual
 * h when p->residual is set ("MoE", section 4: h_out = h + y_MoE), with the router
 * variants of p->score_mode / p->select_bias / MOE_FLAG_BF16_WEIGHTS and the expert
 * capacity of p->capacity_factor when it is > 0.  No host synchronisation; every step
 * reads its sizes from the device, so the call can be captured in a CUDA graph.
 * workspace: at least moe_workspace_size(T, D, E, K, f, f_s) bytes, 256-byte aligned.
 * Errors: MOE_ERR_ARG / _UNSUPPORTED / _ALIGN / _WORKSPACE from the host checks before
 * anything is enqueued; MOE_ERR_CUDA when a launch fails; device-side problems are left
 * in the workspace's status word (moe_read_device_status).
 * Concurrency: the kernels are persistent (one CTA, or CTA pair, per SM) and the last one
 * converts the output after a grid-wide step that needs all of its CTAs resident; work
 * that holds SMs for seconds on other streams can make that step give up after its 2 s
 * bound, leaving MOE_ERR_TIMEOUT in the status word instead of hanging.
 */
MOE_API int moe_layer_forward(const moe_layer_params* p, moe_bf16* out, void* workspace,
                      size_t ws_bytes, void* stream);

/*
 * What moe_layer_forward runs for these parameters (host only; nothing is launched and no
 * pointer of p is dereferenced, only p's shapes, flags and which pointers are NULL are
 * read).  *step_mask (if not NULL) gets bit MOE_EV_x set for every step whose interval,
 * between step events x and x + 1, launches a kernel: steps that are fused into another
 * step's kernel (the shared expert into the routed launches when it is as wide as the
 * routed experts, the combine into the last down kernel) have their bit clear.  *launches
 * (if not NULL) gets the number of kernels one call launches on the device the caller has
 * current.  Errors as the host checks of moe_layer_forward.
 */
MOE_API int moe_layer_plan(const moe_layer_params* p, unsigned* step_mask, int* launches);

/* Kernels this library has launched in this process so far (all devices, all calls). */
MOE_API unsigned long long moe_launch_count(void);

/*
 * Bound of the layer's grid-wide wait, in nanoseconds (failure detection; no counterpart on
 * the source pages).  The last kernel of moe_layer_forward converts the output only after
 * every CTA of its grid has added its tiles: each CTA takes a ticket and waits for the
 * others for at most this long, and a CTA that gives up records MOE_ERR_TIMEOUT in the
 * workspace's status word and returns without converting its share of the output.
 * Applies to the layer calls enqueued after it, on every device (a CUDA graph keeps the
 * value it was captured with); returns the previous bound.  Default 2000000000 (2 s).
 * 0 makes every CTA but the last to arrive give up at its first look: a way to drive the
 * timeout path, and its report, without a hung or faulted GPU.  The waits inside the
 * kernels' copy/MMA pipelines keep their own fixed 2 s bound.
 */
MOE_API unsigned long long moe_set_grid_wait_budget_ns(unsigned long long ns);

/*
 * Synchronously reads (and clears) the device status word of a workspace after the
 * work on `stream` completes: MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE.  This call
 * synchronises `stream`; it is a diagnostic, not part of the layer.
 */
MOE_API int moe_read_device_status(void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_API_H */
