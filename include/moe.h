/*
 * moe.h -- C ABI of the sparsely-gated Mixture-of-Experts FFN layer for one
 * NVIDIA B200 (sm_100a).  Library: sparse_mixture_experts_10_b200/libmoe.so.
 *
 * The layer computes, for every token row x of a batch (Shazeer et al. 2017,
 * as explained in the qiita article "Outrageously Large Neural Networks",
 * section "Sparsely-Gated MoE layer formula"):
 *
 *     y = sum_{i in TopK(x)} G(x)_i * E_i(x),   G(x) = softmax(KeepTopK(x W_g, k))
 *
 * with only the selected experts evaluated.  The argument names follow the
 * Config of the page "MoE(Mixture of Experts)" (sharin-2a1.pages.dev/parts/moe),
 * section (1): DModel, DHidden, NExperts, TopK.
 *
 * Conventions for every entry point
 *  - Pointers named as device buffers are CUDA device memory owned by the
 *    caller.  The library never allocates or frees memory, never keeps a
 *    pointer after a call returns, and never synchronises the stream except in
 *    moe_get_device_status().  Work is enqueued on `stream` (a cudaStream_t;
 *    NULL = the legacy default stream) and runs asynchronously.
 *  - Arrays are row-major and contiguous; leading dimensions are implied by
 *    the shapes given.  "dtype" arrays hold fp32 (MOE_F32) or bf16 (MOE_BF16)
 *    elements as selected by moe_config.dtype; biases are always fp32.
 *  - bf16 layers need DModel and DHidden to be multiples of 8 (16-byte rows
 *    for the tensor-memory-accelerator copies); fp32 layers need multiples of 4.
 *  - Return value: MOE_OK (0) or a negative MOE_ERR_* code.  Argument errors
 *    are found on the host before anything is enqueued.  Errors raised inside
 *    kernels (a bounded wait that ran out, an index out of range) are sticky in
 *    a device status word read by moe_get_device_status().
 *  - Results are deterministic: the same inputs give bitwise-identical
 *    outputs on the same GPU.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream); declared opaquely so that this
 * header does not need the CUDA headers. */
typedef struct CUstream_st *moe_stream_t;

/* Element types of x, the weight matrices and the hidden activations. */
enum { MOE_F32 = 0, MOE_BF16 = 1 };

/* Expert FFN kinds.
 *  MOE_ACT_GELU   GPT-2 FFN ("Extending Raschka's GPT-2: an MoE trained from
 *                 scratch on an RTX 3090", section on how MoE works):
 *                 E(x) = W2 gelu(W1 x + b1) + b2, exact-erf GELU.
 *  MOE_ACT_SWIGLU SwiGLU FFN with the packed gate_up weight (Transformers-v5
 *                 MoE article, section 1 "Weight Loading Refactor": experts
 *                 stacked on dim 0, gate then up concatenated on dim 1):
 *                 E(x) = W_down (silu(W_gate x) * (W_up x)). No biases. */
enum { MOE_ACT_GELU = 0, MOE_ACT_SWIGLU = 1 };

/* Return codes. */
enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,         /* null required pointer, bad size or shape */
    MOE_ERR_WORKSPACE_TOO_SMALL = -2, /* ws_bytes < the size the query returned */
    MOE_ERR_UNSUPPORTED = -3,         /* dtype / act / size combination not built */
    MOE_ERR_CUDA = -4,                /* a CUDA runtime call or launch failed */
    MOE_ERR_DEVICE_TIMEOUT = -5,      /* a kernel's bounded wait ran out (status word) */
    MOE_ERR_DEVICE_BOUNDS = -6        /* a kernel found an index out of range (status word) */
};

/* Bits of the device status word (moe_get_device_status). */
enum {
    MOE_STATUS_TIMEOUT = 1,   /* a bounded wait gave up; the kernel returned early */
    MOE_STATUS_BOUNDS = 2,    /* an expert index or row count was out of range */
    MOE_STATUS_NAN_LOGIT = 4  /* a NaN router logit was ranked as -inf (not fatal) */
};

/* Layer shape ("MoE(Mixture of Experts)", section (1), Config). */
typedef struct {
    int32_t DModel;   /* D: token width */
    int32_t DHidden;  /* H: expert hidden width */
    int32_t NExperts; /* N: number of experts, 1..1024 */
    int32_t TopK;     /* K: experts per token, 1..min(N, 32) */
    int32_t act;      /* MOE_ACT_GELU or MOE_ACT_SWIGLU */
    int32_t dtype;    /* MOE_F32 or MOE_BF16 */
    int32_t has_bias; /* GELU only: expert biases b1, b2 are given */
    int32_t n_shared; /* 0 or 1: a shared expert every token passes through
                         ("MoE(Mixture of Experts)", design notes: DeepSeek-V3's
                         fine-grained experts plus a shared part).  It has the
                         routed experts' form and sizes (GELU with the same
                         has_bias, or SwiGLU) and is added with weight 1 after
                         the routed experts' slot-order sum. */
    float capacity_factor; /* > 0: each expert accepts at most
                         C = ceil(capacity_factor * T * K / N) assignments
                         (computed in double) per call; 0: no limit.
                         "MoE(Mixture of Experts)", design notes (capacity
                         factor: overflow is dropped or sent to the next
                         candidate).  Rows are served in token order and an
                         assignment is accepted while its expert holds fewer
                         than C; what happens to the others is set by
                         overflow.  A dropped assignment adds nothing to y (the
                         kept gate weights are not renormalised).  The
                         statistics (moe_aux) describe the router's choice
                         before the limit. */
    int32_t overflow;  /* with a capacity: MOE_OVERFLOW_DROP, or
                         MOE_OVERFLOW_REROUTE -- each refused assignment of row
                         t, in slot order, goes to the best-ranked expert (by
                         the selection value, ties to the lower index) that row
                         t does not hold yet and that still holds fewer than C,
                         keeping its gate weight; dropped only when no such
                         expert is left.  The reroute is sequential in t (one
                         CTA walks the tokens) and disables the one-kernel
                         decode path.  Ignored without a capacity. */
} moe_config;

/* moe_config.overflow */
enum { MOE_OVERFLOW_DROP = 0, MOE_OVERFLOW_REROUTE = 1 };

/* Layer parameters, all device memory.
 *  W_g [D, N] dtype      router matrix, scores = x W_g (Shazeer gate x W_g)
 *  b_g [N] fp32 or NULL  per-expert router bias added to the scores
 *  W1  [N, H, D] dtype   GELU: first linear, out x in
 *      [N, 2H, D] dtype  SwiGLU: packed gate_up (rows 0..H-1 gate, H..2H-1 up)
 *  b1  [N, H] fp32       GELU with has_bias, else NULL
 *  W2  [N, D, H] dtype   second linear / down projection, out x in
 *  b2  [N, D] fp32       GELU with has_bias, else NULL
 *  b_sel [N] fp32 or NULL  selection-only bias: added (in fp32) to the scores
 *                        for choosing the K experts and for nothing else; the
 *                        gate weights stay the softmax over the kept experts'
 *                        raw scores and the statistics use the raw scores.
 *                        This is the auxiliary-loss-free load balancing of
 *                        DeepSeek-V3 named in "MoE(Mixture of Experts)",
 *                        design notes (the bias itself is adjusted in
 *                        training; here it is an input).
 *  S1  [H, D] / [2H, D] dtype  shared expert's first linear or packed gate_up
 *  sb1 [H] fp32          shared expert bias (GELU with has_bias), else NULL
 *  S2  [D, H] dtype      shared expert's second linear
 *  sb2 [D] fp32          shared expert bias (GELU with has_bias), else NULL
 *  S1, S2 are required when n_shared == 1 and ignored otherwise. */
typedef struct {
    const void *W_g;
    const float *b_g;
    const void *W1;
    const float *b1;
    const void *W2;
    const float *b2;
    const float *b_sel;
    const void *S1;
    const float *sb1;
    const void *S2;
    const float *sb2;
} moe_weights;

/* Per-batch statistics, device memory (any pointer may be NULL to skip it).
 *  counts[N]      tokens routed to each expert ("MoE(Mixture of Experts)",
 *                 section (2), Stats.TokensPerExpert)
 *  importance[N]  sum over tokens of the gate weight given to each expert
 *                 (Shazeer article, load-balancing losses, Importance(X))
 *  p_mean[N]      mean over tokens of the full N-way softmax of the scores
 *  scalars[4]     [0] Switch-style N * sum_e f_e * P_e, f_e = counts/(T*K),
 *                     P_e = p_mean ("Extending Raschka's GPT-2", auxiliary
 *                     loss section)
 *                 [1] N * sum_e f_e^2 ("MoE(Mixture of Experts)", section (3))
 *                 [2] CV(importance)^2, [3] CV(counts)^2 (Shazeer article,
 *                     load-balancing losses; population variance, hard counts
 *                     for Load).  The loss weights are left to the caller.
 * All entries are 0 when T == 0. */
typedef struct {
    int32_t *counts;
    float *importance;
    float *p_mean;
    float *scalars;
} moe_aux;

/* Bytes of device workspace moe_route / moe_forward / moe_aux_stats need for T
 * tokens (0 if the configuration is invalid).  The workspace must be 256-byte
 * aligned.  Its contents need no initialisation and are scratch between calls. */
size_t moe_workspace_size(const moe_config *cfg, int64_t T);

/* Routing only ("MoE(Mixture of Experts)", section (2), Route; Shazeer article,
 * gating, inference form without noise).
 *  x [T, D] dtype (device).
 *  logits [T, N] fp32 or NULL: scores x W_g + b_g, fp32 accumulation.
 *  topk_idx [T, K] int32: selected experts, best first; equal scores go to the
 *      lower expert index (stable descending sort); a NaN score ranks as -inf.
 *  topk_w [T, K] fp32: softmax over the K selected scores, shifted by the best.
 *  counts [N] int32 or NULL: tokens per expert.
 * T == 0 is a no-op that zeroes counts. */
int moe_route(const moe_config *cfg, const void *x, int64_t T, const moe_weights *w,
              float *logits, int32_t *topk_idx, float *topk_w, int32_t *counts,
              void *ws, size_t ws_bytes, moe_stream_t stream);

/* The whole layer ("MoE(Mixture of Experts)", section (2), Forward; Shazeer
 * article, layer formula): route, group the (token, slot) pairs by expert,
 * evaluate each selected expert once per pair on the tensor cores, scale by the
 * gate weight and sum the K contributions of a token in slot order 0..K-1.
 *  x [T, D] dtype (device); y [T, D] in y_dtype (MOE_F32 or MOE_BF16), written
 *      in full; it must not overlap x, the weights or the workspace.  For bf16
 *      layers with T > 64, K <= 2 and an fp32 y, y is cleared before the expert
 *      GEMMs and the down projection adds each token's K scaled rows into it;
 *      with at most two terms on +0 this gives the same bits as the slot-order
 *      sum.
 *  aux: optional statistics (see moe_aux), or NULL.
 * With a shared expert (n_shared == 1) its output is added after the routed
 * sum, y[t] = sum_j w_j E_j(x_t) + S(x_t), and the down projection never adds
 * into y directly.
 * The routing results and intermediates stay in the workspace; their places
 * are given by moe_workspace_layout().  T == 0 is a no-op (aux zeroed). */
int moe_forward(const moe_config *cfg, const void *x, int64_t T, const moe_weights *w,
                void *y, int32_t y_dtype, moe_aux *aux, void *ws, size_t ws_bytes,
                moe_stream_t stream);

/* moe_forward that also records CUDA events between its stages, for timing.
 * stage_events: MOE_N_STAGES + 1 cudaEvent_t handles (created by the caller);
 * event i is recorded on `stream` before stage i and event MOE_N_STAGES after
 * the last; a NULL entry is not recorded.  Stages: 0 route, 1 scan, 2 permute,
 * 3 expert up-projection, 4 expert down-projection, 5 combine, 6 statistics
 * (empty without aux). */
#define MOE_N_STAGES 7
int moe_forward_timed(const moe_config *cfg, const void *x, int64_t T, const moe_weights *w,
                      void *y, int32_t y_dtype, moe_aux *aux, void *ws, size_t ws_bytes,
                      moe_stream_t stream, void *const *stage_events);

/* Statistics from routing results (see moe_aux for the definitions).
 *  logits [T, N] fp32, topk_idx [T, K] int32, topk_w [T, K] fp32 (device).
 *  ws: workspace of at least moe_workspace_size(cfg, T) bytes. */
int moe_aux_stats(const moe_config *cfg, int64_t T, const float *logits, const int32_t *topk_idx,
                  const float *topk_w, moe_aux *out, void *ws, size_t ws_bytes,
                  moe_stream_t stream);

/* moe_aux_stats without a workspace argument.  The pages define no such
 * call: it is a library convenience for callers that cannot allocate device
 * memory or keep a workspace buffer at the point of the call, for instance C
 * code that may not call cudaMalloc there (it can synchronise the whole
 * device) or that has no device allocator of its own.  The results are those
 * of moe_aux_stats for the same arguments (same kernels, same summation
 * order).
 *
 * Scratch: a fixed array of MOE_NOALLOC_SCRATCH_BYTES inside the library, one
 * per device, shared by every call on that device.  The call clears the part
 * that must start at zero itself.  Calls whose work overlaps on the device
 * (different streams, or host threads that do not order their streams) race
 * on that array and give wrong statistics: serialise them.
 *
 * Limit: the call fits when 256 + 3 * round_up_256(ceil(T / 64) * NExperts * 4)
 * <= MOE_NOALLOC_SCRATCH_BYTES, about T * NExperts <= 11 million; otherwise it
 * returns MOE_ERR_WORKSPACE_TOO_SMALL before enqueueing anything.
 *
 * Set-up: the first call on each device (with that device current) looks up
 * the array's device address, once.  Make that first call before capturing
 * the stream into a CUDA graph.  The address is kept for the life of the
 * process: after cudaDeviceReset (or anything else that destroys the device's
 * primary context) the kept address is stale, so do not call this entry point
 * again in that process.
 *
 * Arguments, layouts and other errors as moe_aux_stats. */
#define MOE_NOALLOC_SCRATCH_BYTES (2u << 20)
int moe_aux_stats_noalloc(const moe_config *cfg, int64_t T, const float *logits,
                          const int32_t *topk_idx, const float *topk_w, moe_aux *out,
                          moe_stream_t stream);

/* Statistics under data parallelism ("MoE(Mixture of Experts)", section (3):
 * f_e is the share of ALL routed tokens; Shazeer article, load-balancing
 * losses: Importance(X) and Load(X) sum over the whole batch X).  When the
 * tokens of one batch are split over ranks (each rank runs the layer on its
 * own shard with replicated weights), the losses of the global batch come from
 * each rank's partial sums added over the ranks, then finalised.
 *
 * moe_aux_partials writes one rank's partials as exact integers, so that the
 * sum over ranks (an all-reduce of int64, e.g. NCCL ncclInt64 / ncclSum) is the
 * same on every rank and in any order:
 *   partials[0, N)    tokens routed to each expert
 *   partials[N, 2N)   sum over the slots routed to e of round(w * 2^32)
 *   partials[2N, 3N)  sum over tokens of round(softmax(scores)_e * 2^32), the
 *                     full N-way softmax
 *   partials[3N]      number of tokens T
 * Arguments as moe_aux_stats (routing results in device memory; moe_forward
 * leaves them in its workspace, see moe_get_workspace_layout); partials is
 * MOE_AUX_PARTIALS_LEN(N) int64 of device memory, overwritten.  No workspace.
 * T == 0 writes zeros. */
#define MOE_AUX_PARTIALS_LEN(N) (3 * (int64_t)(N) + 1)
int moe_aux_partials(const moe_config *cfg, int64_t T, const float *logits, const int32_t *topk_idx,
                     const float *topk_w, int64_t *partials, moe_stream_t stream);

/* The statistics of moe_aux (counts, importance, p_mean, the four scalars) from
 * partials summed over ranks (device memory, read on `stream`); any output
 * pointer may be NULL.  Every rank that finalises the same summed partials gets
 * bitwise-identical statistics. */
int moe_aux_finalize(const moe_config *cfg, const int64_t *partials, moe_aux *out, moe_stream_t stream);

/* The same finalisation on the host, for host copies of the summed partials
 * (for instance after an all-reduce over CPU processes); outputs are host
 * arrays ([N], [N], [N], [4]), any of them NULL to skip.  Gives the same bits
 * as moe_aux_finalize.  MOE_ERR_INVALID_ARG on a negative entry. */
int moe_aux_finalize_host(const moe_config *cfg, const int64_t *partials, int32_t *counts, float *importance,
                          float *p_mean, float *scalars);

/* Expert parallelism ("MoE(Mixture of Experts)", design notes: spread the
 * experts over GPUs and an all-to-all sends each token to the GPU of its
 * experts, every layer; Transformers-v5 MoE article, expert parallelism: the
 * experts split on dim 0).  With R ranks, rank r holds experts
 * [r * N/R, (r+1) * N/R) (N a multiple of R) and W_g in full.  A layer call is
 *   1. moe_ep_dispatch on every rank: route its T tokens, group the (token,
 *      slot) pairs by the rank holding their expert (stable: (token, slot)
 *      order inside a rank) and pack them;
 *   2. an all-to-all of send_counts, then of send_x / send_expert / send_w
 *      (the caller's collective, e.g. NCCL);
 *   3. moe_ep_experts on every rank, on the rows it received;
 *   4. the reverse all-to-all of z (same splits, reversed);
 *   5. moe_ep_combine on every rank: each token's K rows in slot order.
 * The result is the layer's y.  Shared experts and capacity limits are not
 * supported on this path (MOE_ERR_UNSUPPORTED).
 *
 * moe_ep_dispatch: cfg is the whole layer's (N experts); x [T, D]; w holds
 * W_g (+ b_g, b_sel); outputs, device memory:
 *   send_x [T*K, D] dtype     the pairs' token rows, rank after rank
 *   send_expert [T*K] int32   each pair's expert index on its rank (0..N/R-1)
 *   send_w [T*K] fp32         each pair's gate weight
 *   send_counts [R] int32     pairs for each rank (send_x rows rank r holds
 *                             start at the exclusive sum of the earlier counts)
 *   send_pos [T*K] int32      the send_x row of slot t*K + j (for the combine)
 *   aux                       statistics of this rank's routing, or NULL
 * ws: moe_ep_workspace_size(cfg, n_ranks, T) bytes. */
size_t moe_ep_workspace_size(const moe_config *cfg, int32_t n_ranks, int64_t T);
int moe_ep_dispatch(const moe_config *cfg, int32_t n_ranks, const void *x, int64_t T, const moe_weights *w,
                    void *send_x, int32_t *send_expert, float *send_w, int32_t *send_counts, int32_t *send_pos,
                    moe_aux *aux, void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_ep_experts: the local experts on M received rows.  cfg_local: NExperts =
 * the rank's N/R experts, TopK = 1, otherwise the layer's.  recv_x [M, D],
 * recv_expert [M] (local indices), recv_w [M] gate weights; w_local: W1, W2
 * (b1, b2) of the local experts (W_g unused).  z_out [M, D] fp32: row i =
 * recv_w[i] * E_{recv_expert[i]}(recv_x[i]).  ws:
 * moe_ep_experts_workspace_size(cfg_local, M) bytes. */
size_t moe_ep_experts_workspace_size(const moe_config *cfg_local, int64_t M);
int moe_ep_experts(const moe_config *cfg_local, const void *recv_x, int64_t M, const int32_t *recv_expert,
                   const float *recv_w, const moe_weights *w_local, float *z_out, void *ws, size_t ws_bytes,
                   moe_stream_t stream);

/* moe_ep_combine: y[t] = z_back[send_pos[t*K]] + ... + z_back[send_pos[t*K+K-1]],
 * left to right; z_back [T*K, D] fp32 are the returned rows in send order; y
 * [T, D] in y_dtype. */
int moe_ep_combine(const moe_config *cfg, const float *z_back, int64_t T, const int32_t *send_pos, void *y,
                   int32_t y_dtype, moe_stream_t stream);

/* Backward pass ("Extending Raschka's GPT-2: an MoE trained from scratch on an
 * RTX 3090", section on making the router trainable: the router learns
 * through the gate weights it produces and through the auxiliary loss).
 * The gradients of  sum(y * dy) + alpha_switch * switch + alpha_importance *
 * cv2_importance  (the moe_aux scalars [0] and [2]; the count-based scalars
 * [1] and [3] are piecewise constant and have no gradient) with respect to
 * x and every parameter, for the routing the forward chooses on the same
 * inputs (recomputed here; no forward state is kept).  All device memory,
 * fp32, overwritten:
 *   dx [T, D]; dW_g [D, N]; db_g [N] (or NULL); dW1 like W1; db1 [N, H] and
 *   db2 [N, D] (GELU with has_bias, else NULL); dW2 [N, D, H].
 * dy [T, D] fp32.  Shared experts and capacity limits are not supported
 * (MOE_ERR_UNSUPPORTED).  ws: moe_backward_workspace_size(cfg, T) bytes. */
typedef struct {
    float *dx;
    float *dW_g;
    float *db_g;
    float *dW1;
    float *db1;
    float *dW2;
    float *db2;
} moe_grads;
size_t moe_backward_workspace_size(const moe_config *cfg, int64_t T);
int moe_backward(const moe_config *cfg, const void *x, int64_t T, const moe_weights *w, const float *dy,
                 float alpha_switch, float alpha_importance, moe_grads *grads, void *ws, size_t ws_bytes,
                 moe_stream_t stream);

/* Where moe_forward leaves its intermediates inside the workspace (byte
 * offsets from ws), for inspection in tests.  Rows of each expert's segment in
 * the permuted buffers start at a multiple of row_align; rows past an expert's
 * count up to the next multiple are padding.
 *  logits [T, N] fp32, topk_idx [T, K] int32, topk_w [T, K] fp32
 *  counts [N] int32, offsets [N+1] int32 (exclusive scan of counts)
 *  row_offsets [N+1] int32 (padded segment starts)
 *  perm_slot [rows_cap] int32: slot t*K+j held by each permuted row, -1 = padding
 *  slot_row [T*K] int32: permuted row of each slot
 *  x_perm [rows_cap, D] dtype, h [rows_cap, H] dtype, z [T*K, D] fp32 */
typedef struct {
    size_t total;
    size_t logits, topk_idx, topk_w, counts, offsets, row_offsets, perm_slot, slot_row;
    size_t x_perm, h, z;
    int64_t rows_cap;
    int32_t row_align;
} moe_workspace_layout;
int moe_get_workspace_layout(const moe_config *cfg, int64_t T, moe_workspace_layout *out);

/* Parameter accounting ("MoE(Mixture of Experts)", section (1)): router D*N
 * plus all N experts (total) or the K active ones, plus the shared expert
 * (n_shared) in both; an expert holds 2*D*H weights (GELU, + H + D with
 * biases) or 3*D*H (SwiGLU).  -1 if invalid. */
int64_t moe_total_params(const moe_config *cfg);
int64_t moe_active_params(const moe_config *cfg);

/* Waits for all work on the current device, returns the sticky device status
 * bits (MOE_STATUS_*) and clears them.  Negative MOE_ERR_CUDA if the device
 * cannot be reached. */
int moe_get_device_status(void);

/* Number of kernels this library has launched in this process (all devices). */
int64_t moe_launch_count(void);

/* Static description of a return code. */
const char *moe_error_string(int code);

/* Self-test of the bounded wait used by every kernel that waits on a barrier:
 * one thread waits on a shared-memory barrier that nothing completes, gives up
 * after timeout_ns nanoseconds, sets MOE_STATUS_TIMEOUT and returns.  Used by
 * tests to show that an expired wait leaves the context usable. */
int moe_selftest_wait_timeout(int64_t timeout_ns, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
