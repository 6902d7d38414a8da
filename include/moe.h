/*
 * moe.h — C ABI of libmoe: the forward pass of the DeepSeekMoE feed-forward
 * layer with noaux_tc routing, on one NVIDIA B200 (sm_100a).
 *
 * What the layer computes (per token x, a row of hidden_size values):
 *   - router: sigmoid scores s_e = sigma(x . router_w[e]) and biased scores
 *     b_e = s_e + e_bias[e]; experts form n_group contiguous groups; a group's
 *     score is the sum of its two largest b; the topk_group best groups are
 *     kept; the num_experts_per_tok best b among the kept groups' experts are
 *     chosen; their weights are the unbiased s, divided by their sum when
 *     norm_topk_prob, times routed_scaling_factor.
 *     ("DeepSeekV3.2-Tiered-Implementations" README, § Architecture: sigmoid
 *     routing with correction bias, topk_method noaux_tc, n_group / topk_group;
 *     "The Evolving Transformer · 07 — DeepSeek V2 & V3", § 06: the bias is a
 *     load-balancing nudge, the weights use the unbiased score.)
 *   - experts: each chosen expert is a SwiGLU MLP, down(silu(gate x) * up x),
 *     and the shared expert(s) run on every token; the output is
 *     shared(x) + sum_j w_j * expert_j(x).
 *     ("The Evolving Transformer · 07", § 02 DeepSeekMoE, MoE.forward, and
 *     § 03 Shared Expert.)
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers (except where a call says "host":
 *     moe_forward_host's x_host / y_host and the host-only placement calls),
 *     row-major and contiguous,
 *     owned by the caller; the library never allocates device memory for
 *     tensors, and never frees or keeps the caller's pointers.  (The one
 *     exception to "allocates nothing" is moe_forward_host, which creates two
 *     copy streams and eight events per device on its first call on that
 *     device and keeps them until the process exits.)
 *     bf16 tensors are passed as void* (IEEE bfloat16 bit patterns).
 *   - Weights use the nn.Linear (out, in) layout: w_gate, w_up [E, I, H],
 *     w_down [E, H, I]; the S shared experts are stored concatenated along the
 *     intermediate axis: ws_gate, ws_up [S*I, H], ws_down [H, S*I] (S separate
 *     SwiGLU experts sum to exactly this).
 *   - `stream` is a cudaStream_t (CUstream) handle; NULL means the legacy
 *     default stream.  Work is enqueued on it and the call returns without
 *     synchronising; results are valid once the stream reaches that point.
 *   - Device pointers must be 16-byte aligned; hidden_size and
 *     moe_intermediate_size must be multiples of 64.
 *   - T = 0 is a valid no-op.  A call never throws across the ABI; it returns
 *     one of the moe_status codes below and, on an argument error, enqueues
 *     nothing.
 *   - Device-side waits are bounded: a wait that gives up writes a device
 *     error word (read with moe_device_status) instead of hanging the GPU.
 *   - Index arrays passed in by the caller (topk_idx, expert_offsets,
 *     expert_counts, perm_src, row_of; for expert parallelism also the expert
 *     ids inside received rows, send_row_of and the placement tables) live on
 *     the device, where the host cannot check them.  Every kernel checks such an entry before using it as
 *     an index: an entry out of range is skipped (it reads and writes nothing;
 *     see each call for what it then produces) and the device error word
 *     records it, so moe_device_status returns MOE_ERR_DEVICE_CHECK.  Arrays
 *     produced by this library always pass these checks.
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

/* Layer configuration; field names follow the DeepSeek-V3 config
 * ("DeepSeekV3.2-Tiered-Implementations" README, § Key Dimensions and
 * § Architecture). */
typedef struct moe_config {
    int32_t hidden_size;            /* H */
    int32_t n_routed_experts;       /* E, 1..256 */
    int32_t num_experts_per_tok;    /* k, 1..32 and <= topk_group * E / n_group */
    int32_t n_group;                /* G, 1..32, divides E */
    int32_t topk_group;             /* TG, 1..G */
    int32_t moe_intermediate_size;  /* I */
    int32_t n_shared_experts;       /* S, >= 0 */
    int32_t norm_topk_prob;         /* 0 or 1 */
    float routed_scaling_factor;
} moe_config;

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* null pointer, T < 0, E % G != 0, TG > G, k out of range, ... */
    MOE_ERR_UNSUPPORTED = 2,  /* H or I not a multiple of 64, E > 256, G > 32, k > 32,
                                 a pointer not 16-byte aligned, sizes beyond int32 rows */
    MOE_ERR_WORKSPACE = 3,    /* workspace null or smaller than moe_workspace_size() */
    MOE_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
    MOE_ERR_TIMEOUT = 5,      /* a bounded device wait gave up (from moe_device_status) */
    MOE_ERR_STATIC_LIMIT = 6, /* moe_dispatch_noalloc: T * E beyond its fixed scratch */
    MOE_ERR_DEVICE_CHECK = 7  /* a device-side check skipped an out-of-range index entry
                                 (from moe_device_status) */
} moe_status;

/* Element type of the layer output y. */
typedef enum moe_dtype {
    MOE_DTYPE_F32 = 0,   /* fp32: the fp32 sum of the expert outputs, unrounded */
    MOE_DTYPE_BF16 = 1   /* bf16: that fp32 sum rounded once, to nearest even */
} moe_dtype;

/* Bytes of scratch needed by moe_forward (and enough for every other call
 * that takes a workspace) for T tokens.  Pure host arithmetic. */
MOE_API int moe_workspace_size(const moe_config *cfg, int64_t T, size_t *bytes);

/*
 * Router (noaux_tc): for each token t, topk_idx[t, 0..k) are the chosen
 * experts in descending biased score (lower expert index first on equal
 * scores) and topk_w[t, 0..k) their routing weights.
 *   x        bf16  [T, H]
 *   router_w fp32  [E, H]      e_bias fp32 [E]
 *   topk_idx int32 [T, k]      topk_w fp32 [T, k]   (outputs)
 * Logits are accumulated in fp32 (gating is kept in high precision, per the
 * knlb.dev DeepSeek-V3 notes, § infrastructure / fp8).  Whatever the values
 * (NaN or infinite scores included, which rank below every finite score),
 * every token gets k distinct expert indices in [0, E) from at most
 * topk_group groups.
 */
MOE_API int moe_route(const moe_config *cfg, int64_t T, const void *x, const float *router_w,
              const float *e_bias, int32_t *topk_idx, float *topk_w,
              void *workspace, size_t workspace_bytes, void *stream);

/*
 * Dispatch: groups the token rows by the expert they are routed to.  The
 * teaching code of "The Evolving Transformer · 07" (§ 02, MoE.forward) selects
 * and gathers each expert's tokens in a loop over experts and slots; here one
 * counting sort does it for all experts.  Rows routed to expert e occupy
 * x_perm[expert_offsets[e] .. expert_offsets[e+1]) in ascending (t, j) order.
 *   topk_idx        int32 [T, k]            (input, from moe_route; each entry in [0, E))
 *   expert_offsets  int32 [E + 1]           expert_offsets[E] == T * k
 *   x_perm          bf16  [T * k, H]        x_perm[r] = x[perm_src[r] / k]
 *   perm_src        int32 [T * k]           source slot t * k + j of row r
 *   row_of          int32 [T, k]            row of slot (t, j); inverse of perm_src
 * A topk_idx entry outside [0, E) is skipped: it gets no row (row_of = -1),
 * expert_offsets[E] is T * k minus the skipped entries, and the device error
 * word records it (moe_device_status: MOE_ERR_DEVICE_CHECK).
 */
MOE_API int moe_dispatch(const moe_config *cfg, int64_t T, const void *x, const int32_t *topk_idx,
                 int32_t *expert_offsets, void *x_perm, int32_t *perm_src, int32_t *row_of,
                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * moe_dispatch for callers that cannot allocate device memory.  The paper has
 * no counterpart to this entry point: it exists for callers that must not
 * call cudaMalloc or any allocating routine themselves, for example a serving
 * process that has handed all free device memory to a fixed pool up front, or
 * an embedding runtime that gives this library only the buffers it already
 * owns.  It computes exactly what moe_dispatch computes, with the same
 * arguments minus the workspace.
 *   Scratch: a file-scope device array of 1 MiB + 4 KiB (263168 int32) holding
 *   the per-block counts and bases and the per-expert totals,
 *   2 * ceil(T / 32) * n_routed_experts + n_routed_experts int32 values;
 *   larger sizes return MOE_ERR_STATIC_LIMIT and enqueue nothing (at
 *   n_routed_experts = 256 the limit is T <= 16384).  The array is part of the
 *   library image: every GPU that loads the library holds it until the
 *   process exits, and nothing is allocated or freed by this call.
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *   call's contents.  Calls that overlap on the GPU (on different streams
 *   without ordering between them) race on it and give undefined results.
 */
MOE_API int moe_dispatch_noalloc(const moe_config *cfg, int64_t T, const void *x,
                                 const int32_t *topk_idx, int32_t *expert_offsets, void *x_perm,
                                 int32_t *perm_src, int32_t *row_of, void *stream);

/*
 * Experts: every routed row r of expert e gives
 *   h_routed[r] = silu(x_perm[r] . w_gate[e]^T) * (x_perm[r] . w_up[e]^T)   bf16 [T*k, I]
 *   y_perm[r]   = topk_w[perm_src[r]] * (h_routed[r] . w_down[e]^T)
 * and every token t runs the shared expert(s) on x itself:
 *   h_shared[t]        = silu(x[t] . ws_gate^T) * (x[t] . ws_up^T)          bf16 [T, S*I]
 *   y_perm[T*k + t]    = h_shared[t] . ws_down^T
 * ("The Evolving Transformer · 07", § 02 and § 03.)  Grouped tensor-core
 * GEMMs over the variable-length expert segments given by expert_offsets
 * (a segment outside [0, T*k) gets no rows and is recorded in the device error
 * word; a perm_src entry outside [0, T*k) gives weight 0, likewise recorded);
 * fp32 accumulation; h is stored as bf16 (it is the next GEMM's operand).
 * y_perm [T*k + T, H] is stored block-scaled: fp16 values plus one scale code
 * per 32 columns in y_perm_scale [T*k + T, ceil(H / 256) * 8] (uint8); a value
 * is fp16 * 2^(code - 141), the code chosen so that the block's largest
 * magnitude lies in [2^14, 2^15) before rounding to fp16 (fp16 precision
 * relative to the block maximum, no overflow).  When S == 0 the shared
 * pointers may be NULL and y_perm needs only T*k rows.
 */
MOE_API int moe_experts(const moe_config *cfg, int64_t T, const void *x, const void *x_perm,
                const int32_t *expert_offsets, const int32_t *perm_src, const float *topk_w,
                const void *w_gate, const void *w_up, const void *w_down,
                const void *ws_gate, const void *ws_up, const void *ws_down,
                void *h_routed, void *h_shared, void *y_perm, void *y_perm_scale, void *stream);

/* The two halves of moe_experts, for callers that schedule them separately:
 * gate_up writes h_routed / h_shared (gate and up projections with the SwiGLU
 * epilogue); down writes y_perm from them (down projection with the routing-
 * weight epilogue).  Arguments as in moe_experts. */
MOE_API int moe_experts_gate_up(const moe_config *cfg, int64_t T, const void *x, const void *x_perm,
                                const int32_t *expert_offsets, const void *w_gate, const void *w_up,
                                const void *ws_gate, const void *ws_up, void *h_routed,
                                void *h_shared, void *stream);
MOE_API int moe_experts_down(const moe_config *cfg, int64_t T, const void *h_routed,
                             const void *h_shared, const int32_t *expert_offsets,
                             const int32_t *perm_src, const float *topk_w, const void *w_down,
                             const void *ws_down, void *y_perm, void *y_perm_scale, void *stream);

/*
 * Combine: y[t] = y_perm[T*k + t] (shared, if S > 0) + sum_{j<k} y_perm[row_of[t, j]],
 * block-scaled y_perm rows (see moe_experts) decoded and summed in fp32 in
 * that order, stored as y_dtype [T, H] (a moe_dtype).  This is the weighted
 * sum of the expert outputs plus the shared expert's output of "The Evolving
 * Transformer · 07" (§ 02, § 03), computed as a deterministic gather rather
 * than by adding into the token rows.  A row_of entry outside [0, T*k)
 * contributes nothing and is recorded in the device error word.
 */
MOE_API int moe_combine(const moe_config *cfg, int64_t T, const void *y_perm,
                const void *y_perm_scale, const int32_t *row_of, void *y, int32_t y_dtype,
                void *stream);

/*
 * The whole layer: route, dispatch, experts, combine, on one stream.
 *   y [T, H] (output) of element type y_dtype (a moe_dtype: fp32, or bf16
 *   rounded once from the fp32 result).  topk_idx_out / topk_w_out: optional [T, k]
 *   copies of the routing (may be NULL).  workspace: at least
 *   moe_workspace_size(cfg, T) bytes of device memory, 256-byte aligned.
 */
MOE_API int moe_forward(const moe_config *cfg, int64_t T, const void *x, const float *router_w,
                const float *e_bias, const void *w_gate, const void *w_up, const void *w_down,
                const void *ws_gate, const void *ws_up, const void *ws_down, void *y,
                int32_t y_dtype, int32_t *topk_idx_out, float *topk_w_out, void *workspace,
                size_t workspace_bytes, void *stream);

/*
 * Auxiliary-loss-free load balancing step, run after a batch has been routed
 * ("The Evolving Transformer · 07", § 06: the per-expert bias is nudged down
 * when the expert is overloaded and up when it is underloaded, with no
 * auxiliary loss).  With load_e = number of entries of topk_idx [T, k] equal to
 * e and the mean load T*k/E:
 *   e_bias[e] -= gamma if load_e > T*k/E;  e_bias[e] += gamma if load_e < T*k/E;
 *   unchanged if equal (the comparison is exact, load_e * E against T * k).
 * e_bias fp32 [E] is updated in place (one fp32 add per expert); expert_load
 * int32 [E] optionally receives the loads (may be NULL).  gamma (the update
 * speed) is not given by the pages; it is the caller's, >= 0.  With T = 0
 * every load equals the mean (0), so no bias moves.  A topk_idx entry outside
 * [0, E) is not counted and is recorded in the device error word.
 */
MOE_API int moe_bias_update(const moe_config *cfg, int64_t T, const int32_t *topk_idx, float *e_bias,
                            float gamma, int32_t *expert_load, void *stream);

/* ------------------------------------------------------------------------
 * MXFP8 expert FFNs ("DeepSeek-V3 notes" (knlb.dev), § fp8: fine-grained
 * block-wise quantisation, E4M3 throughout, scales derived online from each
 * block's maximum, activations cached and dispatched in FP8, gating kept in
 * high precision; "DeepSeekV3.2-Tiered-Implementations", § DeepGEMM: FP8 grouped
 * GEMM for the MoE experts).
 *
 * Format of an MXFP8 matrix [rows, K] (K the contraction axis, a multiple of 128):
 *   q   uint8 [rows, K]   E4M3 bytes (1 sign, 4 exponent bits with bias 7, 3
 *                         mantissa bits; largest finite value 448), row-major;
 *   sf  uint8 scale codes, one per 32 consecutive elements of a row, the scale
 *       being 2^(code - 127); code = 127 + e for the smallest e with
 *       max|block| <= 448 * 2^e (0 for an all-zero block), so nothing saturates.
 *       Stored in 512-byte atoms of 128 rows x 128 K: atom (rb, kb) at byte
 *       (rb * K/128 + kb) * 512, and within it the code of row r (0..127) and
 *       32-block j (0..3) at byte 16 * (r % 32) + 4 * (r / 32) + j.  Rows are
 *       padded to a multiple of 128 (moe_mx_scale_bytes gives the size).
 * Quantised here: the token rows entering the experts (blocks along H), gate and
 * up weights (along H), the SwiGLU output h (along I) and down weights (along I).
 * Routing, products and sums (fp32 accumulation in the tensor core), SwiGLU and
 * the weighted combine are as in the bf16 path.
 * ------------------------------------------------------------------------ */
typedef struct moe_mx_matrix {
    const void *q;   /* E4M3 bytes, [rows, K] */
    const void *sf;  /* scale atoms (layout above) */
} moe_mx_matrix;

/* The layer's expert weights in MXFP8, each in the (out, in) layout of the bf16
 * weights: gate, up [E*I, H]; down [E*H, I]; shared_gate, shared_up [S*I, H];
 * shared_down [H, S*I] (the shared members unused when S = 0). */
typedef struct moe_mx_weights {
    moe_mx_matrix gate, up, down, shared_gate, shared_up, shared_down;
} moe_mx_weights;

/* Bytes of the scale atoms of an MXFP8 matrix [rows, K]; -1 if K is not a
 * positive multiple of 128. */
MOE_API int64_t moe_mx_scale_bytes(int64_t rows, int64_t K);

/* Quantise a bf16 matrix src [rows, K] into q [rows, K] and sf
 * (moe_mx_scale_bytes(rows, K) bytes).  MOE_ERR_UNSUPPORTED unless K % 128 == 0.
 * Used once per weight set (the scheme keeps master weights in higher precision
 * and multiplies FP8 copies). */
MOE_API int moe_mx_quantize(int64_t rows, int64_t K, const void *src, void *q, void *sf, void *stream);

/* Workspace of moe_forward_mx / moe_dispatch_mx.  Shapes: hidden_size a multiple
 * of 256, moe_intermediate_size a multiple of 128 (else MOE_ERR_UNSUPPORTED). */
MOE_API int moe_workspace_size_mx(const moe_config *cfg, int64_t T, size_t *bytes);

/* Rows of the padded routed row space: every expert's segment starts on a
 * multiple of 128 rows, so T*k rows take at most
 * round_up(T*k + 127*n_routed_experts, 128) rows. */
MOE_API int moe_mx_routed_rows(const moe_config *cfg, int64_t T, int64_t *rows);

/* Dispatch with quantisation.  Same counting sort as moe_dispatch (slots in
 * ascending (t, j) order inside each segment) with each expert's segment
 * starting on a multiple of 128 rows:
 *   expert_offsets [E+1] first row of each segment (expert_offsets[E] = end);
 *   expert_counts  [E]   rows routed to each expert;
 *   xq_perm [Rp, H] / xq_perm_sf: the MXFP8 quantisation of x[t] (blocks of 32
 *       along H) in row row_of[t, j]; rows between segments are left unwritten;
 *   xq_shared [round_up(T,128), H] / xq_shared_sf: the same rows in token order
 *       (for the shared experts; unused and may be NULL when S = 0);
 *   perm_src [Rp] flat slot t*k + j of each occupied row; row_of [T, k].
 * Rp = moe_mx_routed_rows. */
MOE_API int moe_dispatch_mx(const moe_config *cfg, int64_t T, const void *x, const int32_t *topk_idx,
                            int32_t *expert_offsets, int32_t *expert_counts, void *xq_perm, void *xq_perm_sf,
                            void *xq_shared, void *xq_shared_sf, int32_t *perm_src, int32_t *row_of,
                            void *workspace, size_t workspace_bytes, void *stream);

/* The gate/up GEMM of the MXFP8 path: for routed expert e, rows
 * expert_offsets[e] .. + expert_counts[e] of xq_perm (as written by
 * moe_dispatch_mx), h = silu(x Wg_e^T) * (x Wu_e^T) with fp32 accumulation,
 * quantised to MXFP8 (blocks of 32 along I) into hq_routed [Rp, I] and its scale
 * atoms hq_routed_sf (moe_mx_scale_bytes(Rp, I)); the shared experts likewise
 * from xq_shared into hq_shared [round_up(T,128), S*I].  Rows of a segment past
 * its count (up to the next multiple of 128) are written as zeros. */
MOE_API int moe_experts_gate_up_mx(const moe_config *cfg, int64_t T, const void *xq_perm, const void *xq_perm_sf,
                                   const void *xq_shared, const void *xq_shared_sf, const int32_t *expert_offsets,
                                   const int32_t *expert_counts, const moe_mx_weights *weights, void *hq_routed,
                                   void *hq_routed_sf, void *hq_shared, void *hq_shared_sf, void *stream);

/* The down GEMM of the MXFP8 path: y_perm row r = topk_w[perm_src[r]] *
 * (h_r Wd_e^T) for the occupied rows of each routed segment, and row Rp + t =
 * h_shared[t] Ws_down^T, in the block-scaled fp16 format of moe_experts
 * (y_perm [Rp + T, H], y_perm_scale [Rp + T, round_up(H/32, 8)]). */
MOE_API int moe_experts_down_mx(const moe_config *cfg, int64_t T, const void *hq_routed, const void *hq_routed_sf,
                                const void *hq_shared, const void *hq_shared_sf, const int32_t *expert_offsets,
                                const int32_t *expert_counts, const int32_t *perm_src, const float *topk_w,
                                const moe_mx_weights *weights, void *y_perm, void *y_perm_scale, void *stream);

/* moe_combine for the MXFP8 path's y_perm, whose shared rows start at row Rp. */
MOE_API int moe_combine_mx(const moe_config *cfg, int64_t T, const void *y_perm, const void *y_perm_scale,
                           const int32_t *row_of, void *y, int32_t y_dtype, void *stream);

/* The layer forward with MXFP8 expert FFNs: route (as moe_route, on the bf16 x),
 * dispatch with quantisation, gate/up GEMM with SwiGLU and h quantised to MXFP8,
 * down GEMM with the routing weights, combine.  Arguments as moe_forward, with
 * the expert weights given as MXFP8 matrices (moe_mx_quantize). */
MOE_API int moe_forward_mx(const moe_config *cfg, int64_t T, const void *x, const float *router_w,
                           const float *e_bias, const moe_mx_weights *weights, void *y, int32_t y_dtype,
                           int32_t *topk_idx_out, float *topk_w_out, void *workspace, size_t workspace_bytes,
                           void *stream);

/* ------------------------------------------------------------------------
 * Backward pass of the layer: gradients of L = sum(y * dy) for an upstream
 * gradient dy, with the expert selection held fixed (the group keep and top-k
 * choice is piecewise constant; the correction bias gets no gradient) — the
 * chain rule of the forward above, checked in float64 by finite differences as
 * the "dsv3-native-reference" page, § NumPy Oracle, does.  Shapes as
 * moe_forward_mx (hidden_size % 256 == 0, moe_intermediate_size % 128 == 0).
 *   dy [T, H] bf16; dx [T, H] fp32; d_router_w [E, H] fp32;
 *   d_w_gate, d_w_up [E, I, H], d_w_down [E, H, I], d_ws_gate, d_ws_up [S*I, H],
 *   d_ws_down [H, S*I], all bf16 (fp32 sums, rounded once).
 * The routing is recomputed (same kernels and inputs as the forward, hence the
 * same selection) and the experts' g = x Wg^T and u = x Wu^T are recomputed
 * rather than kept.  T = 0 writes zero weight gradients.
 * ------------------------------------------------------------------------ */
MOE_API int moe_workspace_size_bwd(const moe_config *cfg, int64_t T, size_t *bytes);

MOE_API int moe_backward(const moe_config *cfg, int64_t T, const void *x, const float *router_w,
                         const float *e_bias, const void *w_gate, const void *w_up, const void *w_down,
                         const void *ws_gate, const void *ws_up, const void *ws_down, const void *dy, float *dx,
                         float *d_router_w, void *d_w_gate, void *d_w_up, void *d_w_down, void *d_ws_gate,
                         void *d_ws_up, void *d_ws_down, void *workspace, size_t workspace_bytes, void *stream);

/* The forward from HOST buffers: x_host [T, H] bf16 and y_host [T, H] (y_dtype)
 * in host memory (pinned, for the copies to run asynchronously), weights on the
 * device.  The batch is cut into chunks of chunk_tokens rows (0 or >= T: one
 * chunk); chunk i's input copy and chunk i-1's output copy run on two internal
 * copy streams while chunk i is computed on `stream`, so transfers overlap the
 * layer.  The two copy streams and the events that order them are created by
 * the first call on each device (with that device current) and kept until the
 * process exits; make that first call before any stream capture.  Rows are
 * independent, so y is moe_forward's on the whole batch: bit for
 * bit when the chunks and the batch take the same router-logit path (at least 2048
 * rows: tensor cores; fewer: CUDA cores), else up to the fp32 summation order of
 * the logits.  The workspace (moe_workspace_size_host) holds two staging slots each
 * for x and y plus the forward's workspace for one chunk.  The call returns
 * after enqueueing; y_host is complete once `stream` reaches that point.
 * Calls from several host threads on one device are serialised. */
MOE_API int moe_workspace_size_host(const moe_config *cfg, int64_t T, int64_t chunk_tokens, int32_t y_dtype,
                                    size_t *bytes);

MOE_API int moe_forward_host(const moe_config *cfg, int64_t T, const void *x_host, const float *router_w,
                             const float *e_bias, const void *w_gate, const void *w_up, const void *w_down,
                             const void *ws_gate, const void *ws_up, const void *ws_down, void *y_host,
                             int32_t y_dtype, int64_t chunk_tokens, void *workspace, size_t workspace_bytes,
                             void *stream);

/* Training pair: moe_forward_train computes the forward (same arguments as
 * moe_forward) and keeps what the backward needs — routing, router logits, the
 * expert-ordered rows and the experts' g = x Wg^T and u = x Wu^T (bf16) — in
 * `context` (moe_workspace_size_bwd bytes); moe_backward_train then gives the
 * gradients of moe_backward without recomputing routing, rows, g or u.  The
 * context must come from moe_forward_train on the same x and weights, unchanged
 * in between.  moe_forward_train's y is moe_forward's (h is formed from the same
 * fp32 accumulators with the same expression): bit for bit when every expert
 * segment has more than 112 rows; moe_forward computes smaller segments
 * transposed, which can round differently in the last place. */
MOE_API int moe_forward_train(const moe_config *cfg, int64_t T, const void *x, const float *router_w,
                              const float *e_bias, const void *w_gate, const void *w_up, const void *w_down,
                              const void *ws_gate, const void *ws_up, const void *ws_down, void *y, int32_t y_dtype,
                              void *context, size_t context_bytes, void *stream);

MOE_API int moe_backward_train(const moe_config *cfg, int64_t T, const void *x, const float *router_w,
                               const void *w_gate, const void *w_up, const void *w_down, const void *ws_gate,
                               const void *ws_up, const void *ws_down, const void *dy, float *dx, float *d_router_w,
                               void *d_w_gate, void *d_w_up, void *d_w_down, void *d_ws_gate, void *d_ws_up,
                               void *d_ws_down, void *context, size_t context_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Expert parallelism: the routed experts spread over `world` ranks (one GPU
 * each), rank r holding experts [r * E/world, (r + 1) * E/world) in the layout
 * of the single-GPU weights (w_gate, w_up [E/world, I, H], w_down
 * [E/world, H, I]); the shared experts and the router are replicated.  ("DeepSeek-
 * V3 notes" (knlb.dev), § infrastructure: expert parallelism with all-to-all
 * dispatch and combine kernels; § architecture: each token is sent to a limited
 * number of nodes — with contiguous expert blocks per rank and groups that do not
 * straddle ranks, to at most topk_group ranks.)
 *
 * A token crosses to a rank once, however many of its k experts live there: the
 * source sends one row per (token, destination rank), the destination runs the
 * token's experts it was sent and sends back one row, their weighted sum.
 *
 * Redundant experts ("DeepSeek-V3 notes" § infrastructure, prefilling: redundant
 * experts for load balance, placed from live statistics): a placement table
 * expert_ranks int32 [E, max_rep] lists for expert e the ranks holding a copy,
 * in its first n_e >= 1 entries (distinct ranks in [0, world)), then -1.  Slot
 * (t, j) of expert e goes to rank expert_ranks[e, t mod n_e], so e's rows split
 * evenly over its copies.  moe_ep_place builds such a table from per-expert
 * loads; a null table means rank e / (E/world) for every e (no copies).  Rank r
 * holds its experts in ascending id order (moe_ep_local_experts gives each id's
 * local index): w_gate, w_up [n_local, I, H], w_down [n_local, H, I].
 *
 * Rows travel in two wire formats (moe_ep_row_bytes):
 *   send row:   H bf16 values of x[t], then k int32 expert ids — slot j's id when
 *               slot j goes to this row's rank, -1 when it goes elsewhere — and
 *               the token's k routing weights (fp32), zero-padded to a multiple
 *               of 16 bytes;
 *   return row: H block-scaled fp16 values (value = fp16 * 2^(code - 141)), then
 *               their H/32 scale codes (one byte per 32 values), padded likewise.
 * One forward on each rank, for its own T tokens:
 *   1. moe_route;
 *   2. moe_ep_send: the send rows, sorted by destination rank (token order within
 *      a rank), the number for each rank, and where each slot's row went;
 *   3. the caller's all-to-all of the counts (one int32 to each rank), then of the
 *      send rows with those block sizes: rank r receives, from each source s in
 *      rank order, s's rows for r;
 *   4. moe_ep_experts: the received rows through the rank's experts, and the
 *      rank's own tokens through the shared experts;
 *   5. the caller's all-to-all of the return rows back (the reverse block sizes),
 *      so that they land in the source's send order;
 *   6. moe_ep_combine.
 * With world = 1 the collectives are copies; the result differs from moe_forward's
 * only by the fp16 rounding of the returned sums.
 * ------------------------------------------------------------------------ */

/* Bytes of one send row and of one return row (formats above); multiples of 16. */
MOE_API int moe_ep_row_bytes(const moe_config *cfg, int64_t *send_row_bytes, int64_t *return_row_bytes);

/* Device workspace (256-byte aligned) for moe_ep_send on T tokens and for
 * moe_ep_experts on R received rows, T own tokens and n_local local experts.
 * MOE_ERR_INVALID_ARG unless 1 <= world, world divides E, 1 <= n_local <= E and
 * R >= 0. */
MOE_API int moe_ep_workspace_size(const moe_config *cfg, int32_t world, int32_t n_local, int64_t T, int64_t R,
                                  size_t *bytes);

/* Host only.  A placement with n_redundant extra copies, from load int64 [E] (rows
 * per expert, e.g. the expert_load of moe_bias_update over recent batches): every
 * expert starts on rank e / (E/world); then, n_redundant times, the expert whose
 * copies carry the most rows each (load / copies; lowest id on ties; fewer than
 * min(max_rep, world) copies) gets one more copy, on the rank with the least
 * load that does not hold it (lowest rank on ties), its load being split evenly
 * over its copies.  Stops early when no copy would carry rows.  Writes
 * expert_ranks int32 [E, max_rep] (format above).  MOE_ERR_INVALID_ARG for E not
 * a multiple of world, max_rep < 1, n_redundant < 0 or a negative load. */
MOE_API int moe_ep_place(int32_t E, int32_t world, const int64_t *load, int32_t n_redundant, int32_t max_rep,
                         int32_t *expert_ranks);

/* Host only.  local_of int32 [E]: expert e's index among rank `rank`'s experts
 * (ascending ids), -1 where the rank holds no copy; *n_local = their number.
 * MOE_ERR_INVALID_ARG for a malformed table (no copy, a rank outside [0, world),
 * a repeated rank, an entry after a -1). */
MOE_API int moe_ep_local_experts(int32_t E, int32_t world, int32_t rank, const int32_t *expert_ranks,
                                 int32_t max_rep, int32_t *local_of, int32_t *n_local);

/* Source side.  In: x bf16 [T, H]; topk_idx int32 / topk_w fp32 [T, k] (from
 * moe_route); expert_ranks [E, max_rep] device table (or null: E/world-expert
 * blocks).  Out: send_rows [T * min(k, world)] rows of send_row_bytes (the
 * first sum(send_counts) written, sorted by destination rank, token order within
 * a rank); send_counts int32 [world]: rows for each rank; send_row_of int32 [T, k]:
 * for the first slot of token t bound for rank d, the index of its send row; -1
 * for the token's other slots bound there.  An expert id outside [0, E), or a
 * malformed table entry, gives no row and is recorded in the device error word.
 * x, send_rows and the workspace 16-byte aligned.  T = 0 only zeroes send_counts. */
MOE_API int moe_ep_send(const moe_config *cfg, int32_t world, int64_t T, const void *x, const int32_t *topk_idx,
                        const float *topk_w, const int32_t *expert_ranks, int32_t max_rep, int32_t *send_counts,
                        void *send_rows, int32_t *send_row_of, void *workspace, size_t workspace_bytes,
                        void *stream);

/* Rank `rank`'s experts.  local_of int32 [E] device map (moe_ep_local_experts)
 * and n_local, or local_of null: the block rank * E/world .. with n_local unused.
 * In: recv_rows [R] send rows from all sources; x bf16 [T, H], the rank's own
 * tokens; w_gate / w_up / w_down the rank's n_local experts.  Out: return_rows
 * [R] rows of return_row_bytes: row i = sum over the slots j of received row i
 * with an id e != -1 of w_j * down_e(silu(gate_e x) * up_e x), summed in fp32 in
 * slot order, then block-scaled to fp16; y_shared [T, H] block-scaled fp16 with
 * y_shared_scale [T, ceil(H/256)*8] codes (the moe_experts format): the shared
 * experts on x (unused when S = 0).  A received id that is not one of this rank's
 * experts gives no row and is recorded in the device error word.  Pointers
 * 16-byte aligned. */
MOE_API int moe_ep_experts(const moe_config *cfg, int32_t world, int32_t rank, const int32_t *local_of,
                           int32_t n_local, int64_t T, const void *x, int64_t R, const void *recv_rows,
                           const void *w_gate, const void *w_up, const void *w_down, const void *ws_gate,
                           const void *ws_up, const void *ws_down, void *return_rows, void *y_shared,
                           void *y_shared_scale, void *workspace, size_t workspace_bytes, void *stream);

/* Source side, after the return rows came back in send order: back_rows holds
 * n_back (= sum(send_counts)) return rows.  y[t] = shared row t + the back rows
 * send_row_of[t, 0..k) (entries -1 skipped), summed in fp32 in that order; y
 * [T, H] of y_dtype (fp32, or bf16 rounded once).  A send_row_of entry outside
 * [-1, n_back) contributes nothing and is recorded in the device error word.
 * MOE_ERR_INVALID_ARG unless 0 <= n_back <= T * min(k, world). */
MOE_API int moe_ep_combine(const moe_config *cfg, int32_t world, int64_t T, int64_t n_back, const void *back_rows,
                           const int32_t *send_row_of, const void *y_shared, const void *y_shared_scale, void *y,
                           int32_t y_dtype, void *stream);

/* Static text for a status code. */
MOE_API const char *moe_status_string(int status);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device: *device_error = 0 when no bounded wait gave up and no
 * device-side check failed, else the nonzero code of the first failure
 * (0x4xx: an index entry out of range was skipped; other codes: a bounded wait
 * gave up).  Returns MOE_OK, MOE_ERR_DEVICE_CHECK for a 0x4xx word,
 * MOE_ERR_TIMEOUT for any other nonzero word, or MOE_ERR_CUDA. */
MOE_API int moe_device_status(void *stream, int32_t *device_error);

/* Number of kernels this library has launched in this process. */
MOE_API uint64_t moe_launch_count(void);

/* Failure-detection self-test: launches one kernel whose thread waits, with the
 * library's bounded-wait routine, on an mbarrier that nothing ever arrives on.
 * After limit_ns (1 ns .. 10 s) the wait gives up, records code 0x901 in the
 * device error word and the kernel returns; the GPU context stays usable.
 * Read the outcome with moe_device_status.  The layer's design has no
 * counterpart on the pages: it exists to test the timeout path without a fault. */
MOE_API int moe_selftest_wait_timeout(uint64_t limit_ns, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
