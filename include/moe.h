/*
 * moe.h - C ABI of the sparse Mixture-of-Experts FFN block on B200.
 *
 * The block computed here (the forward pass, without the residual):
 *
 *   MoE(u_t) = sum_{s in shared} FFN_s(u_t) + sum_{i in TopK(t)} g_{i,t} FFN_i(u_t)
 *   FFN(u)   = W2 (SiLU(W1 u) * W3 u)
 *
 * Entry points, in the order of the path:
 *   moe_check_config, moe_workspace_size      validation and scratch size
 *   moe_route (moe_route_noalloc)             router logits, biased group-limited
 *                                             top-k, gates, counts, offsets
 *   moe_permute                               tokens into expert-contiguous rows
 *   moe_expert_swiglu = moe_expert_gate_up + moe_expert_down
 *                                             every expert's FFN (+ the shared one)
 *   moe_combine                               gate-weighted sum + shared row
 *   moe_forward                               all of the above in one call
 * and around it:
 *   moe_balance_update                        aux-loss-free bias step, entropy
 *   moe_expert_gate_up_gather                 gate/up reading rows of x directly
 *   moe_expert_gelu, moe_forward_gelu         generic experts W2 GELU(W1 u + b1) + b2
 *   moe_backward (_workspace_size), moe_forward_train, moe_backward_saved
 *                                             gradients of the block for training
 *   moe_get_device_error, moe_route_noalloc_device_error,
 *   moe_forward_gathers_rows, moe_selftest_wait_timeout, moe_status_string
 *
 * Sources, cited by page title and section:
 *   [DS] "Sparse MoE FFN" DeepSeek-V3 study note, "How it works": eq. 12
 *        (residual form; the module returns shared + routed without u_t),
 *        the SwiGLU equation (W1, W3 in R^{f x d}, W2 in R^{d x f}), the
 *        "Routing" paragraph (sigmoid affinities, top-K on s + b, 8 groups
 *        keep 4 with group score = sum of top-2, gates = unbiased selected s
 *        renormalised, times route_scale = 2.5) and "Packed forward
 *        (official)" (flatten to (T, d); weights and indices (T, K_r);
 *        per-expert gather, SwiGLU, scale, scatter-add; shared FFN over all T;
 *        no token dropped).
 *   [CS] "Mixture of Experts and Hybrid Architectures" cheat sheet, "The
 *        router in code": route(hidden, W_router, top_k, bias) ->
 *        (top_idx, gates); bias moves selection only; softmax over the chosen
 *        original scores, which sums to 1.
 *   [KB] "Mixture of experts and architecture families", "The router and
 *        load balancing": moe_layer(x, router, experts, k) over x: [tokens, d].
 *   [L2] "Lesson 2 - From the Dense FFN to a Layer of Experts", sections 2
 *        and 4 (routed sum; shared experts with unit weight); sections 1-2
 *        also define the generic expert W2 phi(W1 u + b1) + b2 (phi = GELU)
 *        served by moe_expert_gelu / moe_forward_gelu.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every data pointer is a DEVICE pointer to a row-major, contiguous array
 *    owned by the caller. The library keeps no pointer after a call returns
 *    and allocates no memory: scratch lives in the caller's workspace, sized
 *    by moe_workspace_size().
 *  - Activations, weights, x_perm, y_perm, y_shared, y and the workspace must
 *    be 16-byte aligned; d and f (and f_shared) must be multiples of 8 for
 *    bf16 and of 4 for fp32. Otherwise the call returns MOE_ERR_MISALIGNED.
 *  - dtype selects the storage type of activations and weights (fp32 or
 *    bf16). Router logits, bias, gates and every accumulation are fp32.
 *  - stream is a cudaStream_t (NULL = the legacy default stream). Calls only
 *    enqueue work: none synchronises the host, none copies device data to
 *    the host, so a call may be captured in a CUDA graph.
 *  - Arguments are validated before anything is enqueued. T = 0 is valid:
 *    moe_route then only zeroes expert_counts and expert_offsets, and the
 *    other entry points enqueue nothing.
 *  - Every entry point that takes a workspace needs at least
 *    moe_workspace_size(cfg) bytes of it, else MOE_ERR_WORKSPACE_TOO_SMALL.
 *  - Calls on distinct workspaces are independent and thread-safe. No C++
 *    exception crosses this interface.
 *  - Device-side waits are bounded (about 2 s). A wait that runs out records
 *    MOE_ERR_TIMEOUT in the workspace's error word and its kernel returns;
 *    moe_get_device_error() reports it. Caller-supplied indices (topk_idx,
 *    expert_offsets, inv_row) are bounds-checked on the device: out-of-range
 *    values are skipped or clamped, never dereferenced, and flagged in the
 *    same word where the call has one (moe_combine has none: it skips a
 *    row past T*k silently).
 */
#ifndef MOE_B200_H_
#define MOE_B200_H_

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

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* a size or mode outside the documented range */
  MOE_ERR_MISALIGNED = 2,         /* a pointer or a row stride breaks the 16-byte rule */
  MOE_ERR_UNSUPPORTED = 3,        /* valid, but beyond this build's limits (E, k, groups) */
  MOE_ERR_WORKSPACE_TOO_SMALL = 4,
  MOE_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed */
  MOE_ERR_TIMEOUT = 6             /* a device-side wait ran out (see moe_get_device_error) */
} moe_status;

typedef enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 } moe_dtype;

typedef enum {
  /* gates = route_scale * softmax of the selected RAW logits (max-subtracted) [CS] */
  MOE_GATE_SOFTMAX = 0,
  /* gates = route_scale * s_i / sum_selected s, s = sigmoid(logit)           [DS] */
  MOE_GATE_SIGMOID = 1
} moe_gate_mode;

/* Shape and routing settings of one MoE FFN block. All fields are plain
 * 32-bit values so that the struct has the same layout from any language. */
typedef struct {
  int32_t T;            /* tokens (rows of x)                                      */
  int32_t d;            /* hidden width                                            */
  int32_t E;            /* routed experts, 1..1024                                 */
  int32_t k;            /* experts per token, 1..min(E, 32)                        */
  int32_t f;            /* routed expert inner width (rows of W1, W3)              */
  int32_t dtype;        /* moe_dtype                                               */
  int32_t gate_mode;    /* moe_gate_mode                                           */
  int32_t n_groups;     /* expert groups; 1 = no group limit. E % n_groups == 0,   */
                        /* 1..32, and E / n_groups >= 2 when n_groups > 1          */
  int32_t topk_groups;  /* groups kept per token, 1..n_groups, with                */
                        /* topk_groups * E / n_groups >= k                         */
  float route_scale;    /* > 0; multiplies the renormalised gates (1.0 = none)     */
  int32_t f_shared;     /* shared-expert inner width; 0 = no shared expert         */
} moe_config;

/* Checks a configuration without touching any device. Returns MOE_OK,
 * MOE_ERR_INVALID_ARG or MOE_ERR_UNSUPPORTED. Host-only. */
MOE_API moe_status moe_check_config(const moe_config* cfg);

/* Bytes of workspace that every entry point below accepts for cfg (the
 * largest any of them needs; moe_forward needs all of it). 0 if cfg is not
 * valid. Host-only. Worst case: T*k packed rows plus T shared rows. */
MOE_API size_t moe_workspace_size(const moe_config* cfg);

/*
 * moe_route - the gate: router logits, affinities, biased (optionally
 * group-limited) top-k, gates, and the packing offsets.  [DS] "Routing";
 * [CS] "The router in code".
 *
 *   x            [T][d]     dtype     activations u_t
 *   w_router     [E][d]     dtype     router rows e_i
 *   bias         [E]        fp32      selection bias b_i, or NULL (= 0)
 *   topk_idx     [T][k]     int32     OUT: selected experts, ascending id;
 *                                     ties go to the lower expert / group index
 *   topk_gate    [T][k]     fp32      OUT: gate of each selected expert, from
 *                                     the unbiased affinity
 *   expert_counts  [E]      int32     OUT: tokens per expert
 *   expert_offsets [E+1]    int32     OUT: exclusive prefix sum of counts
 *
 * Selection: b'_e = s_e + bias_e, with s = sigmoid(logit) (MOE_GATE_SIGMOID)
 * or s = logit (MOE_GATE_SOFTMAX). With n_groups > 1, group G = experts
 * [G*E/n_groups, (G+1)*E/n_groups) scores the sum of its two largest b';
 * only the topk_groups best groups stay eligible. Then the k largest
 * eligible b' win. For bf16 with E <= 256 the whole call is one kernel (the
 * router logits never leave the chip as partial sums); the workspace keeps
 * the summed logits [T][E] fp32 either way.
 */
MOE_API moe_status moe_route(const moe_config* cfg, const void* x, const void* w_router,
                     const float* bias, int32_t* topk_idx, float* topk_gate,
                     int32_t* expert_counts, int32_t* expert_offsets,
                     void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_route_maps - moe_route plus the row maps of moe_permute's x_perm = NULL
 * form, from the same single launch: for a batch that is one tile of the
 * fused router (bf16, E <= 256, T <= 128), whose last step already holds the
 * offsets and every chunk's selections. moe_forward takes this path when its
 * gate/up GEMM gathers the token rows (decode-sized batches). [DS]
 * "Routing" and "Packed forward".
 *
 *   x .. expert_offsets   as moe_route
 *   perm_src       [T*k]      int32   OUT: source token of each packed row
 *   inv_row        [T][k]     int32   OUT: packed row of (token, slot)
 *
 * The results equal moe_route followed by moe_permute(x_perm = NULL).
 * Anywhere else (fp32, E > 256, T > 128) it returns MOE_ERR_UNSUPPORTED and
 * writes nothing; moe_route_maps_supported says beforehand.
 */
MOE_API moe_status moe_route_maps(const moe_config* cfg, const void* x, const void* w_router,
                          const float* bias, int32_t* topk_idx, float* topk_gate,
                          int32_t* expert_counts, int32_t* expert_offsets, int32_t* perm_src,
                          int32_t* inv_row, void* workspace, size_t ws_bytes, void* stream);

/* 1 when moe_route_maps runs for cfg, 0 when it would return
 * MOE_ERR_UNSUPPORTED, -1 for an invalid cfg. Host-only. */
MOE_API int moe_route_maps_supported(const moe_config* cfg);

/*
 * moe_permute - gather token rows into expert-contiguous order.
 * [DS] "Packed forward": for each expert, gather the tokens whose indices
 * equal it; [KB] the per-expert mask loop.
 *
 *   x              [T][d]     dtype   activations
 *   topk_idx       [T][k]     int32   from moe_route (each row: k distinct ids)
 *   expert_offsets [E+1]      int32   from moe_route
 *   x_perm         [T*k][d]   dtype   OUT: row offsets[e] + r holds the r-th
 *                                     token (in token order) that chose e;
 *                                     NULL: only perm_src and inv_row are
 *                                     written (x may then be NULL too), for
 *                                     moe_expert_gate_up_gather
 *   perm_src       [T*k]      int32   OUT: source token of each packed row
 *   inv_row        [T][k]     int32   OUT: packed row of (token, slot)
 */
MOE_API moe_status moe_permute(const moe_config* cfg, const void* x, const int32_t* topk_idx,
                       const int32_t* expert_offsets, void* x_perm, int32_t* perm_src,
                       int32_t* inv_row, void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_expert_swiglu - every expert's SwiGLU FFN over its packed rows, plus
 * the shared expert over all T tokens.  [DS] SwiGLU equation and "Packed
 * forward" (the shared FFN runs on all T tokens).
 *
 *   x_perm         [T*k][d]      dtype  packed activations (moe_permute)
 *   expert_offsets [E+1]         int32  segment e = rows [off[e], off[e+1])
 *   w1, w3         [E][f][d]     dtype  W1 (inside SiLU), W3 (multiplier)
 *   w2             [E][d][f]     dtype  W2 (down projection)
 *   x_shared       [T][d]        dtype  shared-expert input, NULL if f_shared == 0
 *   ws1, ws3       [f_shared][d] dtype  shared W1, W3 (NULL if f_shared == 0)
 *   ws2            [d][f_shared] dtype  shared W2     (NULL if f_shared == 0)
 *   y_perm         [T*k][d]      dtype  OUT: FFN_e(row), gate NOT applied
 *   y_shared       [T][d]        dtype  OUT: FFN_shared(x_t) (NULL if f_shared == 0)
 *
 * bf16 runs on tcgen05 tensor cores with fp32 accumulation; the SwiGLU
 * intermediate is rounded to bf16 once. fp32 runs fp32 FMA throughout.
 */
MOE_API moe_status moe_expert_swiglu(const moe_config* cfg, const void* x_perm,
                             const int32_t* expert_offsets, const void* w1, const void* w3,
                             const void* w2, const void* x_shared, const void* ws1,
                             const void* ws3, const void* ws2, void* y_perm, void* y_shared,
                             void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_expert_gate_up - first half of moe_expert_swiglu: the SwiGLU inner
 * activation of every segment.  [DS] SwiGLU equation, SiLU(W1 u) * W3 u.
 *
 *   x_perm, expert_offsets, w1, w3, x_shared, ws1, ws3   as in moe_expert_swiglu
 *   h              [T*k][f]          dtype  OUT: SiLU(W1_e row) * (W3_e row)
 *   h_shared       [T][f_shared]     dtype  OUT: same for the shared expert
 *                                           (NULL if f_shared == 0)
 *
 * bf16: one persistent tcgen05 kernel; both products accumulate in TMEM in
 * fp32, the epilogue applies SiLU and the product in fp32 and rounds once.
 */
MOE_API moe_status moe_expert_gate_up(const moe_config* cfg, const void* x_perm,
                              const int32_t* expert_offsets, const void* w1, const void* w3,
                              const void* x_shared, const void* ws1, const void* ws3, void* h,
                              void* h_shared, void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_expert_gate_up_gather - moe_expert_gate_up without the packed copy of
 * the activations: the GEMM reads each packed row straight from x through
 * perm_src (two gather warps per CTA copy the rows with cp.async into the
 * GEMM's shared-memory slots), so moe_permute can skip writing x_perm.
 * [DS] "Packed forward": gather the tokens of each expert.
 *
 *   x              [T][d]        bf16   activations (also the shared expert's input),
 *                                       16-byte aligned, T*d*2 < 4 GiB
 *   perm_src       [T*k]         int32  source token of each packed row (moe_permute);
 *                                       an entry outside [0, T) reads row 0 and
 *                                       sets MOE_ERR_INVALID_ARG in the error word
 *   expert_offsets, w1, w3, ws1, ws3, h, h_shared   as in moe_expert_gate_up
 *
 * bf16 only (MOE_ERR_UNSUPPORTED for fp32, or when x breaks the limits
 * above). Results are bit-identical to moe_permute + moe_expert_gate_up.
 * moe_forward takes this path itself when the token tiles run on single
 * CTAs (fewer than 128 token rows per tile, e.g. decode), where it is as
 * fast as reading packed rows and saves the permute's copy; on CTA pairs
 * the packed copy is faster and moe_forward uses it.
 */
MOE_API moe_status moe_expert_gate_up_gather(const moe_config* cfg, const void* x,
                                     const int32_t* perm_src, const int32_t* expert_offsets,
                                     const void* w1, const void* w3, const void* ws1,
                                     const void* ws3, void* h, void* h_shared, void* workspace,
                                     size_t ws_bytes, void* stream);

/*
 * moe_expert_down - second half of moe_expert_swiglu: the down projection
 * W2 h of every segment.  [DS] SwiGLU equation, W2 in R^{d x f}.
 *
 *   h              [T*k][f]          dtype  from moe_expert_gate_up
 *   expert_offsets [E+1]             int32
 *   w2             [E][d][f]         dtype
 *   h_shared       [T][f_shared]     dtype  (NULL if f_shared == 0)
 *   ws2            [d][f_shared]     dtype  (NULL if f_shared == 0)
 *   y_perm         [T*k][d]          dtype  OUT
 *   y_shared       [T][d]            dtype  OUT (NULL if f_shared == 0)
 */
MOE_API moe_status moe_expert_down(const moe_config* cfg, const void* h,
                           const int32_t* expert_offsets, const void* w2, const void* h_shared,
                           const void* ws2, void* y_perm, void* y_shared, void* workspace,
                           size_t ws_bytes, void* stream);

/*
 * moe_combine - gate-weighted sum of each token's k expert rows, plus the
 * shared row.  [KB] out[rows] += w * expert(x[rows]); [DS] "Packed forward"
 * (scale by the matching weights, scatter-add into a zero buffer, return y+z).
 *
 *   y[t] = sum_{j<k} topk_gate[t][j] * y_perm[inv_row[t][j]]  (+ y_shared[t])
 *
 * Summed in fp32 in slot order j = 0..k-1, then the shared row, then
 * rounded once to dtype. y_shared may be NULL. y is [T][d] dtype.
 */
MOE_API moe_status moe_combine(const moe_config* cfg, const void* y_perm, const int32_t* inv_row,
                       const float* topk_gate, const void* y_shared, void* y, void* stream);

/*
 * moe_forward - the whole block: route, permute, experts, combine.
 * Inputs as above; y [T][d] dtype receives shared + routed (no residual,
 * [DS] eq. 12). ws1/ws3/ws2 are NULL when f_shared == 0. The gate/up GEMM
 * reads the token rows either from the permute's packed copy or, with
 * single-CTA token tiles, gathered straight from x (moe_forward_gathers_rows
 * says which); the bytes of y are the same either way.
 */
MOE_API moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_router,
                       const float* bias, const void* w1, const void* w3, const void* w2,
                       const void* ws1, const void* ws3, const void* ws2, void* y,
                       void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_expert_gelu - generic (Switch/GShard-style) experts on packed rows.
 * [L2] section 2: E_i(u) = W2_i GELU(W1_i u + b1_i) + b2_i, the expert of
 * section 1's dense FFN with its own weights; GELU(v) = v * Phi(v) with the
 * standard normal CDF (the exact erf form, not the tanh approximation).
 *
 *   x_perm         [T*k][d]  dtype  packed rows (moe_permute's output)
 *   expert_offsets [E+1]     int32  segment e = packed rows [off[e], off[e+1])
 *   w1             [E][f][d] dtype  b1 [E][f] fp32 (NULL: zero)
 *   w2             [E][d][f] dtype  b2 [E][d] fp32 (NULL: zero)
 *   y_perm         [T*k][d]  dtype  OUT: E_e(x_perm[r]) for packed row r of segment e
 *
 * The hidden activation is kept in the workspace in dtype (one rounding
 * after bias + GELU in fp32). Shared experts are not part of this form:
 * cfg->f_shared > 0 returns MOE_ERR_UNSUPPORTED. bf16 runs on the tensor
 * cores, fp32 on the FMA pipes.
 */
MOE_API moe_status moe_expert_gelu(const moe_config* cfg, const void* x_perm,
                           const int32_t* expert_offsets, const void* w1, const float* b1,
                           const void* w2, const float* b2, void* y_perm, void* workspace,
                           size_t ws_bytes, void* stream);

/*
 * moe_forward_gelu - the whole block with generic experts: route (as
 * moe_route), permute, moe_expert_gelu, combine without a shared row.
 * [L2] section 2, boxed equation: MoE(u) = sum_{i in TopK} g_i E_i(u), the
 * gate scaling the whole expert output, b2 included. y [T][d] dtype.
 * cfg->f_shared must be 0 (else MOE_ERR_UNSUPPORTED).
 */
MOE_API moe_status moe_forward_gelu(const moe_config* cfg, const void* x, const void* w_router,
                            const float* bias, const void* w1, const float* b1, const void* w2,
                            const float* b2, void* y, void* workspace, size_t ws_bytes,
                            void* stream);

/*
 * moe_backward - gradients of the block for training: given dy = dL/dy
 * ([T][d], dtype), the gradients of L with respect to x and every weight.
 * The expert choice is piecewise constant in the inputs, so gradients flow
 * through the gates ([DS] "Routing": gates from the unbiased selected s,
 * renormalised, times route_scale; [CS] "The router in code": softmax over
 * the chosen raw scores) and the expert FFNs ([DS] SwiGLU equation); the
 * selection bias gets none (it is moved by moe_balance_update).
 *
 *   x, w_router, bias, w1, w3, w2, ws1, ws3, ws2   as in moe_forward
 *   dy        [T][d]         dtype  IN: gradient with respect to y
 *   dx        [T][d]         dtype  OUT
 *   dw_router [E][d]         dtype  OUT
 *   dw1, dw3  [E][f][d]      dtype  OUT (zero for experts no token chose)
 *   dw2       [E][d][f]      dtype  OUT
 *   dws1, dws3 [f_shared][d], dws2 [d][f_shared]  dtype  OUT (NULL if f_shared == 0)
 *
 * The call recomputes the forward's routing and SwiGLU pre-activations
 * (same kernels, same results as moe_forward), so it needs only the inputs
 * and dy. Every accumulation is fp32; each output is rounded once to dtype.
 * The workspace must hold moe_backward_workspace_size(cfg) bytes (larger
 * than moe_workspace_size). T = 0 writes zero weight gradients.
 */
MOE_API size_t moe_backward_workspace_size(const moe_config* cfg);
MOE_API moe_status moe_backward(const moe_config* cfg, const void* x, const void* w_router,
                        const float* bias, const void* w1, const void* w3, const void* w2,
                        const void* ws1, const void* ws3, const void* ws2, const void* dy, void* dx,
                        void* dw_router, void* dw1, void* dw3, void* dw2, void* dws1, void* dws3,
                        void* dws2, void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_forward_train - moe_forward for training: the same y, and the
 * workspace (at least moe_backward_workspace_size(cfg) bytes) keeps what the
 * backward pass would otherwise recompute: the routing (indices, gates,
 * offsets, packed-row maps, router logits), the packed activations and the
 * SwiGLU pre-activations W1 u and W3 u of every routed and shared row
 * (dtype, written by the gate/up GEMM's epilogue).
 */
MOE_API moe_status moe_forward_train(const moe_config* cfg, const void* x, const void* w_router,
                             const float* bias, const void* w1, const void* w3, const void* w2,
                             const void* ws1, const void* ws3, const void* ws2, void* y,
                             void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_backward_saved - moe_backward on the state moe_forward_train left in
 * `workspace`: no routing, packing or pre-activation GEMMs are recomputed.
 * x and the weights must be the ones that forward call used (they feed the
 * weight gradients and the router's input gradient), and nothing may have
 * written the workspace in between. Outputs as moe_backward's.
 */
MOE_API moe_status moe_backward_saved(const moe_config* cfg, const void* x, const void* w_router,
                              const void* w1, const void* w3, const void* w2, const void* ws1,
                              const void* ws3, const void* ws2, const void* dy, void* dx,
                              void* dw_router, void* dw1, void* dw3, void* dw2, void* dws1, void* dws3,
                              void* dws2, void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_route_noalloc - moe_route for callers that cannot allocate device
 * memory (no workspace argument). Same arguments and outputs as moe_route
 * minus the workspace. The pages have no counterpart: this entry point only
 * changes where the router's scratch lives.
 *
 * Some callers have no way to obtain device scratch when they route: code
 * inside another runtime's allocation-free region, a plugin host that only
 * hands over the tensors it owns, or a process that must not grow its device
 * footprint mid-run. Here the scratch (router logits, per-chunk histograms
 * and bases, error word) is one fixed 24 MiB array in the library's device
 * image, present on every GPU that loads the library until the process
 * exits; the call itself allocates nothing.
 *  - Capacity: the call needs 256 + 4*S*T*E + 8*E*ceil(T/32) + 8*E*ceil(T/128)
 *    bytes (each term rounded up to 256), where S is the number of router
 *    partial sums kept in memory: 1 for fp32 and for bf16 with E <= 256 (one
 *    fused kernel adds the partial sums on chip); for bf16 with more experts,
 *    S = min(8, ceil(d/64), max(1, floor(148 / (ceil(T/128) * ceil(E/256))))).
 *    Beyond 24 MiB it returns MOE_ERR_WORKSPACE_TOO_SMALL before enqueuing
 *    anything.
 *  - The first call on each device looks up the array's device address
 *    (with that device current) and caches it; make that first call before
 *    any stream capture on the device.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; each call clears the error word first and overwrites the rest.
 *    Calls whose work overlaps on the GPU (two streams, two threads) race on
 *    the array and must be serialised by the caller.
 */
MOE_API moe_status moe_route_noalloc(const moe_config* cfg, const void* x, const void* w_router,
                             const float* bias, int32_t* topk_idx, float* topk_gate,
                             int32_t* expert_counts, int32_t* expert_offsets, void* stream);

/*
 * moe_route_noalloc_device_error - the error word of moe_route_noalloc's
 * fixed array on the current device, which no workspace pointer reaches.
 * The pages have no counterpart: like moe_get_device_error, this only reports
 * on the call's own bounded device waits.
 *
 * Synchronises `stream`, reads the word, clears it and returns MOE_OK or
 * MOE_ERR_TIMEOUT (a device wait of a moe_route_noalloc call on this device
 * ran out, so its routing is not to be trusted); MOE_ERR_CUDA if a CUDA call
 * fails, MOE_ERR_UNSUPPORTED for a device ordinal of 64 or more. Allocates
 * nothing. Call it on the stream of the moe_route_noalloc calls it checks,
 * with their device current; like those calls it must not overlap another
 * moe_route_noalloc on the same device.
 */
MOE_API moe_status moe_route_noalloc_device_error(void* stream);

/*
 * moe_forward_gathers_rows - 1 if moe_forward, for this configuration and
 * activation pointer x, has its gate/up GEMM gather the token rows from x
 * (moe_permute writing the maps only, as moe_expert_gate_up_gather), 0 if it
 * reads the permute's packed copy; -1 for an invalid configuration. The
 * pages have no counterpart: the two paths give the same bytes, this tells
 * a caller timing the stages which one to time. The rule: bf16, token tiles
 * of fewer than 128 rows (single-CTA GEMM tiles, e.g. decode), x 16-byte
 * aligned, T*d*2 under 4 GiB.
 */
MOE_API int moe_forward_gathers_rows(const moe_config* cfg, const void* x);

/*
 * moe_balance_update - the aux-loss-free balancing step that follows routing
 * in training, and the routing entropy.  [CS] "Aux-loss-free balance loop":
 * target usage = n_tokens * top_k / n_experts; over target, bias -= gamma;
 * under target, bias += gamma; entropy of the usage rises toward ln(E).
 *
 *   expert_counts [E]  int32  tokens per expert (moe_route's output for cfg->T tokens)
 *   bias          [E]  fp32   IN/OUT selection bias, updated in place (NULL: skip)
 *   gamma                     step size >= 0 (the page's demo uses 0.15)
 *   entropy       [1]  fp32   OUT: -sum_e p_e ln p_e, p = counts / sum(counts),
 *                             accumulated in fp64 (NULL: skip)
 *
 * An expert exactly on target keeps its bias; over/under is decided exactly
 * (count * E against T * k in integers). At least one of bias and entropy
 * must be given. One small kernel; asynchronous on `stream`.
 */
MOE_API moe_status moe_balance_update(const moe_config* cfg, const int32_t* expert_counts,
                              float* bias, float gamma, float* entropy, void* stream);

/* Synchronises `stream`, reads and clears the workspace's device error word.
 * Returns MOE_OK, MOE_ERR_TIMEOUT (a bounded device wait ran out during an
 * earlier call on this workspace), MOE_ERR_INVALID_ARG (a device-side check
 * found a caller index out of range: an expert id outside [0, E) or a
 * packed row outside [0, T*k) in moe_permute, or an expert_offsets entry
 * outside [0, T*k) or below its predecessor in the expert calls; such ids
 * and rows are skipped and such offsets clamped, so no access leaves the
 * caller's buffers, but the outputs are not defined) or MOE_ERR_CUDA. Every
 * entry point that takes a workspace clears the word when it starts. */
MOE_API moe_status moe_get_device_error(void* workspace, void* stream);

/* Launches one kernel that waits on a barrier nothing ever arrives at,
 * with a bound of timeout_ns nanoseconds, so that the bounded-wait path can
 * be exercised without hanging or faulting the GPU. The kernel records
 * MOE_ERR_TIMEOUT in the workspace's error word and returns. */
MOE_API moe_status moe_selftest_wait_timeout(void* workspace, size_t ws_bytes, int64_t timeout_ns,
                                     void* stream);

/* Static description of a status code. Never NULL. */
MOE_API const char* moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H_ */
