/*
 * moe.h -- C ABI of libmoe, the forward pass of a top-k routed
 * Mixture-of-Experts FFN layer on NVIDIA B200 (sm_100a).
 *
 * The layer (pages that define it, by title and section):
 *   router        score = x . W_r, a bias-free linear router, then a softmax
 *                 over all E experts ("MoE: gating, experts, load balancing,
 *                 capacity factor" (dpshk.com/news/6005940) §2.1);
 *   top-k         the k experts with the largest logits, their probabilities
 *                 renormalised to sum to 1 ("Llama-MoE架构解析" (coreui.cn
 *                 /article/2610641) §3.1; MoE-basics page §3.1);
 *   capacity      cap = ceil(T*k/E * capacity_factor); assignments beyond
 *                 an expert's cap are dropped in token order (MoE-basics §2.4);
 *   dispatch      assignments sorted by expert into contiguous groups
 *                 ("Hand-building a LLaMA4-MoE" (dpshk.com/news/5809432) §2.4);
 *   experts       SwiGLU (MoE-basics §2.2; Llama-MoE §2.1) or a two-matrix
 *                 FFN with bias and GELU over one flattened [E, d, ffn] weight
 *                 pool ("How to Loop MoE: Flatten the Experts, Untie the
 *                 Attention" (discosf.com/news/5228035) §2.1; MoE-basics §3.1);
 *   combine       out[t] = sum_j w[t,j] * expert_j(x[t]) (LLaMA4-MoE §2.4);
 *   load balance  f_e, p_e and L_aux = alpha * E * sum_e f_e p_e
 *                 (MoE-basics §2.3; LLaMA4-MoE §3.2).
 *
 * Conventions (all entry points):
 *   - Every tensor pointer is DEVICE memory owned by the caller, row-major,
 *     contiguous, 16-byte aligned, unless the comment says HOST.  The
 *     library never allocates or frees memory and never synchronises, except
 *     in moe_check_device_status (which synchronises the given stream) and
 *     in the moe_pipeline_* object, which owns its buffers and streams.
 *   - "act" tensors (x, x_perm, h, y_perm, out and the weights) have the
 *     config's dtype: float32 (MOE_DT_F32) or bfloat16 (MOE_DT_BF16).
 *     Router logits, probabilities, top-k weights, f, p and L_aux are float32;
 *     indices and counts are int32.  The router logit bias is float32.
 *   - Arguments are validated on the host before any launch; a bad argument
 *     returns MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE
 *     and launches nothing.  A failed launch returns MOE_ERR_CUDA.
 *   - All work is asynchronous on `stream` (0 = legacy default stream).
 *   - Device-side waits inside the kernels are bounded in time; when one
 *     gives up, the kernel records MOE_ERR_TIMEOUT in the workspace status
 *     word and returns; moe_check_device_status reports it.
 *   - Results are deterministic: two calls on the same inputs give
 *     bit-identical outputs (no atomics decide any order or sum).
 *   - Calls that share a workspace must not overlap on the GPU.  Calls with
 *     their own workspaces may be issued from several host threads at once
 *     (the library's per-device one-time setup is thread-safe).
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer */
    MOE_ERR_UNSUPPORTED = 2,  /* valid shape this build does not run (e.g. E > 64) */
    MOE_ERR_WORKSPACE = 3,    /* workspace missing or smaller than moe_workspace_size */
    MOE_ERR_CUDA = 4,         /* a CUDA call or kernel launch failed */
    MOE_ERR_TIMEOUT = 5,      /* a bounded device wait gave up (see moe_check_device_status) */
    MOE_ERR_RANGE = 6         /* a device-side bounds check refused a row (inconsistent counts;
                                 see moe_check_device_status and the expert-parallel calls) */
} moe_status_t;

typedef enum { MOE_DT_F32 = 0, MOE_DT_BF16 = 1 } moe_dtype_t;

typedef enum {
    MOE_ACT_SWIGLU = 0,     /* W_down( silu(x W_gate) * (x W_up) ) */
    MOE_ACT_GELU_BIAS = 1   /* W2( gelu_erf(x W1 + b1) ) + b2 */
} moe_act_t;

/* Router kernel.  All compute the same logits up to fp32 summation order
 * (the two warp-MMA routers exactly the same logits); each is batch-invariant
 * (a token's logits do not depend on T or on the other tokens), and the choice
 * never depends on T, so neither does the routing.
 *   MOE_ROUTER_AUTO      the library's choice for the shape (currently the
 *                        resident-weight warp-MMA router, or the staged one
 *                        where its weight slices do not fit);
 *   MOE_ROUTER_WARP_MMA  warp-level mma.sync; bf16: the router weight resident
 *                        in shared memory across a cluster of 2-8 CTAs, tokens
 *                        streamed by TMA (the staged kernel for shapes whose
 *                        slices do not fit); f32: one thread per token;
 *   MOE_ROUTER_TCGEN05   TMA + tcgen05 tensor cores + TMEM, 128-token tiles:
 *                        bf16, E % 8 == 0, d % 64 == 0, else
 *                        MOE_ERR_UNSUPPORTED;
 *   MOE_ROUTER_WARP_MMA_STAGED  warp-level mma.sync, 32-64 tokens per CTA, the
 *                        router weight staged in shared-memory slabs by every
 *                        CTA (bf16; f32 as MOE_ROUTER_WARP_MMA).
 * Fed logits (logits_in) skip the GEMM and use a warp router's softmax and
 * top-k; MOE_ROUTER_TCGEN05 with fed logits returns MOE_ERR_UNSUPPORTED (that
 * kernel has no GEMM-free path). */
typedef enum {
    MOE_ROUTER_AUTO = 0,
    MOE_ROUTER_WARP_MMA = 1,
    MOE_ROUTER_TCGEN05 = 2,
    MOE_ROUTER_WARP_MMA_STAGED = 3
} moe_router_kernel_t;

/* Expert GEMM kernel (bf16; the f32 path has one kernel).  Same results bit
 * for bit: every output element is one fp32 tensor-core sum over K in the
 * same order, rounded once.
 *   MOE_GEMM_AUTO      the library's choice per GEMM;
 *   MOE_GEMM_ONE_CTA   one CTA per 128-row tile (M=128, N=256);
 *   MOE_GEMM_CTA_PAIR  two CTAs per 256-row tile (tcgen05 cta_group::2), an
 *                      expert's last tile as a 128-row pair tile when it holds
 *                      at most 128 rows. */
typedef enum { MOE_GEMM_AUTO = 0, MOE_GEMM_ONE_CTA = 1, MOE_GEMM_CTA_PAIR = 2 } moe_gemm_kernel_t;

/* How the first expert GEMM of moe_forward / moe_dp_finish gets its rows
 * (bf16; the f32 path always copies).  Same results bit for bit.
 *   MOE_DISPATCH_AUTO    the library's choice (currently COPY: the gathered
 *                        tiles take 32 TMA gathers of four 128-byte rows per
 *                        16 KB stage, which the TMA unit issues about 3x
 *                        slower than the tensor cores consume them, so the
 *                        gathering first GEMM is slower than copy plus TMA
 *                        tiles on B200);
 *   MOE_DISPATCH_COPY    the dispatch kernel copies each kept row to the
 *                        expert-sorted x_perm, which the GEMM reads by TMA;
 *   MOE_DISPATCH_GATHER  the GEMM's producer warp gathers the token rows of x
 *                        straight into its shared-memory tiles with TMA
 *                        tile::gather4 (one-CTA kernel); the dispatch kernel
 *                        writes only slot and src_assign, and x_perm is never
 *                        written. */
typedef enum { MOE_DISPATCH_AUTO = 0, MOE_DISPATCH_COPY = 1, MOE_DISPATCH_GATHER = 2 } moe_dispatch_mode_t;

/* Storage of the routed experts' weights.
 *   MOE_WEIGHTS_NATIVE  the config's dtype;
 *   MOE_WEIGHTS_INT8    INT8 codes with a per-expert, per-output-column fp32
 *                       scale (from moe_quantize_int8; the long-context MoE
 *                       page §3): the layer uses the weights codes * scale.
 *                       bf16 activations only.  Built for decode-sized batches
 *                       (a few rows per expert): it halves the weight bytes the
 *                       FFNs stream.  Shared experts keep native weights. */
typedef enum { MOE_WEIGHTS_NATIVE = 0, MOE_WEIGHTS_INT8 = 1 } moe_weight_format_t;

/* Where moe_forward and moe_dp_finish apply the routing weights topk_w.
 *   MOE_WEIGHTING_AUTO      the library's choice: EPILOGUE where it applies
 *                           (bf16 with native weights), else COMBINE;
 *   MOE_WEIGHTING_COMBINE   y_perm holds each expert's output rounded to the
 *                           dtype, and the combine forms sum_j w[t,j] y(t,j)
 *                           in fp32;
 *   MOE_WEIGHTING_EPILOGUE  bf16 with native weights: the second expert GEMM
 *                           multiplies each fp32 output row (after b2) by its
 *                           routing weight before its one rounding to bf16
 *                           ("Loop-MoE" §2.1 / MoE-basics §4.4: the weighted
 *                           expert output is formed per row), and the combine
 *                           is a plain fp32 sum of the k weighted rows.  The
 *                           other dtypes and INT8 weights fall back to COMBINE.
 * The two orders round differently (last bits of out); both are within the
 * layer's bf16 tolerance.  The expert-parallel calls and moe_combine always
 * weight in the combine. */
typedef enum { MOE_WEIGHTING_AUTO = 0, MOE_WEIGHTING_COMBINE = 1, MOE_WEIGHTING_EPILOGUE = 2 } moe_weighting_t;

/* Layer shape.  Limits: 0 <= T, T*k < 2^31; 1 <= E <= 64; 1 <= k <= min(E, 8).
 * bf16: d % 64 == 0 and ffn % 64 == 0.  f32: d % 4 == 0 and ffn % 4 == 0. */
typedef struct {
    int64_t T;                 /* tokens (batch * sequence) */
    int32_t d;                 /* model (hidden) dimension */
    int32_t ffn;               /* expert intermediate dimension */
    int32_t E;                 /* number of experts */
    int32_t k;                 /* experts per token (top-k) */
    int32_t dtype;             /* moe_dtype_t */
    int32_t act;               /* moe_act_t */
    double capacity_factor;    /* <= 0: no capacity limit (cap = T) */
    float aux_alpha;           /* alpha of L_aux */
    int32_t router_kernel;     /* moe_router_kernel_t (0: library's choice) */
    int32_t gemm_kernel;       /* moe_gemm_kernel_t (0: library's choice) */
    int32_t dispatch;          /* moe_dispatch_mode_t (0: library's choice) */
    int32_t n_shared;          /* shared experts, 0..8 (LLaMA4-MoE §5.2; see moe_forward) */
    int32_t weight_format;     /* moe_weight_format_t of the routed experts */
    int32_t weighting;         /* moe_weighting_t (0: library's choice) */
} moe_config_t;

/* Expert and router parameters (device, config dtype unless stated). */
typedef struct {
    const void* w_router;            /* [d, E] */
    const float* router_logit_bias;  /* [E] float32 added to the logits before the softmax, or NULL */
    const void* w_gate_or_w1;        /* [E, d, ffn]  SwiGLU W_gate | GELU W1 */
    const void* w_up;                /* [E, d, ffn]  SwiGLU W_up   | NULL */
    const void* w_down_or_w2;        /* [E, ffn, d]  SwiGLU W_down | GELU W2 */
    const void* b1;                  /* [E, ffn] GELU only, else NULL */
    const void* b2;                  /* [E, d]   GELU only, else NULL */
    /* shared experts (n_shared > 0), same form and layout per expert as the routed ones */
    const void* shared_gate_or_w1;   /* [S, d, ffn] */
    const void* shared_up;           /* [S, d, ffn] SwiGLU only, else NULL */
    const void* shared_down_or_w2;   /* [S, ffn, d] */
    const void* shared_b1;           /* [S, ffn] GELU only, else NULL */
    const void* shared_b2;           /* [S, d]   GELU only, else NULL */
    /* MOE_WEIGHTS_INT8: w_gate_or_w1 / w_up / w_down_or_w2 hold int8 codes and these their scales */
    const float* gate_or_w1_scale;   /* [E, ffn] */
    const float* up_scale;           /* [E, ffn] SwiGLU only, else NULL */
    const float* down_or_w2_scale;   /* [E, d] */
} moe_weights_t;

/* Outputs of moe_forward (device).  R_max = moe_max_rows(). */
typedef struct {
    void* out;             /* [T, d] layer output, token order */
    int32_t* topk_idx;     /* [T, k] selected experts, best first (ties: lower id) */
    float* topk_w;         /* [T, k] renormalised routing weights */
    int32_t* counts;       /* [E] router selections per expert, before the capacity cut */
    int32_t* offsets;      /* [E+1] start row of each expert's kept rows; offsets[E] = R */
    int32_t* slot;         /* [T, k] row of assignment (t, j) in the expert-sorted buffers, or -1 if dropped */
    int32_t* src_assign;   /* [R_max] t*k + j of each sorted row (first R entries written) */
    float* f;              /* [E] f_e = counts_e / (T*k) */
    float* p;              /* [E] p_e = mean over tokens of the full softmax */
    float* l_aux;          /* [1] alpha * E * sum_e f_e p_e */
    float* logits_out;     /* [T, E] router logits (bias included), or NULL */
    float* probs_out;      /* [T, E] full softmax, or NULL */
} moe_outputs_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_status_string(moe_status_t status);

/* Per-expert capacity, evaluated on the host in double exactly as
 * ceil(((double)T * k / E) * capacity_factor); capacity_factor <= 0 gives T.
 * (MoE-basics §2.4, scaled by k because the buffer holds assignments.) */
moe_status_t moe_capacity(const moe_config_t* cfg, int64_t* cap);

/* Upper bound on dispatched rows: R_max = min(T*k, E*cap).  Size of the
 * src_assign array and row count of x_perm / y_perm buffers. */
moe_status_t moe_max_rows(const moe_config_t* cfg, int64_t* rows);

/* Bytes of workspace the calls below need for this config (x_perm, h, y_perm,
 * per-chunk histograms, probability sums, group bases, and a 64 KB status
 * block at its start). */
moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* bytes);

/* Zero the workspace's 64 KB status block: the status word, and the counters
 * the router and dispatch kernels add into and return to zero within every
 * launch (per-group expert counts, real-token and arrival counts).  Call once
 * after allocating a workspace, before its first use; a status check that
 * reports an error clears the block again itself.  Asynchronous on `stream`. */
moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream);

/* Router + softmax + top-k + renormalisation (MoE-basics §2.1, §3.1;
 * Llama-MoE §3.1).
 *   x [T,d], w_router [d,E]; logit_bias [E] float32 or NULL.
 *   logits_in [T,E] float32 or NULL: when given, these logits (bias already
 *     included) replace x . W_r + bias -- used to feed both this library and a
 *     reference identical logits.
 *   token_mask [T] uint8 or NULL: tokens with 0 are padding (LLaMA4-MoE §4.1
 *     keeps them out of expert selection): their topk_idx is -1 and topk_w 0.
 *   topk_idx [T,k] int32, topk_w [T,k] float32 (outputs).
 *   logits_out, probs_out [T,E] float32 or NULL (optional outputs; written for
 *     every token, padding included).
 * Top-k compares fp32 logits, lower id first on ties.  Needs a workspace. */
moe_status_t moe_router_topk(const moe_config_t* cfg, const void* x, const void* w_router,
                             const float* logit_bias, const float* logits_in, const uint8_t* token_mask,
                             int32_t* topk_idx, float* topk_w, float* logits_out, float* probs_out,
                             void* ws, size_t ws_bytes, cudaStream_t stream);

/* Quantise expert weights w [E, K, N] (config dtype, on the device) to INT8
 * codes q [E, K, N] (int8) and scales scale [E, N] (float32), per expert and
 * output column n: scale = max_k |w[e,k,n]| / 127, q = clamp(rint(w / scale),
 * -127, 127), ties to even, all in fp32; an all-zero column gets scale 0 and
 * codes 0 (the long-context MoE page §3: a scale per expert and per
 * dimension).  For SwiGLU call it for W_gate and W_up (K = d, N = ffn) and
 * W_down (K = ffn, N = d).  Asynchronous on `stream`. */
moe_status_t moe_quantize_int8(const moe_config_t* cfg, const void* w, int64_t K, int64_t N, int8_t* q, float* scale,
                               cudaStream_t stream);

/* Capacity-bounded dispatch (MoE-basics §2.4; LLaMA4-MoE §2.4).
 *   topk_idx [T,k] int32 in [0,E), or -1 (selects nothing: padding).
 *   Outputs: counts [E], offsets [E+1],
 *   slot [T,k], src_assign [R_max] (first offsets[E] entries), and
 *   x_perm [R_max, d] whose row s is x[src_assign[s] / k].
 * Assignment (t,j) has rank = number of earlier assignments (token-major
 * order) to the same expert; it is kept iff rank < cap.  Needs a workspace. */
moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                          int32_t* counts, int32_t* offsets, int32_t* slot, int32_t* src_assign,
                          void* x_perm, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Allocation-free variant of moe_dispatch, for callers that cannot allocate
 * device memory (for instance a plugin that is handed only its input and
 * output buffers by a host framework owning all allocations, or a loop that
 * must not allocate after start-up) and so cannot supply a workspace.  The
 * pages have no counterpart: this is a property of the library, not of the
 * method.  Same arguments, results and errors as moe_dispatch, minus the
 * workspace.  Its scratch (per-chunk histograms, per-group counts and rank
 * bases) is a fixed 632 KiB array in the library's device memory on every GPU
 * that loads it; shapes with ceil(T/32)*E > 131072 (E = 64: T > 65536) return
 * MOE_ERR_UNSUPPORTED.  Each call clears the counts it adds into with a
 * cudaMemsetAsync on that array (no allocation).  The first
 * call on a device looks up that array's address and should come before any
 * stream capture.  All calls on a device share the array: calls that overlap
 * on the GPU race and must be serialised by the caller. */
moe_status_t moe_dispatch_noalloc(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                  int32_t* counts, int32_t* offsets, int32_t* slot, int32_t* src_assign,
                                  void* x_perm, cudaStream_t stream);

/* Expert FFNs over the expert-sorted rows (Loop-MoE §2.1 weight pool;
 * MoE-basics §2.2, §3.1).  Rows [offsets[e], offsets[e+1]) of x_perm [R_max,d]
 * go through expert e; y_perm [R_max, d] receives the results (rows >= R are
 * not written).  bf16 runs on the tensor cores (fp32 accumulation; the
 * intermediate activation is rounded to bf16 once); f32 runs in fp32 FMA.
 * The intermediate [R_max, ffn] activation lives in the workspace. */
moe_status_t moe_expert_ffn(const moe_config_t* cfg, const moe_weights_t* weights, const void* x_perm,
                            const int32_t* offsets, void* y_perm, void* ws, size_t ws_bytes,
                            cudaStream_t stream);

/* Weighted combine back to token order (LLaMA4-MoE §2.4; MoE-basics §3.1):
 * out[t] = sum over j with slot[t,j] >= 0 of topk_w[t,j] * y_perm[slot[t,j]],
 * accumulated in fp32 in ascending j; a token with every assignment dropped
 * gets 0; surviving weights are not renormalised. */
moe_status_t moe_combine(const moe_config_t* cfg, const void* y_perm, const int32_t* slot,
                         const float* topk_w, void* out, cudaStream_t stream);

/* Load-balance statistics (MoE-basics §2.3, §3.1; LLaMA4-MoE §3.2):
 * f_e = counts_e / (T*k), p_e = (1/T) sum_t probs[t,e] (probs [T,E] float32,
 * the full softmax), l_aux = alpha * E * sum_e f_e p_e.  T = 0 gives zeros. */
moe_status_t moe_aux_stats(const moe_config_t* cfg, const int32_t* counts, const float* probs,
                           float* f, float* p, float* l_aux, cudaStream_t stream);

/* The whole layer forward: router, top-k, dispatch, expert FFNs, combine and
 * aux statistics on `stream` (moe_forward_launch_count launches).
 *   logits_in as in moe_router_topk (NULL in normal use).
 *   token_mask [T] uint8 or NULL: padding tokens (0) select no expert, get no
 *     routed output and are left out of f and p, which divide by the number
 *     of real tokens; the capacity stays that of the whole batch.
 *   n_shared > 0: the shared experts (weights->shared_*) run on every token,
 *     padding included, and out[t] = sum_j w[t,j] y(t,j) + sum_s y_s(t),
 *     accumulated in fp32 (routed terms first, then shared experts in order)
 *     and rounded once.
 *   cfg->weighting: whether w[t,j] y(t,j) is formed in the second GEMM's
 *     epilogue (rounded there) or in the combine (moe_weighting_t).
 * Every launch after the router uses programmatic dependent launch: it may
 * start while the kernel before it finishes and waits on the device before
 * reading that kernel's results (no effect on results; the router itself is
 * launched plainly, so consecutive forwards on a stream never overlap). */
moe_status_t moe_forward(const moe_config_t* cfg, const moe_weights_t* weights, const void* x,
                         const float* logits_in, const uint8_t* token_mask, moe_outputs_t* outputs, void* ws,
                         size_t ws_bytes, cudaStream_t stream);

/* ---- Data-parallel sharding of one logical batch ----------------------
 * One batch of T_global tokens split in contiguous slices over `world` ranks
 * (rank r holds its slice as a batch of cfg->T tokens, slices in rank order),
 * with the capacity, the drop order and the load-balance statistics of the
 * WHOLE batch: under data parallelism the per-expert token counts are summed
 * over replicas before the load-balance loss ("Hand-building a LLaMA4-MoE"
 * §3.1), and the capacity cut then drops in the batch's token order.  Results
 * equal a single moe_forward over the whole batch (row indices local).
 *   1. moe_dp_route on every rank: router and top-k of the slice; writes the
 *      slice's per-expert counts local_counts [E] (int32, device),
 *      probability sums local_psum [E] (float64, device) and, if local_real
 *      is not NULL, its number of real tokens local_real [1] (int32, device).
 *   2. the caller all-gathers them in rank order into all_counts [world, E],
 *      all_psum [world, E] and all_real [world] (device), e.g. with NCCL.
 *   3. moe_dp_finish on every rank: capacity left for the slice, dispatch,
 *      expert FFNs, combine; outputs->counts, f, p, l_aux are the whole
 *      batch's (identical on every rank).
 * token_mask (DEVICE [cfg->T] uint8, or NULL) marks padding as in moe_forward:
 * a padding token selects no expert and f and p divide by the whole batch's
 * real tokens, the sum of all_real (all_real NULL: every token is real).
 * With a mask, local_real must be given and exchanged.  The capacity stays
 * that of all T_global tokens.
 * Both calls use the same workspace of moe_dp_workspace_size bytes; outputs
 * src_assign and the sorted-row buffers hold up to moe_dp_max_rows rows. */
moe_status_t moe_dp_workspace_size(const moe_config_t* cfg, int64_t T_global, size_t* bytes);
moe_status_t moe_dp_max_rows(const moe_config_t* cfg, int64_t T_global, int64_t* rows);
moe_status_t moe_dp_route(const moe_config_t* cfg, int64_t T_global, const moe_weights_t* weights, const void* x,
                          const float* logits_in, const uint8_t* token_mask, moe_outputs_t* outputs,
                          int32_t* local_counts, double* local_psum, int32_t* local_real, void* ws, size_t ws_bytes,
                          cudaStream_t stream);
moe_status_t moe_dp_finish(const moe_config_t* cfg, int64_t T_global, const int32_t* all_counts,
                           const double* all_psum, const int32_t* all_real, int32_t world, int32_t rank,
                           const moe_weights_t* weights, const void* x, moe_outputs_t* outputs, void* ws,
                           size_t ws_bytes, cudaStream_t stream);

/* ---- Expert parallelism: experts sharded over ranks --------------------
 * "Hand-building a LLaMA4-MoE" §2.5 and the MoE-basics page §4.1: each GPU
 * holds some of the experts; an all-to-all sends every token to the GPUs
 * holding its experts and a second one brings the results back.  Here `world`
 * ranks (1..8, the GPUs of one NVSwitch node) each hold
 *   - a contiguous slice of one batch of T_global tokens (cfg->T tokens,
 *     slices in rank order), as in the data-parallel calls above, and
 *   - the experts [rank*E/world, (rank+1)*E/world) (E % world == 0), whose
 *     weights are passed as a pool of E/world experts ([E/world, d, ffn] ...);
 *     the router weights and the shared experts are replicated.
 * Capacity, drops and statistics are the whole batch's; every expert's rows
 * reach its rank in the batch's token order, so the layer output equals one
 * moe_forward over the whole batch, bit for bit.
 *
 * Each rank owns two receive buffers of moe_ep_recv_rows rows: x_recv
 * [rows, d] and y_recv [rows, d] (config dtype), on its own GPU.  The
 * dispatch and combine calls take the array of every rank's buffer
 * (x_recv[r] / y_recv[r], r = 0..world-1, HOST array of DEVICE pointers that
 * this rank can dereference: its own buffer and its peers' buffers mapped
 * into this process, e.g. with moe_ipc_open over NVLink).  The kernels
 * store token rows straight into the owners' x_recv (dispatch) and load
 * expert rows straight from the owners' y_recv (combine): the two
 * all-to-alls are fused into the scatter and the weighted sum.
 *
 * Sequence on every rank (the same steps on all ranks, even with no rows):
 *   1. moe_ep_route: router and top-k of the slice, local_counts [E] int32,
 *      local_psum [E] float64 and local_real [1] int32 (device; as in
 *      moe_dp_route, including the padding mask).
 *   2. all-gather local_counts / local_psum / local_real in rank order into
 *      all_counts [world, E] / all_psum [world, E] / all_real [world]
 *      (e.g. NCCL).
 *   3. moe_ep_dispatch: capacity left, rows into the owners' x_recv,
 *      outputs->slot [T,k] = row in the owner's y_recv (or -1), recv_offsets
 *      [E/world + 1] = this rank's received rows per local expert, and the
 *      whole batch's counts, offsets (single-device layout), f, p, l_aux.
 *   4. barrier: every rank's step 3 finished (e.g. a one-word NCCL
 *      all-reduce on the stream).
 *   5. moe_ep_expert_ffn: grouped GEMMs over x_recv -> y_recv with this
 *      rank's experts; the shared experts over the slice's tokens.
 *   6. barrier: every rank's step 5 finished.
 *   7. moe_ep_combine: outputs->out [T,d] of the slice.
 * The receive buffers must not be reused by the next forward's step 3 before
 * every rank's step 7 finished (the all-gather of step 2 orders that).
 * All four calls use one workspace of moe_ep_workspace_size bytes per rank. */
moe_status_t moe_ep_recv_rows(const moe_config_t* cfg, int64_t T_global, int32_t world, int64_t* rows);
moe_status_t moe_ep_workspace_size(const moe_config_t* cfg, int64_t T_global, int32_t world, size_t* bytes);
moe_status_t moe_ep_route(const moe_config_t* cfg, int64_t T_global, int32_t world, const moe_weights_t* weights,
                          const void* x, const float* logits_in, const uint8_t* token_mask, moe_outputs_t* outputs,
                          int32_t* local_counts, double* local_psum, int32_t* local_real, void* ws, size_t ws_bytes,
                          cudaStream_t stream);
/* all_counts / all_psum / all_real: DEVICE [world, E] / [world, E] / [world]
 * as gathered in step 2 (all_real may be NULL: every token is real); counts
 * that do not match the routing make the kernels refuse rows (MOE_ERR_RANGE
 * from moe_check_device_status; memory stays in bounds). */
moe_status_t moe_ep_dispatch(const moe_config_t* cfg, int64_t T_global, const int32_t* all_counts,
                             const double* all_psum, const int32_t* all_real, int32_t world, int32_t rank,
                             const void* x,
                             void* const* x_recv, moe_outputs_t* outputs, int32_t* recv_offsets, void* ws,
                             size_t ws_bytes, cudaStream_t stream);
/* weights: the E/world local experts (and the shared experts); x: the
 * slice's tokens (read only by the shared experts; may be NULL without
 * them); x_recv / y_recv / recv_offsets: this rank's own. */
moe_status_t moe_ep_expert_ffn(const moe_config_t* cfg, int64_t T_global, int32_t world,
                               const moe_weights_t* weights, const void* x, const void* x_recv,
                               const int32_t* recv_offsets, void* y_recv, void* ws, size_t ws_bytes,
                               cudaStream_t stream);
moe_status_t moe_ep_combine(const moe_config_t* cfg, int64_t T_global, int32_t world, const void* const* y_recv,
                            moe_outputs_t* outputs, void* ws, size_t ws_bytes, cudaStream_t stream);

/* ---- Device buffers shared between processes (CUDA IPC) ----------------
 * A record that names a device buffer for other processes of the node.
 * moe_ipc_export fills it for the buffer at dev_ptr (inside any cudaMalloc
 * allocation: the record holds the allocation's handle and dev_ptr's offset
 * in it); moe_ipc_open maps it into the calling process (with peer access
 * enabled, so that kernels load and store it over NVLink) and returns the
 * device pointer of dev_ptr there; moe_ipc_close unmaps it.  The exporting
 * process keeps the allocation alive until every importer has closed it.
 * A process cannot open its own records.  MOE_ERR_CUDA when CUDA refuses. */
typedef struct {
    uint8_t handle[64];   /* cudaIpcMemHandle_t of the allocation */
    uint64_t offset;      /* dev_ptr - allocation base */
    uint64_t bytes;       /* allocation size - offset */
} moe_ipc_buffer_t;
moe_status_t moe_ipc_export(const void* dev_ptr, moe_ipc_buffer_t* record);
moe_status_t moe_ipc_open(const moe_ipc_buffer_t* record, void** dev_ptr);
moe_status_t moe_ipc_close(void* dev_ptr, const moe_ipc_buffer_t* record);

/* moe_forward, recording stage_events[i] on `stream` just before kernel
 * launch i and stage_events[n] after the last launch, n =
 * moe_forward_launch_count(cfg) (stage_events: caller-created CUDA events,
 * at least n+1 of them).  For per-stage timing of the very same launch
 * sequence; the computation is identical to moe_forward.  While `stream` is
 * being captured into a CUDA graph the events are recorded as external records
 * (cudaEventRecordExternal), so the marks still time each replay.
 *
 * Graph capture: moe_forward and moe_forward_profiled make no host
 * synchronisation and allocate nothing, so a forward on fixed buffers may be
 * captured (after one uncaptured call on the device, which sets the kernels'
 * attributes) and replayed; a replay reads x and the weights as they are at
 * replay time. */
moe_status_t moe_forward_profiled(const moe_config_t* cfg, const moe_weights_t* weights, const void* x,
                                  const float* logits_in, const uint8_t* token_mask, moe_outputs_t* outputs,
                                  void* ws, size_t ws_bytes, cudaStream_t stream, cudaEvent_t* stage_events);

/* moe_forward with the token activations in HOST memory: copies x_host
 * (HOST, [T,d], pinned for asynchronous copies) to x_dev (device, [T,d]),
 * runs moe_forward, and copies outputs->out to out_host (HOST, [T,d]) and
 * outputs->l_aux to l_aux_host (HOST, 1 float).  Plain cudaMemcpyAsync on
 * `stream`; the caller synchronises the stream before reading the host
 * buffers. */
moe_status_t moe_forward_hostio(const moe_config_t* cfg, const moe_weights_t* weights, const void* x_host,
                                void* x_dev, moe_outputs_t* outputs, void* out_host, float* l_aux_host,
                                void* ws, size_t ws_bytes, cudaStream_t stream);

/* Synchronises `stream`, then reads the workspace status word.
 * Returns MOE_ERR_TIMEOUT if a bounded device wait gave up since the last
 * check (`*site`, if not NULL, receives the code of the first wait that gave
 * up), else MOE_ERR_RANGE if a device-side bounds check refused a row (the
 * expert-parallel calls given counts that do not match the routing),
 * MOE_ERR_CUDA if the synchronisation failed, else MOE_OK.  After an error it
 * zeroes the whole status block (a launch that gave up may have left its
 * counters partly added), so the workspace is ready for the next call. */
moe_status_t moe_check_device_status(void* ws, size_t ws_bytes, cudaStream_t stream, uint32_t* site);

/* ---- Pipelined forwards on host-resident batches ------------------------
 * A stream of layer forwards whose inputs and outputs live in HOST memory
 * (pinned, e.g. cudaHostAlloc, for the copies to run asynchronously).  Step i
 * copies its batch in, runs moe_forward on it and copies the layer output and
 * L_aux back; the copy in of step i+1, the forward of step i and the copy out
 * of step i-1 run at the same time (three streams; `depth` device buffer
 * slots for x and out).  Each step's results are those of moe_forward on the
 * same batch, bit for bit.  The object allocates its device buffers, workspace
 * and routing outputs with cudaMalloc on the current device at creation and
 * frees them in moe_pipeline_destroy; `weights` (device, caller-owned) must
 * stay valid and unchanged until then.  Not thread-safe: one host thread at a
 * time per pipeline. */
#define MOE_PIPELINE_MAX_DEPTH 4
typedef struct moe_pipeline moe_pipeline_t;

/* depth: 1..MOE_PIPELINE_MAX_DEPTH slots (2 overlaps copy in, forward and
 * copy out).  *pipe receives the object, or NULL on error.  Returns
 * MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED for a bad config, weights or
 * depth (nothing allocated), MOE_ERR_CUDA if an allocation or stream creation
 * failed (everything released). */
moe_status_t moe_pipeline_create(const moe_config_t* cfg, const moe_weights_t* weights, int32_t depth,
                                 moe_pipeline_t** pipe);

/* Queues one step: x_host (HOST, [T,d] config dtype) -> forward ->
 * out_host (HOST, [T,d]) and l_aux_host (HOST, 1 float).  Returns without
 * waiting; x_host must not change and out_host / l_aux_host must not be read
 * until moe_pipeline_wait(ticket) returns.  start_event (if not NULL) is
 * recorded just before the copy in, end_event (if not NULL) just after the
 * copy out, for device-side timing.  *ticket (if not NULL) receives the
 * step's number (0, 1, ...). */
moe_status_t moe_pipeline_submit(moe_pipeline_t* pipe, const void* x_host, void* out_host, float* l_aux_host,
                                 cudaEvent_t start_event, cudaEvent_t end_event, int64_t* ticket);

/* Blocks until step `ticket`'s results are in host memory (ticket < 0: every
 * submitted step).  MOE_ERR_INVALID_ARG for a ticket not yet submitted. */
moe_status_t moe_pipeline_wait(moe_pipeline_t* pipe, int64_t ticket);

/* moe_check_device_status on the pipeline's workspace (synchronises its
 * compute stream). */
moe_status_t moe_pipeline_check(moe_pipeline_t* pipe, uint32_t* site);

/* Waits for every queued step, then frees everything the object holds. */
moe_status_t moe_pipeline_destroy(moe_pipeline_t* pipe);

/* Time limit of every bounded device wait, in milliseconds (default 2000).
 * Applies to launches made after the call; process-wide. */
void moe_set_wait_timeout_ms(uint32_t ms);

/* Self-test of the bounded-wait path: launches one block that waits on an
 * mbarrier phase and on a workspace flag that nothing completes, each with a
 * limit of `timeout_ms`.  Both waits give up; the status word then reports
 * MOE_ERR_TIMEOUT through moe_check_device_status.  Used by the failure
 * tests; faults and hangs nothing. */
moe_status_t moe_selftest_bounded_wait(void* ws, size_t ws_bytes, uint32_t timeout_ms, cudaStream_t stream);

/* Number of kernel launches moe_forward makes for this config. */
int32_t moe_forward_launch_count(const moe_config_t* cfg);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
