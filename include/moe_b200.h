/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) gpt-oss MoE feed-forward block.
 *
 * The block (one call of moe_forward) computes, for every token t:
 *   xn_t   = x_t / sqrt(mean(x_t^2) + eps) * norm_scale
 *              -- RMSNorm: "gpt-oss-20B" hub page (pomoai.com), section 3.2;
 *                 no bias, no mean subtraction: pnsm.cn overview, section 2.3
 *   l_t    = router_w . xn_t + router_b            (fp32 logits)
 *              -- linear router: "gpt-oss-20B" page, section 3.4
 *   S_t    = the top_k largest logits, ties to the lower expert index;
 *   w_t,i  = softmax over the chosen logits
 *              -- top-4 and softmax over the chosen experts: pnsm.cn overview,
 *                 section 2.2; config.json read-out (youleyou.com)
 *   h      = g * sigmoid(1.702 g) * (u + 1),  g = min(z_gate, 7), u = clamp(z_lin, -7, 7),
 *            z = W13_e xn_t + b13_e
 *   o      = W2_e h + b2_e
 *              -- gated SwiGLU with the clamp and the "+1": "gpt-oss-20B" page,
 *                 section 3.3
 *   y_t    = x_t + sum_i w_t,i * o_t,i            (weighted combine + residual)
 * with W13 and W2 in MXFP4 (pnsm.cn overview, sections 1 and 4: MoE weights in
 * MXFP4, about 4.25 bits per weight): 4-bit E2M1 codes, 32 consecutive
 * elements of a row share one E8M0 scale byte s (value 2^(s-127)).
 *
 * Conventions
 *   - Every tensor argument is a DEVICE pointer owned by the caller, row-major,
 *     with no padding.  bf16 tensors are passed as uint16_t bit patterns.
 *     Every pointer must be 16-byte aligned, the two code tensors (w13_codes,
 *     w2_codes) 32-byte aligned (cudaMalloc gives 256).
 *   - Calls are asynchronous on `stream` (a cudaStream_t, may be NULL for the
 *     legacy default stream).  A return value reports argument or launch
 *     errors only; errors raised on the device (a bounded wait that ran out)
 *     are latched in the context and reported by moe_sync_status.
 *   - Return values: MOE_OK (0) or one of the negative MOE_ERR_* codes.  No
 *     C++ exception crosses this boundary.
 *   - The library runs only on compute capability 10.0 (B200, sm_100a);
 *     moe_init returns MOE_ERR_UNSUPPORTED elsewhere.
 *
 * Layouts (E experts, d = d_model, F = d_ff, T tokens, k = top_k)
 *   x, y           bf16 [T, d]
 *   norm_scale     bf16 [d]
 *   router_w       bf16 [E, d]           router_b  fp32 [E]
 *   w13_codes      u8   [E, 2F, d/2]     rows [0,F) are the gate, [F,2F) the
 *                                         linear part; element 2m of a row is the
 *                                         low nibble of byte m
 *   w13_scales     u8   [E, 2F, d/32]    E8M0 byte of each 32-element block
 *   b13            bf16 [E, 2F]
 *   w2_codes       u8   [E, d, F/2]      w2_scales u8 [E, d, F/32]
 *   b2             bf16 [E, d]
 *   topk_idx_out   int32 [T, k]          topk_w_out fp32 [T, k]   (optional)
 */
#ifndef MOE_B200_H
#define MOE_B200_H

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

#define MOE_OK               0
#define MOE_ERR_ARG         -1   /* null pointer, bad size, misalignment, T > T_max, bad top_k */
#define MOE_ERR_CUDA        -2   /* a CUDA runtime call or kernel launch failed */
#define MOE_ERR_TIMEOUT     -3   /* a device-side bounded wait ran out (latched) */
#define MOE_ERR_UNSUPPORTED -4   /* not a compute capability 10.0 device */
#define MOE_ERR_NOMEM       -5   /* device workspace allocation failed */

typedef struct {
    int   T_max;      /* largest token count a moe_forward call may pass */
    int   d_model;    /* d: multiple of 64, 64..6144 */
    int   d_ff;       /* F: multiple of 64, 64..6144 */
    int   n_experts;  /* E: 1..256 */
    int   top_k;      /* largest k a call may pass: 1..min(E, 8) */
    float eps;        /* RMSNorm epsilon, added to the mean square */
} moe_shape_t;

typedef struct moe_ctx moe_ctx_t;

/* Create a context for `shape` on the current CUDA device.  Allocates the
 * device workspace sized for shape->T_max (routing arrays, the fp32 normalised
 * activations, the expert-sorted activations and the SwiGLU output h in the
 * E4M3 terms the block-scaled expert GEMMs read, and the fp32
 * weighted expert rows [T_max*k, d]).  The context owns the workspace; free it with
 * moe_destroy.  Returns MOE_ERR_ARG for an invalid shape, MOE_ERR_UNSUPPORTED
 * off B200, MOE_ERR_NOMEM when the workspace does not fit. */
MOE_API int moe_init(const moe_shape_t *shape, moe_ctx_t **out);

/* Free the context and its workspace (after synchronising its last stream).
 * NULL is accepted. */
MOE_API int moe_destroy(moe_ctx_t *ctx);

/* The whole block for T tokens (0 <= T <= T_max, 1 <= top_k <= shape.top_k):
 * route (RMSNorm, router, top-k, softmax), group the (token, expert) pairs by
 * expert, gate/up grouped GEMM with the SwiGLU epilogue, down grouped GEMM
 * with each row scaled by its routing weight, and y = x + the token's rows in
 * a fixed order, cast to bf16.  It is the stage calls below, except that a
 * decode-sized batch (T <= 64, d_model <= 3072) routes and groups in one
 * launch and, when d_model == d_ff, runs both GEMMs as moe_expert_ffn: the
 * outputs equal the stages' bit for bit.  y must not alias x or any weight.  topk_idx_out / topk_w_out may be NULL; when given
 * they receive the chosen experts (in descending logit order) and their
 * softmax weights. */
MOE_API int moe_forward(moe_ctx_t *ctx, int T,
                const uint16_t *x,
                const uint16_t *router_w, const float *router_b,
                const uint8_t *w13_codes, const uint8_t *w13_scales, const uint16_t *b13,
                const uint8_t *w2_codes, const uint8_t *w2_scales, const uint16_t *b2,
                const uint16_t *norm_scale, int top_k,
                uint16_t *y, int32_t *topk_idx_out, float *topk_w_out,
                void *stream);

/* The five stages of moe_forward, callable one by one on the same context
 * and stream, in this order:
 *   moe_route        RMSNorm, router logits, top-k and softmax;
 *   moe_group        expert histogram, prefix sum and the stable permutation
 *                    of (token, expert) pairs into expert-contiguous rows,
 *                    then the expert-sorted copy of the normalised tokens;
 *   moe_expert_up    gate/up grouped GEMM with the clamped-SwiGLU epilogue;
 *                    for batches over 64 tokens it first reads both weight
 *                    tensors' scale bytes (w13_scales, w2_scales) to plan which
 *                    weight blocks of the two GEMMs take a pass over the third
 *                    E4M3 activation term (blocks with an E8M0 byte >= 126);
 *   moe_expert_down  down grouped GEMM, each row scaled by its routing weight;
 *   moe_finalize     y = x + the token's weighted expert rows (bf16), in a
 *                    fixed order, so results are reproducible run to run.
 * They exist for per-stage timing and tests; intermediate results stay in the
 * context's workspace (see moe_copy_workspace).  moe_finalize needs the same
 * x that moe_route was given.  moe_expert_down reads the routing arrays (and,
 * for batches over 64 tokens, moe_expert_up's pass plan) before it waits for
 * the kernel before it: call it right after moe_expert_up (a call
 * in another order computes nothing useful, but every row index it uses stays
 * inside the workspace).
 *
 * moe_expert_ffn runs moe_expert_up and moe_expert_down as one persistent
 * launch, for decode-sized batches (T <= 64, top_k * T <= 512) of a context with
 * d_model == d_ff: a down work item starts once every gate/up item of its token
 * block has written its h rows (per-token-block counters in the workspace,
 * zeroed by moe_group and by moe_forward's route + group launch, so a moe_group
 * must come before every moe_expert_ffn).  Same outputs as the two calls, bit for
 * bit.  Returns MOE_ERR_UNSUPPORTED (and launches nothing) for other batches and
 * shapes: call the two stages then. */
MOE_API int moe_route(moe_ctx_t *ctx, int T, const uint16_t *x, const uint16_t *norm_scale,
              const uint16_t *router_w, const float *router_b, int top_k, void *stream);
MOE_API int moe_group(moe_ctx_t *ctx, int T, int top_k, void *stream);
MOE_API int moe_expert_up(moe_ctx_t *ctx, int T, int top_k, const uint8_t *w13_codes, const uint8_t *w13_scales,
                  const uint16_t *b13, const uint8_t *w2_scales, void *stream);
MOE_API int moe_expert_down(moe_ctx_t *ctx, int T, int top_k, const uint8_t *w2_codes, const uint8_t *w2_scales,
                    const uint16_t *b2, void *stream);
MOE_API int moe_expert_ffn(moe_ctx_t *ctx, int T, int top_k, const uint8_t *w13_codes, const uint8_t *w13_scales,
                   const uint16_t *b13, const uint8_t *w2_codes, const uint8_t *w2_scales, const uint16_t *b2,
                   void *stream);
MOE_API int moe_finalize(moe_ctx_t *ctx, int T, int top_k, const uint16_t *x, uint16_t *y, int32_t *topk_idx_out,
                 float *topk_w_out, void *stream);

/* Workspace buffers readable through moe_copy_workspace. */
enum {
    MOE_WS_XN = 0,       /* fp32 [T, d]   normalised tokens xn (the experts' input) */
    MOE_WS_TOPK_IDX = 2, /* int32 [T, k]                                         */
    MOE_WS_TOPK_W = 3,   /* fp32 [T, k]                                          */
    MOE_WS_COUNTS = 4,   /* int32 [E]     tokens routed to each expert            */
    MOE_WS_OFFSETS = 5,  /* int32 [E+1]   exclusive prefix of counts              */
    MOE_WS_ROW_TOKEN = 6,/* int32 [T*k]   token of each expert-sorted row         */
    MOE_WS_ROW_W = 7,    /* fp32 [T*k]    routing weight of each expert-sorted row */
    MOE_WS_H = 8,        /* u8 [3, T_max*k, Kf] SwiGLU output h of the expert-sorted rows as
                            E4M3 hi, lo and lo2 terms (planes 0, 1, 2): h ~ hi 2^s + lo 2^(s-4)
                            + lo2 2^s with s the block's scale in MOE_WS_HSF; Kf = d_ff rounded
                            up to 128                                                          */
    MOE_WS_OUT_ROWS = 9, /* fp32 [T*k, d] w * (W2 h + b2), expert-sorted rows      */
    MOE_WS_TILES = 10,   /* int32 [E+1]   exclusive prefix of token blocks        */
    MOE_WS_PAIR_ROW = 11,/* int32 [T*k]   expert-sorted row of pair (token, slot) */
    MOE_WS_XPERM = 12,   /* u8 [3, T_max*k, Kd] normalised tokens in expert-sorted order, E4M3
                            hi, lo and lo2 planes as MOE_WS_H; Kd = d_model rounded up to 128 */
    MOE_WS_XSF = 13,     /* u32 [Kd/128, 2, T_max*k] E8M0 scales of MOE_WS_XPERM: word (g, plane,
                            row), byte i = the scale of 32-block 4g+i; plane 0 scales the hi and
                            the lo2 terms, plane 1 the lo term                                 */
    MOE_WS_HSF = 14      /* u32 [Kf/128, 2, T_max*k] E8M0 scales of MOE_WS_H, same layout      */
};

/* Copy `bytes` bytes of workspace buffer `which` (a MOE_WS_* value) into
 * `dst` (host or device memory) on `stream`.  Returns MOE_ERR_ARG when bytes
 * exceeds the buffer. */
MOE_API int moe_copy_workspace(moe_ctx_t *ctx, int which, void *dst, size_t bytes, void *stream);

/* Synchronise `stream` and return the latched device-side error (clearing
 * it): MOE_OK or MOE_ERR_TIMEOUT.  MOE_ERR_CUDA when the synchronisation
 * itself fails. */
MOE_API int moe_sync_status(moe_ctx_t *ctx, void *stream);

/* Limit of every device-side wait on an mbarrier, in nanoseconds (default
 * 2e9).  A wait that runs out sets the latched error, makes the kernel stop
 * issuing work, drain what it has in flight, free its tensor memory and
 * return. */
MOE_API int moe_set_wait_limit_ns(moe_ctx_t *ctx, unsigned long long ns);

/* Self-test of the bounded wait: launches one CTA that waits on an mbarrier
 * nothing will complete.  With a short limit the wait runs out and
 * moe_sync_status then returns MOE_ERR_TIMEOUT; the context stays usable. */
MOE_API int moe_selftest_wait_timeout(moe_ctx_t *ctx, void *stream);

/* Decode an R x K MXFP4 matrix (codes u8 [R, K/2], scales u8 [R, K/32],
 * device pointers) into fp32 out [R, K] on the device (hardware E2M1
 * conversion to fp16 times the block's power of two, relative to a per-row
 * power of two 2^c_r, then multiplied back).  For tests of the format; the
 * grouped GEMMs hand the codes and scales to the tensor core as they are. */
MOE_API int moe_debug_decode(const uint8_t *codes, const uint8_t *scales, int R, int K, float *out, void *stream);

/* The launch plan of one grouped-GEMM stage, computed on the host alone (no
 * device call), as the library makes it for a call: mode 0 (gate/up) or 1
 * (down), T tokens, top_k, the layer shape, P_max workspace rows (>= T*top_k)
 * and num_sms SMs.  Writes out[0..9] = {token rows per work item, hi and lo
 * rows stacked in one MMA (0/1), shared-memory ring stages, per-item scale
 * factors (0/1), grid size, dynamic shared memory bytes, TMEM columns used,
 * full 128-wide K stages, K stages, weight-row blocks per expert}.  Shape
 * limits as moe_init; returns MOE_ERR_ARG for bad arguments or a plan that
 * does not fit.  For tests of the planner. */
MOE_API int moe_debug_plan(int mode, int T, int top_k, int d_model, int d_ff, int n_experts, int P_max, int num_sms,
                           int *out);

/* The whole block (as moe_forward) without any device allocation, for callers
 * that cannot call cudaMalloc: frameworks whose caching allocator owns all
 * device memory, or plugins whose host does not let library code allocate.
 * (The gpt-oss write-ups have no counterpart of this entry point; it is an
 * integration convenience.)
 *
 * Scratch memory comes from one fixed 8 MiB __device__ array inside the
 * library, held on every GPU that loads it until process exit; no context is
 * needed.  Limits: T <= MOE_NOALLOC_MAX_TOKENS and the workspace for the shape
 * (about T*(4d + 4E) + T*k*(7d + 3F) bytes, d and F rounded up to 128, e.g.
 * 7.96 MiB for 64 tokens of the d_model = d_ff = 2880, top-4, 128-expert
 * layer) must fit in the array; larger requests
 * return MOE_ERR_ARG.  Shape limits otherwise as in moe_init.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current: make it outside any stream
 * capture.  All calls share the one array and the array keeps the last call's
 * contents, so calls that overlap on the GPU (other streams, other host
 * threads on the same device) race; serialise them.  Device-side bounded-wait
 * errors are not reported by this entry point (there is no context to latch
 * them in); the return value covers argument and launch errors. */
#define MOE_NOALLOC_MAX_TOKENS 64
MOE_API int moe_forward_noalloc(int T, int d_model, int d_ff, int n_experts, int top_k, float eps,
                                const uint16_t *x, const uint16_t *router_w, const float *router_b,
                                const uint8_t *w13_codes, const uint8_t *w13_scales, const uint16_t *b13,
                                const uint8_t *w2_codes, const uint8_t *w2_scales, const uint16_t *b2,
                                const uint16_t *norm_scale, uint16_t *y, void *stream);

/* A human-readable name of an error code. */
MOE_API const char *moe_strerror(int code);

/* Library version string. */
MOE_API const char *moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
