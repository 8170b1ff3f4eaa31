/*
 * moe.h -- C ABI of the sigmoid-bias top-k mixture-of-experts feed-forward
 * block, B200 (sm_100a) implementation.
 *
 * The layer is the sparse feed-forward half of a pre-norm block as stated in
 * "LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV Caches"
 * (flozi.net, English page):
 *   section "The exact checkpoint": out = x + FFN(RMSNorm(x)), shape-preserving;
 *   section "The router has two different scores": tokens are rows of
 *     X in R^{N x d}; a router matrix W_r in R^{E x d} gives E logits per token;
 *     sigmoid is applied to each logit independently; a stored E-element bias
 *     takes part in the top-k selection but not in the mixture weights, which
 *     are the selected unbiased scores normalised by their sum plus an epsilon
 *     and multiplied by the routed scaling factor (1 for that checkpoint); each
 *     selected expert is a gated SiLU MLP whose gate and up matrices are packed
 *     together;
 *   section "What to verify in a deployment": tokens are grouped by expert and
 *     the weighted expert outputs accumulated.
 * Per token t:  xn = x_t / sqrt(mean(x_t^2) + eps) * gain
 *               s_e = sigmoid(W_r[e] . xn),  c_e = s_e + bias_e
 *               S = top-k of c (slots by descending c, ties to the lower index)
 *               w_j = routed_scale * s_{S_j} / (sum_j s_{S_j} + eps)
 *               out_t = x_t + sum_j w_j * Wd_e (silu(Wg_e xn) * (Wu_e xn)), e = S_j
 *
 * All pointers passed to these functions are DEVICE pointers unless the name
 * says host. Every function returns 0 (MOE_OK) or a negative moe_err code.
 * A context is not thread-safe: one forward at a time per context.
 */
#ifndef SIGMOID_BIAS_TOP_MOE_H
#define SIGMOID_BIAS_TOP_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Storage type of x, out and the expert matrices. The RMSNorm gain, router
 * matrix and expert bias are always fp32 (the router stays unquantised).
 * MOE_FP8_BLOCK is the FP8 checkpoint's scheme ("LFM2.5-24B-A2B: ein 24B-Reasoning-Modell, das pro Wortstück so wenig verbraucht wie ein 2B-Modell",
 * inferencekey.com, section "Für Engineers", paragraph "Quantisierung":
 * weights FP8 static in 128x128 blocks, activations FP8 dynamic per group of
 * 128): x and out are bf16, the
 * expert matrices are e4m3 codes (1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits, no infinities, largest finite 448) with one fp32 scale per
 * 128x128 block, weight = code value * block scale. Inside the forward each
 * token's input to gate/up and its SiLU(gate)*up row are quantised in groups
 * of 128 columns: s = max|v| / 448, code = e4m3(v / s) rounded to nearest
 * even with saturation (s = 0 and zero codes for an all-zero group). */
typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_FP8_BLOCK = 2 } moe_dtype;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,       /* null pointer, bad enum, n_tokens < 0        */
    MOE_ERR_UNSUPPORTED_SHAPE = -2, /* sizes outside the supported ranges below    */
    MOE_ERR_ALIGNMENT = -3,         /* a pointer is not 16-byte aligned            */
    MOE_ERR_TOO_MANY_TOKENS = -4,   /* n_tokens > max_tokens given at create       */
    MOE_ERR_OOM = -5,               /* workspace allocation failed                 */
    MOE_ERR_CUDA = -6,              /* a CUDA runtime call or launch failed        */
    MOE_ERR_DEVICE_TIMEOUT = -7,    /* a bounded device-side wait ran out          */
    MOE_ERR_DEVICE_BOUNDS = -8,     /* a device-side index check failed            */
    MOE_ERR_NO_DEVICE = -9          /* no CUDA device, or not an sm_100 device     */
} moe_err;

/* Layer parameters: BORROWED device pointers, row-major, caller-owned; they
 * must stay valid and unchanged until moe_destroy. 16-byte aligned. */
typedef struct {
    int dtype;                 /* moe_dtype of w_gate_up, w_down, x and out           */
    const float *norm_gain;    /* [d]        RMSNorm gain, multiplied as stored       */
    const float *router_w;     /* [E][d]     router matrix W_r                        */
    const float *expert_bias;  /* [E]        selection-only expert bias               */
    const void  *w_gate_up;    /* [E][2I][d] rows 0..I-1 gate, rows I..2I-1 up        */
    const void  *w_down;       /* [E][d][I]  down projection                          */
    float        routed_scale; /* multiplies the normalised weights (1 in the page)   */
    /* MOE_FP8_BLOCK only (ignored otherwise): fp32 scales of the 128x128 blocks,
     * block (rb, cb) covering rows rb*128.. and columns cb*128.. of a matrix. */
    const float *w_gate_up_scale; /* [E][2I/128][d/128]                               */
    const float *w_down_scale;    /* [E][d/128][I/128]                                */
} moe_weights;

typedef struct moe_ctx moe_ctx;

/* Validates the shapes, allocates the workspace for up to max_tokens tokens on
 * the current CUDA device and builds the TMA descriptors of the weights.
 * d = hidden width, n_experts = E, d_ff = expert intermediate width I,
 * top_k = k, eps serves both the RMSNorm and the weight normalisation.
 * Supported: 1 <= top_k <= min(n_experts, 8), n_experts <= 256,
 *   MOE_F32: d % 4 == 0, any d_ff >= 1;
 *   MOE_BF16: d % 64 == 0, d_ff % 64 == 0 (tensor-core tiles);
 *   MOE_FP8_BLOCK: d % 128 == 0, d_ff % 128 == 0 (whole scale blocks).
 * On success *out receives the context; on failure *out is set to NULL and
 * nothing stays allocated. Synchronous. The workspace holds the grouped rows,
 * the expert intermediates and outputs of max_tokens * top_k assignments;
 * MOE_FP8_BLOCK layers add an fp32 [max_tokens * top_k][d_ff] buffer for the
 * CTA-pair path (4 bytes per intermediate value; none with MOE_FP8_PAIR=0).
 * The kernels are chosen per forward from the batch size; two environment
 * variables, read here, force the choice between kernels that compute the
 * same result (for testing and tuning): MOE_TC_PAIR=0 (bf16 expert GEMMs
 * on single CTAs instead of the default CTA pairs), MOE_ROUTE_TC=0|1 (SIMT or tensor-core
 * router for bf16 inputs) and MOE_FP8_PAIR=0 (MOE_FP8_BLOCK batches of every
 * size on the persistent FP8 kernel instead of the CTA-pair GEMMs). */
int moe_create(int d, int n_experts, int d_ff, int top_k, float eps,
               const moe_weights *w, int max_tokens, moe_ctx **out);

/* out[N][d] = x + MoE(RMSNorm(x)) for x[N][d] (device, dtype of the weights;
 * bf16 for MOE_FP8_BLOCK).
 * out == x (in place) is allowed; other overlap is not. Asynchronous on
 * `stream` (a cudaStream_t, NULL = legacy default stream): no host sync, no
 * allocation, a fixed sequence of kernel launches, so it can be captured in a
 * CUDA graph. n_tokens == 0 is a no-op. Device-side failures are reported by
 * moe_status. */
int moe_forward(moe_ctx *h, const void *x, void *out, int n_tokens, void *stream);

/* Same as moe_forward for HOST buffers: copies x_host into device staging,
 * runs the forward and brings the result into out_host, then waits for the
 * stream. With pinned out_host (device-mapped) the last kernel stores the
 * rows into it directly; other memory gets a copy from device staging.
 * Pinned x_host gives an asynchronous copy; pageable works. */
int moe_forward_host(moe_ctx *h, const void *x_host, void *out_host, int n_tokens,
                     void *stream);

/* Frees the workspace (not the weights). Waits for the device. NULL is a no-op. */
int moe_destroy(moe_ctx *h);

/* Reads and clears the device status word after waiting for the device:
 * MOE_OK, MOE_ERR_DEVICE_TIMEOUT or MOE_ERR_DEVICE_BOUNDS. */
int moe_status(moe_ctx *h);

/* Device-to-device copy of the last forward's routing into caller buffers
 * (any may be NULL): idx[N][k] int32 expert per slot, w[N][k] fp32 weights,
 * perm[N*k] int32 assignment ids t*k+j grouped by expert (ascending expert,
 * then ascending token), offsets[E+1] int32 exclusive prefix of the per-expert
 * counts. Asynchronous on stream. */
int moe_debug_routing(moe_ctx *h, int32_t *idx, float *w, int32_t *perm,
                      int32_t *offsets, void *stream);

/* MOE_FP8_BLOCK layers: device-to-device copy of the last forward's grouped,
 * quantised expert inputs into caller buffers (either may be NULL):
 * codes[N*k][d] e4m3 (row r is the normalised row of assignment perm[r]) and
 * scales[N*k][d/128] fp32 group scales. MOE_ERR_INVALID_ARG for other dtypes.
 * Asynchronous on stream. */
int moe_debug_fp8_rows(moe_ctx *h, uint8_t *codes, float *scales, void *stream);

/* Per-kernel timing. moe_profile(h, 1) starts (or restarts) profiling: each
 * forward then records CUDA events between its launches on its stream (a ring
 * of 1024 forwards; older entries are folded into running sums as it wraps).
 * moe_kernel_times waits for the recorded forwards and writes up to n MEAN
 * durations in milliseconds per kernel (launch order) over every forward since
 * profiling started, returning the number of kernels per forward, 0 if none
 * was recorded, or a negative moe_err. moe_profile(h, 0) stops recording. */
int moe_profile(moe_ctx *h, int enable);
int moe_kernel_times(moe_ctx *h, float *ms, int n);
/* Name of kernel i of the last forward's launch sequence (static string), or
 * NULL: route, dispatch, gate_up, down, combine; or route, dispatch, experts,
 * combine when the batch was small enough for the fused expert kernel (for
 * MOE_FP8_BLOCK layers: the persistent FP8 kernel); or route, dispatch,
 * gate_up, quantize, down, combine for MOE_FP8_BLOCK batches above that size
 * (the CTA-pair FP8 GEMMs, SiLU(gate)*up quantised by its own kernel). */
const char *moe_kernel_name(moe_ctx *h, int i);

/* Number of kernel launches one forward makes for n_tokens tokens. */
int moe_launches_per_forward(moe_ctx *h, int n_tokens);

/* Test hook of the bounded device waits: launches one kernel that waits on a
 * barrier that nothing signals, with a limit of timeout_us microseconds, and
 * records MOE_ERR_DEVICE_TIMEOUT in the status word. The context stays usable. */
int moe_selftest_timeout(moe_ctx *h, int timeout_us, void *stream);

/* Routing of a batch with no device allocation: for callers that cannot
 * allocate device memory where they route (while a stream is being captured
 * into a CUDA graph, in serving loops that forbid allocator calls because
 * they may synchronise the device, or under a memory planner that owns all
 * device memory). The page describes no such entry point; it is an interface
 * of this library only. Computes, for x[n_tokens][d] (dtype MOE_F32 or
 * MOE_BF16: the storage type of x, so MOE_BF16 for the bf16 x of an
 * MOE_FP8_BLOCK layer, whose router is unquantised; any other dtype gives
 * MOE_ERR_INVALID_ARG) and the fp32 norm_gain[d], router_w[E][d], expert_bias[E], the
 * same idx[n_tokens][top_k] (int32, slot order) and w[n_tokens][top_k] (fp32)
 * as moe_forward's routing (see moe_debug_routing). All pointers are device
 * pointers owned by the caller; x, norm_gain and router_w 16-byte aligned.
 * Limits of the fixed scratch: n_tokens <= 4096 (else MOE_ERR_TOO_MANY_TOKENS),
 * n_experts <= 64 and d <= 2048 (else MOE_ERR_UNSUPPORTED_SHAPE); shapes as
 * moe_create takes them: d % 4 == 0 for MOE_F32 x, d % 64 == 0 for MOE_BF16 x,
 * 1 <= top_k <= min(n_experts, 8) (else MOE_ERR_UNSUPPORTED_SHAPE). The
 * scratch is one array compiled into the library, about 1.1 MB on every GPU
 * that loads it, held until the process exits; a device's first call looks
 * its address up (make that first call before any stream capture). Calls
 * share the array: calls that overlap on the GPU race, calls ordered on one
 * stream do not. Asynchronous on stream. Device-side failure: there is no
 * context and so no moe_status here; if the router's bounded wait for its
 * input copies runs out (1 s), every idx of the call is set to -1 and every
 * w to NaN. */
int moe_route_noalloc(const void *x, int dtype, const float *norm_gain, const float *router_w,
                      const float *expert_bias, int n_tokens, int d, int n_experts, int top_k,
                      float eps, float routed_scale, int32_t *idx, float *w, void *stream);

/* ---------------------------------------------------------------------------
 * Expert parallelism. The page notes that once the experts are spread over
 * devices, dispatch, token regrouping and uneven expert loads decide the cost,
 * and names expert parallelism as how the layer is deployed at scale
 * ("LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV Caches",
 * section "The router has two different scores"); it gives no implementation.
 * Here each rank (one process per GPU) routes and dispatches ITS OWN tokens
 * over all E experts but holds the weights of one contiguous block of
 * experts, [expert_first, expert_first + n_local). A forward is
 *   moe_ep_dispatch -> exchange rows -> moe_ep_experts -> exchange outputs
 *   -> moe_ep_combine,
 * with both exchanges done by the caller (NCCL grouped send/recv or any
 * transport) between the buffers of moe_ep_buffers:
 *   send_rows [max_tokens*k][d]: after moe_ep_dispatch, the normalised rows
 *     grouped by expert (ascending), token order within an expert; the rows
 *     of expert e are rows offsets[e] .. offsets[e+1]-1, offsets being the
 *     exclusive prefix of the counts moe_ep_dispatch returns;
 *   recv_rows [max_recv_rows][d]: the caller places here the rows of the
 *     local experts from every rank, grouped by local expert (ascending),
 *     any fixed order within an expert (source rank order, say);
 *   send_y [max_recv_rows][d]: after moe_ep_experts, the expert output of
 *     each received row, in the same position as the row;
 *   recv_y [max_tokens*k][d]: the caller places here each of its own rows'
 *     outputs, in the position of the row in send_rows.
 * Storage type of rows and outputs = the layer dtype. MOE_F32 and MOE_BF16
 * layers only (MOE_ERR_INVALID_ARG otherwise). Buffers are context-owned
 * device memory, valid until moe_ep_destroy. No kernel of this library reads
 * another GPU's memory. */
typedef struct moe_ep_ctx moe_ep_ctx;

/* As moe_create, except: w->w_gate_up [n_local][2I][d] and w->w_down
 * [n_local][d][I] hold the local experts only (router_w [E][d] and
 * expert_bias [E] stay whole); max_recv_rows bounds the rows one rank may
 * receive (W * max_tokens * k covers any routing). */
int moe_ep_create(int d, int n_experts, int d_ff, int top_k, float eps, const moe_weights *w,
                  int max_tokens, int expert_first, int n_local, int max_recv_rows,
                  moe_ep_ctx **out);

/* Route and dispatch x[n_tokens][d] (device) into send_rows; writes the
 * per-expert row counts [E] to counts_host and waits for the stream (the
 * exchange sizes come from them). */
int moe_ep_dispatch(moe_ep_ctx *h, const void *x, int n_tokens, int32_t *counts_host,
                    void *stream);

/* Device addresses of the four exchange buffers (any may be NULL). */
int moe_ep_buffers(moe_ep_ctx *h, void **send_rows, void **recv_rows, void **send_y,
                   void **recv_y);

/* Both expert contractions of the local experts over the first
 * sum(local_counts_host) rows of recv_rows, local_counts_host[n_local] rows
 * per local expert in order; outputs into send_y. More rows than
 * max_recv_rows give MOE_ERR_TOO_MANY_TOKENS. Asynchronous on stream. */
int moe_ep_experts(moe_ep_ctx *h, const int32_t *local_counts_host, void *stream);

/* out[N][d] = x + sum_j w_j y_j for the last dispatched batch (N tokens),
 * reading recv_y. x is the batch given to moe_ep_dispatch; out == x is
 * allowed. Asynchronous on stream. */
int moe_ep_combine(moe_ep_ctx *h, const void *x, void *out, void *stream);

/* As moe_debug_routing, for the last moe_ep_dispatch (offsets over all E). */
int moe_ep_debug_routing(moe_ep_ctx *h, int32_t *idx, float *w, int32_t *perm,
                         int32_t *offsets, void *stream);

/* As moe_status and moe_destroy. */
int moe_ep_status(moe_ep_ctx *h);
int moe_ep_destroy(moe_ep_ctx *h);

/* Test hook of the FP8 quantisers' division: for n operand pairs (device
 * arrays), q[i] = a[i] / b[i] as the quantisers form it (a reciprocal and
 * one correction step, in paired fp32 operations where b[i] is in the step's
 * range) and q_ref[i] = the IEEE quotient; the two are equal
 * bit for bit wherever the quotient is a normal float. Asynchronous on
 * stream. */
int moe_selftest_fp8_divide(const float *a, const float *b, float *q, float *q_ref, int n,
                            void *stream);

/* Static description of a moe_err code. */
const char *moe_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* SIGMOID_BIAS_TOP_MOE_H */
