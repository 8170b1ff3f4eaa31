/*
 * block.h -- C ABI of the neighbouring steps of the LFM2.5-24B-A2B block on
 * B200 (sm_100a): the dense feed-forward block and the short-convolution
 * (mixer) block. Same library (libmoe.so), conventions and error codes as
 * moe.h.
 *
 * "LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV Caches"
 * (flozi.net, English page):
 *   section "The exact checkpoint": the first two layers are dense and
 *     convolutional; a block preserves [B, T, 2048], normalises (RMSNorm)
 *     before its mixer and before its feed-forward network, and adds a
 *     residual around each;
 *   section "A short convolution is a local mixer, not an embedding lookup":
 *     the normalised row is projected into three width-2048 streams (B, C and
 *     x of the implementation; g, u, v on the page), a = g * v, a depthwise
 *     causal convolution of width three (coefficients indexed by lag), times
 *     u, and a projection back to width 2048; the gates are direct linear
 *     projections (no sigmoid) and the depthwise kernel mixes no channels.
 *
 * Dense block:  out = x + W_down( silu(W_gate xn) * (W_up xn) ),
 *               xn = x / sqrt(mean(x^2) + eps) * gain.
 * Conv block:   [g; u; v] = W_in xn,  a_t = g_t * v_t,
 *               c_t = k[0] a_t + k[1] a_{t-1} + k[2] a_{t-2} (per channel),
 *               out_t = x_t + W_out (u_t * c_t).
 * Readings where the page is silent: no biases; the packed W_in holds g
 * rows, then u rows, then v rows (the implementation's B, C, x order); the
 * taps are stored [d][3] by lag. The conv block runs along sequences: x is
 * [n_seqs][seq_len][d], and each sequence's a before its first position is
 * the caller's state (or zero).
 *
 * bf16 layers (x, out, matrices); the gain, the taps and the state are fp32.
 * All pointers are DEVICE pointers, 16-byte aligned; weights are borrowed
 * until destroy. Forwards are asynchronous on `stream`, allocate nothing and
 * report device-side failures through moe_block_status.
 */
#ifndef SIGMOID_BIAS_TOP_BLOCK_H
#define SIGMOID_BIAS_TOP_BLOCK_H

#include <stdint.h>

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_block_ctx moe_block_ctx;

typedef struct {
    int dtype;               /* MOE_BF16                                          */
    const float *norm_gain;  /* [d]                                               */
    const void *w_gate_up;   /* [2I][d]: rows 0..I-1 gate, rows I..2I-1 up         */
    const void *w_down;      /* [d][I]                                            */
} moe_dense_weights;

typedef struct {
    int dtype;               /* MOE_BF16                                          */
    const float *norm_gain;  /* [d]                                               */
    const void *w_in;        /* [3d][d]: rows of g, then u, then v                 */
    const float *conv;       /* [d][3]: conv[c][l] multiplies a_{t-l} of channel c */
    const void *w_out;       /* [d][d]                                            */
} moe_conv_weights;

/* Dense block of width d and intermediate width d_ff for up to max_tokens
 * tokens. d % 64 == 0, d_ff % 64 == 0; MOE_ERR_INVALID_ARG for other dtypes. */
int moe_dense_create(int d, int d_ff, float eps, const moe_dense_weights *w, int max_tokens,
                     moe_block_ctx **out);

/* out[N][d] = dense block of x[N][d]; out == x (in place) is allowed. */
int moe_dense_forward(moe_block_ctx *h, const void *x, void *out, int n_tokens, void *stream);

/* Short-convolution block of width d (d % 64 == 0) for up to max_tokens
 * positions per forward (n_seqs * seq_len). */
int moe_conv_create(int d, float eps, const moe_conv_weights *w, int max_tokens,
                    moe_block_ctx **out);

/* out[B][T][d] = conv block of x[B][T][d], B = n_seqs, T = seq_len.
 * state_in [B][2][d] fp32 (or NULL for zeros): each sequence's a at
 * positions -2 and -1. state_out [B][2][d] fp32 (or NULL): its a at positions
 * T-2 and T-1 (taken from state_in where T < 2), so a following call with
 * state_in = this state_out continues the sequences (decode: T = 1).
 * state_out may equal state_in. out == x is allowed. */
int moe_conv_forward(moe_block_ctx *h, const void *x, void *out, int n_seqs, int seq_len,
                     const float *state_in, float *state_out, void *stream);

/* As moe_status and moe_destroy. */
int moe_block_status(moe_block_ctx *h);
int moe_block_destroy(moe_block_ctx *h);

/* Per-kernel timing, as moe_profile / moe_kernel_times / moe_kernel_name:
 * CUDA events between the launches of every forward while enabled (the
 * events separate the launches); mean milliseconds per launch; names of the
 * last forward's launches: norm, gate_up, down_residual (dense) or norm,
 * in_gv, in_u_conv, out_residual, state (conv). Small batches, whose GEMMs
 * would leave most of the GPU idle, split K: a GEMM then writes fp32 partial
 * sums ("gate_up_split", "down_split", "in_gv_split", "in_u_split",
 * "out_split") and a second launch adds them and finishes the step
 * ("gate_up_reduce", "down_residual_reduce", "in_gv_reduce",
 * "in_u_conv_reduce", "out_residual_reduce"). The environment variable
 * MOE_BLOCK_SPLIT=0, read at create, keeps every GEMM unsplit (the same
 * result; for testing both paths). */
int moe_block_profile(moe_block_ctx *h, int enable);
int moe_block_kernel_times(moe_block_ctx *h, float *ms, int n);
const char *moe_block_kernel_name(moe_block_ctx *h, int i);

#ifdef __cplusplus
}
#endif
#endif /* SIGMOID_BIAS_TOP_BLOCK_H */
