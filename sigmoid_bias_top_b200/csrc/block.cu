// block.cu -- the neighbouring steps of the block: the dense feed-forward
// block and the short-convolution (mixer) block, declared in include/block.h.
//
// "LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV Caches"
// (flozi.net, English page):
//   section "The exact checkpoint": the first two layers are dense and
//     convolutional; a block normalises before its mixer and before its
//     feed-forward network, adding a residual around each;
//   section "A short convolution is a local mixer, not an embedding lookup":
//     the normalised row is projected into three width-d streams g, u, v
//     (B, C and x of the implementation), a = g * v, a depthwise causal
//     convolution of width three (coefficients by lag), times u, and a
//     projection back to width d; no sigmoid on the gates.
//
// Both blocks run on the CTA-pair tcgen05 GEMM of the experts (gemm_tc2.cu)
// with all tokens as one group and its epilogue mode picking the step:
//   dense: norm -> [SiLU(gate) * up] -> [down + residual]             3 launches
//   conv:  norm -> [g * v -> a] -> [u * conv3(a) -> y] -> [W_out y + residual]
//          (+ the state copy when the caller asks for it)            4 (+1)
// The width-3 convolution needs no launch of its own: the u projection's
// epilogue holds u for its tokens and channels and reads the three a values
// it needs (written by the previous launch) from L2.
#include <stdlib.h>
#include <string.h>

#include <vector>

#include "../../include/block.h"
#include "moe_internal.cuh"

using namespace moe;

namespace {

constexpr int kNormThreads = 256;
constexpr int kMaxLaunches = 8;
constexpr size_t kPartialBytes = size_t(16) << 20;  // fp32 partial sums of split-K GEMMs

// xn[r] = bf16(x[r] * rinv * gain), rinv = 1 / sqrt(mean(x[r]^2) + eps), one
// warp per row (bf16 rows, d % 8 == 0). Block 0 also writes the one-group
// tile plan of the GEMMs: loc = {0, N, 0, ceil(N / 256)}.
template <int kNormU>
__global__ void __launch_bounds__(kNormThreads)
    rmsnorm_rows_kernel(const __nv_bfloat16 *x, const float *gain, __nv_bfloat16 *xn,
                        int32_t *loc, int N, int d, float eps) {
    pdl_trigger();
    pdl_wait();
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        loc[0] = 0;
        loc[1] = N;
        loc[2] = 0;
        loc[3] = (N + kTcPairTileM - 1) / kTcPairTileM;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * (kNormThreads / 32) + warp;
    if (r >= N) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(r) * d);
    uint4 *dst = reinterpret_cast<uint4 *>(xn + static_cast<size_t>(r) * d);
    const int nv = d / 8;
    // kNormU 16-byte vectors per lane are loaded before any is used (one
    // memory round trip per 32 * kNormU vectors of the row instead of one per
    // 32); each lane still adds its values in ascending column order
    float ss = 0.f;
    for (int base = 0; base < nv; base += 32 * kNormU) {
        uint4 q[kNormU];
#pragma unroll
        for (int u = 0; u < kNormU; ++u) {
            const int v = base + u * 32 + lane;
            q[u] = v < nv ? src[v] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kNormU; ++u) {
            const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float a = bf16_to_f32(w[h] & 0xFFFFu), b = bf16_to_f32(w[h] >> 16);
                ss += a * a;
                ss += b * b;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rinv = 1.0f / sqrtf(ss / static_cast<float>(d) + eps);
    for (int base = 0; base < nv; base += 32 * kNormU) {
        uint4 q[kNormU];
        float4 g[kNormU][2];
#pragma unroll
        for (int u = 0; u < kNormU; ++u) {
            const int v = base + u * 32 + lane;
            if (v < nv) {
                q[u] = src[v];
                g[u][0] = *reinterpret_cast<const float4 *>(gain + v * 8);
                g[u][1] = *reinterpret_cast<const float4 *>(gain + v * 8 + 4);
            }
        }
#pragma unroll
        for (int u = 0; u < kNormU; ++u) {
            const int v = base + u * 32 + lane;
            if (v >= nv) continue;
            const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
            const float gg[8] = {g[u][0].x, g[u][0].y, g[u][0].z, g[u][0].w,
                                 g[u][1].x, g[u][1].y, g[u][1].z, g[u][1].w};
            uint32_t o[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(bf16_to_f32(w[h] & 0xFFFFu) * rinv * gg[2 * h],
                                                          bf16_to_f32(w[h] >> 16) * rinv * gg[2 * h + 1]);
                o[h] = *reinterpret_cast<uint32_t *>(&b2);
            }
            dst[v] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// state_out[b][j] = a of position T - 2 + j of sequence b (from the carried
// state_in, or zero, when that position lies before the sequence). One thread
// reads both sources of a (b, channel) before writing, so state_out may be
// state_in.
__global__ void conv_state_kernel(const __nv_bfloat16 *a, const float *state_in, float *state_out,
                                  int B, int T, int d) {
    const size_t n = static_cast<size_t>(B) * d;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const int b = static_cast<int>(i / d), c = static_cast<int>(i % d);
        float v[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int pos = T - 2 + j;
            if (pos >= 0)
                v[j] = __bfloat162float(a[(static_cast<size_t>(b) * T + pos) * d + c]);
            else
                v[j] = state_in ? state_in[(static_cast<size_t>(b) * 2 + pos + 2) * d + c] : 0.f;
        }
        state_out[(static_cast<size_t>(b) * 2) * d + c] = v[0];
        state_out[(static_cast<size_t>(b) * 2 + 1) * d + c] = v[1];
    }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Split-K GEMMs of small batches leave fp32 partial sums part[S][N][width];
// this kernel adds the S slices in slice order (deterministic) and finishes
// the step, for outputs [N][W]:
//   kRedSiluMul: width 2W (gate, then up): act = bf16(silu(sum g) * sum u)
//   kRedMul:     width 2W (g, then v):     a   = bf16(sum g * sum v)
//   kRedConv:    width W (u): y = bf16(sum u * (k0 a_t + k1 a_{t-1} + k2 a_{t-2}))
//                along each sequence of T rows, the carried state before it
//   kRedResid:   width W: out = bf16(x + sum)
// SiLU and the convolution are formed as in the pair GEMM's epilogues.
enum { kRedSiluMul = 0, kRedMul = 1, kRedConv = 2, kRedResid = 3 };

template <int KIND>
__global__ void __launch_bounds__(256)
    block_reduce_kernel(const float *part, int S, int N, int W, const __nv_bfloat16 *x,
                        __nv_bfloat16 *dst, const float *conv, const __nv_bfloat16 *a,
                        const float *state_in, int T) {
    pdl_trigger();
    pdl_wait();
    const bool paired = KIND == kRedSiluMul || KIND == kRedMul;
    const size_t width = paired ? 2 * static_cast<size_t>(W) : static_cast<size_t>(W);
    const size_t n = static_cast<size_t>(N) * W;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const size_t r = i / W, c = i % W;
        float g = 0.f, u = 0.f;
        for (int sl = 0; sl < S; ++sl) {
            const float *row = part + (static_cast<size_t>(sl) * N + r) * width;
            g += row[c];
            if (paired) u += row[W + c];
        }
        float v;
        if (KIND == kRedSiluMul) {
            v = __fdividef(g, 1.0f + __expf(-g)) * u;
        } else if (KIND == kRedMul) {
            v = g * u;
        } else if (KIND == kRedConv) {
            const int b = static_cast<int>(r / T), t = static_cast<int>(r % T);
            const float a0 = __bfloat162float(a[r * W + c]);
            const float a1 = t >= 1 ? __bfloat162float(a[(r - 1) * W + c])
                                    : state_in ? state_in[(static_cast<size_t>(b) * 2 + 1) * W + c] : 0.f;
            const float a2 = t >= 2 ? __bfloat162float(a[(r - 2) * W + c])
                             : state_in ? state_in[(static_cast<size_t>(b) * 2 + t) * W + c] : 0.f;
            v = g * fmaf(conv[c * 3 + 2], a2, fmaf(conv[c * 3 + 1], a1, conv[c * 3] * a0));
        } else {
            v = __bfloat162float(x[i]) + g;
        }
        dst[i] = __float2bfloat16_rn(v);
    }
}

}  // namespace

struct moe_block_ctx {
    int kind;  // 0 dense, 1 conv
    int d, I, max_tokens, device, n_sm;
    float eps;
    const float *gain;
    const void *w1, *w2;   // dense: w_gate_up, w_down; conv: w_in, w_out
    const float *conv;
    void *ws;
    __nv_bfloat16 *xn, *mid, *y;  // xn [cap][d]; dense: act [cap][I]; conv: a [cap][d], y [cap][d]
    int32_t *loc;
    int *status;
    CUtensorMap m_w1, m_w2, m_w3;  // dense: gate/up 4-D, down; conv: g/v 4-D, u rows, w_out
    CUtensorMap m_xn, m_mid;       // token rows: xn, and act (dense) or y (conv)
    float *partial;               // split-K partial sums (kPartialBytes)
    bool split_ok;                // MOE_BLOCK_SPLIT=0 at create keeps every GEMM unsplit
    // the launch sequence of the last forward (it depends on the batch size)
    const char *names[kMaxLaunches + 4];
    int n_names;
    // profiling: events between the launches of every forward since enabled
    bool profile;
    int n_launch;
    std::vector<cudaEvent_t> ev;
    size_t ev_used;
};


static void block_free(moe_block_ctx *h) {
    if (!h) return;
    for (cudaEvent_t e : h->ev) cudaEventDestroy(e);
    if (h->ws) cudaFree(h->ws);
    delete h;
}

static int block_alloc(moe_block_ctx *h, const size_t *sizes, int n, void **ptrs) {
    const char *e = getenv("MOE_BLOCK_SPLIT");  // "0": no split-K (both paths compute the same)
    h->split_ok = !(e && e[0] == '0');
    size_t total = 0, off[8];
    for (int i = 0; i < n; ++i) {
        off[i] = total;
        total += (sizes[i] + 255) & ~static_cast<size_t>(255);
    }
    if (cudaMalloc(&h->ws, total) != cudaSuccess) {
        cudaGetLastError();
        h->ws = nullptr;
        return MOE_ERR_OOM;
    }
    if (cudaMemset(h->ws, 0, total) != cudaSuccess) return MOE_ERR_CUDA;
    for (int i = 0; i < n; ++i) ptrs[i] = static_cast<uint8_t *>(h->ws) + off[i];
    return MOE_OK;
}

static int device_check(int *dev, int *n_sm) {
    if (cudaGetDevice(dev) != cudaSuccess) return MOE_ERR_NO_DEVICE;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, *dev) != cudaSuccess) return MOE_ERR_NO_DEVICE;
    if (prop.major != 10) return MOE_ERR_NO_DEVICE;
    *n_sm = prop.multiProcessorCount;
    return MOE_OK;
}

extern "C" int moe_dense_create(int d, int d_ff, float eps, const moe_dense_weights *w,
                                int max_tokens, moe_block_ctx **out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!w || w->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (d <= 0 || d_ff <= 0 || max_tokens <= 0 || d % 64 != 0 || d_ff % 64 != 0 || d > 32768 ||
        static_cast<long long>(2) * d_ff >= (1LL << 30) || max_tokens >= (1 << 30))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!w->norm_gain || !w->w_gate_up || !w->w_down) return MOE_ERR_INVALID_ARG;
    if (!(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w->norm_gain) || !aligned16(w->w_gate_up) || !aligned16(w->w_down))
        return MOE_ERR_ALIGNMENT;
    int dev, n_sm, rc;
    if ((rc = device_check(&dev, &n_sm)) != MOE_OK) return rc;
    moe_block_ctx *h = new (std::nothrow) moe_block_ctx();
    if (!h) return MOE_ERR_OOM;
    h->kind = 0; h->d = d; h->I = d_ff; h->max_tokens = max_tokens; h->device = dev;
    h->n_sm = n_sm; h->eps = eps; h->gain = w->norm_gain; h->w1 = w->w_gate_up;
    h->w2 = w->w_down; h->n_launch = 3;
    const size_t C = max_tokens;
    const size_t sizes[] = {C * d * 2, C * d_ff * 2, 4 * 4, 256, kPartialBytes};
    void *p[5];
    if ((rc = block_alloc(h, sizes, 5, p)) != MOE_OK) { block_free(h); return rc; }
    h->partial = static_cast<float *>(p[4]);
    h->xn = static_cast<__nv_bfloat16 *>(p[0]);
    h->mid = static_cast<__nv_bfloat16 *>(p[1]);
    h->loc = static_cast<int32_t *>(p[2]);
    h->status = static_cast<int *>(p[3]);
    if ((rc = tc_encode_pair_4d(&h->m_w1, w->w_gate_up, 2 * static_cast<uint64_t>(d_ff), d,
                                d_ff)) != MOE_OK ||
        (rc = tc_encode_2d(&h->m_w2, w->w_down, d, d_ff, 128)) != MOE_OK ||
        (rc = tc_encode_2d(&h->m_xn, h->xn, C, d, 128)) != MOE_OK ||
        (rc = tc_encode_2d(&h->m_mid, h->mid, C, d_ff, 128)) != MOE_OK) {
        block_free(h);
        return rc;
    }
    *out = h;
    return MOE_OK;
}

extern "C" int moe_conv_create(int d, float eps, const moe_conv_weights *w, int max_tokens,
                               moe_block_ctx **out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!w || w->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (d <= 0 || max_tokens <= 0 || d % 64 != 0 || d > 32768 || max_tokens >= (1 << 30))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!w->norm_gain || !w->w_in || !w->conv || !w->w_out) return MOE_ERR_INVALID_ARG;
    if (!(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w->norm_gain) || !aligned16(w->w_in) || !aligned16(w->w_out))
        return MOE_ERR_ALIGNMENT;
    int dev, n_sm, rc;
    if ((rc = device_check(&dev, &n_sm)) != MOE_OK) return rc;
    moe_block_ctx *h = new (std::nothrow) moe_block_ctx();
    if (!h) return MOE_ERR_OOM;
    h->kind = 1; h->d = d; h->I = d; h->max_tokens = max_tokens; h->device = dev;
    h->n_sm = n_sm; h->eps = eps; h->gain = w->norm_gain; h->w1 = w->w_in; h->w2 = w->w_out;
    h->conv = w->conv; h->n_launch = 4;
    const size_t C = max_tokens;
    const size_t sizes[] = {C * d * 2, C * d * 2, C * d * 2, 4 * 4, 256, kPartialBytes};
    void *p[6];
    if ((rc = block_alloc(h, sizes, 6, p)) != MOE_OK) { block_free(h); return rc; }
    h->partial = static_cast<float *>(p[5]);
    h->xn = static_cast<__nv_bfloat16 *>(p[0]);
    h->mid = static_cast<__nv_bfloat16 *>(p[1]);
    h->y = static_cast<__nv_bfloat16 *>(p[2]);
    h->loc = static_cast<int32_t *>(p[3]);
    h->status = static_cast<int *>(p[4]);
    const __nv_bfloat16 *w_in = static_cast<const __nv_bfloat16 *>(w->w_in);
    if ((rc = tc_encode_pair_4d(&h->m_w1, w_in, 3 * static_cast<uint64_t>(d), d,
                                2 * static_cast<uint64_t>(d))) != MOE_OK ||
        (rc = tc_encode_2d(&h->m_w2, w_in + static_cast<size_t>(d) * d, d, d, 128)) != MOE_OK ||
        (rc = tc_encode_2d(&h->m_w3, w->w_out, d, d, 128)) != MOE_OK ||
        (rc = tc_encode_2d(&h->m_xn, h->xn, C, d, 128)) != MOE_OK ||
        (rc = tc_encode_2d(&h->m_mid, h->y, C, d, 128)) != MOE_OK) {
        block_free(h);
        return rc;
    }
    *out = h;
    return MOE_OK;
}

static int call_check(moe_block_ctx *h, int n_tokens) {
    if (!h || n_tokens < 0) return MOE_ERR_INVALID_ARG;
    if (n_tokens > h->max_tokens) return MOE_ERR_TOO_MANY_TOKENS;
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// The profiling events of the next forward (n_launch + 1 of them), or null.
static cudaEvent_t *next_events(moe_block_ctx *h) {
    if (!h->profile) return nullptr;
    const size_t need = h->ev_used + kMaxLaunches + 1;
    while (h->ev.size() < need) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
        h->ev.push_back(e);
    }
    cudaEvent_t *p = &h->ev[h->ev_used];
    h->ev_used = need;
    return p;
}

// Few rows: each warp keeps a whole 2048-wide row in flight (latency-bound:
// 7.3 -> 5 us for 32 rows); many rows: one vector per lane at a time, which
// keeps the occupancy that hides the latency there (8 in flight cost 13%).
static int norm_launch(moe_block_ctx *h, const void *x, int N, cudaStream_t s) {
    const int blocks = (N + kNormThreads / 32 - 1) / (kNormThreads / 32);
    auto kern = N <= 512 ? rmsnorm_rows_kernel<8> : rmsnorm_rows_kernel<1>;
    return launch_k(kern, dim3(blocks), dim3(kNormThreads), 0, s,
                    static_cast<const __nv_bfloat16 *>(x), h->gain, h->xn, h->loc, N, h->d,
                    h->eps);
}

// Parameters of one all-token GEMM. Paired-row modes take I as the features
// and d as K; plain modes take d as the outputs and I as K.
static GroupedParams group_params(moe_block_ctx *h, bool paired, int n_out, int k_dim) {
    GroupedParams gp = {};
    gp.offsets = h->loc;
    gp.mt_start = h->loc + 2;
    gp.status = h->status;
    gp.E = 1;
    gp.k = 1;
    gp.rows_cap = h->max_tokens;
    gp.I = paired ? n_out : k_dim;
    gp.d = paired ? k_dim : n_out;
    return gp;
}

// K slices for one all-token pair GEMM: split while its items (token tiles x
// weight tiles) leave CTA pairs idle, aiming at two items per pair, within
// the partial buffer, every slice non-empty. 1 = no split.
static int pick_split(const moe_block_ctx *h, int N, int items, int K, size_t width) {
    const int pairs = h->n_sm / 2;
    if (!h->split_ok || items >= pairs) return 1;
    const int nk = (K + kTcPairBK - 1) / kTcPairBK;
    int want = (2 * pairs + items - 1) / items;
    const size_t cap = kPartialBytes / (static_cast<size_t>(N) * width * 4);
    if (static_cast<size_t>(want) > cap) want = static_cast<int>(cap);
    if (want > nk) want = nk;
    if (want <= 1) return 1;
    const int nkc = (nk + want - 1) / want;
    return (nk + nkc - 1) / nkc;
}

template <int KIND>
static int reduce_launch(moe_block_ctx *h, int S, int N, int W, const void *x, void *dst,
                         const void *a, const float *state_in, int T, cudaStream_t s) {
    const size_t n = static_cast<size_t>(N) * W;
    int blocks = static_cast<int>((n + 255) / 256);
    if (blocks > 8 * h->n_sm) blocks = 8 * h->n_sm;
    return launch_k(block_reduce_kernel<KIND>, dim3(blocks), dim3(256), 0, s,
                    static_cast<const float *>(h->partial), S, N, W,
                    static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(dst),
                    static_cast<const float *>(h->conv), static_cast<const __nv_bfloat16 *>(a),
                    state_in, T);
}

#define BLOCK_MARK(name)                                                            \
    do {                                                                            \
        if (ne > 0) h->names[ne - 1] = (name);                                      \
        if (ev && cudaEventRecord(ev[ne], s) != cudaSuccess) return MOE_ERR_CUDA;   \
        ++ne;                                                                       \
    } while (0)
#define BLOCK_TRY(expr)                         \
    do {                                        \
        if ((rc = (expr)) != MOE_OK) return rc; \
    } while (0)

extern "C" int moe_dense_forward(moe_block_ctx *h, const void *x, void *out, int n_tokens,
                                 void *stream) {
    int rc = call_check(h, n_tokens);
    if (rc != MOE_OK) return rc;
    if (h->kind != 0) return MOE_ERR_INVALID_ARG;
    if (n_tokens == 0) return MOE_OK;
    if (!x || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out)) return MOE_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaEvent_t *ev = next_events(h);
    const int N = n_tokens, d = h->d, I = h->I;
    const int tiles = (N + kTcPairTileM - 1) / kTcPairTileM;
    int ne = 0;
    BLOCK_MARK(nullptr);
    BLOCK_TRY(norm_launch(h, x, N, s));
    BLOCK_MARK("norm");
    // gate/up: SiLU(gate) * up into act
    const int s1 = pick_split(h, N, tiles * ((I + 127) / 128), d, 2 * static_cast<size_t>(I));
    GroupedParams gp = group_params(h, true, I, d);
    if (s1 > 1) {
        gp.ksplit = s1; gp.partial = h->partial; gp.partial_rows = N;
        BLOCK_TRY(launch_gemm_tc2_mode(kEpiPartialPaired, h->m_w1, h->m_xn, gp, h->n_sm, s));
        BLOCK_MARK("gate_up_split");
        BLOCK_TRY(reduce_launch<kRedSiluMul>(h, s1, N, I, nullptr, h->mid, nullptr, nullptr, 1, s));
        BLOCK_MARK("gate_up_reduce");
    } else {
        gp.c = h->mid;
        BLOCK_TRY(launch_gemm_tc2_mode(kEpiSiluMul, h->m_w1, h->m_xn, gp, h->n_sm, s));
        BLOCK_MARK("gate_up");
    }
    // down + residual
    const int s2 = pick_split(h, N, tiles * ((d + 255) / 256), I, d);
    gp = group_params(h, false, d, I);
    if (s2 > 1) {
        gp.ksplit = s2; gp.partial = h->partial; gp.partial_rows = N;
        BLOCK_TRY(launch_gemm_tc2_mode(kEpiPartial, h->m_w2, h->m_mid, gp, h->n_sm, s));
        BLOCK_MARK("down_split");
        BLOCK_TRY(reduce_launch<kRedResid>(h, s2, N, d, x, out, nullptr, nullptr, 1, s));
        BLOCK_MARK("down_residual_reduce");
    } else {
        gp.c = out;
        gp.resid = x;
        // the act rows (N x I) outweigh W_down (d x I) as soon as N > d: then
        // each token tile is read once while the weight tiles stay in L2
        gp.wt_fastest = N > d;
        BLOCK_TRY(launch_gemm_tc2_mode(kEpiResid, h->m_w2, h->m_mid, gp, h->n_sm, s));
        BLOCK_MARK("down_residual");
    }
    h->n_names = ne - 1;
    return MOE_OK;
}

extern "C" int moe_conv_forward(moe_block_ctx *h, const void *x, void *out, int n_seqs,
                                int seq_len, const float *state_in, float *state_out,
                                void *stream) {
    if (!h || n_seqs < 0 || seq_len < 0) return MOE_ERR_INVALID_ARG;
    const long long n = static_cast<long long>(n_seqs) * seq_len;
    if (n > h->max_tokens) return MOE_ERR_TOO_MANY_TOKENS;
    int rc = call_check(h, static_cast<int>(n));
    if (rc != MOE_OK) return rc;
    if (h->kind != 1) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (n == 0) {
        // no positions: the state passes through unchanged
        if (state_out && n_seqs > 0 && state_out != state_in) {
            const size_t bytes = static_cast<size_t>(n_seqs) * 2 * h->d * 4;
            cudaError_t e = state_in ? cudaMemcpyAsync(state_out, state_in, bytes,
                                                       cudaMemcpyDeviceToDevice, s)
                                     : cudaMemsetAsync(state_out, 0, bytes, s);
            if (e != cudaSuccess) return MOE_ERR_CUDA;
        }
        return MOE_OK;
    }
    if (!x || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out)) return MOE_ERR_ALIGNMENT;
    const int N = static_cast<int>(n), d = h->d;
    const int tiles = (N + kTcPairTileM - 1) / kTcPairTileM;
    cudaEvent_t *ev = next_events(h);
    int ne = 0;
    BLOCK_MARK(nullptr);
    BLOCK_TRY(norm_launch(h, x, N, s));
    BLOCK_MARK("norm");
    // a = g * v
    const int s1 = pick_split(h, N, tiles * ((d + 127) / 128), d, 2 * static_cast<size_t>(d));
    GroupedParams gp = group_params(h, true, d, d);
    if (s1 > 1) {
        gp.ksplit = s1; gp.partial = h->partial; gp.partial_rows = N;
        BLOCK_TRY(launch_gemm_tc2_mode(kEpiPartialPaired, h->m_w1, h->m_xn, gp, h->n_sm, s));
        BLOCK_MARK("in_gv_split");
        BLOCK_TRY(reduce_launch<kRedMul>(h, s1, N, d, nullptr, h->mid, nullptr, nullptr, 1, s));
        BLOCK_MARK("in_gv_reduce");
    } else {
        gp.c = h->mid;
        BLOCK_TRY(launch_gemm_tc2_mode(kEpiMul, h->m_w1, h->m_xn, gp, h->n_sm, s));
        BLOCK_MARK("in_gv");
    }
    // y = u * (k0 a_t + k1 a_{t-1} + k2 a_{t-2}) along each sequence
    const int s2 = pick_split(h, N, tiles * ((d + 255) / 256), d, d);
    gp = group_params(h, false, d, d);
    if (s2 > 1) {
        gp.ksplit = s2; gp.partial = h->partial; gp.partial_rows = N;
        BLOCK_TRY(launch_gemm_tc2_mode(kEpiPartial, h->m_w2, h->m_xn, gp, h->n_sm, s));
        BLOCK_MARK("in_u_split");
        BLOCK_TRY(reduce_launch<kRedConv>(h, s2, N, d, nullptr, h->y, h->mid, state_in, seq_len, s));
        BLOCK_MARK("in_u_conv_reduce");
    } else {
        gp.c = h->y;
        gp.aux = h->mid;
        gp.conv = h->conv;
        gp.state_in = state_in;
        gp.seq_len = seq_len;
        BLOCK_TRY(launch_gemm_tc2_mode(kEpiConv, h->m_w2, h->m_xn, gp, h->n_sm, s));
        BLOCK_MARK("in_u_conv");
    }
    // out = x + W_out y
    const int s3 = pick_split(h, N, tiles * ((d + 255) / 256), d, d);
    gp = group_params(h, false, d, d);
    if (s3 > 1) {
        gp.ksplit = s3; gp.partial = h->partial; gp.partial_rows = N;
        BLOCK_TRY(launch_gemm_tc2_mode(kEpiPartial, h->m_w3, h->m_mid, gp, h->n_sm, s));
        BLOCK_MARK("out_split");
        BLOCK_TRY(reduce_launch<kRedResid>(h, s3, N, d, x, out, nullptr, nullptr, 1, s));
        BLOCK_MARK("out_residual_reduce");
    } else {
        gp.c = out;
        gp.resid = x;
        BLOCK_TRY(launch_gemm_tc2_mode(kEpiResid, h->m_w3, h->m_mid, gp, h->n_sm, s));
        BLOCK_MARK("out_residual");
    }
    if (state_out) {
        const size_t m = static_cast<size_t>(n_seqs) * d;
        const int blocks = static_cast<int>((m + 255) / 256 < 1024 ? (m + 255) / 256 : 1024);
        conv_state_kernel<<<blocks, 256, 0, s>>>(h->mid, state_in, state_out, n_seqs, seq_len, d);
        if (cudaPeekAtLastError() != cudaSuccess) return MOE_ERR_CUDA;
        BLOCK_MARK("state");
    }
    h->n_names = ne - 1;
    return MOE_OK;
}

#undef BLOCK_MARK
#undef BLOCK_TRY

extern "C" int moe_block_status(moe_block_ctx *h) {
    if (!h) return MOE_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    if (v & kStatusTimeout) return MOE_ERR_DEVICE_TIMEOUT;
    if (v & kStatusBounds) return MOE_ERR_DEVICE_BOUNDS;
    return MOE_OK;
}

extern "C" int moe_block_destroy(moe_block_ctx *h) {
    if (!h) return MOE_OK;
    const int rc = cudaDeviceSynchronize() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    block_free(h);
    return rc;
}

extern "C" int moe_block_profile(moe_block_ctx *h, int enable) {
    if (!h) return MOE_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    h->profile = enable != 0;
    h->ev_used = 0;
    return MOE_OK;
}

extern "C" int moe_block_kernel_times(moe_block_ctx *h, float *ms, int n) {
    if (!h || (n > 0 && !ms)) return MOE_ERR_INVALID_ARG;
    if (h->ev_used == 0) return 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    const int per = kMaxLaunches + 1;
    const size_t fwd = h->ev_used / per;
    double sum[kMaxLaunches] = {0};
    int k = 0;
    for (size_t f = 0; f < fwd; ++f) {
        cudaEvent_t *e = &h->ev[f * per];
        for (int i = 0; i < kMaxLaunches; ++i) {
            float t = 0.f;
            if (cudaEventElapsedTime(&t, e[i], e[i + 1]) != cudaSuccess) {
                cudaGetLastError();  // an event this forward did not record
                break;
            }
            sum[i] += t;
            if (i + 1 > k) k = i + 1;
        }
    }
    for (int i = 0; i < k && i < n; ++i) ms[i] = static_cast<float>(sum[i] / fwd);
    return k;
}

extern "C" const char *moe_block_kernel_name(moe_block_ctx *h, int i) {
    if (!h || i < 0 || i >= h->n_names) return nullptr;
    return h->names[i];
}
