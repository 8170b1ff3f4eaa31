// route.cu -- fused pre-FFN RMSNorm, fp32 router, per-logit sigmoid, biased
// top-k selection and weight normalisation (SIMT fp32, no tensor cores).
//
// Follows "LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV
// Caches" (flozi.net, English page), section "The router has two different
// scores": W_r[E x d] gives E logits per token, sigmoid is applied to each
// logit independently, the stored bias is added after the activation and only
// steers the top-k choice, and the mixture weights are the selected unbiased
// scores over (their sum + eps), times the routed scale. The router stays in
// fp32 (the FP8 release leaves the router gates unquantised: inferencekey.com,
// "LFM2.5-24B-A2B: ein 24B-Reasoning-Modell, das pro Wortstück so wenig
// verbraucht wie ein 2B-Modell", section "Für Engineers"), fed by the fp32
// normalised row, never by its bf16 copy.
//
// Two kernels, chosen by batch size:
// The RMSNorm gain is folded into the router matrix once, at context creation
// (W' = W_r * gain, column-wise), and 1/rms is applied to each token's dot
// products: l_e = rinv * sum_j x_j W'_ej, the same value as W_r[e] . xn up to
// fp32 rounding, with no per-element scaling in the inner loops.
//   small batches: a cluster of 8 CTAs per group of TT tokens; CTA r stages
//     its E/8 rows of W' and the group's rows of x in shared memory (bulk
//     copies) and computes their logits with its 8 warps tiled over (tokens x
//     experts), lanes splitting d, in one pass that also sums the squares;
//     the logits go to CTA 0 through distributed shared memory, which then
//     selects and normalises;
//   large batches: one CTA per 32 tokens computes the 32 x 64 logit tile as a
//     register-tiled SGEMM over d (4 x 4 outputs per thread, double-buffered
//     shared-memory chunks of x and of W' transposed to [d][E]); its two
//     halves take alternate chunks and their partial sums are added in a
//     fixed order.
// Both end with the same per-token selection: sigmoid, c = s + b, k rounds of
// a warp arg-max (ties to the lower expert index), weights, and the count of
// selected experts added to the token chunk's histogram (the dispatch input).
// They store the per-token 1/rms; the dispatch writes the normalised rows
// (x * rinv * gain, the same fp32 products) in grouped order for the experts.
#include <cooperative_groups.h>

#include "moe_internal.cuh"

namespace cg = cooperative_groups;

namespace moe {
namespace {

template <typename T>
struct Vec4;
template <>
struct Vec4<float> {
    static __device__ __forceinline__ float4 load(const float *p) {
        return *reinterpret_cast<const float4 *>(p);
    }
    static __device__ __forceinline__ void store(float *p, float4 v) {
        *reinterpret_cast<float4 *>(p) = v;
    }
};
template <>
struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load(const __nv_bfloat16 *p) {
        uint2 u = *reinterpret_cast<const uint2 *>(p);
        return make_float4(bf16_to_f32(u.x & 0xFFFFu), bf16_to_f32(u.x >> 16),
                           bf16_to_f32(u.y & 0xFFFFu), bf16_to_f32(u.y >> 16));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float4 v) {
        __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
        __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t *>(&a);
        u.y = *reinterpret_cast<uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(p) = u;
    }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// 1 / sqrt(mean(x^2) + eps) of one row, by one warp: lane-strided partial
// sums in ascending column order (eight loads in flight), then a butterfly.
template <typename T>
__device__ __forceinline__ float row_rinv(const T *xr, int d, float eps, int lane) {
    constexpr int B = 8;
    float ss = 0.f;
    for (int base = lane * 4; base < d; base += 128 * B) {
        float4 v[B];
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int j = base + u * 128;
            v[u] = j < d ? Vec4<T>::load(xr + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < B; ++u) {
            ss += v[u].x * v[u].x;
            ss += v[u].y * v[u].y;
            ss += v[u].z * v[u].z;
            ss += v[u].w * v[u].w;
        }
    }
    ss = warp_sum(ss);
    return 1.0f / sqrtf(ss / static_cast<float>(d) + eps);
}

// Adds a CTA's expert counts to the histogram of the token chunk it lies in.
__device__ __forceinline__ void flush_hist(const RouteParams &p, const int *hist, int t0) {
    int32_t *row = p.chunk_hist + static_cast<size_t>(t0 / p.chunk_tokens) * p.E;
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
        if (hist[e]) atomicAdd(&row[e], hist[e]);
}

// ---------------------------------------------------------------------------
// Small batches: cluster of 8 CTAs, CTA r owns experts [r*EG, (r+1)*EG).

constexpr int kSmallThreads = 256;
constexpr int kClusterCtas = 8;

template <typename T, int TT, int EG>
__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kSmallThreads)
    route_small_kernel(RouteParams p) {
    // TT tokens per cluster, EG experts per CTA, 8 warps tiled WT x WE
    constexpr int WE = EG < 4 ? EG : 4;   // warps along the experts
    constexpr int WT = 8 / WE;            // warps along the tokens
    constexpr int EPW = EG / WE;          // experts per warp
    constexpr int TPW = TT / WT;          // tokens per warp
    extern __shared__ float4 smem_f4[];
    float *wsl = reinterpret_cast<float *>(smem_f4);  // [EG][d] router rows times gain
    T *xs = reinterpret_cast<T *>(wsl + EG * p.d);    // [TT][d] this group's rows of x
    float *sc = reinterpret_cast<float *>(
        reinterpret_cast<uint8_t *>(xs) + ((static_cast<size_t>(TT) * p.d * sizeof(T) + 15) & ~size_t(15)));
    float *bias_s = sc + TT * p.E;                    // [E]
    float *rinv_s = bias_s + p.E;                     // [TT]
    int *hist = reinterpret_cast<int *>(rinv_s + TT);  // [E]

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int d = p.d, E = p.E;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = (blockIdx.x / kClusterCtas) * TT;
    const int ntok = min(TT, p.N - t0);
    const int e0 = rank * EG;

    // layer parameters first (no earlier kernel writes them): the router rows
    // by one bulk copy, the bias into shared memory
    __shared__ uint64_t wbar, xbar;
    if (threadIdx.x == 0) {
        mbar_init(&wbar, 1);
        mbar_init(&xbar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const uint32_t wbytes = static_cast<uint32_t>(EG) * d * 4;
    if (threadIdx.x == 0) {
        const float *src = p.router_wg + static_cast<size_t>(e0) * d;
        mbar_arrive_expect_tx(&wbar, wbytes);
        for (uint32_t off = 0; off < wbytes; off += 32768u)
            bulk_copy_g2s(wsl + off / 4, src + off / 4, min(32768u, wbytes - off), &wbar);
    }
    for (int e = threadIdx.x; e < E; e += kSmallThreads) {
        hist[e] = 0;
        bias_s[e] = p.bias[e];
    }
    pdl_trigger();
    pdl_wait();
    // this group's rows of x (consecutive tokens) by one bulk copy
    const uint32_t xbytes = static_cast<uint32_t>(ntok) * d * sizeof(T);
    if (threadIdx.x == 0) {
        const uint8_t *src = reinterpret_cast<const uint8_t *>(static_cast<const T *>(p.x) +
                                                               static_cast<size_t>(t0) * d);
        mbar_arrive_expect_tx(&xbar, xbytes);
        for (uint32_t off = 0; off < xbytes; off += 32768u)
            bulk_copy_g2s(reinterpret_cast<uint8_t *>(xs) + off, src + off,
                          min(32768u, xbytes - off), &xbar);
    }
    const uint64_t dl = globaltimer_ns() + 1000000000ull;
    if (!mbar_wait(&wbar, 0, dl) || !mbar_wait(&xbar, 0, dl)) set_status(p.status, kStatusTimeout);

    // warps tile (token groups x expert groups): warp = wt * WE + we takes
    // tokens [wt*TPW, +TPW) and experts [we*EPW, +EPW) of this CTA, so each
    // row of x and of W' read from shared memory feeds several outputs.
    // Lanes take 4 columns of each 128-column chunk.
    const int we = warp % WE, wt = warp / WE;
    const T *xr[TPW];
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
        const int tl = wt * TPW + i;
        xr[i] = xs + static_cast<size_t>(tl < ntok ? tl : 0) * d;
    }
    const float *wr = wsl + static_cast<size_t>(we * EPW) * d;
    float acc[EPW][TPW], ss[TPW];
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
        ss[i] = 0.f;
#pragma unroll
        for (int e = 0; e < EPW; ++e) acc[e][i] = 0.f;
    }
#pragma unroll 4
    for (int j = lane * 4; j < d; j += 128) {
        float4 xv[TPW];
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
            xv[i] = Vec4<T>::load(xr[i] + j);
            if (we == 0) {  // the first expert group also sums the squares
                ss[i] += xv[i].x * xv[i].x;
                ss[i] += xv[i].y * xv[i].y;
                ss[i] += xv[i].z * xv[i].z;
                ss[i] += xv[i].w * xv[i].w;
            }
        }
#pragma unroll
        for (int e = 0; e < EPW; ++e) {
            const float4 w = *reinterpret_cast<const float4 *>(wr + e * d + j);
#pragma unroll
            for (int i = 0; i < TPW; ++i) {
                float a = acc[e][i];
                a = fmaf(w.x, xv[i].x, a);
                a = fmaf(w.y, xv[i].y, a);
                a = fmaf(w.z, xv[i].z, a);
                a = fmaf(w.w, xv[i].w, a);
                acc[e][i] = a;
            }
        }
    }
    if (we == 0) {
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
            const int tl = wt * TPW + i;
            const float tot = warp_sum(ss[i]);
            if (lane == 0) {
                const float r = tl < ntok ? 1.0f / sqrtf(tot / static_cast<float>(d) + p.eps) : 0.f;
                rinv_s[tl] = r;
                if (tl < ntok && rank == 0) p.rinv[t0 + tl] = r;
            }
        }
    }
    __syncthreads();
    float *sc0 = cluster.map_shared_rank(sc, 0);
#pragma unroll
    for (int e = 0; e < EPW; ++e)
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
            const int tl = wt * TPW + i;
            const float v = warp_sum(acc[e][i]) * rinv_s[tl];
            if (lane == 0) sc0[tl * E + e0 + we * EPW + e] = v;
        }
    cluster.sync();
    if (rank != 0) return;

    for (int tl = warp; tl < ntok; tl += kSmallThreads / 32)
        select_token(p, sc + tl * E, bias_s, static_cast<size_t>(t0 + tl), hist, lane);
    __syncthreads();
    flush_hist(p, hist, t0);
}

// ---------------------------------------------------------------------------
// Large batches: 32 tokens x all experts per CTA, register-tiled SGEMM; the
// two halves of the CTA take alternate d-chunks and their partial sums are
// added in a fixed order.

constexpr int kLargeThreads = 256;
constexpr int LT = 32;   // tokens per CTA
constexpr int LKC = 32;  // d per shared-memory chunk
constexpr int LXS = LT + 4;
constexpr int kGroupThreads = 128;

size_t large_smem(int E) {
    return (2 * 2 * LKC * LXS + 2 * 2 * LKC * 64 + LT * 64 + LT * static_cast<size_t>(E) + LT) * 4 +
           2 * static_cast<size_t>(E) * 4;
}

template <typename T>
__global__ void __launch_bounds__(kLargeThreads) route_large_kernel(RouteParams p) {
    extern __shared__ float4 smem_f4[];
    float *xs_all = reinterpret_cast<float *>(smem_f4);        // [2 grp][2 buf][LKC][LXS]
    float *ws_all = xs_all + 2 * 2 * LKC * LXS;                // [2 grp][2 buf][LKC][64]
    float *red = ws_all + 2 * 2 * LKC * 64;                    // [LT][64] second half's sums
    float *sc = red + LT * 64;                                 // [LT][E]
    float *rinv_s = sc + LT * p.E;                             // [LT]
    float *bias_s = rinv_s + LT;                               // [E]
    int *hist = reinterpret_cast<int *>(bias_s + p.E);         // [E]

    const int d = p.d, E = p.E, Ep = p.e_pad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = tid / kGroupThreads, gt = tid % kGroupThreads;
    const int t0 = blockIdx.x * LT;
    const int ntok = min(LT, p.N - t0);
    for (int e = tid; e < E; e += kLargeThreads) {
        hist[e] = 0;
        bias_s[e] = p.bias[e];
    }
    pdl_trigger();
    pdl_wait();
    for (int tl = warp; tl < LT; tl += kLargeThreads / 32) {
        const float r = tl < ntok ? row_rinv<T>(static_cast<const T *>(p.x) +
                                                    static_cast<size_t>(t0 + tl) * d,
                                                d, p.eps, lane)
                                  : 0.f;
        if (lane == 0) {
            rinv_s[tl] = r;
            if (tl < ntok) p.rinv[t0 + tl] = r;
        }
    }
    __syncthreads();

    // loader roles: x -- token xt (the lane, so the transposed stores of a
    // warp hit 32 distinct banks), 8 consecutive columns at xq*8 (the warp);
    // W'^T -- 4 float4 slots
    const int xt = gt & 31, xq = gt >> 5;
    const bool xvalid = xt < ntok;
    const T *xrow = static_cast<const T *>(p.x) + static_cast<size_t>(xvalid ? t0 + xt : 0) * d;
    // compute roles: tokens ty*4.., experts tx*4..
    const int ty = gt >> 4, tx = gt & 15;
    const int nchunk = (d + LKC - 1) / LKC;
    const int rounds = (nchunk + 1) / 2;  // chunk 2*r + grp in round r
    float *xs_g = xs_all + grp * 2 * LKC * LXS;
    float *ws_g = ws_all + grp * 2 * LKC * 64;

    for (int eb = 0; eb < E; eb += 64) {
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
        float4 xa, xb, wv[4];
        auto fetch = [&](int c) {
            const int k0 = c * LKC;
            const int j = k0 + xq * 8;
            if (c < nchunk && j < d) {
                xa = Vec4<T>::load(xrow + j);
                xb = (j + 4 < d) ? Vec4<T>::load(xrow + j + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                xa = xb = make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int slot = gt + kGroupThreads * i;  // 512 float4 = 32 rows x 16
                const int row = k0 + (slot >> 4), col = eb + (slot & 15) * 4;
                wv[i] = (c < nchunk && row < d)
                            ? __ldg(reinterpret_cast<const float4 *>(
                                  p.router_wt + static_cast<size_t>(row) * Ep + col))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        };
        fetch(grp);
        for (int r = 0; r < rounds; ++r) {
            const int c = 2 * r + grp;
            const int buf = r & 1;
            float *xs = xs_g + buf * LKC * LXS;
            float *ws = ws_g + buf * LKC * 64;
            const float v[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) xs[(xq * 8 + q) * LXS + xt] = v[q];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int slot = gt + kGroupThreads * i;
                *reinterpret_cast<float4 *>(&ws[(slot >> 4) * 64 + (slot & 15) * 4]) = wv[i];
            }
            __syncthreads();
            fetch(c + 2);
#pragma unroll
            for (int kk = 0; kk < LKC; ++kk) {
                const float4 a = *reinterpret_cast<const float4 *>(&xs[kk * LXS + ty * 4]);
                const float4 b = *reinterpret_cast<const float4 *>(&ws[kk * 64 + tx * 4]);
                const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
        }
        if (grp == 1)
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) red[(ty * 4 + i) * 64 + tx * 4 + j] = acc[i][j];
        __syncthreads();
        if (grp == 0)
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int e = eb + tx * 4 + j;
                    if (e < E)
                        sc[(ty * 4 + i) * E + e] =
                            (acc[i][j] + red[(ty * 4 + i) * 64 + tx * 4 + j]) * rinv_s[ty * 4 + i];
                }
        __syncthreads();
    }

    for (int tl = warp; tl < ntok; tl += kLargeThreads / 32)
        select_token(p, sc + tl * E, bias_s, static_cast<size_t>(t0 + tl), hist, lane);
    __syncthreads();
    flush_hist(p, hist, t0);
}


size_t small_smem(int EG, int TT, int d, int E, int elem) {
    return static_cast<size_t>(EG) * d * 4 + ((static_cast<size_t>(TT) * d * elem + 15) & ~size_t(15)) +
           (static_cast<size_t>(TT) * E + 2 * static_cast<size_t>(E) + TT) * 4;
}

template <typename T, int TT, int EG>
int launch_small(const RouteParams &p, cudaStream_t s) {
    const int groups = (p.N + TT - 1) / TT;
    const size_t smem = small_smem(EG, TT, p.d, p.E, sizeof(T));
    auto kern = route_small_kernel<T, TT, EG>;
    if (ensure_smem(kern, smem) != MOE_OK) return MOE_ERR_CUDA;
    return launch_k(kern, dim3(groups * kClusterCtas), dim3(kSmallThreads), smem, s, p);
}

template <typename T, int TT>
int launch_small_eg(const RouteParams &p, cudaStream_t s) {
    switch (p.E / kClusterCtas) {
        case 1: return launch_small<T, TT, 1>(p, s);
        case 2: return launch_small<T, TT, 2>(p, s);
        case 4: return launch_small<T, TT, 4>(p, s);
        case 8: return launch_small<T, TT, 8>(p, s);
        case 16: return launch_small<T, TT, 16>(p, s);
        default: return MOE_ERR_INVALID_ARG;
    }
}

template <typename T>
int launch_small_t(const RouteParams &p, int tt, cudaStream_t s) {
    switch (tt) {
        case 8: return launch_small_eg<T, 8>(p, s);
        case 16: return launch_small_eg<T, 16>(p, s);
        case 32: return launch_small_eg<T, 32>(p, s);
        default: return MOE_ERR_INVALID_ARG;
    }
}

template <typename T>
int launch_large(const RouteParams &p, cudaStream_t s) {
    const size_t smem = large_smem(p.E);
    auto kern = route_large_kernel<T>;
    if (ensure_smem(kern, smem) != MOE_OK) return MOE_ERR_CUDA;
    return launch_k(kern, dim3((p.N + LT - 1) / LT), dim3(kLargeThreads), smem, s, p);
}

// W' = W_r * gain (column-wise), stored as [E][d] (wg) and as [d][e_pad] with
// zero columns past E (wt).
__global__ void prepare_router_kernel(const float *w, const float *gain, float *wg, float *wt,
                                      int E, int e_pad, int d) {
    const size_t n = static_cast<size_t>(d) * e_pad;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const int j = static_cast<int>(i / e_pad), e = static_cast<int>(i % e_pad);
        const float v = e < E ? w[static_cast<size_t>(e) * d + j] * gain[j] : 0.f;
        wt[i] = v;
        if (e < E) wg[static_cast<size_t>(e) * d + j] = v;
    }
}

}  // namespace

int launch_prepare_router(const float *w, const float *gain, float *wg, float *wt, int E,
                          int e_pad, int d, cudaStream_t s) {
    prepare_router_kernel<<<256, 256, 0, s>>>(w, gain, wg, wt, E, e_pad, d);
    return cudaPeekAtLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

bool route_small_ok(int d, int E) {
    if (E % kClusterCtas != 0) return false;
    const int eg = E / kClusterCtas;
    if (eg != 1 && eg != 2 && eg != 4 && eg != 8 && eg != 16) return false;
    return small_smem(eg, 8, d, E, 4) <= 200 * 1024;  // at least the 8-token groups fit
}

int route_plan(int N, int d, int E, int *toks_per_group) {
    // the cluster kernel while its groups give fewer CTAs than the tiled
    // kernel would need to fill the GPU twice; the tiled kernel beyond. The
    // group shrinks until its router rows and token rows fit in shared memory.
    if (route_small_ok(d, E) && N < 4096) {
        int tt = N <= 64 ? 8 : N <= 256 ? 16 : 32;
        while (tt > 8 && small_smem(E / kClusterCtas, tt, d, E, 4) > 200 * 1024) tt /= 2;
        *toks_per_group = tt;
        return kRouteSmall;
    }
    *toks_per_group = LT;
    return kRouteLarge;
}

int launch_route(const RouteParams &p, int dtype, int kind, int toks_per_group, cudaStream_t s) {
    if (kind == kRouteSmall)
        return dtype == MOE_F32 ? launch_small_t<float>(p, toks_per_group, s)
                                : launch_small_t<__nv_bfloat16>(p, toks_per_group, s);
    return dtype == MOE_F32 ? launch_large<float>(p, s) : launch_large<__nv_bfloat16>(p, s);
}

}  // namespace moe
