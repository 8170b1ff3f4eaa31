// route.cu -- fused pre-FFN RMSNorm, fp32 router, per-logit sigmoid, biased
// top-k selection and weight normalisation (one kernel, SIMT fp32).
//
// Follows "LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV
// Caches" (flozi.net, English page), section "The router has two different
// scores": W_r[E x d] gives E logits per token, sigmoid is applied to each
// logit independently, the stored bias is added after the activation and only
// steers the top-k choice, and the mixture weights are the selected unbiased
// scores over (their sum + eps), times the routed scale. The router stays in
// fp32 (the FP8 release leaves the router gates unquantised, page 5, "Für
// Engineers"), fed by the fp32 normalised row, never by its bf16 copy.
//
// One CTA of 256 threads handles TT consecutive tokens:
//   A) one warp per token: sum of squares (fixed lane-strided order, then a
//      butterfly), xn = x * (1/sqrt(ms + eps)) * gain kept in fp32 in shared
//      memory and stored in the storage dtype for the experts;
//   B) warp w owns experts w, w+8, ...; lanes split d in float4 chunks; each
//      router row chunk is read once from L2 and used for all TT tokens;
//      partial dot products are reduced across the warp;
//   C) one warp per token: sigmoid, c = s + b, k rounds of a warp arg-max
//      (ties to the lower expert index), weights, per-CTA expert histogram.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kEB = 8;  // experts per register block in phase B

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

template <typename T, int TT>
__global__ void __launch_bounds__(kThreads) route_kernel(RouteParams p) {
    extern __shared__ float4 smem_f4[];
    float *xn_s = reinterpret_cast<float *>(smem_f4);  // [TT][d]
    float *sc = xn_s + TT * p.d;                       // [TT][E] logits, then scores
    int *hist = reinterpret_cast<int *>(sc + TT * p.E);  // [E]

    const int d = p.d, E = p.E, k = p.k;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * TT;
    const int ntok = min(TT, p.N - t0);

    for (int e = threadIdx.x; e < E; e += kThreads) hist[e] = 0;

    // A) RMSNorm
    for (int tl = warp; tl < TT; tl += kWarps) {
        float *row_s = xn_s + tl * d;
        if (tl < ntok) {
            const T *xr = static_cast<const T *>(p.x) + static_cast<size_t>(t0 + tl) * d;
            T *xo = static_cast<T *>(p.xn) + static_cast<size_t>(t0 + tl) * d;
            float ss = 0.f;
            for (int j = lane * 4; j < d; j += 128) {
                float4 v = Vec4<T>::load(xr + j);
                ss += v.x * v.x;
                ss += v.y * v.y;
                ss += v.z * v.z;
                ss += v.w * v.w;
            }
            ss = warp_sum(ss);
            const float rinv = 1.0f / sqrtf(ss / static_cast<float>(d) + p.eps);
            for (int j = lane * 4; j < d; j += 128) {
                float4 v = Vec4<T>::load(xr + j);
                float4 g = *reinterpret_cast<const float4 *>(p.gain + j);
                float4 o = make_float4(v.x * rinv * g.x, v.y * rinv * g.y, v.z * rinv * g.z,
                                       v.w * rinv * g.w);
                *reinterpret_cast<float4 *>(row_s + j) = o;
                Vec4<T>::store(xo + j, o);
            }
        } else {
            for (int j = lane * 4; j < d; j += 128)
                *reinterpret_cast<float4 *>(row_s + j) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    __syncthreads();

    // B) logits l[t][e] = W_r[e] . xn_t
    for (int eb0 = warp * kEB; eb0 < E; eb0 += kWarps * kEB) {
        float acc[kEB][TT];
#pragma unroll
        for (int i = 0; i < kEB; ++i)
#pragma unroll
            for (int t = 0; t < TT; ++t) acc[i][t] = 0.f;
        for (int j = lane * 4; j < d; j += 128) {
            float4 wv[kEB];
#pragma unroll
            for (int i = 0; i < kEB; ++i) {
                const int e = eb0 + i;
                wv[i] = (e < E) ? __ldg(reinterpret_cast<const float4 *>(
                                      p.router_w + static_cast<size_t>(e) * d + j))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const float4 xv = *reinterpret_cast<const float4 *>(xn_s + t * d + j);
#pragma unroll
                for (int i = 0; i < kEB; ++i) {
                    float a = acc[i][t];
                    a = fmaf(wv[i].x, xv.x, a);
                    a = fmaf(wv[i].y, xv.y, a);
                    a = fmaf(wv[i].z, xv.z, a);
                    a = fmaf(wv[i].w, xv.w, a);
                    acc[i][t] = a;
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kEB; ++i)
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const float v = warp_sum(acc[i][t]);
                const int e = eb0 + i;
                if (lane == 0 && e < E) sc[t * E + e] = v;
            }
    }
    __syncthreads();

    // C) sigmoid, biased top-k, normalised unbiased weights
    for (int tl = warp; tl < ntok; tl += kWarps) {
        float c_reg[kMaxExperts / 32];
        uint32_t taken = 0;  // bit i: expert lane + 32 i already selected
        float *srow = sc + tl * E;
#pragma unroll
        for (int i = 0; i < kMaxExperts / 32; ++i) {
            const int e = lane + 32 * i;
            c_reg[i] = -INFINITY;
            if (e < E) {
                const float s = 1.0f / (1.0f + expf(-srow[e]));
                const float c = s + p.bias[e];
                c_reg[i] = (c == c) ? c : -INFINITY;  // a NaN score never wins
                srow[e] = s;  // each lane rewrites only its own experts
            } else {
                taken |= 1u << i;
            }
        }
        __syncwarp();
        int sel[kMaxTopK];
        float ssel[kMaxTopK];
        for (int j = 0; j < k; ++j) {
            float bc = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < kMaxExperts / 32; ++i) {
                const int e = lane + 32 * i;
                // ascending e within a lane: ties keep the lower index
                if (!(taken & (1u << i)) && (c_reg[i] > bc || be == 0x7fffffff)) {
                    bc = c_reg[i];
                    be = e;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float oc = __shfl_xor_sync(0xffffffffu, bc, o);
                const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                if (oe != 0x7fffffff && (be == 0x7fffffff || oc > bc || (oc == bc && oe < be))) {
                    bc = oc;
                    be = oe;
                }
            }
            // k <= E guarantees an untaken expert exists, so be < E here
            sel[j] = be;
            ssel[j] = srow[be];
#pragma unroll
            for (int i = 0; i < kMaxExperts / 32; ++i)
                if (lane + 32 * i == be) taken |= 1u << i;
        }
        if (lane == 0) {
            float sum = 0.f;
            for (int j = 0; j < k; ++j) sum += ssel[j];
            const float den = sum + p.eps;
            const size_t t = static_cast<size_t>(t0 + tl);
            for (int j = 0; j < k; ++j) {
                p.idx[t * k + j] = sel[j];
                p.wts[t * k + j] = p.scale * (ssel[j] / den);
                atomicAdd(&hist[sel[j]], 1);
            }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads)
        p.hist[static_cast<size_t>(blockIdx.x) * E + e] = hist[e];
}

template <typename T, int TT>
int launch_tt(const RouteParams &p, cudaStream_t s) {
    const int nblk = (p.N + TT - 1) / TT;
    const size_t smem = (static_cast<size_t>(TT) * p.d + static_cast<size_t>(TT) * p.E) * 4 +
                        static_cast<size_t>(p.E) * 4;
    auto kern = route_kernel<T, TT>;
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    kern<<<nblk, kThreads, smem, s>>>(p);
    return cudaPeekAtLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <typename T>
int launch_t(const RouteParams &p, int tt, cudaStream_t s) {
    switch (tt) {
        case 1: return launch_tt<T, 1>(p, s);
        case 2: return launch_tt<T, 2>(p, s);
        case 4: return launch_tt<T, 4>(p, s);
        case 8: return launch_tt<T, 8>(p, s);
        default: return MOE_ERR_INVALID_ARG;
    }
}

}  // namespace

int launch_route(const RouteParams &p, int dtype, int toks_per_blk, cudaStream_t s) {
    if (dtype == MOE_F32) return launch_t<float>(p, toks_per_blk, s);
    return launch_t<__nv_bfloat16>(p, toks_per_blk, s);
}

}  // namespace moe
