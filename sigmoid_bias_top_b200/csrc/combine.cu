// combine.cu -- deterministic weighted combine plus residual:
//   out[t] = x[t] + sum_{j=0..k-1} w[t][j] * y[row(t, j)]
// with the sum in fp32 in fixed slot order and one final rounding to the
// storage dtype; no atomics, so the result is bitwise reproducible.
//
// The page ("LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV
// Caches", flozi.net, English page) states the residual structure in section
// "The exact checkpoint" and the weighted accumulation of the grouped expert
// outputs in section "What to verify in a deployment".
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;

struct F32x4 {
    using Raw = uint4;
    static constexpr int V = 4;
    static __device__ __forceinline__ void to_f(const Raw &r, float *f) {
        f[0] = __uint_as_float(r.x); f[1] = __uint_as_float(r.y);
        f[2] = __uint_as_float(r.z); f[3] = __uint_as_float(r.w);
    }
    static __device__ __forceinline__ Raw from_f(const float *f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                          __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};

struct Bf16x8 {
    using Raw = uint4;
    static constexpr int V = 8;
    static __device__ __forceinline__ void to_f(const Raw &r, float *f) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = bf16_to_f32(w[i] & 0xFFFFu);
            f[2 * i + 1] = bf16_to_f32(w[i] >> 16);
        }
    }
    static __device__ __forceinline__ Raw from_f(const float *f) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <typename P>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineParams p) {
    constexpr int V = P::V;
    const int t = blockIdx.x;
    const int k = p.k;
    pdl_trigger();
    pdl_wait();
    if (t == 0)  // the dispatch has consumed the chunk histogram: clear it for the next forward
        for (int i = threadIdx.x; i < p.chunk_hist_n; i += kThreads) p.chunk_hist[i] = 0;
    const int nvec = p.d / V;
    const int total = p.N * k;
    const uint4 *x = static_cast<const uint4 *>(p.x) + static_cast<size_t>(t) * nvec;
    const uint4 *y = static_cast<const uint4 *>(p.y);
    uint4 *out = static_cast<uint4 *>(p.out) + static_cast<size_t>(t) * nvec;
    for (int v = threadIdx.x; v < nvec; v += kThreads) {
        float acc[V], yv[V];
        P::to_f(x[v], acc);
        // slots in groups of four, the four loads of a group in flight together
        for (int j0 = 0; j0 < k; j0 += 4) {
            uint4 raw[4];
            float wj[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                wj[u] = 0.f;
                if (j0 + u < k) {
                    int r = p.inv[static_cast<size_t>(t) * k + j0 + u];
                    wj[u] = p.wts[static_cast<size_t>(t) * k + j0 + u];
                    if (r < 0 || r >= total) {  // never read outside y; report instead
                        set_status(p.status, kStatusBounds);
                        r = 0;
                        wj[u] = 0.f;
                    }
                    raw[u] = y[static_cast<size_t>(r) * nvec + v];
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (j0 + u < k) {
                    P::to_f(raw[u], yv);
#pragma unroll
                    for (int i = 0; i < V; ++i) acc[i] = fmaf(wj[u], yv[i], acc[i]);
                }
            }
        }
        out[v] = P::from_f(acc);
    }
}

}  // namespace

int launch_combine(const CombineParams &p, int dtype, cudaStream_t s) {
    if (dtype == MOE_F32) return launch_k(combine_kernel<F32x4>, dim3(p.N), dim3(kThreads), 0, s, p);
    return launch_k(combine_kernel<Bf16x8>, dim3(p.N), dim3(kThreads), 0, s, p);
}

}  // namespace moe
