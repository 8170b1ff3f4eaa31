// gemm_simt.cu -- fp32 grouped GEMMs on the CUDA cores, for layers stored in
// fp32 (tensor-core formats cannot hold the 1e-5 relative tolerance that fp32
// storage calls for).
//
// Each expert e owns the contiguous row range [offsets[e], offsets[e+1]) of the
// grouped activations. The gated SiLU expert of "LFM2.5-24B-A2B: Biased
// Routing, Short Convolutions and Ten KV Caches" (flozi.net, English page,
// section "The router has two different scores") is computed in two grouped
// contractions:
//   gate/up: act[r][f] = silu(xp[r] . Wg_e[f]) * (xp[r] . Wu_e[f]), with the
//            gate rows 0..I-1 and up rows I..2I-1 of the packed [2I][d] matrix;
//   down:    y[r][n]   = act[r] . Wd_e[n].
// A CTA computes a 64-row x 64-column tile with a 4x4 register block per
// thread; blockIdx.x walks the per-expert row tiles through the prefix
// mt_start, blockIdx.y the output columns.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = kSimtTileM, BN = 64, BK = 16, kThreads = 256;

template <typename T>
__device__ __forceinline__ float ld_f(const T *p, size_t i);
template <>
__device__ __forceinline__ float ld_f<float>(const float *p, size_t i) { return p[i]; }
template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }

// Largest e in [0, E) with mts[e] <= q (mts non-decreasing, mts[0] = 0).
__device__ __forceinline__ int find_expert(const int32_t *mts, int E, int q) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mts[mid] <= q) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <typename T, bool GATE_UP>
__global__ void __launch_bounds__(kThreads) grouped_simt_kernel(GroupedParams p) {
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[GATE_UP ? 2 : 1][BK][BN + 4];
    const int E = p.E;
    const int mt = blockIdx.x;
    pdl_trigger();
    pdl_wait();
    if (mt >= p.mt_start[E]) return;
    const int e = find_expert(p.mt_start, E, mt);
    const int row0 = p.offsets[e] + (mt - p.mt_start[e]) * BM;
    const int rows = min(BM, p.offsets[e + 1] - row0);
    const int K = GATE_UP ? p.d : p.I;
    const int NOUT = GATE_UP ? p.I : p.d;
    const int n0 = blockIdx.y * BN;
    if (row0 < 0 || row0 + rows > p.rows_cap) {
        if (threadIdx.x == 0) set_status(p.status, kStatusBounds);
        return;
    }
    const T *A = static_cast<const T *>(p.a);
    const T *W = static_cast<const T *>(p.w) +
                 static_cast<size_t>(e) * (GATE_UP ? 2 * p.I : p.d) * K;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[2][4][4] = {};

    for (int k0 = 0; k0 < K; k0 += BK) {
        for (int i = threadIdx.x; i < BM * BK; i += kThreads) {
            const int r = i / BK, kk = i % BK;
            As[kk][r] = (r < rows && k0 + kk < K)
                            ? ld_f(A, static_cast<size_t>(row0 + r) * K + k0 + kk) : 0.f;
        }
        for (int i = threadIdx.x; i < BN * BK; i += kThreads) {
            const int n = i / BK, kk = i % BK;
            const bool ok = (n0 + n < NOUT) && (k0 + kk < K);
            Bs[0][kk][n] = ok ? ld_f(W, static_cast<size_t>(n0 + n) * K + k0 + kk) : 0.f;
            if (GATE_UP)
                Bs[GATE_UP ? 1 : 0][kk][n] =
                    ok ? ld_f(W, static_cast<size_t>(p.I + n0 + n) * K + k0 + kk) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[4], b0[4], b1[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = As[kk][ty * 4 + i];
                b0[i] = Bs[0][kk][tx * 4 + i];
                b1[i] = GATE_UP ? Bs[GATE_UP ? 1 : 0][kk][tx * 4 + i] : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[0][i][j] = fmaf(a[i], b0[j], acc[0][i][j]);
                    if (GATE_UP) acc[1][i][j] = fmaf(a[i], b1[j], acc[1][i][j]);
                }
        }
        __syncthreads();
    }

    T *C = static_cast<T *>(p.c);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i;
        if (r >= rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= NOUT) continue;
            float v;
            if (GATE_UP) {
                const float g = acc[0][i][j];
                v = g / (1.0f + expf(-g)) * acc[1][i][j];
            } else {
                v = acc[0][i][j];
            }
            C[static_cast<size_t>(row0 + r) * NOUT + n] = from_f<T>(v);
        }
    }
}

}  // namespace

int launch_gemm_simt_gate_up(const GroupedParams &p, int max_mtiles, cudaStream_t s) {
    return launch_k(grouped_simt_kernel<float, true>, dim3(max_mtiles, (p.I + BN - 1) / BN),
                    dim3(kThreads), 0, s, p);
}

int launch_gemm_simt_down(const GroupedParams &p, int max_mtiles, cudaStream_t s) {
    return launch_k(grouped_simt_kernel<float, false>, dim3(max_mtiles, (p.d + BN - 1) / BN),
                    dim3(kThreads), 0, s, p);
}

}  // namespace moe
