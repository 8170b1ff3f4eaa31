// dispatch.cu -- grouping of the N*k token-expert assignments by expert:
// a deterministic counting sort ordered by (expert, token), with no atomics on
// the order-defining path.
//
// The page ("LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV
// Caches", flozi.net, English page, section "What to verify in a deployment")
// states that the default expert path groups tokens by expert; section "The
// router has two different scores" notes that a batch can activate many or all
// experts with uneven loads, so dispatch and regrouping matter.
//
// The route kernel already wrote one expert histogram per route CTA (a block
// of consecutive tokens). Here:
//   scan:    column prefix sums over the route CTAs give, for every (CTA,
//            expert), the first row that CTA's tokens take in the expert's
//            group; the per-expert counts and their exclusive prefix
//            (offsets) follow, plus the prefix of per-expert row tiles that
//            the grouped GEMMs schedule their work by.
//   scatter: each CTA ranks its own assignments among equal experts in
//            (token, slot) order, writes perm / inv, and copies the
//            normalised rows into grouped order (xp).
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) dispatch_scan_kernel(DispatchParams p) {
    __shared__ int seg_sum[kScanThreads];
    __shared__ int cnt[kMaxExperts];
    const int E = p.E, nblk = p.nblk;
    int G = 1;  // threads per expert: largest power of two with G * E <= 1024
    while (G * 2 * E <= kScanThreads) G *= 2;
    const int tid = threadIdx.x;
    const int e = tid / G, g = tid % G;
    const int L = (nblk + G - 1) / G;
    const int b0 = g * L, b1 = min(nblk, b0 + L);
    const bool active = e < E;

    int local = 0;
    if (active)
        for (int b = b0; b < b1; ++b) local += p.hist[static_cast<size_t>(b) * E + e];
    seg_sum[tid] = local;
    __syncthreads();
    // exclusive prefix of the G segments of expert e, and the expert's total
    int before = 0, total = 0;
    if (active) {
        for (int q = 0; q < G; ++q) {
            const int v = seg_sum[e * G + q];
            if (q < g) before += v;
            total += v;
        }
        if (g == 0) cnt[e] = total;
    }
    __syncthreads();
    if (tid == 0) {
        int off = 0, mt = 0;
        for (int x = 0; x < E; ++x) {
            p.offsets[x] = off;
            p.mt_start[x] = mt;
            p.counts[x] = cnt[x];
            off += cnt[x];
            mt += (cnt[x] + p.tile_m - 1) / p.tile_m;
        }
        p.offsets[E] = off;
        p.mt_start[E] = mt;
    }
    __syncthreads();
    if (active) {
        int run = p.offsets[e] + before;
        for (int b = b0; b < b1; ++b) {
            const size_t i = static_cast<size_t>(b) * E + e;
            p.base[i] = run;
            run += p.hist[i];
        }
    }
}

constexpr int kScatterThreads = 256;

__global__ void __launch_bounds__(kScatterThreads) dispatch_scatter_kernel(DispatchParams p) {
    __shared__ int pos_s[kMaxTopK * 8];
    const int b = blockIdx.x;
    const int t0 = b * p.toks_per_blk;
    const int ntok = min(p.toks_per_blk, p.N - t0);
    const int k = p.k, E = p.E;
    const int na = ntok * k;
    const int total = p.N * k;
    const int32_t *idx = p.idx + static_cast<size_t>(t0) * k;
    if (threadIdx.x < na) {
        const int a = threadIdx.x;
        const int e = idx[a];
        int pos = -1;
        if (e >= 0 && e < E) {
            int rank = 0;
            for (int q = 0; q < a; ++q) rank += (idx[q] == e);
            pos = p.base[static_cast<size_t>(b) * E + e] + rank;
            if (pos < 0 || pos >= total) pos = -1;
        }
        if (pos < 0) {
            set_status(p.status, kStatusBounds);
        } else {
            p.perm[pos] = t0 * k + a;
            p.inv[t0 * k + a] = pos;
        }
        pos_s[a] = pos;
    }
    __syncthreads();
    if (p.xp == nullptr) return;
    const int nvec = p.d * p.elem_bytes / 16;
    const uint4 *src = static_cast<const uint4 *>(p.xn);
    uint4 *dst = static_cast<uint4 *>(p.xp);
    for (int i = threadIdx.x; i < na * nvec; i += kScatterThreads) {
        const int a = i / nvec, v = i - a * nvec;
        const int pos = pos_s[a];
        if (pos >= 0)
            dst[static_cast<size_t>(pos) * nvec + v] =
                src[static_cast<size_t>(t0 + a / k) * nvec + v];
    }
}

}  // namespace

int launch_dispatch_scan(const DispatchParams &p, cudaStream_t s) {
    dispatch_scan_kernel<<<1, kScanThreads, 0, s>>>(p);
    return cudaPeekAtLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_dispatch_scatter(const DispatchParams &p, cudaStream_t s) {
    if (p.toks_per_blk * p.k > kMaxTopK * 8) return MOE_ERR_INVALID_ARG;
    dispatch_scatter_kernel<<<p.nblk, kScatterThreads, 0, s>>>(p);
    return cudaPeekAtLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
