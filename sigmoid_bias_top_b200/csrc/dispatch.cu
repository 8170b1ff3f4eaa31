// dispatch.cu -- grouping of the N*k token-expert assignments by expert: a
// deterministic counting sort ordered by (expert, token), with no atomics on
// the order-defining path, plus the copy of each assignment's normalised row
// into its grouped position.
//
// The page ("LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV
// Caches", flozi.net, English page, section "What to verify in a deployment")
// states that the default expert path groups tokens by expert; section "The
// router has two different scores" notes that a batch can activate many or all
// experts with uneven loads, so dispatch and regrouping matter.
//
// Tokens are split into chunks of chunk_tokens consecutive tokens; the route
// kernels have already added each chunk's per-expert counts to chunk_hist.
// `replicas` CTAs per chunk then each
//   1. read the whole (chunks x E) histogram and form the per-expert totals,
//      their exclusive prefix over experts (offsets) and the prefix over the
//      chunks before their own (CTA 0 also publishes offsets, counts and the
//      prefix of per-expert row tiles that the grouped GEMMs schedule by);
//   2. rank the chunk's assignments among equal experts in (token, slot)
//      order: each warp takes a contiguous slice, counts it per expert in
//      rounds of 32 (__match_any_sync), the warps' counts are prefixed, and a
//      second pass assigns positions;
//   3. replica 0 writes perm (grouped row -> assignment t*k+j) and inv (the
//      reverse); the replicas share out the chunk's tokens, split into column
//      segments, one warp per (token, segment): the segment of the normalised
//      row x[t] * rinv[t] * gain (the same fp32 products as the router's
//      input, rounded once to the storage type) is formed once and stored at
//      each of the token's k grouped positions.
// The grouped rows let the gate/up GEMM load contiguous 128-row TMA boxes.
// For FP8_BLOCK layers ("LFM2.5-24B-A2B: ein 24B-Reasoning-Modell, das pro Wortstück so wenig verbraucht wie ein 2B-Modell",
// inferencekey.com, section "Für Engineers", paragraph "Quantisierung":
// activations FP8, dynamic per group of 128) step 3 writes
// e4m3 codes instead: each group of 128 normalised values (16 lanes) takes
// s = amax / 448 and codes e4m3(v / s), nearest-even and saturating, with the
// scale stored beside the codes.
#include <cuda_fp8.h>

#include "moe_fp8.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Exclusive prefix sum of v over threads 0..n-1 (n <= kThreads); every thread
// of the block must call it. Returns the prefix; *total gets the sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int n, int *warp_sums, int *total) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int x = tid < n ? v : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kWarps ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < kWarps; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kWarps) warp_sums[lane] = w;  // inclusive
    }
    __syncthreads();
    const int before = warp > 0 ? warp_sums[warp - 1] : 0;
    *total = warp_sums[kWarps - 1];
    const int incl = x + before;
    __syncthreads();  // warp_sums may be reused by the next call
    return incl - (tid < n ? v : 0);
}

// One group of 8 normalised values per lane, 16 lanes per group of 128: the
// group's scale (shared by the half-warp) and the lane's 8 e4m3 codes.
__device__ __forceinline__ uint2 quant8(const float (&v)[8], float *scale) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float s = div_rn(m, 448.f, __frcp_rn(448.f));  // the IEEE quotient m / 448
    uint32_t w[2] = {0u, 0u};
    if (s > 0.f) {
        // the half-warp's divisor is tested once for its 8 quotients per lane
        float q[8];
        if (div_rn_step_ok(s)) {
            const float rs = __frcp_rn(s);
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const float2 qq = div_rn_step2(make_float2(v[i], v[i + 1]), s, rs);
                q[i] = qq.x;
                q[i + 1] = qq.y;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(v[i], s);
        }
#pragma unroll
        for (int i = 0; i < 8; i += 2) {  // byte i of the 8 = value i (x of a pair in the low byte)
            const uint32_t c = __nv_cvt_float2_to_fp8x2(make_float2(q[i], q[i + 1]), __NV_SATFINITE, __NV_E4M3);
            w[i >> 2] |= c << (8 * (i & 3));
        }
    }
    *scale = s;
    return make_uint2(w[0], w[1]);
}

template <bool kQuant>
__global__ void __launch_bounds__(kThreads, 4)
    dispatch_kernel(DispatchParams p, uint8_t *xq, float *xs) {
    extern __shared__ int4 smem_v[];
    const int E = p.E, nchunk = p.nchunk, k = p.k, d = p.d;
    float *gs = reinterpret_cast<float *>(smem_v);      // [d] RMSNorm gain
    int *hist = reinterpret_cast<int *>(gs + d);        // [nchunk][E]
    int *base = hist + nchunk * E;                      // [E] this chunk's first row per expert
    int *wcnt = base + E;                               // [kWarps][E]
    int *pos_s = wcnt + kWarps * E;                     // [chunk_tokens * k]
    __shared__ int warp_sums[kWarps];
    const int c = blockIdx.x / p.replicas, rep = blockIdx.x % p.replicas;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    for (int i = tid; i < d / 4; i += kThreads)  // a layer parameter: no earlier kernel writes it
        reinterpret_cast<float4 *>(gs)[i] = __ldg(reinterpret_cast<const float4 *>(p.gain) + i);
    pdl_trigger();
    pdl_wait();
    for (int i = tid; i < nchunk * E; i += kThreads) hist[i] = p.chunk_hist[i];
    for (int i = tid; i < kWarps * E; i += kThreads) wcnt[i] = 0;
    __syncthreads();

    // 1. per-expert totals, chunk prefix, expert prefix (E <= kThreads)
    int before = 0, all = 0;
    if (tid < E) {
        for (int q = 0; q < nchunk; ++q) {
            const int v = hist[q * E + tid];
            before += q < c ? v : 0;
            all += v;
        }
    }
    int total_rows = 0, total_tiles = 0;
    const int off = block_exclusive_scan(all, E, warp_sums, &total_rows);
    const int tiles = (all + p.tile_m - 1) / p.tile_m;
    const int mt = block_exclusive_scan(tiles, E, warp_sums, &total_tiles);
    if (tid < E) {
        base[tid] = off + before;
        if (blockIdx.x == 0) {
            p.offsets[tid] = off;
            p.counts[tid] = all;
            p.mt_start[tid] = mt;
        }
    }
    if (blockIdx.x == 0 && tid == 0) {
        p.offsets[E] = total_rows;
        p.mt_start[E] = total_tiles;
    }
    if (blockIdx.x == 0 && p.sched)
        for (int i = tid; i < p.sched_n; i += kThreads) p.sched[i] = 0;
    __syncthreads();

    // 2. this chunk's assignments a = t*k + j, t in [t0, t1)
    const int t0 = c * p.chunk_tokens;
    const int t1 = min(p.N, t0 + p.chunk_tokens);
    const int a0 = t0 * k, na = max(0, (t1 - t0) * k);
    const int per_warp = (na + kWarps - 1) / kWarps;
    const int wa0 = a0 + warp * per_warp, wa1 = min(a0 + na, wa0 + per_warp);

    // pass 1: per-warp expert counts
    for (int r = wa0; r < wa1; r += 32) {
        const int a = r + lane;
        const bool act = a < wa1;
        const unsigned live = __ballot_sync(0xffffffffu, act);
        const int e = act ? p.idx[a] : -1;
        const bool ok = act && e >= 0 && e < E;
        const unsigned same = __match_any_sync(0xffffffffu, ok ? e : -1);
        if (ok && (same & live & ((1u << lane) - 1u)) == 0)  // first lane of its group
            wcnt[warp * E + e] += __popc(same & live);
        if (act && !ok) set_status(p.status, kStatusBounds);
    }
    __syncthreads();
    if (tid < E) {  // exclusive prefix over warps, from the chunk's base
        int run = base[tid];
        for (int w = 0; w < kWarps; ++w) {
            const int v = wcnt[w * E + tid];
            wcnt[w * E + tid] = run;
            run += v;
        }
    }
    __syncthreads();
    // pass 2: positions
    const int total = p.N * k;
    for (int r = wa0; r < wa1; r += 32) {
        const int a = r + lane;
        const bool act = a < wa1;
        const unsigned live = __ballot_sync(0xffffffffu, act);
        const int e = act ? p.idx[a] : -1;
        const bool ok = act && e >= 0 && e < E;
        const unsigned same = __match_any_sync(0xffffffffu, ok ? e : -1) & live;
        int pos = -1;
        if (ok) pos = wcnt[warp * E + e] + __popc(same & ((1u << lane) - 1u));
        __syncwarp();
        if (ok && (same & ((1u << lane) - 1u)) == 0) wcnt[warp * E + e] += __popc(same);
        __syncwarp();
        if (ok && (pos < 0 || pos >= total)) {
            set_status(p.status, kStatusBounds);
            pos = -1;
        }
        if (act) pos_s[a - a0] = ok ? pos : -1;
        if (ok && pos >= 0 && rep == 0) {
            p.perm[pos] = a;
            p.inv[a] = pos;
        }
    }
    __syncthreads();

    // 3. normalised rows. A token's row is the same for its k assignments, so
    // it is normalised (and for FP8 quantised) once and stored at each of
    // its k grouped positions. Work unit: one token x one column segment (a
    // run of 32-vector blocks), one warp per unit; the segments split each
    // row as far as needed to give every warp of the launch a unit.
    const int ntc = max(0, t1 - t0);
    const int vpr = kQuant ? d / 8 : d * p.elem_bytes / 16;  // 16-byte vectors per row
    const int nblk = (vpr + 31) / 32;
    const int warps_all = kWarps * p.replicas;
    int nseg = warps_all / max(ntc, 1);
    nseg = nseg < 1 ? 1 : nseg > nblk ? nblk : nseg;
    const int units = ntc * nseg;
    const uint4 *xv = static_cast<const uint4 *>(p.x);
    for (int u0 = rep + warp * p.replicas; u0 < units; u0 += warps_all) {
        const int tl = u0 / nseg, sg = u0 % nseg;
        const int t = t0 + tl;
        const int *dst = pos_s + tl * k;  // grouped positions of the token's k slots
        const float r = p.rinv[t];
        const uint4 *src = xv + static_cast<size_t>(t) * vpr;
        const int v_begin = (sg * nblk / nseg) * 32;
        const int v_end = min(vpr, ((sg + 1) * nblk / nseg) * 32);
        if constexpr (kQuant) {
            // bf16 input; d % 128 == 0, so each half-warp's 16 vectors (128
            // values) are one quantisation group, all in or all out of the row
            const int gpr = d / kFp8Block;
            constexpr int U = 4;
            for (int v0 = v_begin; v0 < v_end; v0 += 32 * U) {
                uint4 raw[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    raw[u] = v < v_end ? src[v] : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    const bool in = v < v_end;
                    const float *g = gs + (in ? v : 0) * 8;
                    const float4 g0 = *reinterpret_cast<const float4 *>(g);
                    const float4 g1 = *reinterpret_cast<const float4 *>(g + 4);
                    const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                    const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
                    // (x r) g per value, two values per paired multiply
                    float xnv[8];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const float2 xr = __fmul2_rn(
                            make_float2(bf16_to_f32(w[h] & 0xFFFFu), bf16_to_f32(w[h] >> 16)),
                            make_float2(r, r));
                        const float2 o = __fmul2_rn(xr, make_float2(gg[2 * h], gg[2 * h + 1]));
                        xnv[2 * h] = o.x;
                        xnv[2 * h + 1] = o.y;
                    }
                    float sc;
                    const uint2 codes = quant8(xnv, &sc);  // every lane takes part
                    if (in) {
                        for (int j = 0; j < k; ++j) {
                            const int pos = dst[j];
                            if (pos < 0) continue;
                            reinterpret_cast<uint2 *>(xq + static_cast<size_t>(pos) * d)[v] = codes;
                            if ((lane & 15) == 0) xs[static_cast<size_t>(pos) * gpr + v / 16] = sc;
                        }
                    }
                }
            }
        } else {
            const int epv = 16 / p.elem_bytes;  // elements per vector
            uint4 *xpv = static_cast<uint4 *>(p.xp);
            constexpr int U = 8;
            for (int v0 = v_begin; v0 < v_end; v0 += 32 * U) {
                uint4 raw[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < v_end) raw[u] = src[v];
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v >= v_end) continue;
                    const float *g = gs + v * epv;
                    uint4 o;
                    if (p.elem_bytes == 2) {
                        const float4 g0 = *reinterpret_cast<const float4 *>(g);
                        const float4 g1 = *reinterpret_cast<const float4 *>(g + 4);
                        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                        const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
                        uint32_t q[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(
                                bf16_to_f32(w[h] & 0xFFFFu) * r * gg[2 * h],
                                bf16_to_f32(w[h] >> 16) * r * gg[2 * h + 1]);
                            q[h] = *reinterpret_cast<uint32_t *>(&b2);
                        }
                        o = make_uint4(q[0], q[1], q[2], q[3]);
                    } else {
                        const float4 g0 = *reinterpret_cast<const float4 *>(g);
                        o = make_uint4(__float_as_uint(__uint_as_float(raw[u].x) * r * g0.x),
                                       __float_as_uint(__uint_as_float(raw[u].y) * r * g0.y),
                                       __float_as_uint(__uint_as_float(raw[u].z) * r * g0.z),
                                       __float_as_uint(__uint_as_float(raw[u].w) * r * g0.w));
                    }
                    for (int j = 0; j < k; ++j) {
                        const int pos = dst[j];
                        if (pos >= 0) xpv[static_cast<size_t>(pos) * vpr + v] = o;
                    }
                }
            }
        }
    }
}

}  // namespace

size_t dispatch_smem(int nchunk, int E, int chunk_assign, int d) {
    return (static_cast<size_t>(d) + static_cast<size_t>(nchunk) * E + E +
            static_cast<size_t>(kWarps) * E + static_cast<size_t>(chunk_assign)) * 4;
}

namespace {
template <bool kQuant>
int launch_dispatch_t(const DispatchParams &p, uint8_t *xq, float *xs, cudaStream_t s) {
    const size_t smem = dispatch_smem(p.nchunk, p.E, p.chunk_tokens * p.k, p.d);
    if (ensure_smem(dispatch_kernel<kQuant>, smem) != MOE_OK) return MOE_ERR_CUDA;
    // All CTAs resident at once: a second wave of a few CTAs would repeat the
    // whole prologue (histogram, ranking) after the first wave's copies.
    thread_local size_t last_smem = 0;
    thread_local int last_dev = -1, resident = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (smem != last_smem || dev != last_dev) {
        int per_sm = 0, n_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dispatch_kernel<kQuant>, kThreads,
                                                          smem) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        resident = per_sm * n_sm;
        last_smem = smem;
        last_dev = dev;
    }
    DispatchParams q = p;
    const int fit = resident / p.nchunk;
    q.replicas = fit < 1 ? 1 : fit < p.replicas ? fit : p.replicas;
    return launch_k(dispatch_kernel<kQuant>, dim3(q.nchunk * q.replicas), dim3(kThreads), smem, s,
                    q, xq, xs);
}
}  // namespace

int launch_dispatch(const DispatchParams &p, cudaStream_t s) {
    return launch_dispatch_t<false>(p, nullptr, nullptr, s);
}

int launch_dispatch_fp8(const DispatchParams &p, uint8_t *xq, float *xs, cudaStream_t s) {
    return launch_dispatch_t<true>(p, xq, xs, s);
}

}  // namespace moe
