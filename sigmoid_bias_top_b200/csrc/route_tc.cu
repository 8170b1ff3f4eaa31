// route_tc.cu -- the fp32 router of bf16 batches on the tensor cores.
//
// "LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV Caches"
// (flozi.net, English page), section "The router has two different scores":
// E logits per token from the fp32 router matrix applied to the normalised
// row, a sigmoid per logit, the stored bias added only for the top-k choice,
// and mixture weights from the selected unbiased scores over (their sum +
// eps) times the routed scale. The RMSNorm gain is folded into the router
// matrix (W' = W_r * gain, column-wise) and 1/rms scales each token's dot
// products, as in the SIMT router.
//
// Exactness of the fp32 dot products on bf16 tensor cores: the rows of x are
// bf16 and enter the MMA exactly. W' (fp32) is split once, at context
// creation, into three bf16 matrices W' = B1 + B2 + B3 + r with
// B1 = bf16(W'), B2 = bf16(W' - B1), B3 = bf16(W' - B1 - B2) (each
// difference exact in fp32 by Sterbenz), |r| <= 2^-24 |W'| or so. A product
// of two bf16 numbers is exact in fp32, so one M128 x N(3E) MMA over K = d
// with fp32 accumulation gives D1, D2, D3 = x . B1, x . B2, x . B3, and
// l_e = rinv * (D1_e + (D2_e + D3_e)) carries only fp32 accumulation
// rounding, the same order of error as the SIMT fp32 dot product.
//
// One CTA per 128 tokens, or a cluster of four or two splitting K when the
// clusters fit in one wave (each takes its share of the stages; the others
// leave their partial dot products and sums of squares in shared memory, the
// first reads them through DSMEM after a cluster barrier and adds them in
// rank order).
// Per CTA (192 threads): warp 0 issues the TMA loads of the
// x tile (128 rows x 64) and of [B1; B2; B3] (3E rows x 64) per stage; warp 1
// allocates TMEM and issues tcgen05.mma; warps 2..5 (thread = token = TMEM
// lane) sum the squares of their token's row from each shared-memory stage
// while the MMA runs (the stage is freed once the MMA and the four warps are
// done with it), then read the 3E accumulator columns of their token and
// leave the partial dot products in shared memory. In the first CTA the same
// threads add the cluster's partials (rank order), form the logits, compute
// the sigmoids eight experts at a time and select the top k in k rounds of
// arg-max over the keys in shared memory (ties keep the lower index), then
// write the weights and the expert counts of the token's dispatch chunk.
// All waits are bounded (1 s) and report MOE_ERR_DEVICE_TIMEOUT.
#include <cooperative_groups.h>

#include "moe_internal.cuh"

namespace cg = cooperative_groups;

namespace moe {
namespace {

constexpr int TM = 128;  // tokens per CTA = MMA M
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int kMaxStages = 5;  // stages in use: as many as shared memory holds
constexpr int X_BYTES = TM * BK * 2;  // 16 KB
constexpr int TMEM_COLS = 256;
constexpr int kThreads = 192;
constexpr int kHistChunks = TM / 32 + 1;  // dispatch chunks (multiples of 32 tokens) a tile meets
constexpr uint64_t kWaitNs = 1000000000ull;

struct Ctl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, Ctl *ctl, int *status) {
    if (mbar_try_wait(bar, parity)) return true;
    if (mbar_wait(bar, parity, globaltimer_ns() + kWaitNs)) return true;
    set_status(status, kStatusTimeout);
    atomicExch(&ctl->abort, 1);
    return false;
}

__device__ __forceinline__ bool aborted(Ctl *ctl) {
    return *reinterpret_cast<volatile int *>(&ctl->abort) != 0;
}


template <int KS>
__global__ void __launch_bounds__(kThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                    const __grid_constant__ CUtensorMap tmW, RouteParams p, int ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int E = p.E, NB = 3 * E;
    const int stage_bytes = X_BYTES + NB * BK * 2;  // a multiple of 1024 (E % 16 == 0)
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + ns * stage_bytes);
    int *hist = reinterpret_cast<int *>(ctl + 1);  // [kHistChunks][E]
    float *bias_s = reinterpret_cast<float *>(hist + kHistChunks * E);  // [E]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // KS CTAs (a cluster) share one 128-token tile, CTA `rank` taking the
    // K stages [kb0, kb1); rank 0 adds the others' partial sums and selects
    const int rank = KS > 1 ? static_cast<int>(cg::this_cluster().block_rank()) : 0;
    const int t0 = (blockIdx.x / KS) * TM;
    if (threadIdx.x == 0) {
        for (int s = 0; s < ns; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1 + 4);  // the MMA commit and the four epilogue warps
        }
        mbar_init(&ctl->tfull, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i < kHistChunks * E; i += kThreads) hist[i] = 0;
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
    }
    pdl_trigger();
    // x may be the output of the previous kernel, and the histogram and the
    // routing buffers are read (and the histogram cleared) by the previous
    // forward's last kernels
    pdl_wait();
    for (int i = threadIdx.x; i < E; i += kThreads) bias_s[i] = p.bias[i];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    const int nk_all = p.d / BK;
    const int kb0 = rank * nk_all / KS, kb1 = (rank + 1) * nk_all / KS;
    const int nk = kb1 - kb0;  // stages of this CTA (may be 0 for tiny d)

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_parity[kMaxStages];
            bool issued[kMaxStages];
            for (int i = 0; i < kMaxStages; ++i) issued[i] = false;
            for (int kb = 0; kb < nk && !aborted(ctl); ++kb) {
                if (!wait_bar(&ctl->empty[s], ph ^ 1u, ctl, p.status)) break;
                uint8_t *sx = smem + s * stage_bytes;
                mbar_arrive_expect_tx(&ctl->full[s], static_cast<uint32_t>(stage_bytes));
                tma_load_2d(sx, &tmX, (kb0 + kb) * BK, t0, &ctl->full[s]);
                tma_load_2d(sx + X_BYTES, &tmW, (kb0 + kb) * BK, 0, &ctl->full[s]);
                issued[s] = true;
                issued_parity[s] = ph;
                if (++s == ns) { s = 0; ph ^= 1u; }
            }
            if (aborted(ctl)) {  // let our own copies land before the CTA exits
                const uint64_t dl = globaltimer_ns() + kWaitNs;
                for (int i = 0; i < ns; ++i)
                    if (issued[i]) mbar_wait(&ctl->full[i], issued_parity[i], dl);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            const uint32_t idesc = idesc_bf16_f32(TM, NB);
            int s = 0;
            uint32_t ph = 0;
            for (int kb = 0; kb < nk; ++kb) {
                if (!wait_bar(&ctl->full[s], ph, ctl, p.status)) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * stage_bytes);
                const uint32_t b0 = a0 + X_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / UK; ++kk)
                    umma_bf16(tmem_base, sw128_kmajor_desc(a0 + kk * UK * 2),
                              sw128_kmajor_desc(b0 + kk * UK * 2), idesc, (kb | kk) != 0 ? 1u : 0u);
                umma_commit(&ctl->empty[s]);
                if (++s == ns) { s = 0; ph ^= 1u; }
            }
            // publishes the partial sums (at once if this CTA had no stages);
            // waited for here too, before TMEM is freed
            umma_commit(&ctl->tfull);
            mbar_wait(&ctl->tfull, 0, globaltimer_ns() + kWaitNs);
        }
    } else {
        // ---------------- squares, then logits and selection (warps 2..5) ----------------
        const int q = warp & 3;      // TMEM lane quarter of this warp
        const int r = q * 32 + lane;  // tile row = token
        float ss0 = 0.f, ss1 = 0.f;
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
            if (!wait_bar(&ctl->full[s], ph, ctl, p.status)) { ok = false; break; }
            // the 128-byte row of this token (its 16-byte pieces are permuted
            // by the swizzle, which does not change their sum of squares);
            // lane l starts at piece l mod 8, so a warp's loads spread over
            // all banks instead of the rows' common four
            const uint4 *row = reinterpret_cast<const uint4 *>(smem + s * stage_bytes + r * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 u = row[(c + lane) & 7];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float a = bf16_to_f32(w[h] & 0xFFFFu), b = bf16_to_f32(w[h] >> 16);
                    ss0 = fmaf(a, a, ss0);
                    ss1 = fmaf(b, b, ss1);
                }
            }
            // the reads must have completed (their values consumed) before
            // the stage is released to the next TMA write (async proxy)
            asm volatile("" ::"f"(ss0), "f"(ss1) : "memory");
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->empty[s]);
            if (++s == ns) { s = 0; ph ^= 1u; }
        }
        // this CTA's partial dot products x . W'_e ([e][row]) and partial sum
        // of squares ([row]) go to the stage memory, idle once all four
        // epilogue warps have read their last rows of x (named barrier 1,
        // reached by every epilogue thread, also after a time-out) and the
        // MMAs are done (tfull)
        asm volatile("bar.sync 1, 128;" ::: "memory");
        float *part = reinterpret_cast<float *>(smem);
        float *ssp = part + E * TM;
        const bool have = ok && wait_bar(&ctl->tfull, 0, ctl, p.status);
        if (have) tc_fence_after();
        const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
        for (int c0 = 0; c0 < E; c0 += 8) {  // E % 16 == 0
            uint32_t d1[8], d2[8], d3[8];
            if (have && nk > 0) {
                tmem_ld_32x32b_x8(t_lane + c0, d1);
                tmem_ld_32x32b_x8(t_lane + E + c0, d2);
                tmem_ld_32x32b_x8(t_lane + 2 * E + c0, d3);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) d1[j] = d2[j] = d3[j] = 0u;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                part[(c0 + j) * TM + r] =
                    __uint_as_float(d1[j]) + (__uint_as_float(d2[j]) + __uint_as_float(d3[j]));
        }
        ssp[r] = ss0 + ss1;
    }

    // the partial sums of every CTA of the cluster are in place
    tc_fence_before();
    if (KS > 1) cg::this_cluster().sync(); else __syncthreads();

    if (warp >= 2 && rank == 0) {
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const size_t t = static_cast<size_t>(t0) + r;
        float *part = reinterpret_cast<float *>(smem);
        float *ssp = part + E * TM;
        float ss = ssp[r];
        for (int h = 1; h < KS; ++h) ss += cg::this_cluster().map_shared_rank(ssp, h)[r];
        const float rinv = 1.0f / sqrtf(ss / static_cast<float>(p.d) + p.eps);
        // sigmoid scores in place of the partials and the biased-score keys
        // beside them, eight experts at a time (independent exp / divide
        // chains)
        float *sc = part;
        uint32_t *kk = reinterpret_cast<uint32_t *>(
            smem + ((static_cast<size_t>(E) * TM * 4 + TM * 4 + 1023) & ~size_t(1023)));  // [E][TM]
#pragma unroll 1
        for (int c0 = 0; c0 < E; c0 += 8) {
            float dsum[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) dsum[j] = part[(c0 + j) * TM + r];
            for (int h = 1; h < KS; ++h) {
                const float *peer = cg::this_cluster().map_shared_rank(part, h);
#pragma unroll
                for (int j = 0; j < 8; ++j) dsum[j] += peer[(c0 + j) * TM + r];
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float sg = 1.0f / (1.0f + expf(-rinv * dsum[j]));
                const float cb = sg + bias_s[c0 + j];
                sc[(c0 + j) * TM + r] = sg;
                kk[(c0 + j) * TM + r] = (cb == cb) ? float_key(cb) : 1u;  // NaN ranks lowest
            }
        }
        // k rounds of arg-max over the keys (0 = taken): eight partial maxima
        // over the experts e = u mod 8 in ascending order (strictly greater
        // keeps the lower expert), combined by larger key, then lower expert
        int se[kMaxTopK];
        float sv[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            se[j] = 0;
            sv[j] = 0.f;
            if (j < p.k) {
                uint32_t bk[8];
                int be[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) { bk[u] = 0u; be[u] = E; }
#pragma unroll 2
                for (int e0 = 0; e0 < E; e0 += 8) {
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const uint32_t v = kk[(e0 + u) * TM + r];
                        if (v > bk[u]) { bk[u] = v; be[u] = e0 + u; }
                    }
                }
                uint32_t K = bk[0];
                int B = be[0];
#pragma unroll
                for (int u = 1; u < 8; ++u)
                    if (bk[u] > K || (bk[u] == K && be[u] < B)) { K = bk[u]; B = be[u]; }
                // k <= E: an untaken expert remains, so B < E
                se[j] = B;
                sv[j] = sc[B * TM + r];
                kk[B * TM + r] = 0u;
            }
        }
        if (t < static_cast<size_t>(p.N)) {
            p.rinv[t] = rinv;
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j)
                if (j < p.k) sum += sv[j];
            const float den = sum + p.eps;
            const int hc = static_cast<int>(t / p.chunk_tokens) - t0 / p.chunk_tokens;
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                if (j < p.k) {
                    p.idx[t * p.k + j] = se[j];
                    p.wts[t * p.k + j] = p.scale * (sv[j] / den);
                    atomicAdd(&hist[hc * E + se[j]], 1);
                }
            }
        }
    }

    // the other CTAs keep their partial sums until rank 0 has read them
    if (KS > 1) cg::this_cluster().sync();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
    // the tile's expert counts, per dispatch chunk
    const int c_first = t0 / p.chunk_tokens;
    for (int i = threadIdx.x; i < kHistChunks * E; i += kThreads) {
        const int hc = i / E, e = i - hc * E;
        if (hist[i]) atomicAdd(&p.chunk_hist[static_cast<size_t>(c_first + hc) * E + e], hist[i]);
    }
}

__global__ void split_router_kernel(const float *wg, __nv_bfloat16 *w3, int E, int d) {
    const size_t n = static_cast<size_t>(E) * d;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const float w = wg[i];
        const __nv_bfloat16 b1 = __float2bfloat16_rn(w);
        const float r1 = w - __bfloat162float(b1);
        const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(b2);
        w3[i] = b1;
        w3[n + i] = b2;
        w3[2 * n + i] = __float2bfloat16_rn(r2);
    }
}

size_t smem_bytes(int E, int ns) {
    return 1024 + ns * (X_BYTES + static_cast<size_t>(3 * E) * BK * 2) + sizeof(Ctl) +
           (kHistChunks + 1) * static_cast<size_t>(E) * 4;
}

constexpr size_t kSmemCap = 227 * 1024;

int stages_for(int E) {
    int ns = kMaxStages;
    while (ns > 2 && smem_bytes(E, ns) > kSmemCap) --ns;
    return ns;
}

}  // namespace

bool route_tc_ok(int d, int E) {
    return E % 16 == 0 && 3 * E <= 240 && d % BK == 0 && smem_bytes(E, stages_for(E)) <= kSmemCap;
}

int launch_split_router(const float *wg, void *w3, int E, int d, cudaStream_t s) {
    split_router_kernel<<<256, 256, 0, s>>>(wg, static_cast<__nv_bfloat16 *>(w3), E, d);
    return cudaPeekAtLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <int KS>
int launch_ks(const CUtensorMap &xm, const CUtensorMap &w3_map, const RouteParams &p, int ns,
              size_t smem, int tiles, cudaStream_t s) {
    auto kern = route_tc_kernel<KS>;
    if (ensure_smem(kern, smem) != MOE_OK) return MOE_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(KS * tiles);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = KS;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = KS > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, xm, w3_map, p, ns) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_route_tc(const RouteParams &p, const CUtensorMap &w3_map, cudaStream_t s) {
    if (p.N <= 0) return MOE_OK;
    if (p.chunk_tokens % 32 != 0) return MOE_ERR_INVALID_ARG;
    CUtensorMap xm;
    int rc = tc_encode_2d(&xm, p.x, static_cast<uint64_t>(p.N), static_cast<uint64_t>(p.d), TM);
    if (rc != MOE_OK) return rc;
    const int ns = stages_for(p.E);
    const size_t smem = smem_bytes(p.E, ns);
    thread_local int n_sm = 0, n_sm_dev = -1;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev != n_sm_dev) {
        if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        n_sm_dev = dev;
    }
    // split K over a cluster of 4 or 2 CTAs while the clusters still fit in
    // one wave (one CTA per SM): the per-CTA pipeline latency, not bandwidth,
    // bounds this kernel
    const int tiles = (p.N + TM - 1) / TM;
    if (4 * tiles <= n_sm) return launch_ks<4>(xm, w3_map, p, ns, smem, tiles, s);
    if (2 * tiles <= n_sm) return launch_ks<2>(xm, w3_map, p, ns, smem, tiles, s);
    return launch_ks<1>(xm, w3_map, p, ns, smem, tiles, s);
}

}  // namespace moe
