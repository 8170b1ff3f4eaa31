// moe_api.cu -- the C ABI declared in include/moe.h: argument validation,
// workspace ownership, TMA descriptor set-up and the launch sequence of one
// forward of the sigmoid-bias top-k MoE block.
//
// Launch sequence (all on the caller's stream, no host synchronisation):
//   1 route     RMSNorm + fp32 router + sigmoid + biased top-k + weights, and the
//               per-chunk expert histogram (SIMT fp32; for bf16 batches of 512
//               tokens and more the router GEMM runs on the tensor cores with
//               the router matrix split into three bf16 parts)
//   2 dispatch  per-expert counts, offsets, row-tile prefix, perm / inv
//   3 gate_up   grouped GEMM over the grouped normalised rows, SiLU(gate)*up
//               (tcgen05 for bf16: tiles of 256 weight rows x up to 256
//               tokens on CTA pairs, or with MOE_TC_PAIR=0 128-token tiles on
//               single CTAs; SIMT for fp32)
//   4 down      grouped GEMM
// (bf16 batches of at most 32 rows per expert on average fuse 3 and 4 into one
// persistent kernel. FP8_BLOCK layers always do: their dispatch writes e4m3
// rows with group scales and one persistent kernel runs both contractions.)
//   5 combine   out = x + sum_j w_j y_j in fixed slot order
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <unordered_map>
#include <vector>

#include "moe_fp8.cuh"

using namespace moe;

namespace {
constexpr int kEvPerFwd = 8;     // event marks per forward (launches + 1, rounded up)
constexpr int kRingForwards = 1024;
}

struct moe_ctx {
    int d, E, I, k, dtype, max_tokens, device, n_sm;
    int xdtype;   // storage type of x and out: bf16 for FP8_BLOCK layers, else dtype
    float eps, scale;
    moe_weights w;
    size_t elem;  // bytes per element of x / out

    // FP8_BLOCK layers: e4m3 rows and group scales (carved from xp and act)
    bool fp8;
    void *fp8_maps;
    void *fp8_pair_maps; // the CTA-pair FP8 GEMMs of large batches
    int fp8_pair_mode;   // -1 above the small-batch load, 0 never, 1 whenever not small
    uint8_t *xq, *aq;
    float *xs, *as;
    float *a32;          // CTA-pair path: SiLU(gate)*up in fp32 [rows_cap][I] before quantisation

    void *ws;  // one allocation, carved below
    void *xp, *act, *y, *x_stage, *out_stage;
    int32_t *idx, *chunk_hist, *counts, *offsets, *mt_start, *perm, *inv;
    float *wts, *router_wt, *router_wg, *rinv;
    void *router_w3;     // bf16 [3E][d]: W' split into three bf16 matrices (tensor-core router)
    CUtensorMap w3_map;  // its TMA map (box 64 x 3E)
    bool route_tc;       // the tensor-core router is available (bf16, E % 16 == 0, 3E <= 240)
    int route_tc_mode;   // -1 by batch size, 0 never, 1 whenever available
    int *status;
    int rows_cap, e_pad, max_chunks;

    TcMaps maps;
    void *decode_maps;   // tensor maps of the fused small-batch kernel
    int32_t *sched;      // [1 + E] its work counter and per-expert completion counts
    bool use_tc;
    int pair_mode;       // CTA-pair GEMMs: 0 never, else (default) whenever not fused

    int last_n;
    bool last_fused;  // the last forward used the fused small-batch expert kernel
    bool last_fp8_pair;  // ... or the CTA-pair FP8 GEMMs with their quantiser between

    // profiling: a ring of event sets, one set (kEvPerFwd events) per forward
    bool profile;
    std::vector<cudaEvent_t> ring;
    long long head, pending_from;  // forwards recorded / first not yet accumulated
    int n_kernels;
    double sum_ms[kEvPerFwd];
    long long n_fwd;
};

static const char *kKernelNames[] = {"route", "dispatch", "gate_up", "down", "combine"};
static const char *kFusedKernelNames[] = {"route", "dispatch", "experts", "combine"};
static const char *kFp8PairKernelNames[] = {"route", "dispatch", "gate_up", "quantize", "down",
                                            "combine"};

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int moe::ensure_smem_ptr(const void *kern, size_t smem) {
    static std::mutex mu;
    static std::unordered_map<const void *, size_t> set;  // per process (one device each)
    if (smem <= 48 * 1024) return MOE_OK;
    std::lock_guard<std::mutex> lock(mu);
    size_t &cur = set[kern];
    if (smem <= cur) return MOE_OK;
    const cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(smem));
    if (err != cudaSuccess) {
        if (getenv("MOE_DEBUG"))
            fprintf(stderr, "moe: shared memory of %zu bytes refused: %s\n", smem,
                    cudaGetErrorString(err));
        return MOE_ERR_CUDA;
    }
    cur = smem;
    return MOE_OK;
}

extern "C" const char *moe_strerror(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case MOE_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case MOE_ERR_TOO_MANY_TOKENS: return "n_tokens exceeds max_tokens";
        case MOE_ERR_OOM: return "device allocation failed";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case MOE_ERR_DEVICE_BOUNDS: return "device-side index out of bounds";
        case MOE_ERR_NO_DEVICE: return "no sm_100 CUDA device";
        default: return "unknown error";
    }
}

static int check_shapes(int d, int E, int I, int k, int dtype, int max_tokens) {
    if (dtype != MOE_F32 && dtype != MOE_BF16 && dtype != MOE_FP8_BLOCK) return MOE_ERR_INVALID_ARG;
    if (d <= 0 || E <= 0 || I <= 0 || k <= 0 || max_tokens <= 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (E > kMaxExperts || k > kMaxTopK || k > E) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (d % 4 != 0 || d > 32768) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (dtype == MOE_BF16 && (d % 64 != 0 || I % 64 != 0)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (dtype == MOE_FP8_BLOCK && (d % kFp8Block != 0 || I % kFp8Block != 0))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    // 32-bit row indices and TMA coordinates
    if (static_cast<long long>(max_tokens) * k >= (1LL << 30)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(E) * 2 * I >= (1LL << 30) ||
        static_cast<long long>(E) * d >= (1LL << 30))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

extern "C" int moe_create(int d, int n_experts, int d_ff, int top_k, float eps,
                          const moe_weights *w, int max_tokens, moe_ctx **out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!w) return MOE_ERR_INVALID_ARG;
    int rc = check_shapes(d, n_experts, d_ff, top_k, w->dtype, max_tokens);
    if (rc != MOE_OK) return rc;
    if (!w->norm_gain || !w->router_w || !w->expert_bias || !w->w_gate_up || !w->w_down)
        return MOE_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !(w->routed_scale == w->routed_scale)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w->norm_gain) || !aligned16(w->router_w) || !aligned16(w->w_gate_up) ||
        !aligned16(w->w_down))
        return MOE_ERR_ALIGNMENT;
    if (w->dtype == MOE_FP8_BLOCK) {
        if (!w->w_gate_up_scale || !w->w_down_scale) return MOE_ERR_INVALID_ARG;
        if (!aligned16(w->w_gate_up_scale) || !aligned16(w->w_down_scale)) return MOE_ERR_ALIGNMENT;
    }

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_NO_DEVICE;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_NO_DEVICE;
    if (prop.major != 10) return MOE_ERR_NO_DEVICE;

    moe_ctx *h = new (std::nothrow) moe_ctx();
    if (!h) return MOE_ERR_OOM;
    h->d = d; h->E = n_experts; h->I = d_ff; h->k = top_k; h->dtype = w->dtype;
    h->max_tokens = max_tokens; h->device = dev; h->n_sm = prop.multiProcessorCount;
    h->eps = eps; h->scale = w->routed_scale; h->w = *w;
    h->fp8 = (w->dtype == MOE_FP8_BLOCK);
    h->xdtype = h->fp8 ? MOE_BF16 : w->dtype;
    h->elem = (h->xdtype == MOE_F32) ? 4 : 2;
    h->use_tc = (w->dtype == MOE_BF16);
    h->rows_cap = max_tokens * top_k;
    {
        // MOE_TC_PAIR=0 / 1 overrides the choice between the single-CTA and
        // the CTA-pair grouped GEMMs (both compute the same result).
        const char *e = getenv("MOE_TC_PAIR");
        h->pair_mode = (e && e[0] == '0') ? 0 : (e && e[0] == '1') ? 1 : -1;
        // MOE_ROUTE_TC=0 / 1 likewise for the tensor-core and the SIMT routers
        e = getenv("MOE_ROUTE_TC");
        h->route_tc_mode = (e && e[0] == '0') ? 0 : (e && e[0] == '1') ? 1 : -1;
        // MOE_FP8_PAIR=0 keeps FP8_BLOCK batches of every size on the persistent
        // kernel instead of the CTA-pair GEMMs (both compute the same result)
        e = getenv("MOE_FP8_PAIR");
        h->fp8_pair_mode = (e && e[0] == '0') ? 0 : -1;
    }
    h->route_tc = (h->use_tc || h->fp8) && route_tc_ok(d, n_experts);

    h->e_pad = (n_experts + 63) / 64 * 64;
    h->max_chunks = max_dispatch_chunks(n_experts);

    // workspace layout (every block 256-byte aligned)
    const size_t N = max_tokens, R = h->rows_cap, E = n_experts;
    const size_t sizes[] = {
        R * d * h->elem,                      // xp
        R * d_ff * h->elem,                   // act
        R * d * h->elem,                      // y
        N * d * h->elem,                      // x_stage
        N * d * h->elem,                      // out_stage
        N * top_k * 4,                        // idx
        static_cast<size_t>(h->max_chunks) * E * 4,  // chunk_hist
        E * 4,                                // counts
        (E + 1) * 4,                          // offsets
        (E + 1) * 4,                          // mt_start
        R * 4,                                // perm
        R * 4,                                // inv
        N * top_k * 4,                        // wts
        static_cast<size_t>(d) * h->e_pad * 4,  // router_wt
        N * 4,                                // rinv
        E * static_cast<size_t>(d) * 4,       // router_wg
        (E + 1) * 4,                          // sched
        256,                                  // status
        3 * E * static_cast<size_t>(d) * 2,   // router_w3
        (h->fp8 && h->fp8_pair_mode != 0) ? R * d_ff * 4 : 0,  // a32
    };
    const int nblocks = sizeof(sizes) / sizeof(sizes[0]);
    size_t total = 0, off[20];
    for (int i = 0; i < nblocks; ++i) {
        off[i] = total;
        total += (sizes[i] + 255) & ~static_cast<size_t>(255);
    }
    if (getenv("MOE_TEST_FAIL_ALLOC") != nullptr ||
        cudaMalloc(&h->ws, total) != cudaSuccess) {
        cudaGetLastError();
        delete h;
        return MOE_ERR_OOM;
    }
    uint8_t *b = static_cast<uint8_t *>(h->ws);
    h->xp = b + off[0]; h->act = b + off[1]; h->y = b + off[2];
    h->x_stage = b + off[3]; h->out_stage = b + off[4];
    h->idx = reinterpret_cast<int32_t *>(b + off[5]);
    h->chunk_hist = reinterpret_cast<int32_t *>(b + off[6]);
    h->counts = reinterpret_cast<int32_t *>(b + off[7]);
    h->offsets = reinterpret_cast<int32_t *>(b + off[8]);
    h->mt_start = reinterpret_cast<int32_t *>(b + off[9]);
    h->perm = reinterpret_cast<int32_t *>(b + off[10]);
    h->inv = reinterpret_cast<int32_t *>(b + off[11]);
    h->wts = reinterpret_cast<float *>(b + off[12]);
    h->router_wt = reinterpret_cast<float *>(b + off[13]);
    h->rinv = reinterpret_cast<float *>(b + off[14]);
    h->router_wg = reinterpret_cast<float *>(b + off[15]);
    h->sched = reinterpret_cast<int32_t *>(b + off[16]);
    h->status = reinterpret_cast<int *>(b + off[17]);
    h->router_w3 = b + off[18];
    h->a32 = reinterpret_cast<float *>(b + off[19]);
    if (h->fp8) {  // codes then scales, inside the (2-byte element) xp and act blocks
        h->xq = static_cast<uint8_t *>(h->xp);
        h->xs = reinterpret_cast<float *>(h->xq + R * d);
        h->aq = static_cast<uint8_t *>(h->act);
        h->as = reinterpret_cast<float *>(h->aq + R * d_ff);
    }
    if (cudaMemset(h->ws, 0, total) != cudaSuccess) {
        cudaFree(h->ws);
        delete h;
        return MOE_ERR_CUDA;
    }
    if (launch_prepare_router(w->router_w, w->norm_gain, h->router_wg, h->router_wt, n_experts,
                              h->e_pad, d, 0) != MOE_OK ||
        (h->route_tc && launch_split_router(h->router_wg, h->router_w3, n_experts, d, 0) != MOE_OK) ||
        cudaDeviceSynchronize() != cudaSuccess) {
        cudaFree(h->ws);
        delete h;
        return MOE_ERR_CUDA;
    }
    if (h->use_tc) {
        rc = tc_build_maps(&h->maps, h->xp, h->act, w->w_gate_up, w->w_down, h->rows_cap,
                           n_experts, d, d_ff);
        if (rc == MOE_OK)
            rc = decode_build_maps(&h->decode_maps, h->xp, h->act, w->w_gate_up, w->w_down,
                                   h->rows_cap, n_experts, d, d_ff);
        if (rc == MOE_OK && h->route_tc)
            rc = tc_encode_2d(&h->w3_map, h->router_w3, 3 * static_cast<uint64_t>(n_experts), d,
                              3 * n_experts);
        if (rc != MOE_OK) {
            if (h->decode_maps) decode_free_maps(h->decode_maps);
            cudaFree(h->ws);
            delete h;
            return rc;
        }
    }
    if (h->fp8) {
        rc = fp8_build_maps(&h->fp8_maps, h->xq, h->aq, w->w_gate_up, w->w_down, h->rows_cap,
                            n_experts, d, d_ff);
        if (rc == MOE_OK)
            rc = fp8_pair_build_maps(&h->fp8_pair_maps, h->xq, h->aq, w->w_gate_up, w->w_down,
                                     h->rows_cap, n_experts, d, d_ff);
        if (rc == MOE_OK && h->route_tc)
            rc = tc_encode_2d(&h->w3_map, h->router_w3, 3 * static_cast<uint64_t>(n_experts), d,
                              3 * n_experts);
        if (rc != MOE_OK) {
            if (h->fp8_maps) fp8_free_maps(h->fp8_maps);
            if (h->fp8_pair_maps) fp8_pair_free_maps(h->fp8_pair_maps);
            cudaFree(h->ws);
            delete h;
            return rc;
        }
    }
    *out = h;
    return MOE_OK;
}

// The fused small-batch expert kernel (both contractions in one persistent
// launch) serves bf16 layers while the mean load stays at or below
// kDecodeRowsPerExpert grouped rows per expert; larger batches use the two
// row-tiled grouped GEMMs.
static bool small_batch(const moe_ctx *h, int N) {
    return static_cast<long long>(N) * h->k <= static_cast<long long>(kDecodeRowsPerExpert) * h->E;
}

// FP8_BLOCK layers above the small-batch load run the two CTA-pair FP8 GEMMs
// (token tiles up to 128, K blocks promoted per tile); below it, and with
// MOE_FP8_PAIR=0, the persistent FP8 kernel takes both contractions.
static bool use_fp8_pair(const moe_ctx *h, int N) {
    return h->fp8 && h->fp8_pair_mode != 0 && !small_batch(h, N);
}

static bool use_fused_experts(const moe_ctx *h, int N) {
    if (h->fp8) return !use_fp8_pair(h, N);
    return h->use_tc && small_batch(h, N);
}

// The tensor-core router (bf16 batches) from kRouteTcMinTokens tokens on; the
// SIMT routers below that.
constexpr int kRouteTcMinTokens = 512;
static bool use_route_tc(const moe_ctx *h, int N) {
    if (!h->route_tc || h->route_tc_mode == 0) return false;
    return h->route_tc_mode == 1 || N >= kRouteTcMinTokens;
}

// bf16 GEMMs on CTA pairs (256 weight rows x up to 256 tokens) for every
// batch the fused expert kernel does not take. Their token tiles pad each
// expert's rows to 16, where the single-CTA GEMMs pad them to a 128-row M
// tile, so the pairs are as fast or faster at every batch size measured
// (640 to 8192 tokens at E = 64, k = 4: 1% at 640, 17% at 3072); the
// single-CTA GEMMs stay behind MOE_TC_PAIR=0 as an independent second path.
static bool use_pair_gemms(const moe_ctx *h) {
    return h->use_tc && h->pair_mode != 0;
}

// Adds the durations of up to `count` (all if < 0) recorded forwards, oldest
// first, to the per-kernel sums.
static int accumulate(moe_ctx *h, long long count) {
    while (h->pending_from < h->head && count-- != 0) {
        cudaEvent_t *ev = &h->ring[static_cast<size_t>(h->pending_from % kRingForwards) * kEvPerFwd];
        if (cudaEventSynchronize(ev[h->n_kernels]) != cudaSuccess) return MOE_ERR_CUDA;
        for (int i = 0; i < h->n_kernels; ++i) {
            float ms = 0.f;
            if (cudaEventElapsedTime(&ms, ev[i], ev[i + 1]) != cudaSuccess) return MOE_ERR_CUDA;
            h->sum_ms[i] += ms;
        }
        h->n_fwd++;
        h->pending_from++;
    }
    return MOE_OK;
}

static void free_ring(moe_ctx *h) {
    for (cudaEvent_t e : h->ring) cudaEventDestroy(e);
    h->ring.clear();
}

static int forward_impl(moe_ctx *h, const void *x, void *out, int N, cudaStream_t s) {
    int rc;
    const bool prof = h->profile;
    int ne = 0;
    cudaEvent_t *ev = nullptr;
    if (prof) {
        if (h->head - h->pending_from >= kRingForwards && (rc = accumulate(h, 1)) != MOE_OK)
            return rc;
        ev = &h->ring[static_cast<size_t>(h->head % kRingForwards) * kEvPerFwd];
    }
#define MOE_MARK()                                                          \
    do {                                                                    \
        if (prof && cudaEventRecord(ev[ne++], s) != cudaSuccess) return MOE_ERR_CUDA; \
    } while (0)
#define MOE_TRY(expr)                     \
    do {                                  \
        if ((rc = (expr)) != MOE_OK) return rc; \
    } while (0)

    int tt = 0;
    const int kind = route_plan(N, h->d, h->E, &tt);
    int nchunk = 1, chunk_tokens = N;
    chunk_plan(N, h->k, h->max_chunks, &nchunk, &chunk_tokens);
    const bool fused = use_fused_experts(h, N);
    const bool fp8_pair = use_fp8_pair(h, N);
    const bool pair = !fused && use_pair_gemms(h);
    const int tile_m = fp8_pair ? kFp8PairTileM
                       : !h->use_tc ? kSimtTileM : pair ? kTcPairTileM : kTcTileM;

    MOE_MARK();
    RouteParams rp;
    rp.x = x; rp.gain = h->w.norm_gain; rp.router_w = h->w.router_w; rp.router_wt = h->router_wt;
    rp.router_wg = h->router_wg;
    rp.bias = h->w.expert_bias; rp.rinv = h->rinv; rp.idx = h->idx; rp.wts = h->wts;
    rp.chunk_hist = h->chunk_hist; rp.status = h->status;
    rp.N = N; rp.d = h->d; rp.E = h->E; rp.k = h->k; rp.e_pad = h->e_pad;
    rp.chunk_tokens = chunk_tokens; rp.eps = h->eps; rp.scale = h->scale;
    if (use_route_tc(h, N))
        MOE_TRY(launch_route_tc(rp, h->w3_map, s));
    else
        MOE_TRY(launch_route(rp, h->xdtype, kind, tt, s));
    MOE_MARK();

    DispatchParams dp;
    dp.idx = h->idx; dp.chunk_hist = h->chunk_hist; dp.counts = h->counts;
    dp.offsets = h->offsets; dp.mt_start = h->mt_start; dp.perm = h->perm; dp.inv = h->inv;
    dp.status = h->status; dp.x = x; dp.gain = h->w.norm_gain; dp.rinv = h->rinv; dp.xp = h->xp;
    dp.N = N; dp.d = h->d; dp.E = h->E; dp.k = h->k; dp.nchunk = nchunk;
    dp.chunk_tokens = chunk_tokens; dp.tile_m = tile_m;
    dp.elem_bytes = static_cast<int>(h->elem);
    dp.sched = fused ? h->sched : nullptr;
    dp.sched_n = h->E + 1;
    // several CTAs per chunk share the row copies: about four CTAs per SM in all
    dp.replicas = (4 * h->n_sm + nchunk - 1) / nchunk;
    if (dp.replicas > 64) dp.replicas = 64;
    if (h->fp8)
        MOE_TRY(launch_dispatch_fp8(dp, h->xq, h->xs, s));
    else
        MOE_TRY(launch_dispatch(dp, s));
    MOE_MARK();

    GroupedParams gp = {};
    gp.offsets = h->offsets; gp.mt_start = h->mt_start; gp.status = h->status;
    gp.E = h->E; gp.d = h->d; gp.I = h->I; gp.k = h->k; gp.rows_cap = h->rows_cap;
    const int max_mtiles = (N * h->k + tile_m - 1) / tile_m + h->E;

    if (fp8_pair) {
        Fp8PairParams fp;
        fp.offsets = h->offsets; fp.mt_start = h->mt_start;
        fp.sgu = h->w.w_gate_up_scale; fp.sdn = h->w.w_down_scale;
        fp.xs = h->xs; fp.as_in = h->as; fp.a32 = h->a32; fp.aq = h->aq; fp.as_out = h->as;
        fp.y = h->y; fp.status = h->status; fp.E = h->E; fp.d = h->d; fp.I = h->I;
        MOE_TRY(launch_fp8_pair_gate_up(h->fp8_pair_maps, fp, h->n_sm, s));
        MOE_MARK();
        MOE_TRY(launch_fp8_quantize_act(fp, h->n_sm, s));
        MOE_MARK();
        MOE_TRY(launch_fp8_pair_down(h->fp8_pair_maps, fp, h->n_sm, s));
        MOE_MARK();
    } else if (h->fp8) {
        Fp8ExpertParams fp;
        fp.offsets = h->offsets; fp.sgu = h->w.w_gate_up_scale; fp.sdn = h->w.w_down_scale;
        fp.xs = h->xs; fp.aq = h->aq; fp.as = h->as; fp.y = h->y; fp.sched = h->sched;
        fp.status = h->status; fp.E = h->E; fp.d = h->d; fp.I = h->I;
        // passes of 32 tokens (more TMEM buffers) while the mean load is small
        const bool small = static_cast<long long>(N) * h->k <=
                           static_cast<long long>(kDecodeRowsPerExpert) * h->E;
        MOE_TRY(launch_fp8_experts(h->fp8_maps, fp, h->n_sm, small ? 32 : 64, s));
        MOE_MARK();
    } else if (fused) {
        DecodeParams fp;
        fp.offsets = h->offsets; fp.act = h->act; fp.y = h->y; fp.sched = h->sched;
        fp.status = h->status; fp.E = h->E; fp.d = h->d; fp.I = h->I;
        MOE_TRY(launch_decode_experts(h->decode_maps, fp, h->n_sm, s));
        MOE_MARK();
    } else {
        gp.a = h->xp; gp.w = h->w.w_gate_up; gp.c = h->act;
        if (pair)
            MOE_TRY(launch_gemm_tc2_gate_up(h->maps, gp, h->n_sm, s));
        else if (h->use_tc)
            MOE_TRY(launch_gemm_tc_gate_up(h->maps, gp, h->n_sm, s));
        else
            MOE_TRY(launch_gemm_simt_gate_up(gp, max_mtiles, s));
        MOE_MARK();

        gp.a = h->act; gp.w = h->w.w_down; gp.c = h->y;
        if (pair)
            MOE_TRY(launch_gemm_tc2_down(h->maps, gp, h->n_sm, s));
        else if (h->use_tc)
            MOE_TRY(launch_gemm_tc_down(h->maps, gp, h->n_sm, s));
        else
            MOE_TRY(launch_gemm_simt_down(gp, max_mtiles, s));
        MOE_MARK();
    }

    CombineParams cp;
    cp.x = x; cp.y = h->y; cp.wts = h->wts; cp.inv = h->inv; cp.out = out; cp.status = h->status;
    cp.chunk_hist = h->chunk_hist; cp.chunk_hist_n = nchunk * h->E;
    cp.N = N; cp.d = h->d; cp.k = h->k;
    MOE_TRY(launch_combine(cp, h->xdtype, s));
    MOE_MARK();
#undef MOE_MARK
#undef MOE_TRY
    if (prof) {
        h->n_kernels = ne - 1;
        h->head++;
    }
    h->last_n = N;
    h->last_fused = fused;
    h->last_fp8_pair = fp8_pair;
    return MOE_OK;
}

static int check_call(moe_ctx *h, int n_tokens) {
    if (!h) return MOE_ERR_INVALID_ARG;
    if (n_tokens < 0) return MOE_ERR_INVALID_ARG;
    if (n_tokens > h->max_tokens) return MOE_ERR_TOO_MANY_TOKENS;
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

extern "C" int moe_forward(moe_ctx *h, const void *x, void *out, int n_tokens, void *stream) {
    int rc = check_call(h, n_tokens);
    if (rc != MOE_OK) return rc;
    if (n_tokens == 0) return MOE_OK;
    if (!x || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out)) return MOE_ERR_ALIGNMENT;
    return forward_impl(h, x, out, n_tokens, static_cast<cudaStream_t>(stream));
}

extern "C" int moe_forward_host(moe_ctx *h, const void *x_host, void *out_host, int n_tokens,
                                void *stream) {
    int rc = check_call(h, n_tokens);
    if (rc != MOE_OK) return rc;
    if (n_tokens == 0) return MOE_OK;
    if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t bytes = static_cast<size_t>(n_tokens) * h->d * h->elem;
    // Pinned (page-locked) host memory is mapped into the device's address
    // space: the last kernel then stores the rows there itself, and no copy
    // back (with its own start-up) follows. Other host memory goes through
    // the device staging buffer.
    void *out_dev = nullptr;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, out_host) == cudaSuccess) {
        if (attr.type == cudaMemoryTypeHost && attr.devicePointer && aligned16(attr.devicePointer))
            out_dev = attr.devicePointer;
    } else {
        cudaGetLastError();  // pageable memory unknown to CUDA: not an error here
    }
    if (cudaMemcpyAsync(h->x_stage, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    rc = forward_impl(h, h->x_stage, out_dev ? out_dev : h->out_stage, n_tokens, s);
    if (rc != MOE_OK) return rc;
    if (!out_dev &&
        cudaMemcpyAsync(out_host, h->out_stage, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return cudaStreamSynchronize(s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_destroy(moe_ctx *h) {
    if (!h) return MOE_OK;
    int rc = MOE_OK;
    if (cudaDeviceSynchronize() != cudaSuccess) rc = MOE_ERR_CUDA;
    free_ring(h);
    if (h->decode_maps) decode_free_maps(h->decode_maps);
    if (h->fp8_maps) fp8_free_maps(h->fp8_maps);
    if (h->fp8_pair_maps) fp8_pair_free_maps(h->fp8_pair_maps);
    if (cudaFree(h->ws) != cudaSuccess) rc = MOE_ERR_CUDA;
    delete h;
    return rc;
}

extern "C" int moe_status(moe_ctx *h) {
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

extern "C" int moe_debug_routing(moe_ctx *h, int32_t *idx, float *w, int32_t *perm,
                                 int32_t *offsets, void *stream) {
    if (!h) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t N = h->last_n, k = h->k;
    if (idx && N && cudaMemcpyAsync(idx, h->idx, N * k * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (w && N && cudaMemcpyAsync(w, h->wts, N * k * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (perm && N && cudaMemcpyAsync(perm, h->perm, N * k * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (offsets && cudaMemcpyAsync(offsets, h->offsets, (h->E + 1) * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

extern "C" int moe_debug_fp8_rows(moe_ctx *h, uint8_t *codes, float *scales, void *stream) {
    if (!h || !h->fp8) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t rows = static_cast<size_t>(h->last_n) * h->k;
    if (codes && rows &&
        cudaMemcpyAsync(codes, h->xq, rows * h->d, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (scales && rows &&
        cudaMemcpyAsync(scales, h->xs, rows * (h->d / kFp8Block) * 4, cudaMemcpyDeviceToDevice,
                        s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

extern "C" int moe_profile(moe_ctx *h, int enable) {
    if (!h) return MOE_ERR_INVALID_ARG;
    if (enable && h->ring.empty()) {
        h->ring.resize(static_cast<size_t>(kRingForwards) * kEvPerFwd);
        for (size_t i = 0; i < h->ring.size(); ++i) {
            if (cudaEventCreate(&h->ring[i]) != cudaSuccess) {
                h->ring.resize(i);
                free_ring(h);
                return MOE_ERR_CUDA;
            }
        }
    }
    h->profile = enable != 0;
    h->head = h->pending_from = h->n_fwd = 0;
    for (int i = 0; i < kEvPerFwd; ++i) h->sum_ms[i] = 0.0;
    return MOE_OK;
}

extern "C" int moe_kernel_times(moe_ctx *h, float *ms, int n) {
    if (!h || (n > 0 && !ms)) return MOE_ERR_INVALID_ARG;
    int rc = accumulate(h, -1);
    if (rc != MOE_OK) return rc;
    if (h->n_fwd == 0) return 0;
    for (int i = 0; i < h->n_kernels && i < n; ++i)
        ms[i] = static_cast<float>(h->sum_ms[i] / static_cast<double>(h->n_fwd));
    return h->n_kernels;
}

extern "C" const char *moe_kernel_name(moe_ctx *h, int i) {
    if (!h) return nullptr;
    if (h->last_fused) return (i >= 0 && i < 4) ? kFusedKernelNames[i] : nullptr;
    if (h->last_fp8_pair) return (i >= 0 && i < 6) ? kFp8PairKernelNames[i] : nullptr;
    return (i >= 0 && i < 5) ? kKernelNames[i] : nullptr;
}

extern "C" int moe_launches_per_forward(moe_ctx *h, int n_tokens) {
    if (!h) return MOE_ERR_INVALID_ARG;
    if (n_tokens <= 0) return 0;
    return use_fused_experts(h, n_tokens) ? 4 : use_fp8_pair(h, n_tokens) ? 6 : 5;
}

extern "C" int moe_selftest_timeout(moe_ctx *h, int timeout_us, void *stream) {
    if (!h || timeout_us <= 0 || timeout_us > 10000000) return MOE_ERR_INVALID_ARG;
    return launch_selftest_timeout(h->status, timeout_us, static_cast<cudaStream_t>(stream));
}
