// moe_ep.cu -- expert parallelism: the layer's experts split over ranks, one
// process per GPU. Every rank routes and dispatches its own tokens over all E
// experts, but holds the weights of one contiguous block of experts only.
//
// The page ("LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV
// Caches", flozi.net, English page, section "The router has two different
// scores") notes that dispatch, token regrouping and uneven expert loads are
// what matters once the experts are spread, and names expert parallelism as
// the way the layer is deployed at scale; it describes no implementation.
//
// One forward on a rank (the exchange between the phases is the caller's,
// e.g. NCCL grouped send/recv through torch.distributed):
//   moe_ep_dispatch  route + dispatch over all E experts: the grouped
//                    normalised rows go to the send buffer (expert-major,
//                    token order within an expert, so the rows bound for one
//                    rank's experts are contiguous); the per-expert counts are
//                    copied to the host (the exchange sizes come from them).
//   (exchange)       rows of this rank's experts arrive in the receive
//                    buffer, expert-major, source-rank order within an expert.
//   moe_ep_experts   gate/up + SiLU*up and down of the local experts over the
//                    received rows (the same grouped kernels as moe_forward),
//                    outputs into the send-back buffer in the received order.
//   (exchange)       each output row returns to the rank and grouped position
//                    its input row came from.
//   moe_ep_combine   out = x + sum_j w_j y_j in slot order, as moe_forward.
// No kernel here reads another GPU's memory; all transfers are the caller's.
#include <stdlib.h>
#include <string.h>

#include <vector>

#include "moe_internal.cuh"

using namespace moe;

struct moe_ep_ctx {
    int d, E, I, k, dtype, max_tokens, device, n_sm;
    int e0, El, recv_cap;  // local experts [e0, e0 + El); receive capacity in rows
    float eps, scale;
    moe_weights w;         // w_gate_up / w_down hold the El local experts only
    size_t elem;
    void *ws;
    void *xp, *y, *xr, *act, *yr;  // send rows, received outputs, received rows, act, outputs
    int32_t *idx, *chunk_hist, *counts, *offsets, *mt_start, *perm, *inv;
    float *wts, *router_wt, *router_wg, *rinv;
    void *router_w3;
    CUtensorMap w3_map;
    bool route_tc, use_tc;
    int *status;
    int32_t *sched;  // [1 + El] the fused expert kernel's counters
    int32_t *loc;    // [2 (El + 1)] local row offsets, then the local row-tile prefix
    int e_pad, max_chunks;
    TcMaps maps;          // over the receive buffer and the local experts
    void *decode_maps;
    int last_n, last_nchunk;
    std::vector<int32_t> host_loc;
};

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void ep_free(moe_ep_ctx *h) {
    if (!h) return;
    if (h->decode_maps) decode_free_maps(h->decode_maps);
    if (h->ws) cudaFree(h->ws);
    delete h;
}

}  // namespace

extern "C" int moe_ep_create(int d, int n_experts, int d_ff, int top_k, float eps,
                             const moe_weights *w, int max_tokens, int expert_first, int n_local,
                             int max_recv_rows, moe_ep_ctx **out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!w) return MOE_ERR_INVALID_ARG;
    if (w->dtype != MOE_F32 && w->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (d <= 0 || n_experts <= 0 || d_ff <= 0 || top_k <= 0 || max_tokens <= 0)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (n_experts > kMaxExperts || top_k > kMaxTopK || top_k > n_experts)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (d % 4 != 0 || d > 32768) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (w->dtype == MOE_BF16 && (d % 64 != 0 || d_ff % 64 != 0)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (expert_first < 0 || n_local <= 0 || expert_first + n_local > n_experts)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (max_recv_rows <= 0 || static_cast<long long>(max_recv_rows) >= (1LL << 30) ||
        static_cast<long long>(max_tokens) * top_k >= (1LL << 30))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(n_local) * 2 * d_ff >= (1LL << 30) ||
        static_cast<long long>(n_experts) * d >= (1LL << 30))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!w->norm_gain || !w->router_w || !w->expert_bias || !w->w_gate_up || !w->w_down)
        return MOE_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !(w->routed_scale == w->routed_scale)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w->norm_gain) || !aligned16(w->router_w) || !aligned16(w->w_gate_up) ||
        !aligned16(w->w_down))
        return MOE_ERR_ALIGNMENT;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_NO_DEVICE;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_NO_DEVICE;
    if (prop.major != 10) return MOE_ERR_NO_DEVICE;

    moe_ep_ctx *h = new (std::nothrow) moe_ep_ctx();
    if (!h) return MOE_ERR_OOM;
    h->d = d; h->E = n_experts; h->I = d_ff; h->k = top_k; h->dtype = w->dtype;
    h->max_tokens = max_tokens; h->device = dev; h->n_sm = prop.multiProcessorCount;
    h->e0 = expert_first; h->El = n_local; h->recv_cap = max_recv_rows;
    h->eps = eps; h->scale = w->routed_scale; h->w = *w;
    h->elem = (w->dtype == MOE_F32) ? 4 : 2;
    h->use_tc = (w->dtype == MOE_BF16);
    h->route_tc = h->use_tc && route_tc_ok(d, n_experts);
    h->e_pad = (n_experts + 63) / 64 * 64;
    h->max_chunks = max_dispatch_chunks(n_experts);
    h->host_loc.assign(2 * (n_local + 1), 0);

    const size_t N = max_tokens, R = static_cast<size_t>(max_tokens) * top_k, C = max_recv_rows;
    const size_t E = n_experts, El = n_local;
    const size_t sizes[] = {
        R * d * h->elem,                               // xp: send rows
        R * d * h->elem,                               // y: received outputs
        C * d * h->elem,                               // xr: received rows
        C * d_ff * h->elem,                            // act
        C * d * h->elem,                               // yr: outputs to send back
        N * top_k * 4,                                 // idx
        static_cast<size_t>(h->max_chunks) * E * 4,    // chunk_hist
        E * 4,                                         // counts
        (E + 1) * 4,                                   // offsets
        (E + 1) * 4,                                   // mt_start
        R * 4,                                         // perm
        R * 4,                                         // inv
        N * top_k * 4,                                 // wts
        static_cast<size_t>(d) * h->e_pad * 4,         // router_wt
        N * 4,                                         // rinv
        E * static_cast<size_t>(d) * 4,                // router_wg
        (El + 1) * 4,                                  // sched
        256,                                           // status
        3 * E * static_cast<size_t>(d) * 2,            // router_w3
        2 * (El + 1) * 4,                              // loc
    };
    constexpr int nblocks = sizeof(sizes) / sizeof(sizes[0]);
    size_t total = 0, off[nblocks];
    for (int i = 0; i < nblocks; ++i) {
        off[i] = total;
        total += (sizes[i] + 255) & ~static_cast<size_t>(255);
    }
    if (cudaMalloc(&h->ws, total) != cudaSuccess) {
        cudaGetLastError();
        h->ws = nullptr;
        ep_free(h);
        return MOE_ERR_OOM;
    }
    uint8_t *b = static_cast<uint8_t *>(h->ws);
    h->xp = b + off[0]; h->y = b + off[1]; h->xr = b + off[2]; h->act = b + off[3];
    h->yr = b + off[4];
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
    h->loc = reinterpret_cast<int32_t *>(b + off[19]);
    if (cudaMemset(h->ws, 0, total) != cudaSuccess ||
        launch_prepare_router(w->router_w, w->norm_gain, h->router_wg, h->router_wt, n_experts,
                              h->e_pad, d, 0) != MOE_OK ||
        (h->route_tc && launch_split_router(h->router_wg, h->router_w3, n_experts, d, 0) != MOE_OK) ||
        cudaDeviceSynchronize() != cudaSuccess) {
        ep_free(h);
        return MOE_ERR_CUDA;
    }
    if (h->use_tc) {
        int rc = tc_build_maps(&h->maps, h->xr, h->act, w->w_gate_up, w->w_down, max_recv_rows,
                               n_local, d, d_ff);
        if (rc == MOE_OK)
            rc = decode_build_maps(&h->decode_maps, h->xr, h->act, w->w_gate_up, w->w_down,
                                   max_recv_rows, n_local, d, d_ff);
        if (rc == MOE_OK && h->route_tc)
            rc = tc_encode_2d(&h->w3_map, h->router_w3, 3 * static_cast<uint64_t>(n_experts), d,
                              3 * n_experts);
        if (rc != MOE_OK) {
            ep_free(h);
            return rc;
        }
    }
    *out = h;
    return MOE_OK;
}

extern "C" int moe_ep_dispatch(moe_ep_ctx *h, const void *x, int n_tokens, int32_t *counts_host,
                               void *stream) {
    if (!h || n_tokens < 0 || !counts_host) return MOE_ERR_INVALID_ARG;
    if (n_tokens > h->max_tokens) return MOE_ERR_TOO_MANY_TOKENS;
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MOE_ERR_INVALID_ARG;
    h->last_n = n_tokens;
    if (n_tokens == 0) {
        memset(counts_host, 0, sizeof(int32_t) * h->E);
        return MOE_OK;
    }
    if (!x) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x)) return MOE_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int N = n_tokens;
    int rc, tt = 0, nchunk = 1, chunk_tokens = N;
    const int kind = route_plan(N, h->d, h->E, &tt);
    chunk_plan(N, h->k, h->max_chunks, &nchunk, &chunk_tokens);
    h->last_nchunk = nchunk;
    // the route kernels add to the chunk histogram: start it at zero here, so
    // that a dispatch never depends on an earlier forward having combined
    if (cudaMemsetAsync(h->chunk_hist, 0, static_cast<size_t>(nchunk) * h->E * 4, s) != cudaSuccess)
        return MOE_ERR_CUDA;

    RouteParams rp;
    rp.x = x; rp.gain = h->w.norm_gain; rp.router_w = h->w.router_w; rp.router_wt = h->router_wt;
    rp.router_wg = h->router_wg;
    rp.bias = h->w.expert_bias; rp.rinv = h->rinv; rp.idx = h->idx; rp.wts = h->wts;
    rp.chunk_hist = h->chunk_hist; rp.status = h->status;
    rp.N = N; rp.d = h->d; rp.E = h->E; rp.k = h->k; rp.e_pad = h->e_pad;
    rp.chunk_tokens = chunk_tokens; rp.eps = h->eps; rp.scale = h->scale;
    if (h->route_tc && N >= 512)
        rc = launch_route_tc(rp, h->w3_map, s);
    else
        rc = launch_route(rp, h->dtype, kind, tt, s);
    if (rc != MOE_OK) return rc;

    DispatchParams dp;
    dp.idx = h->idx; dp.chunk_hist = h->chunk_hist; dp.counts = h->counts;
    dp.offsets = h->offsets; dp.mt_start = h->mt_start; dp.perm = h->perm; dp.inv = h->inv;
    dp.status = h->status; dp.x = x; dp.gain = h->w.norm_gain; dp.rinv = h->rinv; dp.xp = h->xp;
    dp.N = N; dp.d = h->d; dp.E = h->E; dp.k = h->k; dp.nchunk = nchunk;
    dp.chunk_tokens = chunk_tokens; dp.tile_m = kTcPairTileM;
    dp.elem_bytes = static_cast<int>(h->elem);
    dp.sched = nullptr;
    dp.sched_n = 0;
    dp.replicas = (4 * h->n_sm + nchunk - 1) / nchunk;
    if (dp.replicas > 64) dp.replicas = 64;
    if ((rc = launch_dispatch(dp, s)) != MOE_OK) return rc;
    if (cudaMemcpyAsync(counts_host, h->counts, sizeof(int32_t) * h->E, cudaMemcpyDeviceToHost,
                        s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

extern "C" int moe_ep_buffers(moe_ep_ctx *h, void **send_rows, void **recv_rows, void **send_y,
                              void **recv_y) {
    if (!h) return MOE_ERR_INVALID_ARG;
    if (send_rows) *send_rows = h->xp;
    if (recv_rows) *recv_rows = h->xr;
    if (send_y) *send_y = h->yr;
    if (recv_y) *recv_y = h->y;
    return MOE_OK;
}

extern "C" int moe_ep_experts(moe_ep_ctx *h, const int32_t *local_counts_host, void *stream) {
    if (!h || !local_counts_host) return MOE_ERR_INVALID_ARG;
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MOE_ERR_INVALID_ARG;
    const int El = h->El;
    long long rows = 0;
    for (int e = 0; e < El; ++e) {
        if (local_counts_host[e] < 0) return MOE_ERR_INVALID_ARG;
        rows += local_counts_host[e];
    }
    if (rows > h->recv_cap) return MOE_ERR_TOO_MANY_TOKENS;
    if (rows == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool fused = h->use_tc && rows <= static_cast<long long>(kDecodeRowsPerExpert) * El;
    const int tile_m = h->use_tc ? kTcPairTileM : kSimtTileM;
    int32_t *ho = h->host_loc.data(), *hm = ho + El + 1;
    ho[0] = hm[0] = 0;
    for (int e = 0; e < El; ++e) {
        ho[e + 1] = ho[e] + local_counts_host[e];
        hm[e + 1] = hm[e] + (local_counts_host[e] + tile_m - 1) / tile_m;
    }
    // pageable source: the copy has taken the values when the call returns
    if (cudaMemcpyAsync(h->loc, ho, sizeof(int32_t) * 2 * (El + 1), cudaMemcpyHostToDevice, s) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    int rc;
    if (fused) {
        if (cudaMemsetAsync(h->sched, 0, sizeof(int32_t) * (El + 1), s) != cudaSuccess)
            return MOE_ERR_CUDA;
        DecodeParams fp;
        fp.offsets = h->loc; fp.act = h->act; fp.y = h->yr; fp.sched = h->sched;
        fp.status = h->status; fp.E = El; fp.d = h->d; fp.I = h->I;
        return launch_decode_experts(h->decode_maps, fp, h->n_sm, s);
    }
    GroupedParams gp = {};
    gp.offsets = h->loc; gp.mt_start = h->loc + El + 1; gp.status = h->status;
    gp.E = El; gp.d = h->d; gp.I = h->I; gp.k = h->k; gp.rows_cap = h->recv_cap;
    gp.a = h->xr; gp.w = h->w.w_gate_up; gp.c = h->act;
    const int max_mtiles = static_cast<int>((rows + tile_m - 1) / tile_m) + El;
    rc = h->use_tc ? launch_gemm_tc2_gate_up(h->maps, gp, h->n_sm, s)
                   : launch_gemm_simt_gate_up(gp, max_mtiles, s);
    if (rc != MOE_OK) return rc;
    gp.a = h->act; gp.w = h->w.w_down; gp.c = h->yr;
    return h->use_tc ? launch_gemm_tc2_down(h->maps, gp, h->n_sm, s)
                     : launch_gemm_simt_down(gp, max_mtiles, s);
}

extern "C" int moe_ep_combine(moe_ep_ctx *h, const void *x, void *out, void *stream) {
    if (!h) return MOE_ERR_INVALID_ARG;
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MOE_ERR_INVALID_ARG;
    if (h->last_n == 0) return MOE_OK;
    if (!x || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out)) return MOE_ERR_ALIGNMENT;
    CombineParams cp;
    cp.x = x; cp.y = h->y; cp.wts = h->wts; cp.inv = h->inv; cp.out = out; cp.status = h->status;
    cp.chunk_hist = h->chunk_hist; cp.chunk_hist_n = h->last_nchunk * h->E;
    cp.N = h->last_n; cp.d = h->d; cp.k = h->k;
    return launch_combine(cp, h->dtype, static_cast<cudaStream_t>(stream));
}

extern "C" int moe_ep_debug_routing(moe_ep_ctx *h, int32_t *idx, float *w, int32_t *perm,
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
    if (offsets &&
        cudaMemcpyAsync(offsets, h->offsets, (h->E + 1) * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

extern "C" int moe_ep_status(moe_ep_ctx *h) {
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

extern "C" int moe_ep_destroy(moe_ep_ctx *h) {
    if (!h) return MOE_OK;
    int rc = cudaDeviceSynchronize() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    ep_free(h);
    return rc;
}
