// gemm_tc2.cu -- the grouped expert GEMMs of large batches on CTA pairs
// (tcgen05.mma.cta_group::2), with the weights as the 256-row MMA operand and
// the tokens as the N operand ("swap AB").
//
// The gated SiLU expert of "LFM2.5-24B-A2B: Biased Routing, Short Convolutions
// and Ten KV Caches" (flozi.net, English page, section "The router has two
// different scores") over the rows grouped by expert (section "What to verify
// in a deployment"):
//   gate/up: act[r][f] = silu(xp[r] . Wg_e[f]) * (xp[r] . Wu_e[f])
//   down:    y[r][n]   = act[r] . Wd_e[n]
// computed transposed, D[feature][token] = W_e[feature] . a[token]:
//   * M = 256 weight rows per tile, 128 in each CTA of the pair. gate/up: a
//     pair tile covers 128 features; CTA h stages the gate and up rows of
//     features f0+64h..+63 interleaved in groups of 16 (16 gate rows, the 16
//     matching up rows, ...) by one 4-D TMA box, so TMEM lanes l and l+16 of
//     every 32-lane quarter hold gate and up of one feature. down: CTA h
//     stages Wd rows n0+128h..+127.
//   * N = the tokens of one expert's tile, a multiple of 16 up to 256; CTA h
//     stages tokens N/2*h..+N/2-1 and the MMA reads both halves. An expert's
//     c rows are split into ceil(c/256) tiles of equal size rounded up to 16,
//     so at most 15 padded columns per tile are computed, where 256-row tiles
//     of the untransposed product would pad up to 255 rows per expert.
// Per CTA a stage is K = 128: two 64-wide boxes of weights (2 x 16 KB) and two
// 128-row boxes of tokens (2 x 16 KB, of which the MMA reads N/2 rows), so
// one barrier handshake covers eight MMAs; 3 stages.
// Both CTAs' TMA loads complete on the leader's full barrier (the leader
// expects the pair's bytes); the leader's single MMA thread issues the
// cta_group::2 MMAs and its commits arrive on both CTAs' barriers
// (tcgen05.commit with a CTA mask; no load uses multicast). Each CTA's
// epilogue reads its own 128 TMEM lanes and arrives remotely on the leader's
// accumulator-empty barrier. In gate/up the gate and up values of a feature
// sit in lanes 16 apart of one warp: the two threads swap half of each
// 32-token chunk by a register shuffle and each finishes 16 tokens.
// Eight epilogue warps, two per TMEM lane quarter, split each tile's token
// columns in 64-column chunks, so the TMEM drain (shuffles, SiLU, stores)
// keeps up with the MMAs of the next tile.
// All waits are bounded (1 s) and report MOE_ERR_DEVICE_TIMEOUT; the pair
// meets at a cluster barrier before TMEM is freed.
// The same pipeline serves the neighbouring dense and short-convolution
// blocks (one "expert", every token) through its epilogue mode: SiLU(gate) *
// up (kEpiSiluMul), a plain product g * v of paired rows (kEpiMul), a plain
// store (kEpiPlain), the store plus a residual (kEpiResid), or the u stream
// times the depthwise causal width-3 convolution of a stored a (kEpiConv).
// The last two read an input of the output's shape; they move it and the
// output in 16-byte rows through a 4 KB shared-memory tile per epilogue warp
// (32 KB in all, beside the 192 KB of stages), so a chunk costs one memory
// round trip instead of one per 16 scalar loads.
#include <cooperative_groups.h>

#include "moe_internal.cuh"

namespace cg = cooperative_groups;

namespace moe {
namespace {

constexpr int WM = 128;       // weight rows per CTA (MMA M = 256 per pair)
constexpr int TN = 256;       // most tokens per tile (MMA N)
constexpr int SUBK = 64;                          // K of one 128-byte-swizzled box
constexpr int KSUB = 2;                           // boxes per operand and stage
constexpr int BK = SUBK * KSUB;                   // K per stage
static_assert(BK == kTcPairBK, "K per stage");
constexpr int UK = 16;
constexpr int STAGES = 3;
constexpr int B_ROWS = TN / 2;                    // token rows per CTA
constexpr int A_SUB = WM * SUBK * 2;              // 16 KB
constexpr int B_SUB = B_ROWS * SUBK * 2;          // one 128-row box (rows past N/2 unused)
constexpr int A_BYTES = A_SUB * KSUB;
constexpr int B_BYTES = B_SUB * KSUB;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;    // 64 KB
constexpr int TMEM_COLS = 2 * TN;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t kPeerBitMask = 0xFEFFFFFFu;  // shared::cluster address in the pair's even CTA

struct Ctl {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
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

// Tile load whose completion is counted on the barrier at the same offset in
// the pair's even CTA.
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *m, int x, int y,
                                                 uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar) & kPeerBitMask)
        : "memory");
}

// gate/up weight box: {64 K, 16 rows, gate|up, 4 row groups} of the 4-D view
// W[group][gate|up][row][k]; w = first 16-row group.
__device__ __forceinline__ void tma_load_4d_pair(void *dst, const CUtensorMap *m, int x, int w,
                                                 uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(0), "r"(0), "r"(w),
        "r"(smem_u32(bar) & kPeerBitMask)
        : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// One arrival on `bar` in both CTAs of the pair once the issued MMAs complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m;\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

// Arrival on the barrier at the same offset in CTA `rank` of the cluster. It
// orders only this thread's earlier TMEM reads (fenced by the caller), not its
// global stores, which nobody waits for.
__device__ __forceinline__ void mbar_arrive_remote(uint64_t *bar, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(bar)), "r"(rank));
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}

__device__ __forceinline__ int find_expert(const int32_t *mts, int E, int q) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mts[mid] <= q) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Work item: expert e, weight tile wt, token tile of `rows` tokens from
// grouped row t0, computed with N = rows rounded up to 16. Items run expert
// by expert; within an expert the token tile varies fastest (the expert's
// weight tile is read from L2 by consecutive pairs), or with wt_fastest the
// weight tile does (for one large group whose token rows outgrow L2: each
// token tile is then read once while the weights stay in L2).
struct Item {
    int e, wt, t0, rows, N;
};

__device__ __forceinline__ Item decode(int item, int NW, const int32_t *mts, const int32_t *offs,
                                       int E, bool wt_fastest) {
    Item it;
    it.e = find_expert(mts, E, item / NW);
    const int ntt = mts[it.e + 1] - mts[it.e];
    const int local = item - mts[it.e] * NW;
    int tt;
    if (wt_fastest) {  // all weight tiles of a token tile, then the next token tile
        tt = local / NW;
        it.wt = local - tt * NW;
    } else {           // all token tiles of a weight tile, then the next weight tile
        it.wt = local / ntt;
        tt = local - it.wt * ntt;
    }
    const int c = offs[it.e + 1] - offs[it.e];
    const int ts = ((c + ntt - 1) / ntt + 15) & ~15;
    it.t0 = offs[it.e] + tt * ts;
    it.rows = min(ts, c - tt * ts);
    it.N = (it.rows + 15) & ~15;
    return it;
}

// g * sigmoid(g) with the fast exponential and division (the result is
// rounded to bf16); saturates to g for large g and to -0 for large -g.
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_tc2_kernel(const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmT, GroupedParams p) {
    // paired-row modes stage gate/up-style interleaved weight rows (4-D map)
    constexpr bool GATE_UP = MODE == kEpiSiluMul || MODE == kEpiMul || MODE == kEpiPartialPaired;
    constexpr bool PARTIAL = MODE == kEpiPartial || MODE == kEpiPartialPaired;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + STAGES * STAGE_BYTES);
    int32_t *mts = reinterpret_cast<int32_t *>(ctl + 1);  // [E+1]
    int32_t *offs = mts + (p.E + 1);                        // [E+1]

    cg::cluster_group cluster = cg::this_cluster();
    const int half = static_cast<int>(cluster.block_rank());  // 0: the leader
    const bool leader = half == 0;
    const int pair = blockIdx.x / 2, npairs = gridDim.x / 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 2 * kEpiWarps);  // one per epilogue warp of both CTAs
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {  // the same warp in both CTAs: one allocation for the pair
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&ctl->tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmT);
    }
    pdl_trigger();
    pdl_wait();
    for (int i = threadIdx.x; i <= E; i += kThreads) {
        mts[i] = p.mt_start[i];
        offs[i] = p.offsets[i];
    }
    tc_fence_before();
    cluster.sync();  // barriers initialised and TMEM allocated in both CTAs
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;

    const int NOUT = GATE_UP ? p.I : p.d;
    const int NW = GATE_UP ? (p.I + 127) / 128 : (p.d + 2 * WM - 1) / (2 * WM);
    const int K = GATE_UP ? p.d : p.I;
    const int nk = (K + BK - 1) / BK;
    // split-K: item = tile * S + slice; slice ks covers K blocks [ks*nkc, +nkc)
    const int S = PARTIAL && p.ksplit > 1 ? p.ksplit : 1;
    const int nkc = (nk + S - 1) / S;
    const int total = mts[E] * NW * S;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            // weight row (2-D, down) or first 16-row group (4-D, gate/up) of an item
            auto wcoord = [&](const Item &it) {
                return GATE_UP ? (it.e * 2 * p.I + it.wt * 128 + half * 64) / 16
                               : it.e * p.d + it.wt * 2 * WM + half * WM;
            };
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_parity[STAGES];
            bool issued[STAGES];
            for (int i = 0; i < STAGES; ++i) issued[i] = false;
            for (int item = pair; item < total && !aborted(ctl); item += npairs) {
                const Item it = decode(item / S, NW, mts, offs, E, p.wt_fastest != 0);
                const int kb0 = (item % S) * nkc, kb1 = min(nk, kb0 + nkc);
                const int trow = it.t0 + half * (it.N / 2);
                const int wc = wcoord(it);
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!wait_bar(&ctl->empty[s], ph ^ 1u, ctl, p.status)) { ok = false; break; }
                    uint8_t *sa = smem + s * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    // boxes that start inside K (the last stage of a K that is
                    // not a multiple of BK may hold one)
                    const int nsub = min(KSUB, (K - kb * BK + SUBK - 1) / SUBK);
                    if (leader) mbar_arrive_expect_tx(&ctl->full[s], 2 * nsub * (A_SUB + B_SUB));
                    for (int j = 0; j < nsub; ++j) {
                        const int x = kb * BK + j * SUBK;
                        if (GATE_UP)
                            tma_load_4d_pair(sa + j * A_SUB, &tmW, x, wc, &ctl->full[s]);
                        else
                            tma_load_2d_pair(sa + j * A_SUB, &tmW, x, wc, &ctl->full[s]);
                        tma_load_2d_pair(sb + j * B_SUB, &tmT, x, trow, &ctl->full[s]);
                    }
                    issued[s] = true;
                    issued_parity[s] = ph;
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
            }
            if (aborted(ctl) && leader) {  // the pair's copies complete on the leader's barriers
                const uint64_t dl = globaltimer_ns() + kWaitNs;
                for (int i = 0; i < STAGES; ++i)
                    if (issued[i]) mbar_wait(&ctl->full[i], issued_parity[i], dl);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------- MMA issuer (leader only) ----------------
            int s = 0;
            uint32_t ph = 0;
            int tile = 0;
            bool any = false;
            for (int item = pair; item < total && !aborted(ctl); item += npairs, ++tile) {
                const Item it = decode(item / S, NW, mts, offs, E, p.wt_fastest != 0);
                const int kb0 = (item % S) * nkc, kb1 = min(nk, kb0 + nkc);
                const uint32_t idesc = idesc_bf16_f32(2 * WM, it.N);
                const int buf = tile & 1;
                const uint32_t use = static_cast<uint32_t>(tile >> 1);
                if (!wait_bar(&ctl->tempty[buf], (use & 1u) ^ 1u, ctl, p.status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * TN);
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!wait_bar(&ctl->full[s], ph, ctl, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
                    const uint32_t b0 = a0 + A_BYTES;
                    const int nsub = min(KSUB, (K - kb * BK + SUBK - 1) / SUBK);
#pragma unroll
                    for (int j = 0; j < KSUB; ++j) {
                        if (j < nsub) {
#pragma unroll
                            for (int kk = 0; kk < SUBK / UK; ++kk)
                                umma_bf16_pair(d_tmem, sw128_kmajor_desc(a0 + j * A_SUB + kk * UK * 2),
                                               sw128_kmajor_desc(b0 + j * B_SUB + kk * UK * 2), idesc,
                                               (kb != kb0 || j != 0 || kk != 0) ? 1u : 0u);
                        }
                    }
                    any = true;
                    umma_commit_pair(&ctl->empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                umma_commit_pair(&ctl->tfull[buf]);
            }
            if (any) {
                asm volatile(
                    "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                        smem_u32(&ctl->drain))
                    : "memory");
                mbar_wait(&ctl->drain, 0, globaltimer_ns() + kWaitNs);
            }
        }
    } else {
        // ---------------- epilogue (warps 2..9, both CTAs) ----------------
        const int q = warp & 3;            // TMEM lane quarter of this warp
        const int c_first = ((warp - 2) >> 2) * 64;  // its 64-column chunks, every kEpiWarps/4-th
        __nv_bfloat16 *c = static_cast<__nv_bfloat16 *>(p.c);
        // the warp's 64 x 32 bf16 staging tile (kEpiResid, kEpiConv), after the expert tables
        __nv_bfloat16 *stage = reinterpret_cast<__nv_bfloat16 *>(
                                   (reinterpret_cast<uintptr_t>(offs + E + 1) + 15) & ~static_cast<uintptr_t>(15)) +
                               (warp - 2) * 64 * 32;
        int tile = 0;
        for (int item = pair; item < total && !aborted(ctl); item += npairs, ++tile) {
            const int buf = tile & 1;
            const uint32_t use = static_cast<uint32_t>(tile >> 1);
            if (!wait_bar(&ctl->tfull[buf], use & 1u, ctl, p.status)) break;
            tc_fence_after();
            const Item it = decode(item / S, NW, mts, offs, E, p.wt_fastest != 0);
                const int kb0 = (item % S) * nkc, kb1 = min(nk, kb0 + nkc);
            const uint32_t t_lane = tmem_base + static_cast<uint32_t>(buf * TN) +
                                    (static_cast<uint32_t>(q * 32) << 16);
            const int nvalid = min(it.rows, p.rows_cap - it.t0);  // tokens stored
            if constexpr (MODE == kEpiPartialPaired) {
                // raw sums of the K slice: gate rows to columns f, up rows to NOUT + f
                const int f = it.wt * 128 + half * 64 + q * 16 + (lane & 15);
                float *prow = p.partial + (static_cast<size_t>(item % S) * p.partial_rows + it.t0) *
                                              (2 * static_cast<size_t>(NOUT)) +
                              (lane < 16 ? 0 : NOUT) + f;
#pragma unroll 1
                for (int c0 = c_first; c0 < it.N; c0 += 64 * (kEpiWarps / 4)) {
                    uint32_t v[2][32];
                    tmem_ld_32x32b_x32(t_lane + c0, v[0]);
                    tmem_ld_32x32b_x32(t_lane + c0 + 32, v[1]);
                    tmem_ld_wait();
                    const int lim = f < NOUT ? nvalid - c0 : 0;
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        if (j < lim)
                            prow[static_cast<size_t>(c0 + j) * (2 * NOUT)] = __uint_as_float(v[j >> 5][j & 31]);
                }
            } else if constexpr (MODE == kEpiPartial) {
                const int n = it.wt * 2 * WM + half * WM + q * 32 + lane;
                float *prow = p.partial +
                              (static_cast<size_t>(item % S) * p.partial_rows + it.t0) * NOUT + n;
#pragma unroll 1
                for (int c0 = c_first; c0 < it.N; c0 += 64 * (kEpiWarps / 4)) {
                    uint32_t v[2][32];
                    tmem_ld_32x32b_x32(t_lane + c0, v[0]);
                    tmem_ld_32x32b_x32(t_lane + c0 + 32, v[1]);
                    tmem_ld_wait();
                    const int lim = n < NOUT ? nvalid - c0 : 0;
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        if (j < lim) prow[static_cast<size_t>(c0 + j) * NOUT] = __uint_as_float(v[j >> 5][j & 31]);
                }
            } else if constexpr (GATE_UP) {
                // lanes 0..15: gate of features f, lanes 16..31: up of the same f
                const bool is_gate = lane < 16;
                const int f = it.wt * 128 + half * 64 + q * 16 + (lane & 15);
#pragma unroll 1
                for (int c0 = c_first; c0 < it.N; c0 += 64 * (kEpiWarps / 4)) {
                    uint32_t v[2][32];
                    tmem_ld_32x32b_x32(t_lane + c0, v[0]);
                    tmem_ld_32x32b_x32(t_lane + c0 + 32, v[1]);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        // the gate thread finishes tokens 0..15 of the chunk, the up thread 16..31
                        const int tb = c0 + h * 32 + (is_gate ? 0 : 16);
                        const int lim = f < NOUT ? nvalid - tb : 0;
                        __nv_bfloat16 *dst = c + static_cast<size_t>(it.t0 + tb) * NOUT + f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float mine_lo = __uint_as_float(v[h][j]);
                            const float mine_hi = __uint_as_float(v[h][16 + j]);
                            const float got = __shfl_xor_sync(0xffffffffu, is_gate ? mine_hi : mine_lo, 16);
                            const float g = is_gate ? mine_lo : got;
                            const float u = is_gate ? got : mine_hi;
                            const float r = MODE == kEpiSiluMul ? silu(g) * u : g * u;
                            if (j < lim) *dst = __float2bfloat16_rn(r);
                            dst += NOUT;
                        }
                    }
                }
            } else if constexpr (MODE == kEpiPlain) {
                const int n = it.wt * 2 * WM + half * WM + q * 32 + lane;
#pragma unroll 1
                for (int c0 = c_first; c0 < it.N; c0 += 64 * (kEpiWarps / 4)) {
                    uint32_t v[2][32];
                    tmem_ld_32x32b_x32(t_lane + c0, v[0]);
                    tmem_ld_32x32b_x32(t_lane + c0 + 32, v[1]);
                    tmem_ld_wait();
                    if (n < NOUT) {
                        const int lim = nvalid - c0;
                        __nv_bfloat16 *dst = c + static_cast<size_t>(it.t0 + c0) * NOUT + n;
#pragma unroll
                        for (int j = 0; j < 64; ++j) {
                            if (j < lim) *dst = __float2bfloat16_rn(__uint_as_float(v[j >> 5][j & 31]));
                            dst += NOUT;
                        }
                    }
                }
            } else {
                // kEpiResid: out = x + acc; kEpiConv: y = u * (k0 a_t + k1 a_{t-1} + k2 a_{t-2})
                // per sequence. A warp's chunk is 64 token rows of its 32 channels
                // n0..n0+31 (64 contiguous bytes per row). The rows of x or a come
                // in by 16-byte loads, 8 per lane, issued before the TMEM loads
                // (one memory round trip per chunk), and are staged in the warp's
                // 4 KB of shared memory [row][32]; each thread then walks its own
                // channel's column, overwriting every input with its output, and
                // the chunk leaves by 16-byte stores from the same lanes and
                // addresses as the loads. Each lane thus stores exactly the
                // elements it loaded, so out may be x.
                const int n0 = it.wt * 2 * WM + half * WM + q * 32;
                const int n = n0 + lane;
                const bool nval = n < NOUT;
                const int vcol = n0 + (lane & 3) * 8;  // first channel of this lane's 16-byte column
                const bool vval = vcol < NOUT;         // NOUT % 8 == 0: all 8 channels or none
                const __nv_bfloat16 *src =
                    static_cast<const __nv_bfloat16 *>(MODE == kEpiResid ? p.resid : p.aux);
                __nv_bfloat16 *col = stage + lane;
                float k0 = 0.f, k1 = 0.f, k2 = 0.f;
                if (MODE == kEpiConv && nval) {
                    k0 = p.conv[n * 3];
                    k1 = p.conv[n * 3 + 1];
                    k2 = p.conv[n * 3 + 2];
                }
#pragma unroll 1
                for (int c0 = c_first; c0 < it.N; c0 += 64 * (kEpiWarps / 4)) {
                    const int lim = nvalid - c0;
                    const size_t r0 = static_cast<size_t>(it.t0 + c0);
                    uint4 in[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int row = (lane >> 2) + 8 * i;
                        in[i] = make_uint4(0u, 0u, 0u, 0u);
                        if (vval && row < lim)
                            in[i] = *reinterpret_cast<const uint4 *>(src + (r0 + row) * NOUT + vcol);
                    }
                    // kEpiConv: the two a values before the chunk, from a (same
                    // sequence) or the sequence's carried state
                    const int T = p.seq_len;
                    int b = 0, t = 0;
                    float am1 = 0.f, am2 = 0.f;
                    auto hist = [&](int seq, int slot) {  // a of position slot - 2 of seq
                        return p.state_in ? p.state_in[(static_cast<size_t>(seq) * 2 + slot) * NOUT + n] : 0.f;
                    };
                    if (MODE == kEpiConv && nval && lim > 0) {
                        b = (it.t0 + c0) / T;  // rows < 2^30
                        t = it.t0 + c0 - b * T;
                        am1 = t >= 1 ? __bfloat162float(src[(r0 - 1) * NOUT + n]) : hist(b, 1);
                        am2 = t >= 2 ? __bfloat162float(src[(r0 - 2) * NOUT + n])
                                     : t == 1 ? hist(b, 1) : hist(b, 0);
                    }
                    uint32_t v[2][32];
                    tmem_ld_32x32b_x32(t_lane + c0, v[0]);
                    tmem_ld_32x32b_x32(t_lane + c0 + 32, v[1]);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        *reinterpret_cast<uint4 *>(stage + ((lane >> 2) + 8 * i) * 32 + (lane & 3) * 8) = in[i];
                    __syncwarp();
                    // every row of the stage is valid to read (rows past lim hold
                    // zeros and are not stored), so the common paths run without a
                    // branch per row and the shared-memory loads go out 32 at a time
                    if (nval) {
                        if (MODE == kEpiResid || t + min(lim, 64) <= T) {
                            // kEpiConv: no sequence starts after the chunk's first row
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                float xin[32];
#pragma unroll
                                for (int j = 0; j < 32; ++j) xin[j] = __bfloat162float(col[(h * 32 + j) * 32]);
#pragma unroll
                                for (int j = 0; j < 32; ++j) {
                                    const float acc = __uint_as_float(v[h][j]);
                                    if constexpr (MODE == kEpiResid) {
                                        col[(h * 32 + j) * 32] = __float2bfloat16_rn(xin[j] + acc);
                                    } else {
                                        const float cv = fmaf(k2, am2, fmaf(k1, am1, k0 * xin[j]));
                                        col[(h * 32 + j) * 32] = __float2bfloat16_rn(acc * cv);
                                        am2 = am1;
                                        am1 = xin[j];
                                    }
                                }
                            }
                        } else {
                            // kEpiConv across sequence starts: the window restarts
                            // from the carried state of each new sequence
#pragma unroll
                            for (int j = 0; j < 64; ++j) {
                                if (j < lim) {
                                    const float acc = __uint_as_float(v[j >> 5][j & 31]);
                                    const float xin = __bfloat162float(col[j * 32]);
                                    if (t == 0) {  // a new sequence starts at this row
                                        am1 = hist(b, 1);
                                        am2 = hist(b, 0);
                                    }
                                    const float cv = fmaf(k2, am2, fmaf(k1, am1, k0 * xin));
                                    col[j * 32] = __float2bfloat16_rn(acc * cv);
                                    am2 = am1;
                                    am1 = xin;
                                    if (++t == T) { t = 0; ++b; }
                                }
                            }
                        }
                    }
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int row = (lane >> 2) + 8 * i;
                        if (vval && row < lim)
                            *reinterpret_cast<uint4 *>(c + (r0 + row) * NOUT + vcol) =
                                *reinterpret_cast<const uint4 *>(stage + row * 32 + (lane & 3) * 8);
                    }
                    __syncwarp();  // the stores' reads of the stage precede the next chunk's writes
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(&ctl->tempty[buf], 0);  // the leader's barrier
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster.sync();  // the leader's MMAs into this CTA's TMEM have drained
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

constexpr size_t kStageBytes = 16 + kEpiWarps * 64 * 32 * 2;  // staging tiles + alignment

size_t smem_bytes(int E, bool staged) {
    return 1024 + STAGES * STAGE_BYTES + sizeof(Ctl) + 2 * (E + 1) * sizeof(int32_t) +
           (staged ? kStageBytes : 0);
}

// CTA pairs that can be resident at once (an SM without a partner in its GPC
// cannot host half a pair), at most one pair per two SMs.
int resident_pairs(const void *kern, size_t smem, int n_sm) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_sm / 2 * 2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = n_sm / 2;
    }
    return n < n_sm / 2 ? n : n_sm / 2;
}

template <int MODE>
int launch(const CUtensorMap &w, const CUtensorMap &t, const GroupedParams &p, int n_sm,
           cudaStream_t s) {
    auto kern = grouped_tc2_kernel<MODE>;
    const size_t smem = smem_bytes(p.E, MODE == kEpiResid || MODE == kEpiConv);
    if (ensure_smem(kern, smem) != MOE_OK) return MOE_ERR_CUDA;
    static int pairs = 0;  // per kernel, for the device model of the process
    if (pairs == 0) pairs = resident_pairs(reinterpret_cast<const void *>(kern), smem, n_sm);
    return launch_k(kern, dim3(2 * pairs), dim3(kThreads), smem, s, w, t, p);
}

}  // namespace

int launch_gemm_tc2_gate_up(const TcMaps &m, const GroupedParams &p, int n_sm, cudaStream_t s) {
    return launch<kEpiSiluMul>(m.w_gate_up_4d, m.a_gate_up, p, n_sm, s);
}

int launch_gemm_tc2_down(const TcMaps &m, const GroupedParams &p, int n_sm, cudaStream_t s) {
    return launch<kEpiPlain>(m.w_down_half, m.a_down, p, n_sm, s);
}

int launch_gemm_tc2_mode(int mode, const CUtensorMap &w, const CUtensorMap &t,
                         const GroupedParams &p, int n_sm, cudaStream_t s) {
    switch (mode) {
        case kEpiSiluMul: return launch<kEpiSiluMul>(w, t, p, n_sm, s);
        case kEpiPlain: return launch<kEpiPlain>(w, t, p, n_sm, s);
        case kEpiMul: return launch<kEpiMul>(w, t, p, n_sm, s);
        case kEpiConv: return launch<kEpiConv>(w, t, p, n_sm, s);
        case kEpiResid: return launch<kEpiResid>(w, t, p, n_sm, s);
        case kEpiPartialPaired: return launch<kEpiPartialPaired>(w, t, p, n_sm, s);
        case kEpiPartial: return launch<kEpiPartial>(w, t, p, n_sm, s);
        default: return MOE_ERR_INVALID_ARG;
    }
}

}  // namespace moe
