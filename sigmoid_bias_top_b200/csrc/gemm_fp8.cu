// gemm_fp8.cu -- FP8_BLOCK experts: both expert contractions of a batch in ONE
// persistent kernel, e4m3 weights as the tensor-core M operand ("swap-AB").
//
// The gated SiLU expert of "LFM2.5-24B-A2B: Biased Routing, Short Convolutions
// and Ten KV Caches" (flozi.net, English page, section "The router has two
// different scores") with the FP8_BLOCK storage of the FP8 checkpoint
// ("LFM2.5-24B-A2B: ein 24B-Reasoning-Modell, das pro Wortstück so wenig verbraucht wie ein 2B-Modell",
// inferencekey.com, section "Für Engineers", paragraph "Quantisierung":
// weights FP8 in static 128x128 blocks, activations FP8 dynamic per group
// of 128).
//
// Work decomposition as in the bf16 small-batch kernel: an item is one
// 128-row weight tile (gate/up item (e, ft): gate rows ft*128.. and the
// matching up rows of expert e, K = d; down item (e, nt): rows nt*128.. of
// Wd_e, K = I), claimed from one atomic counter, gate/up items first; a down
// item of expert e waits until its I/128 gate/up items have published their
// act rows. Each item runs in passes of 32 tokens (small batches) or 64.
//
// What FP8_BLOCK changes: a stage is one K block of 128 (128 e4m3 = one
// 128-byte swizzle row), and every block has its own scale on both operands
// (weight block scale sw, token group scale sa), so the tensor cores cannot
// accumulate across blocks. Each K block's MMAs (kind::f8f6f4, M128, N32/64,
// K32) start a fresh accumulator in one of 8 (32-token passes) or 4 rotating
// TMEM buffers; the epilogue warps load it (tcgen05.ld) and add
// partial * sw * sa[token] into fp32 registers, while the tensor cores
// already fill the next buffers. At the end of a pass:
//   gate/up: a = SiLU(gate) * up per (token, row); the item's 128 rows are
//     exactly one activation group of 128, so the group maximum is a max
//     over the 128 TMEM lanes (a warp redux per column, then the four lane
//     quadrants through shared memory, met at an mbarrier), s = amax / 448
//     and the codes e4m3(a / s) (the IEEE quotient, formed by div_rn;
//     nearest-even, saturating) go to aq, s to as;
//   down: y = the fp32 sum, rounded once to bf16.
// Roles per CTA (320 threads): warp 0 lane 0 claims items and issues TMA
// (and prefetches the item's block scales into L2); warp 1 owns TMEM (512
// columns) and one thread issues the MMAs; warps 2..9 are the epilogue, two
// per TMEM lane quadrant (two teams taking alternate items, or both warps of
// a quadrant sharing each unit's columns: see Shape); the per-column scale
// products sa * sw of up to eight K blocks are formed once per lane into a
// shared-memory table and read back as float4s. All waits are bounded (1 s)
// and report MOE_ERR_DEVICE_TIMEOUT; on time-out the kernel drains its own
// copies and MMAs, frees TMEM and returns.
#include <cuda_fp8.h>

#include <new>

#include "moe_fp8.cuh"

namespace moe {
namespace {

constexpr int WM = 128;              // weight rows per item (MMA M)
constexpr int TT = 32;               // tokens per token tile
constexpr int BK = kFp8Block;        // K per stage: one scale block, 128 bytes per row
constexpr int UK = 32;               // K per tcgen05.mma kind::f8f6f4
constexpr int STAGES = 5;
constexpr int A_BYTES = WM * BK;     // 16 KB weight tile
constexpr int B_TILE = TT * BK;      // 4 KB token tile
constexpr int TMEM_COLS = 512;
constexpr int RING = 4;
constexpr int kEpiWarps = 8;         // two per TMEM lane quadrant
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int TBL_KB = 8;            // K blocks per chunk of the epilogue's scale table
constexpr int kThreads = 64 + kEpiThreads;

// Sizes that follow from MAXT, the token tiles per pass (1 for small batches,
// 2 otherwise): a K block's partials take 2 * NP TMEM columns (gate, up), so
// fewer tokens per pass leave more K-block buffers for the tensor cores to
// run ahead of the epilogue (8 instead of 4).
//
// The epilogue warps: with one token tile per pass they form two teams of
// four (one warp per TMEM lane quadrant) that take alternate items (all the
// passes of an item go to the same team, so that the team's fence before
// publishing the item covers every row it wrote), each warp
// covering all 32 columns, so that one team's end-of-pass work (SiLU,
// quantisation, publication) and scale loads overlap the other team's K loop;
// with two tiles the eight warps share every unit, the two warps of a
// quadrant taking 16 columns of each tile (the registers of a 64-column warp
// would not fit).
template <int MAXT>
struct Shape {
    static constexpr int NP = TT * MAXT;                          // tokens per pass
    static constexpr int STAGE_BYTES = 2 * A_BYTES + MAXT * B_TILE;
    static constexpr int BUF_COLS = 2 * NP;                       // gate 0..NP-1, up NP..
    static constexpr int NBUF = TMEM_COLS / BUF_COLS;
    static constexpr int TEAMS = MAXT == 1 ? 2 : 1;
    static constexpr int CWW = MAXT == 1 ? 32 : 16;               // columns per tile per warp
    static constexpr int TEAM_THREADS = kEpiThreads / TEAMS;
};
constexpr uint64_t kWaitNs = 1000000000ull;

template <int MAXT>
struct Ctl {
    static constexpr int NBUF = Shape<MAXT>::NBUF, NP = Shape<MAXT>::NP;
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[NBUF];
    uint64_t tempty[NBUF];
    uint64_t ufull[RING];
    uint64_t uempty[RING];
    static constexpr int TEAMS = Shape<MAXT>::TEAMS, CWW = Shape<MAXT>::CWW;
    uint64_t pub[TEAMS];        // every thread of a team has stored an item's act rows
    uint64_t red_bar[TEAMS][2]; // a team's column maxima are in red[team][b]
    uint64_t drain;
    float red[TEAMS][2][4][NP]; // per lane quadrant, per token column: max |a| over its 32 rows
    // per epilogue warp, per K block of the current chunk: sa[col] * sw of
    // each of the warp's MAXT * CWW columns, for gate (0) and up (1)
    float4 tbl[kEpiWarps][2][TBL_KB][MAXT * CWW / 4];
    int ring_item[RING];
    int ring_pass[RING];
    int ring_team[RING];  // the epilogue team of the unit's item (all its passes)
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, int *abort_flag,
                                         int *status) {
    if (mbar_try_wait(bar, parity)) return true;
    if (mbar_wait(bar, parity, globaltimer_ns() + kWaitNs)) return true;
    set_status(status, kStatusTimeout);
    atomicExch(abort_flag, 1);
    return false;
}

__device__ __forceinline__ bool aborted(int *abort_flag) {
    return *reinterpret_cast<volatile int *>(abort_flag) != 0;
}

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Brings the bytes [p, p + bytes) into L2 (no registers written).
__device__ __forceinline__ void prefetch_l2(const void *p, int bytes) {
    const char *c = static_cast<const char *>(p);
    for (int o = 0; o < bytes; o += 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(c + o));
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

struct Unit {
    bool gate_up;
    int e, tile;         // expert, weight tile (ft or nt)
    int row0, rows;      // grouped token rows of this pass
    int ntt;             // token tiles (1 or 2)
    bool last_pass;
};

template <int MAXT>
__device__ __forceinline__ Unit decode(int item, int pass, int n_gu_tiles, int n_dn_tiles, int E,
                                       const int32_t *offs) {
    constexpr int NP = Shape<MAXT>::NP;
    Unit u;
    const int n_gu = E * n_gu_tiles;
    u.gate_up = item < n_gu;
    const int local = u.gate_up ? item : item - n_gu;
    const int per = u.gate_up ? n_gu_tiles : n_dn_tiles;
    u.e = local / per;
    u.tile = local - u.e * per;
    const int beg = offs[u.e], cnt = offs[u.e + 1] - beg;
    u.row0 = beg + pass * NP;
    u.rows = min(NP, cnt - pass * NP);
    u.ntt = (u.rows + TT - 1) / TT;
    u.last_pass = (pass + 1) * NP >= cnt;
    return u;
}

// One epilogue step: NKB consecutive K blocks (TMEM buffers buf, buf+1, ...)
// of NT token tiles, gate and up (GU) or down only: every partial times its
// column's scale product from the table row of that K block, added into the
// fp32 accumulators. Per 16 columns, the loads of all NKB blocks are issued
// before one wait.
template <int MAXT, bool GU, int NT, int NKB>
__device__ __forceinline__ void promote(
    uint32_t t0, int buf, const float4 (*tg)[MAXT * Shape<MAXT>::CWW / 4],
    const float4 (*tu)[MAXT * Shape<MAXT>::CWW / 4], float (&accg)[NT * Shape<MAXT>::CWW],
    float (&accu)[NT * Shape<MAXT>::CWW]) {
    constexpr int NP = Shape<MAXT>::NP, NBUF = Shape<MAXT>::NBUF, BUF_COLS = Shape<MAXT>::BUF_COLS;
    constexpr int CWW = Shape<MAXT>::CWW, NH = CWW / 16;
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int h = 0; h < NH; ++h) {  // 16 columns at a time
            uint32_t g[NKB][16], v[NKB][16];
#pragma unroll
            for (int k = 0; k < NKB; ++k) {
                const uint32_t tb = t0 + static_cast<uint32_t>(((buf + k) % NBUF) * BUF_COLS);
                tmem_ld_32x32b_x16(tb + t * TT + h * 16, g[k]);
                if (GU) tmem_ld_32x32b_x16(tb + NP + t * TT + h * 16, v[k]);
            }
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < NKB; ++k)
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int cc = t * CWW + h * 16 + 4 * c4;  // accumulator / table column
                    const float4 sg = tg[k][cc / 4];
                    accg[cc + 0] = fmaf(__uint_as_float(g[k][4 * c4 + 0]), sg.x, accg[cc + 0]);
                    accg[cc + 1] = fmaf(__uint_as_float(g[k][4 * c4 + 1]), sg.y, accg[cc + 1]);
                    accg[cc + 2] = fmaf(__uint_as_float(g[k][4 * c4 + 2]), sg.z, accg[cc + 2]);
                    accg[cc + 3] = fmaf(__uint_as_float(g[k][4 * c4 + 3]), sg.w, accg[cc + 3]);
                    if (GU) {
                        const float4 su = tu[k][cc / 4];
                        accu[cc + 0] = fmaf(__uint_as_float(v[k][4 * c4 + 0]), su.x, accu[cc + 0]);
                        accu[cc + 1] = fmaf(__uint_as_float(v[k][4 * c4 + 1]), su.y, accu[cc + 1]);
                        accu[cc + 2] = fmaf(__uint_as_float(v[k][4 * c4 + 2]), su.z, accu[cc + 2]);
                        accu[cc + 3] = fmaf(__uint_as_float(v[k][4 * c4 + 3]), su.w, accu[cc + 3]);
                    }
                }
        }
}

// Per-thread state of an epilogue warp across units.
struct EpiState {
    int ew, q, h2, r, lt, lcol;  // warp index, TMEM lane quadrant, column half, row, lane column
    int team;
    uint32_t tmem_base;
    uint32_t nblk, npub, nred;   // K blocks consumed; phases of ctl->pub and ctl->red_bar
};

struct Fp8Maps {
    CUtensorMap w_gate_up;  // e4m3 [E*2I][d] box 128 x 128
    CUtensorMap w_down;     // e4m3 [E*d][I]  box 128 x 128
    CUtensorMap xq;         // e4m3 [rows][d] box 128 x 32
    CUtensorMap aq;         // e4m3 [rows][I] box 128 x 32
};


// The epilogue's work on one unit (item, pass) with NT = u.ntt token tiles:
// the K loop (scale table per chunk of TBL_KB blocks, promotion of every
// block), then the pass's output: bf16 y rows (down) or the quantised
// SiLU(gate)*up codes and group scales (gate/up), published after the last
// pass. Returns false after a timed-out wait (status and abort already set).
template <int MAXT, int NT>
__device__ __forceinline__ bool epi_unit(const Unit &u, Ctl<MAXT> *ctl, const Fp8ExpertParams &p,
                                         EpiState &st, int n_gu_tiles, int n_dn_tiles,
                                         int *done) {
    constexpr int NBUF = Shape<MAXT>::NBUF, CWW = Shape<MAXT>::CWW;
    const int lane = threadIdx.x & 31;
    const int ngd = p.d / kFp8Block, ngi = p.I / kFp8Block;
    const int nk = (u.gate_up ? p.d : p.I) / BK;
    // weight block scales of this item: row blocks of the gate and up tiles
    // (gate/up) or of the Wd tile (down), one per K block
    const float *swg = u.gate_up
        ? p.sgu + (static_cast<size_t>(u.e) * (2 * n_gu_tiles) + u.tile) * ngd
        : p.sdn + (static_cast<size_t>(u.e) * n_dn_tiles + u.tile) * ngi;
    const float *swu = u.gate_up
        ? p.sgu + (static_cast<size_t>(u.e) * (2 * n_gu_tiles) + n_gu_tiles + u.tile) * ngd
        : swg;
    const int ng = u.gate_up ? ngd : ngi;
    // this lane's column (lane / CWW is its token tile, which must exist in
    // this shape); its group scales (row of xs or as)
    const bool lserve = st.lt < MAXT;
    const bool lvalid = st.lt < NT && st.lcol < u.rows;
    const float *sa_row = (u.gate_up ? p.xs : p.as) +
                          static_cast<size_t>(u.row0 + (lvalid ? st.lcol : 0)) * ng;
    float accg[NT * CWW], accu[NT * CWW];
#pragma unroll
    for (int c = 0; c < NT * CWW; ++c) { accg[c] = 0.f; accu[c] = 0.f; }
    const float4 (*tg)[MAXT * CWW / 4] = ctl->tbl[st.ew][0];
    const float4 (*tu)[MAXT * CWW / 4] = ctl->tbl[st.ew][1];
    const uint32_t tq = st.tmem_base + (static_cast<uint32_t>(st.q * 32) << 16) + st.h2 * CWW;
    for (int kb = 0; kb < nk;) {
        if (kb % TBL_KB == 0) {
            // the next chunk of the scale table: lane l writes column l's
            // products for up to TBL_KB K blocks
            const int n = min(TBL_KB, nk - kb);
            __syncwarp();  // every lane is done with the previous chunk
#pragma unroll
            for (int j = 0; j < TBL_KB; ++j) {
                float sg = 0.f, su = 0.f;
                if (j < n) {
                    const float sa = !lvalid ? 0.f
                        : u.gate_up ? __ldg(sa_row + kb + j) : __ldcg(sa_row + kb + j);
                    sg = sa * __ldg(swg + kb + j);
                    if (u.gate_up) su = sa * __ldg(swu + kb + j);
                }
                if (lserve) {
                    reinterpret_cast<float *>(ctl->tbl[st.ew][0][j])[lane] = sg;
                    reinterpret_cast<float *>(ctl->tbl[st.ew][1][j])[lane] = su;
                }
            }
            __syncwarp();
        }
        // two K blocks per step for one 16-column tile while both lie in this chunk
        const int nkb = (NT == 1 && CWW == 16 && kb + 1 < nk && (kb + 1) % TBL_KB != 0) ? 2 : 1;
        const int buf = static_cast<int>(st.nblk % NBUF);
        for (int k = 0; k < nkb; ++k)
            if (!wait_bar(&ctl->tfull[(buf + k) % NBUF], ((st.nblk + k) / NBUF) & 1u, &ctl->abort, p.status))
                return false;
        tc_fence_after();
        const int row = kb % TBL_KB;
        if (u.gate_up) {
            if (CWW == 16 && nkb == 2) promote<MAXT, true, NT, (CWW == 16 ? 2 : 1)>(tq, buf, tg + row, tu + row, accg, accu);
            else promote<MAXT, true, NT, 1>(tq, buf, tg + row, tu + row, accg, accu);
        } else {
            if (CWW == 16 && nkb == 2) promote<MAXT, false, NT, (CWW == 16 ? 2 : 1)>(tq, buf, tg + row, tu + row, accg, accu);
            else promote<MAXT, false, NT, 1>(tq, buf, tg + row, tu + row, accg, accu);
        }
        tc_fence_before();
        __syncwarp();  // the whole warp's loads are done: one arrival per warp
        if (lane == 0)
            for (int k = 0; k < nkb; ++k) mbar_arrive(&ctl->tempty[(buf + k) % NBUF]);
        st.nblk += nkb;
        kb += nkb;
    }

    if (!u.gate_up) {
        __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(p.y);
        const int f = u.tile * WM + st.r;
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int c = 0; c < CWW; ++c) {
                const int col = t * TT + st.h2 * CWW + c;
                if (col < u.rows)
                    y[static_cast<size_t>(u.row0 + col) * p.d + f] = __float2bfloat16_rn(accg[t * CWW + c]);
            }
        return true;
    }

    // a = SiLU(gate) * up; group maximum per token column over the 128 rows:
    // a warp maximum over the bits of |a| (non-negative floats order like
    // their bit patterns), then the four lane quadrants
#pragma unroll
    for (int c = 0; c < NT * CWW; ++c) {
        const float gv = accg[c];
        accg[c] = __fdividef(gv, 1.0f + __expf(-gv)) * accu[c];
    }
    float mine = 0.f;  // the warp maximum of column lcol
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int c = 0; c < CWW; ++c) {
            const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(accg[t * CWW + c])));
            if (lane == t * CWW + c) mine = __uint_as_float(m);
        }
    const int rb = static_cast<int>(st.nred & 1u);
    float (*red)[Shape<MAXT>::NP] = ctl->red[st.team][rb];
    if (lserve) red[st.q][st.lcol] = mine;
    mbar_arrive(&ctl->red_bar[st.team][rb]);
    if (!wait_bar(&ctl->red_bar[st.team][rb], (st.nred >> 1) & 1u, &ctl->abort, p.status))
        return false;
    ++st.nred;
    float sl = 0.f, rl = 0.f;  // the scale of column lcol and RN(1 / scale)
    if (lserve) {
        const float amax = fmaxf(fmaxf(red[0][st.lcol], red[1][st.lcol]),
                                 fmaxf(red[2][st.lcol], red[3][st.lcol]));
        sl = __fdiv_rn(amax, 448.f);
        rl = sl > 0.f ? __frcp_rn(sl) : 0.f;
    }
    if (st.q == 0 && lvalid) p.as[static_cast<size_t>(u.row0 + st.lcol) * ngi + u.tile] = sl;
    const int f = u.tile * WM + st.r;
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int c = 0; c < CWW; ++c) {
            const float sc = __shfl_sync(0xffffffffu, sl, t * CWW + c);
            const float rc = __shfl_sync(0xffffffffu, rl, t * CWW + c);
            const int col = t * TT + st.h2 * CWW + c;
            if (col < u.rows) {
                const uint8_t code = sc > 0.f
                    ? static_cast<uint8_t>(__nv_cvt_float_to_fp8(div_rn(accg[t * CWW + c], sc, rc),
                                                                 __NV_SATFINITE, __NV_E4M3))
                    : static_cast<uint8_t>(0);
                p.aq[static_cast<size_t>(u.row0 + col) * p.I + f] = code;
            }
        }
    if (u.last_pass) {
        // publish the expert's act rows to the down items of other CTAs:
        // every thread fences its stores (also towards the async proxy that
        // the TMA reads use) and arrives; one thread waits for all (bounded)
        // and releases the per-expert counter
        fence_proxy_async_global();
        __threadfence();
        mbar_arrive(&ctl->pub[st.team]);
        const bool lead = Shape<MAXT>::TEAMS == 2 ? (st.ew & 3) == 0 : st.ew == 0;
        if (lead && lane == 0) {  // the team's first warp
            if (wait_bar(&ctl->pub[st.team], st.npub & 1u, &ctl->abort, p.status)) {
                __threadfence();
                atomicAdd(done + u.e, 1);
            }
        }
        ++st.npub;
    }
    return true;
}

template <int MAXT>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_experts_kernel(const __grid_constant__ Fp8Maps maps, Fp8ExpertParams p) {
    constexpr int NP = Shape<MAXT>::NP, NBUF = Shape<MAXT>::NBUF;
    constexpr int BUF_COLS = Shape<MAXT>::BUF_COLS, STAGE_BYTES = Shape<MAXT>::STAGE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Ctl<MAXT> *ctl = reinterpret_cast<Ctl<MAXT> *>(smem + STAGES * STAGE_BYTES);
    int32_t *offs = reinterpret_cast<int32_t *>(ctl + 1);  // [E+1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int n_gu_tiles = p.I / WM;
    const int n_dn_tiles = p.d / WM;
    const int total = E * (n_gu_tiles + n_dn_tiles);
    int *next_item = p.sched;     // claimed-item counter
    int *done = p.sched + 1;      // [E] finished gate/up items per expert

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], Shape<MAXT>::TEAM_THREADS / 32);  // the consuming team's warps
        }
        for (int r = 0; r < RING; ++r) {
            mbar_init(&ctl->ufull[r], 1);
            mbar_init(&ctl->uempty[r], 1 + kEpiThreads);  // the MMA thread, every epilogue thread
        }
        for (int t = 0; t < Shape<MAXT>::TEAMS; ++t) {
            mbar_init(&ctl->pub[t], Shape<MAXT>::TEAM_THREADS);
            mbar_init(&ctl->red_bar[t][0], Shape<MAXT>::TEAM_THREADS);
            mbar_init(&ctl->red_bar[t][1], Shape<MAXT>::TEAM_THREADS);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&maps.w_gate_up);
        tma_prefetch_desc(&maps.w_down);
        tma_prefetch_desc(&maps.xq);
        tma_prefetch_desc(&maps.aq);
    }
    pdl_trigger();
    pdl_wait();
    for (int i = threadIdx.x; i <= E; i += kThreads) offs[i] = p.offsets[i];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------- producer -------------------------
            int s = 0;
            uint32_t ph = 0;
            int useq = 0;
            bool issued[STAGES];
            uint32_t issued_parity[STAGES];
            for (int i = 0; i < STAGES; ++i) issued[i] = false;
            bool ok = true;
            int nitem = 0;  // items with tokens claimed by this CTA
            while (ok && !aborted(&ctl->abort)) {
                const int item = atomicAdd(next_item, 1);
                const bool stop = item >= total;
                int npass = 0, team = 0;
                Unit u0;
                if (!stop) {
                    u0 = decode<MAXT>(item, 0, n_gu_tiles, n_dn_tiles, E, offs);
                    const int cnt = offs[u0.e + 1] - offs[u0.e];
                    if (cnt <= 0) continue;  // expert without tokens: nothing to do
                    npass = (cnt + NP - 1) / NP;
                    // every pass of an item goes to one epilogue team, whose
                    // fence at the last pass then covers all the item's rows
                    team = nitem++ % Shape<MAXT>::TEAMS;
                    // the item's weight block scales, for the epilogue units to come
                    const int ngd = p.d / kFp8Block, ngi = p.I / kFp8Block;
                    if (u0.gate_up) {
                        const float *sg = p.sgu + (static_cast<size_t>(u0.e) * (2 * n_gu_tiles) + u0.tile) * ngd;
                        prefetch_l2(sg, ngd * 4);
                        prefetch_l2(sg + static_cast<size_t>(n_gu_tiles) * ngd, ngd * 4);
                    } else {
                        prefetch_l2(p.sdn + (static_cast<size_t>(u0.e) * n_dn_tiles + u0.tile) * ngi, ngi * 4);
                    }
                    if (!u0.gate_up) {
                        // the expert's act rows must be complete: all its gate/up items
                        const uint64_t dl = globaltimer_ns() + kWaitNs;
                        uint32_t it = 0;
                        while (ld_acquire(done + u0.e) < n_gu_tiles) {
                            if ((++it & 255u) == 0 && globaltimer_ns() > dl) {
                                set_status(p.status, kStatusTimeout);
                                atomicExch(&ctl->abort, 1);
                                ok = false;
                                break;
                            }
                        }
                        if (!ok) break;
                        fence_proxy_async_global();  // aq was written by generic stores
                    }
                }
                for (int pass = 0; pass < (stop ? 1 : npass); ++pass) {
                    const int slot = useq % RING;
                    if (!wait_bar(&ctl->uempty[slot], ((useq / RING) & 1u) ^ 1u, &ctl->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    ctl->ring_item[slot] = stop ? -1 : item;
                    ctl->ring_pass[slot] = pass;
                    ctl->ring_team[slot] = team;
                    mbar_arrive(&ctl->ufull[slot]);
                    ++useq;
                    if (stop) break;
                    const Unit u = decode<MAXT>(item, pass, n_gu_tiles, n_dn_tiles, E, offs);
                    const int nk = (u.gate_up ? p.d : p.I) / BK;
                    const uint32_t bytes = (u.gate_up ? 2 * A_BYTES : A_BYTES) + u.ntt * B_TILE;
                    for (int kb = 0; kb < nk; ++kb) {
                        if (!wait_bar(&ctl->empty[s], ph ^ 1u, &ctl->abort, p.status)) { ok = false; break; }
                        uint8_t *sa = smem + s * STAGE_BYTES;
                        uint8_t *sb = sa + 2 * A_BYTES;
                        mbar_arrive_expect_tx(&ctl->full[s], bytes);
                        if (u.gate_up) {
                            const int rg = u.e * 2 * p.I + u.tile * WM;
                            tma_load_2d(sa, &maps.w_gate_up, kb * BK, rg, &ctl->full[s]);
                            tma_load_2d(sa + A_BYTES, &maps.w_gate_up, kb * BK, rg + p.I, &ctl->full[s]);
                            for (int t = 0; t < u.ntt; ++t)
                                tma_load_2d(sb + t * B_TILE, &maps.xq, kb * BK, u.row0 + t * TT, &ctl->full[s]);
                        } else {
                            tma_load_2d(sa, &maps.w_down, kb * BK, u.e * p.d + u.tile * WM, &ctl->full[s]);
                            for (int t = 0; t < u.ntt; ++t)
                                tma_load_2d(sb + t * B_TILE, &maps.aq, kb * BK, u.row0 + t * TT, &ctl->full[s]);
                        }
                        issued[s] = true;
                        issued_parity[s] = ph;
                        if (++s == STAGES) { s = 0; ph ^= 1u; }
                    }
                    if (!ok) break;
                }
                if (stop) break;
            }
            if (!ok || aborted(&ctl->abort)) {
                // make the other roles leave, then let our own copies land
                atomicExch(&ctl->abort, 1);
                const uint64_t dl = globaltimer_ns() + kWaitNs;
                for (int i = 0; i < STAGES; ++i)
                    if (issued[i]) mbar_wait(&ctl->full[i], issued_parity[i], dl);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // --------------------------- MMA ----------------------------
            int s = 0;
            uint32_t ph = 0;
            int useq = 0;
            uint32_t nblk = 0;  // K blocks issued: buffer nblk % NBUF
            bool any = false, ok = true;
            while (ok && !aborted(&ctl->abort)) {
                const int slot = useq % RING;
                if (!wait_bar(&ctl->ufull[slot], (useq / RING) & 1u, &ctl->abort, p.status)) break;
                const int item = ctl->ring_item[slot], pass = ctl->ring_pass[slot];
                mbar_arrive(&ctl->uempty[slot]);
                ++useq;
                if (item < 0) break;
                const Unit u = decode<MAXT>(item, pass, n_gu_tiles, n_dn_tiles, E, offs);
                const uint32_t idesc = idesc_e4m3_f32(WM, TT * u.ntt);
                const int nk = (u.gate_up ? p.d : p.I) / BK;
                for (int kb = 0; kb < nk; ++kb) {
                    const int buf = static_cast<int>(nblk % NBUF);
                    const uint32_t use = nblk / NBUF;
                    if (!wait_bar(&ctl->tempty[buf], (use & 1u) ^ 1u, &ctl->abort, p.status)) { ok = false; break; }
                    if (!wait_bar(&ctl->full[s], ph, &ctl->abort, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d0 = tmem_base + static_cast<uint32_t>(buf * BUF_COLS);
                    const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
                    const uint32_t b0 = a0 + 2 * A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / UK; ++kk) {
                        const uint32_t acc = kk != 0 ? 1u : 0u;  // a fresh sum per K block
                        const uint64_t bd = sw128_kmajor_desc(b0 + kk * UK);
                        umma_e4m3(d0, sw128_kmajor_desc(a0 + kk * UK), bd, idesc, acc);
                        if (u.gate_up)  // up rows into columns NP..: same tokens, second weight tile
                            umma_e4m3(d0 + NP, sw128_kmajor_desc(a0 + A_BYTES + kk * UK), bd, idesc, acc);
                    }
                    any = true;
                    umma_commit(&ctl->empty[s]);
                    umma_commit(&ctl->tfull[buf]);
                    ++nblk;
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
            }
            if (any) {
                umma_commit(&ctl->drain);
                mbar_wait(&ctl->drain, 0, globaltimer_ns() + kWaitNs);
            }
        }
    } else {
        // ------------------------- epilogue -------------------------
        // thread <-> TMEM lane = weight row: warp w reads lanes 32*(w%4)..+31
        // and CWW columns of each token tile (from column h2 * CWW). Lane l
        // also serves one column for the lane-parallel work: lcol = tile
        // l / CWW, column h2 * CWW + l % CWW of that tile.
        constexpr int TEAMS = Shape<MAXT>::TEAMS, CWW = Shape<MAXT>::CWW;
        EpiState st;
        st.ew = warp - 2;
        st.q = warp & 3;
        st.team = TEAMS == 2 ? st.ew >> 2 : 0;
        st.h2 = TEAMS == 2 ? 0 : st.ew >> 2;
        st.r = st.q * 32 + lane;
        st.lt = lane / CWW;
        st.lcol = st.lt * TT + st.h2 * CWW + lane % CWW;
        st.tmem_base = tmem_base;
        st.nblk = st.npub = st.nred = 0;
        int useq = 0;
        bool ok = true;
        while (ok && !aborted(&ctl->abort)) {
            const int slot = useq % RING;
            if (!wait_bar(&ctl->ufull[slot], (useq / RING) & 1u, &ctl->abort, p.status)) break;
            const int item = ctl->ring_item[slot], pass = ctl->ring_pass[slot];
            const int team = ctl->ring_team[slot];
            mbar_arrive(&ctl->uempty[slot]);
            ++useq;
            if (item < 0) break;
            const Unit u = decode<MAXT>(item, pass, n_gu_tiles, n_dn_tiles, E, offs);
            if (team != st.team) {  // the other team's unit: skip its K blocks
                st.nblk += (u.gate_up ? p.d : p.I) / BK;
                continue;
            }
            if (MAXT == 2 && u.ntt == 2)
                ok = epi_unit<MAXT, MAXT>(u, ctl, p, st, n_gu_tiles, n_dn_tiles, done);
            else
                ok = epi_unit<MAXT, 1>(u, ctl, p, st, n_gu_tiles, n_dn_tiles, done);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <int MAXT>
size_t smem_bytes(int E) {
    return 1024 + STAGES * Shape<MAXT>::STAGE_BYTES + sizeof(Ctl<MAXT>) + (E + 1) * 4;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 2-D map of a row-major [rows][cols] byte matrix, box 128 bytes x box_rows,
// 128-byte swizzle, zero fill outside.
int encode_u8(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return MOE_ERR_CUDA;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = reinterpret_cast<EncodeTiledFn>(fn)(
        m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

struct Fp8MapsHolder {
    Fp8Maps m;
};

int fp8_build_maps(void **holder, const void *xq, const void *aq, const void *wgu,
                   const void *wd, int rows_cap, int E, int d, int I) {
    Fp8MapsHolder *h = new (std::nothrow) Fp8MapsHolder;
    if (!h) return MOE_ERR_OOM;
    int rc;
    if ((rc = encode_u8(&h->m.w_gate_up, wgu, static_cast<uint64_t>(E) * 2 * I, d, WM)) != MOE_OK ||
        (rc = encode_u8(&h->m.w_down, wd, static_cast<uint64_t>(E) * d, I, WM)) != MOE_OK ||
        (rc = encode_u8(&h->m.xq, xq, rows_cap, d, TT)) != MOE_OK ||
        (rc = encode_u8(&h->m.aq, aq, rows_cap, I, TT)) != MOE_OK) {
        delete h;
        return rc;
    }
    *holder = h;
    return MOE_OK;
}

void fp8_free_maps(void *holder) { delete static_cast<Fp8MapsHolder *>(holder); }

namespace {
template <int MAXT>
int launch_t(const Fp8MapsHolder *h, const Fp8ExpertParams &p, int n_sm, cudaStream_t s) {
    const size_t smem = smem_bytes<MAXT>(p.E);
    if (ensure_smem(fp8_experts_kernel<MAXT>, smem) != MOE_OK) return MOE_ERR_CUDA;
    // one CTA must fit an SM (registers and shared memory): checked once per size
    thread_local size_t checked = 0;
    if (checked != smem) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fp8_experts_kernel<MAXT>,
                                                          kThreads, smem) != cudaSuccess ||
            per_sm < 1)
            return MOE_ERR_CUDA;
        checked = smem;
    }
    return launch_k(fp8_experts_kernel<MAXT>, dim3(n_sm), dim3(kThreads), smem, s, h->m, p);
}
}  // namespace

int launch_fp8_experts(const void *holder, const Fp8ExpertParams &p, int n_sm, int pass_tokens,
                       cudaStream_t s) {
    const Fp8MapsHolder *h = static_cast<const Fp8MapsHolder *>(holder);
    return pass_tokens <= TT ? launch_t<1>(h, p, n_sm, s) : launch_t<2>(h, p, n_sm, s);
}

}  // namespace moe
