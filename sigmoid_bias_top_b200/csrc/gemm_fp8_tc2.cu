// gemm_fp8_tc2.cu -- the FP8_BLOCK expert GEMMs of large batches on CTA
// pairs (tcgen05.mma.cta_group::2.kind::f8f6f4), weights as the 256-row MMA
// operand and tokens as N ("swap AB"), one launch per contraction.
//
// The gated SiLU expert of "LFM2.5-24B-A2B: Biased Routing, Short Convolutions
// and Ten KV Caches" (flozi.net, English page, section "The router has two
// different scores") with the FP8_BLOCK storage of the FP8 checkpoint
// ("LFM2.5-24B-A2B: ein 24B-Reasoning-Modell, das pro Wortstück so wenig
// verbraucht wie ein 2B-Modell", inferencekey.com, section "Für Engineers",
// paragraph "Quantisierung": weights FP8 in static 128x128 blocks,
// activations FP8 dynamic per group of 128):
//   gate/up:  a32    = silu(xq . Wg) * (xq . Wu)        (fp32)
//   quantise: aq, as = Q(a32)  per token and group of 128 features
//   down:     y      = bf16( aq . Wd )
// where every product over one 128-wide K block carries the weight block's
// scale sw and the token group's scale sa.
//
// Tiles as in the bf16 pair kernel (gemm_tc2.cu): M = 256 weight rows per
// pair, 128 per CTA. gate/up: CTA h stages the gate and up rows of features
// f0+64h..+63 interleaved in 16-row groups (one 4-D TMA box), so its rows
// lie in two weight row blocks (the gate block and the up block of f0) and
// TMEM lanes l, l+16 of each quarter hold gate and up of one feature. down:
// CTA h stages Wd rows n0+128h..+127, one weight row block. N = the tokens of
// one token tile of an expert (equal tiles of at most 128, rounded to 16),
// N/2 token rows per CTA.
//
// The scales differ per K block, so the tensor cores cannot add one K block
// onto the next: each K block's four MMAs (K = 32) start a fresh sum in one
// of four 128-column TMEM buffers, and the epilogue warps (8 per CTA, two per
// TMEM lane quarter, 64 token columns each) load it and add
// partial * (sa[token][kb] * sw[kb]) into fp32 registers. The gate/up
// epilogue loads 16x256b fragments, in which a thread holds 4 rows x 16 token
// columns rather than 1 row x 64 columns, so it reads 16 factors per K block
// and fragment (sa * sw of the gate rows, then of the up rows) instead of 64;
// the down epilogue keeps one row per thread (32x32b) and reads the 64
// factors of its columns, which lets it store 32 consecutive outputs of a
// token per warp directly. An eleventh warp forms the factors of a chunk of
// 16 K blocks ahead (two chunk buffers), in the order the epilogue reads
// them, issuing all of a chunk's scale loads before using any; 11 warps keep
// the 168-register budget of 10 (the fullest of the four register-file
// quarters holds three warps). In a gate/up tile the lower fragment holds gate and the upper one
// up rows of the same features, so at the tile end each thread forms
// SiLU(gate) * up for its 32 values and stores them in fp32 (each warp store
// fills whole 32-byte sectors). A quantisation group of 128 features spans
// both CTAs of a pair, so its maximum, s = amax / 448 and the codes
// e4m3(a / s) (the IEEE quotient, by a reciprocal and one correction step:
// div_rn; nearest-even, saturating) are left to a separate memory-bound
// kernel (fp8_quantize_act_kernel): exchanging the maxima between the CTAs
// and quantising inside the tile kept the epilogue from the next tile's
// K blocks for longer than the whole quantisation pass takes.
// All waits are bounded (1 s) and report MOE_ERR_DEVICE_TIMEOUT; the pair
// meets at a cluster barrier before TMEM is freed. No load uses multicast.
#include <cooperative_groups.h>
#include <cuda_fp8.h>

#include <new>

#include "moe_fp8.cuh"

namespace cg = cooperative_groups;

namespace moe {
namespace {

constexpr int WM = 128;                  // weight rows per CTA (MMA M = 256 per pair)
constexpr int TN = kFp8PairTileM;        // most tokens per tile (MMA N)
constexpr int BK = kFp8Block;            // K per stage: one scale block, 128 bytes per row
constexpr int UK = 32;                   // K per tcgen05.mma kind::f8f6f4
constexpr int STAGES = 6;
constexpr int A_BYTES = WM * BK;         // 16 KB of weights
constexpr int B_ROWS = TN / 2;           // token rows per CTA
constexpr int B_BYTES = B_ROWS * BK;     // 8 KB of tokens
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NBUF = 4;                  // TMEM buffers of one K block each
constexpr int TMEM_COLS = NBUF * TN;     // 512
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kTblWarp = 2 + kEpiWarps;  // builds the tiles' factor tables
constexpr int kThreads = 64 + kEpiThreads + 32;
constexpr int CW = TN / 2;               // token columns per epilogue warp
constexpr int TBL = 16;                  // K blocks per chunk of the factor tables
constexpr int kEpiBar = 1;               // named barrier of the epilogue threads
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t kPeerBitMask = 0xFEFFFFFFu;  // shared::cluster address in the pair's even CTA

struct Ctl {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[NBUF];
    uint64_t tempty[NBUF];
    uint64_t tbl_full[2];       // a factor-table chunk is written
    uint64_t tbl_empty[2];      // every epilogue warp is done with it
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    // two chunks of promotion factors sa * sw, per K block of the chunk:
    // gate/up: [0] with the gate rows' weight block scale, [1] with the up
    // rows', each over the token columns in fragment order (frag_pos); down:
    // [0] over the token columns in column order
    alignas(16) float fac[2][TBL][2][TN];
};

// Position of token column c in a factor-table row: the epilogue thread with
// fragment column pair mq of column half ch reads its 16 columns
// ch*CW + 8 i + 2 mq + e (i < 8, e < 2) as 16 consecutive floats.
__device__ __forceinline__ int frag_pos(int c) {
    const int ch = c / CW, cc = c % CW;
    return ch * CW + ((cc & 7) >> 1) * 16 + 2 * (cc >> 3) + (cc & 1);
}

// tcgen05.ld .16x256b.x8: 16 TMEM lanes x 64 columns; thread t gets lane
// t/4 (registers 4i, 4i+1) and lane t/4 + 8 (4i+2, 4i+3) of columns
// 8 i + 2 (t % 4) + {0, 1}.
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void load_scales(float (&sv)[16], const float *src) {
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float4 v = s4[k];
        sv[4 * k + 0] = v.x;
        sv[4 * k + 1] = v.y;
        sv[4 * k + 2] = v.z;
        sv[4 * k + 3] = v.w;
    }
}

// acc[4i + 2h + e] += v[4i + 2h + e] * f[2i + e] (f = sa * sw, formed in fp32
// by the table warp)
__device__ __forceinline__ void promote(float (&acc)[32], const uint32_t (&v)[32],
                                        const float (&sv)[16]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float f = sv[2 * i + e];
            acc[4 * i + e] = fmaf(__uint_as_float(v[4 * i + e]), f, acc[4 * i + e]);
            acc[4 * i + 2 + e] = fmaf(__uint_as_float(v[4 * i + 2 + e]), f, acc[4 * i + 2 + e]);
        }
    }
}

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

__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *m, int x, int y,
                                                 uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar) & kPeerBitMask)
        : "memory");
}

// gate/up weight box {128 K bytes, 16 rows, gate|up, 4 row groups}; w = first group
__device__ __forceinline__ void tma_load_4d_pair(void *dst, const CUtensorMap *m, int x, int w,
                                                 uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(0), "r"(0), "r"(w),
        "r"(smem_u32(bar) & kPeerBitMask)
        : "memory");
}

__device__ __forceinline__ void umma_e4m3_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m;\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ uint32_t peer_addr(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}

// Arrival on the barrier at the same offset in CTA `rank`. It orders nothing
// beyond this thread's TMEM reads (fenced by the caller with
// tcgen05.fence::before_thread_sync), which is all a TMEM buffer release needs.
__device__ __forceinline__ void mbar_arrive_remote(uint64_t *bar, uint32_t rank) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(peer_addr(bar, rank))
                 : "memory");
}

// The epilogue threads meet and learn whether any of them passed `v`.
__device__ __forceinline__ bool epi_bar_or(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "n"(kEpiBar), "n"(kEpiThreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ int find_expert(const int32_t *mts, int E, int q) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mts[mid] <= q) lo = mid; else hi = mid - 1;
    }
    return lo;
}

struct Item {
    int e, wt, t0, rows, N;
};

// Expert-major items, the token tile fastest, so consecutive pairs share a
// weight tile in L2; an expert's c rows in ceil(c/TN) equal tiles rounded to 16.
__device__ __forceinline__ Item decode(int item, int NW, const int32_t *mts, const int32_t *offs,
                                       int E) {
    Item it;
    it.e = find_expert(mts, E, item / NW);
    const int ntt = mts[it.e + 1] - mts[it.e];
    const int local = item - mts[it.e] * NW;
    it.wt = local / ntt;
    const int tt = local - it.wt * ntt;
    const int c = offs[it.e + 1] - offs[it.e];
    const int ts = ((c + ntt - 1) / ntt + 15) & ~15;
    it.t0 = offs[it.e] + tt * ts;
    it.rows = min(ts, c - tt * ts);
    it.N = (it.rows + 15) & ~15;
    return it;
}

struct PairMaps {
    CUtensorMap w_gate_up_4d;  // e4m3 [E*2I][d] as {d, 16, 2, groups}, box 128 x 16 x 2 x 4
    CUtensorMap w_down;        // e4m3 [E*d][I], box 128 x 128
    CUtensorMap xq;            // e4m3 [rows][d], box 128 x 64
    CUtensorMap aq;            // e4m3 [rows][I], box 128 x 64
};

template <bool GATE_UP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    fp8_pair_kernel(const __grid_constant__ PairMaps maps, Fp8PairParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + STAGES * STAGE_BYTES);
    int32_t *mts = reinterpret_cast<int32_t *>(ctl + 1);  // [E+1]
    int32_t *offs = mts + (p.E + 1);                        // [E+1]

    cg::cluster_group cluster = cg::this_cluster();
    const int half = static_cast<int>(cluster.block_rank());
    const bool leader = half == 0;
    const int pair = blockIdx.x / 2, npairs = gridDim.x / 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 2 * kEpiWarps);  // one per epilogue warp of both CTAs
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tbl_full[b], 1);
            mbar_init(&ctl->tbl_empty[b], kEpiWarps);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&ctl->tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(GATE_UP ? &maps.w_gate_up_4d : &maps.w_down);
        tma_prefetch_desc(GATE_UP ? &maps.xq : &maps.aq);
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

    // weight tiles per expert: 128 features (gate/up) or 256 output rows (down;
    // with d % 256 == 128 the second CTA of an expert's last tile has no rows)
    const int NW = GATE_UP ? p.I / 128 : (p.d + 2 * WM - 1) / (2 * WM);
    const int K = GATE_UP ? p.d : p.I;
    const int nk = K / BK;
    const int total = mts[E] * NW;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_parity[STAGES];
            bool issued[STAGES];
            for (int i = 0; i < STAGES; ++i) issued[i] = false;
            const CUtensorMap *tm = GATE_UP ? &maps.xq : &maps.aq;
            for (int item = pair; item < total && !aborted(ctl); item += npairs) {
                const Item it = decode(item, NW, mts, offs, E);
                const int trow = it.t0 + half * (it.N / 2);
                const int wc = GATE_UP ? (it.e * 2 * p.I + it.wt * 128 + half * 64) / 16
                                       : it.e * p.d + it.wt * 2 * WM + half * WM;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_bar(&ctl->empty[s], ph ^ 1u, ctl, p.status)) { ok = false; break; }
                    uint8_t *sa = smem + s * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    if (leader) mbar_arrive_expect_tx(&ctl->full[s], 2 * STAGE_BYTES);
                    if (GATE_UP)
                        tma_load_4d_pair(sa, &maps.w_gate_up_4d, kb * BK, wc, &ctl->full[s]);
                    else
                        tma_load_2d_pair(sa, &maps.w_down, kb * BK, wc, &ctl->full[s]);
                    tma_load_2d_pair(sb, tm, kb * BK, trow, &ctl->full[s]);
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
            uint32_t ph = 0, nblk = 0;
            bool any = false;
            for (int item = pair; item < total && !aborted(ctl); item += npairs) {
                const Item it = decode(item, NW, mts, offs, E);
                const uint32_t idesc = idesc_e4m3_f32(2 * WM, it.N);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    const int buf = static_cast<int>(nblk % NBUF);
                    const uint32_t use = nblk / NBUF;
                    if (!wait_bar(&ctl->tempty[buf], (use & 1u) ^ 1u, ctl, p.status)) { ok = false; break; }
                    if (!wait_bar(&ctl->full[s], ph, ctl, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * TN);
                    const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
                    const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / UK; ++kk)  // a fresh sum per K block
                        umma_e4m3_pair(d_tmem, sw128_kmajor_desc(a0 + kk * UK),
                                       sw128_kmajor_desc(b0 + kk * UK), idesc, kk != 0 ? 1u : 0u);
                    any = true;
                    umma_commit_pair(&ctl->empty[s]);
                    umma_commit_pair(&ctl->tfull[buf]);
                    ++nblk;
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
            }
            if (any) {
                asm volatile(
                    "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                        smem_u32(&ctl->drain))
                    : "memory");
                mbar_wait(&ctl->drain, 0, globaltimer_ns() + kWaitNs);
            }
        }
    } else if (warp == kTblWarp) {
        // ---------------- scale tables (warp 10, both CTAs) ----------------
        // per chunk of TBL K blocks of every tile: sa[token][kb] of the tile's
        // TN token columns (lane l takes columns 4l..4l+3) and the weight
        // block scales (lane j < 16: the gate (or down) block of K block
        // kb0+j, lane 16+j the up one). All loads of a chunk are issued
        // before any is used.
        const float *sa_all = GATE_UP ? p.xs : p.as_in;
        const int ng = K / BK;
        uint32_t nchunk = 0;
        for (int item = pair; item < total && !aborted(ctl); item += npairs) {
            const Item it = decode(item, NW, mts, offs, E);
            const bool rows_ok = GATE_UP || it.wt * 2 + half < p.d / 128;
            const float *swg, *swu;
            if (GATE_UP) {
                const size_t rbg = static_cast<size_t>(it.e) * (2 * p.I / 128) + it.wt;
                swg = p.sgu + rbg * ng;
                swu = p.sgu + (rbg + p.I / 128) * ng;
            } else {
                swg = p.sdn + (static_cast<size_t>(it.e) * (p.d / 128) + (rows_ok ? it.wt * 2 + half : 0)) * ng;
                swu = swg;
            }
            bool ok = true;
            for (int kb0 = 0; kb0 < nk; kb0 += TBL, ++nchunk) {
                const int slot = static_cast<int>(nchunk & 1u);
                const bool got = wait_bar(&ctl->tbl_empty[slot], ((nchunk >> 1) & 1u) ^ 1u, ctl, p.status);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                const int n = min(TBL, nk - kb0);
                const int jj = lane & 15;
                const float wsc = jj < n ? __ldg((lane < 16 ? swg : swu) + kb0 + jj) : 0.f;
                float sa[4][TBL];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int col = 4 * lane + c;
                    const bool valid = rows_ok && col < it.rows;
                    const float *sa_row = sa_all + static_cast<size_t>(it.t0 + (valid ? col : 0)) * ng + kb0;
#pragma unroll
                    for (int j = 0; j < TBL; ++j) sa[c][j] = (valid && j < n) ? __ldg(sa_row + j) : 0.f;
                }
                if constexpr (GATE_UP) {
                    int pos[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) pos[c] = frag_pos(4 * lane + c);
#pragma unroll
                    for (int j = 0; j < TBL; ++j) {
                        const float wg = __shfl_sync(0xffffffffu, wsc, j);
                        const float wu = __shfl_sync(0xffffffffu, wsc, 16 + j);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            ctl->fac[slot][j][0][pos[c]] = sa[c][j] * wg;
                            ctl->fac[slot][j][1][pos[c]] = sa[c][j] * wu;
                        }
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < TBL; ++j) {
                        const float w = __shfl_sync(0xffffffffu, wsc, j);
                        *reinterpret_cast<float4 *>(&ctl->fac[slot][j][0][4 * lane]) =
                            make_float4(sa[0][j] * w, sa[1][j] * w, sa[2][j] * w, sa[3][j] * w);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->tbl_full[slot]);
            }
            if (!ok) break;
        }
    } else {
        // ---------------- epilogue (warps 2..9, both CTAs) ----------------
        // Warp (q, ch) owns TMEM lane quarter q and token columns ch*CW..+CW-1.
        // gate/up reads them as two 16x256b fragments: lanes 32q..+15 (gate
        // rows of the quarter's 16 features) and 32q+16..+31 (the up rows of
        // the same features), so a thread holds, for fragment rows fr and
        // fr + 8, 16 token columns ch*CW + 8 i + 2 mq + e of both: 16 factors
        // per K block and fragment instead of one per column. down reads one
        // row per thread (32x32b: lane 32q + lane, 64 columns).
        const int ew = warp - 2;
        const int q = warp & 3;          // TMEM lane quarter
        const int ch = ew >> 2;          // token columns ch*CW .. +CW-1
        const int mq = lane & 3;         // column pair of each 8 columns
        const int fr = lane >> 2;        // fragment rows fr and fr + 8
        // The epilogue threads agree at the start of every tile whether to
        // stop (the abort flag), so they leave the tile loop together; a wait
        // that times out inside a tile skips the rest of its work.
        uint32_t nblk = 0, ntile = 0, nchunk = 0;
        for (int item = pair; item < total; item += npairs, ++ntile) {
            if (epi_bar_or(aborted(ctl))) break;
            const Item it = decode(item, NW, mts, offs, E);
            // this CTA's weight rows exist (always for gate/up; for down, row
            // block 2 wt + half must lie inside the expert's d rows)
            const bool rows_ok = GATE_UP || it.wt * 2 + half < p.d / 128;
            const bool has_cols = ch * CW < it.N;
            if constexpr (!GATE_UP) {
                // down: a thread owns TMEM lane (output row) 32 q + lane and
                // token columns ch*CW..+CW-1 (32x32b loads); its factors are the
                // table's sa * sw of those columns, in column order
                float acc[CW];
#pragma unroll
                for (int j = 0; j < CW; ++j) acc[j] = 0.f;
                const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                        static_cast<uint32_t>(ch * CW);
                bool ok = true;
                int tslot = 0;
                uint32_t v0[32], v1[32];
                {
                    const int buf = static_cast<int>(nblk % NBUF);
                    const bool got = wait_bar(&ctl->tfull[buf], (nblk / NBUF) & 1u, ctl, p.status);
                    if (!__all_sync(0xffffffffu, got)) ok = false;
                    tc_fence_after();
                    if (ok && has_cols) {
                        tmem_ld_32x32b_x32(t_lane + buf * TN, v0);
                        tmem_ld_wait(v0);
                    }
                }
                for (int kb = 0; kb < nk && ok; ++kb) {
                    if (kb % TBL == 0) {
                        tslot = static_cast<int>(nchunk & 1u);
                        const bool got = wait_bar(&ctl->tbl_full[tslot], (nchunk >> 1) & 1u, ctl, p.status);
                        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                    }
                    const int buf = static_cast<int>(nblk % NBUF);
                    const float4 *f4 = reinterpret_cast<const float4 *>(&ctl->fac[tslot][kb % TBL][0][ch * CW]);
                    if (has_cols) {
                        tmem_ld_32x32b_x32(t_lane + buf * TN + 32, v1);
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const float4 f = f4[j4];
                            acc[4 * j4 + 0] = fmaf(__uint_as_float(v0[4 * j4 + 0]), f.x, acc[4 * j4 + 0]);
                            acc[4 * j4 + 1] = fmaf(__uint_as_float(v0[4 * j4 + 1]), f.y, acc[4 * j4 + 1]);
                            acc[4 * j4 + 2] = fmaf(__uint_as_float(v0[4 * j4 + 2]), f.z, acc[4 * j4 + 2]);
                            acc[4 * j4 + 3] = fmaf(__uint_as_float(v0[4 * j4 + 3]), f.w, acc[4 * j4 + 3]);
                        }
                        tmem_ld_wait(v1);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(&ctl->tempty[buf], 0);  // the leader's barrier
                    ++nblk;
                    bool next = false;
                    if (kb + 1 < nk) {
                        const int nbuf = static_cast<int>(nblk % NBUF);
                        const bool got = wait_bar(&ctl->tfull[nbuf], (nblk / NBUF) & 1u, ctl, p.status);
                        if (!__all_sync(0xffffffffu, got)) ok = false;
                        tc_fence_after();
                        next = ok && has_cols;
                        if (next) tmem_ld_32x32b_x32(t_lane + nbuf * TN, v0);
                    }
                    if (has_cols) {
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const float4 f = f4[8 + j4];
                            acc[32 + 4 * j4 + 0] = fmaf(__uint_as_float(v1[4 * j4 + 0]), f.x, acc[32 + 4 * j4 + 0]);
                            acc[32 + 4 * j4 + 1] = fmaf(__uint_as_float(v1[4 * j4 + 1]), f.y, acc[32 + 4 * j4 + 1]);
                            acc[32 + 4 * j4 + 2] = fmaf(__uint_as_float(v1[4 * j4 + 2]), f.z, acc[32 + 4 * j4 + 2]);
                            acc[32 + 4 * j4 + 3] = fmaf(__uint_as_float(v1[4 * j4 + 3]), f.w, acc[32 + 4 * j4 + 3]);
                        }
                    }
                    if (kb % TBL == TBL - 1 || kb == nk - 1) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&ctl->tbl_empty[tslot]);
                        ++nchunk;
                    }
                    if (next) tmem_ld_wait(v0);
                }
                if (has_cols && rows_ok && ok) {
                    const int n = it.wt * 2 * WM + half * WM + q * 32 + lane;
                    const int lim = it.rows - ch * CW;
                    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.y) +
                                         static_cast<size_t>(it.t0 + ch * CW) * p.d + n;
#pragma unroll
                    for (int j = 0; j < CW; ++j) {
                        if (j < lim) *dst = __float2bfloat16_rn(acc[j]);
                        dst += p.d;
                    }
                }
            } else {
                // [4 i + 2 h + e]: fragment row fr + 8 h, column ch*CW + 8 i + 2 mq + e;
                // ag from lanes 32q + 0..15, au from lanes 32q + 16..31
                float ag[32], au[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    ag[j] = 0.f;
                    au[j] = 0.f;
                }
                const uint32_t t_lo = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                      static_cast<uint32_t>(ch * CW);
                const uint32_t t_hi = t_lo + (16u << 16);
                bool ok = true;
                int tslot = 0;
                // Software pipeline: the load of the upper fragment is in flight
                // while the lower one is promoted, and the lower fragment of K
                // block kb + 1 while the upper one of kb is.
                uint32_t vg[32], vu[32];
                {
                    const int buf = static_cast<int>(nblk % NBUF);
                    const bool got = wait_bar(&ctl->tfull[buf], (nblk / NBUF) & 1u, ctl, p.status);
                    if (!__all_sync(0xffffffffu, got)) ok = false;
                    tc_fence_after();
                    if (ok && has_cols) {
                        tmem_ld_16x256b_x8(t_lo + buf * TN, vg);
                        tmem_ld_wait(vg);
                    }
                }
                for (int kb = 0; kb < nk && ok; ++kb) {
                    if (kb % TBL == 0) {  // the next chunk of scales
                        tslot = static_cast<int>(nchunk & 1u);
                        const bool got = wait_bar(&ctl->tbl_full[tslot], (nchunk >> 1) & 1u, ctl, p.status);
                        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                    }
                    const int buf = static_cast<int>(nblk % NBUF);
                    const float *fgk = &ctl->fac[tslot][kb % TBL][0][ch * CW + mq * 16];
                    const float *fuk = &ctl->fac[tslot][kb % TBL][1][ch * CW + mq * 16];
                    if (has_cols) {
                        tmem_ld_16x256b_x8(t_hi + buf * TN, vu);
                        float sv[16];
                        load_scales(sv, fgk);
                        promote(ag, vg, sv);
                        tmem_ld_wait(vu);
                    }
                    // both fragments of this K block are in registers: its buffer is free
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(&ctl->tempty[buf], 0);  // the leader's barrier
                    ++nblk;
                    bool next = false;
                    if (kb + 1 < nk) {
                        const int nbuf = static_cast<int>(nblk % NBUF);
                        const bool got = wait_bar(&ctl->tfull[nbuf], (nblk / NBUF) & 1u, ctl, p.status);
                        if (!__all_sync(0xffffffffu, got)) ok = false;
                        tc_fence_after();
                        next = ok && has_cols;
                        if (next) tmem_ld_16x256b_x8(t_lo + nbuf * TN, vg);
                    }
                    if (has_cols) {
                        float sv[16];  // read again rather than held across the next load
                        load_scales(sv, fuk);
                        promote(au, vu, sv);
                    }
                    if (kb % TBL == TBL - 1 || kb == nk - 1) {  // done with this chunk of scales
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&ctl->tbl_empty[tslot]);
                        ++nchunk;
                    }
                    if (next) tmem_ld_wait(vg);
                }
                // gate/up tile end: a = SiLU(gate) * up of fragment rows fr, fr + 8
                // (features 16 q + fr + 8 h of this CTA's 64) to a32 in fp32;
                // a warp's store covers 8 consecutive features (one 32-byte
                // sector) of 4 tokens
                if (has_cols && ok) {
                    float *abase = p.a32 + static_cast<size_t>(it.t0) * p.I + it.wt * 128 +
                                   half * 64 + q * 16 + fr;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int c = ch * CW + 8 * i + 2 * mq + e;
                            if (c < it.rows) {
                                float *row = abase + static_cast<size_t>(c) * p.I;
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    const float g = ag[4 * i + 2 * h + e];
                                    row[8 * h] = __fdividef(g, 1.0f + __expf(-g)) * au[4 * i + 2 * h + e];
                                }
                            }
                        }
                    }
                }
            }  // gate/up
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster.sync();  // the leader's MMAs into this CTA's TMEM and the peer's DSMEM writes are done
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

// The e4m3 quantisation of SiLU(gate)*up per token and group of 128
// features: a warp takes kQU groups of a row at a time (all loaded before any
// is used), lane l holding features 4l..4l+3 of a group; amax = the group
// maximum of |a|, s = amax / 448 and the codes e4m3(a / s) (both the IEEE
// quotient, by div_rn; nearest-even, saturating), s to as.
constexpr int kQU = 4;
__global__ void __launch_bounds__(256) fp8_quantize_act_kernel(Fp8PairParams p) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int ngo = p.I / kFp8Block;
    const int nch = (ngo + kQU - 1) / kQU;  // chunks of kQU groups per row
    const int units = p.offsets[p.E] * nch;
    const int nwarps = gridDim.x * (blockDim.x / 32);
    const float r448 = __frcp_rn(448.f);
    for (int u = (blockIdx.x * blockDim.x + threadIdx.x) / 32; u < units; u += nwarps) {
        const int r = u / nch, g0 = (u - r * nch) * kQU;
        const float *src = p.a32 + static_cast<size_t>(r) * p.I + 4 * lane;
        uint8_t *dst = p.aq + static_cast<size_t>(r) * p.I + 4 * lane;
        {
            float4 v[kQU];
#pragma unroll
            for (int j = 0; j < kQU; ++j)
                v[j] = g0 + j < ngo ? *reinterpret_cast<const float4 *>(src + (g0 + j) * kFp8Block)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int j = 0; j < kQU; ++j) {
                float m = fmaxf(fmaxf(fabsf(v[j].x), fabsf(v[j].y)), fmaxf(fabsf(v[j].z), fabsf(v[j].w)));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if (g0 + j >= ngo) continue;
                const float sc = div_rn(m, 448.f, r448);
                uint32_t code = 0;
                if (sc > 0.f) {
                    // the group's divisor is tested once for its quotients
                    float4 q;
                    if (div_rn_step_ok(sc)) {
                        const float rc = __frcp_rn(sc);
                        const float2 qa = div_rn_step2(make_float2(v[j].x, v[j].y), sc, rc);
                        const float2 qb = div_rn_step2(make_float2(v[j].z, v[j].w), sc, rc);
                        q = make_float4(qa.x, qa.y, qb.x, qb.y);
                    } else {
                        q = make_float4(__fdiv_rn(v[j].x, sc), __fdiv_rn(v[j].y, sc),
                                        __fdiv_rn(v[j].z, sc), __fdiv_rn(v[j].w, sc));
                    }
                    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(q.x, q.y), __NV_SATFINITE, __NV_E4M3);
                    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(q.z, q.w), __NV_SATFINITE, __NV_E4M3);
                    code = lo | (hi << 16);
                }
                *reinterpret_cast<uint32_t *>(dst + (g0 + j) * kFp8Block) = code;
                if (lane == 0) p.as_out[static_cast<size_t>(r) * ngo + g0 + j] = sc;
            }
        }
    }
}

size_t smem_bytes(int E) {
    return 1024 + STAGES * STAGE_BYTES + sizeof(Ctl) + 2 * (E + 1) * sizeof(int32_t);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<EncodeTiledFn>(fn);
}

// byte matrix [rows][cols], box 128 bytes x box_rows, 128-byte swizzle, zero fill
int encode_u8_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn enc = encoder();
    if (!enc) return MOE_ERR_CUDA;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
               ? MOE_OK : MOE_ERR_CUDA;
}

// 4-D byte view of the packed gate/up codes [E*2I][d]: element (k, y, z, g) =
// row 16 g + y + z I, column k (gate row f, up row f + I); a {128, 16, 2, 4}
// box lands as 16 gate rows, the matching 16 up rows, ... (128 rows).
int encode_u8_gate_up_4d(CUtensorMap *m, const void *base, int E, int d, int I) {
    EncodeTiledFn enc = encoder();
    if (!enc) return MOE_ERR_CUDA;
    const uint64_t groups = (static_cast<uint64_t>(E) * 2 * I - I) / 16;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), 16, 2, groups};
    const cuuint64_t row = static_cast<cuuint64_t>(d);
    const cuuint64_t strides[3] = {row, row * static_cast<cuuint64_t>(I), row * 16};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(BK), 16, 2, 4};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
               ? MOE_OK : MOE_ERR_CUDA;
}

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

template <bool GATE_UP>
int launch(const PairMaps &m, const Fp8PairParams &p, int n_sm, cudaStream_t s) {
    auto kern = fp8_pair_kernel<GATE_UP>;
    const size_t smem = smem_bytes(p.E);
    if (ensure_smem(kern, smem) != MOE_OK) return MOE_ERR_CUDA;
    static int pairs = 0;  // per kernel, for the device model of the process
    if (pairs == 0) pairs = resident_pairs(reinterpret_cast<const void *>(kern), smem, n_sm);
    return launch_k(kern, dim3(2 * pairs), dim3(kThreads), smem, s, m, p);
}

}  // namespace

struct Fp8PairMapsHolder {
    PairMaps m;
};

int fp8_pair_build_maps(void **holder, const void *xq, const void *aq, const void *wgu,
                        const void *wd, int rows_cap, int E, int d, int I) {
    Fp8PairMapsHolder *h = new (std::nothrow) Fp8PairMapsHolder;
    if (!h) return MOE_ERR_OOM;
    int rc;
    if ((rc = encode_u8_gate_up_4d(&h->m.w_gate_up_4d, wgu, E, d, I)) != MOE_OK ||
        (rc = encode_u8_2d(&h->m.w_down, wd, static_cast<uint64_t>(E) * d, I, WM)) != MOE_OK ||
        (rc = encode_u8_2d(&h->m.xq, xq, rows_cap, d, B_ROWS)) != MOE_OK ||
        (rc = encode_u8_2d(&h->m.aq, aq, rows_cap, I, B_ROWS)) != MOE_OK) {
        delete h;
        return rc;
    }
    *holder = h;
    return MOE_OK;
}

void fp8_pair_free_maps(void *holder) { delete static_cast<Fp8PairMapsHolder *>(holder); }

int launch_fp8_pair_gate_up(const void *holder, const Fp8PairParams &p, int n_sm, cudaStream_t s) {
    return launch<true>(static_cast<const Fp8PairMapsHolder *>(holder)->m, p, n_sm, s);
}

int launch_fp8_pair_down(const void *holder, const Fp8PairParams &p, int n_sm, cudaStream_t s) {
    return launch<false>(static_cast<const Fp8PairMapsHolder *>(holder)->m, p, n_sm, s);
}

int launch_fp8_quantize_act(const Fp8PairParams &p, int n_sm, cudaStream_t s) {
    if (p.I % kFp8Block != 0) return MOE_ERR_INVALID_ARG;
    return launch_k(fp8_quantize_act_kernel, dim3(4 * n_sm), dim3(256), 0, s, p);
}

}  // namespace moe
