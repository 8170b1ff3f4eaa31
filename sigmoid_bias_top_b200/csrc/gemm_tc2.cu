// gemm_tc2.cu -- the row-tiled grouped expert GEMMs on CTA pairs
// (tcgen05.mma.cta_group::2): one MMA computes a 256-row x 256-column tile.
//
// The gated SiLU expert of "LFM2.5-24B-A2B: Biased Routing, Short Convolutions
// and Ten KV Caches" (flozi.net, English page, section "The router has two
// different scores") over the rows grouped by expert (section "What to verify
// in a deployment"), for batches with many rows per expert:
//   gate/up: act[r][f] = silu(xp[r] . Wg_e[f]) * (xp[r] . Wu_e[f])
//   down:    y[r][n]   = act[r] . Wd_e[n]
// A cluster of two CTAs shares each tile: CTA r of the pair stages 128 rows of
// the A operand (its half of M) and 128 rows of the B operand (its half of N:
// for gate/up the leader holds the gate rows and the peer the matching up
// rows, so accumulator columns 0..127 are gate and 128..255 up in both CTAs'
// TMEM). Per CTA a stage is 32 KB (A 16 KB + B 16 KB) instead of 48 KB for a
// 128 x 256 single-CTA tile, which cuts the L2-to-SM traffic per MMA by a
// third, and 6 stages fit.
//
// Both CTAs' TMA loads complete on the leader's full barrier (the leader
// expects the pair's bytes); the leader's single MMA thread issues the
// cta_group::2 MMAs and commits to both CTAs' barriers with
// tcgen05.commit.multicast::cluster (no load uses multicast). Each CTA's
// epilogue reads its own 128 TMEM lanes (its rows) and arrives remotely on the
// leader's accumulator-empty barrier. All waits are bounded (1 s) and report
// MOE_ERR_DEVICE_TIMEOUT; the pair meets at a cluster barrier before TMEM is
// freed.
#include <cooperative_groups.h>

#include "moe_internal.cuh"

namespace cg = cooperative_groups;

namespace moe {
namespace {

constexpr int BM = 128;      // rows per CTA (the pair: 256)
constexpr int PM = 2 * BM;   // rows per pair tile
constexpr int BN = 256;      // MMA N (each CTA stages 128 rows of B)
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = (BN / 2) * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 32 KB per CTA
constexpr int TMEM_COLS = 2 * BN;
constexpr int kThreads = 192;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t kPeerBitMask = 0xFEFFFFFFu;  // shared::cluster address of the pair's even CTA

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

__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *m, int x, int y,
                                                 uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar) & kPeerBitMask)
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

// Arrives on `bar` in both CTAs of the pair once the issued MMAs complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m;\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_remote(uint64_t *bar, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(bar)), "r"(rank));
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote)
                 : "memory");
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
    int e, nt, row0, rows;  // row0 / rows: this CTA's half of the pair tile
};

__device__ __forceinline__ Item decode(int item, int NT, const int32_t *mts, const int32_t *offs,
                                       int E, int half) {
    Item it;
    it.e = find_expert(mts, E, item / NT);
    const int mcount = mts[it.e + 1] - mts[it.e];
    const int local = item - mts[it.e] * NT;
    it.nt = local / mcount;
    const int m = local - it.nt * mcount;
    it.row0 = offs[it.e] + m * PM + half * BM;
    it.rows = max(0, min(BM, offs[it.e + 1] - it.row0));
    return it;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

template <bool GATE_UP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_tc2_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, GroupedParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + STAGES * STAGE_BYTES);
    int32_t *mts = reinterpret_cast<int32_t *>(ctl + 1);  // [E+1]
    int32_t *offs = mts + (p.E + 1);                        // [E+1]

    cg::cluster_group cluster = cg::this_cluster();
    const int half = static_cast<int>(cluster.block_rank());  // 0 = leader
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
            mbar_init(&ctl->tempty[b], 2 * 128);  // both CTAs' epilogue threads
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {  // same warp in both CTAs: one allocation for the pair
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&ctl->tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
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
    const int NT = GATE_UP ? (p.I + 127) / 128 : (p.d + BN - 1) / BN;
    const int K = GATE_UP ? p.d : p.I;
    const int nk = (K + BK - 1) / BK;
    const int total = mts[E] * NT;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_parity[STAGES];
            bool issued[STAGES];
            for (int i = 0; i < STAGES; ++i) issued[i] = false;
            for (int item = pair; item < total && !aborted(ctl); item += npairs) {
                const Item it = decode(item, NT, mts, offs, E, half);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_bar(&ctl->empty[s], ph ^ 1u, ctl, p.status)) { ok = false; break; }
                    uint8_t *sa = smem + s * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    if (leader) mbar_arrive_expect_tx(&ctl->full[s], 2 * STAGE_BYTES);
                    tma_load_2d_pair(sa, &tmA, kb * BK, it.row0, &ctl->full[s]);
                    int rb;
                    if (GATE_UP)  // leader: gate rows, peer: the matching up rows
                        rb = it.e * 2 * p.I + it.nt * 128 + (half ? p.I : 0);
                    else
                        rb = it.e * p.d + it.nt * BN + half * (BN / 2);
                    tma_load_2d_pair(sb, &tmB, kb * BK, rb, &ctl->full[s]);
                    issued[s] = true;
                    issued_parity[s] = ph;
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
            }
            if (aborted(ctl) && leader) {  // our copies complete on the leader's barriers
                const uint64_t dl = globaltimer_ns() + kWaitNs;
                for (int i = 0; i < STAGES; ++i)
                    if (issued[i]) mbar_wait(&ctl->full[i], issued_parity[i], dl);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------- MMA issuer (leader only) ----------------
            constexpr uint32_t idesc = idesc_bf16_f32(PM, BN);
            int s = 0;
            uint32_t ph = 0;
            int tile = 0;
            bool any = false;
            for (int item = pair; item < total && !aborted(ctl); item += npairs, ++tile) {
                const int buf = tile & 1;
                const uint32_t use = static_cast<uint32_t>(tile >> 1);
                if (!wait_bar(&ctl->tempty[buf], (use & 1u) ^ 1u, ctl, p.status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_bar(&ctl->full[s], ph, ctl, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
                    const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / UK; ++kk)
                        umma_bf16_pair(d_tmem, sw128_kmajor_desc(a0 + kk * UK * 2),
                                       sw128_kmajor_desc(b0 + kk * UK * 2), idesc,
                                       (kb | kk) != 0 ? 1u : 0u);
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
        // ---------------- epilogue (warps 2..5, both CTAs) ----------------
        const int q = warp & 3;
        const int r = q * 32 + lane;
        int tile = 0;
        for (int item = pair; item < total && !aborted(ctl); item += npairs, ++tile) {
            const int buf = tile & 1;
            const uint32_t use = static_cast<uint32_t>(tile >> 1);
            if (!wait_bar(&ctl->tfull[buf], use & 1u, ctl, p.status)) break;
            tc_fence_after();
            const Item it = decode(item, NT, mts, offs, E, half);
            const uint32_t t_row = tmem_base + static_cast<uint32_t>(buf * BN) +
                                   (static_cast<uint32_t>(q * 32) << 16);
            const bool valid = r < it.rows && it.row0 + r < p.rows_cap;
            __nv_bfloat16 *crow = static_cast<__nv_bfloat16 *>(p.c) +
                                  static_cast<size_t>(valid ? it.row0 + r : 0) * NOUT;
            if (GATE_UP) {
#pragma unroll 1
                for (int c = 0; c < 128; c += 32) {
                    uint32_t g[32], u[32];
                    tmem_ld_32x32b_x32(t_row + c, g);
                    tmem_ld_32x32b_x32(t_row + 128 + c, u);
                    tmem_ld_wait();
                    const int f0 = it.nt * 128 + c;
                    if (valid) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            if (f0 + v * 8 + 8 <= NOUT) {
                                uint4 o;
                                o.x = pack_bf16x2(silu_mul(__uint_as_float(g[v * 8 + 0]), __uint_as_float(u[v * 8 + 0])),
                                                  silu_mul(__uint_as_float(g[v * 8 + 1]), __uint_as_float(u[v * 8 + 1])));
                                o.y = pack_bf16x2(silu_mul(__uint_as_float(g[v * 8 + 2]), __uint_as_float(u[v * 8 + 2])),
                                                  silu_mul(__uint_as_float(g[v * 8 + 3]), __uint_as_float(u[v * 8 + 3])));
                                o.z = pack_bf16x2(silu_mul(__uint_as_float(g[v * 8 + 4]), __uint_as_float(u[v * 8 + 4])),
                                                  silu_mul(__uint_as_float(g[v * 8 + 5]), __uint_as_float(u[v * 8 + 5])));
                                o.w = pack_bf16x2(silu_mul(__uint_as_float(g[v * 8 + 6]), __uint_as_float(u[v * 8 + 6])),
                                                  silu_mul(__uint_as_float(g[v * 8 + 7]), __uint_as_float(u[v * 8 + 7])));
                                *reinterpret_cast<uint4 *>(crow + f0 + v * 8) = o;
                            }
                        }
                    }
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    uint32_t a[32];
                    tmem_ld_32x32b_x32(t_row + c, a);
                    tmem_ld_wait();
                    const int n0 = it.nt * BN + c;
                    if (valid) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            if (n0 + v * 8 + 8 <= NOUT) {
                                uint4 o;
                                o.x = pack_bf16x2(__uint_as_float(a[v * 8 + 0]), __uint_as_float(a[v * 8 + 1]));
                                o.y = pack_bf16x2(__uint_as_float(a[v * 8 + 2]), __uint_as_float(a[v * 8 + 3]));
                                o.z = pack_bf16x2(__uint_as_float(a[v * 8 + 4]), __uint_as_float(a[v * 8 + 5]));
                                o.w = pack_bf16x2(__uint_as_float(a[v * 8 + 6]), __uint_as_float(a[v * 8 + 7]));
                                *reinterpret_cast<uint4 *>(crow + n0 + v * 8) = o;
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive_remote(&ctl->tempty[buf], 0);  // the leader's barrier
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

size_t smem_bytes(int E) {
    return 1024 + STAGES * STAGE_BYTES + sizeof(Ctl) + 2 * (E + 1) * sizeof(int32_t);
}

// CTA pairs that can be resident at once (an SM left without a partner in its
// GPC cannot host half a pair), at most one per two SMs.
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
int launch(const CUtensorMap &a, const CUtensorMap &b, const GroupedParams &p, int n_sm,
           cudaStream_t s) {
    auto kern = grouped_tc2_kernel<GATE_UP>;
    const size_t smem = smem_bytes(p.E);
    if (ensure_smem(kern, smem) != MOE_OK) return MOE_ERR_CUDA;
    static int pairs[2] = {0, 0};  // per kernel; the same device model throughout a process
    if (pairs[GATE_UP] == 0)
        pairs[GATE_UP] = resident_pairs(reinterpret_cast<const void *>(kern), smem, n_sm);
    return launch_k(kern, dim3(2 * pairs[GATE_UP]), dim3(kThreads), smem, s, a, b, p);
}

}  // namespace

int launch_gemm_tc2_gate_up(const TcMaps &m, const GroupedParams &p, int n_sm, cudaStream_t s) {
    return launch<true>(m.a_gate_up, m.w_gate_up, p, n_sm, s);
}

int launch_gemm_tc2_down(const TcMaps &m, const GroupedParams &p, int n_sm, cudaStream_t s) {
    return launch<false>(m.a_down, m.w_down_half, p, n_sm, s);
}

}  // namespace moe
