// gemm_decode.cu -- both expert contractions of a small batch in ONE persistent
// kernel, weights as the tensor-core M operand ("swap-AB").
//
// The gated SiLU expert of "LFM2.5-24B-A2B: Biased Routing, Short Convolutions
// and Ten KV Caches" (flozi.net, English page, section "The router has two
// different scores") over tokens grouped by expert (section "What to verify in
// a deployment"). With few tokens per expert (decoding: 1-30), the time is the
// stream of the active experts' weights through HBM; the design keeps that
// stream dense and evenly spread over the SMs:
//   * a work item is one 128-row weight tile: gate/up item (e, ft) = gate rows
//     ft*128.. and the matching up rows of expert e, K = d; down item (e, nt) =
//     rows nt*128.. of Wd_e, K = I. Each is an MMA with M = 128 weight rows and
//     N = 32 or 64 tokens (the expert's grouped rows), so a stage holds 32 KB
//     (gate/up) or 16 KB (down) of weights and 4-8 KB of tokens: 5 stages;
//   * items are taken from one atomic counter (all gate/up items, expert-major,
//     then all down items), so the SMs finish within about one item of each
//     other and the down items fill the tail of the gate/up work;
//   * a down item of expert e first waits until all I/128 gate/up items of e
//     have published their act rows (per-expert counter, release/acquire, plus
//     a generic-to-async proxy fence before its TMA reads them). Items are
//     claimed in order and only depend on earlier items, which running CTAs
//     own and finish without waiting, so the waits always end.
// Roles per CTA (192 threads): warp 0 lane 0 claims items, waits for
// dependencies and issues TMA; warp 1 allocates TMEM (2 x 128 columns) and one
// thread issues tcgen05.mma (kind::f16, M128, N32/N64, K16) and commits;
// warps 2..5 drain the accumulators (tcgen05.ld 32x32b), apply SiLU(gate)*up
// (gate/up) and store bf16 rows. Units (item, pass of up to 64 tokens) travel
// from the producer to the MMA and epilogue warps through a 4-slot ring in
// shared memory guarded by mbarriers. All waits are bounded (1 s) and report
// MOE_ERR_DEVICE_TIMEOUT; on time-out the kernel drains its own copies and
// MMAs, frees TMEM and returns.
#include <new>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int WM = 128;              // weight rows per item (MMA M)
constexpr int TT = 32;               // tokens per token tile
constexpr int MAXT = 2;              // token tiles per pass (N = 32 or 64)
constexpr int BK = 64;               // K per stage (128-byte swizzle rows)
constexpr int UK = 16;
constexpr int STAGES = 5;
constexpr int A_BYTES = WM * BK * 2;                    // 16 KB weight tile
constexpr int B_TILE = TT * BK * 2;                     // 4 KB token tile
constexpr int STAGE_BYTES = 2 * A_BYTES + MAXT * B_TILE;  // 40 KB
constexpr int BUF_COLS = 128;        // TMEM columns per accumulator buffer
constexpr int TMEM_COLS = 2 * BUF_COLS;
constexpr int RING = 4;
constexpr int kThreads = 192;
constexpr uint64_t kWaitNs = 1000000000ull;

struct Ctl {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t ufull[RING];
    uint64_t uempty[RING];
    uint64_t pub;    // every epilogue thread's act rows of an item are stored
    uint64_t drain;
    int ring_item[RING];
    int ring_pass[RING];
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

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
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

__device__ __forceinline__ Unit decode(int item, int pass, int n_gu_tiles, int n_dn_tiles, int E,
                                       const int32_t *offs) {
    Unit u;
    const int n_gu = E * n_gu_tiles;
    u.gate_up = item < n_gu;
    const int local = u.gate_up ? item : item - n_gu;
    const int per = u.gate_up ? n_gu_tiles : n_dn_tiles;
    u.e = local / per;
    u.tile = local - u.e * per;
    const int beg = offs[u.e], cnt = offs[u.e + 1] - beg;
    u.row0 = beg + pass * (TT * MAXT);
    u.rows = min(TT * MAXT, cnt - pass * (TT * MAXT));
    u.ntt = (u.rows + TT - 1) / TT;
    u.last_pass = (pass + 1) * (TT * MAXT) >= cnt;
    return u;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

struct DecodeMaps {
    CUtensorMap w_gate_up;  // [E*2I][d] box 64 x 128
    CUtensorMap w_down;     // [E*d][I]  box 64 x 128
    CUtensorMap xp;         // [rows][d] box 64 x 32
    CUtensorMap act;        // [rows][I] box 64 x 32
};

__global__ void __launch_bounds__(kThreads, 1)
    decode_experts_kernel(const __grid_constant__ DecodeMaps maps, DecodeParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + STAGES * STAGE_BYTES);
    int32_t *offs = reinterpret_cast<int32_t *>(ctl + 1);  // [E+1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int n_gu_tiles = (p.I + WM - 1) / WM;
    const int n_dn_tiles = (p.d + WM - 1) / WM;
    const int total = E * (n_gu_tiles + n_dn_tiles);
    int *next_item = p.sched;     // claimed-item counter
    int *done = p.sched + 1;      // [E] finished gate/up items per expert

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 128);
        }
        for (int r = 0; r < RING; ++r) {
            mbar_init(&ctl->ufull[r], 1);
            mbar_init(&ctl->uempty[r], 1 + 128);  // the MMA thread and every epilogue thread
        }
        mbar_init(&ctl->pub, 128);
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
        tma_prefetch_desc(&maps.xp);
        tma_prefetch_desc(&maps.act);
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
            while (ok && !aborted(ctl)) {
                const int item = atomicAdd(next_item, 1);
                const bool stop = item >= total;
                int npass = 0;
                Unit u0;
                if (!stop) {
                    u0 = decode(item, 0, n_gu_tiles, n_dn_tiles, E, offs);
                    const int cnt = offs[u0.e + 1] - offs[u0.e];
                    if (cnt <= 0) continue;  // expert without tokens: nothing to do
                    npass = (cnt + TT * MAXT - 1) / (TT * MAXT);
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
                        fence_proxy_async_global();  // act was written by generic stores
                    }
                }
                for (int pass = 0; pass < (stop ? 1 : npass); ++pass) {
                    const int slot = useq % RING;
                    if (!wait_bar(&ctl->uempty[slot], ((useq / RING) & 1u) ^ 1u, ctl, p.status)) {
                        ok = false;
                        break;
                    }
                    ctl->ring_item[slot] = stop ? -1 : item;
                    ctl->ring_pass[slot] = pass;
                    mbar_arrive(&ctl->ufull[slot]);
                    ++useq;
                    if (stop) break;
                    const Unit u = decode(item, pass, n_gu_tiles, n_dn_tiles, E, offs);
                    const int K = u.gate_up ? p.d : p.I;
                    const int nk = (K + BK - 1) / BK;
                    const uint32_t bytes = (u.gate_up ? 2 * A_BYTES : A_BYTES) + u.ntt * B_TILE;
                    for (int kb = 0; kb < nk; ++kb) {
                        if (!wait_bar(&ctl->empty[s], ph ^ 1u, ctl, p.status)) { ok = false; break; }
                        uint8_t *sa = smem + s * STAGE_BYTES;
                        uint8_t *sb = sa + 2 * A_BYTES;
                        mbar_arrive_expect_tx(&ctl->full[s], bytes);
                        if (u.gate_up) {
                            const int rg = u.e * 2 * p.I + u.tile * WM;
                            tma_load_2d(sa, &maps.w_gate_up, kb * BK, rg, &ctl->full[s]);
                            tma_load_2d(sa + A_BYTES, &maps.w_gate_up, kb * BK, rg + p.I, &ctl->full[s]);
                            for (int t = 0; t < u.ntt; ++t)
                                tma_load_2d(sb + t * B_TILE, &maps.xp, kb * BK, u.row0 + t * TT, &ctl->full[s]);
                        } else {
                            tma_load_2d(sa, &maps.w_down, kb * BK, u.e * p.d + u.tile * WM, &ctl->full[s]);
                            for (int t = 0; t < u.ntt; ++t)
                                tma_load_2d(sb + t * B_TILE, &maps.act, kb * BK, u.row0 + t * TT, &ctl->full[s]);
                        }
                        issued[s] = true;
                        issued_parity[s] = ph;
                        if (++s == STAGES) { s = 0; ph ^= 1u; }
                    }
                    if (!ok) break;
                }
                if (stop) break;
            }
            if (!ok || aborted(ctl)) {
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
            bool any = false;
            while (!aborted(ctl)) {
                const int slot = useq % RING;
                if (!wait_bar(&ctl->ufull[slot], (useq / RING) & 1u, ctl, p.status)) break;
                const int item = ctl->ring_item[slot], pass = ctl->ring_pass[slot];
                mbar_arrive(&ctl->uempty[slot]);
                if (item < 0) break;
                const Unit u = decode(item, pass, n_gu_tiles, n_dn_tiles, E, offs);
                const int buf = useq & 1;
                const uint32_t use = static_cast<uint32_t>(useq >> 1);
                ++useq;
                if (!wait_bar(&ctl->tempty[buf], (use & 1u) ^ 1u, ctl, p.status)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + static_cast<uint32_t>(buf * BUF_COLS);
                const uint32_t idesc = idesc_bf16_f32(WM, TT * u.ntt);
                const int K = u.gate_up ? p.d : p.I;
                const int nk = (K + BK - 1) / BK;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_bar(&ctl->full[s], ph, ctl, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
                    const uint32_t b0 = a0 + 2 * A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / UK; ++kk) {
                        const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
                        const uint64_t bd = sw128_kmajor_desc(b0 + kk * UK * 2);
                        umma_bf16(d0, sw128_kmajor_desc(a0 + kk * UK * 2), bd, idesc, acc);
                        if (u.gate_up)  // up rows into columns 64..: same tokens, second weight tile
                            umma_bf16(d0 + BUF_COLS / 2, sw128_kmajor_desc(a0 + A_BYTES + kk * UK * 2),
                                      bd, idesc, acc);
                    }
                    any = true;
                    umma_commit(&ctl->empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&ctl->tfull[buf]);
            }
            if (any) {
                umma_commit(&ctl->drain);
                mbar_wait(&ctl->drain, 0, globaltimer_ns() + kWaitNs);
            }
        }
    } else {
        // ------------------------- epilogue -------------------------
        // thread <-> TMEM lane = weight row: warp w reads lanes 32*(w%4)..+31
        const int q = warp & 3;
        const int r = q * 32 + lane;
        int useq = 0;
        uint32_t npub = 0;  // publishes done (phase of ctl->pub)
        while (!aborted(ctl)) {
            const int slot = useq % RING;
            if (!wait_bar(&ctl->ufull[slot], (useq / RING) & 1u, ctl, p.status)) break;
            const int item = ctl->ring_item[slot], pass = ctl->ring_pass[slot];
            mbar_arrive(&ctl->uempty[slot]);
            if (item < 0) break;
            const Unit u = decode(item, pass, n_gu_tiles, n_dn_tiles, E, offs);
            const int buf = useq & 1;
            const uint32_t use = static_cast<uint32_t>(useq >> 1);
            ++useq;
            if (!wait_bar(&ctl->tfull[buf], use & 1u, ctl, p.status)) break;
            tc_fence_after();
            const uint32_t t0 = tmem_base + static_cast<uint32_t>(buf * BUF_COLS) +
                                (static_cast<uint32_t>(q * 32) << 16);
            const int ncol = u.gate_up ? p.I : p.d;     // output row width
            const int f = u.tile * WM + r;              // output column of this thread
            __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(u.gate_up ? p.act : p.y);
            for (int t = 0; t < u.ntt; ++t) {
                uint32_t g[32], v[32];
                tmem_ld_32x32b_x32(t0 + t * TT, g);
                if (u.gate_up) tmem_ld_32x32b_x32(t0 + BUF_COLS / 2 + t * TT, v);
                tmem_ld_wait();
                if (f < ncol) {
#pragma unroll
                    for (int c = 0; c < TT; ++c) {
                        const int row = t * TT + c;
                        if (row < u.rows) {
                            const float val = u.gate_up
                                ? silu_mul(__uint_as_float(g[c]), __uint_as_float(v[c]))
                                : __uint_as_float(g[c]);
                            out[static_cast<size_t>(u.row0 + row) * ncol + f] = __float2bfloat16_rn(val);
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&ctl->tempty[buf]);
            if (u.gate_up && u.last_pass) {
                // publish the expert's act rows to the down items of other CTAs:
                // every thread fences its stores (also towards the async proxy
                // that the TMA reads use) and arrives; one thread waits for all
                // 128 (bounded) and releases the per-expert counter
                fence_proxy_async_global();
                __threadfence();
                mbar_arrive(&ctl->pub);
                if (r == 0) {
                    if (wait_bar(&ctl->pub, npub & 1u, ctl, p.status)) {
                        __threadfence();
                        atomicAdd(done + u.e, 1);
                    }
                }
                ++npub;
            }
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

size_t smem_bytes(int E) { return 1024 + STAGES * STAGE_BYTES + sizeof(Ctl) + (E + 1) * 4; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int encode(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return MOE_ERR_CUDA;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = reinterpret_cast<EncodeTiledFn>(fn)(
        m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

struct DecodeMapsHolder {
    DecodeMaps m;
};

int decode_build_maps(void **holder, const void *xp, const void *act, const void *wgu,
                      const void *wd, int rows_cap, int E, int d, int I) {
    DecodeMapsHolder *h = new (std::nothrow) DecodeMapsHolder;
    if (!h) return MOE_ERR_OOM;
    int rc;
    if ((rc = encode(&h->m.w_gate_up, wgu, static_cast<uint64_t>(E) * 2 * I, d, WM)) != MOE_OK ||
        (rc = encode(&h->m.w_down, wd, static_cast<uint64_t>(E) * d, I, WM)) != MOE_OK ||
        (rc = encode(&h->m.xp, xp, rows_cap, d, TT)) != MOE_OK ||
        (rc = encode(&h->m.act, act, rows_cap, I, TT)) != MOE_OK) {
        delete h;
        return rc;
    }
    *holder = h;
    return MOE_OK;
}

void decode_free_maps(void *holder) { delete static_cast<DecodeMapsHolder *>(holder); }

int launch_decode_experts(const void *holder, const DecodeParams &p, int n_sm, cudaStream_t s) {
    const DecodeMapsHolder *h = static_cast<const DecodeMapsHolder *>(holder);
    const size_t smem = smem_bytes(p.E);
    if (ensure_smem(decode_experts_kernel, smem) != MOE_OK) return MOE_ERR_CUDA;
    return launch_k(decode_experts_kernel, dim3(n_sm), dim3(kThreads), smem, s, h->m, p);
}

}  // namespace moe
