// gemm_tc.cu -- bf16 grouped GEMMs of the experts on the 5th-generation tensor
// cores (tcgen05, accumulators in TMEM), operands staged by TMA.
//
// The gated SiLU expert of "LFM2.5-24B-A2B: Biased Routing, Short Convolutions
// and Ten KV Caches" (flozi.net, English page, section "The router has two
// different scores") runs as two grouped contractions over the expert-grouped
// rows (section "What to verify in a deployment": tokens grouped by expert):
//   gate/up: act[r][f] = silu(xp[r] . Wg_e[f]) * (xp[r] . Wu_e[f]), xp[r] the
//            normalised row of the token that grouped row r belongs to
//            The packed [2I][d] matrix of expert e gives one 256-wide B tile
//            per 128 output features: 128 gate rows then the 128 matching up
//            rows, loaded as two TMA boxes into one operand. The accumulator
//            row (one token) then holds gate in columns 0..127 and up in
//            columns 128..255, so the SiLU(gate)*up epilogue is thread-local.
//   down:    y[r][n]   = act[r] . Wd_e[n]             (256 output columns/tile)
//
// Kernel structure (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: A tile 128 rows x 64 K, B tile 256 rows x 64 K,
//               128-byte swizzle, 4-stage ring of full/empty mbarriers;
//   warp 1      TMEM allocation (512 columns = two 128x256 fp32 accumulators)
//               and the single MMA-issuing thread: 4 x tcgen05.mma (M128 N256
//               K16) per stage, tcgen05.commit frees the stage / publishes the
//               finished accumulator;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31 = tile rows), bf16 conversion, masked
//               stores of the valid rows; the accumulator is double-buffered,
//               so the epilogue of one tile overlaps the MMAs of the next.
// Work items are (expert e, feature tile nt, row tile m) taken expert-major
// with m fastest, so the CTAs in flight share the weight tiles of the same
// few experts through L2; CTAs stride through the items. Rows past an
// expert's range are computed from neighbouring rows (or TMA zero fill past
// the buffer) and never stored.
//
// Every wait is bounded (1 s); on time-out the kernel records
// MOE_ERR_DEVICE_TIMEOUT in the status word, drains its own copies and MMAs
// in flight (again bounded), frees TMEM and returns.
#include <dlfcn.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = kTcTileM;  // rows (tokens) per tile = MMA M
constexpr int BN = 256;       // MMA N
constexpr int BK = 64;        // K per stage: one 128-byte swizzle row of bf16
constexpr int UK = 16;        // K per tcgen05.mma (kind::f16)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * BN;
constexpr int kThreads = 192;
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s

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

// Largest e in [0, E) with mts[e] <= q.
__device__ __forceinline__ int find_expert(const int32_t *mts, int E, int q) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mts[mid] <= q) lo = mid; else hi = mid - 1;
    }
    return lo;
}

struct Item {
    int e, nt, row0, rows;
};

__device__ __forceinline__ Item decode(int item, int NT, const int32_t *mts,
                                       const int32_t *offs, int E) {
    Item it;
    it.e = find_expert(mts, E, item / NT);
    const int mcount = mts[it.e + 1] - mts[it.e];
    const int local = item - mts[it.e] * NT;
    it.nt = local / mcount;
    const int m = local - it.nt * mcount;
    it.row0 = offs[it.e] + m * BM;
    it.rows = min(BM, offs[it.e + 1] - it.row0);
    return it;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
    return g / (1.0f + expf(-g)) * u;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

template <bool GATE_UP>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, GroupedParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + STAGES * STAGE_BYTES);
    int32_t *mts = reinterpret_cast<int32_t *>(ctl + 1);  // [E+1]
    int32_t *offs = mts + (p.E + 1);                        // [E+1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 128);
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
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    // everything above overlaps the previous kernel; the schedule below is its output
    pdl_trigger();
    pdl_wait();
    for (int i = threadIdx.x; i <= E; i += kThreads) {
        mts[i] = p.mt_start[i];
        offs[i] = p.offsets[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;

    const int NOUT = GATE_UP ? p.I : p.d;       // output columns per expert
    const int NT = GATE_UP ? (p.I + 127) / 128 : (p.d + BN - 1) / BN;
    const int K = GATE_UP ? p.d : p.I;
    const int nk = (K + BK - 1) / BK;
    const int total = mts[E] * NT;

    if (warp == 0) {
        // ---------------- TMA producer (whole warp) ----------------
        // lane 0 issues; A by one box, B by one box (down) or two (gate/up)
        int s = 0;
        uint32_t ph = 0;
        uint32_t issued_parity[STAGES];
        bool issued[STAGES];
        for (int i = 0; i < STAGES; ++i) issued[i] = false;
        for (int item = blockIdx.x; item < total; item += gridDim.x) {
            if (__shfl_sync(0xffffffffu, aborted(ctl) ? 1 : 0, 0)) break;
            const Item it = decode(item, NT, mts, offs, E);
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb) {
                int got = 1;
                if (lane == 0) got = wait_bar(&ctl->empty[s], ph ^ 1u, ctl, p.status) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
                if (lane == 0) {
                    uint8_t *sa = smem + s * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    mbar_arrive_expect_tx(&ctl->full[s], STAGE_BYTES);
                    tma_load_2d(sa, &tmA, kb * BK, it.row0, &ctl->full[s]);
                    if (GATE_UP) {
                        const int rg = it.e * 2 * p.I + it.nt * 128;
                        tma_load_2d(sb, &tmB, kb * BK, rg, &ctl->full[s]);
                        tma_load_2d(sb + B_BYTES / 2, &tmB, kb * BK, rg + p.I, &ctl->full[s]);
                    } else {
                        tma_load_2d(sb, &tmB, kb * BK, it.e * p.d + it.nt * BN, &ctl->full[s]);
                    }
                }
                issued[s] = true;
                issued_parity[s] = ph;
                if (++s == STAGES) { s = 0; ph ^= 1u; }
            }
            if (!ok) break;
        }
        if (lane == 0 && aborted(ctl)) {  // let our own copies land before the CTA exits
            const uint64_t dl = globaltimer_ns() + kWaitNs;
            for (int i = 0; i < STAGES; ++i)
                if (issued[i]) mbar_wait(&ctl->full[i], issued_parity[i], dl);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
            int s = 0;
            uint32_t ph = 0;
            int tile = 0;
            bool any = false;
            for (int item = blockIdx.x; item < total && !aborted(ctl); item += gridDim.x, ++tile) {
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
                    for (int kk = 0; kk < BK / UK; ++kk) {
                        umma_bf16(d_tmem, sw128_kmajor_desc(a0 + kk * UK * 2),
                                  sw128_kmajor_desc(b0 + kk * UK * 2), idesc,
                                  (kb | kk) != 0 ? 1u : 0u);
                    }
                    any = true;
                    umma_commit(&ctl->empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&ctl->tfull[buf]);
            }
            if (any) {  // all MMAs issued by this thread complete before TMEM is freed
                umma_commit(&ctl->drain);
                mbar_wait(&ctl->drain, 0, globaltimer_ns() + kWaitNs);
            }
        }
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int q = warp & 3;           // TMEM lane quarter this warp may access
        const int r = q * 32 + lane;      // tile row of this thread
        int tile = 0;
        for (int item = blockIdx.x; item < total && !aborted(ctl); item += gridDim.x, ++tile) {
            const int buf = tile & 1;
            const uint32_t use = static_cast<uint32_t>(tile >> 1);
            if (!wait_bar(&ctl->tfull[buf], use & 1u, ctl, p.status)) break;
            tc_fence_after();
            const Item it = decode(item, NT, mts, offs, E);
            const uint32_t t_row = tmem_base + static_cast<uint32_t>(buf * BN) +
                                   (static_cast<uint32_t>(q * 32) << 16);
            const bool valid = r < it.rows && it.row0 + r < p.rows_cap;
            __nv_bfloat16 *crow = static_cast<__nv_bfloat16 *>(p.c) +
                                  static_cast<size_t>(it.row0 + (valid ? r : 0)) * NOUT;
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
            mbar_arrive(&ctl->tempty[buf]);
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

__global__ void selftest_timeout_kernel(int *status, int timeout_us) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // nothing ever arrives on `bar`: the wait must give up and report
        if (!mbar_wait(&bar, 0, globaltimer_ns() + static_cast<uint64_t>(timeout_us) * 1000ull))
            set_status(status, kStatusTimeout);
    }
}

size_t smem_bytes(int E) {
    return 1024 + STAGES * STAGE_BYTES + sizeof(Ctl) + 2 * (E + 1) * sizeof(int32_t);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D bf16 map of a row-major [rows][cols] matrix with a (64 x box_rows) box
// and the 128-byte swizzle; reads outside the matrix fill with zeros.
int encode_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn enc = get_encoder();
    if (!enc) return MOE_ERR_CUDA;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// 4-D bf16 view of a packed paired-row matrix [rows_total][d] for the
// CTA-pair kernel: element (k, y, z, g) = row 16 g + y + z up_offset, column
// k, i.e. 16-row group g of the first block (z = 0) or the row up_offset
// further (z = 1). For the experts' gate/up matrices [E*2I][d], up_offset =
// I (gate row f, up row f + I); for the short-convolution input projection
// [g; u; v] = [3d][d], up_offset = 2d pairs g with v. Groups run up to
// rows_total - up_offset rows, so every addressed row lies inside the
// matrix; a box of {64, 16, 2, 4} lands in shared memory as 16 first-block
// rows, the matching 16 partner rows, the next 16, ... (128 rows, 128-byte
// swizzle).
int encode_pair_4d(CUtensorMap *m, const void *base, uint64_t rows_total, int d,
                   uint64_t up_offset) {
    EncodeTiledFn enc = get_encoder();
    if (!enc) return MOE_ERR_CUDA;
    const uint64_t groups = (rows_total - up_offset) / 16;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), 16, 2, groups};
    const cuuint64_t row = static_cast<cuuint64_t>(d) * 2;
    const cuuint64_t strides[3] = {row, row * static_cast<cuuint64_t>(up_offset), row * 16};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(BK), 16, 2, 4};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

template <bool GATE_UP>
int launch(const CUtensorMap &a, const CUtensorMap &b, const GroupedParams &p, int n_sm,
           cudaStream_t s) {
    auto kern = grouped_tc_kernel<GATE_UP>;
    const size_t smem = smem_bytes(p.E);
    if (ensure_smem(kern, smem) != MOE_OK) return MOE_ERR_CUDA;
    return launch_k(kern, dim3(n_sm), dim3(kThreads), smem, s, a, b, p);
}

}  // namespace

int tc_encode_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                 uint32_t box_rows) {
    return encode_2d(m, base, rows, cols, box_rows);
}

int tc_encode_pair_4d(CUtensorMap *m, const void *base, uint64_t rows_total, int d,
                      uint64_t up_offset) {
    return encode_pair_4d(m, base, rows_total, d, up_offset);
}

int tc_build_maps(TcMaps *m, const void *xp, const void *act, const void *wgu, const void *wd,
                  int rows_cap, int E, int d, int I) {
    int rc;
    if ((rc = encode_2d(&m->a_gate_up, xp, rows_cap, d, BM)) != MOE_OK) return rc;
    if ((rc = encode_2d(&m->w_gate_up, wgu, static_cast<uint64_t>(E) * 2 * I, d, 128)) != MOE_OK)
        return rc;
    if ((rc = encode_2d(&m->a_down, act, rows_cap, I, BM)) != MOE_OK) return rc;
    if ((rc = encode_2d(&m->w_down, wd, static_cast<uint64_t>(E) * d, I, BN)) != MOE_OK)
        return rc;
    if (I % 16 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if ((rc = encode_pair_4d(&m->w_gate_up_4d, wgu, static_cast<uint64_t>(E) * 2 * I, d, I)) !=
        MOE_OK)
        return rc;
    if ((rc = encode_2d(&m->w_down_half, wd, static_cast<uint64_t>(E) * d, I, BN / 2)) != MOE_OK)
        return rc;
    return MOE_OK;
}

int launch_gemm_tc_gate_up(const TcMaps &m, const GroupedParams &p, int n_sm, cudaStream_t s) {
    return launch<true>(m.a_gate_up, m.w_gate_up, p, n_sm, s);
}

int launch_gemm_tc_down(const TcMaps &m, const GroupedParams &p, int n_sm, cudaStream_t s) {
    return launch<false>(m.a_down, m.w_down, p, n_sm, s);
}

int launch_selftest_timeout(int *status, int timeout_us, cudaStream_t s) {
    selftest_timeout_kernel<<<1, 32, 0, s>>>(status, timeout_us);
    return cudaPeekAtLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
