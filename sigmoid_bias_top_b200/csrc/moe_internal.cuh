// moe_internal.cuh -- shared definitions of the sm_100a MoE kernels: parameter
// blocks, device status codes, and thin inline-PTX wrappers for mbarriers,
// TMA bulk-tensor copies and the tcgen05 (5th-generation tensor core / TMEM)
// instructions. Formats follow the PTX ISA for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <utility>

#include "../../include/moe.h"

namespace moe {

constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;

// ---------------------------------------------------------------------------
// Device status word (one int per context). Kernels OR in flag bits; the host
// maps them to moe_err codes.
constexpr int kStatusTimeout = 1;
constexpr int kStatusBounds = 2;

__device__ __forceinline__ void set_status(int *status, int bits) {
    if (status) atomicOr(status, bits);
}

// ---------------------------------------------------------------------------
// Parameter blocks

struct RouteParams {
    const void *x;          // [N][d] f32 or bf16
    const float *gain;      // [d]
    const float *router_w;  // [E][d]
    const float *router_wg; // [E][d] router matrix times gain (column-wise)
    const float *router_wt; // [d][e_pad] the same transposed, zero-padded columns
    const float *bias;      // [E]
    float *rinv;            // [N] 1 / sqrt(mean(x^2) + eps) per token
    int32_t *idx;           // [N][k]
    float *wts;             // [N][k]
    int32_t *chunk_hist;    // [nchunk][E] per token-chunk expert counts (added to)
    int *status;
    int N, d, E, k, e_pad, chunk_tokens;
    float eps, scale;
};

struct DispatchParams {
    const void *x;             // [N][d] block input
    const float *gain;         // [d]
    const float *rinv;         // [N]
    void *xp;                  // [N*k][d] normalised rows in grouped order (dtype of x)
    const int32_t *idx;        // [N][k]
    const int32_t *chunk_hist; // [nchunk][E]
    int32_t *counts;           // [E]
    int32_t *offsets;          // [E+1]
    int32_t *mt_start;         // [E+1] prefix of per-expert row tiles (tile rows = tile_m)
    int32_t *perm;             // [N*k] grouped row -> assignment t*k+j
    int32_t *inv;              // [N*k] assignment -> grouped row
    int32_t *sched;            // [sched_n] cleared for the fused small-batch expert kernel
    int *status;
    int N, d, E, k, nchunk, chunk_tokens, tile_m, replicas, elem_bytes, sched_n;
};

struct CombineParams {
    const void *x;          // [N][d]
    const void *y;          // [N*k][d] expert outputs in grouped order
    const float *wts;       // [N][k]
    const int32_t *inv;     // [N*k]
    void *out;              // [N][d]
    int32_t *chunk_hist;    // zeroed here for the next forward
    int chunk_hist_n;
    int *status;
    int N, d, k;
};

struct GroupedParams {
    // shared by the SIMT and the tensor-core grouped GEMMs
    const int32_t *offsets;   // [E+1] row range of each expert in the grouped order
    const int32_t *mt_start;  // [E+1] prefix of per-expert row tiles
    const void *a;            // gate/up: xp [rows][d]; down: act [rows][I]
    const void *w;            // gate/up: [E][2I][d]; down: [E][d][I]
    void *c;                  // gate/up: act [rows][I]; down: y [rows][d]
    int *status;
    int E, d, I, k;
    int rows_cap;             // allocated grouped rows (act, y)
    // epilogue inputs of the dense and short-convolution blocks (CTA-pair kernel);
    // kEpiResid / kEpiConv move c, resid and aux in 16-byte pieces: d % 8 == 0
    // and all three 16-byte aligned
    const void *resid;        // kEpiResid: [rows][d] added to the product
    const void *aux;          // kEpiConv: a [rows][d] (bf16), convolved along each sequence
    const float *conv;        // kEpiConv: taps [d][3] by lag
    const float *state_in;    // kEpiConv: [rows/seq_len][2][d] a of positions -2, -1, or null
    int seq_len;              // kEpiConv: positions per sequence (rows are sequence-major)
    int wt_fastest;           // CTA-pair kernel: weight tiles vary fastest within an expert
    // split-K (CTA-pair kernel, kEpiPartial / kEpiPartialPaired): every tile
    // in ksplit K slices of ceil(nk / ksplit) kTcPairBK-wide blocks, none empty (the
    // caller picks ksplit so); slice ks writes fp32 sums to
    // partial[ks][row][width], row < partial_rows, width = NOUT (plain) or
    // 2 NOUT (paired: the first block's rows, then the partner rows)
    int ksplit;
    float *partial;
    int partial_rows;
};

// Epilogue modes of the CTA-pair GEMM (launch_gemm_tc2_mode).
constexpr int kEpiSiluMul = 0;  // paired rows: silu(gate) * up          (4-D weight map)
constexpr int kEpiPlain = 1;    // plain product                          (2-D weight map)
constexpr int kEpiMul = 2;      // paired rows: gate * up, no activation  (4-D weight map)
constexpr int kEpiConv = 3;     // u * depthwise causal conv of a         (2-D weight map)
constexpr int kEpiResid = 4;    // residual + product                     (2-D weight map)
constexpr int kEpiPartialPaired = 5;  // paired rows, fp32 partial sums of a K slice (4-D)
constexpr int kEpiPartial = 6;        // fp32 partial sums of a K slice         (2-D weight map)
constexpr int kTcPairBK = 128;        // K per stage of the CTA-pair kernel

struct DecodeParams {
    // the fused small-batch expert kernel (gate/up and down in one launch)
    const int32_t *offsets;   // [E+1]
    void *act;                // [rows][I] written by gate/up items, read by down items
    void *y;                  // [rows][d]
    int32_t *sched;           // [1 + E]: claimed-item counter, per-expert finished gate/up items
    int *status;
    int E, d, I;
};

// ---------------------------------------------------------------------------
// Host-side launchers

constexpr int kRouteSmall = 0, kRouteLarge = 1, kRouteTc = 2;
bool route_small_ok(int d, int E);
int route_plan(int N, int d, int E, int *toks_per_group);
int launch_route(const RouteParams &p, int dtype, int kind, int toks_per_group, cudaStream_t s);
int launch_prepare_router(const float *w, const float *gain, float *wg, float *wt, int E,
                          int e_pad, int d, cudaStream_t s);
// The tensor-core router of bf16 batches (W' split into three bf16 matrices).
bool route_tc_ok(int d, int E);
int launch_split_router(const float *wg, void *w3, int E, int d, cudaStream_t s);
int launch_route_tc(const RouteParams &p, const CUtensorMap &w3_map, cudaStream_t s);
size_t dispatch_smem(int nchunk, int E, int chunk_assign, int d);
int launch_dispatch(const DispatchParams &p, cudaStream_t s);
int launch_combine(const CombineParams &p, int dtype, cudaStream_t s);
int launch_gemm_simt_gate_up(const GroupedParams &p, int max_mtiles, cudaStream_t s);
int launch_gemm_simt_down(const GroupedParams &p, int max_mtiles, cudaStream_t s);
constexpr int kSimtTileM = 64;
constexpr int kTcTileM = 128;

struct TcMaps {
    CUtensorMap a_gate_up;  // xp  [rows][d],     box 64 x 128
    CUtensorMap w_gate_up;  // W   [E*2I][d],     box 64 x 128
    CUtensorMap a_down;     // act [rows][I],     box 64 x 128
    CUtensorMap w_down;     // Wd  [E*d][I],      box 64 x 256
    // the CTA-pair kernels (weights as the M operand, tokens as N)
    CUtensorMap w_gate_up_4d;  // W as [group][gate|up][16 rows][d], box 64 x 16 x 2 x 4
    CUtensorMap w_down_half;   // Wd [E*d][I],   box 64 x 128
};
// 2-D bf16 map of a row-major [rows][cols] matrix, box 64 x box_rows,
// 128-byte swizzle, zero fill outside.
int tc_encode_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                 uint32_t box_rows);
int tc_build_maps(TcMaps *m, const void *xp, const void *act, const void *wgu, const void *wd,
                  int rows_cap, int E, int d, int I);
int launch_gemm_tc_gate_up(const TcMaps &m, const GroupedParams &p, int n_sm, cudaStream_t s);
int launch_gemm_tc_down(const TcMaps &m, const GroupedParams &p, int n_sm, cudaStream_t s);
int launch_selftest_timeout(int *status, int timeout_us, cudaStream_t s);
// The same contractions on CTA pairs: 256 weight rows x up to 256 tokens per
// tile (experts split into token tiles of at most kTcPairTileM rows).
constexpr int kTcPairTileM = 256;
int launch_gemm_tc2_gate_up(const TcMaps &m, const GroupedParams &p, int n_sm, cudaStream_t s);
int launch_gemm_tc2_down(const TcMaps &m, const GroupedParams &p, int n_sm, cudaStream_t s);
// Any epilogue mode on given maps: w = weights (4-D paired-row map for
// kEpiSiluMul / kEpiMul, 2-D box-128 map otherwise), t = token rows (box 128).
int launch_gemm_tc2_mode(int mode, const CUtensorMap &w, const CUtensorMap &t,
                         const GroupedParams &p, int n_sm, cudaStream_t s);
// 4-D paired-row view of a row-major [rows_total][d] bf16 matrix: 16-row
// group g of the first block and the rows up_offset further (box 64x16x2x4).
int tc_encode_pair_4d(CUtensorMap *m, const void *base, uint64_t rows_total, int d,
                      uint64_t up_offset);
constexpr int kDecodeRowsPerExpert = 32;  // the fused kernel is used up to this mean load
int decode_build_maps(void **holder, const void *xp, const void *act, const void *wgu,
                      const void *wd, int rows_cap, int E, int d, int I);
void decode_free_maps(void *holder);
int launch_decode_experts(const void *holder, const DecodeParams &p, int n_sm, cudaStream_t s);

// ---------------------------------------------------------------------------
// Launch with programmatic dependent launch: the kernel may be scheduled while
// its predecessor in the stream is still running; it must call pdl_wait()
// before touching anything the predecessor writes or reads.

template <typename... KArgs, typename... Args>
inline int launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                    Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    if (err == cudaSuccess) return MOE_OK;
    if (getenv("MOE_DEBUG")) {  // diagnostics on request: why the launch was refused
        cudaFuncAttributes fa = {};
        cudaFuncGetAttributes(&fa, reinterpret_cast<const void *>(kern));
        fprintf(stderr,
                "moe: launch failed: %s (grid %u, block %u, smem %zu; kernel: %d regs, "
                "max %d threads, max dyn smem %d)\n",
                cudaGetErrorString(err), grid.x, block.x, smem, fa.numRegs, fa.maxThreadsPerBlock,
                fa.maxDynamicSharedSizeBytes);
    }
    return MOE_ERR_CUDA;
}

// Token chunks of the dispatch: about kChunkAssign assignments each, a whole
// number of route groups (32 tokens), histogram within 64 KB of shared memory.
constexpr int kChunkAssign = 512;  // assignments per dispatch chunk (target)
inline int max_dispatch_chunks(int E) { return 16384 / E < 256 ? 16384 / E : 256; }
inline void chunk_plan(int N, int k, int max_chunks, int *nchunk, int *chunk_tokens) {
    int n = (N * k + kChunkAssign - 1) / kChunkAssign;
    n = n < 1 ? 1 : n > max_chunks ? max_chunks : n;
    int ct = (N + n - 1) / n;
    ct = (ct + 31) / 32 * 32;
    *chunk_tokens = ct;
    *nchunk = (N + ct - 1) / ct;
}

// Raises a kernel's dynamic shared-memory limit (once per kernel and size).
int ensure_smem_ptr(const void *kern, size_t smem);
template <typename K>
inline int ensure_smem(K kern, size_t smem) {
    return ensure_smem_ptr(reinterpret_cast<const void *>(kern), smem);
}

// ---------------------------------------------------------------------------
// Small device helpers

// Lets the next kernel in the stream be scheduled (its pdl_wait still waits
// for this whole grid to finish).
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Waits until the preceding kernel in the stream has completed and its
// memory operations are visible (returns at once without a predecessor).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float bf16_to_f32(uint16_t u) {
    return __uint_as_float(static_cast<uint32_t>(u) << 16);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// Per-token expert selection shared by the routers

// Order-preserving integer image of a float (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Selection and weights of one token by one warp. srow[E] holds its logits
// (overwritten with the sigmoid scores); the result goes to idx/wts row t and
// the expert counts to hist (shared). Each round takes the largest biased
// score (warp max of its integer image), then the lowest expert index among
// the lanes holding it: exact fp32 top-k with ties to the lower index.
__device__ __forceinline__ void select_token(const RouteParams &p, float *srow,
                                             const float *bias_s, size_t t, int *hist, int lane) {
    const int E = p.E, k = p.k;
    const int epl = (E + 31) / 32;  // experts per lane
    uint32_t key[kMaxExperts / 32];
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i) {
        const int e = lane + 32 * i;
        key[i] = 0u;  // below every real key: never selected
        if (i < epl && e < E) {
            const float s = 1.0f / (1.0f + expf(-srow[e]));
            const float c = s + bias_s[e];
            key[i] = (c == c) ? float_key(c) : 1u;  // a NaN score ranks below every number
            srow[e] = s;  // each lane rewrites only its own experts
        }
    }
    __syncwarp();
    int sel[kMaxTopK];
    float ssel[kMaxTopK];
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        if (j >= k) break;
        uint32_t bk = 0u;
        int bi = 0;
#pragma unroll
        for (int i = 0; i < kMaxExperts / 32; ++i)
            if (key[i] > bk) {  // ascending expert index: ties keep the lower one
                bk = key[i];
                bi = i;
            }
        const uint32_t top = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t cand = (bk == top && top != 0u) ? static_cast<uint32_t>(lane + 32 * bi) : 0xffffffffu;
        const uint32_t e = __reduce_min_sync(0xffffffffu, cand);
        // k <= E: an unselected expert exists, so e < E here
#pragma unroll
        for (int i = 0; i < kMaxExperts / 32; ++i)
            if (static_cast<uint32_t>(lane + 32 * i) == e) key[i] = 0u;
        sel[j] = static_cast<int>(e);
        ssel[j] = srow[e];
        sum += ssel[j];
    }
    if (lane < k) {  // lane j writes slot j
        const float den = sum + p.eps;
        float sj = 0.f;
        int ej = 0;
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j)
            if (j == lane) {
                sj = ssel[j];
                ej = sel[j];
            }
        p.idx[t * k + lane] = ej;
        p.wts[t * k + lane] = p.scale * (sj / den);
        atomicAdd(&hist[ej], 1);
    }
}

// ---------------------------------------------------------------------------
// mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase of `bar` with the given parity to complete, giving up at
// `deadline` (globaltimer ns). Returns false on time-out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t deadline) {
    for (uint32_t i = 0;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && globaltimer_ns() > deadline) return false;
    }
}

// ---------------------------------------------------------------------------
// TMA (bulk tensor copies global -> shared, completion on an mbarrier)

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *m, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned addresses, size % 16 == 0).
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 16-byte asynchronous copy global -> shared (L2 only); src_bytes < 16 zero-fills.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

// One arrival on `bar` once all of this thread's prior cp.async copies land
// (the barrier's expected count must include it).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Orders shared-memory writes made through the generic proxy (st.shared,
// cp.async) before later async-proxy reads (tcgen05.mma operands).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Same with an L2 eviction-priority hint (a createpolicy value).
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const CUtensorMap *m, int x, int y,
                                                 uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, MMA, commit, TMEM -> register loads

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile stored with the
// 128-byte swizzle (rows of 128 B, 8-row atoms of 1024 B): start address,
// leading-byte offset 16 B (unused for this layout), stride-byte offset 1024 B
// between 8-row groups, descriptor version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(1) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Instruction descriptor of kind::f16 with bf16 A and B (both K-major) and an
// fp32 accumulator, for an M x N tile.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4)                                   // D format: f32
           | (1u << 7)                                 // A format: bf16
           | (1u << 10)                                // B format: bf16
           | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives (once) on `bar` when all previously issued tcgen05.mma of this
// thread have completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives TMEM
// lane (lane base + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// 32 lanes x 8 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// tcgen05.wait::ld that names r, the destination of the loads it waits for,
// as read and written: no use of r can be scheduled above the wait, even
// where independent work (another buffer's arithmetic) sits between the load
// and its use.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

}  // namespace moe
