// moe_fp8.cuh -- the FP8_BLOCK expert path: parameter blocks, launchers and
// the kind::f8f6f4 tensor-core wrappers.
//
// Scheme ("LFM2.5-24B-A2B: ein 24B-Reasoning-Modell, das pro Wortstück so wenig verbraucht wie ein 2B-Modell",
// inferencekey.com, section "Für Engineers", paragraph "Quantisierung"):
// expert weights are stored as FP8 with one scale per 128 x 128 block, and the
// activations entering each expert matrix are quantised to FP8 per token in
// groups of 128. Here the FP8 format is e4m3 (largest finite 448); a weight
// is its code's value times the fp32 scale of its block, and an activation
// group of 128 values v gets s = amax|v| / 448 and codes e4m3(v / s), rounded
// to nearest even with saturation (an all-zero group: s = 0, zero codes).
// The router, the RMSNorm gain and x / out stay as in the bf16 path (bf16
// x and out, fp32 router).
#pragma once

#include "moe_internal.cuh"

namespace moe {

constexpr int kFp8Block = 128;  // weight blocks of 128 x 128, activation groups of 128

struct Fp8ExpertParams {
    const int32_t *offsets;   // [E+1] row range of each expert in the grouped order
    const float *sgu;         // [E][2I/128][d/128] block scales of w_gate_up
    const float *sdn;         // [E][d/128][I/128] block scales of w_down
    const float *xs;          // [rows][d/128] group scales of the grouped input rows
    uint8_t *aq;              // [rows][I] e4m3 codes of SiLU(gate)*up (written, then read)
    float *as;                // [rows][I/128] their group scales
    void *y;                  // [rows][d] bf16 expert outputs
    int32_t *sched;           // [1 + E]: claimed-item counter, finished gate/up items per expert
    int *status;
    int E, d, I;
};

// The large-batch path: two launches of the CTA-pair FP8 GEMM (gemm_fp8_tc2.cu)
// over token tiles of at most kFp8PairTileM rows (the dispatch's row-tile
// prefix mt_start must be built with that tile size).
constexpr int kFp8PairTileM = 128;
struct Fp8PairParams {
    const int32_t *offsets;   // [E+1] row range of each expert in the grouped order
    const int32_t *mt_start;  // [E+1] prefix of per-expert token tiles of kFp8PairTileM rows
    const float *sgu;         // [E][2I/128][d/128] block scales of w_gate_up
    const float *sdn;         // [E][d/128][I/128] block scales of w_down
    const float *xs;          // gate/up input: [rows][d/128] group scales of the grouped rows
    const float *as_in;       // down input: [rows][I/128] group scales of aq
    float *a32;               // gate/up output: [rows][I] fp32 SiLU(gate)*up
    uint8_t *aq;              // quantiser output: [rows][I] e4m3 codes of a32
    float *as_out;            // quantiser output: [rows][I/128] their group scales
    void *y;                  // down output: [rows][d] bf16
    int *status;
    int E, d, I;
};
int fp8_pair_build_maps(void **holder, const void *xq, const void *aq, const void *wgu,
                        const void *wd, int rows_cap, int E, int d, int I);
void fp8_pair_free_maps(void *holder);
int launch_fp8_pair_gate_up(const void *holder, const Fp8PairParams &p, int n_sm, cudaStream_t s);
int launch_fp8_pair_down(const void *holder, const Fp8PairParams &p, int n_sm, cudaStream_t s);
// aq, as_out = the per-group-of-128 e4m3 quantisation of a32, rows offsets[E]
int launch_fp8_quantize_act(const Fp8PairParams &p, int n_sm, cudaStream_t s);

// a / b rounded to nearest (the IEEE quotient) from rb = RN(1/b) (__frcp_rn)
// by Markstein's correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Develop.
// 34(1), 1990): q0 = RN(a rb), r = a - q0 b formed inside a fused
// multiply-add, q = RN(q0 + r rb). The result is the correctly rounded
// quotient while nothing overflows or underflows; b outside [2^-100, 2^100]
// takes the full division instead. Quotients that fall into the fp32
// subnormal range may differ in the last place, which no e4m3 code can see
// (every value below 2^-10 rounds to code 0). Tested against __fdiv_rn by
// moe_selftest_fp8_divide. A caller with one divisor for many quotients tests
// the range once (div_rn_step_ok) and takes div_rn_step or __fdiv_rn for all.
__device__ __forceinline__ bool div_rn_step_ok(float b) { return b >= 0x1p-100f && b <= 0x1p100f; }
__device__ __forceinline__ float div_rn_step(float a, float b, float rb) {
    const float q0 = __fmul_rn(a, rb);
    const float r = fmaf(-q0, b, a);
    return fmaf(r, rb, q0);
}
__device__ __forceinline__ float div_rn(float a, float b, float rb) {
    if (!div_rn_step_ok(b)) return __fdiv_rn(a, b);
    return div_rn_step(a, b, rb);
}
// div_rn_step of two numerators over one divisor, in paired fp32 operations
// (each component rounded as the scalar one; a - q0 b as fma(q0, -b, a), the
// same exact product).
__device__ __forceinline__ float2 div_rn_step2(float2 a, float b, float rb) {
    const float2 rb2 = make_float2(rb, rb);
    const float2 q0 = __fmul2_rn(a, rb2);
    const float2 r = __ffma2_rn(q0, make_float2(-b, -b), a);
    return __ffma2_rn(r, rb2, q0);
}

// Grouped, quantised rows from the dispatch: codes [rows][d], scales [rows][d/128].
int launch_dispatch_fp8(const DispatchParams &p, uint8_t *xq, float *xs, cudaStream_t s);

int fp8_build_maps(void **holder, const void *xq, const void *aq, const void *wgu,
                   const void *wd, int rows_cap, int E, int d, int I);
void fp8_free_maps(void *holder);
// pass_tokens: tokens per pass of a weight tile, 32 (small batches: eight
// TMEM buffers of K-block partials) or 64 (two token tiles, four buffers).
int launch_fp8_experts(const void *holder, const Fp8ExpertParams &p, int n_sm, int pass_tokens,
                       cudaStream_t s);

// Instruction descriptor of kind::f8f6f4 with e4m3 A and B (both K-major) and
// an fp32 accumulator, for an M x N tile (A/B format code 0 = E4M3).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
    return (1u << 4)                                   // D format: f32
           | (0u << 7)                                 // A format: e4m3
           | (0u << 10)                                // B format: e4m3
           | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// D (+)= A * B^T with e4m3 operands from shared memory: K = 32 per instruction.
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

}  // namespace moe
