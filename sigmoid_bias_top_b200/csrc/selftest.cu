// selftest.cu -- device-side checks exposed for the tests.
//
// moe_selftest_fp8_divide: the FP8 quantisers take code = e4m3(v / s) with
// the IEEE quotient, formed by div_rn (a reciprocal and one correction step),
// two quotients at a time by div_rn_step2 where the divisor is in its range;
// this entry point returns that quotient (the paired form's first component
// for even i, its second, on the negated numerator and negated back, for odd
// i) beside __fdiv_rn's for the same operands, so that a test can hold the two
// equal bit for bit.
#include "moe_fp8.cuh"

namespace moe {
namespace {
__global__ void divide_kernel(const float *a, const float *b, float *q, float *q_ref, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const float bb = b[i];
        if (div_rn_step_ok(bb)) {
            const float2 qq = div_rn_step2(make_float2(a[i], -a[i]), bb, __frcp_rn(bb));
            q[i] = (i & 1) ? -qq.y : qq.x;
        } else {
            q[i] = div_rn(a[i], bb, __frcp_rn(bb));
        }
        q_ref[i] = __fdiv_rn(a[i], bb);
    }
}
}  // namespace
}  // namespace moe

extern "C" int moe_selftest_fp8_divide(const float *a, const float *b, float *q, float *q_ref,
                                       int n, void *stream) {
    if (n < 0 || (n > 0 && (!a || !b || !q || !q_ref))) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    int blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    moe::divide_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(a, b, q, q_ref, n);
    return cudaPeekAtLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
