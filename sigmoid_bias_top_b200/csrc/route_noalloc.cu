// route_noalloc.cu -- routing of a batch without any device allocation.
//
// Some callers cannot allocate device memory at the point where they need the
// routing: code being recorded into a CUDA graph (allocation calls are not
// allowed, or would be captured, while a stream is capturing), latency-
// critical serving loops that forbid allocator calls because they can
// synchronise the device, and host applications whose memory planner owns all
// device memory up front. For them moe_route_noalloc computes the same
// routing as a context's forward (per-token expert indices and mixture
// weights) with its scratch memory in a fixed array compiled into this
// library, and makes no allocation or free.
//
// The scratch array is a file-scope __device__ array: every GPU that loads
// the library holds its own copy (about 1.1 MB) until the process exits. Host
// code cannot use the array's name as a device address; the address is taken
// with cudaGetSymbolAddress once per device (on that device's first call, with
// the device current) and cached. All calls on a device share the one array,
// so calls that overlap on the GPU (different streams, no ordering between
// them) race on it; calls on one stream are ordered and safe.
//
// The router's waits for its bulk copies are bounded (1 s). Where a context's
// forward reports such a time-out through moe_status, this entry point has no
// context to hold a status word: its status word sits in the scratch array,
// and a last small kernel turns a recorded time-out into idx = -1 and w = NaN
// for every slot of the call, so that a failed routing cannot be mistaken for
// a result.
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kNaMaxTokens = 4096;
constexpr int kNaMaxExperts = 64;
constexpr int kNaMaxD = 2048;
constexpr int kNaMaxChunks = 1;  // the whole batch is one dispatch chunk here
constexpr size_t kNaWg = static_cast<size_t>(kNaMaxExperts) * kNaMaxD * 4;   // W*gain [E][d]
constexpr size_t kNaWt = static_cast<size_t>(kNaMaxD) * 64 * 4;              // [d][64]
constexpr size_t kNaRinv = static_cast<size_t>(kNaMaxTokens) * 4;
constexpr size_t kNaHist = static_cast<size_t>(kNaMaxChunks) * kNaMaxExperts * 4;
constexpr size_t kNaHistPad = ((kNaHist + 255) / 256) * 256;
constexpr size_t kNaStatus = 256;  // one int: the router's time-out flag
constexpr size_t kNaBytes = kNaWg + kNaWt + kNaRinv + kNaHistPad + kNaStatus;

__device__ __align__(256) unsigned char g_route_scratch[kNaBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once).
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return MOE_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return MOE_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// After the router: if it recorded a time-out, no slot of the call holds a
// result, so every index becomes -1 and every weight NaN. Launched without
// programmatic dependence, so it starts after the router has finished.
__global__ void noalloc_finish_kernel(const int *status, int32_t *idx, float *w, int n) {
    if (*status == 0) return;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        idx[i] = -1;
        w[i] = __int_as_float(0x7fc00000);
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_route_noalloc(const void *x, int dtype, const float *norm_gain,
                                 const float *router_w, const float *expert_bias, int n_tokens,
                                 int d, int n_experts, int top_k, float eps, float routed_scale,
                                 int32_t *idx, float *w, void *stream) {
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (n_tokens < 0) return MOE_ERR_INVALID_ARG;
    if (n_tokens > kNaMaxTokens) return MOE_ERR_TOO_MANY_TOKENS;  // beyond the fixed scratch
    if (n_experts > kNaMaxExperts || d > kNaMaxD) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (d <= 0 || d % 4 != 0 || n_experts <= 0 || top_k <= 0 || top_k > kMaxTopK ||
        top_k > n_experts)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    // bf16 rows as moe_create takes them: the router bulk-copies whole groups
    // of rows, whose byte count must be a multiple of 16
    if (dtype == MOE_BF16 && d % 64 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (n_tokens == 0) return MOE_OK;
    if (!x || !norm_gain || !router_w || !expert_bias || !idx || !w) return MOE_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !(routed_scale == routed_scale)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(norm_gain) || !aligned16(router_w)) return MOE_ERR_ALIGNMENT;

    void *base = nullptr;
    int rc = scratch_address(&base);
    if (rc != MOE_OK) return rc;
    uint8_t *b = static_cast<uint8_t *>(base);
    float *wg = reinterpret_cast<float *>(b);
    float *wt = reinterpret_cast<float *>(b + kNaWg);
    float *rinv = reinterpret_cast<float *>(b + kNaWg + kNaWt);
    int32_t *hist = reinterpret_cast<int32_t *>(b + kNaWg + kNaWt + kNaRinv);
    int *status = reinterpret_cast<int *>(b + kNaWg + kNaWt + kNaRinv + kNaHistPad);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    const int e_pad = 64;
    if ((rc = launch_prepare_router(router_w, norm_gain, wg, wt, n_experts, e_pad, d, s)) != MOE_OK)
        return rc;
    // The histogram is added to by the route kernel and the status word only
    // ever gains bits, so both start at zero (one clear: the status follows
    // the histogram's padded block). The clear also sits between the two
    // kernels on purpose: the route kernel may start early under programmatic
    // launch and copies W*gain before its dependency wait, which is only safe
    // once a non-kernel step has ordered it fully after the kernel that
    // writes W*gain.
    if (cudaMemsetAsync(hist, 0, kNaHistPad + sizeof(int), s) != cudaSuccess)
        return MOE_ERR_CUDA;

    int tt = 0;
    const int kind = route_plan(n_tokens, d, n_experts, &tt);
    RouteParams rp;
    rp.x = x; rp.gain = norm_gain; rp.router_w = router_w; rp.router_wg = wg; rp.router_wt = wt;
    rp.bias = expert_bias; rp.rinv = rinv; rp.idx = idx; rp.wts = w; rp.chunk_hist = hist;
    rp.status = status;
    rp.N = n_tokens; rp.d = d; rp.E = n_experts; rp.k = top_k; rp.e_pad = e_pad;
    rp.chunk_tokens = (n_tokens + 31) / 32 * 32;  // one chunk: the histogram row 0
    rp.eps = eps; rp.scale = routed_scale;
    if ((rc = launch_route(rp, dtype, kind, tt, s)) != MOE_OK) return rc;
    const int n = n_tokens * top_k;
    noalloc_finish_kernel<<<(n + 255) / 256, 256, 0, s>>>(status, idx, w, n);
    return cudaPeekAtLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
