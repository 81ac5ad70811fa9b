// wl_linear_forward_noalloc: the decode-path forward for callers that must
// not allocate device memory.
//
// Some callers cannot call cudaMalloc at the time they run a layer: code that
// runs inside a pre-planned memory arena (an inference engine whose allocator
// owns all of device memory), a caller holding a strict memory budget, or a
// host thread that must not take the driver's allocation locks on its hot path.
// wl_linear_forward draws its scratch (the low-rank product V^T x and its
// partial sums) from a pool that grows with cudaMalloc on first use; this
// entry point instead uses one fixed array in the library's own device image,
// so it never allocates.
//
// The scratch is a file-scope __device__ array of kScratchBytes (4 MiB).  Every
// GPU that loads the library holds it until the process exits.  In host code
// the array's name is only a host-side stand-in, not a device address, so the
// entry point looks the address up with cudaGetSymbolAddress once per device
// (with that device current) and passes that pointer to the kernels.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "../../include/wl.h"
#include "wl_internal.h"

namespace wl {
namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr size_t kWordsBytes = 256;                // status word + arrival counters
constexpr int kCounterWord = 8;                    // words [0, 8): status; [8, 64): counters

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

struct NoAllocDevice {
    bool ready = false;
    unsigned char *scratch = nullptr;  // device address of g_noalloc_scratch
    int num_sms = 0;
    int major = 0;
};

std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[64];

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Once per device, with that device current: resolve the array's device address.
wl_status noalloc_setup(NoAllocDevice **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WL_ERR_CUDA;
    if (dev < 0 || dev >= 64) return WL_ERR_UNSUPPORTED;
    NoAllocDevice &d = g_noalloc_dev[dev];
    if (!d.ready) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return WL_ERR_CUDA;
        }
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
            return WL_ERR_CUDA;
        d.scratch = static_cast<unsigned char *>(ptr);
        d.ready = true;
    }
    if (d.major != 10) return WL_ERR_UNSUPPORTED;
    *out = &d;
    return WL_OK;
}

}  // namespace
}  // namespace wl

extern "C" wl_status wl_linear_forward_noalloc(const wl_bf16 *x, const wl_bf16 *W0, const float *s,
                                               const wl_bf16 *U, const wl_bf16 *V, wl_bf16 *y, int M,
                                               int N, int K, int r, void *stream_ptr) {
    using namespace wl;
    // Host-side checks first; nothing below them touches the device until they pass.
    if (M < 0 || N < 0 || K < 0 || r < 0) return WL_ERR_INVALID_ARG;
    if (r > WL_MAX_RANK) return WL_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return WL_OK;
    if (!y || !s || (K > 0 && (!x || !W0)) || (r > 0 && K > 0 && (!U || !V)))
        return WL_ERR_INVALID_ARG;
    if (K % 8 != 0) return WL_ERR_ALIGNMENT;
    if (K > 0 && (!aligned16(x) || !aligned16(W0))) return WL_ERR_ALIGNMENT;
    if (M > WL_DECODE_MAX_M) return WL_ERR_UNSUPPORTED;

    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    if (K == 0) return cudaMemsetAsync(y, 0, (size_t)M * N * 2, stream) == cudaSuccess ? WL_OK : WL_ERR_CUDA;

    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocDevice *d = nullptr;
    wl_status st = noalloc_setup(&d);
    if (st != WL_OK) return st;

    static DecodeParams dp;  // large (tensor maps); guarded by g_noalloc_mu
    std::memset(&dp, 0, sizeof dp);
    DecodeSeg &sg = dp.a.seg[0];
    sg.W0 = reinterpret_cast<const __nv_bfloat16 *>(W0);
    sg.s = s;
    sg.U = reinterpret_cast<const __nv_bfloat16 *>(U);
    sg.V = reinterpret_cast<const __nv_bfloat16 *>(V);
    sg.y = reinterpret_cast<__nv_bfloat16 *>(y);
    sg.N = N;
    sg.r = r;
    sg.t_off = 0;
    dp.a.nseg = 1;
    dp.a.M = M;
    dp.a.K = K;
    dp.a.t_ld = r;
    dp.a.x = reinterpret_cast<const __nv_bfloat16 *>(x);
    dp.a.timeout_ns = wait_limit_ns();
    DecodePlan plan;
    if ((st = plan_decode(dp, d->num_sms, &plan)) != WL_OK) return st;
    // Scratch: the word block, then the partial sums of V^T x ((grid+1) x M x r fp32).
    if (kWordsBytes + align256(plan.tpart_bytes) > kScratchBytes) return WL_ERR_UNSUPPORTED;

    // The array keeps the previous call's contents: zero the arrival counters,
    // which must start at zero (a call whose wait gave up leaves them set), on
    // the caller's stream.  The status word is kept until
    // wl_noalloc_last_status() reads it.
    int *words = reinterpret_cast<int *>(d->scratch);
    if (cudaMemsetAsync(words + kCounterWord, 0, kWordsBytes - kCounterWord * sizeof(int), stream) != cudaSuccess)
        return WL_ERR_CUDA;
    dp.a.status = words;
    dp.a.sync = reinterpret_cast<unsigned int *>(words + kCounterWord);
    dp.a.Tpart = reinterpret_cast<float *>(d->scratch + kWordsBytes);
    return launch_decode(dp, plan, stream) == cudaSuccess ? WL_OK : WL_ERR_CUDA;
}

extern "C" wl_status wl_noalloc_last_status(void *stream) {
    using namespace wl;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocDevice *d = nullptr;
    wl_status st = noalloc_setup(&d);
    if (st != WL_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return WL_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, d->scratch, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return WL_ERR_CUDA;
    // after an error, clear the whole word block (status and any counters a
    // call that gave up left set)
    if (word != 0 && cudaMemset(d->scratch, 0, kWordsBytes) != cudaSuccess) return WL_ERR_CUDA;
    return static_cast<wl_status>(word);
}
