// mq_linear_unfused_noalloc: the unfused comparison path for callers that
// cannot allocate device memory.
//
// mq_linear_unfused needs M*N fp32 partial outputs between its two kernels
// and takes them from a caller-owned workspace. Some callers have no way to
// provide one: code running inside a fixed memory budget or a pool they do
// not control, plugins that are handed only the input and output buffers,
// or hosts where every device allocation must go through an allocator this
// library cannot see. This entry point keeps those partials in a
// fixed-size array that belongs to the library itself, so the call performs
// no cudaMalloc, cudaFree or other allocating call of any kind.
//
// The array is a file-scope __device__ variable: every GPU on which the
// library's code is loaded holds its kNoallocMaxOutputs floats until the
// process exits. Host code cannot use the variable's name as a device
// address, so the first call on each device (with that device current)
// looks the address up with cudaGetSymbolAddress and caches it, keyed on the
// device and its current CUDA context: a call under another context (after
// cudaDeviceReset, or with a non-primary context current) looks the address
// up again. Make the first call on a device, and the first under a new
// context, before any stream capture. All calls on a device share the one
// array and it keeps the last call's contents; nothing in it has to start at
// zero, because the dense kernel writes all M*N partials before the
// residual kernel reads them. Calls whose GPU work overlaps (other streams,
// other threads) race on the array.

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

constexpr int64_t kNoallocMaxOutputs = MQ_UNFUSED_NOALLOC_MAX_OUTPUTS;

static __device__ __align__(256) float g_unfused_scratch[kNoallocMaxOutputs];

std::mutex g_scratch_mu;
struct ScratchEntry {
    CUcontext ctx = nullptr;
    void *ptr = nullptr;
};
ScratchEntry g_scratch[256];

// The driver's cuCtxGetCurrent, reached through the runtime (the library
// links the CUDA runtime only).
CUresult current_context(CUcontext *ctx) {
    using Fn = CUresult (*)(CUcontext *);
    static Fn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<Fn>(p);
    });
    return fn ? fn(ctx) : CUDA_ERROR_NOT_FOUND;
}

// Device address of g_unfused_scratch on `dev` (the current device) in the
// current context.
mq_status scratch_address(int dev, float **out) {
    if (dev < 0 || dev >= 256) return fail(MQ_ERR_UNSUPPORTED, "device ordinal out of range");
    CUcontext ctx = nullptr;
    if (current_context(&ctx) != CUDA_SUCCESS || !ctx)
        return fail(MQ_ERR_CUDA, "no current CUDA context for the built-in scratch");
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchEntry &e = g_scratch[dev];
    if (!e.ptr || e.ctx != ctx) {
        void *p = nullptr;
        const cudaError_t r = cudaGetSymbolAddress(&p, g_unfused_scratch);
        if (r != cudaSuccess || !p)
            return fail(MQ_ERR_CUDA, std::string("cudaGetSymbolAddress for the built-in "
                                                 "scratch failed: ") +
                                         cudaGetErrorString(r));
        e.ctx = ctx;
        e.ptr = p;
    }
    *out = static_cast<float *>(e.ptr);
    return MQ_OK;
}

}  // namespace
}  // namespace mq

extern "C" mq_status mq_linear_unfused_noalloc(const mq_weight *w, const void *X, int64_t M,
                                               void *Y, mq_stream stream) {
    using namespace mq;
    if (!w) return fail(MQ_ERR_INVALID_ARG, "weight handle is NULL");
    if (M < 0) return fail(MQ_ERR_INVALID_ARG, "M must be >= 0");
    if (M == 0) return MQ_OK;
    if (!X || !Y) return fail(MQ_ERR_INVALID_ARG, "X or Y is NULL");
    if ((reinterpret_cast<uintptr_t>(X) & 15) || (reinterpret_cast<uintptr_t>(Y) & 15))
        return fail(MQ_ERR_INVALID_ARG, "X and Y must be 16-byte aligned");
    const DeviceWeight &d = weight_device(w);
    if (M > kNoallocMaxOutputs / d.N)
        return fail(MQ_ERR_INVALID_ARG,
                    "M*N exceeds the built-in scratch of " +
                        std::to_string(kNoallocMaxOutputs) +
                        " partial outputs; use mq_linear_unfused with a workspace");
    mq_info info;
    if (mq_status st = mq_get_info(w, &info)) return st;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (dev != info.device)
        return fail(MQ_ERR_INVALID_ARG, "the current device is not the device that packed the weight");
    float *part = nullptr;
    if (mq_status st = scratch_address(dev, &part)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    mq_status st = (M <= 16) ? launch_decode(w, X, static_cast<int>(M), Y, s, part)
                             : launch_prefill(w, X, M, Y, s, part);
    if (st) return st;
    return launch_residual_merge(w, X, M, part, Y, s);
}
