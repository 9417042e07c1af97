// mq_read_probe: a pure streaming read of device memory, the attainable HBM
// read ceiling that the decode kernels are measured against.
//
// The decode kernels stream packed weights that no earlier kernel writes, in
// chains of dependent launches. This kernel does only that read, shaped the
// way the bandwidth is best reached on B200 when measured: a persistent grid
// of two CTAs per SM, each CTA a contiguous stretch of the buffer, every
// thread keeping eight 16-byte streaming loads in flight, and programmatic
// dependent launch with the next launch released at the first instruction
// and this one waiting for its predecessor only before its final write. A
// CUDA graph of such launches over buffers sized like a model's layers gives
// the ceiling for a chain of that shape. It is a measuring aid: the paper has
// no counterpart, and nothing of the product path uses it.

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

constexpr int kProbeThreads = 256;
constexpr int kProbeUnroll = 8;

__global__ void __launch_bounds__(kProbeThreads) read_probe_kernel(const uint4 *src, long long n16,
                                                                   unsigned *sink) {
    pdl_launch_dependents();
    const long long a = n16 * blockIdx.x / gridDim.x, b = n16 * (blockIdx.x + 1) / gridDim.x;
    unsigned acc = 0;
    for (long long i0 = a + threadIdx.x; i0 < b; i0 += static_cast<long long>(kProbeThreads) * kProbeUnroll) {
        uint4 v[kProbeUnroll];
#pragma unroll
        for (int u = 0; u < kProbeUnroll; ++u) {
            const long long i = i0 + static_cast<long long>(u) * kProbeThreads;
            v[u] = i < b ? ldg_stream(reinterpret_cast<const uint32_t *>(src + i)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kProbeUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
    }
    pdl_wait();
    // a data-dependent store the compiler cannot drop (practically never taken)
    if (acc == 0x9E3779B9u) atomicAdd(sink, 1u);
}

}  // namespace
}  // namespace mq

extern "C" mq_status mq_read_probe(const void *buf, int64_t bytes, void *sink, mq_stream stream) {
    using namespace mq;
    if (!buf || !sink) return fail(MQ_ERR_INVALID_ARG, "buffer or sink is NULL");
    if (bytes <= 0 || (bytes & 15)) return fail(MQ_ERR_INVALID_ARG, "bytes must be a positive multiple of 16");
    if ((reinterpret_cast<uintptr_t>(buf) & 15) || (reinterpret_cast<uintptr_t>(sink) & 3))
        return fail(MQ_ERR_INVALID_ARG, "buffer must be 16-byte and sink 4-byte aligned");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * sm_count()));
    cfg.blockDim = dim3(kProbeThreads);
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, read_probe_kernel, static_cast<const uint4 *>(buf),
                                             static_cast<long long>(bytes / 16), static_cast<unsigned *>(sink));
    if (e != cudaSuccess) return fail(MQ_ERR_CUDA, std::string("read probe launch: ") + cudaGetErrorString(e));
    return MQ_OK;
}
