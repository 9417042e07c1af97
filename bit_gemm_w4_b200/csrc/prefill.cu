// Prefill launcher. Until the tensor-core kernel lands this runs the decode
// kernel over blocks of 16 tokens (correct for any M, re-reads W per block).

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {

mq_status launch_prefill(const mq_weight *w, const void *X, int64_t M, void *Y,
                         cudaStream_t stream, float *partial) {
    const DeviceWeight &d = weight_device(w);
    const auto *x = static_cast<const __nv_bfloat16 *>(X);
    auto *y = static_cast<__nv_bfloat16 *>(Y);
    for (int64_t m0 = 0; m0 < M; m0 += 16) {
        int mb = static_cast<int>(std::min<int64_t>(16, M - m0));
        mq_status st = launch_decode(w, x + m0 * d.K, mb, y + m0 * d.N, stream,
                                     partial ? partial + m0 * d.N : nullptr);
        if (st) return st;
    }
    return MQ_OK;
}

}  // namespace mq
