// Separate residual kernel of the unfused comparison path:
// Y[m][n] = bf16(P[m][n] + s_r[n] * sum_e q_e * X[m][c_e]).
//
// This is the split execution MosaicQuant "Methodology" 3. argues against:
// a second kernel that reloads the activations and merges the dense
// kernel's partial outputs (fp32 partials, so the result is rounded once).
// One thread per output, consecutive threads along n; each walks its row's
// CSR entries and gathers X through the caches.

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

__global__ void __launch_bounds__(256)
    residual_merge_kernel(const __nv_bfloat16 *__restrict__ X, const float *__restrict__ P,
                          __nv_bfloat16 *__restrict__ Y, const int32_t *__restrict__ row_ptr,
                          const uint16_t *__restrict__ col, const uint8_t *__restrict__ val,
                          const uint16_t *__restrict__ rscale, int64_t M, int N, int K) {
    const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= M * N) return;
    const int64_t m = idx / N;
    const int n = static_cast<int>(idx - m * N);
    const int a = row_ptr[n], b = row_ptr[n + 1];
    const uint16_t *xrow = reinterpret_cast<const uint16_t *>(X) + m * K;
    float part = 0.f;
    for (int e = a; e < b; ++e) {
        const uint32_t byte = val[e >> 1];
        const int q = static_cast<int>(((byte >> ((e & 1) * 4)) & 0xF) ^ 8) - 8;
        part = fmaf(static_cast<float>(q), bf16_bits_to_f32(xrow[col[e]]), part);
    }
    Y[idx] = __float2bfloat16_rn(fmaf(half_bits_to_f32(rscale[n]), part, P[idx]));
}

}  // namespace

mq_status launch_residual_merge(const mq_weight *w, const void *X, int64_t M,
                                const float *partial, void *Y, cudaStream_t stream) {
    const DeviceWeight &d = weight_device(w);
    const int64_t total = M * d.N;
    const unsigned blocks = static_cast<unsigned>((total + 255) / 256);
    residual_merge_kernel<<<blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(X), partial, static_cast<__nv_bfloat16 *>(Y),
        d.row_ptr, d.col, d.val, d.rscale, M, static_cast<int>(d.N), static_cast<int>(d.K));
    cudaError_t e = cudaPeekAtLastError();
    if (e != cudaSuccess)
        return fail(MQ_ERR_CUDA, std::string("residual launch: ") + cudaGetErrorString(e));
    return MQ_OK;
}

}  // namespace mq
