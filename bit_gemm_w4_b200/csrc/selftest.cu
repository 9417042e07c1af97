// Self-test of the bounded mbarrier wait that every pipeline of the library
// uses: a wait on a phase that completed returns true; a wait on a phase
// that nobody completes gives up after its cycle limit, records its code in
// the error word and raises the abort flag; a later wait then returns at
// once without overwriting the first code. Nothing faults and nothing hangs:
// the wait that gives up is bounded by a short, caller-chosen limit.

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

__device__ int g_selftest[4];

__global__ void bounded_wait_kernel(long long limit) {
    __shared__ __align__(8) uint64_t bar[2];
    __shared__ int err_word;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        err_word = 0;
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_arrive(&bar[1]);  // completes phase 0 of bar[1]; nobody arrives on bar[0]
        const bool done = mbar_wait(&bar[1], 0, &err_word, kErrWaitFull, &abort_flag, limit);
        const bool stuck = mbar_wait(&bar[0], 0, &err_word, kErrWaitEmpty, &abort_flag, limit);
        const bool later = mbar_wait(&bar[0], 0, &err_word, kErrWaitMma, &abort_flag, limit);
        g_selftest[0] = done ? 1 : 0;
        g_selftest[1] = stuck ? 1 : 0;
        g_selftest[2] = later ? 1 : 0;
        g_selftest[3] = err_word;
    }
}

}  // namespace

mq_status selftest_bounded_wait(long long limit, int32_t *results) {
    bounded_wait_kernel<<<1, 32>>>(limit);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(results, g_selftest, 4 * sizeof(int32_t));
    if (e != cudaSuccess)
        return fail(MQ_ERR_CUDA, std::string("bounded-wait self-test: ") + cudaGetErrorString(e));
    return MQ_OK;
}

}  // namespace mq
