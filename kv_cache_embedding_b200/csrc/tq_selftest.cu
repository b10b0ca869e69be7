// tq_selftest_wait_timeout: exercises the bounded device-side wait that every
// tensor-core kernel of the library uses, on a barrier nothing completes, so
// that the time-out path (give up, record the status, exit) can be checked
// without faulting or hanging the GPU.
#include "tq_internal.cuh"
#include "tq_sm100.cuh"

namespace tq {
namespace {

__global__ void k_wait_timeout(int* err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);  // expects one arrival; none comes
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !sm100::mbar_wait(&bar, 0, &abort_flag, limit_ns))
        atomicCAS(err, 0, TQ_ERR_DEVICE_TIMEOUT * 1000 - 99);
}

}  // namespace
}  // namespace tq

extern "C" int tq_selftest_wait_timeout(void* d_ws, uint64_t limit_ns, void* stream) {
    if (!d_ws || limit_ns == 0 || limit_ns > 2000000000ull) return TQ_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    TQ_TRY_CUDA(cudaMemsetAsync(d_ws, 0, sizeof(int), s));
    tq::k_wait_timeout<<<1, 32, 0, s>>>((int*)d_ws, limit_ns);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}
