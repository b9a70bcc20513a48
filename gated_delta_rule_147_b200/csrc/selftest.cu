// Diagnostic for the bounded-wait mechanism of the tensor-core kernels: one
// block waits, with the same bounded mbarrier wait the chunk kernel uses, on
// a barrier phase that nothing ever completes. The wait must give up, report
// GDR_DEVICE_TIMEOUT in the caller's status word and let the block end.
#include "common.cuh"

namespace gdr {

__global__ void bounded_wait_probe(int* d_status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    const bool ok = mbar_wait(&bar, 0);  // no thread or copy ever arrives
    if (!__syncthreads_and(ok) && threadIdx.x == 0) flag_status(d_status, GDR_DEVICE_TIMEOUT);
}

}  // namespace gdr

extern "C" gdr_status gdr_selftest_bounded_wait(int* d_status, void* stream) {
    if (!d_status) return GDR_ERR_INVALID_ARG;
    gdr::bounded_wait_probe<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(d_status);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
}
