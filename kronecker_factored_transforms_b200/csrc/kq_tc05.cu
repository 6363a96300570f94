// kq_tc05.cu -- persistent fused kernel on the 5th-generation tensor cores
// (tcgen05.mma with TMEM accumulators), plus the device status word that its
// bounded waits report through.
#include "kq_common.cuh"
#include "kq_internal.h"

namespace kq {

// Nonzero when a bounded wait gave up; each site ORs its own bit.
__device__ unsigned int g_device_error = 0;

cudaError_t read_and_clear_device_error(cudaStream_t stream, unsigned int *code) {
    unsigned int zero = 0;
    cudaError_t err = cudaMemcpyFromSymbolAsync(code, g_device_error, sizeof(unsigned int), 0,
                                                cudaMemcpyDeviceToHost, stream);
    if (err != cudaSuccess) return err;
    err = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(unsigned int), 0,
                                  cudaMemcpyHostToDevice, stream);
    if (err != cudaSuccess) return err;
    return cudaStreamSynchronize(stream);
}

bool tc05_supports(int, int, bool) { return false; }

cudaError_t launch_tc05(const LaunchArgs &) { return cudaErrorNotSupported; }

}  // namespace kq
