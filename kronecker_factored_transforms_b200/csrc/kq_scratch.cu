// kq_scratch.cu -- the static device workspace behind
// kq_transform_quant_two_stage_static: one array of kStaticScratchBytes per
// device, part of the library image, so that entry allocates nothing.  It is
// kept in its own translation unit so that, under CUDA's lazy module loading
// (the default), the array's module -- and with it the 64 MiB on the device --
// is only loaded when the entry first asks for its address.  With eager
// loading (CUDA_MODULE_LOADING=EAGER) every process that loads libkq holds
// the 64 MiB on each device it creates a context on, whether or not it ever
// calls the entry.
#include <mutex>

#include "kq_internal.h"

namespace kq {
namespace {

__device__ __align__(256) unsigned char g_two_stage_scratch[kStaticScratchBytes];

}  // namespace

cudaError_t static_scratch(int device, void **ptr) {
    static std::mutex mu;
    static void *addr[64];  // non-null once the lookup succeeded on that device
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[device]) {
        // With that device current.  Only a successful lookup is kept: a failed
        // one (a transient error, or a first call made while the stream was being
        // captured) is reported and tried again on the next call.
        int cur = -1;
        cudaError_t e = cudaGetDevice(&cur);
        if (e == cudaSuccess && cur != device) e = cudaErrorInvalidDevice;
        void *p = nullptr;
        if (e == cudaSuccess) e = cudaGetSymbolAddress(&p, g_two_stage_scratch);
        if (e != cudaSuccess || !p) {
            *ptr = nullptr;
            return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
        }
        addr[device] = p;
    }
    *ptr = addr[device];
    return cudaSuccess;
}

}  // namespace kq
