// kq_scratch.cu -- the static device workspace behind
// kq_transform_quant_two_stage_static: one array of kStaticScratchBytes per
// device, part of the library image, so that entry allocates nothing.  It is
// kept in its own translation unit so the array's module is only loaded when
// the entry first asks for its address.
#include <mutex>

#include "kq_internal.h"

namespace kq {
namespace {

__device__ __align__(256) unsigned char g_two_stage_scratch[kStaticScratchBytes];

}  // namespace

cudaError_t static_scratch(int device, void **ptr) {
    static std::mutex mu;
    static bool looked_up[64];
    static void *addr[64];
    static cudaError_t status[64];
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!looked_up[device]) {
        // once per device, with that device current
        int cur = -1;
        cudaError_t e = cudaGetDevice(&cur);
        if (e == cudaSuccess && cur != device) e = cudaErrorInvalidDevice;
        void *p = nullptr;
        if (e == cudaSuccess) e = cudaGetSymbolAddress(&p, g_two_stage_scratch);
        addr[device] = e == cudaSuccess ? p : nullptr;
        status[device] = e;
        looked_up[device] = true;
    }
    *ptr = addr[device];
    return status[device];
}

}  // namespace kq
