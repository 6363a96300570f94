// kq_common.cuh -- small device helpers shared by the libkq kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kq {

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float v) {
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t *>(&b);
}

// Two floats -> one 32-bit word holding two bf16 values (first in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// v = hi + lo with hi = bf16(v), lo = bf16(v - hi): about 16 significant bits.
__device__ __forceinline__ void split_bf16(float v, float &hi, float &lo) {
    hi = __bfloat162float(__float2bfloat16_rn(v));
    lo = v - hi;  // exact in fp32
}

// Per-token symmetric INT4 code: clamp(round_half_even(y / s), -8, 7), 0 if s == 0.
__device__ __forceinline__ int quant_int4(float y, float s) {
    if (!(s > 0.0f)) return 0;
    float r = __fdiv_rn(y, s);
    r = fminf(fmaxf(r, -8.0f), 7.0f);
    return static_cast<int>(rintf(r));
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Programmatic dependent launch.  launch_dependents: the next kernel on the
// stream may be scheduled once every CTA of this grid has executed it (its CTAs
// then start on SMs as this grid's CTAs exit).  wait: block until the previous
// kernel's grid has completed and its memory operations are visible (returns at
// once when the launch had no programmatic dependency).
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launches `kern` with programmatic stream serialization: once every CTA of the
// previous kernel on the stream has executed griddepcontrol.launch_dependents,
// this grid may be scheduled, so its launch and on-chip set-up overlap that
// grid's last CTAs.  The kernel must execute griddepcontrol.wait before its
// first global-memory access (after a kernel that never signals, the launch
// simply follows its completion, as without the attribute).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_overlapped(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem,
                                     cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace kq
