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

}  // namespace kq
