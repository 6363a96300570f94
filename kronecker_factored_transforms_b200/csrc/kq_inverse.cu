// kq_inverse.cu -- check entry: dequantise and undo the Kronecker transform.
//
// (P1 (x) P2)^-1 = P1^-1 (x) P2^-1 (FlatQuant page, "Kronecker
// factorization"), so with Y^ = q * s the recovered row is
//   x^~ = P1^-T Y^ P2^-1  and  x^ = x^~ * c.
// One CTA per token; plain fp32 FMA on CUDA cores, intermediates in shared
// memory.  Not a hot path: it exists to check round trips.
#include "kq_common.cuh"
#include "kq_internal.h"

namespace kq {

namespace {

constexpr int kInvThreads = 256;

__global__ void __launch_bounds__(kInvThreads)
    kq_dequant_inverse_kernel(const uint8_t *__restrict__ q, const float *__restrict__ scale,
                              const float *__restrict__ P1inv, const float *__restrict__ P2inv,
                              const float *__restrict__ c, float *__restrict__ x_hat, int64_t T,
                              int n1, int n2) {
    extern __shared__ __align__(16) float sbuf[];
    const int n = n1 * n2;
    float *sY = sbuf;      // Y^[a][b]
    float *sW = sbuf + n;  // W[a][j] = sum_b Y^[a][b] P2inv[b][j]
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const float s = scale[t];
        const uint8_t *qt = q + t * (n / 2);
        for (int k = threadIdx.x; k < n; k += blockDim.x) {
            const uint8_t byte = qt[k >> 1];
            int nib = (k & 1) ? (byte >> 4) : (byte & 0xF);
            if (nib >= 8) nib -= 16;
            sY[k] = float(nib) * s;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < n; e += blockDim.x) {
            const int a = e / n2, j = e - a * n2;
            float acc = 0.0f;
            for (int b = 0; b < n2; ++b) acc = fmaf(sY[a * n2 + b], __ldg(P2inv + b * n2 + j), acc);
            sW[e] = acc;
        }
        __syncthreads();
        float *xt = x_hat + t * n;
        for (int e = threadIdx.x; e < n; e += blockDim.x) {
            const int i = e / n2, j = e - i * n2;
            float acc = 0.0f;
            for (int a = 0; a < n1; ++a) acc = fmaf(__ldg(P1inv + a * n1 + i), sW[a * n2 + j], acc);
            xt[e] = c ? acc * __ldg(c + e) : acc;
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_dequant_inverse(const uint8_t *q, const float *scale, const float *P1inv,
                                   const float *P2inv, const float *c, float *x_hat, int64_t T,
                                   int n1, int n2, cudaStream_t stream) {
    const size_t smem = size_t(2) * n1 * n2 * sizeof(float);
    cudaError_t err = cudaFuncSetAttribute(kq_dequant_inverse_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    int dev = 0, sms = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return err;
    int64_t grid = int64_t(sms) * 4;
    if (grid > T) grid = T;
    kq_dequant_inverse_kernel<<<unsigned(grid), kInvThreads, smem, stream>>>(q, scale, P1inv, P2inv,
                                                                             c, x_hat, T, n1, n2);
    return cudaGetLastError();
}

}  // namespace kq
