// kq_internal.h -- launch plumbing shared between the C ABI and the kernels.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kq {

struct LaunchArgs {
    const uint16_t *x;
    const uint16_t *P1;
    const uint16_t *P2;
    const float *cinv;   // nullptr: c = 1
    float alpha;
    uint8_t *q_out;      // quantise mode
    float *scale_out;
    float *y_out;        // transform-only mode when non-null
    int64_t T;
    int n1, n2;
    int num_sms;
    int device;
    cudaStream_t stream;
};

// General warp-level MMA kernel: every supported shape.
cudaError_t launch_warp_mma(const LaunchArgs &a);

// Persistent tcgen05/TMEM kernel for the shapes it covers (alpha >= 2^-19).
bool tc05_supports(int n1, int n2, bool scaled);
cudaError_t launch_tc05(const LaunchArgs &a);

// Group-pipelined tcgen05/TMEM kernel (n1 = 64, n2 in {64, 128}; alpha >= 2^-19).
bool fused_supports(int n1, int n2, bool scaled);
cudaError_t launch_fused(const LaunchArgs &a);

// Diagnostic: a kernel whose bounded wait on a never-signalled barrier gives up.
cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t stream);

// cuTensorMapEncodeTiled from the driver (null if unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Device address of the status word (for kernels in other translation units).
cudaError_t device_error_word(int device, unsigned int **word);

// Read and clear the device status word set by bounded waits that gave up.
cudaError_t read_and_clear_device_error(cudaStream_t stream, unsigned int *code);

// Check entry: q * s -> P1inv^T Y P2inv -> * c, fp32 on CUDA cores.
cudaError_t launch_dequant_inverse(const uint8_t *q, const float *scale, const float *P1inv,
                                   const float *P2inv, const float *c, float *x_hat, int64_t T,
                                   int n1, int n2, cudaStream_t stream);

// W4A4 product of packed INT4 codes: y = sx[m] sw[o] sum_k qx[m][k] qw[o][k].
cudaError_t launch_w4a4_gemm(const uint8_t *qx, const float *sx, const uint8_t *qw, const float *sw, void *y,
                             bool bf16_out, int64_t M, int64_t N, int64_t K, int device, cudaStream_t stream);

// Per-head transform + INT4 per row: rows of head_dim (64 or 128) values.
cudaError_t launch_rowwise(const uint16_t *x, const uint16_t *Ph, float alpha, uint8_t *q_out, float *scale_out,
                           int64_t R, int head_dim, int num_sms, int device, cudaStream_t stream);
// The same transform with NVFP4 rows: E2M1 codes, an E4M3 scale per 16 values,
// an fp32 scale per row.
cudaError_t launch_rowwise_nvfp4(const uint16_t *x, const uint16_t *Ph, uint8_t *q_out, uint8_t *bscale_out,
                                 float *scale_out, int64_t R, int head_dim, int num_sms, int device,
                                 cudaStream_t stream);

// Two-stage transform + INT4 for factors up to 256 through a workspace of
// two_stage_workspace_bytes(T, n1, n2) bytes (Z^T hi then lo, bf16).
bool two_stage_supports(int n1, int n2);
uint64_t two_stage_workspace_bytes(int64_t T, int n1, int n2);
cudaError_t launch_two_stage(const LaunchArgs &a, void *workspace);

// The static workspace of kq_transform_quant_two_stage_static (one per device).
constexpr uint64_t kStaticScratchBytes = uint64_t(64) << 20;
cudaError_t static_scratch(int device, void **ptr);

}  // namespace kq
