/*
 * kq.h -- C ABI of libkq: fused Kronecker-factored transform + per-token
 * INT4 quantisation on an NVIDIA B200 (sm_100a).
 *
 * The operation (FlatQuant page, "Kronecker factorization" and "The fused
 * kernel"; Kronecker Product page, "Definition" and the identity
 * vec(V)(P1 (x) P2) = vec(P1^T V P2)):
 *
 *   for every token row x (length n = n1*n2, bf16):
 *     x'  = x * cinv                  (per-channel scale 1/c; cinv NULL: c = 1)
 *     X~  = x' read row-major as an n1 x n2 matrix, X~[a][b] = x'[a*n2 + b]
 *     Y~  = P1^T X~ P2                (= x' (P1 (x) P2)),  y[i*n2 + j] = Y~[i][j]
 *     s   = alpha * max_k |y_k| / 7   (one fp32 scale per token; clip after the
 *                                      transform: FlatQuant page, "Per-channel
 *                                      scaling and learnable clipping")
 *     q_k = clamp(round_half_even(y_k / s), -8, 7)   (q = 0 when s = 0)
 *     byte k of the token's output = (q_{2k} & 0xF) | ((q_{2k+1} & 0xF) << 4)
 *
 * Numerics: bf16 operands, fp32 accumulation on the tensor cores.  Every
 * operand that is rounded to bf16 on the way (Z = X~' P2, and x' when cinv
 * is given) is carried as a hi + lo pair of bf16 values, so the fp32 result
 * is accurate to about 2^-16 of the token's absmax.
 *
 * Conventions shared by every entry point:
 *   - All data pointers are DEVICE pointers into memory the caller owns.
 *     The library allocates nothing and keeps no per-call state.
 *   - bf16 arrays are passed as uint16_t bit patterns.  Matrices are dense
 *     and row-major with no padding between rows.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  Inputs are read-only; outputs must not
 *     overlap inputs (checked: KQ_ERR_ARG).
 *   - The transform kernels are launched with programmatic stream
 *     serialization: a launch may be scheduled while the previous kernel on
 *     the stream (when that kernel allows it) is finishing, but it reads and
 *     writes global memory only after that kernel has completed, so stream
 *     order is kept for every buffer.
 *   - T == 0 is a no-op that returns KQ_OK without touching any pointer.
 *   - Arguments are checked before anything is launched; on error nothing
 *     runs and the status says why.  Faults inside a kernel surface at the
 *     caller's next synchronisation, as with any CUDA kernel.
 *   - Supported factor sizes: n1 and n2 multiples of 16 in [16, 128].
 */
#ifndef KQ_H
#define KQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kq_status {
    KQ_OK = 0,
    KQ_ERR_NULL = -1,        /* a required pointer is NULL (with T > 0)             */
    KQ_ERR_SHAPE = -2,       /* T < 0, n1 <= 0, n2 <= 0, or T*n1*n2 overflows      */
    KQ_ERR_UNSUPPORTED = -3, /* a size or parameter the entry does not cover       */
    KQ_ERR_ALIGN = -4,       /* a pointer is not aligned as documented             */
    KQ_ERR_ARG = -5,         /* alpha not finite in (0, 1], or outputs overlap inputs */
    KQ_ERR_CUDA = -6,        /* a CUDA runtime call or a kernel launch failed      */
    KQ_ERR_TIMEOUT = -7      /* a bounded wait inside a kernel gave up (see
                                kq_device_error)                                    */
} kq_status;

/* Same type as cudaStream_t, declared here so the header needs no CUDA headers. */
typedef struct CUstream_st *kq_stream_t;

/*
 * kq_transform_quant -- the fused hot path.  Every supported shape runs on the
 * tensor cores (alpha >= 2^-19): short launches at n1 = 64, n2 in {64, 128}
 * (up to 56 groups of 128/n2 tokens per SM without cinv, 4 with it) in the
 * pair-pipelined kernel, everything else in the batch-pipelined kernel
 * (n2 = 16, 32, 48 padded to 64 columns per token, 80, 96, 112 to 128);
 * kq_kernel_for names the kernel a call runs.  alpha below 2^-19 runs on the
 * warp-level MMA kernel.
 *   x         [T, n1*n2] bf16, 16-byte aligned.
 *   P1        [n1, n1] bf16 (left factor; applied transposed), 16-byte aligned.
 *   P2        [n2, n2] bf16 (right factor), 16-byte aligned.
 *   cinv      [n1*n2] fp32 = 1/c, 16-byte aligned, or NULL for c = 1.
 *   alpha     clip ratio, finite, 0 < alpha <= 1.
 *   q_out     [T, n1*n2/2] uint8 packed INT4 codes, 16-byte aligned.
 *   scale_out [T] fp32 per-token scale s, 4-byte aligned.
 * Only q_out and scale_out are written; no intermediate touches global memory.
 */
kq_status kq_transform_quant(const uint16_t *x, const uint16_t *P1, const uint16_t *P2,
                             const float *cinv, float alpha, uint8_t *q_out, float *scale_out,
                             int64_t T, int n1, int n2, kq_stream_t stream);

/*
 * kq_transform -- check entry: the same transform, y written out in fp32
 * instead of being quantised.  y_out [T, n1*n2] fp32, 16-byte aligned.
 * Other arguments as for kq_transform_quant.
 */
kq_status kq_transform(const uint16_t *x, const uint16_t *P1, const uint16_t *P2,
                       const float *cinv, float *y_out, int64_t T, int n1, int n2,
                       kq_stream_t stream);

/*
 * kq_dequant_inverse -- check entry: undo the quantised transform.
 * The inverse of P1 (x) P2 is P1^-1 (x) P2^-1 (FlatQuant page, "Kronecker
 * factorization"; the page inverts P through its SVD, "Learning the affine
 * transformation"), so with Y^ = q * s:
 *     x^~ = P1^-T Y^ P2^-1,   x^ = x^~ * c.
 *   q      [T, n1*n2/2] packed codes as written by kq_transform_quant, 16-byte aligned.
 *   scale  [T] fp32.
 *   P1inv  [n1, n1] fp32, P2inv [n2, n2] fp32: inverses computed by the caller
 *          (e.g. in fp64 on the host, then rounded to fp32).
 *   c      [n1*n2] fp32 channel scale (the reciprocal of cinv), or NULL for c = 1.
 *   x_hat  [T, n1*n2] fp32 output, 16-byte aligned.
 * Arithmetic is fp32 on CUDA cores; this entry is a checker, not a hot path.
 */
kq_status kq_dequant_inverse(const uint8_t *q, const float *scale, const float *P1inv,
                             const float *P2inv, const float *c, float *x_hat, int64_t T,
                             int n1, int n2, kq_stream_t stream);

/*
 * kq_w4a4_gemm -- the product that consumes the codes (FlatQuant page,
 * "Kronecker factorization": Q(X P) Q(P^-1 W^T), the W4A4 linear layer):
 *
 *     y[m][o] = sx[m] * sw[o] * sum_k qx[m][k] * qw[o][k]
 *
 * qx      [M, K/2] device, packed INT4 activation codes, row-major, as written
 *         by kq_transform_quant (element 2k in the low nibble of byte k,
 *         two's complement); 16-byte aligned.
 * sx      [M] device fp32, one scale per row of qx (kq_transform_quant's
 *         scale_out).
 * qw      [N, K/2] device, packed INT4 weight codes in the same layout: one
 *         row per output channel, e.g. the weight rows transformed with
 *         factors P1^-T, P2^-T and the channel vector c and quantised by
 *         kq_transform_quant; 16-byte aligned.
 * sw      [N] device fp32, one scale per output channel.
 * y       [M, N] device fp32, row-major, written; must not overlap the inputs.
 * K       multiple of 128 in [128, 262144] (every n = n1 n2 of kq_transform_quant);
 *         M, N >= 0 (0 is a no-op).
 * The integer sums are exact (|sum| <= 64 K < 2^24); y is (float(sum) * sx[m])
 * * sw[o] in fp32.  The library allocates nothing; asynchronous on `stream`.
 * Returns KQ_ERR_SHAPE for negative M/N or a K out of range, KQ_ERR_NULL,
 * KQ_ERR_ALIGN, KQ_ERR_ARG for overlapping output, KQ_ERR_CUDA if the launch
 * fails.
 */
kq_status kq_w4a4_gemm(const uint8_t *qx, const float *sx, const uint8_t *qw, const float *sw, float *y,
                       int64_t M, int64_t N, int64_t K, kq_stream_t stream);

/*
 * kq_w4a4_gemm_bf16 -- kq_w4a4_gemm with a bf16 output (the next layer's
 * activation dtype): y [M, N] device bf16 bits, row-major, 2-byte aligned,
 * written; each element is kq_w4a4_gemm's fp32 value rounded to the nearest
 * bf16 (ties to even).  Same arguments, checks and status codes otherwise.
 * Writing half the bytes is what a large product needs: at M = N = K = 8192
 * the fp32 output is the larger part of its memory traffic.
 */
kq_status kq_w4a4_gemm_bf16(const uint8_t *qx, const float *sx, const uint8_t *qw, const float *sw, uint16_t *y,
                            int64_t M, int64_t N, int64_t K, kq_stream_t stream);

/*
 * kq_headwise_transform_quant -- the per-head transform of the key / value
 * cache (FlatQuant page: P_h and P_v keep their full per-head shape; keys and
 * values are transformed per head and quantised before storage).  For every
 * token t and head h, the row x[t, h, :] of head_dim values is multiplied by
 * the full factor Ph and quantised on its own with the INT4 rule of
 * kq_transform_quant (s = alpha * max|y| / 7, round half to even, clamp to
 * [-8, 7], two codes per byte, element 2k in the low nibble).
 *
 * x         [T, heads * head_dim] device bf16, row-major (head-major within a
 *           token), 16-byte aligned.
 * Ph        [head_dim, head_dim] device bf16, row-major, 16-byte aligned.
 * alpha     clip ratio in [2^-19, 1].
 * q_out     [T, heads * head_dim / 2] device uint8, 16-byte aligned, written.
 * scale_out [T, heads] device fp32, written (0 for an all-zero row).
 * head_dim  64 or 128; heads >= 1 (any count, e.g. 8 grouped-query heads);
 *           T * heads < 2^31.
 * Returns KQ_ERR_SHAPE, KQ_ERR_UNSUPPORTED (head_dim, or alpha below 2^-19),
 * KQ_ERR_ARG (alpha outside (0, 1], overlapping buffers), KQ_ERR_NULL,
 * KQ_ERR_ALIGN, KQ_ERR_CUDA.  Asynchronous on `stream`; allocates nothing.
 */
kq_status kq_headwise_transform_quant(const uint16_t *x, const uint16_t *Ph, float alpha, uint8_t *q_out,
                                      float *scale_out, int64_t T, int heads, int head_dim, kq_stream_t stream);

/*
 * kq_headwise_transform_quant_nvfp4 -- the per-head transform of
 * kq_headwise_transform_quant with NVFP4 rows instead of INT4 (the 4-bit
 * floating-point format with two levels of scale that the FlatQuant page
 * leaves open; the High-Rate Quantized Matrix Multiplication page calls it a
 * multi-scaled, group-scaled format).  For every row y = x[t, h, :] Ph of
 * head_dim values:
 *   row scale     s = max|y| / (6 * 448)                       (fp32)
 *   block scale   b = E4M3(max over the block |y| / (6 s))     per 16 values,
 *                 round to nearest even, saturating at 448
 *   element       q = E2M1(y / (decode(b) * s)), round to nearest even,
 *                 saturating at +-6; a value that rounds to zero is +0
 * E2M1 codes: bit 3 the sign, magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; two per
 * byte, element 2k in the low nibble.  A row (block) with a zero scale has
 * zero block (element) codes.
 *
 * x, Ph, T, heads, head_dim: as kq_headwise_transform_quant.
 * q_out       [T, heads * head_dim / 2] device uint8, 16-byte aligned, written.
 * block_scale_out [T, heads * head_dim / 16] device uint8 (E4M3 codes),
 *             8-byte aligned, written.
 * scale_out   [T, heads] device fp32, written.
 * Returns KQ_ERR_SHAPE, KQ_ERR_UNSUPPORTED (head_dim), KQ_ERR_ARG (overlapping
 * buffers), KQ_ERR_NULL, KQ_ERR_ALIGN, KQ_ERR_CUDA.  Asynchronous on
 * `stream`; allocates nothing.
 */
kq_status kq_headwise_transform_quant_nvfp4(const uint16_t *x, const uint16_t *Ph, uint8_t *q_out,
                                            uint8_t *block_scale_out, float *scale_out, int64_t T, int heads,
                                            int head_dim, kq_stream_t stream);

/*
 * kq_transform_quant_two_stage -- kq_transform_quant for factors up to 256
 * (FlatQuant page, "The fused kernel", Figure 8 (c): factors too large for one
 * on-chip pass; the transform runs as two stages with the intermediate in
 * global memory).  Same result and INT4 rule as kq_transform_quant:
 * Y~ = P1^T X~ P2 for the row-major n1 x n2 view X~ of x o cinv, per-token
 * s = alpha * max|y| / 7, codes clamp(round_half_even(y / s), -8, 7), two per
 * byte with element 2k in the low nibble, output element k = i * n2 + j.
 * Stage 1 writes Z^T = (X~ P2)^T of every token to `workspace` as a hi/lo
 * bf16 pair; stage 2 forms P1^T Z per token, quantises and packs.  Neither
 * Y~ nor an fp32 intermediate reaches global memory.
 *
 * x, P1, P2, cinv, alpha, q_out, scale_out, T, n1, n2: as kq_transform_quant,
 *           except that n1 and n2 are multiples of 16 in [16, 256] and
 *           T * n1 * n2 < 2^31.
 * workspace caller-owned device scratch of at least
 *           kq_two_stage_workspace_bytes(T, n1, n2) = 4 * T * n1 * Jp bytes,
 *           Jp = 128 * ceil(n2 / 128) (Z^T rows per token, padded to whole
 *           128-row slices), 16-byte aligned; overwritten, and must stay
 *           untouched until the work on `stream` has finished.
 * Returns KQ_ERR_SHAPE, KQ_ERR_UNSUPPORTED (factor size, or alpha below
 * 2^-19), KQ_ERR_ARG (alpha outside (0, 1], workspace too small, overlapping
 * buffers), KQ_ERR_NULL, KQ_ERR_ALIGN, KQ_ERR_CUDA.  Asynchronous on
 * `stream`; allocates nothing.
 */
kq_status kq_transform_quant_two_stage(const uint16_t *x, const uint16_t *P1, const uint16_t *P2,
                                       const float *cinv, float alpha, uint8_t *q_out, float *scale_out,
                                       void *workspace, uint64_t workspace_bytes, int64_t T, int n1, int n2,
                                       kq_stream_t stream);

/*
 * kq_transform_quant_two_stage_static -- kq_transform_quant_two_stage with
 * its workspace taken from a static device array inside libkq instead of a
 * caller buffer, so the call allocates nothing and needs no scratch from the
 * caller.  The pages have no counterpart for this entry: it is a convenience
 * of this library for callers without an allocator at hand.
 *
 * Arguments and results as kq_transform_quant_two_stage (without workspace
 * and workspace_bytes).  Limit: kq_two_stage_workspace_bytes(T, n1, n2) <=
 * KQ_STATIC_WORKSPACE_BYTES (64 MiB: e.g. T <= 256 at n1 = n2 = 256); a larger
 * request returns KQ_ERR_ARG before anything is launched.
 *
 * The array is ONE per device and process, shared by every call of this entry
 * on that device.  Two calls whose work can overlap on the device -- issued on
 * different streams without an ordering between them, or from several host
 * threads -- race on it and can return wrong codes; calls on one stream are
 * ordered and safe.  The first call on a device looks up the array's address
 * (cudaGetSymbolAddress, which can load the module) and must come before any
 * stream capture on that device; a lookup that fails is reported
 * (KQ_ERR_CUDA) and tried again by the next call.  Nothing is claimed about
 * calling this entry inside a captured graph.
 *
 * Device memory: under CUDA's default lazy module loading the 64 MiB are
 * taken on a device when this entry is first called there, and kept until
 * the process exits.  With CUDA_MODULE_LOADING=EAGER they are taken on every
 * device the process creates a context on as soon as libkq is loaded, even if
 * this entry is never called.
 */
#define KQ_STATIC_WORKSPACE_BYTES (64ull * 1024ull * 1024ull)
kq_status kq_transform_quant_two_stage_static(const uint16_t *x, const uint16_t *P1, const uint16_t *P2,
                                              const float *cinv, float alpha, uint8_t *q_out, float *scale_out,
                                              int64_t T, int n1, int n2, kq_stream_t stream);

/* Workspace bytes kq_transform_quant_two_stage needs: 4 * T * n1 * 128 * ceil(n2 / 128) (0 for T <= 0). */
uint64_t kq_two_stage_workspace_bytes(int64_t T, int n1, int n2);

/*
 * kq_device_error -- read and clear the device-side status word that the
 * kernels set when a bounded wait gives up (they then skip their remaining
 * work instead of hanging).  Synchronises `stream`.  *code receives 0 when
 * no wait timed out since the last call, else a nonzero site code.
 * Returns KQ_ERR_NULL for a NULL code, KQ_ERR_CUDA if the read fails.
 */
kq_status kq_device_error(kq_stream_t stream, int *code);

/*
 * kq_selftest_bounded_wait -- diagnostic for the failure path of the bounded
 * waits.  Launches one tiny kernel on `stream` whose thread waits on a
 * shared-memory barrier that nothing ever signals; after `limit_us`
 * microseconds (1 .. 10,000,000) the wait gives up, records site code 256 in
 * the device status word and the kernel returns normally.  Nothing faults and
 * the context stays usable; kq_device_error then reports 256.
 * Returns KQ_ERR_ARG for a limit outside the range, KQ_ERR_CUDA if the launch
 * fails.
 */
kq_status kq_selftest_bounded_wait(int64_t limit_us, kq_stream_t stream);

/* Human-readable text for a kq_status value (static storage, never NULL). */
const char *kq_status_string(int status);

/*
 * Name of the kernel kq_transform_quant launches for this shape on long inputs
 * (static storage): "kq_tc05_fused_kernel" for every supported shape, or
 * "unsupported".  Host-only; touches no device state.
 */
const char *kq_kernel_name(int n1, int n2, int has_cinv);

/*
 * Name of the kernel kq_transform_quant launches for this call size (T tokens)
 * and clip ratio on the current device (static storage), or "unsupported".
 * Short launches of n1 = 64 and n2 in {64, 128} (at most 56 groups of 128/n2
 * tokens per SM without cinv, 4 with it) run kq_fused_kernel, the pair-pipelined
 * kernel; longer ones
 * and every other shape the kernel that kq_kernel_name names; alpha below
 * 2^-19 kq_warp_mma_kernel.  Reads the device's SM count (148 when no device
 * is visible); launches nothing.
 */
const char *kq_kernel_for(int64_t T, int n1, int n2, int has_cinv, float alpha);

/* Library version: major * 10000 + minor * 100 + patch. */
int kq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KQ_H */
