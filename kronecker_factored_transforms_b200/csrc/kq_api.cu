// kq_api.cu -- the extern "C" boundary of libkq (declared in include/kq.h).
//
// Every entry point validates its arguments on the host before anything is
// launched, then picks a kernel for the shape and launches it on the
// caller's stream.  Nothing is allocated and no per-call state is kept.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/kq.h"
#include "kq_internal.h"

namespace {

constexpr int kVersion = 1 * 10000 + 0 * 100 + 0;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
};
Range range_of(const void *p, uint64_t bytes) {
    uintptr_t b = reinterpret_cast<uintptr_t>(p);
    return Range{b, b + static_cast<uintptr_t>(bytes)};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.hi > a.lo && b.hi > b.lo; }

bool supported_factor(int k) { return k >= 16 && k <= 128 && k % 16 == 0; }

// Shape checks shared by all entries: SHAPE, then UNSUPPORTED, then overflow.
kq_status check_shape(int64_t T, int n1, int n2) {
    if (T < 0 || n1 <= 0 || n2 <= 0) return KQ_ERR_SHAPE;
    if (!supported_factor(n1) || !supported_factor(n2)) return KQ_ERR_UNSUPPORTED;
    const int64_t n = int64_t(n1) * n2;
    if (T > INT64_MAX / (n * 4)) return KQ_ERR_SHAPE;  // largest buffer is T*n*4 bytes
    return KQ_OK;
}

kq_status check_alpha(float alpha) {
    if (!std::isfinite(alpha) || !(alpha > 0.0f) || alpha > 1.0f) return KQ_ERR_ARG;
    return KQ_OK;
}

struct DeviceInfo {
    int device = -1;
    int num_sms = 0;
};

// SM count per device, queried once per device.
kq_status device_info(DeviceInfo &info) {
    static std::mutex mu;
    static int sms_cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return KQ_ERR_CUDA;
    if (sms_cache[dev] == 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return KQ_ERR_CUDA;
        sms_cache[dev] = sms;
    }
    info.device = dev;
    info.num_sms = sms_cache[dev];
    return KQ_OK;
}

// Which transform kernel a quantising call of this size runs.  The pair-pipelined
// kernel (n1 = 64) wins on short launches, where its short start-up and per-group
// pipeline matter most, and the batch-pipelined tcgen05 kernel on long ones.  The
// crossover, measured on B200: without cinv about 56 groups of 128 / n2 tokens per
// SM (64x64: 25.2 against 25.8 us at T = 10000, 39.4 against 39.9 at 16384, 152
// against 148 at 65536); with cinv about 4 (64x128: 6.6 against 6.7 us at T = 256,
// 8.0 both at 512, 11.8 against 11.1 at 1024, 19.5 against 15.3 at 2048).
enum class Kern { Fused, Tc05, WarpMma };
Kern choose_kernel(int64_t T, int n1, int n2, bool scaled, float alpha, bool quant, int num_sms) {
    if (!quant || !(alpha >= 0x1p-19f)) return Kern::WarpMma;  // fp32 y out, or the rounding's range
    // tokens per group: 128 / (n2 padded to 64 or 128)
    const int64_t h = n2 <= 64 ? 2 : 1, groups = (T + h - 1) / h;
    // TMA row coordinates are 32-bit: past 2^31 rows of x both tensor-core kernels give way
    if (T * int64_t(n1) >= (int64_t(1) << 31)) return Kern::WarpMma;
    const int64_t per_sm = scaled ? 4 : 56;
    if (kq::fused_supports(n1, n2, scaled) && groups <= per_sm * num_sms) return Kern::Fused;
    if (kq::tc05_supports(n1, n2, scaled)) return Kern::Tc05;
    return Kern::WarpMma;
}

const char *kernel_name_of(Kern k) {
    switch (k) {
    case Kern::Fused: return "kq_fused_kernel";
    case Kern::Tc05: return "kq_tc05_fused_kernel";
    default: return "kq_warp_mma_kernel";
    }
}

kq_status run_transform(const uint16_t *x, const uint16_t *P1, const uint16_t *P2, const float *cinv,
                        float alpha, uint8_t *q_out, float *scale_out, float *y_out, int64_t T,
                        int n1, int n2, kq_stream_t stream) {
    DeviceInfo info;
    kq_status st = device_info(info);
    if (st != KQ_OK) return st;
    kq::LaunchArgs a;
    a.x = x;
    a.P1 = P1;
    a.P2 = P2;
    a.cinv = cinv;
    a.alpha = alpha;
    a.q_out = q_out;
    a.scale_out = scale_out;
    a.y_out = y_out;
    a.T = T;
    a.n1 = n1;
    a.n2 = n2;
    a.num_sms = info.num_sms;
    a.device = info.device;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    // The tcgen05 kernels round with a 1.5 * 2^23 shift, exact while |y / s| = 7 / alpha < 2^22.
    cudaError_t err;
    switch (choose_kernel(T, n1, n2, cinv != nullptr, alpha, y_out == nullptr, info.num_sms)) {
    case Kern::Fused: err = kq::launch_fused(a); break;
    case Kern::Tc05: err = kq::launch_tc05(a); break;
    default: err = kq::launch_warp_mma(a); break;
    }
    return err == cudaSuccess ? KQ_OK : KQ_ERR_CUDA;
}

}  // namespace

extern "C" {

kq_status kq_transform_quant(const uint16_t *x, const uint16_t *P1, const uint16_t *P2,
                             const float *cinv, float alpha, uint8_t *q_out, float *scale_out,
                             int64_t T, int n1, int n2, kq_stream_t stream) {
    kq_status st = check_shape(T, n1, n2);
    if (st != KQ_OK) return st;
    if ((st = check_alpha(alpha)) != KQ_OK) return st;
    if (T == 0) return KQ_OK;
    if (!x || !P1 || !P2 || !q_out || !scale_out) return KQ_ERR_NULL;
    if (!aligned(x, 16) || !aligned(P1, 16) || !aligned(P2, 16) || !aligned(q_out, 16) ||
        !aligned(scale_out, 4) || (cinv && !aligned(cinv, 16)))
        return KQ_ERR_ALIGN;
    const uint64_t n = uint64_t(n1) * n2;
    const Range in[4] = {range_of(x, uint64_t(T) * n * 2), range_of(P1, uint64_t(n1) * n1 * 2),
                         range_of(P2, uint64_t(n2) * n2 * 2), range_of(cinv, cinv ? n * 4 : 0)};
    const Range rq = range_of(q_out, uint64_t(T) * n / 2), rs = range_of(scale_out, uint64_t(T) * 4);
    for (const Range &r : in)
        if (overlap(r, rq) || overlap(r, rs)) return KQ_ERR_ARG;
    if (overlap(rq, rs)) return KQ_ERR_ARG;
    return run_transform(x, P1, P2, cinv, alpha, q_out, scale_out, nullptr, T, n1, n2, stream);
}

kq_status kq_transform(const uint16_t *x, const uint16_t *P1, const uint16_t *P2, const float *cinv,
                       float *y_out, int64_t T, int n1, int n2, kq_stream_t stream) {
    kq_status st = check_shape(T, n1, n2);
    if (st != KQ_OK) return st;
    if (T == 0) return KQ_OK;
    if (!x || !P1 || !P2 || !y_out) return KQ_ERR_NULL;
    if (!aligned(x, 16) || !aligned(P1, 16) || !aligned(P2, 16) || !aligned(y_out, 16) ||
        (cinv && !aligned(cinv, 16)))
        return KQ_ERR_ALIGN;
    const uint64_t n = uint64_t(n1) * n2;
    const Range in[4] = {range_of(x, uint64_t(T) * n * 2), range_of(P1, uint64_t(n1) * n1 * 2),
                         range_of(P2, uint64_t(n2) * n2 * 2), range_of(cinv, cinv ? n * 4 : 0)};
    const Range ry = range_of(y_out, uint64_t(T) * n * 4);
    for (const Range &r : in)
        if (overlap(r, ry)) return KQ_ERR_ARG;
    return run_transform(x, P1, P2, cinv, 1.0f, nullptr, nullptr, y_out, T, n1, n2, stream);
}

kq_status kq_dequant_inverse(const uint8_t *q, const float *scale, const float *P1inv,
                             const float *P2inv, const float *c, float *x_hat, int64_t T, int n1,
                             int n2, kq_stream_t stream) {
    kq_status st = check_shape(T, n1, n2);
    if (st != KQ_OK) return st;
    if (T == 0) return KQ_OK;
    if (!q || !scale || !P1inv || !P2inv || !x_hat) return KQ_ERR_NULL;
    if (!aligned(q, 16) || !aligned(scale, 4) || !aligned(P1inv, 4) || !aligned(P2inv, 4) ||
        !aligned(x_hat, 16) || (c && !aligned(c, 4)))
        return KQ_ERR_ALIGN;
    const uint64_t n = uint64_t(n1) * n2;
    const Range in[5] = {range_of(q, uint64_t(T) * n / 2), range_of(scale, uint64_t(T) * 4),
                         range_of(P1inv, uint64_t(n1) * n1 * 4), range_of(P2inv, uint64_t(n2) * n2 * 4),
                         range_of(c, c ? n * 4 : 0)};
    const Range rx = range_of(x_hat, uint64_t(T) * n * 4);
    for (const Range &r : in)
        if (overlap(r, rx)) return KQ_ERR_ARG;
    cudaError_t err = kq::launch_dequant_inverse(q, scale, P1inv, P2inv, c, x_hat, T, n1, n2,
                                                 reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KQ_OK : KQ_ERR_CUDA;
}

namespace {
// The checks and the launch of both W4A4 entries; `ob` = output bytes per element.
kq_status w4a4_gemm(const uint8_t *qx, const float *sx, const uint8_t *qw, const float *sw, void *y, int ob,
                    int64_t M, int64_t N, int64_t K, kq_stream_t stream) {
    if (M < 0 || N < 0 || K < 128 || K > 262144 || K % 128 != 0) return KQ_ERR_SHAPE;
    if (M > int64_t(65535) * 128) return KQ_ERR_SHAPE;  // grid rows
    if (M == 0 || N == 0) return KQ_OK;
    if (M > INT64_MAX / N / 4) return KQ_ERR_SHAPE;
    if (!qx || !sx || !qw || !sw || !y) return KQ_ERR_NULL;
    if (!aligned(qx, 16) || !aligned(qw, 16) || !aligned(sx, 4) || !aligned(sw, 4) || !aligned(y, uintptr_t(ob)))
        return KQ_ERR_ALIGN;
    const Range in[4] = {range_of(qx, uint64_t(M) * uint64_t(K) / 2), range_of(sx, uint64_t(M) * 4),
                         range_of(qw, uint64_t(N) * uint64_t(K) / 2), range_of(sw, uint64_t(N) * 4)};
    const Range ry = range_of(y, uint64_t(M) * uint64_t(N) * uint64_t(ob));
    for (const Range &r : in)
        if (overlap(r, ry)) return KQ_ERR_ARG;
    DeviceInfo info;
    kq_status st = device_info(info);
    if (st != KQ_OK) return st;
    cudaError_t err = kq::launch_w4a4_gemm(qx, sx, qw, sw, y, ob == 2, M, N, K, info.device,
                                           reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KQ_OK : KQ_ERR_CUDA;
}
}  // namespace

kq_status kq_w4a4_gemm(const uint8_t *qx, const float *sx, const uint8_t *qw, const float *sw, float *y,
                       int64_t M, int64_t N, int64_t K, kq_stream_t stream) {
    return w4a4_gemm(qx, sx, qw, sw, y, 4, M, N, K, stream);
}

kq_status kq_w4a4_gemm_bf16(const uint8_t *qx, const float *sx, const uint8_t *qw, const float *sw, uint16_t *y,
                            int64_t M, int64_t N, int64_t K, kq_stream_t stream) {
    return w4a4_gemm(qx, sx, qw, sw, y, 2, M, N, K, stream);
}

kq_status kq_headwise_transform_quant(const uint16_t *x, const uint16_t *Ph, float alpha, uint8_t *q_out,
                                      float *scale_out, int64_t T, int heads, int head_dim, kq_stream_t stream) {
    if (T < 0 || heads <= 0 || head_dim <= 0) return KQ_ERR_SHAPE;
    if (head_dim != 64 && head_dim != 128) return KQ_ERR_UNSUPPORTED;
    if (T > (int64_t(1) << 31) / heads) return KQ_ERR_SHAPE;  // rows are TMA coordinates
    kq_status st = check_alpha(alpha);
    if (st != KQ_OK) return st;
    if (!(alpha >= 0x1p-19f)) return KQ_ERR_UNSUPPORTED;  // the code rounding's range
    if (T == 0) return KQ_OK;
    if (!x || !Ph || !q_out || !scale_out) return KQ_ERR_NULL;
    if (!aligned(x, 16) || !aligned(Ph, 16) || !aligned(q_out, 16) || !aligned(scale_out, 4)) return KQ_ERR_ALIGN;
    const int64_t R = T * heads;
    const Range in[2] = {range_of(x, uint64_t(R) * head_dim * 2), range_of(Ph, uint64_t(head_dim) * head_dim * 2)};
    const Range out[2] = {range_of(q_out, uint64_t(R) * head_dim / 2), range_of(scale_out, uint64_t(R) * 4)};
    for (const Range &o : out)
        for (const Range &i : in)
            if (overlap(o, i)) return KQ_ERR_ARG;
    if (overlap(out[0], out[1])) return KQ_ERR_ARG;
    DeviceInfo info;
    if ((st = device_info(info)) != KQ_OK) return st;
    cudaError_t err = kq::launch_rowwise(x, Ph, alpha, q_out, scale_out, R, head_dim, info.num_sms, info.device,
                                         reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KQ_OK : KQ_ERR_CUDA;
}

kq_status kq_headwise_transform_quant_nvfp4(const uint16_t *x, const uint16_t *Ph, uint8_t *q_out,
                                            uint8_t *block_scale_out, float *scale_out, int64_t T, int heads,
                                            int head_dim, kq_stream_t stream) {
    if (T < 0 || heads <= 0 || head_dim <= 0) return KQ_ERR_SHAPE;
    if (head_dim != 64 && head_dim != 128) return KQ_ERR_UNSUPPORTED;
    if (T > (int64_t(1) << 31) / heads) return KQ_ERR_SHAPE;  // rows are TMA coordinates
    if (T == 0) return KQ_OK;
    if (!x || !Ph || !q_out || !block_scale_out || !scale_out) return KQ_ERR_NULL;
    if (!aligned(x, 16) || !aligned(Ph, 16) || !aligned(q_out, 16) || !aligned(block_scale_out, 8) ||
        !aligned(scale_out, 4))
        return KQ_ERR_ALIGN;
    const int64_t R = T * heads;
    const Range in[2] = {range_of(x, uint64_t(R) * head_dim * 2), range_of(Ph, uint64_t(head_dim) * head_dim * 2)};
    const Range out[3] = {range_of(q_out, uint64_t(R) * head_dim / 2), range_of(block_scale_out, uint64_t(R) * head_dim / 16),
                          range_of(scale_out, uint64_t(R) * 4)};
    for (const Range &o : out)
        for (const Range &i : in)
            if (overlap(o, i)) return KQ_ERR_ARG;
    if (overlap(out[0], out[1]) || overlap(out[0], out[2]) || overlap(out[1], out[2])) return KQ_ERR_ARG;
    DeviceInfo info;
    kq_status st = device_info(info);
    if (st != KQ_OK) return st;
    cudaError_t err = kq::launch_rowwise_nvfp4(x, Ph, q_out, block_scale_out, scale_out, R, head_dim, info.num_sms,
                                               info.device, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KQ_OK : KQ_ERR_CUDA;
}

kq_status kq_transform_quant_two_stage(const uint16_t *x, const uint16_t *P1, const uint16_t *P2,
                                       const float *cinv, float alpha, uint8_t *q_out, float *scale_out,
                                       void *workspace, uint64_t workspace_bytes, int64_t T, int n1, int n2,
                                       kq_stream_t stream) {
    if (T < 0 || n1 <= 0 || n2 <= 0) return KQ_ERR_SHAPE;
    if (!kq::two_stage_supports(n1, n2)) return KQ_ERR_UNSUPPORTED;
    const int64_t n = int64_t(n1) * n2;
    if (T >= (int64_t(1) << 31) / n) return KQ_ERR_SHAPE;  // rows and offsets are 32-bit
    kq_status st = check_alpha(alpha);
    if (st != KQ_OK) return st;
    if (!(alpha >= 0x1p-19f)) return KQ_ERR_UNSUPPORTED;  // the code rounding's range
    if (T == 0) return KQ_OK;
    if (!x || !P1 || !P2 || !q_out || !scale_out || !workspace) return KQ_ERR_NULL;
    if (!aligned(x, 16) || !aligned(P1, 16) || !aligned(P2, 16) || !aligned(q_out, 16) ||
        !aligned(workspace, 16) || !aligned(scale_out, 4) || (cinv && !aligned(cinv, 16)))
        return KQ_ERR_ALIGN;
    const uint64_t need = kq::two_stage_workspace_bytes(T, n1, n2);
    if (workspace_bytes < need) return KQ_ERR_ARG;
    const Range in[4] = {range_of(x, uint64_t(T) * n * 2), range_of(P1, uint64_t(n1) * n1 * 2),
                         range_of(P2, uint64_t(n2) * n2 * 2), range_of(cinv, cinv ? uint64_t(n) * 4 : 0)};
    const Range out[3] = {range_of(q_out, uint64_t(T) * n / 2), range_of(scale_out, uint64_t(T) * 4),
                          range_of(workspace, need)};
    for (const Range &o : out)
        for (const Range &i : in)
            if (overlap(o, i)) return KQ_ERR_ARG;
    if (overlap(out[0], out[1]) || overlap(out[0], out[2]) || overlap(out[1], out[2])) return KQ_ERR_ARG;
    DeviceInfo info;
    if ((st = device_info(info)) != KQ_OK) return st;
    kq::LaunchArgs a;
    a.x = x;
    a.P1 = P1;
    a.P2 = P2;
    a.cinv = cinv;
    a.alpha = alpha;
    a.q_out = q_out;
    a.scale_out = scale_out;
    a.y_out = nullptr;
    a.T = T;
    a.n1 = n1;
    a.n2 = n2;
    a.num_sms = info.num_sms;
    a.device = info.device;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    return kq::launch_two_stage(a, workspace) == cudaSuccess ? KQ_OK : KQ_ERR_CUDA;
}

uint64_t kq_two_stage_workspace_bytes(int64_t T, int n1, int n2) {
    if (T <= 0 || n1 <= 0 || n2 <= 0) return 0;
    return kq::two_stage_workspace_bytes(T, n1, n2);
}

kq_status kq_transform_quant_two_stage_static(const uint16_t *x, const uint16_t *P1, const uint16_t *P2,
                                              const float *cinv, float alpha, uint8_t *q_out, float *scale_out,
                                              int64_t T, int n1, int n2, kq_stream_t stream) {
    static_assert(KQ_STATIC_WORKSPACE_BYTES == kq::kStaticScratchBytes, "static workspace size");
    if (T < 0 || n1 <= 0 || n2 <= 0) return KQ_ERR_SHAPE;
    if (!kq::two_stage_supports(n1, n2)) return KQ_ERR_UNSUPPORTED;
    if (T > int64_t(kq::kStaticScratchBytes / kq::two_stage_workspace_bytes(1, n1, n2))) return KQ_ERR_ARG;
    void *scratch = nullptr;
    if (T > 0) {
        DeviceInfo info;
        kq_status st = device_info(info);
        if (st != KQ_OK) return st;
        if (kq::static_scratch(info.device, &scratch) != cudaSuccess) return KQ_ERR_CUDA;
    }
    return kq_transform_quant_two_stage(x, P1, P2, cinv, alpha, q_out, scale_out, scratch, kq::kStaticScratchBytes, T,
                                        n1, n2, stream);
}

kq_status kq_device_error(kq_stream_t stream, int *code) {
    if (!code) return KQ_ERR_NULL;
    unsigned int v = 0;
    if (kq::read_and_clear_device_error(reinterpret_cast<cudaStream_t>(stream), &v) != cudaSuccess)
        return KQ_ERR_CUDA;
    *code = static_cast<int>(v);
    return KQ_OK;
}

kq_status kq_selftest_bounded_wait(int64_t limit_us, kq_stream_t stream) {
    if (limit_us < 1 || limit_us > 10000000) return KQ_ERR_ARG;
    cudaError_t err = kq::launch_selftest_wait(uint64_t(limit_us) * 1000u,
                                               reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KQ_OK : KQ_ERR_CUDA;
}

const char *kq_status_string(int status) {
    switch (status) {
    case KQ_OK: return "ok";
    case KQ_ERR_NULL: return "a required pointer is NULL";
    case KQ_ERR_SHAPE: return "bad shape (T < 0, n1 <= 0, n2 <= 0 or size overflow)";
    case KQ_ERR_UNSUPPORTED:
        return "unsupported size or parameter for this entry (factors: multiples of 16 up to 128, or up to 256 for "
               "the two-stage entries; head_dim 64 or 128; alpha of at least 2^-19 where the entry requires it)";
    case KQ_ERR_ALIGN: return "misaligned pointer";
    case KQ_ERR_ARG: return "bad argument (alpha outside (0, 1] or outputs overlap inputs)";
    case KQ_ERR_CUDA: return "CUDA runtime error";
    case KQ_ERR_TIMEOUT: return "a bounded wait inside a kernel timed out";
    default: return "unknown status";
    }
}

const char *kq_kernel_name(int n1, int n2, int has_cinv) {
    if (!supported_factor(n1) || !supported_factor(n2)) return "unsupported";
    return kq::tc05_supports(n1, n2, has_cinv != 0) ? "kq_tc05_fused_kernel" : "kq_warp_mma_kernel";
}

const char *kq_kernel_for(int64_t T, int n1, int n2, int has_cinv, float alpha) {
    if (T < 0 || !supported_factor(n1) || !supported_factor(n2)) return "unsupported";
    int sms = 148;
    DeviceInfo info;
    if (device_info(info) == KQ_OK) sms = info.num_sms;
    return kernel_name_of(choose_kernel(T, n1, n2, has_cinv != 0, alpha, true, sms));
}

int kq_version(void) { return kVersion; }

}  // extern "C"
