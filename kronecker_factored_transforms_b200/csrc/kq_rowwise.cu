// kq_rowwise.cu -- the per-head transform of the key / value cache with INT4
// per (token, head) row (FlatQuant page: P_h and P_v keep their full per-head
// shape because head dims are small; keys and values are transformed per head
// and quantised before they are stored):
//
//     y[r] = x[r] Ph,  s[r] = alpha max|y[r]| / 7,
//     q[r] = clamp(round_half_even(y[r] / s[r]), -8, 7)
//
// for every row r = (token, head) of head_dim (D = 64 or 128) values, with one
// bf16 factor Ph shared by all rows.
//
// The rows are independent, so the product is a plain [R x D] x [D x D] GEMM:
// tiles of 128 rows by TMA are the A operand (M = 128, one row per TMEM lane),
// Ph^T resident in shared memory the B operand (N = D), one tcgen05 kind::f16
// pass (x and Ph are exact in bf16), the fp32 row in TMEM.  An epilogue thread
// owns one row: its absmax, its scale and its codes stay in the thread; the
// codes leave as 16-byte stores, the scale as one coalesced 4-byte store.
//
// Warps: 0 TMA producer | 1 TMEM allocator + MMA issuer | 4-19 four epilogue
// warpgroups, tile k to warpgroup and TMEM buffer k % 4 | 2-3 idle (all warps
// build Ph^T at start).  Every mbarrier wait is bounded (kq_wait.cuh).
#include <mutex>

#include "kq_common.cuh"
#include "kq_internal.h"
#include "kq_tc05_ptx.cuh"
#include "kq_wait.cuh"

namespace kq {
namespace {

using namespace tc;

constexpr int R_THREADS = 640;
constexpr int R_EPI = 4;  // epilogue warpgroups, one per TMEM accumulator buffer
constexpr int RT = 128;  // rows per tile: MMA M, one per TMEM lane
enum : unsigned { kSiteRow = 128u };

template <int D>
struct RCfg {
    static constexpr int KC = D / 64;                // 64-element K chunks
    static constexpr int CHUNK = RT * 128;           // one [128 rows][64] bf16 chunk: 16 KB
    static constexpr int XTILE = KC * CHUNK;         // a tile's x
    static constexpr int B_BYTES = KC * D * 128;     // Ph^T: [D rows][64] chunks
    static constexpr int NB = R_EPI;                 // TMEM accumulator buffers (NB * D <= 512)
    static constexpr int SX = D == 128 ? 5 : 8;      // x stages
    static constexpr int OFF_B = 0;
    static constexpr int OFF_X = B_BYTES;            // 1024-aligned
    static constexpr int FULL = 0, EMPTY = SX, DFULL = 2 * SX, DEMPTY = 2 * SX + NB, DONE = 2 * SX + 2 * NB;
    static constexpr int NBAR = DONE + 1;
    static constexpr int OFF_BAR = OFF_X + SX * XTILE;
    static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;  // TMEM base, abort flag, the constant 1
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static_assert(NB * D <= 512, "TMEM budget");
    static_assert(OFF_X % 1024 == 0 && CHUNK % 1024 == 0, "swizzle alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

// round_half_even(y * inv) as an int for |y * inv| < 2^22 (alpha >= 2^-19):
// after adding 1.5 * 2^23 the rounded integer sits in the low mantissa bits.
__device__ __forceinline__ int round_code_r(uint32_t ybits, float inv, int one) {
    const uint32_t b = __float_as_uint(fmaf(__uint_as_float(ybits), inv, 12582912.0f));
    int k;
    asm("mad.lo.s32 %0, %1, %2, %3;" : "=r"(k) : "r"(b), "r"(one), "r"(-0x4B400000));
    return k;
}

// Eight codes (value e in nibble e) from eight fp32 values.
__device__ __forceinline__ uint32_t codes8(const uint32_t *v, float inv, int one) {
    uint32_t w = pack_s4x2(round_code_r(v[7], inv, one), round_code_r(v[6], inv, one), 0u);
    w = pack_s4x2(round_code_r(v[5], inv, one), round_code_r(v[4], inv, one), w);
    w = pack_s4x2(round_code_r(v[3], inv, one), round_code_r(v[2], inv, one), w);
    return pack_s4x2(round_code_r(v[1], inv, one), round_code_r(v[0], inv, one), w);
}

// ---- NVFP4: E2M1 elements, an E4M3 scale per 16 values, an fp32 scale per row --
// Two fp32 values -> E4M3 codes (round to nearest even, saturating at 448): b in
// the low byte, a in the high byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(a), "f"(b));
    return d;
}
// The two E4M3 codes of e4m3x2 back to fp32 (exact).
__device__ __forceinline__ void e4m3x2_decode(uint32_t c, float &lo, float &hi) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(uint16_t(c)));
    lo = __half2float(__ushort_as_half(uint16_t(h2)));
    hi = __half2float(__ushort_as_half(uint16_t(h2 >> 16)));
}
// Two fp32 values -> one byte of E2M1 codes (round to nearest even, saturating
// at 6): b in the low nibble, a in the high nibble.
__device__ __forceinline__ uint32_t e2m1x2(float a, float b) {
    uint32_t d;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(d)
        : "f"(a), "f"(b));
    return d;
}
// Eight values times k -> a 32-bit word of E2M1 codes, value e in nibble e; a
// value that rounds to zero is stored as +0 (the conversion keeps the sign).
__device__ __forceinline__ uint32_t fp4x8(const uint32_t *v, float k) {
    uint32_t w = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p)
        w |= e2m1x2(__uint_as_float(v[2 * p + 1]) * k, __uint_as_float(v[2 * p]) * k) << (8 * p);
    const uint32_t nz = (w | (w >> 1) | (w >> 2)) & 0x11111111u;  // nibbles with a nonzero magnitude
    return w & (0x77777777u | (nz << 3));
}

template <int D, bool FP4>
__global__ void __launch_bounds__(R_THREADS, 1)
    kq_rowwise_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint16_t *__restrict__ Ph, float alpha,
                      uint8_t *__restrict__ q_out, float *__restrict__ scale_out, uint8_t *__restrict__ bscale_out,
                      int64_t R, unsigned int *err) {
    using C = RCfg<D>;
    extern __shared__ __align__(1024) unsigned char r_raw[];
    const uint32_t raw_addr = smem_u32(r_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    unsigned char *smem = r_raw + (sbase - raw_addr);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ntiles = (R + RT - 1) / RT;
    auto bar = [&](int i) -> uint32_t { return sbase + uint32_t(C::OFF_BAR + 8 * i); };
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    if (tid == 0) {
        for (int s = 0; s < C::SX; ++s) {
            mbar_init(bar(C::FULL + s), 1);
            mbar_init(bar(C::EMPTY + s), 1);
        }
        for (int b = 0; b < C::NB; ++b) {
            mbar_init(bar(C::DFULL + b), 1);
            mbar_init(bar(C::DEMPTY + b), 4);  // the four warps of the epilogue warpgroup
        }
        mbar_init(bar(C::DONE), 1);
        *s_abort = 0;
        *reinterpret_cast<int *>(smem + C::OFF_MISC + 8) = 1;  // `one` of the code rounding
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_x);
    if (warp == 1) {
        tmem_alloc(sbase + C::OFF_MISC, 512);
        tmem_relinquish();
    }
    // on-chip state only above; global reads and writes after the previous kernel
    griddep_wait();
    // B = Ph^T in 128B-swizzled K-major chunks: row o (output column), K = k.
    // A unit is one row o and eight consecutive k: eight loads (consecutive
    // threads take consecutive o, so each load is coalesced), one 16-byte store
    // (the swizzle spreads consecutive rows over all banks).
    {
        constexpr int UNITS = D * D / 8, PER = (UNITS + R_THREADS - 1) / R_THREADS;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int u = tid + i * R_THREADS;
            if (u < UNITS) {
                const int o = u % D, k0 = 8 * (u / D);
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w[e] = uint32_t(Ph[(k0 + 2 * e) * D + o]) | (uint32_t(Ph[(k0 + 2 * e + 1) * D + o]) << 16);
                *reinterpret_cast<uint4 *>(smem + C::OFF_B + (k0 >> 6) * D * 128 + o * 128 +
                                           ((((k0 & 63) >> 3) ^ (o & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    // The next launch may be scheduled once every CTA holds its SM and its TMEM;
    // it touches global memory only after this grid completes.
    griddep_launch_dependents();

    if (warp == 0) {
        // ---------------- TMA producer: x tiles [128 rows] x [D] ----------------
        Ring r;
        int issued = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, r.next(C::SX)) {
            const bool ok = __all_sync(0xffffffffu, wait_bounded_err(bar(C::EMPTY + r.idx), r.phase ^ 1u, s_abort,
                                                                     kSiteRow, kWaitLimitNs, false, err));
            if (!ok) break;
            if (elect_one()) {
                const uint32_t dst = sbase + uint32_t(C::OFF_X + r.idx * C::XTILE);
                mbar_arrive_expect_tx(bar(C::FULL + r.idx), C::XTILE);
#pragma unroll
                for (int kc = 0; kc < C::KC; ++kc)
                    tma_load_2d(dst + uint32_t(kc * C::CHUNK), &tmap_x, 64 * kc, int(tile * RT), bar(C::FULL + r.idx));
            }
            __syncwarp();
            ++issued;
        }
        Ring rd;
        for (int i = 0; i < issued; ++i, rd.next(C::SX))
            if (i + C::SX >= issued)
                wait_bounded_err(bar(C::FULL + rd.idx), rd.phase, s_abort, kSiteRow, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer: D[row][o] = sum_k x[row][k] Ph[k][o] ----------------
        constexpr uint32_t idesc = idesc_bf16_f32(RT, D);
        const uint32_t bdesc = sdesc_sw128_lo(sbase + uint32_t(C::OFF_B));
        Ring rs, rd;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, rs.next(C::SX), rd.next(C::NB)) {
            bool ok = wait_bounded_err(bar(C::DEMPTY + rd.idx), rd.phase ^ 1u, s_abort, kSiteRow, kWaitLimitNs, false,
                                       err);
            ok = ok && wait_bounded_err(bar(C::FULL + rs.idx), rs.phase, s_abort, kSiteRow, kWaitLimitNs, false, err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t d = tmem + uint32_t(rd.idx * D);
            const uint32_t adesc = sdesc_sw128_lo(sbase + uint32_t(C::OFF_X + rs.idx * C::XTILE));
            if (elect_one()) {
#pragma unroll
                for (int kc = 0; kc < C::KC; ++kc)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t a =
                            (uint64_t(kSdescSw128Hi) << 32) | (adesc + uint32_t((kc * C::CHUNK) >> 4) + 2 * kk);
                        const uint32_t b = bdesc + uint32_t((kc * D * 128) >> 4) + 2 * kk;
                        if ((kc | kk) != 0)
                            mma_ss_split<1>(d, a, b, kSdescSw128Hi, idesc);
                        else
                            mma_ss_split<0>(d, a, b, kSdescSw128Hi, idesc);
                    }
                tc_commit(bar(C::EMPTY + rs.idx));  // x stage free once read
                tc_commit(bar(C::DFULL + rd.idx));  // accumulator ready
            }
            __syncwarp();
        }
        if (elect_one()) tc_commit(bar(C::DONE));
        __syncwarp();
        wait_bounded_err(bar(C::DONE), 0u, s_abort, kSiteRow, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------- epilogue: one row per thread ----------------
        const int ew = (warp - 4) >> 2, q = warp & 3;
        const int one = *reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);
        int64_t k = 0;  // the CTA's tile counter: tile k lives in buffer k % NB, warpgroup k % NB
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++k) {
            if (int(k % R_EPI) != ew) continue;
            const int b = int(k % C::NB);
            const uint32_t ph = uint32_t((k / C::NB) & 1);
            const bool ok = wait_bounded_err(bar(C::DFULL + b), ph, s_abort, kSiteRow, kWaitLimitNs, false, err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t base = tmem + (uint32_t(32 * q) << 16) + uint32_t(b * D);
            const int64_t row = tile * RT + 32 * q + lane;
            // pass 1: the row's absmax
            float m = 0.0f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(base + uint32_t(32 * c), v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    m = fmax3(m, fabsf(__uint_as_float(v[e])), fabsf(__uint_as_float(v[e + 1])));
            }
            // INT4: s = alpha max / 7.  NVFP4: the row scale s = max / (6 * 448).
            const float sc = FP4 ? __fdiv_rn(m, 2688.0f) : alpha * m * (1.0f / 7.0f);
            const float inv = sc > 0.0f ? fminf(__fdividef(1.0f, sc), 3.0e38f) : 0.0f;
            // pass 2: codes, 16 bytes per 32 values (NVFP4: and one E4M3 scale per 16)
            uint8_t *qrow = q_out + row * (D / 2);
            uint32_t bsc[D / 64 > 0 ? D / 64 : 1];  // the row's block-scale codes, four per word
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(base + uint32_t(32 * c), v);
                tmem_wait_ld();
                if (c == D / 32 - 1) {  // this warp's last read of the buffer
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(C::DEMPTY + b));
                }
                uint4 w;
                if constexpr (FP4) {
                    // blocks 2c and 2c + 1: absmax, E4M3 scale code, element codes
                    float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
                    for (int e = 0; e < 16; e += 2) {
                        a0 = fmax3(a0, fabsf(__uint_as_float(v[e])), fabsf(__uint_as_float(v[e + 1])));
                        a1 = fmax3(a1, fabsf(__uint_as_float(v[16 + e])), fabsf(__uint_as_float(v[17 + e])));
                    }
                    const uint32_t bc = e4m3x2(a1 * inv * (1.0f / 6.0f), a0 * inv * (1.0f / 6.0f));
                    float d0, d1;
                    e4m3x2_decode(bc, d0, d1);
                    const float den0 = d0 * sc, den1 = d1 * sc;
                    const float k0 = den0 > 0.0f ? __fdividef(1.0f, den0) : 0.0f;
                    const float k1 = den1 > 0.0f ? __fdividef(1.0f, den1) : 0.0f;
                    w = make_uint4(fp4x8(v, k0), fp4x8(v + 8, k0), fp4x8(v + 16, k1), fp4x8(v + 24, k1));
                    if (c & 1)
                        bsc[c >> 1] |= bc << 16;
                    else
                        bsc[c >> 1] = bc;
                } else {
                    w = make_uint4(codes8(v, inv, one), codes8(v + 8, inv, one), codes8(v + 16, inv, one),
                                   codes8(v + 24, inv, one));
                }
                if (row < R) *reinterpret_cast<uint4 *>(qrow + 16 * c) = w;
            }
            if (row < R) {
                scale_out[row] = sc;
                if constexpr (FP4) {
                    if (D == 128)
                        *reinterpret_cast<uint2 *>(bscale_out + row * (D / 16)) = make_uint2(bsc[0], bsc[1]);
                    else
                        *reinterpret_cast<uint32_t *>(bscale_out + row * (D / 16)) = bsc[0];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, bool FP4>
cudaError_t launch_rowwise_inst(const uint16_t *x, const uint16_t *Ph, float alpha, uint8_t *q_out, float *scale_out,
                                uint8_t *bscale_out, int64_t R, int num_sms, int device, cudaStream_t stream) {
    using C = RCfg<D>;
    auto kern = kq_rowwise_kernel<D, FP4>;
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[device], [&] {
        attr_err[device] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    });
    if (attr_err[device] != cudaSuccess) return attr_err[device];
    unsigned int *err = nullptr;
    cudaError_t e = device_error_word(device, &err);
    if (e != cudaSuccess) return e;
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap tx;
    const cuuint64_t dx[2] = {cuuint64_t(D), cuuint64_t(R)};
    const cuuint64_t sx[1] = {cuuint64_t(D) * 2};
    const cuuint32_t bx[2] = {64u, cuuint32_t(RT)};
    const cuuint32_t estr[2] = {1u, 1u};
    CUresult r = encode(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(x), dx, sx, bx, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const int64_t ntiles = (R + RT - 1) / RT;
    const int64_t grid = ntiles < num_sms ? ntiles : num_sms;
    return launch_overlapped(kern, unsigned(grid), R_THREADS, C::SMEM, stream, tx, Ph, alpha, q_out, scale_out,
                             bscale_out, R, err);
}

}  // namespace

cudaError_t launch_rowwise(const uint16_t *x, const uint16_t *Ph, float alpha, uint8_t *q_out, float *scale_out,
                           int64_t R, int head_dim, int num_sms, int device, cudaStream_t stream) {
    if (R >= (int64_t(1) << 31)) return cudaErrorInvalidValue;  // TMA row coordinate range
    if (head_dim == 128)
        return launch_rowwise_inst<128, false>(x, Ph, alpha, q_out, scale_out, nullptr, R, num_sms, device, stream);
    if (head_dim == 64)
        return launch_rowwise_inst<64, false>(x, Ph, alpha, q_out, scale_out, nullptr, R, num_sms, device, stream);
    return cudaErrorNotSupported;
}

cudaError_t launch_rowwise_nvfp4(const uint16_t *x, const uint16_t *Ph, uint8_t *q_out, uint8_t *bscale_out,
                                 float *scale_out, int64_t R, int head_dim, int num_sms, int device,
                                 cudaStream_t stream) {
    if (R >= (int64_t(1) << 31)) return cudaErrorInvalidValue;  // TMA row coordinate range
    if (head_dim == 128)
        return launch_rowwise_inst<128, true>(x, Ph, 1.0f, q_out, scale_out, bscale_out, R, num_sms, device, stream);
    if (head_dim == 64)
        return launch_rowwise_inst<64, true>(x, Ph, 1.0f, q_out, scale_out, bscale_out, R, num_sms, device, stream);
    return cudaErrorNotSupported;
}

}  // namespace kq
