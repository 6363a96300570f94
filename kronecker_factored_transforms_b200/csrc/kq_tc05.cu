// kq_tc05.cu -- persistent fused Kronecker transform + INT4 kernel on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM), plus the
// device status word that its bounded waits report through.
//
// Method (FlatQuant page, "Kronecker factorization" and "The fused kernel"):
// per token Y~ = P1^T X~ P2 with X~ the row-major n1 x n2 view of x * cinv,
// then per-token absmax, s = alpha * max / 7, round-half-even codes clamped
// to [-8, 7], packed two per byte.  Only codes and scales reach HBM.
//
// Layout of the work (one CTA per SM, 16 warps, groups of H = 128 / n2
// tokens so that the 128 TMEM lanes always hold 128 output columns):
//   TMEM lane l = (h, m): token h of the group, output column j = pi(m) of
//   its n2 columns.  pi interleaves each block of 16 columns (lanes 0-7 take
//   the even columns, lanes 8-15 the odd ones) so that one thread of a
//   16x256b TMEM load holds both nibbles of an output byte.
//   stage 1 (SS MMA)  D1[l][a]  = sum_(h',b) A1[l][(h',b)] * X[a][(h',b)]
//                     A1 = block-diag over h of P2^T (rows permuted by pi),
//                     X  = the group's x tile straight from TMA (K = 128).
//   convert (TMEM)    D1 fp32 -> A2 = hi + lo bf16, in place, chunk by chunk.
//   stage 2 (TS MMA)  D2[l][i]  = sum_a A2[l][a] * P1[a][i]   (A from TMEM)
//   epilogue          absmax over the token's lanes, quantise, pack, bulk store.
// With cinv, warps 4-7 first turn each raw x tile into x' = x * cinv split
// into hi and lo bf16 tiles; stage 1 then accumulates both.
//
// Warp roles: 0 TMA producer | 1 TMEM allocator + MMA issuer | 4-7 x' split
// (cinv only) | 8-11 D1 -> A2 conversion | 12-15 epilogue.  Every mbarrier
// wait is bounded: after about a second it ORs a site bit into
// g_device_error, raises a CTA-wide abort flag and the roles drain and exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kq_common.cuh"
#include "kq_internal.h"
#include "kq_tc05_ptx.cuh"

namespace kq {

// Nonzero when a bounded wait gave up; each site ORs its own bit.
__device__ unsigned int g_device_error = 0;

cudaError_t read_and_clear_device_error(cudaStream_t stream, unsigned int *code) {
    static const unsigned int zero = 0;
    cudaError_t err = cudaMemcpyFromSymbolAsync(code, g_device_error, sizeof(unsigned int), 0,
                                                cudaMemcpyDeviceToHost, stream);
    if (err != cudaSuccess) return err;
    err = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(unsigned int), 0,
                                  cudaMemcpyHostToDevice, stream);
    if (err != cudaSuccess) return err;
    return cudaStreamSynchronize(stream);
}

namespace {

using namespace tc;

constexpr int kTcThreads = 512;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // about one second

enum : unsigned {
    kSiteProducer = 1u,
    kSiteXSplit = 2u,
    kSiteMma = 4u,
    kSiteConvert = 8u,
    kSiteEpilogue = 16u,
    kSiteDrain = 32u,
    kSiteSelfTest = 256u,
};

// Wait for the phase of parity `parity` of mbarrier `bar` to complete, for at
// most `limit_ns`.  Returns false (after flagging `site`) on timeout, or when
// another role already aborted (unless `ignore_abort`).
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort,
                                          unsigned site, uint64_t limit_ns, bool ignore_abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 0) {
            if (!ignore_abort && *abort) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                atomicOr(&g_device_error, site);
                *abort = 1;
                return false;
            }
        }
    }
}

__host__ __device__ constexpr int align_up(int v, int a) { return (v + a - 1) / a * a; }

template <int N1, int N2, bool SCALED>
struct Cfg {
    static constexpr int H = 128 / N2;               // tokens stacked in the TMEM lanes
    static constexpr int N = N1 * N2;
    static constexpr int SX = 4;                     // raw x tile stages
    static constexpr int SC = 2;                     // split x' tile stages (cinv)
    static constexpr int CHUNK = N1 * 128;           // one 64-element K chunk of an x tile
    static constexpr int XTILE = 2 * CHUNK;          // a group's x tile (K = 128)
    static constexpr int NCH2 = (N1 + 63) / 64;      // K chunks of P1^T
    static constexpr int N1P = align_up(N1, 32);     // TMEM columns per region
    static constexpr int TMEM_COLS = 4 * N1P <= 128 ? 128 : (4 * N1P <= 256 ? 256 : 512);
    static constexpr int OUT = H * N / 2;            // output bytes per group
    static constexpr int UNITS = N1 / 8;             // 16-byte units per x'-split thread
    static constexpr int OFF_A1 = 0;                 // 2 chunks x 128 rows x 128 B
    static constexpr int OFF_B2 = 32768;
    static constexpr int OFF_RAW = align_up(OFF_B2 + NCH2 * N1 * 128, 1024);
    static constexpr int OFF_CONV = OFF_RAW + SX * XTILE;
    static constexpr int OFF_OUT = OFF_CONV + (SCALED ? SC * 2 * XTILE : 0);
    static constexpr int NBAR = 2 * SX + 2 * SC + 10 + 1;
    static constexpr int OFF_BAR = align_up(OFF_OUT + 2 * OUT, 16);
    static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;  // tmem base, abort flag, 4 maxima
    static constexpr int SMEM = OFF_MISC + 32 + 1024;    // + slack for 1024-byte alignment
    // barrier indices
    static constexpr int FULL = 0, EMPTY = SX, CFULL = 2 * SX, CEMPTY = 2 * SX + SC;
    static constexpr int D1FULL = 2 * SX + 2 * SC, A2FULL = D1FULL + 2, D1EMPTY = D1FULL + 4;
    static constexpr int D2FULL = D1FULL + 6, D2EMPTY = D1FULL + 8, TEARDOWN = D1FULL + 10;
    static_assert(N2 == 64 || N2 == 128, "stage 1 needs K = H * n2 = 128");
    static_assert(N1 % 16 == 0 && N1 >= 16 && N1 <= 128, "n1 must be a multiple of 16 in [16, 128]");
    static_assert(!SCALED || N1 <= 64, "x' split keeps cinv in registers: n1 <= 64");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    __host__ __device__ static constexpr uint32_t R1(int b) { return uint32_t(b * N1P); }
    __host__ __device__ static constexpr uint32_t R2(int b) { return uint32_t(2 * N1P + b * N1P); }
};

// Byte offset of element (row r, k in [0, 64)) inside one 128B-swizzled chunk.
__device__ __forceinline__ uint32_t swz128(int r, int k) {
    return uint32_t(r * 128 + ((((k >> 3) ^ (r & 7)) << 4) | ((k & 7) << 1)));
}

// INT4 code of y * inv, round half to even, clamped to [-8, 7], as a nibble.
__device__ __forceinline__ uint32_t nibble(uint32_t ybits, float inv) {
    float p = __uint_as_float(ybits) * inv;
    p = fminf(fmaxf(p, -9.0f), 9.0f);
    // Adding 1.5 * 2^23 rounds p to an integer (nearest, ties to even) held in
    // the low mantissa bits.
    int q = __float_as_int(p + 12582912.0f) - 0x4B400000;
    q = min(max(q, -8), 7);
    return uint32_t(q) & 0xFu;
}

template <int N1, int N2, bool SCALED>
__global__ void __launch_bounds__(kTcThreads, 1)
    kq_tc05_fused_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint16_t *__restrict__ P1,
                         const uint16_t *__restrict__ P2, const float *__restrict__ cinv, float alpha,
                         uint8_t *__restrict__ q_out, float *__restrict__ scale_out, int64_t T) {
    using C = Cfg<N1, N2, SCALED>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - raw_addr);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t G = (T + C::H - 1) / C::H;
    const int64_t nk = G > int64_t(blockIdx.x) ? (G - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

    auto bar = [&](int i) -> uint32_t { return sbase + uint32_t(C::OFF_BAR + 8 * i); };
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    float *s_red = reinterpret_cast<float *>(smem + C::OFF_MISC + 16);

    if (tid == 0) {
        for (int s = 0; s < C::SX; ++s) {
            mbar_init(bar(C::FULL + s), 1);
            mbar_init(bar(C::EMPTY + s), SCALED ? 128 : 1);
        }
        for (int c = 0; c < C::SC; ++c) {
            mbar_init(bar(C::CFULL + c), 128);
            mbar_init(bar(C::CEMPTY + c), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(C::D1FULL + b), 1);
            mbar_init(bar(C::A2FULL + b), 128);
            mbar_init(bar(C::D1EMPTY + b), 1);
            mbar_init(bar(C::D2FULL + b), 1);
            mbar_init(bar(C::D2EMPTY + b), 128);
        }
        mbar_init(bar(C::TEARDOWN), 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_x);
    if (warp == 1) {
        tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
        tmem_relinquish();
    }

    // Resident operands, 128B-swizzled K-major.
    // A1[l][k], l = (h, m), k = (h', b): P2[b][pi(m)] when h == h', else 0.
    for (int e = tid; e < 128 * 128; e += kTcThreads) {
        const int l = e >> 7, k = e & 127;
        const int h = l / N2, m = l % N2, hk = k / N2, b = k % N2;
        const int j = (m & ~15) | ((m & 7) << 1) | ((m >> 3) & 1);
        const uint16_t v = (h == hk) ? P2[b * N2 + j] : uint16_t(0);
        *reinterpret_cast<uint16_t *>(smem + C::OFF_A1 + (k >> 6) * 16384 + swz128(l, k & 63)) = v;
    }
    // B2[i][a] = P1[a][i] (rows i, K = a), zero beyond a = n1.
    for (int e = tid; e < C::NCH2 * 64 * N1; e += kTcThreads) {
        const int i = e / (C::NCH2 * 64), ka = e % (C::NCH2 * 64);
        const uint16_t v = ka < N1 ? P1[ka * N1 + i] : uint16_t(0);
        *reinterpret_cast<uint16_t *>(smem + C::OFF_B2 + (ka >> 6) * (N1 * 128) + swz128(i, ka & 63)) = v;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int64_t issued = 0;
            for (int64_t k = 0; k < nk; ++k) {
                const int s = int(k % C::SX);
                if (!wait_bounded(bar(C::EMPTY + s), uint32_t((k / C::SX) & 1) ^ 1u, s_abort,
                                  kSiteProducer, kWaitLimitNs, false))
                    break;
                const int64_t g = blockIdx.x + k * gridDim.x;
                mbar_arrive_expect_tx(bar(C::FULL + s), C::XTILE);
                const uint32_t dst = sbase + C::OFF_RAW + s * C::XTILE;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int xc = (N2 == 128) ? 64 * c : 0;
                    const int64_t row = (N2 == 128) ? g * N1 : (2 * g + c) * N1;
                    tma_load_2d(dst + c * C::CHUNK, &tmap_x, xc, int(row), bar(C::FULL + s));
                }
                issued = k + 1;
            }
            // Drain: the last load issued into each slot has landed.
            for (int s = 0; s < C::SX; ++s) {
                if (issued > s) {
                    const int64_t last = s + ((issued - 1 - s) / C::SX) * C::SX;
                    wait_bounded(bar(C::FULL + s), uint32_t((last / C::SX) & 1), s_abort, kSiteDrain,
                                 kWaitLimitNs, true);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, N1);
            const uint32_t a1 = sbase + C::OFF_A1, b2 = sbase + C::OFF_B2;
            for (int64_t k = 0; k <= nk; ++k) {
                if (k < nk) {  // stage 1 of group k
                    const int b = int(k & 1);
                    if (!wait_bounded(bar(C::D1EMPTY + b), uint32_t((k >> 1) & 1) ^ 1u, s_abort, kSiteMma,
                                      kWaitLimitNs, false))
                        break;
                    uint32_t src0, src1, release;
                    if (SCALED) {
                        const int c2 = int(k % C::SC);
                        if (!wait_bounded(bar(C::CFULL + c2), uint32_t((k / C::SC) & 1), s_abort, kSiteMma,
                                          kWaitLimitNs, false))
                            break;
                        src0 = sbase + C::OFF_CONV + c2 * 2 * C::XTILE;
                        src1 = src0 + C::XTILE;
                        release = bar(C::CEMPTY + c2);
                    } else {
                        const int s = int(k % C::SX);
                        if (!wait_bounded(bar(C::FULL + s), uint32_t((k / C::SX) & 1), s_abort, kSiteMma,
                                          kWaitLimitNs, false))
                            break;
                        src0 = src1 = sbase + C::OFF_RAW + s * C::XTILE;
                        release = bar(C::EMPTY + s);
                    }
                    tc_fence_after();
                    const uint32_t d1 = tmem + C::R1(b);
#pragma unroll
                    for (int pass = 0; pass < (SCALED ? 2 : 1); ++pass) {
                        const uint32_t src = pass ? src1 : src0;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t off = uint32_t((kk & 3) * 32);
                            const uint64_t ad = sdesc_kmajor_sw128(a1 + (kk >> 2) * 16384 + off);
                            const uint64_t bd = sdesc_kmajor_sw128(src + (kk >> 2) * C::CHUNK + off);
                            mma_ss(d1, ad, bd, idesc, (pass | kk) != 0);
                        }
                    }
                    tc_commit(release);
                    tc_commit(bar(C::D1FULL + b));
                }
                if (k >= 1) {  // stage 2 of group k - 1
                    const int64_t kp = k - 1;
                    const int b = int(kp & 1);
                    const uint32_t ph = uint32_t((kp >> 1) & 1);
                    if (!wait_bounded(bar(C::A2FULL + b), ph, s_abort, kSiteMma, kWaitLimitNs, false)) break;
                    if (!wait_bounded(bar(C::D2EMPTY + b), ph ^ 1u, s_abort, kSiteMma, kWaitLimitNs, false))
                        break;
                    tc_fence_after();
                    const uint32_t d2 = tmem + C::R2(b), a2 = tmem + C::R1(b);
#pragma unroll
                    for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
                        for (int kk = 0; kk < N1 / 16; ++kk) {
                            const uint64_t bd =
                                sdesc_kmajor_sw128(b2 + (kk >> 2) * (N1 * 128) + (kk & 3) * 32);
                            mma_ts(d2, a2 + 16 * kk + 8 * pass, bd, idesc, (pass | kk) != 0);
                        }
                    }
                    tc_commit(bar(C::D2FULL + b));
                    tc_commit(bar(C::D1EMPTY + b));
                }
            }
            // Every MMA this thread issued has completed before TMEM is freed.
            tc_commit(bar(C::TEARDOWN));
            wait_bounded(bar(C::TEARDOWN), 0u, s_abort, kSiteDrain, kWaitLimitNs, true);
        }
    } else if (warp >= 4 && warp < 8) {
        // ---------------- x' = x * cinv -> hi / lo bf16 tiles ----------------
        if (SCALED) {
            const int t = tid - 128;
            float cv[C::UNITS][8];
#pragma unroll
            for (int u = 0; u < C::UNITS; ++u) {
                const int e = t + 128 * u;
                const int c = e / (8 * N1), rem = e % (8 * N1), r = rem >> 3, up = rem & 7;
                const int b0 = (N2 == 128 ? 64 * c : 0) + 8 * (up ^ (r & 7));
#pragma unroll
                for (int v = 0; v < 8; ++v) cv[u][v] = cinv[r * N2 + b0 + v];
            }
            for (int64_t k = 0; k < nk; ++k) {
                const int s = int(k % C::SX), c2 = int(k % C::SC);
                bool ok = wait_bounded(bar(C::FULL + s), uint32_t((k / C::SX) & 1), s_abort, kSiteXSplit,
                                       kWaitLimitNs, false);
                ok = ok && wait_bounded(bar(C::CEMPTY + c2), uint32_t((k / C::SC) & 1) ^ 1u, s_abort,
                                        kSiteXSplit, kWaitLimitNs, false);
                if (!__all_sync(0xffffffffu, ok)) break;  // the warp leaves together
                const unsigned char *raw = smem + C::OFF_RAW + s * C::XTILE;
                unsigned char *hi = smem + C::OFF_CONV + c2 * 2 * C::XTILE;
                unsigned char *lo = hi + C::XTILE;
#pragma unroll
                for (int u = 0; u < C::UNITS; ++u) {
                    const int e = t + 128 * u;
                    const uint4 in = *reinterpret_cast<const uint4 *>(raw + e * 16);
                    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
                    uint32_t oh[4], ol[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float v0 = __uint_as_float(w[p] << 16) * cv[u][2 * p];
                        const float v1 = __uint_as_float(w[p] & 0xFFFF0000u) * cv[u][2 * p + 1];
                        float h0, l0, h1, l1;
                        split_bf16(v0, h0, l0);
                        split_bf16(v1, h1, l1);
                        oh[p] = pack_bf16x2(h0, h1);
                        ol[p] = pack_bf16x2(l0, l1);
                    }
                    *reinterpret_cast<uint4 *>(hi + e * 16) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
                    *reinterpret_cast<uint4 *>(lo + e * 16) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
                }
                fence_proxy_async_smem();
                mbar_arrive(bar(C::EMPTY + s));
                mbar_arrive(bar(C::CFULL + c2));
            }
        }
    } else if (warp >= 8 && warp < 12) {
        // ---------------- D1 (fp32) -> A2 (hi, lo bf16) in TMEM ----------------
        const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
        for (int64_t k = 0; k < nk; ++k) {
            const int b = int(k & 1);
            const bool ok = wait_bounded(bar(C::D1FULL + b), uint32_t((k >> 1) & 1), s_abort, kSiteConvert,
                                         kWaitLimitNs, false);
            // reconverge before the warp-collective TMEM loads; leave together
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t col0 = tmem + lane_off + C::R1(b);
            constexpr int NK = N1 / 16;
            constexpr int BATCH = NK < 4 ? NK : 4;
#pragma unroll
            for (int k0 = 0; k0 < NK; k0 += BATCH) {
                uint32_t v[BATCH][16];
#pragma unroll
                for (int q = 0; q < BATCH; ++q)
                    if (k0 + q < NK) tmem_ld_32x32b_x16(col0 + 16 * (k0 + q), v[q]);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < BATCH; ++q) {
                    if (k0 + q < NK) {
                        uint32_t o[16];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            float h0, l0, h1, l1;
                            split_bf16(__uint_as_float(v[q][2 * e]), h0, l0);
                            split_bf16(__uint_as_float(v[q][2 * e + 1]), h1, l1);
                            o[e] = pack_bf16x2(h0, h1);
                            o[8 + e] = pack_bf16x2(l0, l1);
                        }
                        tmem_st_32x32b_x16(col0 + 16 * (k0 + q), o);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::A2FULL + b));
        }
    } else if (warp >= 12) {
        // ---------------- epilogue: absmax, quantise, pack, store ----------------
        const int q = warp & 3;
        const int et = tid - 384;
        const int tok_h = (32 * q) / N2;
        const int g8 = lane >> 2, qq = lane & 3;
        const uint32_t lane_off = uint32_t(32 * q) << 16;
        constexpr int NK = N1 / 16;
        for (int64_t k = 0; k < nk; ++k) {
            const int b = int(k & 1);
            const int64_t g = blockIdx.x + k * gridDim.x;
            const bool ok = wait_bounded(bar(C::D2FULL + b), uint32_t((k >> 1) & 1), s_abort,
                                         kSiteEpilogue, kWaitLimitNs, false);
            // All four warps leave together, so none is left behind in a named barrier.
            const bool warp_ok = __all_sync(0xffffffffu, ok);
            if (named_barrier_any(1, 128, !warp_ok)) break;
            __syncwarp();
            tc_fence_after();
            // pass 1: absmax over this warp's 32 lanes and all n1 columns
            float mx = 0.0f;
            constexpr int BATCH = NK < 4 ? NK : 4;
#pragma unroll
            for (int k0 = 0; k0 < NK; k0 += BATCH) {
                uint32_t v[BATCH][16];
#pragma unroll
                for (int r = 0; r < BATCH; ++r)
                    if (k0 + r < NK) tmem_ld_32x32b_x16(tmem + lane_off + C::R2(b) + 16 * (k0 + r), v[r]);
                tmem_wait_ld();
#pragma unroll
                for (int r = 0; r < BATCH; ++r)
                    if (k0 + r < NK)
#pragma unroll
                        for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(__uint_as_float(v[r][e])));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) s_red[q] = mx;
            if (et == 0) bulk_wait_read<1>();  // staging buffer (k & 1) is free again
            named_barrier_sync(1, 128);
            float m = 0.0f;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if ((32 * w) / N2 == tok_h) m = fmaxf(m, s_red[w]);
            const float s = alpha * m / 7.0f;
            const float inv = s > 0.0f ? 1.0f / s : 0.0f;
            // pass 2: codes, two nibbles per thread per byte (lane g8 even column, g8 + 8 odd)
            unsigned char *stg = smem + C::OFF_OUT + (k & 1) * C::OUT + tok_h * (C::N / 2);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int L0 = 32 * q + 16 * hf;
                const int col_byte = 8 * ((L0 % N2) / 16) + g8;
                const uint32_t taddr = tmem + (uint32_t(L0) << 16) + C::R2(b);
#pragma unroll
                for (int cc = 0; cc < NK; ++cc) {
                    uint32_t r[8];
                    tmem_ld_16x256b_x2(taddr + 16 * cc, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int rep = 0; rep < 2; ++rep) {
                        const int i0 = 16 * cc + 8 * rep + 2 * qq;
                        const uint32_t b0 = nibble(r[4 * rep + 0], inv) | (nibble(r[4 * rep + 2], inv) << 4);
                        const uint32_t b1 = nibble(r[4 * rep + 1], inv) | (nibble(r[4 * rep + 3], inv) << 4);
                        stg[i0 * (N2 / 2) + col_byte] = uint8_t(b0);
                        stg[(i0 + 1) * (N2 / 2) + col_byte] = uint8_t(b1);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(bar(C::D2EMPTY + b));
            fence_proxy_async_smem();
            named_barrier_sync(1, 128);
            const int64_t tok0 = C::H * g;
            if (et == 0) {
                const int64_t valid = (T - tok0) < C::H ? (T - tok0) : C::H;
                bulk_store(q_out + tok0 * (C::N / 2), sbase + C::OFF_OUT + (k & 1) * C::OUT,
                           uint32_t(valid * (C::N / 2)));
                bulk_commit();
            }
            if (lane == 0 && (32 * q) % N2 == 0 && tok0 + tok_h < T) scale_out[tok0 + tok_h] = s;
        }
        if (et == 0) bulk_wait<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// A wait on an mbarrier that nothing ever arrives at: exercises the bounded
// wait and the status word without touching any other state.
__global__ void kq_selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t mbar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_u32(&mbar), 1);
        fence_mbar_init();
        wait_bounded(smem_u32(&mbar), 0u, &abort_flag, kSiteSelfTest, limit_ns, true);
    }
}

// ---------------------------------------------------------------------------
// Host side.

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

template <int N1, int N2, bool SCALED>
cudaError_t launch_inst(const LaunchArgs &a) {
    using C = Cfg<N1, N2, SCALED>;
    auto kern = kq_tc05_fused_kernel<N1, N2, SCALED>;
    static std::once_flag attr_once[64];
    static cudaError_t attr_err[64];
    if (a.device < 0 || a.device >= 64) return cudaErrorInvalidDevice;
    std::call_once(attr_once[a.device], [&] {
        attr_err[a.device] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    });
    if (attr_err[a.device] != cudaSuccess) return attr_err[a.device];

    PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap tmap;
    const cuuint64_t dims[2] = {cuuint64_t(N2), cuuint64_t(a.T) * N1};
    const cuuint64_t strides[1] = {cuuint64_t(N2) * 2};
    const cuuint32_t box[2] = {64u, cuuint32_t(N1)};
    const cuuint32_t estr[2] = {1u, 1u};
    CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(a.x), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const int64_t G = (a.T + C::H - 1) / C::H;
    const int64_t grid = G < a.num_sms ? G : a.num_sms;
    kern<<<unsigned(grid), kTcThreads, C::SMEM, a.stream>>>(tmap, a.P1, a.P2, a.cinv, a.alpha, a.q_out,
                                                            a.scale_out, a.T);
    return cudaGetLastError();
}

template <int N2, bool SCALED>
cudaError_t dispatch_n1(const LaunchArgs &a) {
    switch (a.n1) {
    case 16: return launch_inst<16, N2, SCALED>(a);
    case 32: return launch_inst<32, N2, SCALED>(a);
    case 48: return launch_inst<48, N2, SCALED>(a);
    case 64: return launch_inst<64, N2, SCALED>(a);
    default: break;
    }
    if constexpr (!SCALED) {
        switch (a.n1) {
        case 80: return launch_inst<80, N2, false>(a);
        case 96: return launch_inst<96, N2, false>(a);
        case 112: return launch_inst<112, N2, false>(a);
        case 128: return launch_inst<128, N2, false>(a);
        default: break;
        }
    }
    return cudaErrorNotSupported;
}

}  // namespace

bool tc05_supports(int n1, int n2, bool scaled) {
    if (n2 != 64 && n2 != 128) return false;
    if (n1 < 16 || n1 > 128 || n1 % 16) return false;
    return !scaled || n1 <= 64;
}

cudaError_t launch_tc05(const LaunchArgs &a) {
    if (a.T * int64_t(a.n1) >= (int64_t(1) << 31)) return launch_warp_mma(a);  // TMA row coordinate range
    const bool scaled = a.cinv != nullptr;
    if (a.n2 == 128) return scaled ? dispatch_n1<128, true>(a) : dispatch_n1<128, false>(a);
    return scaled ? dispatch_n1<64, true>(a) : dispatch_n1<64, false>(a);
}

cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t stream) {
    kq_selftest_wait_kernel<<<1, 32, 0, stream>>>(limit_ns);
    return cudaGetLastError();
}

}  // namespace kq
