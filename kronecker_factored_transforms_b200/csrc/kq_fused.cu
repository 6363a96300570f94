// kq_fused.cu -- persistent fused Kronecker transform + INT4 kernel on the
// 5th-generation tensor cores, pipelined per group of tokens.
//
// Method (FlatQuant page, "Kronecker factorization", "Per-channel scaling and
// learnable clipping" and "The fused kernel"): per token Y~ = P1^T X~ P2 with
// X~ the row-major n1 x n2 view of x o cinv, then the token's absmax,
// s = alpha * max / 7, round-half-even codes clamped to [-8, 7], two per byte.
// Only codes and scales reach HBM.
//
// Work unit: a group of H = 128 / n2 tokens, so that the 128 TMEM lanes hold
// the group's 128 output columns j (n2 = 64: two tokens, P2^T block-diagonal).
// TMEM lane m of a token holds column lane_column(m) (kq_tile.cuh), so that
// the epilogue thread of a 16x256b load holds four consecutive columns: two
// whole bytes of every output row.
//
//   stage 1   D1[l][a] = sum_k A1[l][k] X[a][k]: A1 = P2^T (TMEM, resident),
//             X = the group's x tile (K = 128; with cinv its x' = x o cinv hi
//             and lo bf16 tiles, accumulated in two passes), M = 128, N = n1.
//   convert   D1 (fp32) -> A2 = hi + lo bf16 pairs, in place in TMEM.
//   stage 2   D2[l][i] = sum_a A2[l][a] P1[a][i] (A from TMEM, B = P1^T in
//             shared memory; hi and lo passes), M = 128, N = n1.
//   epilogue  absmax over the token's lanes, quantise, pack, 16-bit stores
//             straight to global memory, one fp32 scale per token.
//
// TMEM: P2^T (64 columns), NA = 5 D1/A2 slots and ND = 2 D2 slots of n1
// columns.  One MMA thread issues stage 1 of group j + L before stage 2 of
// group j, so the conversion of a group overlaps the tensor work of the
// groups around it and every slot is reused only long after the MMAs that
// read it completed.
//
// x reaches the kernel in one of two ways.  Without cinv, TMA copies each
// group's x tile (128-byte swizzle, the K-major B layout) into a ring of
// shared-memory slots that stage 1 reads as is.  With cinv, eight warps load
// the group's x with 16-byte global loads (prefetched into L2 a few groups
// ahead), form x' = x o cinv as hi + lo bf16 in registers and store the two
// swizzled tiles; the raw x tile never passes through shared memory.
//
// Warp roles (24 warps): 0 factor copies, then (without cinv) the TMA
// producer | 1 TMEM allocation and MMA issue | 2-3 set-up only | 4-11 x'
// split (cinv) | 12-15 D1 -> A2 conversion | 16-19 and 20-23 two epilogue
// warpgroups on alternate groups (each with its own D2 slot).  Every mbarrier
// wait is bounded: after about a second it ORs a site bit into the device
// status word, raises a CTA-wide abort flag and the roles drain and exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "kq_common.cuh"
#include "kq_internal.h"
#include "kq_tc05_ptx.cuh"
#include "kq_tile.cuh"
#include "kq_wait.cuh"

namespace kq {
namespace {

using namespace tc;
using namespace tile;

enum : unsigned {
    kSiteFProducer = 1u,
    kSiteFSplit = 2u,
    kSiteFMma = 4u,
    kSiteFConvert = 8u,
    kSiteFEpilogue = 16u,
    kSiteFDrain = 32u,
};

constexpr int kFThreads = 1024;  // 32 warps, at most 64 registers per thread
constexpr int kSplitThreads = 512;  // warps 4-19
constexpr int kSplitWarps = kSplitThreads / 32;
constexpr int kConvWarp0 = 4 + kSplitWarps;  // warps 20-23: D1 -> A2 conversion
constexpr int kEpiWarp0 = kConvWarp0 + 4;    // warps 24-31: two epilogue warpgroups
constexpr int kSetupArrivals = 14;  // warps 2, 3, 20-31 arrive once their set-up share is done

__host__ __device__ constexpr int f_align_up(int v, int a) { return (v + a - 1) / a * a; }

template <int N1, int N2, bool SCALED>
struct FCfg {
    static constexpr int H = 128 / N2;            // tokens per group
    static constexpr int CHUNK = N1 * 128;        // bytes of one 64-element K chunk of a group tile
    static constexpr int TILE = 2 * CHUNK;        // one bf16 tile [n1 rows][K = 128]
    static constexpr int XSLOT = SCALED ? 2 * TILE : TILE;  // x' hi + lo, or x
    static constexpr int NA = 4, ND = 3;          // D1/A2 and D2 slots in TMEM
    static constexpr int A1COLS = 64;             // P2^T: 128 K values of bf16 per lane
    static constexpr int TMEM_COLS = 512;
    static constexpr int NX = SCALED ? 6 : 12;    // shared-memory x slots
    static constexpr int OFF_B2 = 0;              // P1^T [n1 rows][K = n1], 128-byte swizzle
    static constexpr int OFF_X = f_align_up(N1 * 128, 1024);
    static constexpr int OFF_BAR = OFF_X + NX * XSLOT;
    static constexpr int CFULL = 0, XFREE = NX, D1FULL = 2 * NX, A2FULL = D1FULL + NA, AFREE = A2FULL + NA,
                         D2FULL = AFREE + NA, D2FREE = D2FULL + ND, FACT = D2FREE + ND, SETUP = FACT + 1,
                         TEARDOWN = SETUP + 1, NBAR = TEARDOWN + 1;
    static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;  // tmem base, abort flag, the constant 1, maxima
    static constexpr int SMEM = OFF_MISC + 96 + 1024;    // + slack for 1024-byte alignment
    // P1 and P2 arrive by bulk copies into the last NSCR x slots, which take x
    // tiles only once the factor operands are built from them.
    static constexpr int P1B = N1 * N1 * 2, P2B = N2 * N2 * 2;
    static constexpr int OFF_SP2 = f_align_up(P1B, 1024);
    static constexpr int NSCR = (OFF_SP2 + P2B + XSLOT - 1) / XSLOT;
    static constexpr int OFF_SCR = OFF_X + (NX - NSCR) * XSLOT;
    __host__ __device__ static constexpr uint32_t SLOT_A(int s) { return uint32_t(A1COLS + s * N1); }
    __host__ __device__ static constexpr uint32_t SLOT_D(int d) { return uint32_t(A1COLS + (NA + d) * N1); }
    static_assert(N1 == 64, "this kernel is built for n1 = 64");
    static_assert(N2 == 64 || N2 == 128, "stage 1 needs K = H * n2 = 128");
    static_assert(A1COLS + (NA + ND) * N1 <= TMEM_COLS, "TMEM budget");
    static_assert(NX > NSCR, "x slots besides the factor scratch");
    static_assert(OFF_X % 1024 == 0 && XSLOT % 1024 == 0 && TILE % 1024 == 0, "swizzle alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(16 * N1 == 2 * kSplitThreads, "two 16-byte x units per split thread and group");
};

// Bulk prefetch of global memory into L2 (no completion to wait for).
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// 16-byte read-only global load that does not allocate in L1 (streamed once).
__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// v = hi + lo with hi = v truncated to bf16 (its top 16 bits, a byte permute)
// and lo = v - hi (exact in fp32) rounded to bf16: about 16 significant bits.
// Takes two fp32 values; returns the two hi values packed (first in the low
// half) and the two lo ones.
__device__ __forceinline__ void split_pair(uint32_t v0, uint32_t v1, uint32_t &hi, uint32_t &lo) {
    const uint64_t v = uint64_t(v0) | (uint64_t(v1) << 32);
    const uint64_t t = uint64_t(v0 & 0xFFFF0000u) | (uint64_t(v1 & 0xFFFF0000u) << 32);
    const uint64_t l = f32x2_sub(v, t);
    hi = __byte_perm(v0, v1, 0x7632);
    lo = pack_bf16x2(__uint_as_float(uint32_t(l)), __uint_as_float(uint32_t(l >> 32)));
}

// round_half_even(y * inv) for |y * inv| < 2^22: adding 1.5 * 2^23 leaves the
// rounded integer in the low mantissa bits (bit pattern 0x4B400000 + k); an
// integer multiply-add with `one` (== 1, read at run time) removes the offset.
constexpr uint32_t kFMagicBits = 0x4B400000u;  // 1.5 * 2^23
__device__ __forceinline__ int f_round_code(uint32_t ybits, float inv, int one) {
    const uint32_t b = __float_as_uint(fmaf(__uint_as_float(ybits), inv, 12582912.0f));
    int k;
    asm("mad.lo.s32 %0, %1, %2, %3;" : "=r"(k) : "r"(b), "r"(one), "r"(-int(kFMagicBits)));
    return k;
}

template <int N1, int N2, bool SCALED>
__global__ void __launch_bounds__(kFThreads, 1)
    kq_fused_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint16_t *__restrict__ x,
                    const uint16_t *__restrict__ P1, const uint16_t *__restrict__ P2, const float *__restrict__ cinv,
                    float alpha, uint8_t *__restrict__ q_out, float *__restrict__ scale_out, int64_t T,
                    unsigned int *err) {
    using C = FCfg<N1, N2, SCALED>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - raw_addr);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Groups of H tokens, dealt round-robin to the CTAs.
    const int64_t G = (T + C::H - 1) / C::H;
    const int nloc = G > int64_t(blockIdx.x) ? int((G - 1 - blockIdx.x) / gridDim.x) + 1 : 0;
    auto group_of = [&](int j) -> int64_t { return int64_t(blockIdx.x) + int64_t(j) * gridDim.x; };

    auto bar = [&](int i) -> uint32_t { return sbase + uint32_t(C::OFF_BAR + 8 * i); };
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    float *s_red = reinterpret_cast<float *>(smem + C::OFF_MISC + 16);  // [2 warpgroups][2 buffers][4 warps]
    auto wait = [&](int b, uint32_t parity, unsigned site) -> bool {
        return wait_bounded_err(bar(b), parity, s_abort, site, kWaitLimitNs, false, err);
    };

    if (tid == 0) {
        for (int s = 0; s < C::NX; ++s) {
            mbar_init(bar(C::CFULL + s), SCALED ? kSplitWarps : 1);
            mbar_init(bar(C::XFREE + s), 1);
        }
        for (int s = 0; s < C::NA; ++s) {
            mbar_init(bar(C::D1FULL + s), 1);
            mbar_init(bar(C::A2FULL + s), 4);
            mbar_init(bar(C::AFREE + s), 1);
        }
        for (int d = 0; d < C::ND; ++d) {
            mbar_init(bar(C::D2FULL + d), 1);
            mbar_init(bar(C::D2FREE + d), 4);
        }
        mbar_init(bar(C::FACT), 1);
        mbar_init(bar(C::SETUP), kSetupArrivals);
        mbar_init(bar(C::TEARDOWN), 2);  // one commit from each MMA issuer
        *s_abort = 0;
        *reinterpret_cast<int *>(smem + C::OFF_MISC + 8) = 1;  // `one` of f_round_code
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0 && !SCALED) prefetch_tensormap(&tmap_x);
    if (warp == 1) {
        tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    // The next launch on the stream may be scheduled once every CTA holds its SM
    // and its TMEM; its CTAs start as this grid's CTAs exit.  Every global access
    // of this grid (x, P1, P2, cinv, codes, scales) follows the previous grid's
    // completion.
    griddep_launch_dependents();
    griddep_wait();

    // ---------------- set-up: P1^T into shared memory, P2^T into TMEM ----------------
    const bool setup_warp = warp == 2 || warp == 3 || warp >= kConvWarp0;
    if (setup_warp) {
        // (on a timeout the abort flag is up and the operands do not matter)
        wait(C::FACT, 0u, kSiteFProducer);
        const uint16_t *P1s = reinterpret_cast<const uint16_t *>(smem + C::OFF_SCR);
        const uint16_t *P2s = reinterpret_cast<const uint16_t *>(smem + C::OFF_SCR + C::OFF_SP2);
        if (warp == 2 || warp == 3 || warp >= kEpiWarp0 + 4) {
            // B2[i][a] = P1[a][i] (rows i, K = a), 128-byte swizzle: a piece is one
            // row i and eight consecutive a; one 16-byte store each.
            constexpr int kThr = 6 * 32, PIECES = 8 * N1, PER = (PIECES + kThr - 1) / kThr;
            const int st = (warp >= kEpiWarp0 + 4 ? 64 + 32 * (warp - kEpiWarp0 - 4) : 32 * (warp - 2)) + lane;
            uint32_t w[PER][4];
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int c = st + u * kThr;
                const int i = c % N1, a0 = 8 * (c / N1);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int a = a0 + 2 * e;
                    const uint32_t lo = c < PIECES ? P1s[a * N1 + i] : 0u;
                    const uint32_t hi = c < PIECES ? P1s[(a + 1) * N1 + i] : 0u;
                    w[u][e] = lo | (hi << 16);
                }
            }
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int c = st + u * kThr;
                if (c < PIECES) {
                    const int i = c % N1, a0 = 8 * (c / N1);
                    *reinterpret_cast<uint4 *>(smem + C::OFF_B2 + swz128(i, a0)) =
                        make_uint4(w[u][0], w[u][1], w[u][2], w[u][3]);
                }
            }
            fence_proxy_async_smem();  // B2 is read by the tensor cores
        }
        if (warp >= kConvWarp0 && warp < kEpiWarp0 + 4) {
            // A1 = block-diag P2^T (rows permuted) into TMEM columns [0, 64): lane l
            // holds row l, K pairs packed per column; warps 20-23 write K in [0, 64),
            // warps 24-27 K in [64, 128).
            const int l = 32 * (warp & 3) + lane;
            const uint32_t taddr = tmem + (uint32_t(32 * (warp & 3)) << 16);
            const int kc0 = warp < kEpiWarp0 ? 0 : 2;
#pragma unroll
            for (int kq = 0; kq < 2; ++kq) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int k = 32 * (kc0 + kq) + 2 * e;
                    w[e] = uint32_t(a1_value<N2>(P2s, l, k)) | (uint32_t(a1_value<N2>(P2s, l, k + 1)) << 16);
                }
                tmem_st_32x32b_x16(taddr + 16 * (kc0 + kq), w);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::SETUP));
    }

    if (warp == 0) {
        // ---------------- factor copies; without cinv the TMA producer ----------------
        if (elect_one()) {
            mbar_arrive_expect_tx(bar(C::FACT), uint32_t(C::P1B + C::P2B));
            bulk_load(sbase + C::OFF_SCR, P1, uint32_t(C::P1B), bar(C::FACT));
            bulk_load(sbase + C::OFF_SCR + C::OFF_SP2, P2, uint32_t(C::P2B), bar(C::FACT));
        }
        __syncwarp();
        if (!SCALED) {
            bool setup_seen = false;
            Ring rx;
            int issued = 0;
            for (int j = 0; j < nloc; ++j, rx.next(C::NX)) {
                if (!setup_seen && j == C::NX - C::NSCR) {
                    // the scratch slots are read by the set-up warps before TMA reuses them
                    if (!__all_sync(0xffffffffu, wait(C::SETUP, 0u, kSiteFProducer))) break;
                    setup_seen = true;
                }
                const bool ok = wait(C::XFREE + rx.idx, rx.phase ^ 1u, kSiteFProducer);
                if (!__all_sync(0xffffffffu, ok)) break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(bar(C::CFULL + rx.idx), C::TILE);
                    const uint32_t dst = sbase + C::OFF_X + rx.idx * C::XSLOT;
                    const int64_t g = group_of(j);
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int xc = (N2 == 128) ? 64 * c : 0;
                        const int64_t row = (N2 == 128) ? g * N1 : (2 * g + c) * N1;
                        tma_load_2d(dst + c * C::CHUNK, &tmap_x, xc, int(row), bar(C::CFULL + rx.idx));
                    }
                }
                __syncwarp();
                ++issued;
            }
            // Drain: every load issued has landed (the slots' last phases completed).
            Ring rd;
            for (int i = 0; i < issued; ++i, rd.next(C::NX))
                if (i + C::NX >= issued)
                    wait_bounded_err(bar(C::CFULL + rd.idx), rd.phase, s_abort, kSiteFDrain, kWaitLimitNs, true, err);
            __syncwarp();
        }
        // the factor copies have landed before the CTA can exit
        wait_bounded_err(bar(C::FACT), 0u, s_abort, kSiteFDrain, kWaitLimitNs, true, err);
    } else if (warp == 1 || warp == 3) {
        // ---------------- MMA issue: warp 1 stage 1, warp 3 stage 2 ----------------
        // Two issuers, so that the latency of one stage's barrier waits and commits
        // (an mbarrier operation takes 100-300 cycles while shared memory is busy)
        // overlaps the other stage's MMAs.  Stage 1 of group j reuses the D1/A2 slot
        // of group j - NA only after stage 2 of that group has completed (AFREE), so
        // stage 1 runs at most NA groups ahead.  Each runs its loop converged; one
        // elected lane issues the MMAs and the commits.
        constexpr uint32_t idesc = idesc_bf16_f32(128, N1);
        const uint32_t b2l = sdesc_sw128_lo(sbase + C::OFF_B2);
        const bool ok0 = __all_sync(0xffffffffu, wait(C::SETUP, 0u, kSiteFMma));
        tc_fence_after();
        if (warp == 1) {
            for (int j = 0; ok0 && j < nloc; ++j) {
                const int xs = j % C::NX, as = j % C::NA;
                bool w = wait(C::CFULL + xs, uint32_t(j / C::NX) & 1u, kSiteFMma);
                w = w && wait(C::AFREE + as, (uint32_t(j / C::NA) & 1u) ^ 1u, kSiteFMma);
                if (!__all_sync(0xffffffffu, w)) break;
                tc_fence_after();
                const uint32_t d = tmem + C::SLOT_A(as);
                const uint32_t xb = sbase + C::OFF_X + xs * C::XSLOT;
                if (elect_one()) {
#pragma unroll
                    for (int pass = 0; pass < (SCALED ? 2 : 1); ++pass) {
                        const uint32_t bl = sdesc_sw128_lo(xb + pass * C::TILE);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t b = bl + uint32_t(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4);
                            if ((pass | kk) != 0)
                                mma_ts_split<1>(d, tmem + 8 * kk, b, kSdescSw128Hi, idesc);
                            else
                                mma_ts_split<0>(d, tmem + 8 * kk, b, kSdescSw128Hi, idesc);
                        }
                    }
                    tc_commit(bar(C::XFREE + xs));   // x slot free once these MMAs have read it
                    tc_commit(bar(C::D1FULL + as));  // D1 complete
                }
                __syncwarp();
            }
        } else {
            for (int j = 0; ok0 && j < nloc; ++j) {
                const int as = j % C::NA, ds = j % C::ND;
                bool w = wait(C::A2FULL + as, uint32_t(j / C::NA) & 1u, kSiteFMma);
                w = w && wait(C::D2FREE + ds, (uint32_t(j / C::ND) & 1u) ^ 1u, kSiteFMma);
                if (!__all_sync(0xffffffffu, w)) break;
                tc_fence_after();
                const uint32_t d = tmem + C::SLOT_D(ds), a2 = tmem + C::SLOT_A(as);
                if (elect_one()) {
#pragma unroll
                    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                        for (int kk = 0; kk < N1 / 16; ++kk) {
                            const uint32_t b = b2l + uint32_t((kk * 32) >> 4);
                            if ((pass | kk) != 0)
                                mma_ts_split<1>(d, a2 + 16 * kk + 8 * pass, b, kSdescSw128Hi, idesc);
                            else
                                mma_ts_split<0>(d, a2 + 16 * kk + 8 * pass, b, kSdescSw128Hi, idesc);
                        }
                    tc_commit(bar(C::D2FULL + ds));  // D2 complete
                    tc_commit(bar(C::AFREE + as));   // D1/A2 slot free
                }
                __syncwarp();
            }
        }
        // Every MMA either issuer issued has completed before TMEM is freed.
        if (elect_one()) tc_commit(bar(C::TEARDOWN));
        __syncwarp();
        wait_bounded_err(bar(C::TEARDOWN), 0u, s_abort, kSiteFDrain, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp >= 4 && warp < kConvWarp0) {
        // ---------------- x' = x o cinv -> hi / lo bf16 tiles ----------------
        if (SCALED) {
            const int t = tid - 128;  // 0 .. 511
            constexpr int UPT = 2;     // 16-byte units per thread per group (1024 units)
            // Unit e = t + 512 u of a group: 8 consecutive x values at byte 16 e of the
            // group's (contiguous) x, which is row r of B chunk c, 16-byte column k8:
            //   n2 = 128: r = e / 16, c = (e / 8) % 2, k8 = e % 8;
            //   n2 = 64:  c = e / 512 (the token), r = (e / 8) % 64, k8 = e % 8.
            // Its cinv values start at channel 8 (e mod (n / 8)).
            // The tile offset of unit u is soff0 + u * SDELTA: unit u = 1 lies 32 rows
            // further down (n2 = 128) or in the second token's chunk (n2 = 64).
            constexpr uint32_t SDELTA = N2 == 128 ? 32 * 128 : C::CHUNK;
            uint32_t soff0;
            uint32_t ch[UPT][4], cl[UPT][4];
            {
                float4 ca[UPT], cb[UPT];
                {
                    const int r = N2 == 128 ? t / 16 : t / 8, c = N2 == 128 ? (t / 8) % 2 : 0, k8 = t % 8;
                    soff0 = uint32_t(c * C::CHUNK + r * 128 + ((k8 ^ (r & 7)) << 4));
                }
#pragma unroll
                for (int u = 0; u < UPT; ++u) {
                    const int e = t + kSplitThreads * u;
                    const int ch0 = 8 * (e % (N1 * N2 / 8));
                    ca[u] = __ldg(reinterpret_cast<const float4 *>(cinv + ch0));
                    cb[u] = __ldg(reinterpret_cast<const float4 *>(cinv + ch0 + 4));
                }
                // cinv = ch + cl, two bf16 values (RN(cinv) and RN of the rest), so that
                // x' needs only packed bf16 arithmetic: hi = RN(x ch),
                // lo = RN(x cl + RN(x ch - hi)), each step one fused rounding; hi + lo is
                // x * cinv to about 2^-14 relative.
#pragma unroll
                for (int u = 0; u < UPT; ++u) {
                    const float cv[8] = {ca[u].x, ca[u].y, ca[u].z, ca[u].w, cb[u].x, cb[u].y, cb[u].z, cb[u].w};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float c0 = cv[2 * p], c1 = cv[2 * p + 1];
                        ch[u][p] = pack_bf16x2(c0, c1);
                        cl[u][p] = pack_bf16x2(c0 - __uint_as_float(ch[u][p] << 16),
                                               c1 - __uint_as_float(ch[u][p] & 0xFFFF0000u));
                    }
                }
            }
            // x of a group: H tokens, contiguous; this thread's unit u is at byte
            // 16 t + 8192 u of it; a unit of a token past T reads as zero (n2 = 64:
            // unit u belongs to token u of the group).
            const unsigned char *xg = reinterpret_cast<const unsigned char *>(x);
            const unsigned char *xt = xg + 16 * t;
            constexpr int64_t GBYTES = int64_t(C::H) * N1 * N2 * 2;
            auto load_group = [&](int j, uint4 (&v)[UPT]) {
                const int64_t g = group_of(j);
                const unsigned char *src = xt + g * GBYTES;
#pragma unroll
                for (int u = 0; u < UPT; ++u) {
                    const bool in = N2 == 128 || g * C::H + u < T;
                    v[u] = in ? ldg_stream(src + 8192 * u) : make_uint4(0u, 0u, 0u, 0u);
                }
            };
            constexpr int PD = 4;  // groups prefetched into L2 ahead of the loads
            const bool prefetcher = t == 0;
            auto prefetch_group = [&](int j) {
                if (j < nloc) {
                    const int64_t g = group_of(j);
                    const int64_t tokens = T - g * C::H < C::H ? T - g * C::H : C::H;
                    prefetch_l2(xg + g * GBYTES, uint32_t(tokens * N1 * N2 * 2));
                }
            };
            if (prefetcher)
                for (int j = 2; j < 2 + PD; ++j) prefetch_group(j);
            // Two groups of loads in flight per thread: group j's values sit in xv[j % 2];
            // once a unit is stored, the same registers take that unit of group j + 2.
            uint4 xv[2][UPT];
#pragma unroll
            for (int b = 0; b < 2; ++b)
                if (b < nloc) load_group(b, xv[b]);
            bool setup_seen = false;
            Ring rx;
            auto body = [&](int j, uint4 (&v)[UPT]) -> bool {
                if (!setup_seen && j == C::NX - C::NSCR) {
                    // the scratch slots are read by the set-up warps before they are overwritten
                    if (!__all_sync(0xffffffffu, wait(C::SETUP, 0u, kSiteFSplit))) return false;
                    setup_seen = true;
                }
                if (!__all_sync(0xffffffffu, wait(C::XFREE + rx.idx, rx.phase ^ 1u, kSiteFSplit))) return false;
                if (prefetcher) prefetch_group(j + 2 + PD);
                unsigned char *hi = smem + C::OFF_X + rx.idx * C::XSLOT;
                unsigned char *lo = hi + C::TILE;
#pragma unroll
                for (int u = 0; u < UPT; ++u) {
                    const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    uint32_t oh[4], ol[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        oh[p] = bf16x2_mul(w[p], ch[u][p]);
                        const uint32_t rest = bf16x2_fma(w[p], ch[u][p], bf16x2_neg(oh[p]));
                        ol[p] = bf16x2_fma(w[p], cl[u][p], rest);
                    }
                    *reinterpret_cast<uint4 *>(hi + soff0 + u * SDELTA) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
                    *reinterpret_cast<uint4 *>(lo + soff0 + u * SDELTA) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
                }
                // the registers take group j + 2 (its loads overlap the next group's work)
                if (j + 2 < nloc) load_group(j + 2, v);
                fence_proxy_async_smem();  // the tiles are read by the tensor cores
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::CFULL + rx.idx));
                rx.next(C::NX);
                return true;
            };
            for (int j = 0; j < nloc; j += 2) {
                if (!body(j, xv[0])) break;
                if (j + 1 < nloc && !body(j + 1, xv[1])) break;
            }
        }
    } else if (warp >= kConvWarp0 && warp < kEpiWarp0) {
        // ---------------- D1 (fp32) -> A2 (hi, lo bf16) in TMEM ----------------
        const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
        for (int j = 0; j < nloc; ++j) {
            const int as = j % C::NA;
            if (!__all_sync(0xffffffffu, wait(C::D1FULL + as, uint32_t(j / C::NA) & 1u, kSiteFConvert))) break;
            tc_fence_after();
            const uint32_t col0 = tmem + lane_off + C::SLOT_A(as);
            constexpr int NK = N1 / 16;
            // 16-column chunks, software-pipelined: chunk k + 1 loads while chunk k
            // is converted and stored.  A chunk's 16 fp32 columns (K = 16 values of a)
            // become 8 columns of hi pairs then 8 of lo pairs.
            uint32_t v[2][16];
            tmem_ld_32x32b_x16(col0, v[0]);
            tmem_wait_ld_tie(v[0]);
#pragma unroll
            for (int k = 0; k < NK; ++k) {
                if (k + 1 < NK) tmem_ld_32x32b_x16(col0 + 16 * (k + 1), v[(k + 1) & 1]);
                uint32_t o[16];
#pragma unroll
                for (int e = 0; e < 8; ++e) split_pair(v[k & 1][2 * e], v[k & 1][2 * e + 1], o[e], o[8 + e]);
                tmem_st_32x32b_x16(col0 + 16 * k, o);
                if (k + 1 < NK) tmem_wait_ld_tie(v[(k + 1) & 1]);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::A2FULL + as));
        }
    } else if (warp >= kEpiWarp0) {
        // ---------------- epilogue: absmax, quantise, pack, store ----------------
        // Warpgroup ew takes the groups j with j % 2 == ew; group j's D2 is in slot
        // j % ND.  A thread
        // reads, with 16x256b loads, lanes g8 and g8 + 8 of both 16-lane halves of its
        // warp's 32 lanes: four consecutive output columns (lane_column), two whole
        // bytes of each output row, stored as one 16-bit word.
        const int ew = (warp - kEpiWarp0) >> 2;
        const int q = warp & 3;
        const uint32_t nbar = 1u + uint32_t(ew);
        const int tok_h = (32 * q) / N2;  // the token of the group this warp's lanes belong to
        const int g8 = lane >> 2, qq = lane & 3;
        float *red = s_red + 8 * ew;
        const int one = *reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);
        constexpr int NK = N1 / 16;
        constexpr int RB = N2 / 2;  // bytes of one output row i of a token
        const uint32_t tq = tmem + (uint32_t(32 * q) << 16);
        const int bcol = ((32 * q) % N2) / 2 + 2 * g8;
        int it = 0;
        for (int j = ew; j < nloc; j += 2, ++it) {
            const int buf = it & 1;
            const int ds = j % C::ND;
            const uint32_t t0 = tq + C::SLOT_D(ds);
            const bool ok = wait(C::D2FULL + ds, uint32_t(j / C::ND) & 1u, kSiteFEpilogue);
            // All four warps leave together, so none is left behind in a named barrier.
            if (named_barrier_any(nbar, 128, !__all_sync(0xffffffffu, ok))) break;
            __syncwarp();
            tc_fence_after();
            // absmax from a first read (32x32b: thread = lane), 16 columns per load
            float mx4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int k0 = 0; k0 < N1; k0 += 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(t0 + k0, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; e += 8) {
                    mx4[0] = fmax3(mx4[0], fabsf(__uint_as_float(v[e])), fabsf(__uint_as_float(v[e + 1])));
                    mx4[1] = fmax3(mx4[1], fabsf(__uint_as_float(v[e + 2])), fabsf(__uint_as_float(v[e + 3])));
                    mx4[2] = fmax3(mx4[2], fabsf(__uint_as_float(v[e + 4])), fabsf(__uint_as_float(v[e + 5])));
                    mx4[3] = fmax3(mx4[3], fabsf(__uint_as_float(v[e + 6])), fabsf(__uint_as_float(v[e + 7])));
                }
            }
            const float mx = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]);
            // non-negative floats order like their bit patterns: one warp reduction
            const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
            if (lane == 0) red[4 * buf + q] = __uint_as_float(wmax);
            named_barrier_sync(nbar, 128);  // maxima visible
            float m = 0.0f;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if ((32 * w) / N2 == tok_h) m = fmaxf(m, red[4 * buf + w]);
            // s = alpha * max / 7 to within an ulp; codes use y * (1/s): both differ from
            // the exact quotients by a few ulps, far inside the rounding-boundary window
            const float s = alpha * m * (1.0f / 7.0f);
            const float inv = s > 0.0f ? fminf(__fdividef(1.0f, s), 3.0e38f) : 0.0f;
            const int64_t tok = group_of(j) * C::H + tok_h;
            const bool live = tok < T;
            // this thread's two bytes of rows i = 16 c0 + 8 rep + 2 qq + d of its token
            uint8_t *gq = q_out + (live ? tok : 0) * int64_t(N1 * RB) + (2 * qq) * RB + bcol;
#pragma unroll
            for (int c0 = 0; c0 < NK; ++c0) {
                uint32_t ra[8], rb[8];  // half 0 (lanes 32 q + [0, 16)) and half 1 (+ [16, 32))
                tmem_ld_16x256b_x2(t0 + 16 * c0, ra);
                tmem_ld_16x256b_x2(t0 + (16u << 16) + 16 * c0, rb);
                tmem_wait_ld();
                if (c0 + 1 == NK) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(C::D2FREE + ds));  // D2 slot free for stage 2
                }
                if (live) {
#pragma unroll
                    for (int rep = 0; rep < 2; ++rep)
#pragma unroll
                        for (int d = 0; d < 2; ++d) {
                            // row 16 c0 + 8 rep + 2 qq + d: columns 4 g8 + (0, 1) from half 0,
                            // + (2, 3) from half 1; even column in the low nibble
                            const uint32_t wb = pack_s4x2(f_round_code(rb[4 * rep + 2 + d], inv, one),
                                                          f_round_code(rb[4 * rep + d], inv, one), 0u);
                            const uint32_t wv = pack_s4x2(f_round_code(ra[4 * rep + 2 + d], inv, one),
                                                          f_round_code(ra[4 * rep + d], inv, one), wb);
                            *reinterpret_cast<uint16_t *>(gq + (16 * c0 + 8 * rep + d) * RB) = uint16_t(wv);
                        }
                }
            }
            if (live && lane == 0 && (32 * q) % N2 == 0) scale_out[tok] = s;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Host side.

template <int N1, int N2, bool SCALED>
cudaError_t launch_fused_inst(const LaunchArgs &a) {
    using C = FCfg<N1, N2, SCALED>;
    auto kern = kq_fused_kernel<N1, N2, SCALED>;
    static std::once_flag attr_once[64];
    static cudaError_t attr_err[64];
    if (a.device < 0 || a.device >= 64) return cudaErrorInvalidDevice;
    std::call_once(attr_once[a.device], [&] {
        attr_err[a.device] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    });
    if (attr_err[a.device] != cudaSuccess) return attr_err[a.device];
    unsigned int *err = nullptr;
    cudaError_t e = device_error_word(a.device, &err);
    if (e != cudaSuccess) return e;

    CUtensorMap tmap;
    memset(&tmap, 0, sizeof(tmap));
    if (!SCALED) {
        PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
        if (!encode) return cudaErrorNotSupported;
        const cuuint64_t dims[2] = {cuuint64_t(N2), cuuint64_t(a.T) * N1};
        const cuuint64_t strides[1] = {cuuint64_t(N2) * 2};
        const cuuint32_t box[2] = {64u, cuuint32_t(N1)};
        const cuuint32_t estr[2] = {1u, 1u};
        CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(a.x), dims, strides,
                            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    const int64_t G = (a.T + C::H - 1) / C::H;
    const int64_t grid = G < a.num_sms ? G : a.num_sms;
    return launch_overlapped(kern, unsigned(grid), kFThreads, C::SMEM, a.stream, tmap, a.x, a.P1, a.P2, a.cinv,
                             a.alpha, a.q_out, a.scale_out, a.T, err);
}

}  // namespace

bool fused_supports(int n1, int n2, bool scaled) {
    (void)n1;
    (void)n2;
    (void)scaled;
    return false;  // not selected yet: slower than kq_tc05_fused_kernel at large T
}

cudaError_t launch_fused(const LaunchArgs &a) {
    const bool scaled = a.cinv != nullptr;
    if (a.n2 == 128) return scaled ? launch_fused_inst<64, 128, true>(a) : launch_fused_inst<64, 128, false>(a);
    return scaled ? launch_fused_inst<64, 64, true>(a) : launch_fused_inst<64, 64, false>(a);
}

}  // namespace kq
