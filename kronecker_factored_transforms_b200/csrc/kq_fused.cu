// kq_fused.cu -- persistent fused Kronecker transform + INT4 kernel on the
// 5th-generation tensor cores, pipelined per pair of token groups; the kernel
// kq_transform_quant runs for short launches at n1 = 64 (up to 56 groups per
// SM without cinv, 4 with it), where the batch-pipelined kernel of kq_tc05.cu
// spends a larger share of the launch filling and draining its pipeline.
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
// whole bytes of every output row.  A CTA takes its groups (dealt round-robin)
// in pairs.
//
//   stage 1   D1[l][a] = sum_k A1[l][k] X[a][k] for both groups of a pair in
//             one MMA (M = 128, N = 2 n1 = 128, K = 128): A1 = P2^T (TMEM,
//             resident), X = the pair's x tile, or with cinv its x' = x o cinv
//             as -hi and lo bf16 tiles accumulated in two passes (the -hi pass
//             with the MMA's negate-B bit).
//   convert   D1 (fp32) -> A2 = hi and -lo bf16 halves, in place in TMEM.
//   stage 2   D2[l][i] = sum_a A2[l][a] P1[a][i] per group (A from TMEM, B =
//             P1^T in shared memory; the -lo pass with negate-B), M = 128, N = n1.
//   epilogue  absmax over the token's lanes, quantise, pack, 16-bit stores
//             straight to global memory, one fp32 scale per token.
//
// TMEM: P2^T (64 columns), two D1/A2 regions of 2 n1 columns (one pair each)
// and three D2 slots of n1 columns (one per epilogue warpgroup).  Stage 1 of a
// pair reuses its region only after stage 2 of the pair two back completed, so
// the tensor pipe runs stage 1 of two pairs, then stage 2 of the two pairs
// before them, and so on.
//
// x reaches the kernel in one of two ways.  Without cinv, TMA copies each
// pair's x tile (128-byte swizzle, the K-major B layout) into a ring of
// shared-memory slots that stage 1 reads as is.  With cinv, the split warps
// load x with 16-byte global loads (prefetched into L2 a few pairs ahead by
// warp 0), form x' = x o cinv as -hi + lo bf16 in registers (three packed bf16
// operations per pair of values, cinv held in registers as two bf16 values)
// and store the two swizzled tiles; the raw x tile never passes through shared
// memory.
//
// Warp roles (32 warps, at most 64 registers per thread): 0 factor copies,
// then the TMA producer (without cinv) or the L2 prefetch (with cinv) | 1
// TMEM allocation and stage-1 MMA issue | 3 stage-2 MMA issue | 4-19 x' split
// (cinv) and the D1 -> A2 conversion, running the split two pairs ahead of
// the conversion | 20-31 three epilogue warpgroups on groups j with j % 3 ==
// warpgroup | 2 idle.  Warps 4-11 and 20-31 build P2^T (TMEM) and P1^T (shared
// memory) at start.  Every mbarrier wait is bounded: after about a second it
// ORs a site bit into the device status word, raises a CTA-wide abort flag and
// the roles drain and exit.
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

constexpr int kFThreads = 1024;   // 32 warps, at most 64 registers per thread
constexpr int kSplitWarp0 = 4;    // warps 4-19: x' split (with cinv) and the D1 -> A2 conversion
constexpr int kSplitWarps = 16;
constexpr int kSplitThreads = 32 * kSplitWarps;
constexpr int kEpiWarp0 = 20;     // warps 20-31: three epilogue warpgroups
constexpr int kEpiGroups = 3;
constexpr int kSetupArrivals = 8 + 12;  // P2^T into TMEM by warps 4-11, P1^T into shared memory by warps 20-31

__host__ __device__ constexpr int f_align_up(int v, int a) { return (v + a - 1) / a * a; }

template <int N1, int N2, bool SCALED>
struct FCfg {
    static constexpr int H = 128 / N2;            // tokens per group
    static constexpr int GCHUNK = N1 * 128;       // one group's rows of a 64-element K chunk (bytes)
    static constexpr int CHUNK = 2 * GCHUNK;      // a pair tile's K chunk: 2 n1 rows of 128 B
    static constexpr int TILE = 2 * CHUNK;        // a pair tile [2 n1 rows][K = 128], bf16
    static constexpr int XSLOT = SCALED ? 2 * TILE : TILE;  // x' hi + lo tiles, or x
    static constexpr int NX = SCALED ? 3 : 6;     // shared-memory pair slots
    static constexpr int NR = 2;                  // TMEM regions of a pair's D1/A2 (2 n1 columns)
    static constexpr int ND = kEpiGroups;         // TMEM D2 slots, one per epilogue warpgroup
    static constexpr int A1COLS = 64;             // P2^T: 128 K values of bf16 per lane
    static constexpr int TMEM_COLS = 512;
    static constexpr int OFF_B2 = 0;              // P1^T [n1 rows][K = n1], 128-byte swizzle
    static constexpr int OFF_X = f_align_up(N1 * 128, 1024);
    static constexpr int OFF_BAR = OFF_X + NX * XSLOT;
    static constexpr int CFULL = 0, XFREE = NX, D1FULL = 2 * NX, A2FULL = D1FULL + NR, AFREE = A2FULL + 2 * NR,
                         D2FULL = AFREE + NR, D2FREE = D2FULL + ND, FACT = D2FREE + ND, SETUP = FACT + 1,
                         TEARDOWN = SETUP + 1, NBAR = TEARDOWN + 1;
    static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;  // tmem base, abort flag, the constant 1, maxima
    static constexpr int SMEM = OFF_MISC + 128 + 1024;   // + slack for 1024-byte alignment
    // P1 and P2 arrive by bulk copies into the last NSCR pair slots, which take
    // x tiles only once the factor operands are built from them.
    static constexpr int P1B = N1 * N1 * 2, P2B = N2 * N2 * 2;
    static constexpr int OFF_SP2 = f_align_up(P1B, 1024);
    static constexpr int NSCR = (OFF_SP2 + P2B + XSLOT - 1) / XSLOT;
    static constexpr int OFF_SCR = OFF_X + (NX - NSCR) * XSLOT;
    __host__ __device__ static constexpr uint32_t SLOT_R(int r) { return uint32_t(A1COLS + r * 2 * N1); }
    __host__ __device__ static constexpr uint32_t SLOT_D(int d) { return uint32_t(A1COLS + (2 * NR + d) * N1); }
    static_assert(N1 == 64, "this kernel is built for n1 = 64");
    static_assert(N2 == 64 || N2 == 128, "stage 1 needs K = H * n2 = 128");
    static_assert(A1COLS + (2 * NR + ND) * N1 <= TMEM_COLS, "TMEM budget");
    static_assert(NX > NSCR && NX >= 3, "pair slots besides the factor scratch");
    static_assert(OFF_X % 1024 == 0 && XSLOT % 1024 == 0 && GCHUNK % 1024 == 0, "swizzle alignment");
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

// v = hi + lo: hi = v truncated to bf16 (its top 16 bits, a byte permute), lo =
// v - hi (exact in fp32) rounded to bf16, about 16 significant bits in all.
// Returns the two hi values packed (first in the low half) and the two NEGATED
// lo values: hi - v is one mixed bf16/fp32 subtraction per value, and stage 2
// multiplies the lo half by -P1^T (the MMA's negate-B bit).
__device__ __forceinline__ void split_pair_neg(uint32_t v0, uint32_t v1, uint32_t &hi, uint32_t &nlo) {
    hi = __byte_perm(v0, v1, 0x7632);
    float n0, n1;
    asm("{\n\t.reg .b16 h0, h1;\n\tmov.b32 {h0, h1}, %2;\n\t"
        "sub.rn.f32.bf16 %0, h0, %3;\n\tsub.rn.f32.bf16 %1, h1, %4;\n\t}"
        : "=f"(n0), "=f"(n1)
        : "r"(hi), "f"(__uint_as_float(v0)), "f"(__uint_as_float(v1)));
    nlo = pack_bf16x2(n0, n1);
}

// round_half_even(y * inv) as an int, for |y * inv| < 2^22: adding 1.5 * 2^23
// leaves the rounded integer in the low mantissa bits (bit pattern 0x4B400000
// + k); an integer multiply-add with `one` (== 1, read at run time) removes
// the offset beside the floating-point work.
constexpr uint32_t kFMagicBits = 0x4B400000u;  // 1.5 * 2^23
__device__ __forceinline__ int round_code(uint32_t ybits, float inv, int one) {
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
    // Groups of H tokens, dealt round-robin to the CTAs; a CTA takes its groups
    // in pairs (local groups 2p and 2p + 1; an odd count leaves the last pair
    // with one group).
    const int64_t G = (T + C::H - 1) / C::H;
    const int nloc = G > int64_t(blockIdx.x) ? int((G - 1 - blockIdx.x) / gridDim.x) + 1 : 0;
    const int npair = (nloc + 1) / 2;
    auto group_of = [&](int j) -> int64_t { return int64_t(blockIdx.x) + int64_t(j) * gridDim.x; };

    auto bar = [&](int i) -> uint32_t { return sbase + uint32_t(C::OFF_BAR + 8 * i); };
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    float *s_red = reinterpret_cast<float *>(smem + C::OFF_MISC + 16);  // [3 warpgroups][2 buffers][4 warps]
    // Inline bounded wait: a polling try_wait loop without a call; every 64 polls it
    // checks the abort flag and the time limit (about a second).
    auto wait = [&](int b, uint32_t parity, unsigned site) -> bool {
        const uint32_t a = bar(b);
        if (mbar_try_wait(a, parity)) return true;
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t it = 1;; ++it) {
            if (mbar_try_wait(a, parity)) return true;
            if ((it & 63u) == 0) {
                if (*s_abort) return false;
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    atomicOr(err, site);
                    *s_abort = 1;
                    return false;
                }
            }
        }
    };

    if (tid == 0) {
        for (int s = 0; s < C::NX; ++s) {
            mbar_init(bar(C::CFULL + s), SCALED ? kSplitWarps : 1);
            mbar_init(bar(C::XFREE + s), 1);
        }
        for (int r = 0; r < C::NR; ++r) {
            mbar_init(bar(C::D1FULL + r), 1);
            mbar_init(bar(C::A2FULL + 2 * r), kSplitWarps);
            mbar_init(bar(C::A2FULL + 2 * r + 1), kSplitWarps);
            mbar_init(bar(C::AFREE + r), 1);
        }
        for (int d = 0; d < C::ND; ++d) {
            mbar_init(bar(C::D2FULL + d), 1);
            mbar_init(bar(C::D2FREE + d), 4);
        }
        mbar_init(bar(C::FACT), 1);
        mbar_init(bar(C::SETUP), kSetupArrivals);
        mbar_init(bar(C::TEARDOWN), 2);
        *s_abort = 0;
        *reinterpret_cast<int *>(smem + C::OFF_MISC + 8) = 1;  // `one` of round_code
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

    // ---------------- set-up: P2^T into TMEM, P1^T into shared memory ----------------
    if ((warp >= kSplitWarp0 && warp < kSplitWarp0 + 8) || warp >= kEpiWarp0) {
        // (on a timeout the abort flag is up and the operands do not matter)
        wait(C::FACT, 0u, kSiteFProducer);
        const uint16_t *P1s = reinterpret_cast<const uint16_t *>(smem + C::OFF_SCR);
        const uint16_t *P2s = reinterpret_cast<const uint16_t *>(smem + C::OFF_SCR + C::OFF_SP2);
        if (warp >= kEpiWarp0) {
            // B2[i][a] = P1[a][i] (rows i, K = a), 128-byte swizzle: a piece is one
            // row i and eight consecutive a; one 16-byte store each.
            constexpr int kThr = 12 * 32, PIECES = 8 * N1, PER = (PIECES + kThr - 1) / kThr;
            const int st = 32 * (warp - kEpiWarp0) + lane;
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int c = st + u * kThr;
                if (c < PIECES) {
                    const int i = c % N1, a0 = 8 * (c / N1);
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w[e] = uint32_t(P1s[(a0 + 2 * e) * N1 + i]) | (uint32_t(P1s[(a0 + 2 * e + 1) * N1 + i]) << 16);
                    *reinterpret_cast<uint4 *>(smem + C::OFF_B2 + swz128(i, a0)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_proxy_async_smem();  // B2 is read by the tensor cores
        } else {
            // A1 = block-diag P2^T (rows permuted, lane_column) into TMEM columns
            // [0, 64): lane l holds row l, K pairs packed per column; warps 4-7 write
            // K in [0, 64), warps 8-11 K in [64, 128).
            const int l = 32 * (warp & 3) + lane;
            const uint32_t taddr = tmem + (uint32_t(32 * (warp & 3)) << 16);
            const int kc0 = warp < kSplitWarp0 + 4 ? 0 : 2;
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
        if (SCALED) {
            // L2 prefetch of the x the split warps load, PD pairs ahead of the pair
            // whose slot has just been released to them (paced by the same barrier).
            constexpr int PD = 3;
            constexpr int64_t GBYTES = int64_t(C::H) * N1 * N2 * 2;
            auto prefetch_pair = [&](int p) {
                for (int h = 0; h < 2; ++h) {
                    const int j = 2 * p + h;
                    if (j < nloc) {
                        const int64_t g = group_of(j);
                        const int64_t tokens = T - g * C::H < C::H ? T - g * C::H : C::H;
                        prefetch_l2(reinterpret_cast<const unsigned char *>(x) + g * GBYTES,
                                    uint32_t(tokens * N1 * N2 * 2));
                    }
                }
            };
            if (elect_one())
                for (int p = 0; p <= PD; ++p) prefetch_pair(p);
            __syncwarp();
            Ring rx;
            for (int p = 0; p + PD + 1 < npair; ++p, rx.next(C::NX)) {
                if (!__all_sync(0xffffffffu, wait(C::XFREE + rx.idx, rx.phase ^ 1u, kSiteFProducer))) break;
                if (elect_one()) prefetch_pair(p + PD + 1);
                __syncwarp();
            }
        } else {
            bool setup_seen = false;
            Ring rx;
            int issued = 0;
            for (int p = 0; p < npair; ++p, rx.next(C::NX)) {
                if (!setup_seen && p == C::NX - C::NSCR) {
                    // the scratch slots are read by the set-up warps before TMA reuses them
                    if (!__all_sync(0xffffffffu, wait(C::SETUP, 0u, kSiteFProducer))) break;
                    setup_seen = true;
                }
                if (!__all_sync(0xffffffffu, wait(C::XFREE + rx.idx, rx.phase ^ 1u, kSiteFProducer))) break;
                if (elect_one()) {
                    const int ng = 2 * p + 1 < nloc ? 2 : 1;
                    mbar_arrive_expect_tx(bar(C::CFULL + rx.idx), uint32_t(ng * 2 * C::GCHUNK));
                    const uint32_t dst = sbase + C::OFF_X + rx.idx * C::XSLOT;
                    for (int h = 0; h < ng; ++h) {
                        const int64_t g = group_of(2 * p + h);
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            const int xc = (N2 == 128) ? 64 * c : 0;
                            const int64_t row = (N2 == 128) ? g * N1 : (2 * g + c) * N1;
                            tma_load_2d(dst + c * C::CHUNK + h * C::GCHUNK, &tmap_x, xc, int(row),
                                        bar(C::CFULL + rx.idx));
                        }
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
        // ---------------- MMA issue: warp 1 stage 1 (pairs), warp 3 stage 2 (groups) ----------------
        // Stage 1 of pair p writes TMEM region p % 2 (N = 2 n1: both groups in one
        // MMA); it reuses the region only after stage 2 of pair p - 2 completed
        // (AFREE).  With two regions the tensor pipe then runs, in steady state,
        // stage 1 of two pairs, stage 2 of the two pairs before them, and so on:
        // no stage-1 MMA directly follows the stage-2 MMAs it waits for.  Two issuers,
        // so that one stage's barrier waits and commits overlap the other stage's
        // MMAs.  One elected lane of each issues the MMAs and the commits.
        const bool ok0 = __all_sync(0xffffffffu, wait(C::SETUP, 0u, kSiteFMma));
        tc_fence_after();
        if (warp == 1) {
            // the hi tile holds -hi (the split's three-operation form): negate B for it
            constexpr uint32_t idesc = idesc_bf16_f32(128, 2 * N1);
            constexpr uint32_t idesc_neg = idesc | (SCALED ? (1u << 14) : 0u);
            Ring rx;
            for (int p = 0; ok0 && p < npair; ++p, rx.next(C::NX)) {
                const int r = p & 1;
                bool w = wait(C::CFULL + rx.idx, rx.phase, kSiteFMma);
                w = w && wait(C::AFREE + r, (uint32_t(p >> 1) & 1u) ^ 1u, kSiteFMma);
                if (!__all_sync(0xffffffffu, w)) break;
                tc_fence_after();
                const uint32_t d = tmem + C::SLOT_R(r);
                const uint32_t xb = sbase + C::OFF_X + rx.idx * C::XSLOT;
                if (elect_one()) {
#pragma unroll
                    for (int pass = 0; pass < (SCALED ? 2 : 1); ++pass) {
                        const uint32_t bl = sdesc_sw128_lo(xb + pass * C::TILE);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t b = bl + uint32_t(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4);
                            if ((pass | kk) != 0)
                                mma_ts_split<1>(d, tmem + 8 * kk, b, kSdescSw128Hi, pass ? idesc : idesc_neg);
                            else
                                mma_ts_split<0>(d, tmem + 8 * kk, b, kSdescSw128Hi, idesc_neg);
                        }
                    }
                    tc_commit(bar(C::XFREE + rx.idx));  // x slot free once these MMAs have read it
                    tc_commit(bar(C::D1FULL + r));      // D1 of both groups complete
                }
                __syncwarp();
            }
        } else {
            // the A2 lo half holds -lo (split_pair_neg): negate B for the lo pass
            constexpr uint32_t idesc = idesc_bf16_f32(128, N1);
            constexpr uint32_t idesc_neg = idesc | (1u << 14);
            const uint32_t b2l = sdesc_sw128_lo(sbase + C::OFF_B2);
            Ring rd;
            for (int j = 0; ok0 && j < nloc; ++j, rd.next(C::ND)) {
                const int p = j >> 1, h = j & 1, r = p & 1;
                const int ds = int(rd.idx);
                bool w = wait(C::A2FULL + 2 * r + h, uint32_t(p >> 1) & 1u, kSiteFMma);
                w = w && wait(C::D2FREE + ds, rd.phase ^ 1u, kSiteFMma);
                if (!__all_sync(0xffffffffu, w)) break;
                tc_fence_after();
                const uint32_t d = tmem + C::SLOT_D(ds), a2 = tmem + C::SLOT_R(r) + uint32_t(h * N1);
                if (elect_one()) {
#pragma unroll
                    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                        for (int kk = 0; kk < N1 / 16; ++kk) {
                            const uint32_t b = b2l + uint32_t((kk * 32) >> 4);
                            if ((pass | kk) != 0)
                                mma_ts_split<1>(d, a2 + 16 * kk + 8 * pass, b, kSdescSw128Hi, pass ? idesc_neg : idesc);
                            else
                                mma_ts_split<0>(d, a2 + 16 * kk + 8 * pass, b, kSdescSw128Hi, idesc);
                        }
                    tc_commit(bar(C::D2FULL + ds));  // D2 complete
                    if (h == 1 || j + 1 == nloc) tc_commit(bar(C::AFREE + r));  // the pair's region free
                }
                __syncwarp();
            }
        }
        // Every MMA either issuer issued has completed before TMEM is freed.
        if (elect_one()) tc_commit(bar(C::TEARDOWN));
        __syncwarp();
        wait_bounded_err(bar(C::TEARDOWN), 0u, s_abort, kSiteFDrain, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp >= kSplitWarp0 && warp < kSplitWarp0 + kSplitWarps) {
        // ---------------- x' split (cinv) and the D1 -> A2 conversion ----------------
        const int q = warp & 3;                  // TMEM lane quadrant
        const int ck = (warp - kSplitWarp0) >> 2;  // this warp's 16-column chunk of each group
        const uint32_t lane_off = uint32_t(32 * q) << 16;
        // Convert pair p: in each group of the pair, this warp's 16 columns of D1
        // (fp32) become 8 columns of hi pairs then 8 of -lo pairs, in place.
        auto convert = [&](int p) -> bool {
            const int r = p & 1;
            if (!__all_sync(0xffffffffu, wait(C::D1FULL + r, uint32_t(p >> 1) & 1u, kSiteFConvert))) return false;
            tc_fence_after();
            const int ng = 2 * p + 1 < nloc ? 2 : 1;
            for (int h = 0; h < ng; ++h) {
                const uint32_t col = tmem + lane_off + C::SLOT_R(r) + uint32_t(h * N1 + 16 * ck);
                uint32_t v[16], o[16];
                tmem_ld_32x32b_x16(col, v);
                tmem_wait_ld_tie(v);
#pragma unroll
                for (int e = 0; e < 8; ++e) split_pair_neg(v[2 * e], v[2 * e + 1], o[e], o[8 + e]);
                tmem_st_32x32b_x16(col, o);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::A2FULL + 2 * r + h));
            }
            return true;
        };
        if (SCALED) {
            const int t = tid - 32 * kSplitWarp0;  // 0 .. 511
            constexpr int UPT = 2;               // 16-byte units per thread per group (1024 units)
            // Unit e = t + 512 u of a group: 8 consecutive x values at byte 16 e of the
            // group's (contiguous) x, which is row r of B chunk c, 16-byte column k8:
            //   n2 = 128: r = e / 16, c = (e / 8) % 2, k8 = e % 8;
            //   n2 = 64:  c = e / 512 (the token), r = (e / 8) % 64, k8 = e % 8.
            // Its cinv values start at channel 8 (e mod (n / 8)).  Group h of a pair
            // takes rows h n1 .. h n1 + n1 - 1 of the pair tile.  The tile offset of
            // unit u is soff0 + u * SDELTA: unit u = 1 lies 32 rows further down
            // (n2 = 128) or in the second token's chunk (n2 = 64).
            constexpr uint32_t SDELTA = N2 == 128 ? 32 * 128 : C::CHUNK;
            uint32_t soff0;
            uint32_t ch[UPT][4], cl[UPT][4];
            {
                const int r = N2 == 128 ? t / 16 : t / 8, c = N2 == 128 ? (t / 8) % 2 : 0, k8 = t % 8;
                soff0 = uint32_t(c * C::CHUNK + r * 128 + ((k8 ^ (r & 7)) << 4));
                float4 ca[UPT], cb[UPT];
#pragma unroll
                for (int u = 0; u < UPT; ++u) {
                    const int e = t + kSplitThreads * u;
                    const int ch0 = 8 * (e % (N1 * N2 / 8));
                    ca[u] = __ldg(reinterpret_cast<const float4 *>(cinv + ch0));
                    cb[u] = __ldg(reinterpret_cast<const float4 *>(cinv + ch0 + 4));
                }
                // cinv = ch + cl, two bf16 values (RN(cinv) and RN of the rest).  The
                // split then needs three packed bf16 operations per pair of values:
                //   nh = RN(x (-ch)) = -hi,  rest = RN(x ch + nh) = x ch - hi (exact),
                //   lo = RN(x cl + rest);
                // hi + lo is x * cinv to about 2^-14 relative.  The hi tile holds -hi;
                // stage 1 multiplies it with the MMA's negate-B bit.
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
            const unsigned char *xt = reinterpret_cast<const unsigned char *>(x) + 16 * t;
            constexpr int64_t GBYTES = int64_t(C::H) * N1 * N2 * 2;
            auto load_pair = [&](int p, uint4 (&v)[2][UPT]) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int j = 2 * p + h;
                    const int64_t g = group_of(j);
                    const unsigned char *src = xt + g * GBYTES;
#pragma unroll
                    for (int u = 0; u < UPT; ++u) {
                        const bool in = j < nloc && (N2 == 128 || g * C::H + u < T);
                        v[h][u] = in ? ldg_stream(src + 8192 * u) : make_uint4(0u, 0u, 0u, 0u);
                    }
                }
            };
            bool setup_seen = false, ok = true;
            Ring rx;
            // The split runs two pairs ahead of the conversion, so that stage 1 of a
            // pair can be queued behind stage 1 of the pair before it.
            for (int p = 0; ok && p < npair + 2; ++p) {
                if (p < npair) {
                    // The pair's loads go out first (L2 hits: warp 0 prefetched the
                    // groups a few pairs ago); the slot wait overlaps them.  The
                    // split runs two pairs ahead of stage 1, so their latency is off its
                    // path, and no loads are in flight during the conversion.
                    uint4 xv[2][UPT];
                    load_pair(p, xv);
                    if (!setup_seen && rx.idx == uint32_t(C::NX - C::NSCR)) {
                        // the scratch slot is read by the set-up warps before it is overwritten
                        if (!__all_sync(0xffffffffu, wait(C::SETUP, 0u, kSiteFSplit))) break;
                        setup_seen = true;
                    }
                    if (!__all_sync(0xffffffffu, wait(C::XFREE + rx.idx, rx.phase ^ 1u, kSiteFSplit))) break;
                    unsigned char *hib = smem + C::OFF_X + rx.idx * C::XSLOT;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (2 * p + h < nloc) {
                            unsigned char *hi = hib + h * C::GCHUNK;
                            unsigned char *lo = hi + C::TILE;
#pragma unroll
                            for (int u = 0; u < UPT; ++u) {
                                const uint32_t w[4] = {xv[h][u].x, xv[h][u].y, xv[h][u].z, xv[h][u].w};
                                uint32_t oh[4], ol[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    oh[e] = bf16x2_mul(w[e], ch[u][e] ^ 0x80008000u);
                                    const uint32_t rest = bf16x2_fma(w[e], ch[u][e], oh[e]);
                                    ol[e] = bf16x2_fma(w[e], cl[u][e], rest);
                                }
                                *reinterpret_cast<uint4 *>(hi + soff0 + u * SDELTA) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
                                *reinterpret_cast<uint4 *>(lo + soff0 + u * SDELTA) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
                            }
                        }
                    }
                    // the next pair's loads (L2 hits: prefetched PD pairs ago) are in
                    // flight during the conversion below
                    fence_proxy_async_smem();  // the tiles are read by the tensor cores
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(C::CFULL + rx.idx));
                    rx.next(C::NX);
                }
                if (p >= 2) ok = convert(p - 2);
            }
        } else {
            for (int p = 0; p < npair; ++p)
                if (!convert(p)) break;
        }
    } else if (warp >= kEpiWarp0) {
        // ---------------- epilogue: absmax, quantise, pack, store ----------------
        // Warpgroup ew takes the groups j with j % 3 == ew, in D2 slot ew.  A thread
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
        const uint32_t t0 = tmem + (uint32_t(32 * q) << 16) + C::SLOT_D(ew);
        const int bcol = ((32 * q) % N2) / 2 + 2 * g8;
        int it = 0;
        for (int j = ew; j < nloc; j += kEpiGroups, ++it) {
            const int buf = it & 1;
            const bool ok = wait(C::D2FULL + ew, uint32_t(it) & 1u, kSiteFEpilogue);
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
                    if (lane == 0) mbar_arrive(bar(C::D2FREE + ew));  // D2 slot free for stage 2
                }
                if (live) {
#pragma unroll
                    for (int rep = 0; rep < 2; ++rep) {
                        // rows 16 c0 + 8 rep + 2 qq + d: columns 4 g8 + (0, 1) from half 0,
                        // + (2, 3) from half 1; even column in the low nibble
                        int ka[4], kb[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            ka[e] = round_code(ra[4 * rep + e], inv, one);
                            kb[e] = round_code(rb[4 * rep + e], inv, one);
                        }
#pragma unroll
                        for (int d = 0; d < 2; ++d) {
                            const uint32_t wb = pack_s4x2(kb[2 + d], kb[d], 0u);
                            const uint32_t wv = pack_s4x2(ka[2 + d], ka[d], wb);
                            *reinterpret_cast<uint16_t *>(gq + (16 * c0 + 8 * rep + d) * RB) = uint16_t(wv);
                        }
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
    (void)scaled;
    return n1 == 64 && (n2 == 64 || n2 == 128);
}

cudaError_t launch_fused(const LaunchArgs &a) {
    const bool scaled = a.cinv != nullptr;
    if (a.n2 == 128) return scaled ? launch_fused_inst<64, 128, true>(a) : launch_fused_inst<64, 128, false>(a);
    return scaled ? launch_fused_inst<64, 64, true>(a) : launch_fused_inst<64, 64, false>(a);
}

}  // namespace kq
