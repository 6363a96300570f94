// kq_tc05.cu -- persistent fused Kronecker transform + INT4 kernel on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM), pipelined
// per batch of token groups: the kernel kq_transform_quant runs for long
// launches and for every shape but n1 = 64 with n2 in {64, 128} (kq_fused.cu
// takes the short launches of those); plus the device status word that the
// bounded waits report through.
//
// Method (FlatQuant page, "Kronecker factorization" and "The fused kernel"):
// per token Y~ = P1^T X~ P2 with X~ the row-major n1 x n2 view of x * cinv,
// then per-token absmax, s = alpha * max / 7, round-half-even codes clamped
// to [-8, 7], packed two per byte.  Only codes and scales reach HBM.
//
// Layout of the work (one CTA per SM, 24 warps, groups of H = 128 / n2 tokens
// so that the 128 TMEM lanes always hold 128 output columns -- n2 = 16, 32, 48
// padded to 64 and 80, 96, 112 to 128, the padding zero; stage 1 runs on
// batches of GB groups, MMAs up to 128 columns wide):
//   TMEM lane l = (h, m): token h of the group, output column
//   j = lane_column(m) of its n2 columns.  Within each block of 32 lanes the
//   columns are interleaved so that the thread of a 16x256b TMEM load that
//   holds lanes g and g + 8 of both 16-lane halves holds four consecutive
//   columns, i.e. two whole output bytes.
//   stage 1           D1[l][a]  = sum_(h',b) A1[l][(h',b)] * X[a][(h',b)]
//                     A1 = block-diag over h of P2^T (rows permuted as above),
//                     resident in TMEM (in shared memory for n1 > 96
//                     without cinv, and at n1 = 128 with a padded n2);
//                     X  = the group's x tile straight from TMA (K = 128).
//   convert (TMEM)    D1 fp32 -> A2 = hi and -lo bf16, in place, chunk by chunk
//                     (hi = the top 16 bits, -lo = hi - D1 by one mixed
//                     bf16/fp32 subtraction).
//   stage 2 (TS MMA)  D2[l][i]  = sum_a A2[l][a] * P1[a][i]   (A from TMEM; the
//                     -lo pass with the MMA's negate-B bit)
//   epilogue          absmax over the token's lanes, quantise, pack into a
//                     swizzled staging tile, one TMA store per group to HBM
//                     (padded n2: plain rows, one bulk copy per group).
// With cinv, the x' split warps turn each raw x tile into x' = x * cinv
// split into a hi bf16 tile (written over x) and a lo bf16 tile; stage 1
// then accumulates both (for n1 > 64 the lo tile holds -lo and its pass
// negates B).  TMEM holds P2^T, two D1/A2 regions (batches) and one to
// three D2 regions (groups; one, taken in turn by the two epilogue
// warpgroups, with cinv at n1 > 96).
//
// Warp roles: 0 TMA producer | 1 TMEM allocator + stage-1 MMA issuer | 5
// stage-2 MMA issuer | 2-4, 6-7, 20, 22-23 x' split (cinv only) | 8-11 P2^T
// into TMEM, then D1 -> A2 conversion | 12-15 and 16-19 two epilogue
// warpgroups taking alternate groups | 21 idle.  Every mbarrier
// wait is bounded: after about a second it ORs a site bit into
// g_device_error, raises a CTA-wide abort flag and the roles drain and exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kq_common.cuh"
#include "kq_internal.h"
#include "kq_tc05_ptx.cuh"
#include "kq_tile.cuh"
#include "kq_wait.cuh"

namespace kq {

// Nonzero when a bounded wait gave up; each site ORs its own bit.
__device__ unsigned int g_device_error = 0;

// The word's device address, looked up once per device.  Only a successful
// lookup is kept: a failed one (e.g. made during a stream capture) is returned
// to the caller and tried again by the next launch.
cudaError_t device_error_word(int device, unsigned int **word) {
    static std::mutex mu;
    static unsigned int *addr[64];
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[device]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_device_error);
        if (e != cudaSuccess) {
            *word = nullptr;
            return e;
        }
        addr[device] = static_cast<unsigned int *>(p);
    }
    *word = addr[device];
    return cudaSuccess;
}

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
using namespace tile;

constexpr int kTcThreads = 768;  // 24 warps, at most 80 registers per thread
constexpr int kSetupWarps = 15;  // warps 1, 5, 8-19, 21 build the factor operands
constexpr int kXThreads = 256;   // x' split: warps 2-4, 6-7, 20, 22-23

// Warp w runs on scheduler w % 4.  The x' split warps avoid scheduler 1, which
// runs the MMA issuers: their instruction streams are short but on the
// critical path.
// Returns the x' split warp's index in [0, 8), or -1.
__device__ __forceinline__ int xsplit_index(int warp) {
    switch (warp) {
    case 2: return 0;
    case 3: return 1;
    case 4: return 2;
    case 6: return 3;
    case 7: return 4;
    case 20: return 5;
    case 22: return 6;
    case 23: return 7;
    default: return -1;
    }
}
enum : unsigned {
    kSiteProducer = 1u,
    kSiteXSplit = 2u,
    kSiteMma = 4u,
    kSiteConvert = 8u,
    kSiteEpilogue = 16u,
    kSiteDrain = 32u,
    kSiteSelfTest = 256u,
};

// Bounded waits (kq_wait.cuh) reporting through g_device_error.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort,
                                             unsigned site, uint64_t limit_ns, bool ignore_abort) {
    return wait_bounded_err(bar, parity, abort, site, limit_ns, ignore_abort, &g_device_error);
}

__host__ __device__ constexpr int align_up(int v, int a) { return (v + a - 1) / a * a; }
__host__ __device__ constexpr int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int imax(int a, int b) { return a > b ? a : b; }

template <int N1, int N2, bool SCALED>
struct Cfg {
    // The tile layout works on N2P = 64 or 128 columns per token; n2 = 16, 32, 48
    // (80, 96, 112) is padded to 64 (128): the x boxes read zeros past n2, the
    // padded rows and columns of P2^T are zero, and no code is stored for them.
    // (Stacking four or eight tokens of n2 = 32 or 16 in one 128-byte row of a K
    // chunk would waste nothing, but a 128-byte-swizzled TMA box narrower than
    // 128 bytes still takes 128 bytes per row in shared memory, so one box cannot
    // place two tokens side by side.)
    static constexpr int N2P = N2 <= 64 ? 64 : 128;
    static constexpr bool PADDED = N2 != N2P;
    // codes staged in plain row order and stored by one bulk copy per group (rows
    // of n2/2 bytes that are not 32 or 64: no swizzled tensor store for them)
    static constexpr bool PLAIN = PADDED;
    static constexpr int H = 128 / N2P;              // tokens stacked in the TMEM lanes
    // Stage 1 runs on batches of GB groups so that its MMAs are N = GB * n1 wide
    // (up to 128).
    static constexpr int GB = N1 <= 64 ? imin(8, 128 / N1) : 1;
    static constexpr int NS1 = GB * N1;              // stage-1 MMA N
    static constexpr int CHUNK = NS1 * 128;          // one 64-element K chunk of a batch tile
    static constexpr int XTILE = 2 * CHUNK;          // a batch's x tile (K = 128)
    static constexpr int NCH2 = (N1 + 63) / 64;      // K chunks of P1^T
    static constexpr int N1P = align_up(N1, 32);     // TMEM columns of a D2 region
    static constexpr int R1W = align_up(NS1, 32);    // TMEM columns of a D1/A2 region
    // P2^T lives in TMEM (stage 1 reads A from TMEM) when the columns allow it.
    // With cinv and n1 > 96 it does so at the cost of a single D2 region that the
    // two epilogue warpgroups take in turn (SHARED_D2): stage 1's two passes then
    // read only the x' tiles from shared memory, which bounds that case.
    // (not at n1 = 128 with a padded n2, which runs short of registers that way)
    static constexpr bool SHARED_D2 = SCALED && N1 > 96 && !(N1 == 128 && PADDED);
    static constexpr bool A1_TMEM = N1P <= 96 || SHARED_D2;
    static constexpr int A1COLS = A1_TMEM ? 64 : 0;  // 128 K-elements of bf16
    static constexpr int NB2 = SHARED_D2 ? 1 : ((A1COLS + 2 * R1W + 3 * N1P <= 512) ? 3 : 2);  // D2 regions
    // D2FULL barriers: one per D2 region, or with SHARED_D2 one per epilogue warpgroup
    static constexpr int ND2F = SHARED_D2 ? 2 : NB2;
    static constexpr int NB1 = imin(4, (512 - A1COLS - NB2 * N1P) / R1W);        // D1/A2 regions (batches)
    static constexpr int TMEM_USED = A1COLS + NB1 * R1W + NB2 * N1P;
    static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : (TMEM_USED <= 256 ? 256 : 512);
    static constexpr int RB = N2 / 2;                // bytes of one output row (codes)
    // staging bytes per group: a multiple of 1024 (the swizzled TMA-store tile) or,
    // PLAIN, of 128 (rows in plain order, written out by one bulk copy)
    static constexpr int STG = H * N1 * RB;
    static constexpr int OFF_B2 = 0;
    static constexpr int OFF_A1 = align_up(OFF_B2 + NCH2 * N1 * 128, 1024);
    static constexpr int OFF_STG = OFF_A1 + (A1_TMEM ? 0 : 32768);  // 2 epilogues x 2 staging buffers
    static constexpr int OFF_RAW = align_up(OFF_STG + 4 * STG, 1024);
    static constexpr int BUDGET = 222 * 1024 - OFF_RAW - 2048;
    static constexpr int SC = (SCALED && BUDGET >= 10 * XTILE) ? 4 : 2;  // lo-half tile stages (cinv)
    static constexpr int SX = imax(2, imin(8, (BUDGET - (SCALED ? SC * XTILE : 0)) / XTILE));  // raw x stages
    static constexpr int OFF_CONV = OFF_RAW + SX * XTILE;
    static constexpr int NBAR = 2 * SX + 2 * SC + 3 * NB1 + ND2F + NB2 + 2;
    // P1 and P2 arrive first, by bulk copies into the last NSCR x stages, which
    // take x tiles only once the factor operands are built from them.  With cinv
    // and n1 >= 112 only two x stages fit; the scratch then takes the lo-half
    // stages that follow them (SCR_CONV), which the split warps fill only after
    // the factor operands are built.
    static constexpr int P1B = N1 * N1 * 2, P2B = N2 * N2 * 2;
    static constexpr int OFF_SP2 = align_up(P1B, 1024);  // P2 within the scratch
    static constexpr int NSCR = (OFF_SP2 + P2B + XTILE - 1) / XTILE;
    static constexpr bool SCR_CONV = SCALED && SX <= NSCR;
    static constexpr int NSCR_RAW = SCR_CONV ? imax(0, NSCR - SC) : NSCR;  // x stages in the scratch
    static constexpr int OFF_SCR = OFF_RAW + (SX + (SCR_CONV ? SC : 0) - NSCR) * XTILE;
    static constexpr int OFF_BAR = align_up(OFF_CONV + (SCALED ? SC * XTILE : 0), 16);
    static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;  // tmem base, abort flag, the constant 1, 2 x 2 x 4 maxima
    static constexpr int SMEM = OFF_MISC + 80 + 1024;    // + slack for 1024-byte alignment
    // barrier indices
    static constexpr int FULL = 0, EMPTY = SX, CFULL = 2 * SX, CEMPTY = 2 * SX + SC;
    static constexpr int D1FULL = 2 * SX + 2 * SC, A2FULL = D1FULL + NB1, D1EMPTY = A2FULL + NB1;
    static constexpr int D2FULL = D1EMPTY + NB1, D2EMPTY = D2FULL + ND2F, TEARDOWN = D2EMPTY + NB2;
    static constexpr int FACT = TEARDOWN + 1;  // P1 and P2 landed in the scratch
    static_assert(SX > NSCR_RAW && NSCR - NSCR_RAW <= (SCALED ? SC : 0) , "at least one x stage besides the factor scratch");
    static_assert(N2 % 16 == 0 && N2 >= 16 && N2 <= 128, "stage 1 needs K = H * n2 (padded) = 128");
    static_assert(N1 % 16 == 0 && N1 >= 16 && N1 <= 128, "n1 must be a multiple of 16 in [16, 128]");
    static_assert(NS1 % 16 == 0 && NS1 <= 128, "stage-1 MMA width");
    static_assert(NB1 >= 2, "stage-1 regions");
    static_assert(TMEM_USED <= 512, "TMEM budget");
    static_assert((PLAIN ? STG % 128 : STG % 1024) == 0 && OFF_STG % 1024 == 0 && OFF_RAW % 1024 == 0,
                  "swizzle and bulk-copy alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    __host__ __device__ static constexpr uint32_t R1(int b) { return uint32_t(A1COLS + b * R1W); }
    __host__ __device__ static constexpr uint32_t R2(int b) { return uint32_t(A1COLS + NB1 * R1W + b * N1P); }
};

// Threads of the named barrier that ends the setup: the setup warps, the TMA
// producer and, when the factor scratch overlaps the lo-half stages, the split warps.
template <class C>
__host__ __device__ constexpr int setup_barrier_threads() {
    return kSetupWarps * 32 + 32 + (C::SCR_CONV ? kXThreads : 0);
}

// v = hi + lo with hi = v truncated to bf16 (its top 16 bits, a byte permute)
// and lo = v - hi (exact in fp32) rounded to bf16: about 16 significant bits in
// all.  Returns the two hi values packed (first in the low half) and the two
// NEGATED lo values: hi - v is one mixed bf16/fp32 subtraction per value, and
// stage 2 multiplies the lo half by -P1^T (the MMA's negate-B bit).
__device__ __forceinline__ void split_pair_neg(uint32_t v0, uint32_t v1, uint32_t &hi, uint32_t &nlo) {
    hi = __byte_perm(v0, v1, 0x7632);
    float n0, n1;
    asm("{\n\t.reg .b16 h0, h1;\n\tmov.b32 {h0, h1}, %2;\n\t"
        "sub.rn.f32.bf16 %0, h0, %3;\n\tsub.rn.f32.bf16 %1, h1, %4;\n\t}"
        : "=f"(n0), "=f"(n1)
        : "r"(hi), "f"(__uint_as_float(v0)), "f"(__uint_as_float(v1)));
    nlo = pack_bf16x2(n0, n1);
}

// round_half_even(y * inv) as an int, valid for |y * inv| < 2^22 (alpha >= 2^-19):
// adding 1.5 * 2^23 leaves the rounded integer in the low mantissa bits (bit
// pattern 0x4B400000 + k).  The offset is removed by an integer multiply-add
// with `one` (== 1, loaded at run time), which runs beside the floating-point
// work instead of on the logic pipe.  (A packed fp32x2 multiply-add for two
// values at once needs register pairs the TMEM loads do not provide: it measured
// 1-4 % slower over the whole kernel.)
constexpr uint32_t kRoundMagicBits = 0x4B400000u;  // 1.5 * 2^23
__device__ __forceinline__ int round_code(uint32_t ybits, float inv, int one) {
    const uint32_t b = __float_as_uint(fmaf(__uint_as_float(ybits), inv, 12582912.0f));
    int k;
    asm("mad.lo.s32 %0, %1, %2, %3;" : "=r"(k) : "r"(b), "r"(one), "r"(-int(kRoundMagicBits)));
    return k;
}


template <int N1, int N2, bool SCALED>
__global__ void __launch_bounds__(kTcThreads, 1)
    kq_tc05_fused_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_q,
                         const uint16_t *__restrict__ P1,
                         const uint16_t *__restrict__ P2, const float *__restrict__ cinv, float alpha,
                         uint8_t *__restrict__ q_out, float *__restrict__ scale_out, int64_t T) {
    using C = Cfg<N1, N2, SCALED>;
    constexpr int N2P = C::N2P;
    static_assert(C::PLAIN || staging_addresses_match<N1, N2>(), "epilogue staging addresses");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - raw_addr);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Work units: groups of H tokens; batches of GB groups, dealt round-robin to CTAs.
    const int64_t G = (T + C::H - 1) / C::H;
    const int64_t NBt = (G + C::GB - 1) / C::GB;
    const int64_t nb = NBt > int64_t(blockIdx.x) ? (NBt - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

    auto bar = [&](int i) -> uint32_t { return sbase + uint32_t(C::OFF_BAR + 8 * i); };
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    float *s_red = reinterpret_cast<float *>(smem + C::OFF_MISC + 16);

    if (tid == 0) {
        for (int s = 0; s < C::SX; ++s) {
            mbar_init(bar(C::FULL + s), 1);
            mbar_init(bar(C::EMPTY + s), 1);
        }
        for (int c = 0; c < C::SC; ++c) {
            mbar_init(bar(C::CFULL + c), kXThreads);
            mbar_init(bar(C::CEMPTY + c), 1);
        }
        for (int b = 0; b < C::NB1; ++b) {
            mbar_init(bar(C::D1FULL + b), 1);
            mbar_init(bar(C::A2FULL + b), 128);
            mbar_init(bar(C::D1EMPTY + b), 1);
        }
        for (int b = 0; b < C::ND2F; ++b) mbar_init(bar(C::D2FULL + b), 1);
        for (int b = 0; b < C::NB2; ++b) {
            mbar_init(bar(C::D2EMPTY + b), 128);
        }
        mbar_init(bar(C::TEARDOWN), 2);  // one commit from each MMA issuer
        mbar_init(bar(C::FACT), 1);
        *s_abort = 0;
        *reinterpret_cast<int *>(smem + C::OFF_MISC + 8) = 1;  // `one` of round_code
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_x);
        prefetch_tensormap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
        tmem_relinquish();
    }

    // Barriers and the TMEM address are published.  The TMA producer copies P1
    // and P2 into the scratch stages first, then starts the stream of x tiles;
    // the setup warps build the factor operands from the scratch while the x'
    // split warps load cinv.
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    // The next launch on the stream may be scheduled once every CTA of this grid
    // has got here, i.e. holds its SM and its TMEM (so a CTA of that launch can
    // never hold TMEM that this grid still waits for); its CTAs take SMs as this
    // grid's CTAs exit and touch global memory only after this grid completes.
    griddep_launch_dependents();
    // Everything above touched only on-chip state; every global read (x, P1, P2,
    // cinv) and write (codes, scales) comes after the previous kernel on the
    // stream has completed.
    griddep_wait();
    const int setup_idx = warp == 1 ? 0 : warp == 5 ? 1 : (warp >= 8 && warp < 20) ? warp - 6 : warp == 21 ? 14 : -1;
    if (setup_idx >= 0) {
        constexpr int kSetupThreads = kSetupWarps * 32;
        const int st = 32 * setup_idx + lane;
        // P1 and P2 as the producer's first bulk copies put them in the scratch
        // (on a timeout the abort flag is up and the operands do not matter)
        wait_bounded(bar(C::FACT), 0u, s_abort, kSiteProducer, kWaitLimitNs, false);
        const uint16_t *P1s = reinterpret_cast<const uint16_t *>(smem + C::OFF_SCR);
        const uint16_t *P2s = reinterpret_cast<const uint16_t *>(smem + C::OFF_SCR + C::OFF_SP2);
        // B2[i][a] = P1[a][i] (rows i, K = a), 128B-swizzled K-major, zero beyond a = n1.
        {
            // A piece is one row i and eight consecutive a (zero past n1): eight
            // loads (consecutive threads take consecutive i, so each is
            // coalesced) and one 16-byte store (the swizzle spreads consecutive
            // rows over all banks).
            constexpr int PIECES = C::NCH2 * 8 * N1, PER = (PIECES + kSetupThreads - 1) / kSetupThreads;
            uint32_t w[PER][4];
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int c = st + u * kSetupThreads;
                const int i = c % N1, a0 = 8 * (c / N1);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int a = a0 + 2 * e;
                    const uint32_t lo = (c < PIECES && a < N1) ? P1s[a * N1 + i] : 0u;
                    const uint32_t hi = (c < PIECES && a + 1 < N1) ? P1s[(a + 1) * N1 + i] : 0u;
                    w[u][e] = lo | (hi << 16);
                }
            }
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int c = st + u * kSetupThreads;
                if (c < PIECES) {
                    const int i = c % N1, a0 = 8 * (c / N1);
                    *reinterpret_cast<uint4 *>(smem + C::OFF_B2 + (a0 >> 6) * (N1 * 128) + swz128(i, a0 & 63)) =
                        make_uint4(w[u][0], w[u][1], w[u][2], w[u][3]);
                }
            }
        }
        if (!C::A1_TMEM) {
            // A1[(h, m)][(h', b)] = P2[b][lane_column(m)] if h == h' else 0, 128B-swizzled
            // K-major, built like B2: a piece is one row l and eight consecutive k, eight
            // loads (consecutive threads take consecutive l, i.e. 32 distinct columns
            // of one row of P2) and one 16-byte store.
            constexpr int PIECES = 128 * 16, PER = (PIECES + kSetupThreads - 1) / kSetupThreads;
            uint32_t w[PER][4];
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int c = st + u * kSetupThreads;
                const int l = c % 128, k0 = 8 * (c / 128);
                const int h = l / N2P, j = lane_column(l % N2P), hk = k0 / N2P, b0 = k0 % N2P;
                // (eight K values never straddle n2: both are multiples of 8)
                const bool on = c < PIECES && h == hk && j < N2 && b0 < N2;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t lo = on ? P2s[(b0 + 2 * e) * N2 + j] : 0u;
                    const uint32_t hi = on ? P2s[(b0 + 2 * e + 1) * N2 + j] : 0u;
                    w[u][e] = lo | (hi << 16);
                }
            }
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int c = st + u * kSetupThreads;
                if (c < PIECES) {
                    const int l = c % 128, k0 = 8 * (c / 128);
                    *reinterpret_cast<uint4 *>(smem + C::OFF_A1 + (k0 >> 6) * 16384 + swz128(l, k0 & 63)) =
                        make_uint4(w[u][0], w[u][1], w[u][2], w[u][3]);
                }
            }
        }
        fence_proxy_async_smem();
        if (C::A1_TMEM && warp >= 8 && warp < 16) {
            // A1 into TMEM columns [0, 64): lane l holds row l, K pairs packed per
            // column; warps 8-11 write K in [0, 64), warps 12-15 K in [64, 128).
            const int l = 32 * (warp & 3) + lane;
            const uint32_t taddr = tmem + (uint32_t(32 * (warp & 3)) << 16);
            const int kc0 = warp < 12 ? 0 : 2;
            uint32_t w[2][16];  // every load first, then the two stores
#pragma unroll
            for (int kq = 0; kq < 2; ++kq)
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int k = 32 * (kc0 + kq) + 2 * e;
                    w[kq][e] = uint32_t(a1_value<N2, N2P>(P2s, l, k)) |
                               (uint32_t(a1_value<N2, N2P>(P2s, l, k + 1)) << 16);
                }
#pragma unroll
            for (int kq = 0; kq < 2; ++kq) tmem_st_32x32b_x16(taddr + 16 * (kc0 + kq), w[kq]);
            tmem_wait_st();
        }
        fence_proxy_async_smem();  // the scratch is read before TMA writes reuse it
        tc_fence_before();
        named_barrier_sync(3, setup_barrier_threads<C>());  // with the TMA producer (and the split warps)
        tc_fence_after();
    }
    // Buffer hand-offs from the tensor pipe are commits by the MMA warp: stage 1
    // of a batch completing frees its x (and lo) tile and fills its D1 region;
    // stage 2 of a group completing fills a D2 region; stage 2 of a whole batch
    // completing frees its D1/A2 region.
    if (warp == 0) {
        // ---------------- TMA producer: one batch tile per slot ----------------
        // The whole warp runs the loop (converged); one elected lane issues.
        // Its first copies are P1 and P2 (into the scratch stages), ahead of the
        // stream of x tiles; the scratch stages take x tiles only after the
        // setup warps have built the factor operands from them.
        if (elect_one()) {
            mbar_arrive_expect_tx(bar(C::FACT), uint32_t(C::P1B + C::P2B));
            bulk_load(sbase + C::OFF_SCR, P1, uint32_t(C::P1B), bar(C::FACT));
            bulk_load(sbase + C::OFF_SCR + C::OFF_SP2, P2, uint32_t(C::P2B), bar(C::FACT));
        }
        __syncwarp();
        bool setup_seen = false;
        Ring rx;
        uint32_t issued = 0;
        int64_t g0 = int64_t(blockIdx.x) * C::GB;
        const int64_t gstep = int64_t(gridDim.x) * C::GB;
        for (int64_t j = 0; j < nb; ++j, g0 += gstep, rx.next(C::SX)) {
            if (!setup_seen && j == C::SX - C::NSCR_RAW) {
                named_barrier_sync(3, setup_barrier_threads<C>());
                setup_seen = true;
            }
            const bool ok = wait_bounded(bar(C::EMPTY + rx.idx), rx.phase ^ 1u, s_abort, kSiteProducer,
                                         kWaitLimitNs, false);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (elect_one()) {
                mbar_arrive_expect_tx(bar(C::FULL + rx.idx), C::XTILE);
                const uint32_t dst = sbase + C::OFF_RAW + rx.idx * C::XTILE;
#pragma unroll
                for (int gp = 0; gp < C::GB; ++gp) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int64_t g = g0 + gp;
                        const int xc = (N2P == 128) ? 64 * c : 0;  // columns past n2 read as zero
                        const int64_t row = (N2P == 128) ? g * N1 : (2 * g + c) * N1;
                        tma_load_2d(dst + c * C::CHUNK + gp * (N1 * 128), &tmap_x, xc, int(row),
                                    bar(C::FULL + rx.idx));
                    }
                }
            }
            __syncwarp();
            ++issued;
        }
        if (!setup_seen) named_barrier_sync(3, setup_barrier_threads<C>());  // fewer batches than free stages
        // Drain: every load issued has landed (the slots' last phases completed).
        wait_bounded(bar(C::FACT), 0u, s_abort, kSiteDrain, kWaitLimitNs, true);
        Ring rd;
        for (uint32_t i = 0; i < issued; ++i, rd.next(C::SX))
            if (i + C::SX >= issued)
                wait_bounded(bar(C::FULL + rd.idx), rd.phase, s_abort, kSiteDrain, kWaitLimitNs, true);
        __syncwarp();
    } else if (warp == 1 || warp == 5) {
        // ---------------- MMA issuers: warp 1 stage 1, warp 5 stage 2 ----------------
        // Each runs its loop and waits converged (every operand warp-uniform); one
        // elected lane issues the MMAs and commits.  Two issuers keep the latency of
        // one stage's waits and commits off the other's critical path; each commit
        // covers the MMAs its own thread issued.
        constexpr uint32_t idesc1 = idesc_bf16_f32(128, C::NS1);
        constexpr uint32_t idesc2 = idesc_bf16_f32(128, N1);
        // The A2 lo half holds -lo (split_pair_neg): stage 2 negates B on the lo pass.
        constexpr uint32_t idesc2n = idesc2 | (1u << 14);
        const uint32_t b2l = sdesc_sw128_lo(sbase + C::OFF_B2);
        const uint64_t a1d = sdesc_kmajor_sw128(sbase + C::OFF_A1);
        // descriptor start addresses are in 16-byte units in the low bits
        auto koff1 = [](int kk) { return uint32_t(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4); };
        auto koff2 = [](int kk) { return uint32_t(((kk >> 2) * (N1 * 128) + (kk & 3) * 32) >> 4); };
        if (warp == 1) {
            Ring rin, rxs, r1;  // input tiles, raw slots, D1/A2 regions
            for (int64_t j = 0; j < nb; ++j) {
                bool ok = wait_bounded(bar(C::D1EMPTY + r1.idx), r1.phase ^ 1u, s_abort, kSiteMma, kWaitLimitNs,
                                       false);
                uint32_t src, src_lo;
                if (SCALED) {
                    ok = ok && wait_bounded(bar(C::CFULL + rin.idx), rin.phase, s_abort, kSiteMma, kWaitLimitNs,
                                            false);
                    src = sbase + C::OFF_RAW + rxs.idx * C::XTILE;      // hi half, in place of x
                    src_lo = sbase + C::OFF_CONV + rin.idx * C::XTILE;  // lo half
                } else {
                    ok = ok && wait_bounded(bar(C::FULL + rin.idx), rin.phase, s_abort, kSiteMma, kWaitLimitNs,
                                            false);
                    src = src_lo = sbase + C::OFF_RAW + rin.idx * C::XTILE;
                }
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();
                const uint32_t d1 = tmem + C::R1(int(r1.idx));
                const uint32_t bl_hi = sdesc_sw128_lo(src), bl_lo = sdesc_sw128_lo(src_lo);
                if (elect_one()) {
#pragma unroll
                    for (int pass = 0; pass < (SCALED ? 2 : 1); ++pass) {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t b = (pass ? bl_lo : bl_hi) + koff1(kk);
                            // n1 > 64 with cinv: the lo tile holds -lo
                            const uint32_t id1 = (SCALED && N1 > 64 && pass == 1) ? (idesc1 | (1u << 14)) : idesc1;
                            if (C::A1_TMEM) {
                                if ((pass | kk) != 0)
                                    mma_ts_split<1>(d1, tmem + 8 * kk, b, kSdescSw128Hi, id1);
                                else
                                    mma_ts_split<0>(d1, tmem + 8 * kk, b, kSdescSw128Hi, id1);
                            } else {
                                const uint64_t a = a1d + uint64_t(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                                if ((pass | kk) != 0)
                                    mma_ss_split<1>(d1, a, b, kSdescSw128Hi, id1);
                                else
                                    mma_ss_split<0>(d1, a, b, kSdescSw128Hi, id1);
                            }
                        }
                    }
                    tc_commit(bar(C::EMPTY + rxs.idx));  // x (hi) tile slot free
                    if (SCALED) tc_commit(bar(C::CEMPTY + rin.idx));  // lo tile free
                    tc_commit(bar(C::D1FULL + r1.idx));
                }
                __syncwarp();
                rin.next(SCALED ? C::SC : C::SX);
                rxs.next(C::SX);
                r1.next(C::NB1);
            }
        } else {
            Ring r1p, r2;  // D1/A2 regions, D2 regions
            uint32_t li = 0;  // groups issued (SHARED_D2: D2FULL of warpgroup li % 2)
            for (int64_t j = 0; j < nb; ++j) {
                bool ok = wait_bounded(bar(C::A2FULL + r1p.idx), r1p.phase, s_abort, kSiteMma, kWaitLimitNs, false);
                if (!__all_sync(0xffffffffu, ok)) break;
                const uint32_t a2b = tmem + C::R1(int(r1p.idx));
#pragma unroll
                for (int gp = 0; gp < C::GB; ++gp) {
                    ok = __all_sync(0xffffffffu, wait_bounded(bar(C::D2EMPTY + r2.idx), r2.phase ^ 1u, s_abort,
                                                              kSiteMma, kWaitLimitNs, false));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t d2 = tmem + C::R2(int(r2.idx)), a2 = a2b + gp * N1;
                    if (elect_one()) {
#pragma unroll
                        for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                            for (int kk = 0; kk < N1 / 16; ++kk) {
                                if ((pass | kk) != 0)
                                    mma_ts_split<1>(d2, a2 + 16 * kk + 8 * pass, b2l + koff2(kk), kSdescSw128Hi,
                                                    pass ? idesc2n : idesc2);
                                else
                                    mma_ts_split<0>(d2, a2 + 16 * kk + 8 * pass, b2l + koff2(kk), kSdescSw128Hi,
                                                    idesc2);
                            }
                        tc_commit(bar(C::D2FULL + (C::SHARED_D2 ? (li & 1u) : r2.idx)));
                    }
                    __syncwarp();
                    r2.next(C::NB2);
                    ++li;
                }
                if (!ok) break;
                if (elect_one()) tc_commit(bar(C::D1EMPTY + r1p.idx));  // A2 region free
                __syncwarp();
                r1p.next(C::NB1);
            }
        }
        // Every MMA either issuer issued has completed before TMEM is freed.
        if (elect_one()) tc_commit(bar(C::TEARDOWN));
        __syncwarp();
        wait_bounded(bar(C::TEARDOWN), 0u, s_abort, kSiteDrain, kWaitLimitNs, true);
        __syncwarp();
    } else if (xsplit_index(warp) >= 0) {
        // ---------------- x' = x * cinv -> hi / lo bf16 tiles ----------------
        if constexpr (SCALED && N1 > 64) {
            // n1 > 64: 5 to 8 units per thread.  The first UR (3 or 4) units keep their cinv in
            // registers as two bf16 values, cinv = ch + cl (RN(cinv) and RN of the
            // rest): hi = RN(x ch), -lo = RN(-x cl + RN(-x ch + hi)), three packed bf16
            // operations per pair.  The other units read their cinv through the
            // read-only cache (UG x 8 KB per CTA, which stays in L1), form x' = x cinv
            // in fp32 (one packed multiply per pair) and split it into hi = x'
            // truncated to bf16 and -lo = RN(hi - x') (a mixed bf16/fp32 subtraction).
            // Either way the lo tile holds -lo, which stage 1 multiplies with the
            // MMA's negate-B bit; hi + lo is x cinv to about 2^-14 relative.
            const int t = 32 * xsplit_index(warp) + lane;  // 0 .. kXThreads - 1
            constexpr int UPT = 16 * N1 / kXThreads;       // units per thread per token
            // register units, cached units (three register units where four leave the
            // kernel short of registers: n1 = 96, and n1 >= 112 with a padded n2 or stacked tokens)
            constexpr int UR = (N1 == 96 || (C::PADDED && N1 == 112) || (C::H > 1 && N1 >= 112)) ? 3 : 4;
            constexpr int UG = UPT - UR;
            static_assert(C::GB == 1 && UG >= 1 && UG <= 5, "one group per batch for n1 > 64");
            // unit e = t + kXThreads u: row r of chunk c, 16-byte column up of the
            // swizzled tile, i.e. channels r n2 + b0 .. + 7
            // (-1 for a unit of the zero padding past n2)
            auto chan0 = [&](int u) {
                const int e = t + kXThreads * u;
                const int c = e / (8 * N1), rem = e % (8 * N1), r = rem >> 3, up = rem & 7;
                const int b0 = (N2P == 128 ? 64 * c : 0) + 8 * (up ^ (r & 7));  // column within a token
                return (!C::PADDED || b0 < N2) ? r * N2 + b0 : -1;
            };
            auto load_c8 = [&](int ch, float4 &a, float4 &b) {
                if (!C::PADDED || ch >= 0) {
                    a = __ldg(reinterpret_cast<const float4 *>(cinv + ch));
                    b = __ldg(reinterpret_cast<const float4 *>(cinv + ch + 4));
                } else {
                    a = b = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                }
            };
            auto tile_off = [&](int u) {
                const int e = t + kXThreads * u;
                return (e / (8 * N1)) * C::CHUNK + (e % (8 * N1)) * 16;
            };
            uint32_t ch[UR][4], ncl[UR][4];
            {
                float4 ca[UR], cb[UR];  // every load first
#pragma unroll
                for (int u = 0; u < UR; ++u) load_c8(chan0(u), ca[u], cb[u]);
#pragma unroll
                for (int u = 0; u < UR; ++u) {
                    const float cv[8] = {ca[u].x, ca[u].y, ca[u].z, ca[u].w, cb[u].x, cb[u].y, cb[u].z, cb[u].w};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float c0 = cv[2 * p], c1 = cv[2 * p + 1];
                        ch[u][p] = pack_bf16x2(c0, c1);
                        ncl[u][p] = bf16x2_neg(pack_bf16x2(c0 - __uint_as_float(ch[u][p] << 16),
                                                           c1 - __uint_as_float(ch[u][p] & 0xFFFF0000u)));
                    }
                }
            }
            // the lo-half stages may hold the factor scratch until the setup is done
            if constexpr (C::SCR_CONV) named_barrier_sync(3, setup_barrier_threads<C>());
            Ring rx, rc;
            for (int64_t j = 0; j < nb; ++j, rx.next(C::SX), rc.next(C::SC)) {
                bool ok = wait_bounded(bar(C::FULL + rx.idx), rx.phase, s_abort, kSiteXSplit, kWaitLimitNs, false);
                ok = ok && wait_bounded(bar(C::CEMPTY + rc.idx), rc.phase ^ 1u, s_abort, kSiteXSplit,
                                        kWaitLimitNs, false);
                if (!__all_sync(0xffffffffu, ok)) break;  // the warp leaves together
                unsigned char *raw = smem + C::OFF_RAW + rx.idx * C::XTILE;  // x in, hi half out
                unsigned char *lo = smem + C::OFF_CONV + rc.idx * C::XTILE;
                // the first cached units' loads are in flight during the register units
                constexpr int PF = UG < 2 ? UG : 2;
                float4 ga[UG], gb[UG];
#pragma unroll
                for (int g = 0; g < PF; ++g) load_c8(chan0(UR + g), ga[g], gb[g]);
#pragma unroll
                for (int u = 0; u < UR; ++u) {
                    const int off = tile_off(u);
                    const uint4 in = *reinterpret_cast<const uint4 *>(raw + off);
                    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
                    uint32_t oh[4], ol[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        oh[p] = bf16x2_mul(w[p], ch[u][p]);
                        const uint32_t nrest = bf16x2_fma(w[p], bf16x2_neg(ch[u][p]), oh[p]);
                        ol[p] = bf16x2_fma(w[p], ncl[u][p], nrest);
                    }
                    *reinterpret_cast<uint4 *>(raw + off) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
                    *reinterpret_cast<uint4 *>(lo + off) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
                }
#pragma unroll
                for (int g = 0; g < UG; ++g) {
                    if (g + PF < UG) load_c8(chan0(UR + g + PF), ga[g + PF], gb[g + PF]);  // keep PF loads in flight
                    const int off = tile_off(UR + g);
                    const uint4 in = *reinterpret_cast<const uint4 *>(raw + off);
                    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
                    const float cv[8] = {ga[g].x, ga[g].y, ga[g].z, ga[g].w, gb[g].x, gb[g].y, gb[g].z, gb[g].w};
                    uint32_t oh[4], ol[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const uint64_t xp = uint64_t(w[p] << 16) | (uint64_t(w[p] & 0xFFFF0000u) << 32);
                        const uint64_t cp = uint64_t(__float_as_uint(cv[2 * p])) |
                                            (uint64_t(__float_as_uint(cv[2 * p + 1])) << 32);
                        const uint64_t v = f32x2_mul(xp, cp);
                        split_pair_neg(uint32_t(v), uint32_t(v >> 32), oh[p], ol[p]);
                    }
                    *reinterpret_cast<uint4 *>(raw + off) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
                    *reinterpret_cast<uint4 *>(lo + off) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
                }
                fence_proxy_async_smem();
                mbar_arrive(bar(C::CFULL + rc.idx));
            }
        } else if constexpr (SCALED) {
            const int t = 32 * xsplit_index(warp) + lane;  // 0 .. kXThreads - 1
            constexpr int UPT = 16 * N1 / kXThreads;             // units per thread per group
            // thread t handles unit e = t + kXThreads u (u < UPT) of every group of the
            // batch; its cinv values depend only on (u, t).  cinv = ch + cl, two bf16
            // values (RN(cinv) and RN of the rest), so that x' needs only packed bf16
            // arithmetic: hi = RN(x ch), lo = RN(x cl + RN(x ch - hi)).  Each step is one
            // fused rounding; hi + lo is x * cinv to about 2^-14 relative.
            uint32_t ch[UPT][4], cl[UPT][4];
            float4 ca[UPT], cb[UPT];  // every load first
#pragma unroll
            for (int u = 0; u < UPT; ++u) {
                const int e = t + kXThreads * u;
                const int c = e / (8 * N1), rem = e % (8 * N1), r = rem >> 3, up = rem & 7;
                const int b0 = (N2P == 128 ? 64 * c : 0) + 8 * (up ^ (r & 7));  // column within a token
                if (!C::PADDED || b0 < N2) {
                    ca[u] = __ldg(reinterpret_cast<const float4 *>(cinv + r * N2 + b0));
                    cb[u] = __ldg(reinterpret_cast<const float4 *>(cinv + r * N2 + b0 + 4));
                } else {  // zero padding past n2
                    ca[u] = cb[u] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                }
            }
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
            Ring rx, rc;
            for (int64_t j = 0; j < nb; ++j, rx.next(C::SX), rc.next(C::SC)) {
                bool ok = wait_bounded(bar(C::FULL + rx.idx), rx.phase, s_abort, kSiteXSplit, kWaitLimitNs, false);
                ok = ok && wait_bounded(bar(C::CEMPTY + rc.idx), rc.phase ^ 1u, s_abort, kSiteXSplit,
                                        kWaitLimitNs, false);
                if (!__all_sync(0xffffffffu, ok)) break;  // the warp leaves together
                unsigned char *raw = smem + C::OFF_RAW + rx.idx * C::XTILE;  // x in, hi half out
                unsigned char *lo = smem + C::OFF_CONV + rc.idx * C::XTILE;
#pragma unroll
                for (int gp = 0; gp < C::GB; ++gp) {
#pragma unroll
                    for (int u = 0; u < UPT; ++u) {
                        const int e = t + kXThreads * u;
                        const int c = e / (8 * N1), rem = e % (8 * N1);
                        const int off = c * C::CHUNK + gp * (N1 * 128) + rem * 16;
                        const uint4 in = *reinterpret_cast<const uint4 *>(raw + off);
                        const uint32_t w[4] = {in.x, in.y, in.z, in.w};
                        uint32_t oh[4], ol[4];
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            oh[p] = bf16x2_mul(w[p], ch[u][p]);
                            const uint32_t rest = bf16x2_fma(w[p], ch[u][p], bf16x2_neg(oh[p]));
                            ol[p] = bf16x2_fma(w[p], cl[u][p], rest);
                        }
                        *reinterpret_cast<uint4 *>(raw + off) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
                        *reinterpret_cast<uint4 *>(lo + off) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(bar(C::CFULL + rc.idx));
            }
        }
    } else if (warp >= 8 && warp < 12) {
        // ---------------- D1 (fp32) -> A2 (hi, lo bf16) in TMEM ----------------
        const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
        Ring r1;
        for (int64_t j = 0; j < nb; ++j, r1.next(C::NB1)) {
            const bool ok = wait_bounded(bar(C::D1FULL + r1.idx), r1.phase, s_abort, kSiteConvert, kWaitLimitNs,
                                         false);
            // reconverge before the warp-collective TMEM loads; leave together
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t col0 = tmem + lane_off + C::R1(int(r1.idx));
            constexpr int NK = C::NS1 / 16;
            // Chunks of 16 columns, software-pipelined: chunk k + 1 is loaded while
            // chunk k is converted and stored, so only the first load's latency is
            // exposed.  (The wait ties the registers it makes valid, so no use of
            // them is scheduled above it.)
            uint32_t v[2][16];
            tmem_ld_32x32b_x16(col0, v[0]);
            tmem_wait_ld_tie(v[0]);
#pragma unroll
            for (int k = 0; k < NK; ++k) {
                if (k + 1 < NK) tmem_ld_32x32b_x16(col0 + 16 * (k + 1), v[(k + 1) & 1]);
                // chunk of 16 columns -> 8 hi words then 8 -lo words, in place
                uint32_t o[16];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    split_pair_neg(v[k & 1][2 * e], v[k & 1][2 * e + 1], o[e], o[8 + e]);
                tmem_st_32x32b_x16(col0 + 16 * k, o);
                if (k + 1 < NK) tmem_wait_ld_tie(v[(k + 1) & 1]);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::A2FULL + r1.idx));
        }
    } else if (warp >= 12 && warp < 20) {
        // ---------------- epilogue: absmax, quantise, pack, store ----------------
        // Two epilogue warpgroups take alternate groups.  Each thread reads, with
        // 16x256b loads, lanes g8 and g8 + 8 of both 16-lane halves of its warp's
        // 32 lanes: four consecutive output columns (see lane_column), i.e. two
        // whole bytes of each output row it covers, stored as one 16-bit word.
        const int ew = (warp - 12) >> 2;  // which epilogue warpgroup
        const int q = warp & 3;
        const int et = tid - 384 - 128 * ew;
        const uint32_t nbar = 1u + uint32_t(ew);
        const int tok_h = (32 * q) / N2P;
        const int g8 = lane >> 2, qq = lane & 3;
        float *red = s_red + 8 * ew;
        const int one = *reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);
        constexpr int NK = N1 / 16;
        // 32-column TMEM loads; 16-column ones where the split warps hold cinv in
        // registers (n1 > 64), which leaves fewer registers to this role
        constexpr bool WIDE = N1 % 32 == 0 && !(SCALED && N1 > 64);
        const uint32_t ng = uint32_t(nb) * C::GB;
        const uint32_t stg0 = sbase + C::OFF_STG + 2 * ew * C::STG;
        // One thread per warpgroup writes a finished staging tile to HBM with a
        // TMA store (the tensor map clips rows past the last token) or, for a padded
        // n2, whose code rows are not a multiple of 16 bytes, with one bulk copy of
        // the group's valid tokens (contiguous in q_out).
        const bool storer = et == 0;
        auto store_group = [&](int64_t gprev, int sb) {
            if (storer) {
                if constexpr (C::PLAIN) {
                    // the last batch of a CTA can end in groups past the last token
                    // (G not a multiple of GB): nothing of theirs is stored
                    const int64_t tok0 = C::H * gprev, ntok = T - tok0 < C::H ? T - tok0 : C::H;
                    if (ntok > 0)
                        bulk_store(q_out + tok0 * (N1 * C::RB), stg0 + uint32_t(sb) * C::STG,
                                   uint32_t(ntok * N1 * C::RB));
                } else {
                    tma_store_2d(&tmap_q, 0, int(C::H * gprev * N1), stg0 + uint32_t(sb) * C::STG);
                }
                bulk_commit();
            }
        };
        int64_t g_prev = -1;
        int it = 0;
        for (uint32_t gi = uint32_t(ew); gi < ng; gi += 2, ++it) {
            const uint32_t b = gi % C::NB2, ph = (gi / C::NB2) & 1u;
            const uint32_t jb = gi / C::GB, gp = gi % C::GB;
            const int64_t g = (int64_t(blockIdx.x) + int64_t(jb) * gridDim.x) * C::GB + gp;
            const int buf = it & 1;
            const bool ok = wait_bounded(bar(C::D2FULL + (C::SHARED_D2 ? uint32_t(ew) : b)),
                                         C::SHARED_D2 ? uint32_t(it & 1) : ph, s_abort, kSiteEpilogue, kWaitLimitNs,
                                         false);
            // All four warps leave together, so none is left behind in a named barrier.
            const bool warp_ok = __all_sync(0xffffffffu, ok);
            if (named_barrier_any(nbar, 128, !warp_ok)) break;
            __syncwarp();
            tc_fence_after();
            // absmax from a first read (32x32b, thread = lane), 32 columns per load
            float mx4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            {
                const uint32_t lane_off = uint32_t(32 * q) << 16;
                if (WIDE) {
#pragma unroll
                    for (int k0 = 0; k0 < N1; k0 += 32) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(tmem + lane_off + C::R2(int(b)) + k0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            mx4[0] = fmax3(mx4[0], fabsf(__uint_as_float(v[e])), fabsf(__uint_as_float(v[e + 1])));
                            mx4[1] = fmax3(mx4[1], fabsf(__uint_as_float(v[e + 2])), fabsf(__uint_as_float(v[e + 3])));
                            mx4[2] = fmax3(mx4[2], fabsf(__uint_as_float(v[e + 4])), fabsf(__uint_as_float(v[e + 5])));
                            mx4[3] = fmax3(mx4[3], fabsf(__uint_as_float(v[e + 6])), fabsf(__uint_as_float(v[e + 7])));
                        }
                    }
                } else {
#pragma unroll
                    for (int k0 = 0; k0 < NK; ++k0) {
                        uint32_t v[16];
                        tmem_ld_32x32b_x16(tmem + lane_off + C::R2(int(b)) + 16 * k0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; e += 8) {
                            mx4[0] = fmax3(mx4[0], fabsf(__uint_as_float(v[e])), fabsf(__uint_as_float(v[e + 1])));
                            mx4[1] = fmax3(mx4[1], fabsf(__uint_as_float(v[e + 2])), fabsf(__uint_as_float(v[e + 3])));
                            mx4[2] = fmax3(mx4[2], fabsf(__uint_as_float(v[e + 4])), fabsf(__uint_as_float(v[e + 5])));
                            mx4[3] = fmax3(mx4[3], fabsf(__uint_as_float(v[e + 6])), fabsf(__uint_as_float(v[e + 7])));
                        }
                    }
                }
            }
            const float mx = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]);
            // non-negative floats order like their bit patterns: one warp reduction
            const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
            if (lane == 0) red[4 * buf + q] = __uint_as_float(wmax);
            // the store that read this group's staging buffer (two groups back) is done
            if (storer) bulk_wait_read<0>();
            // maxima visible; every thread finished writing its previous group's staging rows
            named_barrier_sync(nbar, 128);
            if (g_prev >= 0) store_group(g_prev, buf ^ 1);
            float m = 0.0f;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if ((32 * w) / N2P == tok_h) m = fmaxf(m, red[4 * buf + w]);
            // s = alpha * max / 7 to within an ulp; codes use y * (1/s): both differ from the
            // exact quotients by a few ulps, far inside the rounding-boundary window
            const float s = alpha * m * (1.0f / 7.0f);
            const float inv = s > 0.0f ? fminf(__fdividef(1.0f, s), 3.0e38f) : 0.0f;
            unsigned char *stg = smem + C::OFF_STG + (2 * ew + buf) * C::STG;
            // this thread's two bytes of every row: columns 4 g8 .. 4 g8 + 3 of the warp's 32.
            // It writes rows row0 + 16 c + 8 rep + 2 qq + d, whose swizzle term of
            // stg_offset is the same for all of them: qq (64-byte rows; row0 is a
            // multiple of 16) or qq >> 1 (32-byte rows).  So every store is one base
            // address plus a constant.
            const int row0 = tok_h * N1, bcol = ((32 * q) % N2P) / 2 + 2 * g8;
            // plain staging: rows in order, and no store for the columns past n2
            const bool keep = !C::PADDED || bcol < C::RB;
            const int swz_t = N2P == 128 ? qq : (qq >> 1);
            unsigned char *tbase = stg + (row0 + 2 * qq) * C::RB +
                                   (C::PLAIN ? bcol : ((((bcol >> 4) ^ swz_t) << 4) | (bcol & 15)));
            const uint32_t t0 = tmem + (uint32_t(32 * q) << 16) + C::R2(int(b));
            constexpr int CB = WIDE ? 2 : 1;  // 16-column chunks per load
#pragma unroll
            for (int c0 = 0; c0 < NK; c0 += CB) {
                // half 0 (lanes 32 q + [0, 16)) and half 1 (lanes 32 q + [16, 32))
                uint32_t ra[8 * CB], rb[8 * CB];
                if (CB == 2) {
                    tmem_ld_16x256b_x4(t0 + 16 * c0, *reinterpret_cast<uint32_t(*)[16]>(ra));
                    tmem_ld_16x256b_x4(t0 + (16u << 16) + 16 * c0, *reinterpret_cast<uint32_t(*)[16]>(rb));
                } else {
                    tmem_ld_16x256b_x2(t0 + 16 * c0, *reinterpret_cast<uint32_t(*)[8]>(ra));
                    tmem_ld_16x256b_x2(t0 + (16u << 16) + 16 * c0, *reinterpret_cast<uint32_t(*)[8]>(rb));
                }
                tmem_wait_ld();
                if (c0 + CB >= NK) {
                    tc_fence_before();
                    mbar_arrive(bar(C::D2EMPTY + b));  // D2 region free for the next stage 2
                }
#pragma unroll
                for (int rep = 0; rep < 2 * CB; ++rep) {
                    // rows i0 + d, i0 = 16 c0 + 8 rep + 2 qq: registers 4 rep + d hold the even
                    // column, 4 rep + 2 + d the odd one, of half 0 (ra) and half 1 (rb)
                    int ka[4], kb[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        ka[e] = round_code(ra[4 * rep + e], inv, one);
                        kb[e] = round_code(rb[4 * rep + e], inv, one);
                    }
#pragma unroll
                    for (int d = 0; d < 2; ++d) {
                        // row i0 + d: columns 4 g8 + (0, 1) from half 0, + (2, 3) from half 1;
                        // byte = even column in the low nibble, odd in the high one
                        const uint32_t wb = pack_s4x2(kb[2 + d], kb[d], 0u);
                        const uint32_t w = pack_s4x2(ka[2 + d], ka[d], wb);
                        if (keep) *reinterpret_cast<uint16_t *>(tbase + (16 * c0 + 8 * rep + d) * C::RB) = uint16_t(w);
                    }
                }
            }
            fence_proxy_async_smem();  // staging writes visible to the TMA store
            const int64_t tok0 = C::H * g;
            if (lane == 0 && (32 * q) % N2P == 0 && tok0 + tok_h < T) scale_out[tok0 + tok_h] = s;
            g_prev = g;
        }
        // the last group's rows: everyone has written them once all pass this barrier
        named_barrier_sync(nbar, 128);
        if (g_prev >= 0) store_group(g_prev, (it - 1) & 1);
        if (storer) bulk_wait<0>();  // staging is read (and written out) before the CTA exits
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

    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap tmap;
    const cuuint32_t estr[2] = {1u, 1u};
    // x as [T n1 rows][n2 columns]; one box = 64 columns (zeros past n2) by n1 rows,
    // a full 128-byte swizzle row per tile row
    const cuuint64_t dims[2] = {cuuint64_t(N2), cuuint64_t(a.T) * N1};
    const cuuint64_t strides[1] = {cuuint64_t(N2) * 2};
    const cuuint32_t box[2] = {64u, cuuint32_t(N1)};
    CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(a.x), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // codes: rows of n2/2 bytes, one box = one group's H * n1 rows, swizzled like the staging tile
    // (plain staging stores its codes by bulk copies instead; the map is then unused)
    CUtensorMap tmap_q = tmap;
    if constexpr (!C::PLAIN) {
        const cuuint64_t qdims[2] = {cuuint64_t(C::RB), cuuint64_t(a.T) * N1};
        const cuuint64_t qstrides[1] = {cuuint64_t(C::RB)};
        const cuuint32_t qbox[2] = {cuuint32_t(C::RB), cuuint32_t(C::H * N1)};
        r = encode(&tmap_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.q_out, qdims, qstrides, qbox, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, N2 == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    const int64_t G = (a.T + C::H - 1) / C::H;
    const int64_t NBt = (G + C::GB - 1) / C::GB;
    const int64_t grid = NBt < a.num_sms ? NBt : a.num_sms;
    // Launched with programmatic stream serialization: when the previous kernel on
    // the stream is another launch of this kernel, this grid's launch and set-up
    // overlap that grid's last CTAs (see griddep_launch_dependents / griddep_wait).
    return launch_overlapped(kern, unsigned(grid), kTcThreads, C::SMEM, a.stream, tmap, tmap_q, a.P1, a.P2, a.cinv,
                             a.alpha, a.q_out, a.scale_out, a.T);
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
    switch (a.n1) {
    case 80: return launch_inst<80, N2, SCALED>(a);
    case 96: return launch_inst<96, N2, SCALED>(a);
    case 112: return launch_inst<112, N2, SCALED>(a);
    case 128: return launch_inst<128, N2, SCALED>(a);
    default: break;
    }
    return cudaErrorNotSupported;
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

bool tc05_supports(int n1, int n2, bool scaled) {
    (void)scaled;
    if (n2 < 16 || n2 > 128 || n2 % 16 != 0) return false;  // n2 = 16, 32, 48, 80, 96, 112 run padded
    return n1 >= 16 && n1 <= 128 && n1 % 16 == 0;
}

cudaError_t launch_tc05(const LaunchArgs &a) {
    if (a.T * int64_t(a.n1) >= (int64_t(1) << 31)) return launch_warp_mma(a);  // TMA row coordinate range
    const bool scaled = a.cinv != nullptr;
    switch (a.n2) {
    case 16: return scaled ? dispatch_n1<16, true>(a) : dispatch_n1<16, false>(a);
    case 32: return scaled ? dispatch_n1<32, true>(a) : dispatch_n1<32, false>(a);
    case 48: return scaled ? dispatch_n1<48, true>(a) : dispatch_n1<48, false>(a);
    case 64: return scaled ? dispatch_n1<64, true>(a) : dispatch_n1<64, false>(a);
    case 80: return scaled ? dispatch_n1<80, true>(a) : dispatch_n1<80, false>(a);
    case 96: return scaled ? dispatch_n1<96, true>(a) : dispatch_n1<96, false>(a);
    case 112: return scaled ? dispatch_n1<112, true>(a) : dispatch_n1<112, false>(a);
    case 128: return scaled ? dispatch_n1<128, true>(a) : dispatch_n1<128, false>(a);
    default: return cudaErrorNotSupported;
    }
}

cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t stream) {
    kq_selftest_wait_kernel<<<1, 32, 0, stream>>>(limit_ns);
    return cudaGetLastError();
}

}  // namespace kq
