// kq_two_stage.cu -- Kronecker transform + INT4 for factors above 128
// (FlatQuant page, "The fused kernel", Figure 8 (c): when the factors are too
// large for one on-chip pass, the transform runs as two stages with the
// intermediate in global memory).
//
// For a token, with X~ the row-major n1 x n2 view of x' = x o cinv:
//   stage 1  Z^T[j][a] = sum_b P2[b][j] X~[a][b]   (all tokens at once: a tall product)
//   stage 2  Y~[i][j]  = sum_a P1[a][i] Z[a][j]    (per token), then the token's
//            absmax, s = alpha max / 7, round-half-even codes clamped to [-8, 7],
//            nibble packing (element 2k in the low nibble of byte k).
//
// The intermediate leaves stage 1 as a hi/lo bf16 pair (Z = hi + lo, about 16
// significant bits, the same split the fused kernel applies on chip) in a
// caller-provided workspace of 4 T n bytes: hi [T][n2][n1] then lo [T][n2][n1].
// One token's whole Y~ (n / 128 TMEM columns, at most 512) stays in TMEM until
// its absmax is known, so the codes leave from the stage-2 kernel and neither
// Y~ nor an fp32 intermediate is ever written.  Factors are multiples of 16 up
// to 256 (n up to 65536).
//
// Stage 1 (512 threads, one 128-wide slice of j per CTA, persistent over row
// tiles of 128 rows (t, a)): warp 0 TMA loads of x tiles [128 rows] x [64 b];
// warp 1 TMEM allocation and MMA issue (A = the slice of P2^T, resident in
// TMEM; B = the x' hi and lo tiles; N = 128); warps 4-11 split x o cinv into
// hi/lo tiles (without cinv the MMA reads the loaded tile as is); warps 12-15
// write P2^T into TMEM, then split each accumulator tile into Z^T hi/lo and
// store it.
//
// Stage 2 (384 threads, persistent over tokens): warp 0 TMA loads of Z^T hi/lo
// tiles [128 j] x [64 a]; warp 1 TMEM allocation and MMA issue (A = the Z^T
// tiles, B = P1^T resident in shared memory, N = n1); warps 4-11 the epilogue
// (two warpgroups, each half of every 128-lane block's columns).
//
// Every mbarrier wait is bounded (kq_wait.cuh); a wait that gives up records
// site 512 in the device status word and every role leaves its loop.
#include <mutex>

#include "kq_common.cuh"
#include "kq_internal.h"
#include "kq_tc05_ptx.cuh"
#include "kq_wait.cuh"

namespace kq {
namespace {

using namespace tc;

enum : unsigned { kSiteTwoStage = 512u };

constexpr int kMaxFactor = 256;
constexpr int RT = 128;                 // rows of a tile (stage 1: rows (t, a); stage 2: lanes j)
constexpr int KCH = 64;                 // K elements per chunk: one 128-byte swizzle row of bf16
constexpr int TILE = RT * KCH * 2;      // 16 KB: one bf16 tile [128][64]

// 32 lanes x 32 bits, 8 columns: thread t <- lane t, registers = columns.
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr));
}

// v = hi + lo for two fp32 values: hi = v truncated to bf16 (its top 16 bits),
// lo = v - hi (exact in fp32) rounded to bf16.  Returns both pairs packed,
// first value in the low half.
__device__ __forceinline__ void hi_lo_pair(float v0, float v1, uint32_t &hi, uint32_t &lo) {
    const uint32_t b0 = __float_as_uint(v0), b1 = __float_as_uint(v1);
    const float r0 = v0 - __uint_as_float(b0 & 0xFFFF0000u), r1 = v1 - __uint_as_float(b1 & 0xFFFF0000u);
    hi = __byte_perm(b0, b1, 0x7632);
    lo = pack_bf16x2(r0, r1);
}

// round_half_even(y * inv) as an int for |y * inv| < 2^22 (alpha >= 2^-19):
// after adding 1.5 * 2^23 the rounded integer sits in the low mantissa bits.
__device__ __forceinline__ int round_code_ts(uint32_t ybits, float inv, int one) {
    const uint32_t b = __float_as_uint(fmaf(__uint_as_float(ybits), inv, 12582912.0f));
    int k;
    asm("mad.lo.s32 %0, %1, %2, %3;" : "=r"(k) : "r"(b), "r"(one), "r"(-0x4B400000));
    return k;
}

__device__ __forceinline__ uint32_t align1024(uint32_t a) { return (a + 1023u) & ~1023u; }

// ============================================================================
// Stage 1: Z^T hi/lo = split(P2^T X~'^T), one 128-wide slice of j per CTA
// ============================================================================
constexpr int S1_THREADS = 512;
constexpr int S1_NX = 4;                                   // loaded x stages
constexpr int S1_NS = 2;                                   // hi/lo stages
constexpr int S1_OFF_S = S1_NX * TILE;                     // 64 KB
constexpr int S1_OFF_BAR = S1_OFF_S + S1_NS * 2 * TILE;    // 128 KB
constexpr int B1_XFULL = 0, B1_XEMPTY = S1_NX, B1_SFULL = 2 * S1_NX, B1_SEMPTY = 2 * S1_NX + S1_NS,
              B1_DFULL = 2 * S1_NX + 2 * S1_NS, B1_DEMPTY = B1_DFULL + 2, B1_DONE = B1_DEMPTY + 2,
              B1_COUNT = B1_DONE + 1;
constexpr int S1_OFF_MISC = S1_OFF_BAR + 8 * B1_COUNT;     // TMEM base, abort flag
constexpr int S1_SMEM = S1_OFF_MISC + 16 + 1024;           // + slack for 1024-byte alignment
constexpr uint32_t S1_TMEM_COLS = 512;
constexpr uint32_t S1_DCOL = 128;                          // D1 buffers at columns 128 and 256
static_assert(S1_SMEM <= 227 * 1024, "shared memory budget");

template <bool SCALED>
__global__ void __launch_bounds__(S1_THREADS, 1)
    kq_two_stage_s1_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint16_t *__restrict__ P2,
                           const float *__restrict__ cinv, uint16_t *__restrict__ zhi,
                           uint16_t *__restrict__ zlo, int64_t T, int n1, int n2, int ctas_per_slice,
                           unsigned int *err) {
    extern __shared__ __align__(1024) unsigned char s1_raw[];
    const uint32_t raw_addr = smem_u32(s1_raw);
    const uint32_t sbase = align1024(raw_addr);
    unsigned char *smem = s1_raw + (sbase - raw_addr);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int jt = int(blockIdx.x) % ((n2 + RT - 1) / RT);     // slice of j
    const int first = int(blockIdx.x) / ((n2 + RT - 1) / RT);  // first row tile
    const int64_t rows = T * n1;
    const int ntiles = int((rows + RT - 1) / RT);
    const int KC = (n2 + KCH - 1) / KCH;                         // K chunks per row tile
    auto bar = [&](int i) -> uint32_t { return sbase + uint32_t(S1_OFF_BAR + 8 * i); };
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + S1_OFF_MISC + 4);

    if (tid == 0) {
        for (int s = 0; s < S1_NX; ++s) {
            mbar_init(bar(B1_XFULL + s), 1);
            mbar_init(bar(B1_XEMPTY + s), SCALED ? 8 : 1);  // split warps, or the MMA commit
        }
        for (int s = 0; s < S1_NS; ++s) {
            mbar_init(bar(B1_SFULL + s), 8);
            mbar_init(bar(B1_SEMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B1_DFULL + b), 1);
            mbar_init(bar(B1_DEMPTY + b), 4);
        }
        mbar_init(bar(B1_DONE), 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_x);
    if (warp == 1) {
        tmem_alloc(sbase + S1_OFF_MISC, S1_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + S1_OFF_MISC);

    if (warp >= 12) {
        // A1 = this CTA's slice of P2^T into TMEM columns [0, KC * 32): lane m holds
        // row j = 128 jt + m, K pairs (b, b + 1) packed per column; zero outside n2.
        const int jg = RT * jt + 32 * (warp & 3) + lane;
        const uint32_t taddr = tmem + (uint32_t(32 * (warp & 3)) << 16);
        for (int c16 = 0; c16 < 2 * KC; ++c16) {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int b = 32 * c16 + 2 * e;
                const uint32_t v0 = (jg < n2 && b < n2) ? P2[b * n2 + jg] : 0u;
                const uint32_t v1 = (jg < n2 && b + 1 < n2) ? P2[(b + 1) * n2 + jg] : 0u;
                w[e] = v0 | (v1 << 16);
            }
            tmem_st_32x32b_x16(taddr + 16 * c16, w);
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == 0) {
        // ---------------- TMA producer: x tiles [128 rows (t, a)] x [64 b] ----------------
        Ring r;
        int issued = 0;
        for (int tile = first; tile < ntiles; tile += ctas_per_slice) {
            bool ok = true;
            for (int kc = 0; kc < KC; ++kc, r.next(S1_NX)) {
                ok = __all_sync(0xffffffffu, wait_bounded_err(bar(B1_XEMPTY + r.idx), r.phase ^ 1u, s_abort,
                                                              kSiteTwoStage, kWaitLimitNs, false, err));
                if (!ok) break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(bar(B1_XFULL + r.idx), TILE);
                    tma_load_2d(sbase + uint32_t(r.idx * TILE), &tmap_x, kc * KCH, tile * RT, bar(B1_XFULL + r.idx));
                }
                __syncwarp();
                ++issued;
            }
            if (!ok) break;
        }
        // every load issued has landed before the CTA can exit
        Ring rd;
        for (int i = 0; i < issued; ++i, rd.next(S1_NX))
            if (i + S1_NX >= issued)
                wait_bounded_err(bar(B1_XFULL + rd.idx), rd.phase, s_abort, kSiteTwoStage, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer: D1[j][row] = sum_b P2^T[j][b] x'[row][b] ----------------
        constexpr uint32_t idesc = idesc_bf16_f32(128, RT);
        Ring rs, rd;
        for (int tile = first; tile < ntiles; tile += ctas_per_slice, rd.next(2)) {
            bool ok = wait_bounded_err(bar(B1_DEMPTY + rd.idx), rd.phase ^ 1u, s_abort, kSiteTwoStage,
                                       kWaitLimitNs, false, err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t d = tmem + S1_DCOL + 128u * rd.idx;
            for (int kc = 0; kc < KC; ++kc, rs.next(SCALED ? S1_NS : S1_NX)) {
                ok = __all_sync(0xffffffffu, wait_bounded_err(bar((SCALED ? B1_SFULL : B1_XFULL) + rs.idx), rs.phase,
                                                              s_abort, kSiteTwoStage, kWaitLimitNs, false, err));
                if (!ok) break;
                tc_fence_after();
                const uint32_t hi = SCALED ? sbase + uint32_t(S1_OFF_S + rs.idx * 2 * TILE)
                                           : sbase + uint32_t(rs.idx * TILE);
                const uint32_t bh = sdesc_sw128_lo(hi), bl = sdesc_sw128_lo(hi + TILE);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < KCH / 16; ++kk) {
                        const uint32_t a = tmem + uint32_t(32 * kc + 8 * kk);
                        if ((kc | kk) != 0)
                            mma_ts_split<1>(d, a, bh + 2 * kk, kSdescSw128Hi, idesc);
                        else
                            mma_ts_split<0>(d, a, bh + 2 * kk, kSdescSw128Hi, idesc);
                        if (SCALED) mma_ts_split<1>(d, a, bl + 2 * kk, kSdescSw128Hi, idesc);
                    }
                    tc_commit(bar((SCALED ? B1_SEMPTY : B1_XEMPTY) + rs.idx));  // stage free once read
                }
                __syncwarp();
            }
            if (!ok) break;
            if (elect_one()) tc_commit(bar(B1_DFULL + rd.idx));
            __syncwarp();
        }
        // DONE completes once every MMA this warp issued has completed
        if (elect_one()) tc_commit(bar(B1_DONE));
        __syncwarp();
        wait_bounded_err(bar(B1_DONE), 0u, s_abort, kSiteTwoStage, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (SCALED && warp >= 4 && warp < 12) {
        // ---------------- x' = x o cinv split into hi/lo bf16 tiles ----------------
        // Thread xt takes 16-byte chunk c = xt % 8 (8 values of b) of rows
        // xt / 8 + 32 i; the swizzled offset is the same in every tile.
        const int xt = tid - 128;
        const int c = xt & 7;
        Ring rx, rs;
        for (int tile = first; tile < ntiles; tile += ctas_per_slice) {
            bool ok = true;
            for (int kc = 0; kc < KC; ++kc, rx.next(S1_NX), rs.next(S1_NS)) {
                ok = wait_bounded_err(bar(B1_XFULL + rx.idx), rx.phase, s_abort, kSiteTwoStage, kWaitLimitNs, false,
                                      err);
                ok = ok && wait_bounded_err(bar(B1_SEMPTY + rs.idx), rs.phase ^ 1u, s_abort, kSiteTwoStage,
                                            kWaitLimitNs, false, err);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                const unsigned char *src = smem + rx.idx * TILE;
                unsigned char *dhi = smem + S1_OFF_S + rs.idx * 2 * TILE;
                const int b = kc * KCH + 8 * c;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = (xt >> 3) + 32 * i;
                    const uint32_t off = uint32_t(r * 128 + ((c ^ (r & 7)) << 4));
                    const uint4 v = *reinterpret_cast<const uint4 *>(src + off);
                    float4 c0 = make_float4(0.f, 0.f, 0.f, 0.f), c1 = c0;
                    if (b < n2) {  // chunks past n2 hold zeros from the load
                        const int a = (tile * RT + r) % n1;
                        const float4 *cp = reinterpret_cast<const float4 *>(cinv + a * n2 + b);
                        c0 = __ldg(cp);
                        c1 = __ldg(cp + 1);
                    }
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                    const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                    uint32_t h[4], l[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        hi_lo_pair(__uint_as_float(w[e] << 16) * cs[2 * e],
                                   __uint_as_float(w[e] & 0xFFFF0000u) * cs[2 * e + 1], h[e], l[e]);
                    *reinterpret_cast<uint4 *>(dhi + off) = make_uint4(h[0], h[1], h[2], h[3]);
                    *reinterpret_cast<uint4 *>(dhi + TILE + off) = make_uint4(l[0], l[1], l[2], l[3]);
                }
                fence_proxy_async_smem();  // tiles visible to the tensor cores
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(bar(B1_XEMPTY + rx.idx));
                    mbar_arrive(bar(B1_SFULL + rs.idx));
                }
            }
            if (!ok) break;
        }
    } else if (warp >= 12) {
        // ---------------- epilogue: D1 -> Z^T hi/lo in the workspace ----------------
        // Thread = TMEM lane = j; each group of 8 consecutive rows of a tile is 8
        // consecutive a of one token (n1 is a multiple of 16), stored as 16 bytes.
        const int q = warp & 3;
        const int jg = RT * jt + 32 * q + lane;
        const bool jvalid = jg < n2;
        Ring rd;
        for (int tile = first; tile < ntiles; tile += ctas_per_slice, rd.next(2)) {
            const bool ok = wait_bounded_err(bar(B1_DFULL + rd.idx), rd.phase, s_abort, kSiteTwoStage,
                                             kWaitLimitNs, false, err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t col0 = tmem + (uint32_t(32 * q) << 16) + S1_DCOL + 128u * rd.idx;
#pragma unroll 1
            for (int cc = 0; cc < RT / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(col0 + 32 * cc, v);
                tmem_wait_ld();
                if (jvalid) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int R0 = tile * RT + 32 * cc + 8 * g;
                        if (R0 < rows) {
                            const int t = R0 / n1;
                            const int a0 = R0 - t * n1;
                            uint32_t h[4], l[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                hi_lo_pair(__uint_as_float(v[8 * g + 2 * e]), __uint_as_float(v[8 * g + 2 * e + 1]),
                                           h[e], l[e]);
                            const int64_t off = (int64_t(t) * n2 + jg) * n1 + a0;
                            *reinterpret_cast<uint4 *>(zhi + off) = make_uint4(h[0], h[1], h[2], h[3]);
                            *reinterpret_cast<uint4 *>(zlo + off) = make_uint4(l[0], l[1], l[2], l[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B1_DEMPTY + rd.idx));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, S1_TMEM_COLS);
    }
}

// ============================================================================
// Stage 2: Y~ = P1^T Z per token, absmax, INT4 codes, packed store
// ============================================================================
constexpr int S2_THREADS = 384;
constexpr int S2_MAX_NA = 4;
constexpr int S2_SMEM_MAX = 227 * 1024;

// Shared-memory carve-up of the stage-2 kernel for one shape (byte offsets
// from the 1024-aligned base).
struct S2Layout {
    int n1, n2, J, AC, NA, NB, dcols;
    int off_b2, off_a, off_stg, off_bar, off_red, off_misc, smem;
    // barriers
    __host__ __device__ int AFULL() const { return 0; }
    __host__ __device__ int AEMPTY() const { return NA; }
    __host__ __device__ int DFULL() const { return 2 * NA; }
    __host__ __device__ int DEMPTY() const { return 2 * NA + NB; }
    __host__ __device__ int DONE() const { return 2 * NA + 2 * NB; }
    __host__ __device__ int nbar() const { return DONE() + 1; }
};

__host__ __device__ inline S2Layout s2_layout(int n1, int n2) {
    S2Layout L{};
    L.n1 = n1;
    L.n2 = n2;
    L.J = (n2 + RT - 1) / RT;
    L.AC = (n1 + KCH - 1) / KCH;
    L.dcols = L.J * n1;
    L.NB = 2 * L.dcols <= 512 ? 2 : 1;
    L.off_b2 = 0;
    const int b2 = L.AC * n1 * 128;                 // P1^T chunks [n1 rows][128 B]
    L.off_a = (b2 + 1023) & ~1023;
    const int stg = n1 * n2 / 2;                    // one token's codes
    const int fixed = 1024 /* alignment slack */ + L.off_a + stg + 8 * (2 * S2_MAX_NA + 5) + 64 + 16;
    int na = (S2_SMEM_MAX - fixed) / (2 * TILE);
    L.NA = na > S2_MAX_NA ? S2_MAX_NA : na;
    L.off_stg = L.off_a + L.NA * 2 * TILE;
    L.off_bar = (L.off_stg + stg + 7) & ~7;
    L.off_red = L.off_bar + 8 * L.nbar();
    L.off_misc = L.off_red + 64;                    // 2 x 8 floats
    L.smem = L.off_misc + 16 + 1024;
    return L;
}

__global__ void __launch_bounds__(S2_THREADS, 1)
    kq_two_stage_s2_kernel(const __grid_constant__ CUtensorMap tmap_zhi, const __grid_constant__ CUtensorMap tmap_zlo,
                           const uint16_t *__restrict__ P1, float alpha, uint8_t *__restrict__ q_out,
                           float *__restrict__ scale_out, int64_t T, int n1, int n2, unsigned int *err) {
    extern __shared__ __align__(1024) unsigned char s2_raw[];
    const uint32_t raw_addr = smem_u32(s2_raw);
    const uint32_t sbase = align1024(raw_addr);
    unsigned char *smem = s2_raw + (sbase - raw_addr);
    const S2Layout L = s2_layout(n1, n2);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = n1 * n2;
    auto bar = [&](int i) -> uint32_t { return sbase + uint32_t(L.off_bar + 8 * i); };
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + L.off_misc + 4);

    if (tid == 0) {
        for (int s = 0; s < L.NA; ++s) {
            mbar_init(bar(L.AFULL() + s), 1);
            mbar_init(bar(L.AEMPTY() + s), 1);
        }
        for (int b = 0; b < L.NB; ++b) {
            mbar_init(bar(L.DFULL() + b), 1);
            mbar_init(bar(L.DEMPTY() + b), 8);  // one arrive per epilogue warp
        }
        mbar_init(bar(L.DONE()), 1);
        *s_abort = 0;
        *reinterpret_cast<int *>(smem + L.off_misc + 8) = 1;  // `one` of the code rounding
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_zhi);
        prefetch_tensormap(&tmap_zlo);
    }
    if (warp == 1) {
        tmem_alloc(sbase + uint32_t(L.off_misc), 512);
        tmem_relinquish();
    }
    // B2 = P1^T in 128B-swizzled K-major chunks: row i, K = a; zero for a >= n1.
    for (int idx = tid; idx < L.AC * KCH * n1; idx += S2_THREADS) {
        const int a = idx / n1, i = idx - a * n1;
        const uint16_t v = a < n1 ? P1[a * n1 + i] : uint16_t(0);
        const int k = a & (KCH - 1);
        *reinterpret_cast<uint16_t *>(smem + L.off_b2 + (a >> 6) * n1 * 128 + i * 128 +
                                      ((((k >> 3) ^ (i & 7)) << 4) | ((k & 7) << 1))) = v;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + L.off_misc);

    if (warp == 0) {
        // ---------------- TMA producer: Z^T hi/lo tiles [128 j] x [64 a] ----------------
        Ring r;
        int issued = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < T && ok; t += gridDim.x)
            for (int jt = 0; jt < L.J && ok; ++jt)
                for (int ac = 0; ac < L.AC; ++ac, r.next(L.NA)) {
                    ok = wait_bounded_err(bar(L.AEMPTY() + r.idx), r.phase ^ 1u, s_abort, kSiteTwoStage,
                                          kWaitLimitNs, false, err);
                    if (!__all_sync(0xffffffffu, ok)) {
                        ok = false;
                        break;
                    }
                    if (elect_one()) {
                        const uint32_t dst = sbase + uint32_t(L.off_a + r.idx * 2 * TILE);
                        const int y = int(t * n2) + RT * jt;
                        mbar_arrive_expect_tx(bar(L.AFULL() + r.idx), 2 * TILE);
                        tma_load_2d(dst, &tmap_zhi, ac * KCH, y, bar(L.AFULL() + r.idx));
                        tma_load_2d(dst + TILE, &tmap_zlo, ac * KCH, y, bar(L.AFULL() + r.idx));
                    }
                    __syncwarp();
                    ++issued;
                }
        Ring rd;
        for (int i = 0; i < issued; ++i, rd.next(L.NA))
            if (i + L.NA >= issued)
                wait_bounded_err(bar(L.AFULL() + rd.idx), rd.phase, s_abort, kSiteTwoStage, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer: D2[j][i] = sum_a Z^T[j][a] P1^T[i][a] ----------------
        const uint32_t idesc = idesc_bf16_f32(128, n1);
        const uint32_t b2 = sdesc_sw128_lo(sbase + uint32_t(L.off_b2));
        Ring ra, rd;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < T && ok; t += gridDim.x, rd.next(L.NB)) {
            ok = wait_bounded_err(bar(L.DEMPTY() + rd.idx), rd.phase ^ 1u, s_abort, kSiteTwoStage, kWaitLimitNs,
                                  false, err);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int jt = 0; jt < L.J && ok; ++jt) {
                const uint32_t d = tmem + uint32_t(rd.idx * L.dcols + jt * n1);
                for (int ac = 0; ac < L.AC; ++ac, ra.next(L.NA)) {
                    ok = wait_bounded_err(bar(L.AFULL() + ra.idx), ra.phase, s_abort, kSiteTwoStage, kWaitLimitNs,
                                          false, err);
                    if (!__all_sync(0xffffffffu, ok)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ah = sdesc_sw128_lo(sbase + uint32_t(L.off_a + ra.idx * 2 * TILE));
                    const uint32_t al = ah + uint32_t(TILE >> 4);
                    const uint32_t bc = b2 + uint32_t((ac * n1 * 128) >> 4);
                    if (elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < KCH / 16; ++kk) {
                            const uint64_t dh = (uint64_t(kSdescSw128Hi) << 32) | (ah + 2 * kk);
                            const uint64_t dl = (uint64_t(kSdescSw128Hi) << 32) | (al + 2 * kk);
                            if ((ac | kk) != 0)
                                mma_ss_split<1>(d, dh, bc + 2 * kk, kSdescSw128Hi, idesc);
                            else
                                mma_ss_split<0>(d, dh, bc + 2 * kk, kSdescSw128Hi, idesc);
                            mma_ss_split<1>(d, dl, bc + 2 * kk, kSdescSw128Hi, idesc);
                        }
                        tc_commit(bar(L.AEMPTY() + ra.idx));
                    }
                    __syncwarp();
                }
            }
            if (!ok) break;
            if (elect_one()) tc_commit(bar(L.DFULL() + rd.idx));
            __syncwarp();
        }
        if (elect_one()) tc_commit(bar(L.DONE()));
        __syncwarp();
        wait_bounded_err(bar(L.DONE()), 0u, s_abort, kSiteTwoStage, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------- epilogue: absmax, codes, packing, one bulk store per token ----------------
        // Thread = TMEM lane = column j of a 128-lane block; warpgroup ew takes
        // columns (i) [ew h, ew h + h) of every block, h = n1 / 2.
        const int ew = (warp - 4) >> 2, q = warp & 3, et = tid - 128;
        const int h = n1 / 2;
        const int one = *reinterpret_cast<volatile int *>(smem + L.off_misc + 8);
        float *red = reinterpret_cast<float *>(smem + L.off_red);
        unsigned char *stg = smem + L.off_stg;
        Ring rd;
        int par = 0;
        for (int64_t t = blockIdx.x; t < T; t += gridDim.x, rd.next(L.NB), par ^= 1) {
            bool ok = wait_bounded_err(bar(L.DFULL() + rd.idx), rd.phase, s_abort, kSiteTwoStage, kWaitLimitNs,
                                       false, err);
            ok = __all_sync(0xffffffffu, ok);
            if (named_barrier_any(3, 256, !ok)) break;  // all epilogue warps leave together
            tc_fence_after();
            const uint32_t lanes = tmem + (uint32_t(32 * q) << 16) + uint32_t(rd.idx * L.dcols + ew * h);
            // pass 1: absmax over the valid lanes
            float m = 0.0f;
            for (int jt = 0; jt < L.J; ++jt) {
                const bool valid = RT * jt + 32 * q + lane < n2;
                for (int c8 = 0; c8 < h; c8 += 8) {
                    uint32_t v[8];
                    tmem_ld_32x32b_x8(lanes + uint32_t(jt * n1 + c8), v);
                    tmem_wait_ld();
                    if (valid) {
#pragma unroll
                        for (int e = 0; e < 8; e += 2)
                            m = fmax3(m, fabsf(__uint_as_float(v[e])), fabsf(__uint_as_float(v[e + 1])));
                    }
                }
            }
            const unsigned mw = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
            if (lane == 0) red[8 * par + (warp - 4)] = __uint_as_float(mw);
            if (et == 0) bulk_wait_read<0>();  // the previous token's codes have left the staging buffer
            named_barrier_sync(1, 256);
            float M = red[8 * par];
#pragma unroll
            for (int w = 1; w < 8; ++w) M = fmaxf(M, red[8 * par + w]);
            const float s = alpha * M * (1.0f / 7.0f);
            const float inv = s > 0.0f ? fminf(__fdividef(1.0f, s), 3.0e38f) : 0.0f;
            if (et == 0) scale_out[t] = s;
            // pass 2: codes; lanes j .. j + 7 gather one 32-bit word of row i
            for (int jt = 0; jt < L.J; ++jt) {
                const int jg = RT * jt + 32 * q + lane;
                const bool store = jg < n2 && (lane & 7) == 0;
                for (int c8 = 0; c8 < h; c8 += 8) {
                    uint32_t v[8];
                    tmem_ld_32x32b_x8(lanes + uint32_t(jt * n1 + c8), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int code = round_code_ts(v[e], inv, one);
                        const int nb = __shfl_xor_sync(0xffffffffu, code, 1);
                        const uint32_t b8 = pack_s4x2(nb, code, 0u);  // even lane: own code low, neighbour high
                        const uint32_t b16 = b8 | (__shfl_xor_sync(0xffffffffu, b8, 2) << 8);
                        const uint32_t b32 = b16 | (__shfl_xor_sync(0xffffffffu, b16, 4) << 16);
                        if (store) {
                            const int i = ew * h + c8 + e;
                            *reinterpret_cast<uint32_t *>(stg + ((i * n2 + jg) >> 1)) = b32;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L.DEMPTY() + rd.idx));
            fence_proxy_async_smem();  // staging writes visible to the bulk copy
            named_barrier_sync(2, 256);
            if (et == 0) {
                bulk_store(q_out + t * (n / 2), sbase + uint32_t(L.off_stg), uint32_t(n / 2));
                bulk_commit();
            }
        }
        if (et == 0) bulk_wait<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

CUresult encode_bf16_2d(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) return CUDA_ERROR_NOT_SUPPORTED;
    const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    const cuuint64_t stride[1] = {cuuint64_t(cols * 2)};
    const cuuint32_t box[2] = {cuuint32_t(KCH), cuuint32_t(RT)};
    const cuuint32_t estr[2] = {1u, 1u};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, stride, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace

bool two_stage_supports(int n1, int n2) {
    return n1 >= 16 && n2 >= 16 && n1 <= kMaxFactor && n2 <= kMaxFactor && n1 % 16 == 0 && n2 % 16 == 0;
}

uint64_t two_stage_workspace_bytes(int64_t T, int n1, int n2) { return uint64_t(T) * uint64_t(n1) * n2 * 4; }

cudaError_t launch_two_stage(const LaunchArgs &a, void *workspace) {
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    if (a.device < 0 || a.device >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[a.device], [&] {
        cudaError_t e = cudaFuncSetAttribute(kq_two_stage_s1_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             S1_SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kq_two_stage_s1_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     S1_SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kq_two_stage_s2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     S2_SMEM_MAX);
        attr_err[a.device] = e;
    });
    if (attr_err[a.device] != cudaSuccess) return attr_err[a.device];
    if (!two_stage_supports(a.n1, a.n2)) return cudaErrorInvalidValue;
    if (a.T == 0) return cudaSuccess;
    const S2Layout L = s2_layout(a.n1, a.n2);
    if (L.NA < 2 || L.smem > S2_SMEM_MAX) return cudaErrorInvalidValue;
    unsigned int *err = nullptr;
    cudaError_t e = device_error_word(a.device, &err);
    if (e != cudaSuccess) return e;

    const int64_t n = int64_t(a.n1) * a.n2;
    uint16_t *zhi = static_cast<uint16_t *>(workspace);
    uint16_t *zlo = zhi + a.T * n;
    CUtensorMap tx, th, tl;
    if (encode_bf16_2d(&tx, a.x, uint64_t(a.n2), uint64_t(a.T) * a.n1) != CUDA_SUCCESS ||
        encode_bf16_2d(&th, zhi, uint64_t(a.n1), uint64_t(a.T) * a.n2) != CUDA_SUCCESS ||
        encode_bf16_2d(&tl, zlo, uint64_t(a.n1), uint64_t(a.T) * a.n2) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    // stage 1: J slices of j, each walked by ctas_per_slice CTAs over the row tiles
    const int J = (a.n2 + RT - 1) / RT;
    const int64_t ntiles = (a.T * a.n1 + RT - 1) / RT;
    int per = a.num_sms / J;
    if (per < 1) per = 1;
    if (per > ntiles) per = int(ntiles);
    if (a.cinv)
        kq_two_stage_s1_kernel<true><<<unsigned(J * per), S1_THREADS, S1_SMEM, a.stream>>>(
            tx, a.P2, a.cinv, zhi, zlo, a.T, a.n1, a.n2, per, err);
    else
        kq_two_stage_s1_kernel<false><<<unsigned(J * per), S1_THREADS, S1_SMEM, a.stream>>>(
            tx, a.P2, nullptr, zhi, zlo, a.T, a.n1, a.n2, per, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    // stage 2: one CTA per SM, tokens strided
    const int64_t g2 = a.T < a.num_sms ? a.T : a.num_sms;
    kq_two_stage_s2_kernel<<<unsigned(g2), S2_THREADS, L.smem, a.stream>>>(th, tl, a.P1, a.alpha, a.q_out,
                                                                           a.scale_out, a.T, a.n1, a.n2, err);
    return cudaGetLastError();
}

}  // namespace kq
