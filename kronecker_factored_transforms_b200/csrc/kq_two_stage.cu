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
// caller-provided workspace: hi [T][Jp][n1] then lo [T][Jp][n1] with
// Jp = 128 ceil(n2 / 128) rows per token (rows j >= n2 hold zeros).  One
// token's whole Y~ (at most 512 TMEM columns) stays in TMEM until its absmax
// is known, so the codes leave from the stage-2 kernel and neither Y~ nor an
// fp32 intermediate is ever written.  Factors are multiples of 16 up to 256.
//
// Stage 1 (640 threads, persistent over tiles of 64 rows (t, a)): warp 0 TMA
// loads of x tiles [64 rows] x [64 b]; warp 1 TMEM allocation and MMA issue
// (A = P2^T in 128-row slices of j, resident in TMEM; B = the x' hi and lo
// tiles; N = 64); warps 4-11 split x o cinv into hi/lo tiles, cinv tiles
// arriving by TMA with the x tiles (without cinv the MMA reads the loaded x
// tile as is); warps
// 12-19 (two warpgroups) write P2^T into TMEM, then split each accumulator
// into Z^T hi/lo and store it with per-warp TMA tensor stores of [32 j] x
// [16 a] boxes, the warpgroups taking alternate 32-row halves.
//
// Lane order: TMEM lane m of slice s holds j = 128 s + lane_column(m) (within
// each block of 32 lanes, lane 16 f + 8 s' + g holds column 4 g + 2 f + s'),
// and Z^T row m of the slice is stored in that order, so that a stage-2
// epilogue thread reading 16x256b rows holds four consecutive j of an output
// row: two whole bytes of codes.
//
// Stage 2 (384 threads, persistent over tokens): warp 0 TMA loads of Z^T hi/lo
// tiles [128 j] x [64 a]; warp 1 TMEM allocation and MMA issue (A = the Z^T
// tiles, B = P1^T resident in shared memory, N = n1), one 128-lane slice of j
// at a time; warps 4-11 the epilogue (two warpgroups, each half of every
// slice's columns; two bytes of codes per thread and output row, no shuffles,
// stored straight to global memory).  Full/empty barriers per slice let the next token's MMAs
// start on a slice as soon as its codes are formed.
//
// Every mbarrier wait is bounded (kq_wait.cuh); a wait that gives up records
// site 512 in the device status word and every role leaves its loop.
#include <mutex>

#include "kq_common.cuh"
#include "kq_internal.h"
#include "kq_tc05_ptx.cuh"
#include "kq_tile.cuh"
#include "kq_wait.cuh"

namespace kq {
namespace {

using namespace tc;

enum : unsigned { kSiteTwoStage = 512u };

constexpr int kMaxFactor = 256;
constexpr int RT = 128;                 // TMEM lanes: one slice of j
constexpr int KCH = 64;                 // K elements per chunk: one 128-byte swizzle row of bf16
constexpr int TILE = RT * KCH * 2;      // 16 KB: one bf16 tile [128][64]

__host__ __device__ constexpr int slices(int n2) { return (n2 + RT - 1) / RT; }

// 16 lanes x 256 bits, 8 columns: thread t gets lane t/4 in regs 0, 1 and lane
// t/4 + 8 in regs 2, 3, columns 2 (t % 4) and 2 (t % 4) + 1.
__device__ __forceinline__ void tmem_ld_16x256b_x1(uint32_t taddr, uint32_t (&r)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}

// One run of up to 32 columns (cnt, a multiple of 8) of both 16-lane halves of a
// warp's 32 lanes, in the 16x256b layout: ra[u] from lanes base + {g, g + 8},
// rb[u] from lanes base + 16 + {g, g + 8}, columns 8 u + 2 (lane % 4) + {0, 1}.
// Whole runs of 32 take one .x4 load per half; shorter ones .x1 loads.
__device__ __forceinline__ void load_run(uint32_t taddr, int cnt, uint32_t (&ra)[4][4], uint32_t (&rb)[4][4]) {
    if (cnt == 32) {
        tmem_ld_16x256b_x4(taddr, *reinterpret_cast<uint32_t(*)[16]>(&ra[0][0]));
        tmem_ld_16x256b_x4(taddr + (16u << 16), *reinterpret_cast<uint32_t(*)[16]>(&rb[0][0]));
    } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (8 * u < cnt) {
                tmem_ld_16x256b_x1(taddr + uint32_t(8 * u), ra[u]);
                tmem_ld_16x256b_x1(taddr + (16u << 16) + uint32_t(8 * u), rb[u]);
            }
    }
    tmem_wait_ld();
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
// Stage 1: Z^T hi/lo = split(P2^T X~'^T)
// ============================================================================
constexpr int R1 = 64;                                     // rows (t, a) per tile: MMA N
constexpr int XT = R1 * KCH * 2;                           // 8 KB: one x tile [64][64]
constexpr int S1_THREADS = 640;
constexpr int S1_NX = 4;                                   // loaded x stages
constexpr int S1_NS = 4;                                   // hi/lo stages
constexpr int SBOX = 32 * 16 * 2;                          // 1 KB: one store box [32 j][16 a]
constexpr int SG = 4 * SBOX;                               // 4 KB: a warp's hi and lo boxes of 32 rows
constexpr int CT = R1 * KCH * 4;                           // 16 KB: the cinv tile of an x tile [64][64] fp32
constexpr int S1_OFF_C = S1_NX * XT;                       // 32 KB: cinv stages
constexpr int S1_OFF_S = S1_OFF_C + S1_NX * CT;            // 96 KB
constexpr int S1_OFF_STG = S1_OFF_S + S1_NS * 2 * XT;      // 160 KB: two staging buffers per epilogue warp
constexpr int S1_OFF_BAR = S1_OFF_STG + 8 * 2 * SG;        // 224 KB
constexpr int B1_XFULL = 0, B1_XEMPTY = S1_NX, B1_SFULL = 2 * S1_NX, B1_SEMPTY = 2 * S1_NX + S1_NS,
              B1_DFULL = 2 * S1_NX + 2 * S1_NS, B1_DEMPTY = B1_DFULL + 2, B1_DONE = B1_DEMPTY + 2,
              B1_COUNT = B1_DONE + 1;
constexpr int S1_OFF_MISC = S1_OFF_BAR + 8 * B1_COUNT;     // TMEM base, abort flag
constexpr int S1_SMEM = S1_OFF_MISC + 16 + 1024;           // + slack for 1024-byte alignment
constexpr uint32_t S1_TMEM_COLS = 512;
constexpr uint32_t S1_DCOL = 256;                          // A1 slices at 0 and 128; D1 [2 buffers][2 slices][64]
static_assert(S1_SMEM <= 227 * 1024, "shared memory budget");
static_assert(S1_OFF_BAR >= kMaxFactor * kMaxFactor * 2, "P2 staging at start fits before the barriers");

template <bool SCALED>
__global__ void __launch_bounds__(S1_THREADS, 1)
    kq_two_stage_s1_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                           const __grid_constant__ CUtensorMap tmap_shi, const __grid_constant__ CUtensorMap tmap_slo,
                           const uint16_t *__restrict__ P2, int64_t T, int n1, int n2, unsigned int *err) {
    extern __shared__ __align__(1024) unsigned char s1_raw[];
    const uint32_t raw_addr = smem_u32(s1_raw);
    const uint32_t sbase = align1024(raw_addr);
    unsigned char *smem = s1_raw + (sbase - raw_addr);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int J = slices(n2), Jp = RT * J;
    const int rows = int(T * n1);                 // < 2^31 (checked by the entry)
    const int ntiles = (rows + R1 - 1) / R1;
    const int KC = (n2 + KCH - 1) / KCH;          // K chunks per tile
    const int first = int(blockIdx.x), stride = int(gridDim.x);
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
            mbar_init(bar(B1_DEMPTY + b), 8);  // one arrive per epilogue warp
        }
        mbar_init(bar(B1_DONE), 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_x);
        if (SCALED) prefetch_tensormap(&tmap_c);
        prefetch_tensormap(&tmap_shi);
        prefetch_tensormap(&tmap_slo);
    }
    if (warp == 1) {
        tmem_alloc(sbase + S1_OFF_MISC, S1_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + S1_OFF_MISC);
    // The next launch (stage 2) may be scheduled once every CTA holds its SM and
    // its TMEM; it touches global memory only after this grid completes.
    griddep_launch_dependents();
    // on-chip state only above; global reads and writes after the previous kernel
    griddep_wait();

    // P2 into shared memory first (row-major, the pipeline buffers are not in
    // use yet): 16-byte loads, eight per thread in flight.
    {
        const int units = n2 * n2 / 8;
        for (int u0 = tid; u0 < units; u0 += 8 * S1_THREADS) {
            uint4 v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int u = u0 + q * S1_THREADS;
                if (u < units) v[q] = __ldg(reinterpret_cast<const uint4 *>(P2) + u);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int u = u0 + q * S1_THREADS;
                if (u < units) *reinterpret_cast<uint4 *>(smem + 16 * u) = v[q];
            }
        }
    }
    __syncthreads();
    if (warp >= 12) {
        // A1 = P2^T into TMEM: slice s at columns [128 s, 128 s + 32 KC); lane m
        // holds row j = 128 s + lane_column(m), K pairs (b, b + 1) packed per
        // column; zero outside n2 (rows j >= n2 give zero accumulators).
        // Warpgroup 12-15 writes slice 0, 16-19 slice 1.
        const uint16_t *P2s = reinterpret_cast<const uint16_t *>(smem);
        const uint32_t lanes = tmem + (uint32_t(32 * (warp & 3)) << 16);
        for (int s = (warp - 12) >> 2; s < J; s += 2) {
            const int jg = RT * s + tile::lane_column(32 * (warp & 3) + lane);
            for (int c16 = 0; c16 < 2 * KC; ++c16) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int b = 32 * c16 + 2 * e;
                    const uint32_t v0 = (jg < n2 && b < n2) ? P2s[b * n2 + jg] : 0u;
                    const uint32_t v1 = (jg < n2 && b + 1 < n2) ? P2s[(b + 1) * n2 + jg] : 0u;
                    w[e] = v0 | (v1 << 16);
                }
                tmem_st_32x32b_x16(lanes + uint32_t(RT * s + 16 * c16), w);
            }
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();  // the staged P2 is read before TMA writes reuse the buffers
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == 0) {
        // ---------------- TMA producer: x tiles [64 rows (t, a)] x [64 b] ----------------
        // (and with cinv its [64 a] x [64 b] tile, as four 16-row boxes: 16
        // consecutive rows stay in one token since n1 is a multiple of 16)
        Ring r;
        int issued = 0;
        bool ok = true;
        for (int tile = first; tile < ntiles && ok; tile += stride)
            for (int kc = 0; kc < KC; ++kc, r.next(S1_NX)) {
                ok = __all_sync(0xffffffffu, wait_bounded_err(bar(B1_XEMPTY + r.idx), r.phase ^ 1u, s_abort,
                                                              kSiteTwoStage, kWaitLimitNs, false, err));
                if (!ok) break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(bar(B1_XFULL + r.idx), SCALED ? XT + CT : XT);
                    tma_load_2d(sbase + uint32_t(r.idx * XT), &tmap_x, kc * KCH, tile * R1, bar(B1_XFULL + r.idx));
                    if (SCALED) {
#pragma unroll
                        for (int b = 0; b < 4; ++b)
                            tma_load_2d(sbase + uint32_t(S1_OFF_C + r.idx * CT + b * (CT / 4)), &tmap_c, kc * KCH,
                                        (tile * R1 + 16 * b) % n1, bar(B1_XFULL + r.idx));
                    }
                }
                __syncwarp();
                ++issued;
            }
        // every load issued has landed before the CTA can exit
        Ring rd;
        for (int i = 0; i < issued; ++i, rd.next(S1_NX))
            if (i + S1_NX >= issued)
                wait_bounded_err(bar(B1_XFULL + rd.idx), rd.phase, s_abort, kSiteTwoStage, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer: D1[s][j][row] = sum_b P2^T[128 s + j][b] x'[row][b] ----------------
        constexpr uint32_t idesc = idesc_bf16_f32(128, R1);
        Ring rs, rd;
        bool ok = true;
        for (int tile = first; tile < ntiles && ok; tile += stride, rd.next(2)) {
            ok = __all_sync(0xffffffffu, wait_bounded_err(bar(B1_DEMPTY + rd.idx), rd.phase ^ 1u, s_abort,
                                                          kSiteTwoStage, kWaitLimitNs, false, err));
            if (!ok) break;
            tc_fence_after();
            for (int kc = 0; kc < KC; ++kc, rs.next(SCALED ? S1_NS : S1_NX)) {
                ok = __all_sync(0xffffffffu, wait_bounded_err(bar((SCALED ? B1_SFULL : B1_XFULL) + rs.idx), rs.phase,
                                                              s_abort, kSiteTwoStage, kWaitLimitNs, false, err));
                if (!ok) break;
                tc_fence_after();
                const uint32_t hi = SCALED ? sbase + uint32_t(S1_OFF_S + rs.idx * 2 * XT) : sbase + uint32_t(rs.idx * XT);
                const uint32_t bh = sdesc_sw128_lo(hi), bl = sdesc_sw128_lo(hi + XT);
                if (elect_one()) {
                    for (int s = 0; s < J; ++s) {
                        const uint32_t d = tmem + S1_DCOL + 128u * rd.idx + uint32_t(R1 * s);
#pragma unroll
                        for (int kk = 0; kk < KCH / 16; ++kk) {
                            const uint32_t a = tmem + uint32_t(RT * s + 32 * kc + 8 * kk);
                            if ((kc | kk) != 0)
                                mma_ts_split<1>(d, a, bh + 2 * kk, kSdescSw128Hi, idesc);
                            else
                                mma_ts_split<0>(d, a, bh + 2 * kk, kSdescSw128Hi, idesc);
                            if (SCALED) mma_ts_split<1>(d, a, bl + 2 * kk, kSdescSw128Hi, idesc);
                        }
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
        // xt / 8 and xt / 8 + 32; the swizzled offset is the same in every tile,
        // and the matching cinv values sit at row r, bytes [32 c, 32 c + 32) of
        // the stage's cinv tile.
        const int xt = tid - 128;
        const int c = xt & 7;
        Ring rx, rs;
        for (int tile = first; tile < ntiles; tile += stride) {
            bool ok = true;
            for (int kc = 0; kc < KC; ++kc, rx.next(S1_NX), rs.next(S1_NS)) {
                ok = wait_bounded_err(bar(B1_XFULL + rx.idx), rx.phase, s_abort, kSiteTwoStage, kWaitLimitNs, false,
                                      err);
                ok = ok && wait_bounded_err(bar(B1_SEMPTY + rs.idx), rs.phase ^ 1u, s_abort, kSiteTwoStage,
                                            kWaitLimitNs, false, err);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                const unsigned char *src = smem + rx.idx * XT;
                const unsigned char *csrc = smem + S1_OFF_C + rx.idx * CT;
                unsigned char *dhi = smem + S1_OFF_S + rs.idx * 2 * XT;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int r = (xt >> 3) + 32 * i;
                    const uint32_t off = uint32_t(r * 128 + ((c ^ (r & 7)) << 4));
                    const uint4 v = *reinterpret_cast<const uint4 *>(src + off);
                    const float4 c0 = *reinterpret_cast<const float4 *>(csrc + r * 256 + 32 * c);
                    const float4 c1 = *reinterpret_cast<const float4 *>(csrc + r * 256 + 32 * c + 16);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                    const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                    uint32_t h[4], l[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        hi_lo_pair(__uint_as_float(w[e] << 16) * cs[2 * e],
                                   __uint_as_float(w[e] & 0xFFFF0000u) * cs[2 * e + 1], h[e], l[e]);
                    *reinterpret_cast<uint4 *>(dhi + off) = make_uint4(h[0], h[1], h[2], h[3]);
                    *reinterpret_cast<uint4 *>(dhi + XT + off) = make_uint4(l[0], l[1], l[2], l[3]);
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
        // ---------------- epilogue: D1 -> Z^T hi/lo boxes -> TMA stores ----------------
        // Thread = TMEM lane = row m of a slice.  Each warp turns its 32 lanes of a
        // 32-row half of the accumulator into two [32 m][16 a] boxes of hi and
        // two of lo (16 consecutive rows stay in one token since n1 is a
        // multiple of 16), staged in its own two shared buffers and stored by
        // its own TMA stores: no barrier between warps.  Warpgroups 12-15 and
        // 16-19 take alternate halves.
        const int ew = (warp - 12) >> 2, q = warp & 3;
        unsigned char *wstg = smem + S1_OFF_STG + (warp - 12) * 2 * SG;
        const uint32_t wsa = sbase + uint32_t(S1_OFF_STG + (warp - 12) * 2 * SG);
        const int sw = (lane >> 2) & 1;  // chunk order that spreads the 16-byte stores over all banks
        Ring rd;
        int sb = 0;
        for (int tile = first; tile < ntiles; tile += stride, rd.next(2)) {
            const bool ok = wait_bounded_err(bar(B1_DFULL + rd.idx), rd.phase, s_abort, kSiteTwoStage, kWaitLimitNs,
                                             false, err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            for (int s = 0; s < J; ++s)
                for (int hf = ew; hf < 2; hf += 2) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem + (uint32_t(32 * q) << 16) + S1_DCOL + 128u * rd.idx +
                                           uint32_t(R1 * s + 32 * hf),
                                       v);
                    tmem_wait_ld();
                    if (s == J - 1) {  // this warp's last read of the buffer
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(B1_DEMPTY + rd.idx));
                    }
                    uint32_t h[16], l[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        hi_lo_pair(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]), h[e], l[e]);
                    if (lane == 0) bulk_wait_read<1>();  // the stores that used this buffer have read it
                    __syncwarp();
                    unsigned char *stg = wstg + sb * SG;
#pragma unroll
                    for (int bx = 0; bx < 2; ++bx) {
                        const uint4 h0 = make_uint4(h[8 * bx], h[8 * bx + 1], h[8 * bx + 2], h[8 * bx + 3]);
                        const uint4 h1 = make_uint4(h[8 * bx + 4], h[8 * bx + 5], h[8 * bx + 6], h[8 * bx + 7]);
                        const uint4 l0 = make_uint4(l[8 * bx], l[8 * bx + 1], l[8 * bx + 2], l[8 * bx + 3]);
                        const uint4 l1 = make_uint4(l[8 * bx + 4], l[8 * bx + 5], l[8 * bx + 6], l[8 * bx + 7]);
                        const uint32_t off = uint32_t(bx * SBOX + lane * 32);
                        const uint32_t o_first = sw ? 16u : 0u, o_second = sw ? 0u : 16u;
                        *reinterpret_cast<uint4 *>(stg + off + o_first) = sw ? h1 : h0;
                        *reinterpret_cast<uint4 *>(stg + 2 * SBOX + off + o_first) = sw ? l1 : l0;
                        *reinterpret_cast<uint4 *>(stg + off + o_second) = sw ? h0 : h1;
                        *reinterpret_cast<uint4 *>(stg + 2 * SBOX + off + o_second) = sw ? l0 : l1;
                    }
                    fence_proxy_async_smem();  // staging visible to the tensor stores
                    __syncwarp();
                    if (lane == 0) {
                        const uint32_t sa = wsa + uint32_t(sb * SG);
#pragma unroll
                        for (int bx = 0; bx < 2; ++bx) {
                            const int R = tile * R1 + 32 * hf + 16 * bx;
                            if (R < rows) {
                                const int t = R / n1, a0 = R - t * n1;
                                const int y = t * Jp + RT * s + 32 * q;
                                tma_store_2d(&tmap_shi, a0, y, sa + uint32_t(bx * SBOX));
                                tma_store_2d(&tmap_slo, a0, y, sa + uint32_t(2 * SBOX + bx * SBOX));
                            }
                        }
                        bulk_commit();
                    }
                    sb ^= 1;
                }
        }
        if (lane == 0) bulk_wait<0>();
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
// from the 1024-aligned base) and its barrier indices.
struct S2Layout {
    int n1, n2, J, AC, NA, NB, dcols;
    int off_b2, off_a, off_bar, off_red, off_misc, smem;
    __host__ __device__ int AFULL(int s) const { return s; }
    __host__ __device__ int AEMPTY(int s) const { return NA + s; }
    __host__ __device__ int DFULL(int b, int s) const { return 2 * NA + b * J + s; }
    __host__ __device__ int DEMPTY(int b, int s) const { return 2 * NA + NB * J + b * J + s; }
    __host__ __device__ int DONE() const { return 2 * NA + 2 * NB * J; }
    __host__ __device__ int nbar() const { return DONE() + 1; }
};

__host__ __device__ inline S2Layout s2_layout(int n1, int n2) {
    S2Layout L{};
    L.n1 = n1;
    L.n2 = n2;
    L.J = slices(n2);
    L.AC = (n1 + KCH - 1) / KCH;
    L.dcols = L.J * n1;
    L.NB = 2 * L.dcols <= 512 ? 2 : 1;
    L.off_b2 = 0;
    const int b2 = L.AC * n1 * 128;                 // P1^T chunks [n1 rows][128 B]
    L.off_a = (b2 + 1023) & ~1023;
    const int fixed = 1024 /* alignment slack */ + L.off_a + 8 * (2 * S2_MAX_NA + 9) + 64 + 16;
    const int na = (S2_SMEM_MAX - fixed) / (2 * TILE);
    L.NA = na > S2_MAX_NA ? S2_MAX_NA : na;
    L.off_bar = L.off_a + L.NA * 2 * TILE;
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
    const int n = n1 * n2, Jp = RT * L.J;
    auto bar = [&](int i) -> uint32_t { return sbase + uint32_t(L.off_bar + 8 * i); };
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + L.off_misc + 4);

    if (tid == 0) {
        for (int s = 0; s < L.NA; ++s) {
            mbar_init(bar(L.AFULL(s)), 1);
            mbar_init(bar(L.AEMPTY(s)), 1);
        }
        for (int b = 0; b < L.NB; ++b)
            for (int s = 0; s < L.J; ++s) {
                mbar_init(bar(L.DFULL(b, s)), 1);
                mbar_init(bar(L.DEMPTY(b, s)), 8);  // one arrive per epilogue warp
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
    // on-chip state only above; the workspace that stage 1 wrote, P1 and the
    // outputs are touched only after the previous kernel (stage 1) has completed
    griddep_wait();
    // B2 = P1^T in 128B-swizzled K-major chunks: row i, K = a; zero for a >= n1.
    // A unit is one row i and eight consecutive a: eight loads (consecutive
    // threads take consecutive i, so each load is coalesced), one 16-byte store
    // (the swizzle spreads consecutive rows over all banks); four units in
    // flight per thread.
    {
        const int units = L.AC * KCH / 8 * n1;
        for (int u0 = tid; u0 < units; u0 += 4 * S2_THREADS) {
            uint32_t w[4][4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int u = u0 + q * S2_THREADS;
                const int i = u % n1, a0 = 8 * (u / n1);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int a = a0 + 2 * e;
                    const uint32_t lo = (u < units && a < n1) ? P1[a * n1 + i] : 0u;
                    const uint32_t hi = (u < units && a + 1 < n1) ? P1[(a + 1) * n1 + i] : 0u;
                    w[q][e] = lo | (hi << 16);
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int u = u0 + q * S2_THREADS;
                if (u < units) {
                    const int i = u % n1, a0 = 8 * (u / n1);
                    *reinterpret_cast<uint4 *>(smem + L.off_b2 + (a0 >> 6) * n1 * 128 + i * 128 +
                                               ((((a0 & 63) >> 3) ^ (i & 7)) << 4)) =
                        make_uint4(w[q][0], w[q][1], w[q][2], w[q][3]);
                }
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + L.off_misc);
    // The next launch may be scheduled once every CTA holds its SM and its TMEM;
    // it touches global memory only after this grid completes.
    griddep_launch_dependents();

    if (warp == 0) {
        // ---------------- TMA producer: Z^T hi/lo tiles [128 j] x [64 a] ----------------
        Ring r;
        int issued = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < T && ok; t += gridDim.x)
            for (int s = 0; s < L.J && ok; ++s)
                for (int ac = 0; ac < L.AC; ++ac, r.next(L.NA)) {
                    ok = __all_sync(0xffffffffu, wait_bounded_err(bar(L.AEMPTY(r.idx)), r.phase ^ 1u, s_abort,
                                                                  kSiteTwoStage, kWaitLimitNs, false, err));
                    if (!ok) break;
                    if (elect_one()) {
                        const uint32_t dst = sbase + uint32_t(L.off_a + r.idx * 2 * TILE);
                        const int y = int(t) * Jp + RT * s;
                        mbar_arrive_expect_tx(bar(L.AFULL(r.idx)), 2 * TILE);
                        tma_load_2d(dst, &tmap_zhi, ac * KCH, y, bar(L.AFULL(r.idx)));
                        tma_load_2d(dst + TILE, &tmap_zlo, ac * KCH, y, bar(L.AFULL(r.idx)));
                    }
                    __syncwarp();
                    ++issued;
                }
        Ring rd;
        for (int i = 0; i < issued; ++i, rd.next(L.NA))
            if (i + L.NA >= issued)
                wait_bounded_err(bar(L.AFULL(rd.idx)), rd.phase, s_abort, kSiteTwoStage, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer: D2[s][j][i] = sum_a Z^T[128 s + j][a] P1^T[i][a] ----------------
        const uint32_t idesc = idesc_bf16_f32(128, n1);
        const uint32_t b2 = sdesc_sw128_lo(sbase + uint32_t(L.off_b2));
        Ring ra, rd;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < T && ok; t += gridDim.x, rd.next(L.NB)) {
            for (int s = 0; s < L.J && ok; ++s) {
                ok = __all_sync(0xffffffffu, wait_bounded_err(bar(L.DEMPTY(rd.idx, s)), rd.phase ^ 1u, s_abort,
                                                              kSiteTwoStage, kWaitLimitNs, false, err));
                if (!ok) break;
                tc_fence_after();
                const uint32_t d = tmem + uint32_t(rd.idx * L.dcols + s * n1);
                for (int ac = 0; ac < L.AC; ++ac, ra.next(L.NA)) {
                    ok = __all_sync(0xffffffffu, wait_bounded_err(bar(L.AFULL(ra.idx)), ra.phase, s_abort,
                                                                  kSiteTwoStage, kWaitLimitNs, false, err));
                    if (!ok) break;
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
                        tc_commit(bar(L.AEMPTY(ra.idx)));
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (elect_one()) tc_commit(bar(L.DFULL(rd.idx, s)));  // this slice of the token is ready
                __syncwarp();
            }
        }
        if (elect_one()) tc_commit(bar(L.DONE()));
        __syncwarp();
        wait_bounded_err(bar(L.DONE()), 0u, s_abort, kSiteTwoStage, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------- epilogue: absmax, codes, packing, one bulk store per token ----------------
        // Warpgroup ew takes columns (i) [ew h, ew h + h) of every slice, h = n1 / 2,
        // in runs of up to 32.  With 16x256b loads of both 16-lane halves of its
        // warp's lanes, thread (g, cp) = (lane / 4, lane % 4) holds lanes
        // 32 q + g + {0, 8, 16, 24}, i.e. (by the lane order stage 1 wrote) the
        // four consecutive columns j = 128 s + 32 q + 4 g + {0, 1, 2, 3}, for the
        // rows i = 8 u + 2 cp + {0, 1} of each run of 8: two bytes of codes each.
        const int ew = (warp - 4) >> 2, q = warp & 3, et = tid - 128;
        const int g = lane >> 2, cp = lane & 3;
        const int h = n1 / 2;
        const int one = *reinterpret_cast<volatile int *>(smem + L.off_misc + 8);
        float *red = reinterpret_cast<float *>(smem + L.off_red);
        Ring rd;
        int par = 0;
        for (int64_t t = blockIdx.x; t < T; t += gridDim.x, rd.next(L.NB), par ^= 1) {
            const uint32_t lanes = tmem + (uint32_t(32 * q) << 16) + uint32_t(rd.idx * L.dcols + ew * h);
            // pass 1: absmax over the valid columns, slice by slice as they complete
            float m = 0.0f;
            bool ok = true;
            for (int s = 0; s < L.J; ++s) {
                ok = ok && wait_bounded_err(bar(L.DFULL(rd.idx, s)), rd.phase, s_abort, kSiteTwoStage, kWaitLimitNs,
                                            false, err);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const bool valid = RT * s + 32 * q + 4 * g < n2;
                for (int c = 0; c < h; c += 32) {
                    const int cnt = h - c < 32 ? h - c : 32;  // a multiple of 8
                    uint32_t ra[4][4], rb[4][4];
                    load_run(lanes + uint32_t(s * n1 + c), cnt, ra, rb);
                    if (valid) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (8 * u < cnt) {
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    m = fmax3(m, fabsf(__uint_as_float(ra[u][e])), fabsf(__uint_as_float(rb[u][e])));
                            }
                    }
                }
            }
            const unsigned mw = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
            if (lane == 0) red[8 * par + (warp - 4)] = __uint_as_float(mw);
            if (named_barrier_any(1, 256, !ok)) break;  // all epilogue warps leave together
            float M = red[8 * par];
#pragma unroll
            for (int w = 1; w < 8; ++w) M = fmaxf(M, red[8 * par + w]);
            const float sc = alpha * M * (1.0f / 7.0f);
            const float inv = sc > 0.0f ? fminf(__fdividef(1.0f, sc), 3.0e38f) : 0.0f;
            if (et == 0) scale_out[t] = sc;
            // pass 2: codes, two bytes (columns 4 g .. 4 g + 3) per row i, stored
            // straight to the token's row of q_out (the eight groups g of a warp
            // fill 16 contiguous bytes of each row)
            uint8_t *qt = q_out + t * (n / 2);
            for (int s = 0; s < L.J; ++s) {
                const int jb = RT * s + 32 * q + 4 * g;
                const bool store = jb < n2;
                for (int c = 0; c < h; c += 32) {
                    const int cnt = h - c < 32 ? h - c : 32;
                    uint32_t ra[4][4], rb[4][4];
                    load_run(lanes + uint32_t(s * n1 + c), cnt, ra, rb);
                    if (c + 32 >= h) {  // this warp's last read of the slice
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(L.DEMPTY(rd.idx, s)));
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (8 * u < cnt) {
#pragma unroll
                            for (int d = 0; d < 2; ++d) {
                                const uint32_t hi = pack_s4x2(round_code_ts(rb[u][2 + d], inv, one),
                                                              round_code_ts(rb[u][d], inv, one), 0u);
                                const uint32_t w = pack_s4x2(round_code_ts(ra[u][2 + d], inv, one),
                                                             round_code_ts(ra[u][d], inv, one), hi);
                                if (store) {
                                    const int i = ew * h + c + 8 * u + 2 * cp + d;
                                    *reinterpret_cast<uint16_t *>(qt + ((i * n2 + jb) >> 1)) = uint16_t(w);
                                }
                            }
                        }
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

CUresult encode_bf16_2d(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                        uint32_t box_rows, CUtensorMapSwizzle swizzle) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) return CUDA_ERROR_NOT_SUPPORTED;
    const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    const cuuint64_t stride[1] = {cuuint64_t(cols * 2)};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, stride, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace

bool two_stage_supports(int n1, int n2) {
    return n1 >= 16 && n2 >= 16 && n1 <= kMaxFactor && n2 <= kMaxFactor && n1 % 16 == 0 && n2 % 16 == 0;
}

uint64_t two_stage_workspace_bytes(int64_t T, int n1, int n2) {
    return uint64_t(T) * uint64_t(n1) * uint64_t(RT * slices(n2)) * 4;
}

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

    const uint64_t zrows = uint64_t(a.T) * uint64_t(RT * slices(a.n2));  // Z^T rows, padded per token
    uint16_t *zhi = static_cast<uint16_t *>(workspace);
    uint16_t *zlo = zhi + zrows * uint64_t(a.n1);
    CUtensorMap tx, tc, shi, slo, lhi, llo;
    if (encode_bf16_2d(&tx, a.x, uint64_t(a.n2), uint64_t(a.T) * a.n1, KCH, R1, CU_TENSOR_MAP_SWIZZLE_128B) !=
            CUDA_SUCCESS ||
        encode_bf16_2d(&shi, zhi, uint64_t(a.n1), zrows, 16, 32, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS ||
        encode_bf16_2d(&slo, zlo, uint64_t(a.n1), zrows, 16, 32, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS ||
        encode_bf16_2d(&lhi, zhi, uint64_t(a.n1), zrows, KCH, RT, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        encode_bf16_2d(&llo, zlo, uint64_t(a.n1), zrows, KCH, RT, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    if (a.cinv) {
        // cinv as [n1 rows][n2 cols] fp32; boxes [16 rows][64 cols], columns past n2 read as zero
        PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
        const cuuint64_t dims[2] = {cuuint64_t(a.n2), cuuint64_t(a.n1)};
        const cuuint64_t stride[1] = {cuuint64_t(a.n2) * 4};
        const cuuint32_t box[2] = {cuuint32_t(KCH), 16u};
        const cuuint32_t estr[2] = {1u, 1u};
        if (!encode || encode(&tc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(a.cinv), dims, stride, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    } else {
        tc = tx;  // unused without cinv
    }

    // stage 1: persistent CTAs over 64-row tiles
    const int64_t ntiles = (a.T * a.n1 + R1 - 1) / R1;
    const int64_t g1 = ntiles < a.num_sms ? ntiles : a.num_sms;
    e = launch_overlapped(a.cinv ? kq_two_stage_s1_kernel<true> : kq_two_stage_s1_kernel<false>, unsigned(g1),
                          S1_THREADS, S1_SMEM, a.stream, tx, tc, shi, slo, a.P2, a.T, a.n1, a.n2, err);
    if (e != cudaSuccess) return e;

    // stage 2: one CTA per SM, tokens strided
    const int64_t g2 = a.T < a.num_sms ? a.T : a.num_sms;
    return launch_overlapped(kq_two_stage_s2_kernel, unsigned(g2), S2_THREADS, size_t(L.smem), a.stream, lhi, llo,
                             a.P1, a.alpha, a.q_out, a.scale_out, a.T, a.n1, a.n2, err);
}

}  // namespace kq
