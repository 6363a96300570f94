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
// The rows are independent, so they are processed as slots of 16 rows: TMEM
// lanes hold the output column j of H = 128 / D slots (lane_column order, as in
// the fused transform kernel), D1 columns the rows of the slot.  One batch is 8
// groups of H slots: stage 1 of the transform kernel with N = 128, A = Ph^T
// (block-diagonal over the slots) resident in TMEM, B = the rows' x tile by TMA.
// There is no second factor, so the epilogue reads D1 itself, once: per row
// (one D1 column) the absmax over the slot's lanes -- a local max, xor
// shuffles within the warp and a shared-memory step across the warps of the
// slot -- then codes, 16-bit stores into a swizzled staging tile and one TMA
// store per group.
//
// Warps: 0 TMA producer | 1 TMEM allocator + MMA issuer | 4-7 and 8-11 two
// epilogue warpgroups on alternate batches (they also write Ph^T into TMEM at
// start) | 2-3 idle.  Every mbarrier wait is bounded (kq_wait.cuh).
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

constexpr int R_THREADS = 384;
constexpr int RP = 16;  // rows per slot
enum : unsigned { kSiteRowProducer = 128u, kSiteRowMma = 128u, kSiteRowEpilogue = 128u };

constexpr int align_up_r(int v, int a) { return (v + a - 1) / a * a; }

template <int D>
struct RCfg {
    static constexpr int H = 128 / D;                // slots stacked in the TMEM lanes
    static constexpr int GB = 8;                     // groups per batch: stage-1 N = GB * RP = 128
    static constexpr int NS1 = GB * RP;
    static constexpr int CHUNK = NS1 * 128;          // one 64-element K chunk of a batch tile
    static constexpr int XTILE = 2 * CHUNK;          // 32 KB
    static constexpr int A1COLS = 64;                // Ph^T block-diagonal: 128 K-elements of bf16
    static constexpr int R1W = NS1;                  // D1 region: 128 fp32 columns
    static constexpr int NB1 = (512 - A1COLS) / R1W; // 3
    static constexpr int RB = D / 2;                 // code bytes per row
    static constexpr int STG = H * RP * RB;          // staging bytes per group: 1 KB
    static constexpr int BSTG = GB * STG;            // per batch: 8 KB
    static constexpr int OFF_STG = 0;                // 2 epilogues x 2 batch staging tiles
    static constexpr int OFF_RAW = align_up_r(OFF_STG + 4 * BSTG, 1024);
    static constexpr int SX = 5;                     // x tile stages
    static constexpr int FULL = 0, EMPTY = SX, D1FULL = 2 * SX, D1EMPTY = 2 * SX + NB1, TEARDOWN = 2 * SX + 2 * NB1;
    static constexpr int NBAR = TEARDOWN + 1;
    static constexpr int OFF_BAR = OFF_RAW + SX * XTILE;
    static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;  // TMEM base, abort flag, the constant 1, maxima
    static constexpr int OFF_RED = OFF_MISC + 16;        // [2 epilogues][2 batches][GB][4 warps][16] fp32
    static constexpr int SMEM = OFF_RED + 2 * 2 * GB * 4 * RP * 4 + 1024;
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static_assert(STG % 1024 == 0 && OFF_RAW % 1024 == 0, "swizzle alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    __host__ __device__ static constexpr uint32_t R1(int b) { return uint32_t(A1COLS + b * R1W); }
};

// round_half_even(y * inv) as an int (see the fused transform kernel's epilogue).
__device__ __forceinline__ int round_code_r(uint32_t ybits, float inv, int one) {
    const uint32_t b = __float_as_uint(fmaf(__uint_as_float(ybits), inv, 12582912.0f));
    int k;
    asm("mad.lo.s32 %0, %1, %2, %3;" : "=r"(k) : "r"(b), "r"(one), "r"(-0x4B400000));
    return k;
}

template <int D>
__global__ void __launch_bounds__(R_THREADS, 1)
    kq_rowwise_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_q,
                      const uint16_t *__restrict__ Ph, float alpha, float *__restrict__ scale_out, int64_t R,
                      unsigned int *err) {
    using C = RCfg<D>;
    static_assert(staging_addresses_match<RP, D>(), "epilogue staging addresses");
    extern __shared__ __align__(1024) unsigned char rsm_raw[];
    const uint32_t raw_addr = smem_u32(rsm_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    unsigned char *smem = rsm_raw + (sbase - raw_addr);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // groups of H slots of RP rows; batches of GB groups dealt round-robin to CTAs
    const int64_t G = (R + C::H * RP - 1) / (C::H * RP);
    const int64_t NBt = (G + C::GB - 1) / C::GB;
    const int64_t nb = NBt > int64_t(blockIdx.x) ? (NBt - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    auto bar = [&](int i) -> uint32_t { return sbase + uint32_t(C::OFF_BAR + 8 * i); };
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    float *s_red = reinterpret_cast<float *>(smem + C::OFF_RED);

    if (tid == 0) {
        for (int s = 0; s < C::SX; ++s) {
            mbar_init(bar(C::FULL + s), 1);
            mbar_init(bar(C::EMPTY + s), 1);
        }
        for (int b = 0; b < C::NB1; ++b) {
            mbar_init(bar(C::D1FULL + b), 1);
            mbar_init(bar(C::D1EMPTY + b), 4);  // the four warps of the epilogue warpgroup
        }
        mbar_init(bar(C::TEARDOWN), 1);
        *s_abort = 0;
        *reinterpret_cast<int *>(smem + C::OFF_MISC + 8) = 1;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_x);
        prefetch_tensormap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(sbase + C::OFF_MISC, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    if (warp >= 4 && warp < 12) {
        // A1 (block-diagonal Ph^T, rows in lane order) into TMEM columns [0, 64):
        // warps 4-7 write K in [0, 64), warps 8-11 K in [64, 128).
        const int l = 32 * (warp & 3) + lane;
        const uint32_t taddr = tmem + (uint32_t(32 * (warp & 3)) << 16);
        const int kc0 = warp < 8 ? 0 : 2;
#pragma unroll
        for (int kq = 0; kq < 2; ++kq) {
            const int kc = kc0 + kq;
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int k = 32 * kc + 2 * e;
                w[e] = uint32_t(a1_value<D>(Ph, l, k)) | (uint32_t(a1_value<D>(Ph, l, k + 1)) << 16);
            }
            tmem_st_32x32b_x16(taddr + 16 * kc, w);
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == 0) {
        // ---------------- TMA producer: one batch tile per slot ----------------
        Ring rx;
        uint32_t issued = 0;
        int64_t g0 = int64_t(blockIdx.x) * C::GB;
        const int64_t gstep = int64_t(gridDim.x) * C::GB;
        for (int64_t j = 0; j < nb; ++j, g0 += gstep, rx.next(C::SX)) {
            const bool ok = wait_bounded_err(bar(C::EMPTY + rx.idx), rx.phase ^ 1u, s_abort, kSiteRowProducer,
                                             kWaitLimitNs, false, err);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (elect_one()) {
                mbar_arrive_expect_tx(bar(C::FULL + rx.idx), C::XTILE);
                const uint32_t dst = sbase + C::OFF_RAW + rx.idx * C::XTILE;
#pragma unroll
                for (int gp = 0; gp < C::GB; ++gp) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int64_t g = g0 + gp;
                        const int xc = (D == 128) ? 64 * c : 0;
                        const int64_t row = (D == 128) ? g * RP : (2 * g + c) * RP;
                        tma_load_2d(dst + c * C::CHUNK + gp * (RP * 128), &tmap_x, xc, int(row),
                                    bar(C::FULL + rx.idx));
                    }
                }
            }
            __syncwarp();
            ++issued;
        }
        Ring rd;
        for (uint32_t i = 0; i < issued; ++i, rd.next(C::SX))
            if (i + C::SX >= issued)
                wait_bounded_err(bar(C::FULL + rd.idx), rd.phase, s_abort, kSiteRowProducer, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer: D1 = Ph^T x^T for each batch ----------------
        constexpr uint32_t idesc = idesc_bf16_f32(128, C::NS1);
        auto koff = [](int kk) { return uint32_t(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4); };
        Ring rxs, r1;
        for (int64_t j = 0; j < nb; ++j, rxs.next(C::SX), r1.next(C::NB1)) {
            bool ok = wait_bounded_err(bar(C::D1EMPTY + r1.idx), r1.phase ^ 1u, s_abort, kSiteRowMma, kWaitLimitNs,
                                       false, err);
            ok = ok && wait_bounded_err(bar(C::FULL + rxs.idx), rxs.phase, s_abort, kSiteRowMma, kWaitLimitNs,
                                        false, err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t d1 = tmem + C::R1(int(r1.idx));
            const uint32_t bl = sdesc_sw128_lo(sbase + C::OFF_RAW + rxs.idx * C::XTILE);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    if (kk != 0)
                        mma_ts_split<1>(d1, tmem + 8 * kk, bl + koff(kk), kSdescSw128Hi, idesc);
                    else
                        mma_ts_split<0>(d1, tmem + 8 * kk, bl + koff(kk), kSdescSw128Hi, idesc);
                }
                tc_commit(bar(C::EMPTY + rxs.idx));
                tc_commit(bar(C::D1FULL + r1.idx));
            }
            __syncwarp();
        }
        if (elect_one()) tc_commit(bar(C::TEARDOWN));
        __syncwarp();
        wait_bounded_err(bar(C::TEARDOWN), 0u, s_abort, kSiteRowMma, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp >= 4 && warp < 12) {
        // ---------------- epilogue: per-row absmax, codes, staging, TMA store ----------------
        // The two warpgroups take alternate batches (GB groups): a first pass over
        // the groups finds the row maxima, one barrier, a second pass codes them;
        // one TMA store writes the batch's rows.
        const int ew = (warp - 4) >> 2;
        const int q = warp & 3;
        const int et = tid - 128 - 128 * ew;
        const uint32_t nbar = 1u + uint32_t(ew);
        const int slot = (32 * q) / D;           // slot of this warp's lanes
        const int g8 = lane >> 2, qq = lane & 3;
        const int one = *reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);
        float *red = s_red + ew * (2 * C::GB * 4 * RP);  // [2 buffers][GB groups][4 warps][16 rows]
        const uint32_t stg0 = sbase + C::OFF_STG + 2 * ew * C::BSTG;
        const bool storer = et == 0;
        auto store_batch = [&](int64_t gfirst, int sb) {
            if (storer) {
                tma_store_2d(&tmap_q, 0, int(C::H * gfirst * RP), stg0 + uint32_t(sb) * C::BSTG);
                bulk_commit();
            }
        };
        // this thread's two bytes of every row of its slot (see the transform kernel)
        const int row0 = slot * RP, bcol = ((32 * q) % D) / 2 + 2 * g8;
        const int swz_t = D == 128 ? qq : (qq >> 1);
        const int toff = (row0 + 2 * qq) * C::RB + ((((bcol >> 4) ^ swz_t) << 4) | (bcol & 15));
        int64_t gprev = -1;
        int it = 0;
        for (int64_t jb = ew; jb < nb; jb += 2, ++it) {
            const uint32_t b = uint32_t(jb % C::NB1), ph = uint32_t((jb / C::NB1) & 1);
            const int64_t g0 = (int64_t(blockIdx.x) + jb * gridDim.x) * C::GB;  // first group of the batch
            const int buf = it & 1;
            const bool ok = wait_bounded_err(bar(C::D1FULL + b), ph, s_abort, kSiteRowEpilogue, kWaitLimitNs,
                                             false, err);
            const bool warp_ok = __all_sync(0xffffffffu, ok);
            if (named_barrier_any(nbar, 128, !warp_ok)) break;
            __syncwarp();
            tc_fence_after();
            const uint32_t colb = tmem + C::R1(int(b)) + (uint32_t(32 * q) << 16);
            // pass 1: row maxima.  A 16x256b load per 16-lane half gives this thread
            // lanes g8, g8 + 8 of both halves (four output columns) of rows
            // 8 rep + 2 qq + d of each group; one x8 load covers four groups, so a
            // batch takes two load rounds.  xor shuffles finish each row over the
            // warp's lanes.
#pragma unroll 1
            for (int g4 = 0; g4 < C::GB; g4 += 4) {
                uint32_t ra[32], rb[32];
                tmem_ld_16x256b_x8(colb + uint32_t(RP * g4), ra);
                tmem_ld_16x256b_x8(colb + (16u << 16) + uint32_t(RP * g4), rb);
                tmem_wait_ld();
#pragma unroll
                for (int gl = 0; gl < 4; ++gl)
#pragma unroll
                    for (int rep = 0; rep < 2; ++rep)
#pragma unroll
                        for (int d = 0; d < 2; ++d) {
                            const int o = 4 * (2 * gl + rep);
                            float m = fmax3(fabsf(__uint_as_float(ra[o + d])), fabsf(__uint_as_float(ra[o + 2 + d])),
                                            fabsf(__uint_as_float(rb[o + d])));
                            m = fmaxf(m, fabsf(__uint_as_float(rb[o + 2 + d])));
#pragma unroll
                            for (int off = 4; off < 32; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
                            if (g8 == 0) red[((buf * C::GB + g4 + gl) * 4 + q) * RP + 8 * rep + 2 * qq + d] = m;
                        }
            }
            if (storer) bulk_wait_read<0>();  // the store that read this staging tile is done
            named_barrier_sync(nbar, 128);
            if (gprev >= 0) store_batch(gprev, buf ^ 1);
            unsigned char *stgb = smem + C::OFF_STG + (2 * ew + buf) * C::BSTG + toff;
            // pass 2: scales and codes, four groups per load round
#pragma unroll 1
            for (int g4 = 0; g4 < C::GB; g4 += 4) {
                uint32_t ra[32], rb[32];
                tmem_ld_16x256b_x8(colb + uint32_t(RP * g4), ra);
                tmem_ld_16x256b_x8(colb + (16u << 16) + uint32_t(RP * g4), rb);
                tmem_wait_ld();
                if (g4 + 4 >= C::GB) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(C::D1EMPTY + b));  // this warp is done with the region
                }
#pragma unroll
                for (int gl = 0; gl < 4; ++gl) {
                    const int gp = g4 + gl;
                    unsigned char *tbase = stgb + gp * C::STG;
#pragma unroll
                    for (int rep = 0; rep < 2; ++rep)
#pragma unroll
                        for (int d = 0; d < 2; ++d) {
                            const int i = 8 * rep + 2 * qq + d;
                            float m = 0.0f;
#pragma unroll
                            for (int w = 0; w < 4; ++w)
                                if ((32 * w) / D == slot) m = fmaxf(m, red[((buf * C::GB + gp) * 4 + w) * RP + i]);
                            const float sc = alpha * m * (1.0f / 7.0f);
                            const float iv = sc > 0.0f ? fminf(__fdividef(1.0f, sc), 3.0e38f) : 0.0f;
                            // the scale of row i of the slot: written once, by the slot's first warp
                            if ((32 * q) % D == 0 && g8 == 0) {
                                const int64_t r = (C::H * (g0 + gp) + slot) * RP + i;
                                if (r < R) scale_out[r] = sc;
                            }
                            const int o = 4 * (2 * gl + rep);
                            const uint32_t wb = pack_s4x2(round_code_r(rb[o + 2 + d], iv, one),
                                                          round_code_r(rb[o + d], iv, one), 0u);
                            const uint32_t w = pack_s4x2(round_code_r(ra[o + 2 + d], iv, one),
                                                         round_code_r(ra[o + d], iv, one), wb);
                            *reinterpret_cast<uint16_t *>(tbase + (8 * rep + d) * C::RB) = uint16_t(w);
                        }
                }
            }
            fence_proxy_async_smem();
            gprev = g0;
        }
        named_barrier_sync(nbar, 128);
        if (gprev >= 0) store_batch(gprev, (it - 1) & 1);
        if (storer) bulk_wait<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D>
cudaError_t launch_rowwise_inst(const uint16_t *x, const uint16_t *Ph, float alpha, uint8_t *q_out, float *scale_out,
                                int64_t R, int num_sms, int device, cudaStream_t stream) {
    using C = RCfg<D>;
    auto kern = kq_rowwise_kernel<D>;
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
    CUtensorMap tx, tq;
    const cuuint64_t dx[2] = {cuuint64_t(D), cuuint64_t(R)};
    const cuuint64_t sx[1] = {cuuint64_t(D) * 2};
    const cuuint32_t bx[2] = {64u, cuuint32_t(RP)};
    const cuuint32_t estr[2] = {1u, 1u};
    CUresult r = encode(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(x), dx, sx, bx, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const cuuint64_t dq[2] = {cuuint64_t(C::RB), cuuint64_t(R)};
    const cuuint64_t sq[1] = {cuuint64_t(C::RB)};
    const cuuint32_t bq[2] = {cuuint32_t(C::RB), cuuint32_t(C::GB * C::H * RP)};  // one batch
    r = encode(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q_out, dq, sq, bq, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const int64_t G = (R + C::H * RP - 1) / (C::H * RP);
    const int64_t NBt = (G + C::GB - 1) / C::GB;
    const int64_t grid = NBt < num_sms ? NBt : num_sms;
    kern<<<unsigned(grid), R_THREADS, C::SMEM, stream>>>(tx, tq, Ph, alpha, scale_out, R, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rowwise(const uint16_t *x, const uint16_t *Ph, float alpha, uint8_t *q_out, float *scale_out,
                           int64_t R, int head_dim, int num_sms, int device, cudaStream_t stream) {
    if (R >= (int64_t(1) << 31)) return cudaErrorInvalidValue;  // TMA row coordinate range
    if (head_dim == 128) return launch_rowwise_inst<128>(x, Ph, alpha, q_out, scale_out, R, num_sms, device, stream);
    if (head_dim == 64) return launch_rowwise_inst<64>(x, Ph, alpha, q_out, scale_out, R, num_sms, device, stream);
    return cudaErrorNotSupported;
}

}  // namespace kq
