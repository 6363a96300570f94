// kq_gemm.cu -- the W4A4 product that consumes the packed codes
// (FlatQuant page, "Kronecker factorization": Q(X P) Q(P^-1 W^T)):
//
//     y[m][o] = sx[m] * sw[o] * sum_k qx[m][k] * qw[o][k]
//
// qx [M, K/2] and qw [N, K/2] hold two's-complement INT4 codes, element 2k in
// the low nibble of byte k (the layout kq_transform_quant writes), sx [M] and
// sw [N] the per-token and per-output-channel fp32 scales, y [M, N] fp32, or
// bf16 (the fp32 value rounded to nearest even), which halves the output bytes
// that dominate the traffic of a large product.
//
// The 5th-generation tensor cores have no 4-bit integer kind, so each 128-code
// K chunk goes: packed tiles by TMA -> eight expander warps widen every code q
// to the int8 16 q (a mask keeps the high nibble where it is, a shift moves the
// low one up) -> tcgen05.mma kind::i8 (s8 x s8 -> s32 in TMEM).  The widened
// activation tile goes straight into TMEM (the MMA's A operand, one row per
// lane, four K bytes per column), the widened weight tile into shared memory
// (B), which keeps a third of the widened bytes off the shared-memory pipe.
// Within every 8-code group the expanders write the even codes before the odd
// ones, the same way for both operands, which leaves every dot product
// unchanged.  The s32 sums are 256 times the code sums and exact
// (|sum| <= 16384 K < 2^31); the epilogue shifts the factor out and applies
// (float(sum) * sx[m]) * sw[o].
//
// One CTA per 256 x 128 output tile: two 128-row activation tiles in TMEM (the
// A operands of two MMAs) share one widened weight tile in shared memory, so
// each widened weight byte written to shared memory feeds two MMAs; that keeps
// the shared-memory traffic per output a seventh below a 128 x 256 tile's.
// Warps: 0 TMA producer | 1 TMEM allocator + MMA issuer | 4-11 expanders, then
// the epilogue | 2-3 idle.
// Every mbarrier wait is bounded (kq_wait.cuh).
#include <mutex>

#include "kq_common.cuh"
#include "kq_internal.h"
#include "kq_tc05_ptx.cuh"
#include "kq_wait.cuh"

namespace kq {
namespace {

using namespace tc;

constexpr int TM = 256, TN = 128, KC = 128;            // tile rows (two MMA tiles), columns, codes per K chunk
constexpr int PA = TM * KC / 2, PB = TN * KC / 2;       // packed bytes per chunk: 16 KB, 8 KB
constexpr int EB = TN * KC;                             // widened int8 weight bytes per chunk: 16 KB
constexpr int NS = 5, NE = 4;                           // packed stages, widened stages
constexpr int G_THREADS = 384;                          // 12 warps
constexpr int XW0 = 4, NXW = 8;                         // expander / epilogue warps 4-11
constexpr int OFF_E = NS * (PA + PB);                   // 120 KB: widened weight stages (1024-aligned)
constexpr int OFF_BAR = OFF_E + NE * EB;
constexpr int FULL = 0, EMPTY = NS, XFULL = 2 * NS, XEMPTY = 2 * NS + NE, DONE = 2 * NS + 2 * NE;
constexpr int NBAR = DONE + 1;
constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;            // TMEM base, abort flag
constexpr int G_SMEM = OFF_MISC + 16 + 1024;            // + slack for 1024-byte alignment
constexpr uint32_t TMEM_COLS = 512;  // s32 accumulators [0, 128) and [128, 256) + widened activations
constexpr uint32_t ACOL = 2 * TN;    // widened activation stage e: tile h at columns 256 + 64 e + 32 h
static_assert(ACOL + NE * 2 * (KC / 4) <= TMEM_COLS, "TMEM budget");
static_assert(OFF_E % 1024 == 0 && EB % 1024 == 0 && (PA + PB) % 1024 == 0, "swizzle atoms");
static_assert(G_SMEM <= 227 * 1024, "shared memory budget");

enum : unsigned { kSiteGemm = 64u };

// Instruction descriptor: signed int8 A and B (K-major), s32 accumulator, M x N.
__host__ __device__ constexpr uint32_t idesc_s8_s32(int M, int N) {
    return (2u << 4)                      // accumulator format: s32
           | (1u << 7)                    // A format: signed 8-bit
           | (1u << 10)                   // B format: signed 8-bit
           | (uint32_t(N >> 3) << 17)     // N / 8
           | (uint32_t(M >> 4) << 24);    // M / 16
}

// D (+)= A B^T with A in TMEM and B in shared memory, described by the low
// half of its 128B-swizzle descriptor.
template <int ACC>
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 bd;\n\tmov.b64 bd, {%2, %3};\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], bd, %4, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b_lo), "r"(kSdescSw128Hi), "r"(idesc), "n"(ACC)
        : "memory");
}

// Byte offset of the 16-byte chunk `c` of row `r` in a 128B-swizzled K-major tile.
__device__ __forceinline__ uint32_t sw128_chunk(int r, int c) { return uint32_t(r * 128 + ((c ^ (r & 7)) << 4)); }

// y[n .. n + 3] of one row: fp32 as is, or rounded to bf16 (nearest even);
// one 16-byte (fp32) or 8-byte (bf16) store where `vec` allows it.
template <bool BF16>
__device__ __forceinline__ void store_out4(void *yrow, int64_t n, int64_t N, bool vec, const float (&r4)[4]) {
    if constexpr (BF16) {
        uint16_t *p = static_cast<uint16_t *>(yrow) + n;
        const __nv_bfloat162 a = __floats2bfloat162_rn(r4[0], r4[1]), b = __floats2bfloat162_rn(r4[2], r4[3]);
        if (vec && n + 3 < N) {
            *reinterpret_cast<uint2 *>(p) = make_uint2(*reinterpret_cast<const uint32_t *>(&a),
                                                       *reinterpret_cast<const uint32_t *>(&b));
        } else {
            const uint16_t h[4] = {__bfloat16_as_ushort(a.x), __bfloat16_as_ushort(a.y), __bfloat16_as_ushort(b.x),
                                   __bfloat16_as_ushort(b.y)};
#pragma unroll
            for (int t = 0; t < 4; ++t)
                if (n + t < N) p[t] = h[t];
        }
    } else {
        float *p = static_cast<float *>(yrow) + n;
        if (vec && n + 3 < N) {
            *reinterpret_cast<float4 *>(p) = make_float4(r4[0], r4[1], r4[2], r4[3]);
        } else {
#pragma unroll
            for (int t = 0; t < 4; ++t)
                if (n + t < N) p[t] = r4[t];
        }
    }
}

template <bool BF16>
__global__ void __launch_bounds__(G_THREADS, 1)
    kq_w4a4_tc_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const float *__restrict__ sx, const float *__restrict__ sw, void *__restrict__ y,
                      int64_t M, int64_t N, int64_t K, unsigned int *err) {
    extern __shared__ __align__(1024) unsigned char gsm_raw[];
    const uint32_t raw_addr = smem_u32(gsm_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    unsigned char *smem = gsm_raw + (sbase - raw_addr);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t m0 = int64_t(blockIdx.y) * TM, n0 = int64_t(blockIdx.x) * TN;
    const int KT = int(K / KC);
    auto bar = [&](int i) -> uint32_t { return sbase + uint32_t(OFF_BAR + 8 * i); };
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(FULL + s), 1);
            mbar_init(bar(EMPTY + s), NXW);  // one arrive per expander warp
        }
        for (int e = 0; e < NE; ++e) {
            mbar_init(bar(XFULL + e), NXW);
            mbar_init(bar(XEMPTY + e), 1);
        }
        mbar_init(bar(DONE), 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_a);
        prefetch_tensormap(&tmap_b);
    }
    if (warp == 1) {
        tmem_alloc(sbase + OFF_MISC, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + OFF_MISC);

    if (warp == 0) {
        // ---------------- TMA producer: packed A and B tiles of each K chunk ----------------
        Ring r;
        int issued = 0;
        for (int kt = 0; kt < KT; ++kt, r.next(NS)) {
            const bool ok = wait_bounded_err(bar(EMPTY + r.idx), r.phase ^ 1u, s_abort, kSiteGemm, kWaitLimitNs,
                                             false, err);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (elect_one()) {
                const uint32_t dst = sbase + uint32_t(r.idx * (PA + PB));
                mbar_arrive_expect_tx(bar(FULL + r.idx), PA + PB);
                tma_load_2d(dst, &tmap_a, kt * (KC / 2), int(m0), bar(FULL + r.idx));
                tma_load_2d(dst + PA, &tmap_b, kt * (KC / 2), int(n0), bar(FULL + r.idx));
            }
            __syncwarp();
            ++issued;
        }
        // every load issued has landed before the CTA can exit
        Ring rd;
        for (int i = 0; i < issued; ++i, rd.next(NS))
            if (i + NS >= issued)
                wait_bounded_err(bar(FULL + rd.idx), rd.phase, s_abort, kSiteGemm, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        constexpr uint32_t idesc = idesc_s8_s32(128, TN);
        Ring r;
        for (int kt = 0; kt < KT; ++kt, r.next(NE)) {
            const bool ok = wait_bounded_err(bar(XFULL + r.idx), r.phase, s_abort, kSiteGemm, kWaitLimitNs, false,
                                             err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t bl = sdesc_sw128_lo(sbase + uint32_t(OFF_E + r.idx * EB));
            const uint32_t at = tmem + ACOL + uint32_t(r.idx * 2 * (KC / 4));
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < KC / 32; ++kk) {  // K = 32 int8 per MMA: 8 TMEM columns, +32 bytes of B
#pragma unroll
                    for (int h = 0; h < 2; ++h) {      // the two 128-row tiles share the B slice
                        const uint32_t d = tmem + uint32_t(h * TN), a = at + uint32_t(h * (KC / 4)) + 8 * kk;
                        if ((kt | kk) != 0)
                            mma_i8_ts<1>(d, a, bl + 2 * kk, idesc);
                        else
                            mma_i8_ts<0>(d, a, bl + 2 * kk, idesc);
                    }
                }
                tc_commit(bar(XEMPTY + r.idx));  // widened stage free once these MMAs complete
            }
            __syncwarp();
        }
        // DONE completes once every MMA this thread issued has completed
        if (elect_one()) tc_commit(bar(DONE));
        __syncwarp();
        wait_bounded_err(bar(DONE), 0u, s_abort, kSiteGemm, kWaitLimitNs, true, err);
        __syncwarp();
    } else if (warp >= XW0 && warp < XW0 + NXW) {
        // ---------------- expanders: packed INT4 -> int8 (x16) ----------------
        // Activations: thread (warp w, lane) widens row am = 128 hh + 32 (w % 4) +
        // lane of the 256-row tile (hh = (w - 4) / 4): its four 16-byte units of
        // the packed tile (64B swizzle: unit c of row m at m * 64 + 16 (c ^ ((m >> 1)
        // & 3)), so the eight rows of a shared-memory phase hit eight bank groups)
        // become 32 TMEM columns of lane am % 128 in MMA tile hh.  Weights: two
        // 16-byte units per thread into the 128B-swizzled K-major shared tile.
        const int xt = tid - XW0 * 32;                // 0 .. 255
        const int hh = (warp - XW0) >> 2, qa = warp & 3;
        const int am = 128 * hh + 32 * qa + lane;     // activation row of the tile
        constexpr int UB = TN * (KC / 32);            // 16-byte packed weight units per chunk: 512
        constexpr int UPB = UB / (NXW * 32);          // 2 per thread
        static_assert(UB % (NXW * 32) == 0, "unit split");
        Ring rs, re;
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt, rs.next(NS), re.next(NE)) {
            ok = wait_bounded_err(bar(FULL + rs.idx), rs.phase, s_abort, kSiteGemm, kWaitLimitNs, false, err);
            ok = ok && wait_bounded_err(bar(XEMPTY + re.idx), re.phase ^ 1u, s_abort, kSiteGemm, kWaitLimitNs,
                                        false, err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const unsigned char *pk = smem + rs.idx * (PA + PB);
            unsigned char *ex = smem + OFF_E + re.idx * EB;
            uint4 va[4], vb[UPB];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                va[c] = *reinterpret_cast<const uint4 *>(pk + am * 64 + ((c ^ ((am >> 1) & 3)) << 4));
#pragma unroll
            for (int i = 0; i < UPB; ++i)
                vb[i] = *reinterpret_cast<const uint4 *>(pk + PA + (xt + i * NXW * 32) * 16);
            // activations -> TMEM: unit c gives columns 8 c .. 8 c + 7 of this row's tile
            uint32_t o[2][16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t w[4] = {va[c].x, va[c].y, va[c].z, va[c].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    o[c >> 1][8 * (c & 1) + 2 * j] = (w[j] << 4) & 0xF0F0F0F0u;  // even codes of the 8-code group, x16
                    o[c >> 1][8 * (c & 1) + 2 * j + 1] = w[j] & 0xF0F0F0F0u;     // odd codes, x16
                }
            }
            const uint32_t tcol = tmem + (uint32_t(32 * qa) << 16) + ACOL + uint32_t((2 * re.idx + hh) * (KC / 4));
            tmem_st_32x32b_x16(tcol, o[0]);
            tmem_st_32x32b_x16(tcol + 16, o[1]);
            // weights -> shared memory
#pragma unroll
            for (int i = 0; i < UPB; ++i) {
                const int ub = xt + i * NXW * 32;
                const int r = ub >> 2, q = ub & 3;  // row, 16-byte unit within the row's 64 packed bytes
                const uint32_t w[4] = {vb[i].x, vb[i].y, vb[i].z, vb[i].w};
                uint32_t e[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    e[2 * j] = (w[j] << 4) & 0xF0F0F0F0u;
                    e[2 * j + 1] = w[j] & 0xF0F0F0F0u;
                }
                *reinterpret_cast<uint4 *>(ex + sw128_chunk(r, 2 * q)) = make_uint4(e[0], e[1], e[2], e[3]);
                *reinterpret_cast<uint4 *>(ex + sw128_chunk(r, 2 * q + 1)) = make_uint4(e[4], e[5], e[6], e[7]);
            }
            tmem_wait_st();
            fence_proxy_async_smem();  // widened weight tile visible to the tensor cores
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(EMPTY + rs.idx));  // packed stage read
                mbar_arrive(bar(XFULL + re.idx));  // widened stage written
            }
        }
        // ---------------- epilogue: TMEM -> scales -> y ----------------
        const bool done = wait_bounded_err(bar(DONE), 0u, s_abort, kSiteGemm, kWaitLimitNs, false, err);
        if (__all_sync(0xffffffffu, done && ok)) {
            tc_fence_after();
            const int q = warp & 3, h = (warp - XW0) >> 2;  // lane quarter, 128-row tile
            const int64_t m = m0 + 128 * h + 32 * q + lane;
            const float fx = m < M ? sx[m] : 0.0f;
            constexpr int OB = BF16 ? 2 : 4;  // output bytes per element
            void *yrow = static_cast<unsigned char *>(y) + (m < M ? m : 0) * N * OB;
            // vector stores only where every row start is aligned for them
            const bool vec = (N % 4) == 0 && (reinterpret_cast<uintptr_t>(y) & (4 * OB - 1)) == 0;
#pragma unroll 1
            for (int c = 0; c < TN / 32; ++c) {
                uint32_t a[32];
                tmem_ld_32x32b_x32(tmem + (uint32_t(32 * q) << 16) + uint32_t(TN * h + 32 * c), a);
                tmem_wait_ld();
                const int64_t nb = n0 + 32 * c;
                if (m < M) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const int64_t n = nb + e;
                        float r4[4];
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            r4[t] = (float(int(a[e + t]) >> 8) * fx) * (n + t < N ? sw[n + t] : 0.0f);
                        store_out4<BF16>(yrow, n, N, vec, r4);
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
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace

cudaError_t launch_w4a4_gemm(const uint8_t *qx, const float *sx, const uint8_t *qw, const float *sw, void *y,
                             bool bf16_out, int64_t M, int64_t N, int64_t K, int device, cudaStream_t stream) {
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[device], [&] {
        attr_err[device] = cudaFuncSetAttribute(kq_w4a4_tc_kernel<false>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM);
        if (attr_err[device] == cudaSuccess)
            attr_err[device] = cudaFuncSetAttribute(kq_w4a4_tc_kernel<true>,
                                                    cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM);
    });
    if (attr_err[device] != cudaSuccess) return attr_err[device];
    unsigned int *err = nullptr;
    cudaError_t e = device_error_word(device, &err);
    if (e != cudaSuccess) return e;
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    // packed codes: rows of K/2 bytes; one box = one K chunk (64 bytes) of TM or TN rows
    CUtensorMap ta, tb;
    const cuuint64_t da[2] = {cuuint64_t(K / 2), cuuint64_t(M)}, db[2] = {cuuint64_t(K / 2), cuuint64_t(N)};
    const cuuint64_t stride[1] = {cuuint64_t(K / 2)};
    const cuuint32_t boxa[2] = {cuuint32_t(KC / 2), cuuint32_t(TM)}, boxb[2] = {cuuint32_t(KC / 2), cuuint32_t(TN)};
    const cuuint32_t estr[2] = {1u, 1u};
    CUresult r = encode(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(qx), da, stride, boxa, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    r = encode(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(qw), db, stride, boxb, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const dim3 grid(unsigned((N + TN - 1) / TN), unsigned((M + TM - 1) / TM));
    if (bf16_out)
        kq_w4a4_tc_kernel<true><<<grid, G_THREADS, G_SMEM, stream>>>(ta, tb, sx, sw, y, M, N, K, err);
    else
        kq_w4a4_tc_kernel<false><<<grid, G_THREADS, G_SMEM, stream>>>(ta, tb, sx, sw, y, M, N, K, err);
    return cudaGetLastError();
}

}  // namespace kq
