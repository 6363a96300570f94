// kq_gemm.cu -- the W4A4 product that consumes the packed codes
// (FlatQuant page, "Kronecker factorization": Q(X P) Q(P^-1 W^T)):
//
//     y[m][o] = sx[m] * sw[o] * sum_k qx[m][k] * qw[o][k]
//
// qx [M, K/2] and qw [N, K/2] hold two's-complement INT4 codes, element 2k in
// the low nibble of byte k (the layout kq_transform_quant writes), sx [M] and
// sw [N] the per-token and per-output-channel fp32 scales, y [M, N] fp32.
//
// Tensor cores read the nibbles as they are: mma.sync m16n8k64 with s4
// operands and s32 accumulators (the sum is exact), fed by ldmatrix from a
// 4-stage cp.async ring.  Tile 128 x 128 x 128 per CTA, 8 warps of 64 x 32.
// The integer sum is converted to fp32 (exact: |sum| <= 64 K < 2^24) and
// multiplied by sx[m], then by sw[o].
#include <mutex>

#include "kq_common.cuh"
#include "kq_internal.h"

namespace kq {
namespace {

constexpr int BM = 128, BN = 128;      // tile rows (tokens) and columns (output channels)
constexpr int BKB = 64;                // K bytes per stage (128 codes)
constexpr int STAGES = 4;
constexpr int GEMM_THREADS = 256;      // 8 warps: 2 along M x 4 along N, 64 x 32 each
constexpr int STAGE_BYTES = (BM + BN) * BKB;
constexpr int GEMM_SMEM = STAGES * STAGE_BYTES;

// Rows of 64 bytes (four 16-byte chunks); chunk c of row r is stored at chunk
// c ^ ((r >> 1) & 3), so the eight rows an ldmatrix reads hit 32 distinct banks.
__device__ __forceinline__ uint32_t tile_off(int r, int chunk) {
    return uint32_t(r * BKB + ((chunk ^ ((r >> 1) & 3)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_s4(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k64.row.col.s32.s4.s4.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(GEMM_THREADS, 1)
    kq_w4a4_gemm_kernel(const uint8_t *__restrict__ qx, const float *__restrict__ sx,
                        const uint8_t *__restrict__ qw, const float *__restrict__ sw, float *__restrict__ y,
                        int64_t M, int64_t N, int64_t K) {
    extern __shared__ __align__(128) unsigned char gsm[];
    const uint32_t sbase = smem_u32(gsm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wm = warp >> 2, wn = warp & 3;
    const int64_t m0 = int64_t(blockIdx.y) * BM, n0 = int64_t(blockIdx.x) * BN;
    const int64_t kbytes = K / 2;
    const int KT = int(K / (2 * BKB));

    // Each thread copies two 16-byte chunks of A and two of B per stage.
    auto load_stage = [&](int kt, int slot) {
        const uint32_t sa = sbase + uint32_t(slot * STAGE_BYTES), sb = sa + BM * BKB;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = tid + h * GEMM_THREADS, r = c >> 2, ch = c & 3;
            const int64_t ga = m0 + r, gb = n0 + r;
            const bool va = ga < M, vb = gb < N;
            // rows past the end read nothing (size 0) and the chunk is zero-filled
            const uint8_t *pa = qx + (va ? ga : 0) * kbytes + int64_t(kt) * BKB + ch * 16;
            const uint8_t *pb = qw + (vb ? gb : 0) * kbytes + int64_t(kt) * BKB + ch * 16;
            cp_async16(sa + tile_off(r, ch), pa, va);
            cp_async16(sb + tile_off(r, ch), pb, vb);
        }
    };

    int acc[4][4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0;

#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
        if (s < KT) load_stage(s, s);
        cp_async_commit();
    }

    // ldmatrix row addresses: thread t serves matrix t / 8, row t % 8
    const int mat = lane >> 3, mr = lane & 7;
    for (int kt = 0; kt < KT; ++kt) {
        cp_async_wait<STAGES - 2>();
        __syncthreads();  // tile kt landed for everyone; slot (kt - 1) % STAGES is free
        if (kt + STAGES - 1 < KT) load_stage(kt + STAGES - 1, (kt + STAGES - 1) % STAGES);
        cp_async_commit();

        const uint32_t sa = sbase + uint32_t((kt % STAGES) * STAGE_BYTES), sb = sa + BM * BKB;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {  // two k64 steps per stage
            uint32_t a[4][4], b[4][2];
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                // matrices: rows +0 / +8 of the m16 tile, bytes [0,16) / [16,32) of the k64 step
                const int r = wm * 64 + mt * 16 + (mat & 1) * 8 + mr;
                ldmatrix_x4(sa + tile_off(r, 2 * kk + (mat >> 1)), a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
            }
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                // matrices: n8 tile 2 np (k halves 0, 1), then n8 tile 2 np + 1
                const int r = wn * 32 + (2 * np + (mat >> 1)) * 8 + mr;
                ldmatrix_x4(sb + tile_off(r, 2 * kk + (mat & 1)), b[2 * np][0], b[2 * np][1], b[2 * np + 1][0],
                            b[2 * np + 1][1]);
            }
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) mma_s4(acc[mt][nt], a[mt], b[nt][0], b[nt][1]);
        }
    }
    cp_async_wait<0>();

    // epilogue: accumulator (row g (+8), columns 2 tig, 2 tig + 1) of each m16n8 tile
    const int g = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int64_t m = m0 + wm * 64 + mt * 16 + g + 8 * hr;
            if (m >= M) continue;
            const float fx = sx[m];
            float *yrow = y + m * N;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int64_t n = n0 + wn * 32 + nt * 8 + 2 * tig;
                if (n < N) yrow[n] = (float(acc[mt][nt][2 * hr]) * fx) * sw[n];
                if (n + 1 < N) yrow[n + 1] = (float(acc[mt][nt][2 * hr + 1]) * fx) * sw[n + 1];
            }
        }
    }
}

}  // namespace

cudaError_t launch_w4a4_gemm(const uint8_t *qx, const float *sx, const uint8_t *qw, const float *sw, float *y,
                             int64_t M, int64_t N, int64_t K, int device, cudaStream_t stream) {
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[device], [&] {
        attr_err[device] = cudaFuncSetAttribute(kq_w4a4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                GEMM_SMEM);
    });
    if (attr_err[device] != cudaSuccess) return attr_err[device];
    const dim3 grid(unsigned((N + BN - 1) / BN), unsigned((M + BM - 1) / BM));
    kq_w4a4_gemm_kernel<<<grid, GEMM_THREADS, GEMM_SMEM, stream>>>(qx, sx, qw, sw, y, M, N, K);
    return cudaGetLastError();
}

}  // namespace kq
