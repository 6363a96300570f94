// kq_warp_mma.cu -- general fused Kronecker transform + INT4 kernel on the
// warp-level tensor-core path (mma.sync m16n8k16, bf16 in, fp32 accumulate).
//
// It covers every supported shape (n1, n2 multiples of 16 up to 128) and runs
// what the tcgen05 kernels do not: the fp32 check entry kq_transform, clip
// ratios below 2^-19, and inputs of 2^31 rows of x or more.
//
// Method (FlatQuant page, "Kronecker factorization" and "The fused kernel"):
// for a token, Y~ = P1^T X~ P2 with X~ the row-major n1 x n2 view of x * cinv.
// Each warp owns 16 output columns j of one token:
//   stage 1  Z^T[j][a] = sum_b P2^T[j][b] X~[a][b]   (M = j, N = a, K = b)
//   stage 2  Y~[i][j]  = sum_a P1^T[i][a] Z[a][j]     (M = i, N = j, K = a)
// The stage-1 accumulator fragment (rows j, columns a) is exactly the stage-2
// B fragment (k = a, n = j), so Z never leaves registers.  Z is split into
// hi + lo bf16 halves (and x * cinv too when cinv is given), each multiplied
// separately into the same fp32 accumulator.  The epilogue reduces the
// token's absmax across warps through shared memory, quantises, packs
// nibbles into a shared staging row and writes it out with 16-byte stores.
#include "kq_common.cuh"
#include "kq_internal.h"

namespace kq {

namespace {

constexpr int kMax = 128;      // largest n1 / n2
constexpr int kWarps = 8;      // warps per CTA
constexpr int kThreads = kWarps * 32;

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void cp_async_16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

struct Geometry {
    int n1, n2, n, wpt, tpi, xs, p1s, tile;  // tile: bf16 elements per stage
};

__host__ __device__ inline Geometry make_geometry(int n1, int n2) {
    Geometry g;
    g.n1 = n1;
    g.n2 = n2;
    g.n = n1 * n2;
    g.wpt = n2 / 16;
    g.tpi = kWarps / g.wpt > 0 ? kWarps / g.wpt : 1;
    g.xs = n2 + 8;   // padded row stride: 16-byte rows shifted by one bank group
    g.p1s = n1 + 8;
    g.tile = g.tpi * n1 * g.xs;
    return g;
}

// Shared memory carve-up (bytes): P1^T | x stages (2) | lo tile | cinv | reduction | out rows
struct Layout {
    size_t p1t, xst, lo, cinv, red, out, total;
};

__host__ __device__ inline Layout make_layout(const Geometry &g, bool scaled, bool quant) {
    Layout L;
    size_t off = 0;
    L.p1t = off;
    off += size_t(g.n1) * g.p1s * 2;
    L.xst = off;
    off += size_t(2) * g.tile * 2;
    L.lo = off;
    off += scaled ? size_t(g.tile) * 2 : 0;
    L.cinv = off;
    off += scaled ? size_t(g.n) * 4 : 0;
    L.red = off;
    off += 64 * 4;
    L.out = off;
    off += quant ? size_t(g.tpi) * g.n / 2 : 0;
    L.total = off;
    return L;
}

template <bool SCALED, bool QUANT>
__global__ void __launch_bounds__(kThreads, 1)
    kq_warp_mma_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ P1,
                       const uint16_t *__restrict__ P2, const float *__restrict__ cinv, float alpha,
                       uint8_t *__restrict__ q_out, float *__restrict__ scale_out,
                       float *__restrict__ y_out, int64_t T, int n1, int n2) {
    extern __shared__ __align__(128) unsigned char smem[];
    const Geometry G = make_geometry(n1, n2);
    const Layout L = make_layout(G, SCALED, QUANT);
    uint16_t *sP1T = reinterpret_cast<uint16_t *>(smem + L.p1t);
    uint16_t *sX = reinterpret_cast<uint16_t *>(smem + L.xst);
    uint16_t *sLo = reinterpret_cast<uint16_t *>(smem + L.lo);
    float *sC = reinterpret_cast<float *>(smem + L.cinv);
    float *sRed = reinterpret_cast<float *>(smem + L.red);
    uint8_t *sOut = smem + L.out;

    // The next launch on the stream may be scheduled once every CTA of this grid
    // has started (the grid fits on the GPU at once); every global access below
    // comes after the previous kernel on the stream has completed.
    griddep_launch_dependents();
    griddep_wait();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, q4 = lane & 3;
    const int slot = warp / G.wpt, jb = warp % G.wpt, j0 = 16 * jb;
    const bool active = slot < G.tpi;  // warps beyond tpi*wpt only join barriers
    const int nk1 = n2 / 16;           // stage-1 k-steps (b)
    const int nc = n1 / 8;             // stage-1 n-tiles (a)
    const int nk2 = n1 / 16;           // stage-2 k-steps (a) == m-tiles (i)

    // P1^T into shared memory: sP1T[i][a] = P1[a][i].
    for (int e = tid; e < n1 * n1; e += kThreads) {
        int a = e / n1, i = e - a * n1;
        sP1T[i * G.p1s + a] = P1[e];
    }
    if (SCALED)
        for (int e = tid; e < G.n; e += kThreads) sC[e] = cinv[e];

    // P2^T A-fragments for this warp's 16 rows j (loaded once per CTA).
    uint32_t aP2[kMax / 16][4];
#pragma unroll
    for (int ks = 0; ks < kMax / 16; ++ks) {
        if (ks < nk1 && active) {
            const int k0 = 16 * ks + 2 * q4;
            const int ja = j0 + g, jbb = j0 + 8 + g;
            aP2[ks][0] = uint32_t(P2[k0 * n2 + ja]) | (uint32_t(P2[(k0 + 1) * n2 + ja]) << 16);
            aP2[ks][1] = uint32_t(P2[k0 * n2 + jbb]) | (uint32_t(P2[(k0 + 1) * n2 + jbb]) << 16);
            aP2[ks][2] = uint32_t(P2[(k0 + 8) * n2 + ja]) | (uint32_t(P2[(k0 + 9) * n2 + ja]) << 16);
            aP2[ks][3] = uint32_t(P2[(k0 + 8) * n2 + jbb]) | (uint32_t(P2[(k0 + 9) * n2 + jbb]) << 16);
        } else {
            aP2[ks][0] = aP2[ks][1] = aP2[ks][2] = aP2[ks][3] = 0u;
        }
    }

    const int64_t n_iter = (T + G.tpi - 1) / G.tpi;
    const int chunks_row = n2 / 8;              // 16-byte chunks per row of X~
    const int chunks_tok = G.n / 8;

    auto load_stage = [&](int64_t it, int st) {
        uint16_t *dst0 = sX + st * G.tile;
        for (int e = tid; e < G.tpi * chunks_tok; e += kThreads) {
            const int s = e / chunks_tok, c = e - s * chunks_tok;
            const int64_t t = it * G.tpi + s;
            if (t < T) {
                const int a = c / chunks_row, c8 = c - a * chunks_row;
                cp_async_16(dst0 + (s * n1 + a) * G.xs + c8 * 8, x + t * G.n + a * n2 + c8 * 8);
            }
        }
    };

    int64_t it = blockIdx.x;
    int stage = 0;
    if (it < n_iter) load_stage(it, 0);
    cp_async_commit();

    for (; it < n_iter; it += gridDim.x, stage ^= 1) {
        const int64_t nxt = it + gridDim.x;
        if (nxt < n_iter) load_stage(nxt, stage ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();

        uint16_t *tile = sX + stage * G.tile;
        if (SCALED) {
            // x' = x * cinv, split into hi (in place) and lo (separate tile).
            for (int e = tid; e < G.tpi * chunks_tok; e += kThreads) {
                const int s = e / chunks_tok, c = e - s * chunks_tok;
                const int a = c / chunks_row, c8 = c - a * chunks_row;
                const int off = (s * n1 + a) * G.xs + c8 * 8;
                const int k0 = a * n2 + c8 * 8;
                uint4 raw = *reinterpret_cast<const uint4 *>(tile + off);
                const uint16_t *h = reinterpret_cast<const uint16_t *>(&raw);
                uint16_t hi[8], lo[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    float v = bf16_bits_to_float(h[u]) * sC[k0 + u];
                    float vh, vl;
                    split_bf16(v, vh, vl);
                    hi[u] = float_to_bf16_bits(vh);
                    lo[u] = float_to_bf16_bits(vl);
                }
                *reinterpret_cast<uint4 *>(tile + off) = *reinterpret_cast<const uint4 *>(hi);
                *reinterpret_cast<uint4 *>(sLo + off) = *reinterpret_cast<const uint4 *>(lo);
            }
            __syncthreads();
        }

        const int64_t t = it * G.tpi + slot;
        const bool valid = active && t < T;

        float accY[kMax / 16][2][4];
#pragma unroll
        for (int i2 = 0; i2 < kMax / 16; ++i2)
#pragma unroll
            for (int jt = 0; jt < 2; ++jt)
#pragma unroll
                for (int r = 0; r < 4; ++r) accY[i2][jt][r] = 0.0f;

        if (active) {
            // ---- stage 1: Z^T[j0..j0+15][a] -------------------------------
            float accZ[kMax / 8][4];
#pragma unroll
            for (int c = 0; c < kMax / 8; ++c)
#pragma unroll
                for (int r = 0; r < 4; ++r) accZ[c][r] = 0.0f;
            const int mat = lane >> 3, mr = lane & 7;
#pragma unroll
            for (int pass = 0; pass < (SCALED ? 2 : 1); ++pass) {
                const uint16_t *src = (pass ? sLo : sX + stage * G.tile) + slot * n1 * G.xs;
#pragma unroll
                for (int ks = 0; ks < kMax / 16; ++ks) {
                    if (ks < nk1) {
#pragma unroll
                        for (int c = 0; c < kMax / 8; c += 2) {
                            if (c < nc) {
                                uint32_t b[4];
                                ldmatrix_x4(b, src + (8 * (c + (mat >> 1)) + mr) * G.xs + 16 * ks +
                                                   8 * (mat & 1));
                                mma_bf16_16816(accZ[c], aP2[ks], b[0], b[1]);
                                mma_bf16_16816(accZ[c + 1], aP2[ks], b[2], b[3]);
                            }
                        }
                    }
                }
            }
            // ---- Z -> hi/lo bf16 B fragments (k = a, n = j) -------------------
            uint32_t bHi[kMax / 16][2][2], bLo[kMax / 16][2][2];
#pragma unroll
            for (int k2 = 0; k2 < kMax / 16; ++k2)
#pragma unroll
                for (int jt = 0; jt < 2; ++jt) {
                    float h0, l0, h1, l1, h2, l2, h3, l3;
                    split_bf16(accZ[2 * k2][2 * jt], h0, l0);
                    split_bf16(accZ[2 * k2][2 * jt + 1], h1, l1);
                    split_bf16(accZ[2 * k2 + 1][2 * jt], h2, l2);
                    split_bf16(accZ[2 * k2 + 1][2 * jt + 1], h3, l3);
                    bHi[k2][jt][0] = pack_bf16x2(h0, h1);
                    bHi[k2][jt][1] = pack_bf16x2(h2, h3);
                    bLo[k2][jt][0] = pack_bf16x2(l0, l1);
                    bLo[k2][jt][1] = pack_bf16x2(l2, l3);
                }
            // ---- stage 2: Y~[i][j0..j0+15] = P1^T Z ----------------------------
#pragma unroll
            for (int i2 = 0; i2 < kMax / 16; ++i2) {
                if (i2 < nk2) {
#pragma unroll
                    for (int k2 = 0; k2 < kMax / 16; ++k2) {
                        if (k2 < nk2) {
                            uint32_t a[4];
                            ldmatrix_x4(a, sP1T + (16 * i2 + 8 * (mat & 1) + mr) * G.p1s + 16 * k2 +
                                               8 * (mat >> 1));
#pragma unroll
                            for (int jt = 0; jt < 2; ++jt) {
                                mma_bf16_16816(accY[i2][jt], a, bHi[k2][jt][0], bHi[k2][jt][1]);
                                mma_bf16_16816(accY[i2][jt], a, bLo[k2][jt][0], bLo[k2][jt][1]);
                            }
                        }
                    }
                }
            }
        }

        if (QUANT) {
            // ---- per-token absmax across the token's warps -------------------
            float mloc = 0.0f;
#pragma unroll
            for (int i2 = 0; i2 < kMax / 16; ++i2)
                if (i2 < nk2)
#pragma unroll
                    for (int jt = 0; jt < 2; ++jt)
#pragma unroll
                        for (int r = 0; r < 4; ++r) mloc = fmaxf(mloc, fabsf(accY[i2][jt][r]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
            if (active && lane == 0) sRed[slot * G.wpt + jb] = mloc;
            __syncthreads();
            float m = 0.0f;
            if (active)
                for (int w = 0; w < G.wpt; ++w) m = fmaxf(m, sRed[slot * G.wpt + w]);
            const float s = alpha * m / 7.0f;
            if (active) {
                uint8_t *ob = sOut + slot * (G.n / 2);
#pragma unroll
                for (int i2 = 0; i2 < kMax / 16; ++i2)
                    if (i2 < nk2)
#pragma unroll
                        for (int jt = 0; jt < 2; ++jt) {
                            const int r0 = 16 * i2 + g, col = (j0 + 8 * jt + 2 * q4) >> 1;
                            const int c0 = quant_int4(accY[i2][jt][0], s);
                            const int c1 = quant_int4(accY[i2][jt][1], s);
                            const int c2 = quant_int4(accY[i2][jt][2], s);
                            const int c3 = quant_int4(accY[i2][jt][3], s);
                            ob[r0 * (n2 / 2) + col] = uint8_t((c0 & 0xF) | ((c1 & 0xF) << 4));
                            ob[(r0 + 8) * (n2 / 2) + col] = uint8_t((c2 & 0xF) | ((c3 & 0xF) << 4));
                        }
                if (valid && lane == 0 && jb == 0) scale_out[t] = s;
            }
            __syncthreads();
            const int v16_tok = G.n / 32;  // 16-byte vectors per token of output
            for (int e = tid; e < G.tpi * v16_tok; e += kThreads) {
                const int s2 = e / v16_tok, v = e - s2 * v16_tok;
                const int64_t t2 = it * G.tpi + s2;
                if (t2 < T)
                    reinterpret_cast<uint4 *>(q_out + t2 * (G.n / 2))[v] =
                        reinterpret_cast<const uint4 *>(sOut + s2 * (G.n / 2))[v];
            }
        } else if (valid) {
            float *yt = y_out + t * G.n;
#pragma unroll
            for (int i2 = 0; i2 < kMax / 16; ++i2)
                if (i2 < nk2)
#pragma unroll
                    for (int jt = 0; jt < 2; ++jt) {
                        const int r0 = 16 * i2 + g, col = j0 + 8 * jt + 2 * q4;
                        *reinterpret_cast<float2 *>(yt + r0 * n2 + col) =
                            make_float2(accY[i2][jt][0], accY[i2][jt][1]);
                        *reinterpret_cast<float2 *>(yt + (r0 + 8) * n2 + col) =
                            make_float2(accY[i2][jt][2], accY[i2][jt][3]);
                    }
        }
        __syncthreads();
    }
    cp_async_wait<0>();
}

template <bool SCALED, bool QUANT>
cudaError_t launch_variant(const LaunchArgs &a) {
    const Geometry G = make_geometry(a.n1, a.n2);
    const Layout L = make_layout(G, SCALED, QUANT);
    auto kern = kq_warp_mma_kernel<SCALED, QUANT>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(L.total));
    if (err != cudaSuccess) return err;
    int occ = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, L.total);
    if (err != cudaSuccess) return err;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    const int64_t n_iter = (a.T + G.tpi - 1) / G.tpi;
    int64_t grid = int64_t(a.num_sms) * occ;
    if (grid > n_iter) grid = n_iter;
    return launch_overlapped(kern, static_cast<unsigned>(grid), kThreads, L.total, a.stream, a.x, a.P1, a.P2, a.cinv,
                             a.alpha, a.q_out, a.scale_out, a.y_out, a.T, a.n1, a.n2);
}

}  // namespace

cudaError_t launch_warp_mma(const LaunchArgs &a) {
    const bool scaled = a.cinv != nullptr, quant = a.y_out == nullptr;
    if (scaled)
        return quant ? launch_variant<true, true>(a) : launch_variant<true, false>(a);
    return quant ? launch_variant<false, true>(a) : launch_variant<false, false>(a);
}

}  // namespace kq
