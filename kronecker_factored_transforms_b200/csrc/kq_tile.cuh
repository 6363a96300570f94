// kq_tile.cuh -- layouts shared by the tcgen05 transform kernels: the 128-byte
// swizzle of K-major bf16 tiles, the TMEM lane permutation of the output
// columns, the block-diagonal P^T operand and the swizzled staging rows of
// the packed codes.
#pragma once

#include <stdint.h>

namespace kq {
namespace tile {

// Offset of byte b of staging row r: rows of n2/2 bytes with the 16-byte chunks
// permuted the way a TMA store with 64-byte (n2 = 128) or 32-byte (n2 = 64)
// swizzle reads them back in order.  It also spreads the epilogue's 16-bit
// stores over all banks.
template <int N2>
__host__ __device__ constexpr uint32_t stg_offset(int r, int b) {
    const int swz = N2 == 128 ? (r >> 1) & 3 : (r >> 2) & 1;
    return uint32_t(r * (N2 / 2) + ((((b >> 4) ^ swz) << 4) | (b & 15)));
}

// The epilogue writes staging row row0 + 16 c + 8 rep + 2 qq + d, byte column
// bcol, at base(qq, bcol) + (16 c + 8 rep + d) * n2/2; checked here against
// stg_offset for every thread and store of an n1 x n2 group.
template <int N1, int N2>
__host__ __device__ constexpr bool staging_addresses_match() {
    constexpr int H = 128 / N2, RB = N2 / 2;
    for (int q = 0; q < 4; ++q)
        for (int g8 = 0; g8 < 8; ++g8)
            for (int qq = 0; qq < 4; ++qq) {
                const int row0 = ((32 * q) / N2) * N1, bcol = ((32 * q) % N2) / 2 + 2 * g8;
                const int swz_t = N2 == 128 ? qq : (qq >> 1);
                const int base = (row0 + 2 * qq) * RB + ((((bcol >> 4) ^ swz_t) << 4) | (bcol & 15));
                for (int c = 0; c < N1 / 16; ++c)
                    for (int rep = 0; rep < 2; ++rep)
                        for (int d = 0; d < 2; ++d) {
                            const int r = row0 + 16 * c + 8 * rep + 2 * qq + d;
                            if (r >= H * N1 || uint32_t(base + (16 * c + 8 * rep + d) * RB) != stg_offset<N2>(r, bcol) ||
                                uint32_t(base + (16 * c + 8 * rep + d) * RB) + 2 > uint32_t(H * N1 * RB))
                                return false;
                        }
            }
    return true;
}

// Byte offset of element (row r, k in [0, 64)) inside one 128B-swizzled chunk.
__device__ __forceinline__ uint32_t swz128(int r, int k) {
    return uint32_t(r * 128 + ((((k >> 3) ^ (r & 7)) << 4) | ((k & 7) << 1)));
}

// Output column held by TMEM lane m of a token (m < n2).  Within each block of
// 32 lanes, lane 16 f + 8 s + g holds column 4 g + 2 f + s, so the thread
// that a 16x256b load gives lanes g and g + 8 of both 16-lane halves holds
// four consecutive columns: two whole bytes of every output row.
__host__ __device__ constexpr int lane_column(int m) {
    return (m & ~31) | ((m & 7) << 2) | (((m >> 4) & 1) << 1) | ((m >> 3) & 1);
}

// Inverse of lane_column: the lane (within a token) that holds output column j.
__host__ __device__ constexpr int lane_of_column(int j) {
    return (j & ~31) | (((j >> 1) & 1) << 4) | ((j & 1) << 3) | ((j >> 2) & 7);
}

__host__ __device__ constexpr bool lane_maps_invert() {
    for (int m = 0; m < 128; ++m)
        if (lane_of_column(lane_column(m)) != m || lane_column(m) >= 128) return false;
    return true;
}
static_assert(lane_maps_invert(), "lane_of_column inverts lane_column");

// Row l of A1 = block-diag over the stacked tokens of P2^T, rows permuted:
// A1[l][k] = P2[b][lane_column(m)] for l = (h, m), k = (h, b); zero off the
// diagonal blocks.  Tokens take N2P >= n2 lanes and K values each; rows and
// columns past n2 (a padded n2) are zero.
template <int N2, int N2P = N2>
__device__ __forceinline__ uint16_t a1_value(const uint16_t *__restrict__ P2, int l, int k) {
    const int h = l / N2P, m = l % N2P, hk = k / N2P, b = k % N2P, j = lane_column(m);
    return (h == hk && b < N2 && j < N2) ? P2[b * N2 + j] : uint16_t(0);
}

}  // namespace tile
}  // namespace kq
