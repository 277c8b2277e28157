// Checkpoint [N, K/8] -> kernel [K, N/8] int4 weight repack (bit-exact).
//
// Operation: section "2. 가중치 레이아웃 재포장 (Weight Repacking)" of the vLLM
// PR #37352 analysis page. Checkpoint word (n, c) holds q[8c + j, n] in nibble j;
// kernel word (k, d) holds q[k, 8d + j] in nibble j.
//
// Design (HBM-bound permutation, 8 bytes moved per 16 nibbles... i.e. one read
// and one write of every byte):
//   - a CTA owns a 256 (n) x 256 (k) tile: 256 checkpoint rows of 32 words in,
//     256 kernel rows of 32 words out;
//   - lane = checkpoint word column, so every warp load is one 128-byte row
//     segment; each thread gathers the 8 words of an 8x8 nibble block (8
//     consecutive n, one word of 8 consecutive k) and transposes it in registers
//     with three rounds of masked block swaps (4x4, 2x2, 1x1 nibble blocks);
//   - the 8 transposed words are parked in a 32 KB shared tile with an XOR
//     swizzle (column ^= row/8) so both the scattered writes and the row reads
//     are bank-conflict free, then every warp stores whole 128-byte output rows.
#include "common.cuh"

namespace w4a16 {
namespace {

constexpr int kTileWords = 32;            // words per tile row, both sides
constexpr int kTileRows = 8 * kTileWords; // 256 rows (n on input, k on output)
constexpr int kThreads = 256;

// Transpose an 8x8 matrix of nibbles held as 8 words (row i = word i, column j =
// nibble j) in place, by swapping off-diagonal blocks of size 4, then 2, then 1.
__device__ __forceinline__ void nibble_transpose8(uint32_t (&x)[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t t = ((x[i] >> 16) ^ x[i + 4]) & 0x0000FFFFu;
        x[i] ^= t << 16;
        x[i + 4] ^= t;
    }
#pragma unroll
    for (int base = 0; base < 8; base += 4) {
#pragma unroll
        for (int i = base; i < base + 2; ++i) {
            uint32_t t = ((x[i] >> 8) ^ x[i + 2]) & 0x00FF00FFu;
            x[i] ^= t << 8;
            x[i + 2] ^= t;
        }
    }
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        uint32_t t = ((x[i] >> 4) ^ x[i + 1]) & 0x0F0F0F0Fu;
        x[i] ^= t << 4;
        x[i + 1] ^= t;
    }
}

__global__ void __launch_bounds__(kThreads)
repack_kernel(const uint32_t* __restrict__ ckpt, uint32_t* __restrict__ out, int64_t N, int64_t K) {
    __shared__ uint32_t tile[kTileRows * kTileWords];  // [k_local][n_word ^ swz]
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t kw_total = K / 8;   // checkpoint words per row
    const int64_t nw_total = N / 8;   // kernel words per row
    const int64_t kw0 = (int64_t)blockIdx.x * kTileWords;  // first checkpoint word column
    const int64_t n0 = (int64_t)blockIdx.y * kTileRows;    // first n row

    const int64_t kw = kw0 + lane;
    // Each warp transposes n-blocks b = warp, warp + 8, warp + 16, warp + 24.
#pragma unroll
    for (int bb = 0; bb < kTileWords / 8; ++bb) {
        const int b = warp + 8 * bb;
        uint32_t x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t n = n0 + 8 * b + i;
            x[i] = (n < N && kw < kw_total) ? __ldg(ckpt + n * kw_total + kw) : 0u;
        }
        nibble_transpose8(x);
        // x[i] now holds q[k = 8*kw + i, n = n0 + 8b .. n0 + 8b + 7]
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = 8 * lane + i;  // k_local; r / 8 == lane
            tile[r * kTileWords + (b ^ lane)] = x[i];
        }
    }
    __syncthreads();
    const int64_t k0 = kw0 * 8;
    const int64_t nw = (n0 >> 3) + lane;
#pragma unroll 4
    for (int r = warp; r < kTileRows; r += kThreads / 32) {
        const int64_t k = k0 + r;
        if (k < K && nw < nw_total)
            out[k * nw_total + nw] = tile[r * kTileWords + (lane ^ (r >> 3))];
    }
}

}  // namespace

cudaError_t launch_repack(const uint32_t* ckpt, uint32_t* out, int64_t N, int64_t K, cudaStream_t st) {
    const int64_t gx = (K / 8 + kTileWords - 1) / kTileWords;
    const int64_t gy = (N + kTileRows - 1) / kTileRows;
    if (gx > 0x7fffffff || gy > 65535) return cudaErrorInvalidValue;
    repack_kernel<<<dim3((unsigned)gx, (unsigned)gy), kThreads, 0, st>>>(ckpt, out, N, K);
    return cudaGetLastError();
}

}  // namespace w4a16
