// Checkpoint [N, K/8] -> kernel [K, N/8] int4 weight repack (bit-exact), and the
// whole-layer load conversion that also moves the per-group scales [N, K/G] ->
// [K/G, N] and zeros [N/8, K/G] -> [K/G, N/8] in the same launch.
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

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Transpose an 8x8 matrix of nibbles held as 8 words (row i = word i, column j =
// nibble j) in place, by exchanging off-diagonal blocks of size 4, then 2, then 1:
// the 16-bit and 8-bit levels are byte permutes (prmt), the nibble level a shift
// and a bit select per word. Measured on B200: the shift/xor form of all three
// levels left the repack ALU-bound (ALU pipe ~70 %, issue ~73 %).
__device__ __forceinline__ void nibble_transpose8(uint32_t (&x)[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {   // 16-bit halves: x[i] = (lo x[i], lo x[i+4]), x[i+4] = (hi, hi)
        const uint32_t a = x[i], b = x[i + 4];
        x[i] = prmt(a, b, 0x5410);
        x[i + 4] = prmt(a, b, 0x7632);
    }
#pragma unroll
    for (int base = 0; base < 8; base += 4) {
#pragma unroll
        for (int i = base; i < base + 2; ++i) {   // bytes: x[i] = (a0 b0 a2 b2), x[i+2] = (a1 b1 a3 b3)
            const uint32_t a = x[i], b = x[i + 2];
            x[i] = prmt(a, b, 0x6240);
            x[i + 2] = prmt(a, b, 0x7351);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; i += 2) {   // nibbles of each byte: x[i] = (lo b, lo a), x[i+1] = (hi b, hi a)
        const uint32_t a = x[i], b = x[i + 1];
        x[i] = (a & 0x0F0F0F0Fu) | ((b << 4) & 0xF0F0F0F0u);
        x[i + 1] = ((a >> 4) & 0x0F0F0F0Fu) | (b & 0xF0F0F0F0u);
    }
}

// One 256 (n) x 256 (k) tile of the weight repack; (bx, by) = (k-word tile, n tile).
__device__ __forceinline__ void repack_tile(const uint32_t* __restrict__ ckpt, uint32_t* __restrict__ out, int64_t N,
                                            int64_t K, int64_t bx, int64_t by, uint32_t* tile) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t kw_total = K / 8;   // checkpoint words per row
    const int64_t nw_total = N / 8;   // kernel words per row
    const int64_t kw0 = bx * kTileWords;  // first checkpoint word column
    const int64_t n0 = by * kTileRows;    // first n row
    const bool full = n0 + kTileRows <= N && kw0 + kTileWords <= kw_total;   // no bounds checks needed

    const int64_t kw = kw0 + lane;
    // Each warp transposes n-blocks b = warp, warp + 8, warp + 16, warp + 24. All 32 loads are
    // issued before the first transpose, so that each thread keeps 128 bytes in flight.
    constexpr int kBlocks = kTileWords / 8;
    uint32_t x[kBlocks][8];
    if (full) {
        const uint32_t* src = ckpt + (n0 + 8 * warp) * kw_total + kw;   // row n0 + 8 warp
        const int64_t block_step = 64 * kw_total;                        // 8 blocks of 8 rows
#pragma unroll
        for (int bb = 0; bb < kBlocks; ++bb) {
            const uint32_t* row = src + bb * block_step;
#pragma unroll
            for (int i = 0; i < 8; ++i) x[bb][i] = __ldg(row + i * kw_total);
        }
    } else {
#pragma unroll
        for (int bb = 0; bb < kBlocks; ++bb)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int64_t n = n0 + 8 * (warp + 8 * bb) + i;
                x[bb][i] = (n < N && kw < kw_total) ? __ldg(ckpt + n * kw_total + kw) : 0u;
            }
    }
#pragma unroll
    for (int bb = 0; bb < kBlocks; ++bb) {
        const int b = warp + 8 * bb;
        nibble_transpose8(x[bb]);
        // x[bb][i] now holds q[k = 8*kw + i, n = n0 + 8b .. n0 + 8b + 7]
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = 8 * lane + i;  // k_local; r / 8 == lane
            tile[r * kTileWords + (b ^ lane)] = x[bb][i];
        }
    }
    __syncthreads();
    const int64_t k0 = kw0 * 8;
    const int64_t nw = (n0 >> 3) + lane;
    if (full) {
        uint32_t* dst = out + (k0 + warp) * nw_total + nw;
        const int64_t step = (int64_t)(kThreads / 32) * nw_total;
#pragma unroll 8
        for (int r = warp; r < kTileRows; r += kThreads / 32, dst += step) *dst = tile[r * kTileWords + (lane ^ (r >> 3))];
    } else {
#pragma unroll 4
        for (int r = warp; r < kTileRows; r += kThreads / 32) {
            const int64_t k = k0 + r;
            if (k < K && nw < nw_total)
                out[k * nw_total + nw] = tile[r * kTileWords + (lane ^ (r >> 3))];
        }
    }
}

__global__ void __launch_bounds__(kThreads)
repack_kernel(const uint32_t* __restrict__ ckpt, uint32_t* __restrict__ out, int64_t N, int64_t K) {
    __shared__ uint32_t tile[kTileRows * kTileWords];  // [k_local][n_word ^ swz]
    repack_tile(ckpt, out, N, K, blockIdx.x, blockIdx.y, tile);
}

// out[c][r] = in[r][c] for one 32 x 32 tile (tr, tc) of an R x C matrix of T.
// Lane = column on both sides, so loads and stores are row segments; the tile's
// row pitch of 33 elements keeps the column reads of 32-bit T conflict free.
template <typename T>
__device__ __forceinline__ void transpose_tile(const T* __restrict__ in, T* __restrict__ out, int64_t R, int64_t C,
                                               int64_t tr, int64_t tc, T* tile) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t r0 = tr * 32, c0 = tc * 32;
#pragma unroll
    for (int y = warp; y < 32; y += kThreads / 32) {
        const int64_t r = r0 + y, c = c0 + lane;
        if (r < R && c < C) tile[y * 33 + lane] = in[r * C + c];
    }
    __syncthreads();
#pragma unroll
    for (int y = warp; y < 32; y += kThreads / 32) {
        const int64_t c = c0 + y, r = r0 + lane;
        if (r < R && c < C) out[c * R + r] = tile[lane * 33 + y];
    }
}

struct CtLoadArgs {
    const uint32_t* ckpt;   // [N, K/8]
    const uint16_t* s_ng;   // [N, K/G]
    const uint32_t* z_n8g;  // [N/8, K/G] or null
    uint32_t* b_kn8;        // [K, N/8]
    uint16_t* s_gn;         // [K/G, N]
    uint32_t* z_gn8;        // [K/G, N/8] or null
    int64_t N, K, ngroups;
    int64_t rep_x, rep_blocks;   // weight tiles: x extent, count
    int64_t s_tc, s_blocks;      // scale tiles: column-tile extent, count
    int64_t z_tc;                // zero tiles: column-tile extent
};

// The whole layer in one launch: blocks [0, rep_blocks) repack weight tiles, the
// next s_blocks transpose scale tiles, the rest transpose zero tiles.
__global__ void __launch_bounds__(kThreads) ct_load_kernel(const CtLoadArgs p) {
    __shared__ uint32_t smem[kTileRows * kTileWords];
    int64_t b = blockIdx.x;
    if (b < p.rep_blocks) {
        repack_tile(p.ckpt, p.b_kn8, p.N, p.K, b % p.rep_x, b / p.rep_x, smem);
        return;
    }
    b -= p.rep_blocks;
    if (b < p.s_blocks) {
        transpose_tile<uint16_t>(p.s_ng, p.s_gn, p.N, p.ngroups, b / p.s_tc, b % p.s_tc,
                                 reinterpret_cast<uint16_t*>(smem));
        return;
    }
    b -= p.s_blocks;
    transpose_tile<uint32_t>(p.z_n8g, p.z_gn8, p.N / 8, p.ngroups, b / p.z_tc, b % p.z_tc, smem);
}

}  // namespace

cudaError_t launch_repack(const uint32_t* ckpt, uint32_t* out, int64_t N, int64_t K, cudaStream_t st) {
    const int64_t gx = (K / 8 + kTileWords - 1) / kTileWords;
    const int64_t gy = (N + kTileRows - 1) / kTileRows;
    if (gx > 0x7fffffff || gy > 65535) return cudaErrorInvalidValue;
    repack_kernel<<<dim3((unsigned)gx, (unsigned)gy), kThreads, 0, st>>>(ckpt, out, N, K);
    return cudaGetLastError();
}

cudaError_t launch_ct_load(const uint32_t* ckpt, const uint16_t* s_ng, const uint32_t* z_n8g, uint32_t* b_kn8,
                           uint16_t* s_gn, uint32_t* z_gn8, int64_t N, int64_t K, int64_t ngroups, cudaStream_t st) {
    CtLoadArgs p{ckpt, s_ng, z_n8g, b_kn8, s_gn, z_gn8, N, K, ngroups, 0, 0, 0, 0, 0};
    p.rep_x = (K / 8 + kTileWords - 1) / kTileWords;
    p.rep_blocks = p.rep_x * ((N + kTileRows - 1) / kTileRows);
    p.s_tc = (ngroups + 31) / 32;
    p.s_blocks = p.s_tc * ((N + 31) / 32);
    p.z_tc = p.s_tc;
    const int64_t z_blocks = z_n8g ? p.z_tc * ((N / 8 + 31) / 32) : 0;
    const int64_t blocks = p.rep_blocks + p.s_blocks + z_blocks;
    if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
    ct_load_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace w4a16
