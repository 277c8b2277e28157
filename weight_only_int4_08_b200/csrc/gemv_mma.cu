// Split-K GEMV for M <= 8 whose multiply-accumulate runs on warp-level tensor
// instructions (mma.sync.m16n8k16, fp16 inputs, fp32 accumulation), with the
// CUDA cores doing only the nibble unpack.
//
// Operation (vLLM PR #37352 analysis page, "코드 분석 1", `_w4a16_reference`):
//   out[m, n] = fp16( sum_g s[g, n] * sum_{k in g} a[m, k] * (q[k, n] - z[g, n]) ),
// fp32 accumulation; (q - z) is formed exactly in fp16, its products with the
// fp16 activations are exact in the fp32 accumulator, and the group scale is
// applied in fp32 to each group's accumulator.
//
// Why tensor instructions for a GEMV: measured on B200, the pure CUDA-core
// inner loop (fp32 "magic number" unpack, packed FADD2/FFMA2) executes about
// 41 instructions per packed word of 8 weights and is issue-bound well below
// the HBM rate. Here a register holds two k-rows of four columns after one
// ldmatrix.trans, and 9 instructions turn it into four exact (q - z) fp16 pairs
// (0x6400 magic OR, fp16 subtract or fused scale-subtract); one mma.sync then
// does 16 x 16 x 8 multiply-adds. The MMA's batch dimension (8) is padded for
// M < 8; tensor throughput is not the bound.
//
// Work decomposition: a CTA owns a 128-column tile (16 packed words per row)
// and a K slab (split-K over gridDim.y); each of its 8 warps streams its own
// run of 32-row blocks through a private ring of shared-memory stages filled
// by 2-D TMA loads (64-byte swizzle, which makes the transposed ldmatrix reads
// bank-conflict free). Swap-AB: the MMA's rows are output columns
// (A = dequantised weights, transposed by ldmatrix), its columns the
// activation rows (B). Warps are reduced through shared memory; split-K slabs
// by the last-arriving CTA in slab order (deterministic).
//
// Register layout (lane = 4 g + t): ldmatrix.trans gives thread (g, t) the
// k-pair t of an 8-row matrix for columns 4g..4g+3 of a 32-column chunk; MMA 1
// takes columns 4g (row g) and 4g+1 (row g+8), MMA 2 columns 4g+2 and 4g+3;
// the accumulator d0..d3 = (row g, batch 2t), (row g, 2t+1), (row g+8, 2t),
// (row g+8, 2t+1).
#include "common.cuh"
#include "ptx.cuh"

#include <algorithm>
#include <atomic>

namespace w4a16 {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = 8;
constexpr int kTileN = 128;
constexpr int kTileWords = kTileN / 8;            // 16 packed words = 64 B per row
constexpr int kRows = 32;                         // rows per TMA stage
constexpr int kStage = kRows * kTileWords * 4;    // 2 KB
constexpr int kRing = 4;                          // stages in flight per warp
constexpr int kRingBytes = kWarps * kRing * kStage;
constexpr int kMaxRowsPerCta = 2048;

struct MmaArgs {
    const __half* a;      // [M, K]
    const __half* s;      // [K/G, N]
    const uint32_t* z;    // [K/G, N/8] or nullptr
    __half* out;          // [M, N] (row block)
    float* partials;      // [split][MT][N]
    uint32_t* counters;   // [col_tiles]
    int* status;
    int64_t N, K;
    int G, zp_bias, split, s_vec, stall_loads;
    uint64_t wait_ns;
};

__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

__device__ __forceinline__ void mma16816(float& d0, float& d1, float& d2, float& d3, uint32_t a0, uint32_t a1,
                                         uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

constexpr uint32_t kMagic = 0x64006400u;   // fp16 1024.0 in both halves
constexpr uint32_t kSixteenth = 0x2C002C00u;  // fp16 1/16 in both halves

// Per chunk (32 columns) and thread: four columns 4g..4g+3. Low-nibble columns
// (j = 0, 2) subtract (1024 + z); high-nibble columns (j = 1, 3), unpacked as
// 1024 + 16 q, are scaled by 1/16 and lose (64 + z) in one fused fp16 op.
struct ChunkMeta {
    uint32_t bias[4];   // j even: (1024 + z) x2; j odd: -(64 + z) x2  (fp16 bits)
    float s[4];         // fp32 scales of the four columns
};

template <int MT>
__global__ void __launch_bounds__(kThreads)
gemv_mma_kernel(const __grid_constant__ CUtensorMap bmap, MmaArgs p) {
    extern __shared__ __align__(1024) unsigned char s_dyn[];
    unsigned char* ring = s_dyn;                                            // [8][kRing][2 KB]
    uint32_t* s_act = reinterpret_cast<uint32_t*>(s_dyn + kRingBytes);      // [MT][rows/2] fp16 pairs
    __shared__ __align__(8) uint64_t s_full[kWarps][kRing];
    __shared__ int s_last;
    __shared__ volatile int s_abort;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t nw = p.N / 8;

    const int64_t nblk_total = (p.K + kRows - 1) / kRows;
    const int64_t blk_begin = nblk_total * blockIdx.y / p.split;
    const int64_t blk_end = nblk_total * (blockIdx.y + 1) / p.split;
    const int64_t r_begin = blk_begin * kRows;
    const int64_t r_end = min(blk_end * kRows, p.K);
    const int rows_cta = (int)(r_end - r_begin);      // a multiple of 16
    const int nblk = (int)(blk_end - blk_begin);
    const int b_lo = nblk * warp / kWarps, b_hi = nblk * (warp + 1) / kWarps;
    const int nmine = b_hi - b_lo;

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int w = 0; w < kWarps; ++w)
            for (int j = 0; j < kRing; ++j) ptx::mbar_init(ptx::smem_addr(&s_full[w][j]), 1);
        ptx::mbar_fence_init();
    }
    __syncthreads();

    auto arm = [&](int j) {
        const int slot = j % kRing;
        const uint32_t bar = ptx::smem_addr(&s_full[warp][slot]);
        ptx::mbar_arrive_expect_tx(bar, (uint32_t)kStage);
        ptx::tma_load_2d(ptx::smem_addr(ring + (size_t)(warp * kRing + slot) * kStage), &bmap,
                         (int32_t)(blockIdx.x * kTileWords), (int32_t)(r_begin + (int64_t)(b_lo + j) * kRows), bar);
    };
    if (lane == 0 && !p.stall_loads) {
        ptx::prefetch_tensormap(&bmap);
        for (int j = 0; j < min(kRing, nmine); ++j) arm(j);
    }
    // Activations of this slab as fp16 pairs (k, k+1).
    const int half_rows = rows_cta / 2;
    for (int i = threadIdx.x; i < MT * half_rows; i += kThreads) {
        const int m = i / half_rows, r2 = i - m * half_rows;
        s_act[i] = *reinterpret_cast<const uint32_t*>(p.a + (int64_t)m * p.K + r_begin + 2 * r2);
    }
    __syncthreads();

    float tot[4][8], acc[4][8];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 8; ++i) tot[c][i] = 0.f;
    ChunkMeta meta[4];
    int64_t g_cur = -1, g_next = 0;
    const int64_t word0 = (int64_t)blockIdx.x * kTileWords + g / 2;   // + 4c: the word holding my columns
    const int zshift = 16 * (g & 1);   // my first column is nibble 4 (g & 1) of that word
    const int64_t ncol0 = (int64_t)blockIdx.x * kTileN + 4 * g;        // + 32c + j: my columns

    auto group_end = [&]() {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            tot[c][0] = fmaf(meta[c].s[0], acc[c][0], tot[c][0]);
            tot[c][1] = fmaf(meta[c].s[0], acc[c][1], tot[c][1]);
            tot[c][2] = fmaf(meta[c].s[1], acc[c][2], tot[c][2]);
            tot[c][3] = fmaf(meta[c].s[1], acc[c][3], tot[c][3]);
            tot[c][4] = fmaf(meta[c].s[2], acc[c][4], tot[c][4]);
            tot[c][5] = fmaf(meta[c].s[2], acc[c][5], tot[c][5]);
            tot[c][6] = fmaf(meta[c].s[3], acc[c][6], tot[c][6]);
            tot[c][7] = fmaf(meta[c].s[3], acc[c][7], tot[c][7]);
        }
    };
    auto group_start = [&](int64_t gg) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int64_t word = word0 + 4 * c;
            const bool ok = word < nw;
            uint32_t zw = (uint32_t)p.zp_bias * 0x1111u;
            if (p.z && ok) zw = __ldg(p.z + gg * nw + word) >> zshift;
            meta[c].bias[0] = (0x6400u + (zw & 0xFu)) * 0x00010001u;
            // -(64 + z): 0xD400 is -64 and one unit of the fraction is 1/16 there
            meta[c].bias[1] = (0xD400u + 16u * ((zw >> 4) & 0xFu)) * 0x00010001u;
            meta[c].bias[2] = (0x6400u + ((zw >> 8) & 0xFu)) * 0x00010001u;
            meta[c].bias[3] = (0xD400u + 16u * ((zw >> 12) & 0xFu)) * 0x00010001u;
            const __half* sp = p.s + gg * p.N + ncol0 + 32 * c;
#pragma unroll
            for (int j = 0; j < 4; ++j) meta[c].s[j] = ok ? __half2float(__ldg(sp + j)) : 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[c][i] = 0.f;
        }
    };

    int consumed = 0;
    for (int j = 0; j < nmine; ++j) {
        const int slot = j % kRing;
        const bool okw = ptx::mbar_wait(ptx::smem_addr(&s_full[warp][slot]), (uint32_t)((j / kRing) & 1), &s_abort,
                                        p.wait_ns);
        if (!__all_sync(0xffffffffu, okw)) break;
        consumed = j + 1;
        const int64_t rs = r_begin + (int64_t)(b_lo + j) * kRows;
        const int64_t re = min(rs + kRows, r_end);
        // Four chunks x four 8-row matrices, transposed: R[c][i] holds k-rows 8i + 2t, 8i + 2t + 1
        // of columns 32c + 4g .. 32c + 4g + 3. My address row is `lane`; the 64-byte swizzle
        // moves 16-byte chunk c of row r to chunk c ^ ((r >> 1) & 3).
        const uint32_t sbase = ptx::smem_addr(ring + (size_t)(warp * kRing + slot) * kStage) + lane * 64;
        uint32_t R[4][4];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::ldmatrix_x4_trans(sbase + 16 * (c ^ ((lane >> 1) & 3)), R[c]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t k0 = rs + 16 * h;
            if (k0 >= re) break;
            if (k0 >= g_next) {
                if (g_cur >= 0) group_end();
                g_cur = k0 / p.G;
                g_next = (g_cur + 1) * p.G;
                group_start(g_cur);
            }
            // B fragment: batch row g (zero past M), k-pairs t and t + 4 of this 16-k step.
            uint32_t b0 = 0u, b1 = 0u;
            if (g < MT) {
                const uint32_t* ap = s_act + g * (rows_cta / 2) + (k0 - r_begin) / 2 + t;
                b0 = ap[0];
                b1 = ap[4];
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t x0 = R[c][2 * h], x1 = R[c][2 * h + 1];
                const uint32_t y0 = x0 >> 8, y1 = x1 >> 8;
                const uint32_t e0a = hsub2((x0 & 0x000F000Fu) | kMagic, meta[c].bias[0]);
                const uint32_t e1a = hfma2((x0 & 0x00F000F0u) | kMagic, kSixteenth, meta[c].bias[1]);
                const uint32_t e0b = hsub2((x1 & 0x000F000Fu) | kMagic, meta[c].bias[0]);
                const uint32_t e1b = hfma2((x1 & 0x00F000F0u) | kMagic, kSixteenth, meta[c].bias[1]);
                const uint32_t e2a = hsub2((y0 & 0x000F000Fu) | kMagic, meta[c].bias[2]);
                const uint32_t e3a = hfma2((y0 & 0x00F000F0u) | kMagic, kSixteenth, meta[c].bias[3]);
                const uint32_t e2b = hsub2((y1 & 0x000F000Fu) | kMagic, meta[c].bias[2]);
                const uint32_t e3b = hfma2((y1 & 0x00F000F0u) | kMagic, kSixteenth, meta[c].bias[3]);
                mma16816(acc[c][0], acc[c][1], acc[c][2], acc[c][3], e0a, e1a, e0b, e1b, b0, b1);
                mma16816(acc[c][4], acc[c][5], acc[c][6], acc[c][7], e2a, e3a, e2b, e3b, b0, b1);
            }
        }
        // Every lane has consumed its ldmatrix results: the stage can be refilled.
        __syncwarp();
        if (lane == 0 && j + kRing < nmine && !p.stall_loads) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            arm(j + kRing);
        }
    }
    if (g_cur >= 0) group_end();

    if (s_abort) {
        if (lane == 0) {
            for (int j = consumed; j < min(nmine, consumed + kRing) && !p.stall_loads; ++j) {
                volatile int dummy = 0;
                ptx::mbar_wait(ptx::smem_addr(&s_full[warp][j % kRing]), (uint32_t)((j / kRing) & 1), &dummy, p.wait_ns);
            }
            if (p.status) atomicExch(p.status, (int)W4A16_ERR_TIMEOUT);
        }
    }
    __syncthreads();  // rings are free: reuse them for the warp reduction
    if (s_abort) return;

    // Warp reduction: s_red[w][m][128] (m < MT); thread values map to
    // (column 32c + 4g + j, batch 2t + (i & 1)) with j = 0,1 from MMA 1 and 2,3 from MMA 2.
    float* s_red = reinterpret_cast<float*>(s_dyn);
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int m = 2 * t + (i & 1);
            const int jcol = (i < 4) ? (i >> 1) : 2 + ((i - 4) >> 1);
            if (m < MT) s_red[(warp * MT + m) * kTileN + 32 * c + 4 * g + jcol] = tot[c][i];
        }
    __syncthreads();
    const int64_t n0 = (int64_t)blockIdx.x * kTileN;
    for (int item = threadIdx.x; item < MT * kTileN; item += kThreads) {
        const int m = item / kTileN, nl = item % kTileN;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += s_red[(w * MT + m) * kTileN + nl];
        const int64_t n = n0 + nl;
        if (n < p.N) {
            if (p.split == 1) p.out[(int64_t)m * p.N + n] = __float2half_rn(v);
            else p.partials[((int64_t)blockIdx.y * MT + m) * p.N + n] = v;
        }
    }
    if (p.split == 1) return;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t ticket = atomicAdd(p.counters + blockIdx.x, 1u);
        s_last = (ticket == (uint32_t)p.split - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int item = threadIdx.x; item < MT * kTileN; item += kThreads) {
        const int m = item / kTileN, nl = item % kTileN;
        const int64_t n = n0 + nl;
        if (n >= p.N) continue;
        float v = 0.f;
        for (int y = 0; y < p.split; ++y) v += __ldcg(p.partials + ((int64_t)y * MT + m) * p.N + n);
        p.out[(int64_t)m * p.N + n] = __float2half_rn(v);
    }
    if (threadIdx.x == 0) p.counters[blockIdx.x] = 0u;
}

using MmaFn = void (*)(CUtensorMap, MmaArgs);

MmaFn select_mma(int mt) {
    switch (mt) {
        case 1: return gemv_mma_kernel<1>;
        case 2: return gemv_mma_kernel<2>;
        case 3: return gemv_mma_kernel<3>;
        case 4: return gemv_mma_kernel<4>;
        case 5: return gemv_mma_kernel<5>;
        case 6: return gemv_mma_kernel<6>;
        case 7: return gemv_mma_kernel<7>;
        default: return gemv_mma_kernel<8>;
    }
}

std::atomic<int> g_mma_occ[9];

size_t act_smem(int mt, int64_t rows) { return (size_t)mt * (size_t)rows * 2; }

int mma_ctas_per_sm(int mt) {
    int n = g_mma_occ[mt].load(std::memory_order_relaxed);
    if (n > 0) return n;
    MmaFn k = select_mma(mt);
    cudaFuncAttributes fa{};
    int regs = 255;
    if (cudaFuncGetAttributes(&fa, k) == cudaSuccess && fa.numRegs > 0) regs = fa.numRegs;
    const size_t smem = kRingBytes + act_smem(mt, kMaxRowsPerCta) + fa.sharedSizeBytes + 1024;
    const int by_smem = (int)((228 * 1024) / smem);
    const int by_regs = 65536 / (((regs + 7) / 8 * 8) * kThreads);
    n = std::max(1, std::min(by_smem, by_regs));
    g_mma_occ[mt].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace

bool gemv_mma_supported(int64_t N, const void* a, const void* b) {
    return N % 32 == 0 && (reinterpret_cast<uintptr_t>(b) % 16) == 0 && (reinterpret_cast<uintptr_t>(a) % 4) == 0;
}

GemvPlan plan_gemv_mma(int64_t M, int64_t N, int64_t K, int32_t G, int split_k_request, int sm_count) {
    (void)G;
    GemvPlan pl{};
    pl.tma = true;
    pl.mma = true;
    pl.vec = 1;
    pl.m_rows = (int)std::min<int64_t>(M, 8);
    pl.col_tiles = (int)((N + kTileN - 1) / kTileN);
    const int64_t nblk = (K + kRows - 1) / kRows;
    int64_t split;
    if (split_k_request > 0) {
        split = std::min<int64_t>(split_k_request, nblk);
    } else {
        // Fill whole waves of resident CTAs best; count the fp32 partials a split writes and
        // reads as traffic against the packed weights; at most kMaxRowsPerCta rows per CTA.
        const int64_t slots = (int64_t)std::max(sm_count, 1) * mma_ctas_per_sm(pl.m_rows);
        const int64_t smin = std::max<int64_t>(1, (K + kMaxRowsPerCta - 1) / kMaxRowsPerCta);
        double best = -1.0;
        split = smin;
        for (int64_t sp = smin; sp <= std::min<int64_t>(nblk, 64); ++sp) {
            const int64_t ctas = (int64_t)pl.col_tiles * sp;
            const double waves = (double)((ctas + slots - 1) / slots);
            const double fill = (double)ctas / (waves * (double)slots);
            const double wb = (double)K * (double)N / 2;
            const double pb = sp > 1 ? 2.0 * sp * pl.m_rows * (double)N * 4 : 0.0;
            const double score = fill * wb / (wb + pb) / (1.0 + 0.02 * waves);
            if (score > best + 1e-9) {
                best = score;
                split = sp;
            }
        }
    }
    pl.split_k = (int)std::max<int64_t>(1, split);
    pl.counters_off = kWsHeader;
    pl.partials_off = align_up(kWsHeader + (size_t)pl.col_tiles * 4, 256);
    pl.ws_bytes = pl.partials_off + (pl.split_k > 1 ? (size_t)pl.split_k * pl.m_rows * (size_t)N * 4 : 0);
    return pl;
}

cudaError_t launch_gemv_mma(const __half* a, const uint32_t* b, const __half* s, const uint32_t* z, int64_t M,
                            int64_t N, int64_t K, int32_t G, int32_t zp_bias, __half* out, void* workspace,
                            const GemvPlan& pl, const WaitPolicy& wp, cudaStream_t st) {
    CUtensorMap bmap;
    const cuuint64_t dims[2] = {(cuuint64_t)(N / 8), (cuuint64_t)K};
    const cuuint64_t strides[1] = {(cuuint64_t)(N / 8) * 4};
    const cuuint32_t box[2] = {(cuuint32_t)kTileWords, (cuuint32_t)kRows};
    const cuuint32_t estr[2] = {1, 1};
    cudaError_t e = encode_tensor_map(&bmap, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, (void*)b, dims, strides, box, estr,
                                      CU_TENSOR_MAP_SWIZZLE_64B);
    if (e != cudaSuccess) return e;
    const int64_t nblk = (K + kRows - 1) / kRows;
    const int64_t rows_max = (nblk + pl.split_k - 1) / pl.split_k * kRows;
    char* ws = static_cast<char*>(workspace);
    for (int64_t m0 = 0; m0 < M; m0 += 8) {
        const int mt = (int)std::min<int64_t>(8, M - m0);
        MmaArgs args;
        args.a = a + m0 * K;
        args.s = s;
        args.z = z;
        args.out = out + m0 * N;
        args.partials = reinterpret_cast<float*>(ws + pl.partials_off);
        args.counters = reinterpret_cast<uint32_t*>(ws + pl.counters_off);
        args.status = reinterpret_cast<int*>(ws);
        args.N = N;
        args.K = K;
        args.G = G;
        args.zp_bias = zp_bias;
        args.split = pl.split_k;
        args.s_vec = 0;
        args.stall_loads = wp.stall_loads;
        args.wait_ns = wp.limit_ns;
        const size_t smem = kRingBytes + act_smem(mt, rows_max);
        MmaFn k = select_mma(mt);
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k<<<dim3((unsigned)pl.col_tiles, (unsigned)pl.split_k), kThreads, smem, st>>>(bmap, args);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace w4a16
