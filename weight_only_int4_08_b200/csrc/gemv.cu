// CUDA-core split-K GEMV for the W4A16 layer, M <= 8 activation rows per launch.
//
// Operation (vLLM PR #37352 analysis page, "코드 분석 1", `_w4a16_reference`):
//   out[m, n] = fp16( sum_g s[g, n] * sum_{k in g} a[m, k] * (q[k, n] - z[g, n]) )
// with fp32 accumulation. The scale is applied once per group in fp32, after the
// group's products a * (q - z), which are exact in fp32 (an 11-bit fp16
// significand times a 4-bit integer).
//
// Work decomposition (the weight stream is the whole cost: K*N/2 bytes):
//   - a CTA (256 threads, 8 warps) owns a 256-column tile (32 packed words per
//     row) and a contiguous slab of K rows (split-K: gridDim.y slabs);
//   - inside a warp, lane = (k-lane, chunk-lane): CL = 32/VEC chunk lanes read
//     VEC consecutive words each, so every load instruction moves whole
//     128-byte row segments (the one-block-per-row / warp-reduction GEMV of the
//     "Criando do zero um motor de inferência" page, section 3.2, turned so the
//     reduction runs over K because the packed words run along N);
//   - each of the CTA's 8*VEC k-threads walks a contiguous run of rows, split at
//     group boundaries; per group it accumulates sum_k a*(q - z') with the zero
//     folded out (sum a*q - z * sum a), then adds s * (that) into its totals;
//   - k-threads are reduced with __shfl_xor_sync inside the warp and through
//     shared memory across warps; CTAs of one column tile are reduced by the
//     last-arriving CTA, which sums the fp32 partials in slab order (fixed
//     order, no floating-point atomics: results are bit-reproducible).
//
// Nibble unpack: OR-ing a nibble field (w & (0xF << 4i)) into the fraction of
// the float 2^23 (bits 0x4B000000) gives exactly 2^23 + 2^(4i) q. One packed
// fp32 subtract (FADD2) removes 2^23, leaving 2^(4i) q exactly; the 2^(4i)
// factor is folded into the per-column scale at the group end. Packed fp32
// FMA (FFMA2, sm_100) then does two columns per instruction.
#include "common.cuh"

#include <algorithm>

namespace w4a16 {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTileWords = 32;             // packed words per column tile (256 columns)
constexpr int kTileCols = 8 * kTileWords;
constexpr int kMaxRowsPerCta = 1024;       // bounds the staged activations

struct GemvArgs {
    const __half* a;      // [M, K]
    const uint32_t* b;    // [K, N/8]
    const __half* s;      // [K/G, N]
    const uint32_t* z;    // [K/G, N/8] or nullptr
    __half* out;          // [M, N]
    float* partials;      // [split][MT][N]
    uint32_t* counters;   // [col_tiles]
    int64_t N, K;
    int G, zp_bias, split;
};

// 2^23 + 2^(4i) q for the nibble field `bits` (already masked in place).
__device__ __forceinline__ float magic(uint32_t bits) { return __uint_as_float(bits | 0x4B000000u); }

// Unpack one packed word into four column pairs holding 2^(4(j%4)) * q_j.
__device__ __forceinline__ void unpack_word(uint32_t w, float2 (&d)[4]) {
    const float2 bias = make_float2(-8388608.0f, -8388608.0f);
    const uint32_t h = w >> 16;
    d[0] = __fadd2_rn(make_float2(magic(w & 0x000Fu), magic(w & 0x00F0u)), bias);
    d[1] = __fadd2_rn(make_float2(magic(w & 0x0F00u), magic(w & 0xF000u)), bias);
    d[2] = __fadd2_rn(make_float2(magic(h & 0x000Fu), magic(h & 0x00F0u)), bias);
    d[3] = __fadd2_rn(make_float2(magic(h & 0x0F00u), magic(h & 0xF000u)), bias);
}

template <int VEC>
__device__ __forceinline__ void load_words(const uint32_t* p, uint32_t (&w)[VEC]) {
    if constexpr (VEC == 4) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (VEC == 2) {
        uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        w[0] = v.x; w[1] = v.y;
    } else {
        w[0] = __ldg(p);
    }
}

template <int MT, int VEC>
__global__ void __launch_bounds__(kThreads, (MT <= 3 ? 2 : 1))
gemv_kernel(GemvArgs p) {
    constexpr int CL = kTileWords / VEC;   // chunk lanes per warp
    constexpr int KL = 32 / CL;            // k lanes per warp (== VEC)
    constexpr int KT = kWarps * KL;        // k-threads per CTA
    constexpr int NP = 4 * VEC;            // column pairs per thread
    constexpr int U = 8;                   // rows per load batch (8 * VEC words in flight)

    extern __shared__ float2 s_act[];      // [MT][rows_cta] pairs (a, a)
    __shared__ float s_red[kWarps][kTileCols];
    __shared__ int s_last;

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int cl = lane % CL;
    const int kl = lane / CL;
    const int kthread = warp * KL + kl;

    const int64_t nw_total = p.N / 8;
    const int64_t w0 = (int64_t)blockIdx.x * kTileWords + cl * VEC;
    const bool col_ok = w0 < nw_total;

    const int64_t K = p.K;
    const int64_t r_begin = K * blockIdx.y / p.split;
    const int64_t r_end = K * (blockIdx.y + 1) / p.split;
    const int rows_cta = (int)(r_end - r_begin);

    // Stage this slab's activations as fp32 pairs (a, a) for the packed FMA.
    for (int i = threadIdx.x; i < MT * rows_cta; i += kThreads) {
        const int m = i / rows_cta, r = i - m * rows_cta;
        const float v = __half2float(p.a[(int64_t)m * K + r_begin + r]);
        s_act[i] = make_float2(v, v);
    }
    __syncthreads();

    const int64_t lo = r_begin + (int64_t)rows_cta * kthread / KT;
    const int64_t hi = r_begin + (int64_t)rows_cta * (kthread + 1) / KT;

    float2 tot[MT][NP];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int i = 0; i < NP; ++i) tot[m][i] = make_float2(0.f, 0.f);

    int64_t r = lo;
    while (r < hi) {
        const int64_t g = r / p.G;
        const int64_t seg_end = min(hi, (g + 1) * (int64_t)p.G);
        float2 gacc[MT][NP];
        float asum[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            asum[m] = 0.f;
#pragma unroll
            for (int i = 0; i < NP; ++i) gacc[m][i] = make_float2(0.f, 0.f);
        }
        for (int64_t rb = r; rb < seg_end; rb += U) {
            uint32_t wv[U][VEC];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (col_ok && rb + u < seg_end) {
                    load_words<VEC>(p.b + (rb + u) * nw_total + w0, wv[u]);
                } else {
#pragma unroll
                    for (int v = 0; v < VEC; ++v) wv[u][v] = 0u;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const bool row_ok = rb + u < seg_end;
                float2 av[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    av[m] = row_ok ? s_act[m * rows_cta + (int)(rb + u - r_begin)] : make_float2(0.f, 0.f);
                    asum[m] += av[m].x;
                }
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    float2 d[4];
                    unpack_word(wv[u][v], d);
#pragma unroll
                    for (int m = 0; m < MT; ++m)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            gacc[m][4 * v + i] = __ffma2_rn(av[m], d[i], gacc[m][4 * v + i]);
                }
            }
        }
        r = seg_end;
        // Group end: tot += s * (gacc * 2^-(4(j%4)) - z * sum a).
        if (col_ok) {
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                const int64_t word = w0 + v;
                const uint32_t zw = p.z ? __ldg(p.z + g * nw_total + word) : 0u;
                const __half* sp = p.s + g * p.N + word * 8;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float sc = __half2float(__ldg(sp + j));
                    const float zf = p.z ? (float)((zw >> (4 * j)) & 0xFu) : (float)p.zp_bias;
                    const float f = (j % 4 == 0) ? 1.0f : (j % 4 == 1) ? 0.0625f : (j % 4 == 2) ? 0.00390625f : 0.000244140625f;
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        float2& gp = gacc[m][4 * v + j / 2];
                        float2& tp = tot[m][4 * v + j / 2];
                        const float ga = (j & 1) ? gp.y : gp.x;
                        const float t = fmaf(-zf, asum[m], ga * f);
                        if (j & 1) tp.y = fmaf(sc, t, tp.y); else tp.x = fmaf(sc, t, tp.x);
                    }
                }
            }
        }
    }

    // Reduce the KL k-lanes of each warp (lanes differing in the bits above CL).
#pragma unroll
    for (int off = CL; off < 32; off <<= 1)
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                tot[m][i].x += __shfl_xor_sync(0xffffffffu, tot[m][i].x, off);
                tot[m][i].y += __shfl_xor_sync(0xffffffffu, tot[m][i].y, off);
            }

    const int64_t n0 = (int64_t)blockIdx.x * kTileCols;
    const int64_t n = n0 + threadIdx.x;
    const bool n_ok = n < p.N;
    float part[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        if (kl == 0) {
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                const int c = 8 * cl * VEC + 2 * i;
                s_red[warp][c] = tot[m][i].x;
                s_red[warp][c + 1] = tot[m][i].y;
            }
        }
        __syncthreads();
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) acc += s_red[w][threadIdx.x];
        part[m] = acc;
        __syncthreads();
    }

    if (p.split == 1) {
        if (n_ok)
#pragma unroll
            for (int m = 0; m < MT; ++m) p.out[(int64_t)m * p.N + n] = __float2half_rn(part[m]);
        return;
    }

    // Split-K: publish this slab's partial, the last CTA of the tile sums all slabs in order.
    if (n_ok)
#pragma unroll
        for (int m = 0; m < MT; ++m)
            p.partials[((int64_t)blockIdx.y * MT + m) * p.N + n] = part[m];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t ticket = atomicAdd(p.counters + blockIdx.x, 1u);
        s_last = (ticket == (uint32_t)p.split - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (n_ok) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float acc = 0.f;
            for (int y = 0; y < p.split; ++y) acc += __ldcg(p.partials + ((int64_t)y * MT + m) * p.N + n);
            p.out[(int64_t)m * p.N + n] = __float2half_rn(acc);
        }
    }
    if (threadIdx.x == 0) p.counters[blockIdx.x] = 0u;  // leave the workspace as found
}

template <int MT, int VEC>
cudaError_t launch_one(const GemvArgs& args, dim3 grid, size_t smem, cudaStream_t st) {
    auto kern = gemv_kernel<MT, VEC>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<grid, kThreads, smem, st>>>(args);
    return cudaGetLastError();
}

template <int MT>
cudaError_t launch_vec(int vec, const GemvArgs& args, dim3 grid, size_t smem, cudaStream_t st) {
    // Only the (rows, vector width) pairs plan_gemv can pick are instantiated.
    if constexpr (MT == 1) {
        if (vec == 4) return launch_one<MT, 4>(args, grid, smem, st);
        if (vec == 2) return launch_one<MT, 2>(args, grid, smem, st);
    } else if constexpr (MT == 2) {
        if (vec >= 2) return launch_one<MT, 2>(args, grid, smem, st);
    }
    return launch_one<MT, 1>(args, grid, smem, st);
}

}  // namespace

GemvPlan plan_gemv(int64_t M, int64_t N, int64_t K, int32_t G, int split_k_request, int sm_count, int max_vec) {
    (void)G;
    GemvPlan pl{};
    pl.m_rows = (int)std::min<int64_t>(M, 8);
    const int64_t nw = N / 8;
    int vec = (nw % 4 == 0) ? 4 : (nw % 2 == 0) ? 2 : 1;
    // Register budget: MT * 8 * VEC columns, twice (group and running sums).
    vec = std::min(vec, std::max(max_vec, 1));
    if (pl.m_rows >= 3) vec = 1;
    else if (pl.m_rows == 2) vec = std::min(vec, 2);
    pl.vec = vec;
    pl.col_tiles = (int)((N + kTileCols - 1) / kTileCols);
    const int ctas_per_sm = pl.m_rows <= 3 ? 2 : 1;
    const int64_t target = (int64_t)std::max(sm_count, 1) * ctas_per_sm;
    int64_t split = split_k_request > 0 ? split_k_request : (target + pl.col_tiles - 1) / pl.col_tiles;
    if (split_k_request <= 0) {
        // At least one row per warp; independent of VEC so the workspace query
        // (made without the weight pointer) matches every launch.
        split = std::max<int64_t>(split, (K + kMaxRowsPerCta - 1) / kMaxRowsPerCta);
        split = std::min<int64_t>(split, std::max<int64_t>(1, K / kWarps));
        split = std::min<int64_t>(split, 256);
    }
    pl.split_k = (int)std::max<int64_t>(1, split);
    pl.counters_off = kWsHeader;
    pl.partials_off = align_up(kWsHeader + (size_t)pl.col_tiles * 4, 256);
    pl.ws_bytes = pl.split_k > 1 ? pl.partials_off + (size_t)pl.split_k * pl.m_rows * (size_t)N * 4 : 0;
    return pl;
}

size_t gemv_smem_bytes(int64_t M, int64_t K, int split_k) {
    const int64_t rows_cta = (K + split_k - 1) / split_k;
    return (size_t)std::min<int64_t>(M, 8) * (size_t)rows_cta * sizeof(float2);
}

cudaError_t launch_gemv(const __half* a, const uint32_t* b, const __half* s, const uint32_t* z,
                        int64_t M, int64_t N, int64_t K, int32_t G, int32_t zp_bias, __half* out,
                        void* workspace, const GemvPlan& pl, cudaStream_t st) {
    const int64_t rows_cta = (K + pl.split_k - 1) / pl.split_k;
    for (int64_t m0 = 0; m0 < M; m0 += 8) {
        const int mt = (int)std::min<int64_t>(8, M - m0);
        GemvArgs args;
        args.a = a + m0 * K;
        args.b = b;
        args.s = s;
        args.z = z;
        args.out = out + m0 * N;
        args.partials = pl.split_k > 1 ? reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.partials_off) : nullptr;
        args.counters = pl.split_k > 1 ? reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + pl.counters_off) : nullptr;
        args.N = N;
        args.K = K;
        args.G = G;
        args.zp_bias = zp_bias;
        args.split = pl.split_k;
        const dim3 grid((unsigned)pl.col_tiles, (unsigned)pl.split_k);
        const size_t smem = (size_t)mt * (size_t)rows_cta * sizeof(float2);
        cudaError_t e;
        switch (mt) {
            case 1: e = launch_vec<1>(pl.vec, args, grid, smem, st); break;
            case 2: e = launch_vec<2>(pl.vec, args, grid, smem, st); break;
            case 3: e = launch_vec<3>(pl.vec, args, grid, smem, st); break;
            case 4: e = launch_vec<4>(pl.vec, args, grid, smem, st); break;
            case 5: e = launch_vec<5>(pl.vec, args, grid, smem, st); break;
            case 6: e = launch_vec<6>(pl.vec, args, grid, smem, st); break;
            case 7: e = launch_vec<7>(pl.vec, args, grid, smem, st); break;
            default: e = launch_vec<8>(pl.vec, args, grid, smem, st); break;
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace w4a16
