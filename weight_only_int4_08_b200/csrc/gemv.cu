// CUDA-core split-K GEMV for the W4A16 layer, M <= 8 activation rows per launch.
//
// Operation (vLLM PR #37352 analysis page, "코드 분석 1", `_w4a16_reference`):
//   out[m, n] = fp16( sum_g s[g, n] * sum_{k in g} a[m, k] * (q[k, n] - z[g, n]) )
// with fp32 accumulation. The scale is applied once per group in fp32, after the
// group's sums of a * (q - z), whose products are exact in fp32 (an 11-bit fp16
// significand times a small integer).
//
// Work decomposition (the weight stream is the whole cost: K*N/2 bytes):
//   - a CTA (8 warps) owns a column tile of 32*V packed words (256*V columns)
//     and a contiguous slab of K rows (split-K: gridDim.y slabs);
//   - lane l of every warp owns words [V*l, V*l + V) of the tile, so a row of
//     the tile is one 128*V-byte segment (the one-block-per-row, warp-reduction
//     GEMV of the "Criando do zero um motor de inferência" page, section 3.2,
//     turned so the reduction runs over K because the packed words run along N);
//   - each warp walks a contiguous run of rows; all its lanes take the same
//     path (group boundaries are per warp);
//   - the 8 warps are reduced through shared memory; the CTAs of one column
//     tile by the last-arriving CTA, which sums the fp32 partials in slab
//     order (fixed order, no floating-point atomics: bit-reproducible);
//   - the grid is sized from the occupancy query so every CTA runs in a single
//     wave (split = resident CTA slots / column tiles).
//
// Two kernels share that structure:
//   gemv_tma: every warp streams its rows through a private ring of shared
//     memory stages filled by 2-D TMA tile loads (cp.async.bulk.tensor) and
//     tracked by mbarriers, so several stages are in flight while it computes
//     (needs N % 32 == 0 and a 16-byte aligned weight pointer);
//   gemv_ldg: plain vector loads into registers, U rows per batch (any N % 8
//     == 0, any 4-byte alignment).
//
// Inner loop: OR each nibble field (w & 0xF<<4i) into the fraction of 2^23
// (bits 0x4B000000) to get exactly 2^23 + 2^(4i) q. The group's zero word is
// unpacked the same way, so one packed fp32 add (FADD2, of the negated zero
// pair) leaves exactly 2^(4i) (q - z) for two columns, and one packed fp32 FMA
// (FFMA2) accumulates them against the activation; the power of two 2^(4i) is
// folded into the group-end scale. A column with q == z adds exactly nothing.
#include "common.cuh"
#include "ptx.cuh"

#include <algorithm>
#include <atomic>

namespace w4a16 {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRowsPerCta = 1024;          // bounds the staged activations
constexpr int kRing = 4;                      // TMA stages per warp
constexpr int kStageBytes = 2048;             // bytes per TMA stage
#ifndef W4A16_GEMV_SCALAR_FMA
#define W4A16_GEMV_SCALAR_FMA 0               // 1: scalar fp32 add/FMA instead of the packed forms
#endif
#ifndef W4A16_GEMV_M1_VEC
#define W4A16_GEMV_M1_VEC 2                   // packed words per lane for one activation row
#endif

struct GemvArgs {
    const __half* a;      // [M, K]
    const uint32_t* b;    // [K, N/8]
    const __half* s;      // [K/G, N]
    const uint32_t* z;    // [K/G, N/8] or nullptr
    OutPtr out;           // [M, N]
    float* partials;      // [split][MT][N]
    uint32_t* counters;   // [col_tiles]
    int* status;          // workspace status word (TMA kernel), or nullptr
    int64_t N, K;
    int G, zp_bias, split;
    int rows_per_stage;   // TMA kernel: rows per ring stage (box height)
    int s_vec;            // scales pointer is 16-byte aligned (vector loads)
    int stall_loads;      // tests only: issue no loads (every wait runs out)
    uint64_t wait_ns;     // limit on each device-side wait
};

template <int V>
__device__ __forceinline__ void load_words(const uint32_t* p, uint32_t (&w)[V]) {
    if constexpr (V == 4) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (V == 2) {
        uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        w[0] = v.x; w[1] = v.y;
    } else {
        w[0] = __ldg(p);
    }
}

template <int V>
__device__ __forceinline__ void lds_words(const uint32_t* p, uint32_t (&w)[V]) {
    if constexpr (V == 2) {
        uint2 v = *reinterpret_cast<const uint2*>(p);
        w[0] = v.x; w[1] = v.y;
    } else if constexpr (V == 4) {
        uint4 v = *reinterpret_cast<const uint4*>(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
        w[0] = *p;
    }
}

// fp32 form of the exponent-bias ("magic number") unpack (Kim et al. 2022; Frantar et al. 2024,
// MARLIN), from the IEEE-754 layout: 0x4B000000 is 2^23, whose ulp is 1, so OR-ing an integer
// below 2^23 into its mantissa gives exactly 2^23 + that integer.
__device__ __forceinline__ float magic(uint32_t bits) { return __uint_as_float(bits | 0x4B000000u); }

// Column pairs (0,1) (2,3) (4,5) (6,7) of one packed word as 2^23 + 2^(4(j%4)) * q_j.
__device__ __forceinline__ void unpack_raw(uint32_t w, float2 (&d)[4]) {
    const uint32_t h = w >> 16;
    d[0] = make_float2(magic(w & 0x000Fu), magic(w & 0x00F0u));
    d[1] = make_float2(magic(w & 0x0F00u), magic(w & 0xF000u));
    d[2] = make_float2(magic(h & 0x000Fu), magic(h & 0x00F0u));
    d[3] = make_float2(magic(h & 0x0F00u), magic(h & 0xF000u));
}

// Group metadata for the lane's V words: 8*V fp16 scales and, per column pair,
// -(2^23 + 2^(4(j%4)) z_j).
template <int V>
struct GroupMeta {
    uint32_t s[V][4];   // 8 halves per word
    float2 nz[V][4];
};

template <int V>
__device__ __forceinline__ void load_meta(const GemvArgs& p, int64_t g, int64_t w0, GroupMeta<V>& gm) {
    const int64_t nw = p.N / 8;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const __half* sp = p.s + g * p.N + (w0 + v) * 8;
        if (p.s_vec) {
            const uint4 sv = __ldg(reinterpret_cast<const uint4*>(sp));
            gm.s[v][0] = sv.x; gm.s[v][1] = sv.y; gm.s[v][2] = sv.z; gm.s[v][3] = sv.w;
        } else {  // scales not 16-byte aligned: eight 2-byte loads
            const unsigned short* sh = reinterpret_cast<const unsigned short*>(sp);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                gm.s[v][i] = (uint32_t)__ldg(sh + 2 * i) | ((uint32_t)__ldg(sh + 2 * i + 1) << 16);
        }
        const uint32_t zw = p.z ? __ldg(p.z + g * nw + w0 + v) : (uint32_t)p.zp_bias * 0x11111111u;
        float2 zr[4];
        unpack_raw(zw, zr);
#pragma unroll
        for (int i = 0; i < 4; ++i) gm.nz[v][i] = make_float2(-zr[i].x, -zr[i].y);
    }
}

// One row: gacc[m][c] += a[m] * 2^(4(c%4)) (q - z) for the lane's 8*V columns.
template <int MT, int V>
__device__ __forceinline__ void accumulate_row(float2 (&gacc)[MT][4 * V], const uint32_t (&wv)[V],
                                               const GroupMeta<V>& gm, const float2* act, int stride) {
    float2 d[V][4];
#pragma unroll
    for (int v = 0; v < V; ++v) {
        unpack_raw(wv[v], d[v]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#if W4A16_GEMV_SCALAR_FMA
            d[v][i].x += gm.nz[v][i].x;
            d[v][i].y += gm.nz[v][i].y;
#else
            d[v][i] = __fadd2_rn(d[v][i], gm.nz[v][i]);
#endif
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        const float2 av = act[m * stride];
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#if W4A16_GEMV_SCALAR_FMA
                gacc[m][4 * v + i].x = fmaf(av.x, d[v][i].x, gacc[m][4 * v + i].x);
                gacc[m][4 * v + i].y = fmaf(av.x, d[v][i].y, gacc[m][4 * v + i].y);
#else
                gacc[m][4 * v + i] = __ffma2_rn(av, d[v][i], gacc[m][4 * v + i]);
#endif
            }
    }
}

// tot += s * 2^-(4(c%4)) * gacc.
template <int MT, int V>
__device__ __forceinline__ void group_end(float2 (&tot)[MT][4 * V], const float2 (&gacc)[MT][4 * V],
                                          const GroupMeta<V>& gm) {
#pragma unroll
    for (int v = 0; v < V; ++v) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // columns 2i and 2i+1 of word v: factors 2^-(4(2i%4)), 2^-(4((2i+1)%4))
            const float f0 = (i & 1) ? 0.00390625f : 1.0f;
            const float f1 = (i & 1) ? 0.000244140625f : 0.0625f;
            const uint32_t sp = gm.s[v][i];
            const float2 sc = make_float2(__half2float(__ushort_as_half((uint16_t)(sp & 0xFFFFu))) * f0,
                                          __half2float(__ushort_as_half((uint16_t)(sp >> 16))) * f1);
#pragma unroll
            for (int m = 0; m < MT; ++m) tot[m][4 * v + i] = __ffma2_rn(sc, gacc[m][4 * v + i], tot[m][4 * v + i]);
        }
    }
}

template <int MT, int V>
__device__ __forceinline__ void zero_acc(float2 (&x)[MT][4 * V]) {
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int c = 0; c < 4 * V; ++c) x[m][c] = make_float2(0.f, 0.f);
}

// Reduce the 8 warps' totals through shared memory (s_red: 8 * 32 * (8V + 1)
// floats), then write the output (one slab) or the slab's partial and, in the
// last-arriving CTA of the column tile, the ordered sum of all slabs.
template <int MT, int V>
__device__ __forceinline__ void finish_cta(const GemvArgs& p, const float2 (&tot)[MT][4 * V], float* s_red, int* s_last) {
    constexpr int NC = 8 * V;
    constexpr int kTileCols = 32 * NC;
    constexpr int PER = kTileCols / kThreads;  // == V
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float part[MT][PER];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        // tile column c = lane * NC + j lives at s_red[warp][c + lane] (padded rows)
#pragma unroll
        for (int c = 0; c < NC / 2; ++c) {
            s_red[warp * 32 * (NC + 1) + lane * (NC + 1) + 2 * c] = tot[m][c].x;
            s_red[warp * 32 * (NC + 1) + lane * (NC + 1) + 2 * c + 1] = tot[m][c].y;
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const int col = threadIdx.x + q * kThreads;
            const int idx = col + col / NC;
            float acc = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) acc += s_red[w * 32 * (NC + 1) + idx];
            part[m][q] = acc;
        }
        __syncthreads();
    }
    const int64_t n0 = (int64_t)blockIdx.x * kTileCols;
    if (p.split == 1) {
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const int64_t n = n0 + threadIdx.x + q * kThreads;
            if (n < p.N)
#pragma unroll
                for (int m = 0; m < MT; ++m) p.out.put((int64_t)m * p.N + n, part[m][q]);
        }
        return;
    }
#pragma unroll
    for (int q = 0; q < PER; ++q) {
        const int64_t n = n0 + threadIdx.x + q * kThreads;
        if (n < p.N)
#pragma unroll
            for (int m = 0; m < MT; ++m) p.partials[((int64_t)blockIdx.y * MT + m) * p.N + n] = part[m][q];
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t ticket = atomicAdd(p.counters + blockIdx.x, 1u);
        *s_last = (ticket == (uint32_t)p.split - 1);
    }
    __syncthreads();
    if (!*s_last) return;
    __threadfence();
#pragma unroll
    for (int q = 0; q < PER; ++q) {
        const int64_t n = n0 + threadIdx.x + q * kThreads;
        if (n < p.N) {
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                float acc = 0.f;
                for (int y = 0; y < p.split; ++y) acc += __ldcg(p.partials + ((int64_t)y * MT + m) * p.N + n);
                p.out.put((int64_t)m * p.N + n, acc);
            }
        }
    }
    if (threadIdx.x == 0) p.counters[blockIdx.x] = 0u;  // leave the workspace as found
}

// Stage this slab's activation rows in shared memory as (a, a) pairs.
template <int MT>
__device__ __forceinline__ void stage_acts(const GemvArgs& p, float2* s_act, int64_t r_begin, int rows) {
    for (int i = threadIdx.x; i < MT * rows; i += kThreads) {
        const int m = i / rows, r = i - m * rows;
        const float v = __half2float(p.a[(int64_t)m * p.K + r_begin + r]);
        s_act[i] = make_float2(v, v);
    }
}

template <int V>
constexpr size_t red_bytes() { return (size_t)kWarps * 32 * (8 * V + 1) * sizeof(float); }

// ============================================================== TMA kernel ====
// Slabs are whole multiples of the stage height R (except the last one, cut by
// K); each warp takes a contiguous run of R-row blocks of its CTA's slab and
// keeps kRing of them in flight in its own ring of shared-memory stages.
// Dynamic shared memory: [ring 8 x kRing x 2 KB][activations]; the warp
// reduction reuses the ring once every warp is done with it.
template <int MT, int V>
__global__ void __launch_bounds__(kThreads)
gemv_tma_kernel(const __grid_constant__ CUtensorMap bmap, GemvArgs p) {
    constexpr int TW = 32 * V;  // words per tile row
    static_assert(red_bytes<V>() <= (size_t)kWarps * kRing * kStageBytes, "reduction buffer must fit in the ring");
    const int R = p.rows_per_stage;

    extern __shared__ __align__(1024) unsigned char s_dyn[];
    uint32_t* ring = reinterpret_cast<uint32_t*>(s_dyn);                       // [8][kRing][R][TW]
    float2* s_act = reinterpret_cast<float2*>(s_dyn + (size_t)kWarps * kRing * kStageBytes);
    __shared__ __align__(8) uint64_t s_full[kWarps][kRing];
    __shared__ int s_last;
    __shared__ volatile int s_abort;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t nw = p.N / 8;
    const int64_t w0 = (int64_t)blockIdx.x * TW + lane * V;
    const bool col_ok = w0 < nw;

    const int64_t nblk_total = (p.K + R - 1) / R;
    const int64_t blk_begin = nblk_total * blockIdx.y / p.split;
    const int64_t blk_end = nblk_total * (blockIdx.y + 1) / p.split;
    const int64_t r_begin = blk_begin * R;
    const int64_t r_end = min(blk_end * R, p.K);
    const int rows_cta = (int)(r_end - r_begin);

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int w = 0; w < kWarps; ++w)
            for (int j = 0; j < kRing; ++j) ptx::mbar_init(ptx::smem_addr(&s_full[w][j]), 1);
        ptx::mbar_fence_init();
    }
    // This warp's blocks [b_lo, b_hi) (indices relative to blk_begin).
    const int nblk = (int)(blk_end - blk_begin);
    const int b_lo = nblk * warp / kWarps, b_hi = nblk * (warp + 1) / kWarps;
    __syncthreads();

    auto arm = [&](int j) {  // issue the load of this warp's j-th block into ring slot j % kRing
        const int slot = j % kRing;
        const uint32_t bar = ptx::smem_addr(&s_full[warp][slot]);
        ptx::mbar_arrive_expect_tx(bar, (uint32_t)kStageBytes);
        const uint32_t dst = ptx::smem_addr(ring + ((size_t)warp * kRing + slot) * (kStageBytes / 4));
        ptx::tma_load_2d(dst, &bmap, (int32_t)(blockIdx.x * TW), (int32_t)(r_begin + (int64_t)(b_lo + j) * R), bar);
    };
    const int nmine = b_hi - b_lo;
    if (lane == 0 && !p.stall_loads) {
        ptx::prefetch_tensormap(&bmap);
        for (int j = 0; j < min(kRing, nmine); ++j) arm(j);
    }
    stage_acts<MT>(p, s_act, r_begin, rows_cta);
    __syncthreads();

    float2 tot[MT][4 * V], gacc[MT][4 * V];
    zero_acc<MT, V>(tot);
    GroupMeta<V> gm;
    int64_t g = -1, g_next = 0;

    int consumed = 0;
    for (int j = 0; j < nmine; ++j) {
        const int slot = j % kRing;
        // warp-uniform outcome: every lane takes the same path below
        const bool okw = ptx::mbar_wait(ptx::smem_addr(&s_full[warp][slot]), (uint32_t)((j / kRing) & 1), &s_abort,
                                        p.wait_ns);
        if (!__all_sync(0xffffffffu, okw)) break;
        consumed = j + 1;
        const uint32_t* buf = ring + ((size_t)warp * kRing + slot) * (kStageBytes / 4) + lane * V;
        const int64_t rs = r_begin + (int64_t)(b_lo + j) * R;     // first row of the block
        const int64_t re = min(rs + R, r_end);
        int64_t r = rs;
        while (r < re) {
            if (r >= g_next) {
                if (g >= 0 && col_ok) group_end<MT, V>(tot, gacc, gm);
                g = r / p.G;
                g_next = (g + 1) * p.G;
                if (col_ok) load_meta<V>(p, g, w0, gm);
                zero_acc<MT, V>(gacc);
            }
            const int64_t se = min(re, g_next);
            const float2* act = s_act + (r - r_begin);
            const uint32_t* rowp = buf + (r - rs) * TW;
            int cnt = (int)(se - r);
            for (; cnt >= 4; cnt -= 4, r += 4, act += 4, rowp += 4 * TW) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t wv[V];
                    lds_words<V>(rowp + u * TW, wv);
                    accumulate_row<MT, V>(gacc, wv, gm, act + u, rows_cta);
                }
            }
            for (; cnt > 0; --cnt, ++r, ++act, rowp += TW) {
                uint32_t wv[V];
                lds_words<V>(rowp, wv);
                accumulate_row<MT, V>(gacc, wv, gm, act, rows_cta);
            }
        }
        __syncwarp();
        if (lane == 0 && j + kRing < nmine && !p.stall_loads) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // our reads before the async refill
            arm(j + kRing);
        }
    }
    if (g >= 0 && col_ok) group_end<MT, V>(tot, gacc, gm);

    if (s_abort) {
        // Drain this warp's loads still in flight (bounded) before the CTA exits.
        if (lane == 0) {
            for (int j = consumed; j < min(nmine, consumed + kRing) && !p.stall_loads; ++j) {
                volatile int dummy = 0;
                ptx::mbar_wait(ptx::smem_addr(&s_full[warp][j % kRing]), (uint32_t)((j / kRing) & 1), &dummy, p.wait_ns);
            }
            if (p.status) atomicExch(p.status, (int)W4A16_ERR_TIMEOUT);
        }
    }
    __syncthreads();  // every warp is done with its ring: the reduction may reuse it
    if (s_abort) return;
    finish_cta<MT, V>(p, tot, reinterpret_cast<float*>(s_dyn), &s_last);
}

// ============================================================== LDG kernel ====
template <int MT, int V>
__global__ void __launch_bounds__(kThreads)
gemv_ldg_kernel(GemvArgs p) {
    constexpr int U = (V == 1) ? 16 : 8;  // rows per load batch
    extern __shared__ __align__(1024) unsigned char s_dyn[];
    float2* s_act = reinterpret_cast<float2*>(s_dyn);  // [MT][rows_cta]
    __shared__ float s_red[kWarps * 32 * (8 * V + 1)];
    __shared__ int s_last;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t nw = p.N / 8;
    const int64_t w0 = (int64_t)blockIdx.x * (32 * V) + lane * V;
    const bool col_ok = w0 < nw;
    const int64_t r_begin = p.K * blockIdx.y / p.split;
    const int64_t r_end = p.K * (blockIdx.y + 1) / p.split;
    const int rows_cta = (int)(r_end - r_begin);

    stage_acts<MT>(p, s_act, r_begin, rows_cta);
    __syncthreads();

    const int lo = rows_cta * warp / kWarps, hi = rows_cta * (warp + 1) / kWarps;
    float2 tot[MT][4 * V], gacc[MT][4 * V];
    zero_acc<MT, V>(tot);
    const uint32_t* bp = p.b + w0 + r_begin * nw;
    int r = lo;
    while (r < hi) {
        const int64_t g = (r_begin + r) / p.G;
        const int seg_end = (int)min((int64_t)hi, (g + 1) * (int64_t)p.G - r_begin);
        GroupMeta<V> gm;
        if (col_ok) load_meta<V>(p, g, w0, gm);
        zero_acc<MT, V>(gacc);
        for (int rb = r; rb < seg_end; rb += U) {
            const int nrows = min(U, seg_end - rb);
            const uint32_t* rp = bp + (int64_t)rb * nw;
            uint32_t wv[U][V];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (col_ok && u < nrows) {
                    load_words<V>(rp + u * nw, wv[u]);
                } else {
#pragma unroll
                    for (int v = 0; v < V; ++v) wv[u][v] = 0u;
                }
            }
            if (col_ok) {
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (u < nrows) accumulate_row<MT, V>(gacc, wv[u], gm, s_act + rb + u, rows_cta);
            }
        }
        r = seg_end;
        if (col_ok) group_end<MT, V>(tot, gacc, gm);
    }
    finish_cta<MT, V>(p, tot, s_red, &s_last);
}

// ================================================================ host side ===
using LdgFn = void (*)(GemvArgs);
using TmaFn = void (*)(CUtensorMap, GemvArgs);

// Only the (rows, vector width) pairs plan_gemv can pick are instantiated.
LdgFn select_ldg(int mt, int vec) {
    switch (mt) {
        case 1: return vec == 4 ? gemv_ldg_kernel<1, 4> : vec == 2 ? gemv_ldg_kernel<1, 2> : gemv_ldg_kernel<1, 1>;
        case 2: return vec >= 2 ? gemv_ldg_kernel<2, 2> : gemv_ldg_kernel<2, 1>;
        case 3: return gemv_ldg_kernel<3, 1>;
        case 4: return gemv_ldg_kernel<4, 1>;
        case 5: return gemv_ldg_kernel<5, 1>;
        case 6: return gemv_ldg_kernel<6, 1>;
        case 7: return gemv_ldg_kernel<7, 1>;
        default: return gemv_ldg_kernel<8, 1>;
    }
}

TmaFn select_tma(int mt, int vec) {
    switch (mt) {
        case 1: return vec >= 2 ? gemv_tma_kernel<1, 2> : gemv_tma_kernel<1, 1>;
        case 2: return gemv_tma_kernel<2, 1>;
        case 3: return gemv_tma_kernel<3, 1>;
        case 4: return gemv_tma_kernel<4, 1>;
        case 5: return gemv_tma_kernel<5, 1>;
        case 6: return gemv_tma_kernel<6, 1>;
        case 7: return gemv_tma_kernel<7, 1>;
        default: return gemv_tma_kernel<8, 1>;
    }
}

// Rows per TMA stage: one stage is R x (32*V) words = kStageBytes.
int tma_rows(int vec) { return kStageBytes / (128 * vec); }

constexpr size_t kRingBytes = (size_t)kWarps * kRing * kStageBytes;

// Resident CTAs per SM for each (kernel kind, rows, vector width), cached per process.
std::atomic<int> g_occ[2][9][5];

int ctas_per_sm(bool tma, int mt, int vec) {
    int n = g_occ[tma][mt][vec].load(std::memory_order_relaxed);
    if (n > 0) return n;
    size_t smem = (size_t)mt * kMaxRowsPerCta * sizeof(float2);
    cudaError_t e;
    if (tma) {
        smem += kRingBytes;
        TmaFn k = select_tma(mt, vec);
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kThreads, smem);
    } else {
        LdgFn k = select_ldg(mt, vec);
        if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kThreads, smem);
    }
    if (e != cudaSuccess || n < 1) n = 1;
    g_occ[tma][mt][vec].store(n, std::memory_order_relaxed);
    return n;
}

// Host encoding of the 2-D tensor map over the packed weights [K, N/8] (int32).
cudaError_t make_bmap(CUtensorMap* map, const uint32_t* b, int64_t N, int64_t K, int vec) {
    const cuuint64_t dims[2] = {(cuuint64_t)(N / 8), (cuuint64_t)K};
    const cuuint64_t strides[1] = {(cuuint64_t)(N / 8) * 4};
    const cuuint32_t box[2] = {(cuuint32_t)(32 * vec), (cuuint32_t)tma_rows(vec)};
    const cuuint32_t estr[2] = {1, 1};
    return encode_tensor_map(map, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, (void*)b, dims, strides, box, estr,
                             CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace

GemvPlan plan_gemv(int64_t M, int64_t N, int64_t K, int32_t G, int split_k_request, int sm_count, int max_vec,
                   bool tma_ok) {
    (void)G;
    GemvPlan pl{};
    pl.m_rows = (int)std::min<int64_t>(M, 8);
    const int64_t nw = N / 8;
    pl.tma = tma_ok && (nw % 4 == 0) && max_vec >= 4;
    int vec;
    if (pl.tma) {
        vec = pl.m_rows == 1 ? W4A16_GEMV_M1_VEC : 1;
    } else {
        vec = (nw % 4 == 0) ? 4 : (nw % 2 == 0) ? 2 : 1;
        vec = std::min(vec, std::max(max_vec, 1));
        // Register budget: two sums (group and running) of MT * 8 * VEC columns.
        if (pl.m_rows >= 3) vec = 1;
        else if (pl.m_rows == 2) vec = std::min(vec, 2);
    }
    pl.vec = vec;
    const int64_t tile_cols = 256 * vec;
    pl.col_tiles = (int)((N + tile_cols - 1) / tile_cols);
    int64_t split;
    if (split_k_request > 0) {
        split = split_k_request;
    } else {
        // One wave: as many slabs per column tile as resident CTA slots allow,
        // at least 8 rows per warp, at most kMaxRowsPerCta staged rows per CTA.
        const int64_t slots = (int64_t)std::max(sm_count, 1) * ctas_per_sm(pl.tma, pl.m_rows, vec);
        split = std::max<int64_t>(1, slots / pl.col_tiles);
        split = std::max<int64_t>(split, (K + kMaxRowsPerCta - 1) / kMaxRowsPerCta);
        split = std::min<int64_t>(split, std::max<int64_t>(1, K / (kWarps * 8)));
        split = std::min<int64_t>(split, 256);
    }
    pl.split_k = (int)std::max<int64_t>(1, split);
    if (pl.tma) {  // slabs are whole stages: no more slabs than stages
        const int64_t nblk = (K + tma_rows(vec) - 1) / tma_rows(vec);
        pl.split_k = (int)std::min<int64_t>(pl.split_k, nblk);
    }
    pl.counters_off = kWsHeader;
    pl.partials_off = align_up(kWsHeader + (size_t)pl.col_tiles * 4, 256);
    pl.ws_bytes = pl.split_k > 1 ? pl.partials_off + (size_t)pl.split_k * pl.m_rows * (size_t)N * 4
                                 : (pl.tma ? kWsHeader : 0);
    return pl;
}

size_t gemv_smem_bytes(int64_t M, int64_t K, int split_k) {
    const int64_t rows_cta = (K + split_k - 1) / split_k + 32;  // TMA slabs round up to whole stages
    return (size_t)std::min<int64_t>(M, 8) * (size_t)rows_cta * sizeof(float2);
}

cudaError_t launch_gemv(const __half* a, const uint32_t* b, const __half* s, const uint32_t* z,
                        int64_t M, int64_t N, int64_t K, int32_t G, int32_t zp_bias, OutPtr out,
                        void* workspace, const GemvPlan& pl, const WaitPolicy& wp, cudaStream_t st) {
    CUtensorMap bmap;
    if (pl.tma) {
        cudaError_t e = make_bmap(&bmap, b, N, K, pl.vec);
        if (e != cudaSuccess) return e;
    }
    const int R = tma_rows(pl.vec);
    // Largest slab: whole stages for the TMA kernel, an even split of rows otherwise.
    const int64_t rows_cta = pl.tma ? ((K + R - 1) / R + pl.split_k - 1) / pl.split_k * R
                                    : (K + pl.split_k - 1) / pl.split_k;
    for (int64_t m0 = 0; m0 < M; m0 += 8) {
        const int mt = (int)std::min<int64_t>(8, M - m0);
        GemvArgs args;
        args.a = a + m0 * K;
        args.b = b;
        args.s = s;
        args.z = z;
        args.out = out.rows(m0, N);
        args.partials = pl.split_k > 1 ? reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.partials_off) : nullptr;
        args.counters = pl.split_k > 1 ? reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + pl.counters_off) : nullptr;
        args.status = workspace ? static_cast<int*>(workspace) : nullptr;
        args.N = N;
        args.K = K;
        args.G = G;
        args.zp_bias = zp_bias;
        args.split = pl.split_k;
        args.rows_per_stage = R;
        args.s_vec = (reinterpret_cast<uintptr_t>(s) % 16) == 0;
        args.stall_loads = wp.stall_loads;
        args.wait_ns = wp.limit_ns;
        const dim3 grid((unsigned)pl.col_tiles, (unsigned)pl.split_k);
        size_t smem = (size_t)mt * (size_t)rows_cta * sizeof(float2);
        cudaError_t e;
        if (pl.tma) {
            smem += kRingBytes;
            TmaFn k = select_tma(mt, pl.vec);
            e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            k<<<grid, kThreads, smem, st>>>(bmap, args);
        } else {
            LdgFn k = select_ldg(mt, pl.vec);
            if (smem > 48 * 1024) {
                e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
                if (e != cudaSuccess) return e;
            }
            k<<<grid, kThreads, smem, st>>>(args);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace w4a16
