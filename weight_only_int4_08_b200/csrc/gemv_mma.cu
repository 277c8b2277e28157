// Stream-K GEMV for M <= 8 activation rows per launch, whose multiply-add runs
// on warp-level tensor instructions (mma.sync.m16n8k16, fp16 inputs, fp32
// accumulation) with the CUDA cores doing only the nibble unpack.
//
// Operation (vLLM PR #37352 analysis page, "코드 분석 1", `_w4a16_reference`):
//   out[m, n] = fp16( sum_g s[g, n] * sum_{k in g} a[m, k] * (q[k, n] - z[g, n]) ),
// fp32 accumulation; (q - z) is formed exactly in fp16, its products with the
// fp16 activations are exact in the fp32 accumulator, and the group scale is
// applied in fp32 to each group's accumulator.
//
// Why tensor instructions for a GEMV: the pure CUDA-core inner loop (fp32
// "magic number" unpack, packed FADD2/FFMA2) executes about 41 instructions per
// packed word of 8 weights on B200 and is issue-bound below the HBM rate. Here
// a register holds two k-rows of four columns after one ldmatrix.trans, and 9
// instructions turn it into four exact (q - z) fp16 pairs (0x6400 magic OR,
// fp16 subtract or fused scale-subtract); one mma.sync does 16 x 16 x 8
// multiply-adds. The MMA's batch dimension (8) is padded for M < 8.
//
// Work decomposition (stream-K): the weight matrix is cut into units of one
// 128-column tile x 128 rows (8 KB of packed weights), ordered tile by tile
// along K. A single wave of resident CTAs takes equal contiguous runs of that
// order, so every SM streams the same number of bytes whatever N and K are. A
// CTA's run covers pieces ("fragments") of one to a few tiles; within a
// fragment its 8 warps take equal runs of units, each through a private ring
// of two shared-memory stages filled by 2-D TMA loads (weights with 64-byte
// swizzle, which makes the transposed ldmatrix reads bank-conflict free, and
// the activations of the same rows) and tracked by one mbarrier per stage.
// The stage shape follows measurements on B200: streaming a 29 MB matrix,
// TMA boxes of 64 B x 16..32 rows ran up to 2x slower than boxes of 4 KB and
// more, and about 128 KB in flight per SM was enough; and one resident CTA per
// SM with 128-row stages needs fewer instructions per byte (no register cap,
// half the per-stage bookkeeping) than two CTAs with 64-row stages. Scales and
// zero words are copied one group ahead into a small per-warp shared buffer
// (cp.async; the first group before the wait on the previous kernel); each
// group's scaled sums are added to fp32 totals kept in registers. At the end of
// a fragment the totals go to shared memory and the warps are reduced in warp
// order; a tile covered by one CTA is written directly, otherwise the CTAs of
// the thread-block cluster that share it store their parts into the first one's
// shared memory, which adds them in rank order after one cluster barrier (fixed
// order, no floating-point atomics: bit-reproducible).
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

#ifndef W4A16_SK_WARPS
#define W4A16_SK_WARPS 8
#endif
// Warps per CTA: 8 (one CTA per SM), or 4 (two CTAs per SM) for launches of up to 8 rows on
// layers with more 128-column tiles than the GPU has SMs. Measured on B200 at M=1 (CUDA graphs,
// programmatic dependent launch, weights larger than L2): K=4096, N=28672 (224 tiles) 23.0 ->
// 16.4 us with 4 warps; K=4096, N=14336 (112 tiles) 9.96 against 11.37 us, and every narrower
// layer measured, stay faster with 8.
constexpr int kWarpsMax = W4A16_SK_WARPS;
constexpr int kWarpsWide = 4;
constexpr int kTileN = 128;
constexpr int kTileWords = kTileN / 8;            // 16 packed words = 64 B per row
#ifndef W4A16_SK_ROWS
#define W4A16_SK_ROWS 128
#endif
#ifndef W4A16_SK_RING
#define W4A16_SK_RING 2
#endif
constexpr int kRing = W4A16_SK_RING;              // stages in flight per warp
#ifndef W4A16_SK_MAX_CLUSTER
#define W4A16_SK_MAX_CLUSTER 4
#endif
// Thread-block cluster size limit (above 8: non-portable). Measured on B200 over the decode,
// small-batch and layer shapes: a limit of 4 was as fast as or faster than 8 on every shape
// (K=4096, N=6144: 9.6 -> 8.1 us) and 16 was slower; clusters cost more than the finer
// split they buy.
constexpr int kMaxCluster = W4A16_SK_MAX_CLUSTER;
constexpr int kMaxMT = 16;                        // activation rows per launch: two 8-row MMA tiles

// MMA batch tiles (8 activation rows each) of a launch of MT rows.
__host__ __device__ constexpr int n_tiles(int mt) { return (mt + 7) / 8; }
// Rows per unit / TMA stage (a multiple of 32): 128 for one batch tile; 64 for two, so that the
// larger activation stages and totals still fit one CTA's shared memory.
__host__ __device__ constexpr int rows_for(int mt) { return mt > 8 ? 64 : W4A16_SK_ROWS; }
__host__ __device__ constexpr int wstage_bytes(int mt) { return rows_for(mt) * kTileWords * 4; }
// Activation slot of one stage: MT rows x rows_for(MT) fp16. With 64-row stages (128 B per row)
// and more than four rows the rows are loaded with 128-byte swizzle (so that ldmatrix reads of 8
// rows hit 8 different bank groups), which needs 1024-byte aligned slots; otherwise the few
// conflicts are cheaper than the padding.
__host__ __device__ constexpr bool a_swizzled(int mt) { return mt > 4 && rows_for(mt) == 64; }
__host__ __device__ constexpr int a_slot_bytes(int mt) {
    return a_swizzled(mt) ? (2 * 64 * mt + 1023) / 1024 * 1024 : 2 * rows_for(mt) * mt;
}
// Per warp, two group buffers: the tile's 128 scales (256 B) and 16 zero words (64 B).
constexpr int kGrpBytes = 2 * kTileN + 4 * kTileWords;
// Accumulator values per thread and chunk kept across groups: entry i of each batch tile's MMA
// accumulators (only the even entries, batch 2t, matter for one activation row).
__host__ __device__ constexpr int tot_per_tile(int mt) { return mt > 1 ? 8 : 4; }
__host__ __device__ constexpr int tot_per_chunk(int mt) { return tot_per_tile(mt) * n_tiles(mt); }
// Dynamic shared memory: weight ring, activation ring, fp32 totals, group buffers, and the
// warp-reduced sums of the (at most two) fragments shared with other CTAs.
// recv: the launch's layout splits tiles between CTAs, whose owners receive the other parts.
__host__ __device__ constexpr size_t sk_smem_bytes(int warps, int mt, bool recv = false) {
    return (size_t)warps * kRing * (wstage_bytes(mt) + a_slot_bytes(mt)) +
           (size_t)warps * 4 * tot_per_chunk(mt) * 32 * 4 + (size_t)warps * 2 * kGrpBytes + 2 * (size_t)mt * kTileN * 4 +
           (recv ? (size_t)(kMaxCluster - 1) * mt * kTileN * 4 : 0);
}

struct SkArgs {
    const __half* s;      // [K/G, N]
    const uint32_t* z;    // [K/G, N/8] or nullptr
    OutPtr out;           // [M, N] (this launch's row block)
    int* status;
    int64_t N, K;
    int tiles;            // 128-column tiles
    int tiles_per_cluster;
    int G, zp_bias, nblk, stall_loads;
    uint32_t magic;       // kMagic, passed at run time so that the and-or unpack compiles to one LOP3
    int shares_mask;      // bit 0: a full cluster splits a tile between CTAs; bit 1: the last, shorter one does
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
__device__ __forceinline__ void cp_async_8(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
// Four 8x8 matrices, not transposed: thread t receives row t / 4, columns 2 (t % 4), 2 (t % 4) + 1.
__device__ __forceinline__ void ldmatrix_x4(uint32_t saddr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr)
                 : "memory");
}
// Two transposed 8x8 matrices (rows given by threads 0..15).
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t saddr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(saddr)
                 : "memory");
}

// The unpack is the exponent-bias ("magic number") technique published by Kim et al. 2022 ("Who
// Says Elephants Can't Run") and Frantar et al. 2024 ("MARLIN"), written here from the IEEE-754
// layout: OR a nibble into the mantissa of an fp16 whose ulp is 1 (1024.0 = 0x6400) and the
// value is exactly 1024 + q; subtracting 1024 + z leaves q - z exactly.
constexpr uint32_t kMagic = 0x64006400u;      // fp16 1024.0 in both halves
// Measured on B200: with both masks of (x & mask) | kMagic as compile-time constants the
// compiler emits two logic instructions per unpacked register pair; with kMagic in a register
// (a kernel argument) it emits one.
constexpr uint32_t kSixteenth = 0x2C002C00u;  // fp16 1/16 in both halves

// Rank whose run of a cluster's units contains unit u (counted from the cluster's first unit);
// runs are [floor(r U / S), floor((r + 1) U / S)).
__device__ __forceinline__ int rank_of(int64_t u, int64_t U, int S) { return (int)(((u + 1) * S - 1) / U); }

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_cluster(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
// Shared-memory address of the same variable in CTA `rank` of the cluster, and a load from it.
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ float ld_cluster(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

#ifndef W4A16_SK_MIN_CTAS
#define W4A16_SK_MIN_CTAS 1   // one resident CTA per SM: no register cap (a cap of 128 cost ~15 % in moves)
#endif
// FAST: the group size is a multiple of the unit (kRows), so a group starts only at a unit start
// (and K is a multiple of kRows); otherwise groups are tracked per 16-row step.
template <int kWarps, int MT, bool FAST>
__global__ void __launch_bounds__(32 * kWarps, W4A16_SK_MIN_CTAS)
gemv_sk_kernel(const __grid_constant__ CUtensorMap bmap, const __grid_constant__ CUtensorMap amap, SkArgs p) {
    constexpr int kThreads = 32 * kWarps;
    constexpr int kRows = rows_for(MT);            // rows per unit / stage
    constexpr int kSteps = kRows / 16;             // 16-row MMA steps per stage
    constexpr int kWStage = wstage_bytes(MT);
    constexpr int kWRingBytes = kWarps * kRing * kWStage;
    constexpr int kASlot = a_slot_bytes(MT);
    constexpr int NT = n_tiles(MT);                // 8-row batch tiles
    constexpr int NB = tot_per_tile(MT);
    constexpr int NI = tot_per_chunk(MT);
    extern __shared__ __align__(1024) unsigned char s_dyn[];
    unsigned char* wring = s_dyn;                                        // [warp][kRing][kRows][64 B], 64-byte swizzle
    unsigned char* aring = s_dyn + kWRingBytes;                          // [warp][kRing][MT][kRows] fp16
    float* tots = reinterpret_cast<float*>(aring + kWarps * kRing * kASlot);  // [warp][c * NI + i][lane]
    unsigned char* grps = reinterpret_cast<unsigned char*>(tots + kWarps * 4 * NI * 32);  // [warp][2][kGrpBytes]
    float* keep = reinterpret_cast<float*>(grps + kWarps * 2 * kGrpBytes);                // [2][MT][128]
    float* recv = keep + 2 * MT * kTileN;   // [kMaxCluster - 1][MT][128]: parts of a shared tile I own
                                            // (allocated when the layout shares tiles)
    __shared__ __align__(8) uint64_t s_full[kWarps][kRing];
    __shared__ __align__(16) uint4 s_zero;   // the B rows past MT read these zeros
    __shared__ volatile int s_abort;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2;
    float* tmine = tots + warp * 4 * NI * 32 + lane;
    unsigned char* grp = grps + warp * 2 * kGrpBytes;
    const int nblk = p.nblk, G = p.G, K = (int)p.K;
    const int nw = (int)(p.N / 8);
    // My cluster owns tiles [tile_lo, tile_hi); its units (tile-major, kRows-row blocks) are split in
    // S equal contiguous runs, mine being run `rank`. Unit counts fit in 32 bits (the weights would
    // not fit in memory otherwise; the host checks).
    const int S = (int)cluster_nctarank(), rank = (int)cluster_ctarank();
    const int tile_lo = (int)(blockIdx.x / S) * p.tiles_per_cluster;
    const int tile_hi = min(tile_lo + p.tiles_per_cluster, p.tiles);
    const int ubase = tile_lo * nblk, U = (tile_hi - tile_lo) * nblk;
    // (32-bit arithmetic unless a cluster holds 2^29 units or more)
    auto split_at = [&](int r) -> int {
        return U < (1 << 29) ? (int)((uint32_t)U * (uint32_t)r / (uint32_t)S) : (int)((int64_t)U * r / S);
    };
    const int u0 = ubase + split_at(rank), u1 = ubase + split_at(rank + 1);
    const int t0 = u0 / nblk;
    const int nfrag = u1 > u0 ? (u1 - 1) / nblk - t0 + 1 : 0;

    // This warp's units of fragment f: k-blocks [lo, hi) of tile t0 + f.
    auto frag_lo_hi = [&](int f, int& lo, int& hi) {
        const int tb = (t0 + f) * nblk;
        const int a = max(u0, tb) - tb, b = min(u1, tb + nblk) - tb;
        lo = a + (b - a) * warp / kWarps;
        hi = a + (b - a) * (warp + 1) / kWarps;
    };

    // Each warp's ring is waited on by that warp alone: its lane 0 initialises the ring's barriers and
    // issues the first loads before the block-wide barrier, which only the abort flag and the zero row
    // need (neither is read before it).
    if (threadIdx.x == 0) {
        s_abort = 0;
        s_zero = make_uint4(0u, 0u, 0u, 0u);
    }
    if (lane == 0) {
        for (int j = 0; j < kRing; ++j) ptx::mbar_init(ptx::smem_addr(&s_full[warp][j]), 1);
        ptx::mbar_fence_init();
    }
    __syncwarp();
    // Shared tiles: the CTAs that share a tile with its first (owning) CTA store their parts into
    // the owner's shared memory before the cluster barrier at the end, and the owner adds them up
    // after it; nobody reads another CTA's shared memory, so nobody waits for another to finish
    // reading. Remote stores need the owner to have started: every CTA arrives here and waits (after
    // its first loads, by when all have arrived) before its first remote store. Every CTA of a
    // cluster computes the same cluster_shares, so all of them or none take the cluster barriers.
    const bool cluster_shares =
        (tile_hi - tile_lo == p.tiles_per_cluster ? p.shares_mask & 1 : p.shares_mask & 2) != 0;

    // Per-warp shared-memory addresses of ring slot 0 (slot j adds j times the slot size).
    const uint32_t bar0 = ptx::smem_addr(&s_full[warp][0]);
    const uint32_t w0 = ptx::smem_addr(wring + warp * kRing * kWStage);
    const uint32_t a0 = ptx::smem_addr(aring + warp * kRing * kASlot);

    // With programmatic dependent launch the next kernel on the stream may start now; it waits for
    // this one to finish before it touches anything this one writes.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // Load issue (lane 0): a cursor over this warp's units, one stage per unit. A stage's barrier
    // expects the weight box and the activation box; the activations may be issued later.
    int pf = 0, pkb = 0, phi = 0, armed = 0;
    frag_lo_hi(0, pkb, phi);
    auto arm_w = [&]() -> int {   // the unit's k-block, or -1 when the warp has no more units
        while (pkb >= phi) {
            if (pf + 1 >= nfrag) return -1;
            ++pf;
            frag_lo_hi(pf, pkb, phi);
        }
        const int slot = armed % kRing;
        const uint32_t bar = bar0 + 8 * slot;
        ptx::mbar_arrive_expect_tx(bar, (uint32_t)(kWStage + 2 * kRows * MT));
        ptx::tma_load_2d(w0 + slot * kWStage, &bmap, (t0 + pf) * kTileWords, pkb * kRows, bar);
        ++armed;
        return pkb++;
    };
    auto issue_a = [&](int slot, int kb) {
        ptx::tma_load_2d(a0 + slot * kASlot, &amap, kb * kRows, 0, bar0 + 8 * slot);
    };
    auto arm_next = [&]() {
        const int slot = armed % kRing;
        const int kb = arm_w();
        if (kb >= 0) issue_a(slot, kb);
    };
    // Prologue: the first stages' weights (independent of any earlier kernel) go out first; the
    // activations, written by the kernel before this one, only after it has completed.
    int first_kb[kRing];
    if (lane == 0 && !p.stall_loads) {
        ptx::prefetch_tensormap(&bmap);
        ptx::prefetch_tensormap(&amap);
#pragma unroll
        for (int j = 0; j < kRing; ++j) first_kb[j] = arm_w();
    }
    // Copy group gg's scales and zero words of a tile into group buffer gg & 1 (lane l copies scales
    // 4l..4l+3, lanes 0..15 the zero words), one group ahead of use. Chunks past N get zero scales.
    auto load_meta = [&](int tile, int gg) {
        unsigned char* gb = grp + (gg & 1) * kGrpBytes;
        if ((int64_t)tile * kTileN + 32 * (lane / 8) < p.N)
            cp_async_8(ptx::smem_addr(gb + 8 * lane), p.s + (int64_t)tile * kTileN + 4 * lane + (int64_t)gg * p.N);
        else
            *reinterpret_cast<uint2*>(gb + 8 * lane) = make_uint2(0u, 0u);
        if (p.z && lane < kTileWords && tile * kTileWords + lane < nw)
            cp_async_4(ptx::smem_addr(gb + 2 * kTileN + 4 * lane), p.z + (int64_t)tile * kTileWords + lane + (int64_t)gg * nw);
        cp_async_commit();
    };
    // The first fragment's first group goes out before the wait for the previous kernel: like the
    // weights, scales and zeros are written by no kernel this one may overlap. Measured on B200
    // (per-warp timeline, K=N=4096, M=1, one 8 KB unit per warp): the first group's copy issued
    // after the wait held the warp ~0.3 us once its weights had landed.
    if (nfrag > 0) {
        int lo0, hi0;
        frag_lo_hi(0, lo0, hi0);
        if (lo0 < hi0) load_meta(t0, lo0 * kRows / G);
    }
    __syncthreads();   // the abort flag and the zero row are set
    if (cluster_shares) cluster_arrive_relaxed();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (cluster_shares) cluster_wait();   // every CTA of the cluster has started
    if (lane == 0 && !p.stall_loads) {
#pragma unroll
        for (int j = 0; j < kRing; ++j)
            if (first_kb[j] >= 0) issue_a(j, first_kb[j]);
    }

    const int zshift = 16 * (g & 1);  // my first column is nibble 4 (g & 1) of its zero word
    const uint32_t magic = p.magic;
    int consumed = 0;
    bool failed = false;

    uint32_t bias[4][4];  // j even: (1024 + z) x2; j odd: -(64 + z) x2 (fp16 bits)
    auto set_bias = [&](int c, uint32_t zw) {
        bias[c][0] = (0x6400u + (zw & 0xFu)) * 0x00010001u;
        // -(64 + z): 0xD400 is -64 and one unit of the fraction is 1/16 there
        bias[c][1] = (0xD400u + 16u * ((zw >> 4) & 0xFu)) * 0x00010001u;
        bias[c][2] = (0x6400u + ((zw >> 8) & 0xFu)) * 0x00010001u;
        bias[c][3] = (0xD400u + 16u * ((zw >> 12) & 0xFu)) * 0x00010001u;
    };
    if (!p.z) {  // one zero point for every column and group
#pragma unroll
        for (int c = 0; c < 4; ++c) set_bias(c, (uint32_t)p.zp_bias * 0x1111u);
    }
    // B-fragment ldmatrix address of lane (activation row 8 nt + lane % 8, 8-k block lane / 8) in
    // ring slot 0, or the zero row past MT; each ldmatrix covers two 16-row steps.
    const int br = lane & 7, bc = lane >> 3;
    auto b_off = [&](int nt) -> uint32_t {
        return 8 * nt + br < MT ? a0 + (8 * nt + br) * 2 * kRows : ptx::smem_addr(&s_zero);
    };
    auto b_col = [&](int nt, int h2) -> uint32_t {   // 16-byte column block 4 h2 + bc of that row
        return 8 * nt + br < MT ? 16 * (a_swizzled(MT) ? ((4 * h2 + bc) ^ br) : (4 * h2 + bc)) : 0;
    };
    auto b_slot = [&](int nt) -> uint32_t { return 8 * nt + br < MT ? kASlot : 0; };
    // Weight ldmatrix.trans address of lane (row lane, 16-byte chunk c) under the 64-byte swizzle:
    // row r holds chunk c at chunk c ^ ((r >> 1) & 3).
    const uint32_t w_row = lane * 64;
    const int w_sw = (lane >> 1) & 3;

    for (int f = 0; f < nfrag; ++f) {
        const int tile = t0 + f;
        int lo, hi;
        frag_lo_hi(f, lo, hi);
        const int rend = min(hi * kRows, K);

        float acc[4][NT][8];
        // The fragment's scaled group sums, in registers (4 NI values per lane, stored to shared
        // memory once at the fragment's end). Measured on B200: at one row (per-warp timeline) the
        // 16 load-FMA-store steps on shared memory they replaced took ~0.24 us per group; at 9-16
        // rows (64 per group, the kernel at 234-237 registers without spills) they cost 4-10 %, e.g.
        // K=4096, N=14336, M=16 16.2 -> 14.7 us.
        float treg[4 * NI];
#pragma unroll
        for (int k = 0; k < 4 * NI; ++k) treg[k] = 0.f;

        auto load_group = [&](int gg) { load_meta(tile, gg); };
        // Groups advance one at a time: g_cur is the open group (from g_first), g_next its end row.
        const int g_first = lo * kRows / G;
        int g_cur = g_first - 1, g_next = g_first * G;
        auto group_end = [&]() {
            const unsigned char* gb = grp + (g_cur & 1) * kGrpBytes;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint2 sc = *reinterpret_cast<const uint2*>(gb + 64 * c + 8 * g);
                const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&sc.x));
                const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&sc.y));
                const float sj[4] = {s01.x, s01.y, s23.x, s23.y};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if (MT > 1 || (i & 1) == 0) {
                            const int k = c * NI + nt * NB + (MT > 1 ? i : i / 2);
                            treg[k] = fmaf(sj[i >> 1], acc[c][nt][i], treg[k]);
                        }
            }
        };
        // Start group gg (its buffer was filled one group earlier) and prefetch the next one.
        auto group_start = [&](int gg) {
            cp_async_wait_all();
            __syncwarp();   // every lane's copies have landed; every lane is done with the other buffer
            const unsigned char* gb = grp + (gg & 1) * kGrpBytes;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (p.z) set_bias(c, *reinterpret_cast<const uint32_t*>(gb + 2 * kTileN + 4 * (4 * c + g / 2)) >> zshift);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[c][nt][i] = 0.f;
            }
            if (g_next < rend) load_group(gg + 1);   // g_next is the first row of group gg + 1
        };
        auto advance_group = [&]() {
            if (g_cur >= g_first) group_end();
            ++g_cur;
            g_next += G;
            group_start(g_cur);
        };
        // Dequantise two 8-row matrices of chunk c (k-rows r..r+7 in x0, r+8..r+15 in x1) and
        // multiply them with the activation fragments of 16-row step h (one per batch tile).
        uint32_t bf[kSteps][NT][2];
        auto mma_chunk = [&](int c, uint32_t x0, uint32_t x1, int h) {
            {
                const uint32_t e0a = hsub2((x0 & 0x000F000Fu) | magic, bias[c][0]);
                const uint32_t e1a = hfma2((x0 & 0x00F000F0u) | magic, kSixteenth, bias[c][1]);
                const uint32_t e0b = hsub2((x1 & 0x000F000Fu) | magic, bias[c][0]);
                const uint32_t e1b = hfma2((x1 & 0x00F000F0u) | magic, kSixteenth, bias[c][1]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    mma16816(acc[c][nt][0], acc[c][nt][1], acc[c][nt][2], acc[c][nt][3], e0a, e1a, e0b, e1b,
                             bf[h][nt][0], bf[h][nt][1]);
            }
            {
                const uint32_t y0 = x0 >> 8, y1 = x1 >> 8;
                const uint32_t e2a = hsub2((y0 & 0x000F000Fu) | magic, bias[c][2]);
                const uint32_t e3a = hfma2((y0 & 0x00F000F0u) | magic, kSixteenth, bias[c][3]);
                const uint32_t e2b = hsub2((y1 & 0x000F000Fu) | magic, bias[c][2]);
                const uint32_t e3b = hfma2((y1 & 0x00F000F0u) | magic, kSixteenth, bias[c][3]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    mma16816(acc[c][nt][4], acc[c][nt][5], acc[c][nt][6], acc[c][nt][7], e2a, e3a, e2b, e3b,
                             bf[h][nt][0], bf[h][nt][1]);
            }
        };

        if (lo < hi && f > 0) load_group(g_first);   // (fragment 0's went out before the wait)
        for (int kb = lo; kb < hi && !failed; ++kb) {
            const int slot = consumed % kRing;
            const bool okw = ptx::mbar_wait(bar0 + 8 * slot, (uint32_t)((consumed / kRing) & 1), &s_abort, p.wait_ns);
            if (!__all_sync(0xffffffffu, okw)) {
                failed = true;
                break;
            }
            ++consumed;
            const int rs = kb * kRows;
            const uint32_t wst = w0 + slot * kWStage;
            // B fragments (batch row 8 nt + g, k-pairs t and t + 4 of each 16-row step), two steps per
            // ldmatrix.
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int h2 = 0; h2 < kSteps / 2; ++h2) {
                    uint32_t B[4];
                    ldmatrix_x4(b_off(nt) + slot * b_slot(nt) + b_col(nt, h2), B);
                    bf[2 * h2][nt][0] = B[0];
                    bf[2 * h2][nt][1] = B[1];
                    bf[2 * h2 + 1][nt][0] = B[2];
                    bf[2 * h2 + 1][nt][1] = B[3];
                }
            if constexpr (FAST) {
                if (rs >= g_next) advance_group();
#pragma unroll
                for (int q = 0; q < kRows / 32; ++q) {
                    // rows 32q + lane of all four chunks; ((32q + lane) >> 1) & 3 == (lane >> 1) & 3
                    uint32_t R[4][4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) ptx::ldmatrix_x4_trans(wst + 32 * q * 64 + w_row + 16 * (c ^ w_sw), R[c]);
                    // chunks innermost: consecutive MMAs update different accumulators
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int c = 0; c < 4; ++c) mma_chunk(c, R[c][2 * hh], R[c][2 * hh + 1], 2 * q + hh);
                }
            } else {
#pragma unroll
                for (int h = 0; h < kSteps; ++h) {
                    const int k0 = rs + 16 * h;
                    if (k0 >= rend) break;
                    if (k0 >= g_next) advance_group();
                    const int row = 16 * h + (lane & 15);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t x0, x1;
                        ldmatrix_x2_trans(wst + row * 64 + 16 * (c ^ ((row >> 1) & 3)), x0, x1);
                        mma_chunk(c, x0, x1, h);
                    }
                }
            }
            // Every lane has read the stage: it can be refilled.
            __syncwarp();
            // (The ldmatrix results were consumed above, so the reads are complete before the copy
            // that overwrites the stage is issued.)
            if (lane == 0 && !p.stall_loads) arm_next();
        }
        if (g_cur >= g_first && !failed) group_end();

        // ---- reduce fragment f over the warps (warp order) ----
        // A tile held by this CTA alone is written out now; the first and the last fragment may be
        // shared with other CTAs of the cluster and are kept (keep[0], keep[1]) for the exchange.
#pragma unroll
        for (int k = 0; k < 4 * NI; ++k) tmine[32 * k] = treg[k];
        __syncthreads();
        // s_abort is read by every thread between two barriers with no wait in between: uniform.
        if (s_abort == 0) {
            const int first = rank_of(tile * nblk - ubase, U, S);
            const bool shared_tile = first != rank_of((tile + 1) * nblk - 1 - ubase, U, S);
            float* kp = keep + (f == 0 ? 0 : MT * kTileN);
            // a part for the owner: slot rank - first - 1 of its receive buffer
            const uint32_t rp = shared_tile && first != rank
                                    ? map_rank(ptx::smem_addr(recv + (rank - first - 1) * MT * kTileN), (uint32_t)first)
                                    : 0u;
            for (int item = threadIdx.x; item < MT * kTileN; item += kThreads) {
                const int m = item / kTileN, nl = item % kTileN;
                const int64_t n = (int64_t)tile * kTileN + nl;
                // (m, nl) is entry i = 2 (nl % 4) + (m % 2) of batch tile m / 8 of chunk nl / 32, held by
                // lane 4 ((nl % 32) / 4) + (m % 8) / 2
                const int mm = m & 7, i = 2 * (nl & 3) + (mm & 1);
                const int src = 32 * ((nl >> 5) * NI + (m >> 3) * NB + (MT > 1 ? i : i / 2)) + 4 * ((nl & 31) >> 2) +
                                (mm >> 1);
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) v += tots[w * 4 * NI * 32 + src];
                if (!shared_tile) {
                    if (n < p.N) p.out.put((int64_t)m * p.N + n, v);
                } else if (first == rank) {
                    kp[item] = v;
                } else {
                    st_cluster(rp + 4 * item, v);
                }
            }
        }
        __syncthreads();  // the totals are free again
    }

    // ---- tiles shared within the cluster: the first CTA touching a tile adds its own part and the
    // parts the others stored into its receive buffer, in rank order, then writes the tile ----
    // Only a cluster whose rank boundaries cut through a tile has shared tiles; the others (every CTA
    // runs whole tiles) take no cluster barrier. Measured on B200: the two barriers of the earlier
    // exchange (read the parts remotely, then wait for every reader) cost a CTA ~1.6 us at the end
    // of a decode launch; this one has a single barrier, after which only the owners work.
    if (cluster_shares) cluster_sync();   // every part has been stored (release / acquire)
    if (cluster_shares && s_abort == 0) {
#pragma unroll
        for (int d = 0; d < 2; ++d) {
            if (d >= nfrag || (d == 1 && nfrag == 1)) continue;
            const int tile = t0 + (d == 0 ? 0 : nfrag - 1);
            const int first = rank_of(tile * nblk - ubase, U, S), last = rank_of((tile + 1) * nblk - 1 - ubase, U, S);
            if (first == last || first != rank) continue;
            const float* own = keep + (d == 0 ? 0 : MT * kTileN);
            for (int item = threadIdx.x; item < MT * kTileN; item += kThreads) {
                const int m = item / kTileN, nl = item % kTileN;
                const int64_t n = (int64_t)tile * kTileN + nl;
                if (n >= p.N) continue;
                float v = 0.f;
                v += own[item];
                for (int rr = first + 1; rr <= last; ++rr) v += recv[(rr - first - 1) * MT * kTileN + item];
                p.out.put((int64_t)m * p.N + n, v);
            }
        }
    }

    // A wait gave up: let the copies already issued land before the CTA's shared memory goes away.
    cp_async_wait_all();
    if (lane == 0 && consumed < armed) {
        for (int j = consumed; j < armed; ++j) {
            volatile int dummy = 0;
            ptx::mbar_wait(bar0 + 8 * (j % kRing), (uint32_t)((j / kRing) & 1), &dummy, p.wait_ns);
        }
    }
    if (failed && lane == 0 && p.status) atomicExch(p.status, (int)W4A16_ERR_TIMEOUT);
}

using SkFn = void (*)(CUtensorMap, CUtensorMap, SkArgs);

template <int W, bool FAST>
SkFn select_sk_t(int mt) {
    switch (mt) {
        case 1: return gemv_sk_kernel<W, 1, FAST>;
        case 2: return gemv_sk_kernel<W, 2, FAST>;
        case 3: return gemv_sk_kernel<W, 3, FAST>;
        case 4: return gemv_sk_kernel<W, 4, FAST>;
        case 5: return gemv_sk_kernel<W, 5, FAST>;
        case 6: return gemv_sk_kernel<W, 6, FAST>;
        case 7: return gemv_sk_kernel<W, 7, FAST>;
        case 8: return gemv_sk_kernel<W, 8, FAST>;
        default: break;
    }
    if constexpr (W == kWarpsMax) {
        switch (mt) {
            case 9: return gemv_sk_kernel<W, 9, FAST>;
            case 10: return gemv_sk_kernel<W, 10, FAST>;
            case 11: return gemv_sk_kernel<W, 11, FAST>;
            case 12: return gemv_sk_kernel<W, 12, FAST>;
            case 13: return gemv_sk_kernel<W, 13, FAST>;
            case 14: return gemv_sk_kernel<W, 14, FAST>;
            case 15: return gemv_sk_kernel<W, 15, FAST>;
            default: return gemv_sk_kernel<W, 16, FAST>;
        }
    }
    return nullptr;   // 4-warp CTAs serve launches of up to 8 rows only
}
// Occupancy queries use the FAST instance (both have the same shared memory and launch bounds).
SkFn select_sk(int warps, int mt, bool fast = true) {
    if (warps == kWarpsWide && kWarpsWide != kWarpsMax)
        return fast ? select_sk_t<kWarpsWide, true>(mt) : select_sk_t<kWarpsWide, false>(mt);
    return fast ? select_sk_t<kWarpsMax, true>(mt) : select_sk_t<kWarpsMax, false>(mt);
}
// Index of a warp count in the per-configuration caches below.
int wix(int warps) { return warps == kWarpsMax ? 0 : 1; }

std::atomic<int> g_sk_occ[2][kMaxMT + 1];

// Resident CTAs per SM from the kernel's registers and shared memory.
int sk_ctas_per_sm(int warps, int mt) {
    int n = g_sk_occ[wix(warps)][mt].load(std::memory_order_relaxed);
    if (n > 0) return n;
    cudaFuncAttributes fa{};
    int regs = 255;
    size_t static_smem = 1024;
    if (cudaFuncGetAttributes(&fa, select_sk(warps, mt)) == cudaSuccess && fa.numRegs > 0) {
        regs = fa.numRegs;
        static_smem = fa.sharedSizeBytes;
    }
    const size_t smem = sk_smem_bytes(warps, mt) + static_smem + 1024;   // + the per-CTA reservation
    const int by_smem = (int)((228 * 1024) / smem);
    const int by_regs = 65536 / (((regs + 7) / 8 * 8) * 32 * warps);
    n = std::max(1, std::min(by_smem, by_regs));
    g_sk_occ[wix(warps)][mt].store(n, std::memory_order_relaxed);
    return n;
}

std::atomic<int> g_sk_clusters[2][kMaxMT + 1][kMaxCluster + 1];

// Clusters of S CTAs that can be resident at once (clusters are placed within one GPC each, so
// this can be less than the resident CTAs divided by S).
int sk_max_clusters(int warps, int mt, int S) {
    int n = g_sk_clusters[wix(warps)][mt][S].load(std::memory_order_relaxed);
    if (n > 0) return n;
    SkFn k = select_sk(warps, mt);
    const size_t smem = sk_smem_bytes(warps, mt);
    n = 0;
    if (kMaxCluster > 8) cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)S);
        cfg.blockDim = dim3(32 * warps);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)S;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();  // a failed query must not leak into the next launch check
    if (n <= 0) n = 1;
    g_sk_clusters[wix(warps)][mt][S].store(n, std::memory_order_relaxed);
    return n;
}

// Cluster layout of one launch of mt activation rows: S CTAs per cluster over k whole tiles each,
// all resident at once; the fewest units per CTA wins, then the most CTAs. An explicit split asks
// for that many CTAs per tile (at most a cluster, at most one per unit).
struct SkLayout {
    int cluster, cluster_tiles, ctas, warps;
    int64_t nblk;
};
int sk_warps(int mt, int64_t N, int sm_count) {
    const int64_t T = (N + kTileN - 1) / kTileN;
    return mt <= 8 && T > sm_count ? kWarpsWide : kWarpsMax;
}
SkLayout sk_layout(int mt, int64_t N, int64_t K, int split_k_request, int sm_count) {
    const int64_t T = (N + kTileN - 1) / kTileN, nblk = (K + rows_for(mt) - 1) / rows_for(mt);
    const int warps = sk_warps(mt, N, sm_count);
    int best_s = 1, best_k = 1;
    if (split_k_request > 0) {
        best_s = (int)std::min<int64_t>(std::min(split_k_request, kMaxCluster), nblk);
    } else {
        const int64_t slots = (int64_t)std::max(sm_count, 1) * sk_ctas_per_sm(warps, mt);
        int64_t best_cost = INT64_MAX, best_ctas = 0;
        for (int S = 1; S <= kMaxCluster; ++S) {
            const int64_t qmax = std::min<int64_t>({T, slots / S, (int64_t)sk_max_clusters(warps, mt, S)});
            for (int64_t Q = 1; Q <= qmax; ++Q) {
                const int64_t k = (T + Q - 1) / Q;
                if ((Q - 1) * k >= T) continue;   // the same k with fewer clusters
                const int64_t ctas = Q * S;
                if (S > nblk) continue;   // every CTA of every cluster (the last one may be short) gets a unit
                const int64_t cost = (k * nblk + S - 1) / S;
                if (cost < best_cost || (cost == best_cost && ctas > best_ctas)) {
                    best_cost = cost;
                    best_ctas = ctas;
                    best_s = S;
                    best_k = (int)k;
                }
            }
        }
    }
    SkLayout l;
    l.cluster = best_s;
    l.cluster_tiles = best_k;
    l.ctas = (int)((T + best_k - 1) / best_k) * best_s;
    l.warps = warps;
    l.nblk = nblk;
    return l;
}

}  // namespace

bool gemv_mma_supported(int64_t N, int64_t K, const void* a, const void* b, const void* s, const void* z) {
    (void)z;   // zeros are read with 4-byte copies
    const int64_t units = (N + kTileN - 1) / kTileN * ((K + 63) / 64);   // counted in 32 bits (64-row units at most)
    return N % 32 == 0 && units < ((int64_t)1 << 31) && (reinterpret_cast<uintptr_t>(b) % 16) == 0 &&
           (reinterpret_cast<uintptr_t>(a) % 16) == 0 && (reinterpret_cast<uintptr_t>(s) % 8) == 0;
}

GemvPlan plan_gemv_mma(int64_t M, int64_t N, int64_t K, int32_t G, int split_k_request, int sm_count) {
    (void)G;
    GemvPlan pl{};
    pl.tma = true;
    pl.mma = true;
    pl.vec = 1;
    pl.m_rows = (int)std::min<int64_t>(M, kMaxMT);
    pl.col_tiles = (int)((N + kTileN - 1) / kTileN);
    const SkLayout l = sk_layout(pl.m_rows, N, K, split_k_request, sm_count);
    pl.cluster = l.cluster;
    pl.cluster_tiles = l.cluster_tiles;
    pl.warps = l.warps;
    pl.split_k = l.ctas;
    pl.split_k_request = split_k_request;
    pl.ws_bytes = 0;  // partial sums stay in the clusters' shared memory
    return pl;
}

cudaError_t launch_gemv_mma(const __half* a, const uint32_t* b, const __half* s, const uint32_t* z, int64_t M,
                            int64_t N, int64_t K, int32_t G, int32_t zp_bias, OutPtr out, void* workspace,
                            const GemvPlan& pl, const WaitPolicy& wp, cudaStream_t st) {
    char* ws = static_cast<char*>(workspace);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int split_req = pl.split_k_request;
    for (int64_t m0 = 0; m0 < M; m0 += kMaxMT) {
        const int mt = (int)std::min<int64_t>(kMaxMT, M - m0);
        const int rows = rows_for(mt);
        // Row blocks of another size than the first take their own layout (stage rows differ).
        const SkLayout l = mt == pl.m_rows ? SkLayout{pl.cluster, pl.cluster_tiles, pl.split_k, pl.warps, (K + rows - 1) / rows}
                                           : sk_layout(mt, N, K, split_req, sms);
        CUtensorMap bmap, amap;
        {
            const cuuint64_t dims[2] = {(cuuint64_t)(N / 8), (cuuint64_t)K};
            const cuuint64_t strides[1] = {(cuuint64_t)(N / 8) * 4};
            const cuuint32_t box[2] = {(cuuint32_t)kTileWords, (cuuint32_t)rows};
            const cuuint32_t estr[2] = {1, 1};
            cudaError_t e = encode_tensor_map(&bmap, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, (void*)b, dims, strides, box,
                                              estr, CU_TENSOR_MAP_SWIZZLE_64B);
            if (e != cudaSuccess) return e;
        }
        {
            const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)mt};
            const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
            const cuuint32_t box[2] = {(cuuint32_t)rows, (cuuint32_t)mt};
            const cuuint32_t estr[2] = {1, 1};
            cudaError_t e = encode_tensor_map(&amap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void*)(a + m0 * K), dims,
                                              strides, box, estr,
                                              a_swizzled(mt) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
            if (e != cudaSuccess) return e;
        }
        SkArgs args;
        args.s = s;
        args.z = z;
        args.out = out.rows(m0, N);
        args.status = workspace ? reinterpret_cast<int*>(ws) : nullptr;
        args.N = N;
        args.K = K;
        args.tiles = pl.col_tiles;
        args.tiles_per_cluster = l.cluster_tiles;
        args.G = G;
        args.zp_bias = zp_bias;
        args.nblk = (int)l.nblk;
        args.magic = kMagic;
        {
            // A cluster of S CTAs over `tiles` whole tiles splits a tile between CTAs when a rank
            // boundary of its units falls inside one.
            const int64_t T = pl.col_tiles, k = l.cluster_tiles;
            auto shares = [&](int64_t tiles) {
                const int64_t U = tiles * l.nblk;
                for (int r = 1; r < l.cluster; ++r)
                    if ((U * r / l.cluster) % l.nblk != 0) return true;
                return false;
            };
            const int64_t last_tiles = T - (T - 1) / k * k;
            args.shares_mask = (shares(k) ? 1 : 0) | (shares(last_tiles) ? 2 : 0);
        }
        args.stall_loads = wp.stall_loads;
        args.wait_ns = wp.limit_ns;
        const size_t smem = sk_smem_bytes(l.warps, mt, args.shares_mask != 0);
        SkFn k = select_sk(l.warps, mt, G % rows == 0);
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (l.cluster > 8) {
            e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
        }
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)l.ctas);
        cfg.blockDim = dim3(32 * l.warps);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)l.cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = wp.pdl ? 2 : 1;
        e = cudaLaunchKernelEx(&cfg, k, bmap, amap, args);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace w4a16
