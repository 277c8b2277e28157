// Tensor-core (tcgen05 / TMEM) W4A16 GEMM for M >= 9 activation rows.
//
// Operation (vLLM PR #37352 analysis page, "코드 분석 1", `_w4a16_reference`):
//   out[m, n] = fp16( sum_g s[g, n] * sum_{k in g} a[m, k] * (q[k, n] - z[g, n]) ),
// fp32 accumulation. The weights are the big operand, so the MMA is "swapped":
// the MMA's M dimension is N (128 output columns per CTA, one per TMEM lane),
// its N dimension is the activation rows (padded to MN, a multiple of 16), and
//   D[n, m] += A[n, k] * B[k, m],  A = (q - z)^T from TMEM, B = activations^T.
//
// (q - z) is an integer in [-15, 15]: exact in fp16, and its products with the
// fp16 activations are exact in the fp32 accumulator, so each group's partial
// sum D_g is exact up to fp32 summation; the fp16 scale is applied in fp32 when
// D_g is read back (tot += s[g, n] * D_g), never rounded into the weights. The exact unpack is
// the exponent-bias ("magic number") technique of Kim et al. 2022 and Frantar et al. 2024
// (MARLIN), derived here from the fp16 layout: 0x6400 | q is 1024 + q.
//
// Roles (one CTA = one 128-column tile x one K slab; 19 warps, 15 at MN = 16):
//   warps 0-7   dequantisers: warp p owns TMEM lanes 32(p%4)..+31 and tile
//               columns 32(p%4)..+31 (one 16-byte chunk of each weight row);
//               warps 0-3 take the even stages and 4-7 the odd ones;
//               ldmatrix.trans hands every thread two k-rows of 4 columns per
//               register, which become exact fp16 (q - z) pairs (0x6400 magic +
//               fp16 subtract) written to TMEM with tcgen05.st.16x128b.x4;
//   warp 8      weight producer: per stage of 128 k-rows, one 2-D TMA load of
//               the tile's packed words [128 rows x 64 B] (64-byte swizzle) into
//               a ring of up to 16 stages;
//   warp 9      activation producer: per stage, two TMA loads of the activation
//               tile [MN x 64] (128-byte swizzle, the canonical K-major layout of
//               operand B), into an 8-stage ring (4 above MN = 48);
//   warp 10     TMEM allocator and MMA issuer: tcgen05.mma.kind::f16 with A
//               from TMEM and B from shared memory, 8 per stage (K = 16 each);
//               a fresh accumulator per group segment, in a ring of TMEM
//               buffers, and a tcgen05.commit to an mbarrier at each segment
//               end. When G is a multiple of 128 (segments are whole stages) the
//               stage loop is unrolled over the ring so that every operand
//               address is a constant offset: measured on B200, the issue loop's
//               own instructions and barrier waits, not the tensor core, set the
//               MMA rate at these small N (about 220 cycles per MMA with per-MMA
//               bookkeeping, 62 with this form and one wait per stage, 36 for
//               the MMAs alone at N = 32);
//   warps 11-18 epilogue (11-14 at MN = 16): tcgen05.ld of each finished group
//               segment, scaled by s[g, n] in fp32 into register totals; then the
//               fp16 (or fp32) output, or the fp32 split-K partial and the
//               last-CTA ordered reduction.
// Every mbarrier wait is bounded; a wait that runs out sets the workspace
// status word to W4A16_ERR_TIMEOUT, and all roles drain and leave, freeing TMEM.
//
// Lane/column bookkeeping: dequantiser thread t of warp p (q = p % 4, t0 = t % 4,
// t1 = t / 4) holds tile columns 32q + 4 t1 + {0, 1, 2, 3} (nibbles 4(t1%2)..
// of packed word 4q + t1/2) and writes them to TMEM lanes {t1, t1+8, t1+16,
// t1+24} (+32q): lane L holds column 32q + 4 (L % 8) + L / 8. Columns at odd
// nibble positions come out of the unpack scaled by 16 (exact), undone in the
// epilogue. The thread's k-pair in each 8-row matrix is t0, i.e. TMEM column
// (k - k_stage) / 2 of the stage's A slot, in natural k order.
#include "common.cuh"
#include "ptx.cuh"

#include <algorithm>
#include <atomic>

namespace w4a16 {
namespace {

constexpr int kBlockN = 128;                    // MMA M = TMEM lanes = output columns per CTA
constexpr int kTileWords = kBlockN / 8;         // 16 packed words per k-row of the tile
constexpr int kStageK = 128;                    // k-rows per pipeline stage
constexpr int kWStageBytes = kStageK * kTileWords * 4;   // 128 rows x 64 B, 64-byte swizzle
constexpr int kBoxK = 64;                       // activation TMA box width (128 B: the 128-byte swizzle's limit)
constexpr int kBoxes = kStageK / kBoxK;         // activation boxes per stage
constexpr int kMmaPerStage = kStageK / 16;      // K = 16 per tcgen05.mma.kind::f16
constexpr int kAColsPerStage = kStageK / 2;     // TMEM columns of one A slot (two fp16 per column)
constexpr int kTmemStages = 4;                  // A slots in TMEM
// Dequantiser warps: groups of four (one per TMEM lane quarter) that take turns on the stages. A
// group's stage ends with a wait for its TMEM stores; a second group keeps another stage in flight
// meanwhile. Measured on B200 (K=4096, N=14336, PDL): M = 128 33.4 -> 27.9 us with two groups
// (and the two epilogue warpgroups below).
__host__ __device__ constexpr int deq_warps(int mn) { return (void)mn, 8; }
// Weight producers: stage i of the weight ring is issued by producer i % P (one: measured on
// B200 at M = 32, four issuing warps did not raise the weight rate).
__host__ __device__ constexpr int wproducer_warps(int mn) { return (void)mn, 1; }
// Epilogue warps: one warpgroup at MN = 16, else two that split the accumulator's columns (rows
// of A) into halves of MN / 2. Each epilogue thread loads its share of every group's accumulator
// from TMEM and adds it, scaled, to per-row totals in registers; measured on B200 (M = 128,
// dequantisers and MMAs doing no work), one warpgroup spent ~0.7 us per group on it. At M = 32
// two warpgroups save ~0.6 us per call; at MN = 48 (K=4096, N=6144) one warpgroup made the call
// slower (44.8 us) than MN = 64 with two (34.4 us).
__host__ __device__ constexpr int epi_warps(int mn) { return mn >= 32 ? 8 : 4; }
// Warps: dequantisers, weight producers, an activation producer, the MMA issuer, the epilogue.
__host__ __device__ constexpr int tc_threads(int mn) {
    return (deq_warps(mn) + wproducer_warps(mn) + 2 + epi_warps(mn)) * 32;
}

template <int MN>
struct TcCfg {
    // Weights and activations have rings of their own. A weight slot is free again as soon as its
    // dequantiser group has read it; an activation slot only when the stage's MMAs have completed.
    // Measured on B200 (M = 32, per-stage timeline): with one ring released by the MMA commit, a
    // slot was busy ~1.3 us after its data landed and a refill took ~2.85 us to land, which set
    // the stage rate (12 slots per ~4.1 us).
    static constexpr int kAStages = MN <= 48 ? 8 : 4;   // a multiple of kTmemStages (unrolled MMA loop)
    static constexpr int kBoxBytes = MN * kBoxK * 2;        // one activation box: MN rows x 128 B
    static constexpr int kBStageBytes = kBoxes * kBoxBytes;
    static constexpr int kWStagesFit = (200 * 1024 - kAStages * kBStageBytes) / kWStageBytes;
    static constexpr int kWStages = (kWStagesFit > 16 ? 16 : kWStagesFit) / wproducer_warps(MN) * wproducer_warps(MN);
    // Accumulator buffers in TMEM: the MMAs of segment g + kDBufs wait for the epilogue to have read
    // segment g. Measured on B200 (M = 32, per-stage timeline): with two buffers that round trip
    // (MMA completion, commit, epilogue read-out) set the stage rate at ~0.45 us, the MMA warp
    // running ~1.2 us behind the dequantisers; the columns left after the A slots allow more.
    static constexpr int kDBufs = MN <= 32 ? 8 : MN <= 64 ? 4 : 2;
    static constexpr int kDCol = kTmemStages * kAColsPerStage;   // first accumulator column
    static constexpr int kColsNeeded = kDCol + kDBufs * MN;
    static constexpr int kTmemCols = kColsNeeded <= 32 ? 32 : kColsNeeded <= 64 ? 64 : kColsNeeded <= 128 ? 128
                                   : kColsNeeded <= 256 ? 256 : 512;
    static constexpr size_t kSmemBytes = 1024 /*align slack*/ + (size_t)kAStages * kBStageBytes +
                                         (size_t)kWStages * kWStageBytes;
};

struct TcArgs {
    const uint32_t* b;     // [K, N/8]
    const __half* s;       // [K/G, N]
    const uint32_t* z;     // [K/G, N/8] or nullptr
    OutPtr out;            // [M, N] (already offset to this row block)
    float* partials;       // [split][mblk][N]
    uint32_t* counters;    // [n_tiles]
    int* status;           // workspace status word
    int64_t N, K;
    int G, zp_bias, split, mblk, m0;
    uint32_t magic;        // 0x64006400, passed at run time so that (x & mask) | magic is one logic op
    int stall_loads;       // tests only: the producer issues nothing (every wait runs out)
    uint64_t wait_ns;      // limit on each device-side wait
};

__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Shared-memory matrix descriptor for a K-major operand tile in the 128-byte
// swizzle layout: rows of 64 fp16 (128 B), 8-row atoms 1024 B apart.
__device__ __forceinline__ uint64_t kmajor_sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4)      // start address, 16-byte units
         | ((uint64_t)1 << 16)                       // leading byte offset (unused for this layout)
         | ((uint64_t)(1024 >> 4) << 32)             // stride byte offset: 8 rows x 128 B
         | ((uint64_t)1 << 46)                       // descriptor version (sm_100)
         | ((uint64_t)2 << 61);                      // 128-byte swizzle
}

// Instruction descriptor: fp16 A and B (K-major), fp32 D, M = 128, N = MN.
template <int MN>
__device__ __forceinline__ uint32_t idesc_f16() {
    return (1u << 4) | ((uint32_t)(MN >> 3) << 17) | ((uint32_t)(kBlockN >> 4) << 24);
}

// The slab's rows; a segment of 16-k MMA steps ends at a group end or at the slab end.
struct SegIter {
    int64_t k_lo, k_hi;  // slab rows
    int G;
};

// FAST: G is a multiple of the stage (kStageK rows), so group segments are whole stages.
template <int MN, bool FAST>
__global__ void __launch_bounds__(tc_threads(MN), 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap wmap, TcArgs p) {
    using C = TcCfg<MN>;
    constexpr int kDeqWarps = deq_warps(MN);
    constexpr int kWProducers = wproducer_warps(MN);
    constexpr int kWProducer = kDeqWarps, kAProducer = kDeqWarps + kWProducers, kMmaWarp = kAProducer + 1,
                  kEpiWarp0 = kMmaWarp + 1;
    constexpr int kEpiWarps = epi_warps(MN), kEpiThreads = 32 * kEpiWarps;
    constexpr int EH = MN / (kEpiWarps / 4);   // accumulator columns (rows of A) per epilogue warpgroup
    constexpr int WS = C::kWStages, AS = C::kAStages;
    static_assert(WS % kWProducers == 0, "every weight slot has one producer");
    extern __shared__ __align__(1024) unsigned char s_raw[];
    unsigned char* s_base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(s_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char* s_b = s_base;                                   // [AS][2][MN x 128 B], 1024-aligned boxes
    unsigned char* s_w = s_base + (size_t)AS * C::kBStageBytes;    // [WS][128 rows x 64 B], 1024-aligned stages

    // weight ring (TMA / dequantiser group) and activation ring (TMA / MMA commit)
    __shared__ __align__(8) uint64_t bar_wfull[WS], bar_wempty[WS], bar_full[AS], bar_empty[AS];
    __shared__ __align__(8) uint64_t bar_afull[kTmemStages], bar_aempty[kTmemStages];
    constexpr int DB = C::kDBufs;
    __shared__ __align__(8) uint64_t bar_dfull[DB], bar_dempty[DB], bar_drain;
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;
    __shared__ int s_last;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = blockIdx.x;
    const int64_t nstage_all = p.K / kStageK;
    const int64_t st_lo = nstage_all * blockIdx.y / p.split, st_hi = nstage_all * (blockIdx.y + 1) / p.split;
    const int nst = (int)(st_hi - st_lo);
    const SegIter seg{st_lo * kStageK, st_hi * kStageK, p.G};

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int i = 0; i < WS; ++i) {
            ptx::mbar_init(ptx::smem_addr(&bar_wfull[i]), 1);
            ptx::mbar_init(ptx::smem_addr(&bar_wempty[i]), 4);   // the four warps of a dequantiser group
        }
        for (int i = 0; i < AS; ++i) {
            ptx::mbar_init(ptx::smem_addr(&bar_full[i]), 1);
            ptx::mbar_init(ptx::smem_addr(&bar_empty[i]), 1);
        }
        for (int i = 0; i < kTmemStages; ++i) {
            ptx::mbar_init(ptx::smem_addr(&bar_afull[i]), 128);   // one group of four warps per stage
            ptx::mbar_init(ptx::smem_addr(&bar_aempty[i]), 1);
        }
        for (int i = 0; i < DB; ++i) {
            ptx::mbar_init(ptx::smem_addr(&bar_dfull[i]), 1);
            ptx::mbar_init(ptx::smem_addr(&bar_dempty[i]), 32 * kEpiWarps);
        }
        ptx::mbar_init(ptx::smem_addr(&bar_drain), 1);
        ptx::mbar_fence_init();
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_addr(&s_tmem), C::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = s_tmem;
    // With programmatic dependent launch the next kernel on the stream may be scheduled now. This
    // one waits for the kernel before it (griddepcontrol.wait) only where it reads what that kernel
    // may have written (the activations) and before it writes (output, workspace); the weights,
    // scales and zeros stream from the start. Without the launch attribute both are no-ops.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == kAProducer) {
        // ------------------------------------------------- activation producer
        // The activation ring, in stage order: two 2-D TMA boxes per stage (MN rows x 64 k each,
        // 128-byte swizzle, rows past M read as zero). Converged loop, one elected lane issuing.
        const bool leader = ptx::elect_one();
        if (leader) ptx::prefetch_tensormap(&amap);
        asm volatile("griddepcontrol.wait;" ::: "memory");   // the activations come from the kernel before
        int issued = 0;
        for (int i = 0; i < nst && !p.stall_loads; ++i) {
            const int s = i % AS;
            const bool okw = ptx::mbar_wait(ptx::smem_addr(&bar_empty[s]), ((i / AS) & 1) ^ 1, &s_abort, p.wait_ns);
            if (!__all_sync(0xffffffffu, okw)) break;
            if (leader) {
                const uint32_t full = ptx::smem_addr(&bar_full[s]);
                ptx::mbar_arrive_expect_tx(full, (uint32_t)C::kBStageBytes);
                const int32_t k0 = (int32_t)((st_lo + i) * kStageK);
#pragma unroll
                for (int x = 0; x < kBoxes; ++x)
                    ptx::tma_load_2d(ptx::smem_addr(s_b + (size_t)s * C::kBStageBytes + x * C::kBoxBytes), &amap,
                                     k0 + x * kBoxK, p.m0, full);
            }
            __syncwarp();
            issued = i + 1;
        }
        if (s_abort && leader) {  // let copies already issued land before the CTA leaves
            volatile int dummy = 0;
            for (int i = max(0, issued - AS); i < issued; ++i)
                ptx::mbar_wait(ptx::smem_addr(&bar_full[i % AS]), (i / AS) & 1, &dummy, p.wait_ns);
        }
    } else if (warp >= kWProducer && warp < kAProducer) {
        // ------------------------------------------------------------ weight producers
        // Weight producer p streams weight stages p, p + P, ... Converged loops, one elected lane
        // issuing (as for the MMA warp).
        const int R = WS;
        const int first = warp - kWProducer, step = kWProducers;
        uint64_t* fullb = bar_wfull;
        uint64_t* emptyb = bar_wempty;
        const bool leader = ptx::elect_one();
        if (leader) ptx::prefetch_tensormap(&wmap);
        const uint32_t tx = (uint32_t)kWStageBytes;
        int issued = -1;   // last stage this warp issued
        for (int i = first; i < nst && !p.stall_loads; i += step) {
            const int s = i % R;
            const bool okw = ptx::mbar_wait(ptx::smem_addr(&emptyb[s]), ((i / R) & 1) ^ 1, &s_abort, p.wait_ns);
            if (!__all_sync(0xffffffffu, okw)) break;
            if (leader) {
                const uint32_t full = ptx::smem_addr(&fullb[s]);
                ptx::mbar_arrive_expect_tx(full, tx);
                const int32_t k0 = (int32_t)((st_lo + i) * kStageK);
                ptx::tma_load_2d(ptx::smem_addr(s_w + (size_t)s * kWStageBytes), &wmap, tile * kTileWords, k0, full);
            }
            __syncwarp();
            issued = i;
        }
        if (s_abort && leader) {  // let copies already issued land before the CTA leaves
            volatile int dummy = 0;
            for (int i = issued; i >= 0 && i > issued - R; i -= step)
                ptx::mbar_wait(ptx::smem_addr(&fullb[i % R]), (i / R) & 1, &dummy, p.wait_ns);
        }
    } else if (warp < kDeqWarps) {
        // -------------------------------------------------------- dequantisers
        constexpr int kDeqGroups = kDeqWarps / 4;
        const int q = warp & 3, dg = warp >> 2;   // TMEM lane quarter / column chunk; my group
        const int t1 = lane >> 2;
        const int64_t nw = p.N / 8;
        const int64_t word = (int64_t)tile * kTileWords + 4 * q + (t1 >> 1);  // holds my 4 columns
        const int nib0 = 4 * (t1 & 1);                                       // their first nibble
        const int64_t ngroups = p.K / p.G;
        // g_next_k is the end of the open group. A warp that dequantises every other stage may skip
        // groups, so the group is found from the row; its zero word is prefetched for the group
        // after it.
        int64_t g_next_k = st_lo * kStageK / p.G * p.G, g_pref = -1;
        uint32_t zw_next = 0u;
        bool have_next = false;
        uint32_t bias0 = 0, bias1 = 0, bias2 = 0, bias3 = 0;
        const uint32_t magic = p.magic;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        // (1024 + z) for low-nibble columns, (1024 + 16 z) for high ones, in both halves
        auto set_bias = [&](uint32_t zw) {
            bias0 = (0x6400u + (zw & 0xFu)) * 0x00010001u;
            bias1 = (0x6400u + 16u * ((zw >> 4) & 0xFu)) * 0x00010001u;
            bias2 = (0x6400u + ((zw >> 8) & 0xFu)) * 0x00010001u;
            bias3 = (0x6400u + 16u * ((zw >> 12) & 0xFu)) * 0x00010001u;
        };
        auto enter_group = [&](int64_t kk) {
            const int64_t g = kk / p.G;
            g_next_k = (g + 1) * p.G;
            uint32_t zraw = 0u;
            if (p.z) {
                zraw = have_next && g == g_pref ? zw_next : __ldg(p.z + g * nw + word);
                g_pref = g + 1;
                have_next = g_pref < ngroups;
                if (have_next) zw_next = __ldg(p.z + g_pref * nw + word);
            }
            set_bias(p.z ? (zraw >> (4 * nib0)) : (uint32_t)p.zp_bias * 0x1111u);
        };
        // FAST: one group per stage; the zero words of my next four stages are loaded ahead in a
        // register ring (a DRAM round trip is longer than one or two stages).
        auto zero_of_stage = [&](int st) -> uint32_t {
            return (p.z && st < nst) ? __ldg(p.z + (st_lo + st) * kStageK / p.G * nw + word) : 0u;
        };
        uint32_t zr0 = 0u, zr1 = 0u, zr2 = 0u, zr3 = 0u;
        if (FAST) {
            if (p.z) {
                zr0 = zero_of_stage(dg);
                zr1 = zero_of_stage(dg + kDeqGroups);
                zr2 = zero_of_stage(dg + 2 * kDeqGroups);
                zr3 = zero_of_stage(dg + 3 * kDeqGroups);
            } else {
                set_bias((uint32_t)p.zp_bias * 0x1111u);
            }
        }
        for (int i = dg; i < nst; i += kDeqGroups) {
            const int s = i % WS, ts = i % kTmemStages;
            // Wait outcomes are made warp-uniform: the tcgen05 stores below are .sync.aligned. The
            // stage's activations are waited for here too, so that the MMA warp's one wait (for the
            // TMEM slot) also orders the activation tile before its MMAs.
            bool okw = ptx::mbar_wait(ptx::smem_addr(&bar_wfull[s]), (i / WS) & 1, &s_abort, p.wait_ns);
            okw = okw && ptx::mbar_wait(ptx::smem_addr(&bar_full[i % AS]), (i / AS) & 1, &s_abort, p.wait_ns);
            okw = okw && ptx::mbar_wait(ptx::smem_addr(&bar_aempty[ts]), ((i / kTmemStages) & 1) ^ 1, &s_abort,
                                        p.wait_ns);
            if (!__all_sync(0xffffffffu, okw)) break;
            ptx::tc_fence_after();
            const uint32_t wbase = ptx::smem_addr(s_w + (size_t)s * kWStageBytes);
            if (FAST && p.z) {
                set_bias(zr0 >> (4 * nib0));
                zr0 = zr1;
                zr1 = zr2;
                zr2 = zr3;
                zr3 = zero_of_stage(i + 4 * kDeqGroups);
            }
#pragma unroll
            for (int hh = 0; hh < kStageK / 32; ++hh) {
                // rows 32hh .. 32hh + 31 as four 8x8 matrices of 16-bit halves; my address row is
                // 32hh + lane; 16-byte chunk q of it, moved by the 64-byte swizzle
                const int row = 32 * hh + lane;
                uint32_t R[4];
                ptx::ldmatrix_x4_trans(wbase + row * 64 + 16 * (q ^ ((row >> 1) & 3)), R);
                const int64_t k_half = (st_lo + i) * kStageK + 32 * hh;   // first k of these 32 rows
                uint32_t lo[8], hi[8];
#pragma unroll
                for (int mi = 0; mi < 4; ++mi) {
                    // G % 16 == 0: an 8-row matrix never straddles a group boundary
                    if (!FAST && k_half + 8 * mi >= g_next_k) enter_group(k_half + 8 * mi);
                    const uint32_t x = R[mi], y = x >> 8;
                    lo[2 * mi] = hsub2((x & 0x000F000Fu) | magic, bias0);
                    lo[2 * mi + 1] = hsub2((x & 0x00F000F0u) | magic, bias1);
                    hi[2 * mi] = hsub2((y & 0x000F000Fu) | magic, bias2);
                    hi[2 * mi + 1] = hsub2((y & 0x00F000F0u) | magic, bias3);
                }
                const uint32_t col = (uint32_t)(ts * kAColsPerStage + 16 * hh);
                ptx::tmem_st_16x128b_x4(lane_base + col, lo);
                ptx::tmem_st_16x128b_x4(lane_base + (16u << 16) + col, hi);
                if (hh == kStageK / 32 - 1) {
                    // the weight stage is read: its slot can be refilled
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bar_wempty[s]));
                }
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            ptx::mbar_arrive(ptx::smem_addr(&bar_afull[ts]));
        }
    } else if (warp == kMmaWarp) {
        // ----------------------------------------------------------- MMA issuer
        // The whole warp runs the loop (so the operands stay warp-uniform) and one elected lane
        // issues the MMAs and commits.
        const bool leader = ptx::elect_one();
        const uint32_t idesc = idesc_f16<MN>();
        int sg = 0;              // segment counter
        if constexpr (FAST) {
            // Segments are whole stages: `rem` counts the stages left in the open group. The stage
            // loop is unrolled over the ring, so slot, A-slot and B-descriptor offsets are constants.
            const int gs = p.G / kStageK;
            int rem = gs - (int)(st_lo % gs);
            const uint64_t bdesc0 = kmajor_sw128_desc(ptx::smem_addr(s_b));
            const uint32_t t_d = tmem + (uint32_t)C::kDCol;
            bool ok = true;
            for (int i0 = 0; i0 < nst && ok; i0 += AS) {
#pragma unroll
                for (int u = 0; u < AS; ++u) {
                    const int i = i0 + u;
                    if (i >= nst) break;
                    constexpr int kTsMask = kTmemStages - 1;
                    const int ts = u & kTsMask;
                    const bool seg_start = rem == gs || i == 0;
                    const bool seg_end = rem == 1 || i == nst - 1;
                    const int db = sg % DB;
                    // The stage's A slot is complete only after every thread of its dequantiser group
                    // has waited for the stage's TMA barrier, so this wait also orders the activation
                    // tile before the MMAs (a second wait on that barrier cost ~150 cycles per stage).
                    bool okw = ptx::mbar_wait(ptx::smem_addr(&bar_afull[ts]), (i / kTmemStages) & 1, &s_abort,
                                              p.wait_ns);
                    if (seg_start)
                        okw = okw && ptx::mbar_wait(ptx::smem_addr(&bar_dempty[db]), ((sg / DB) & 1) ^ 1, &s_abort,
                                                    p.wait_ns);
                    if (!__all_sync(0xffffffffu, okw)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    if (leader) {
                        const uint32_t d = t_d + (uint32_t)(db * MN);
                        const uint32_t a = tmem + (uint32_t)(ts * kAColsPerStage);
                        const uint64_t b = bdesc0 + (uint64_t)((u * C::kBStageBytes) >> 4);
#pragma unroll
                        for (int j = 0; j < kMmaPerStage; ++j) {
                            // A: 8 TMEM columns per 16 k; B: box j / 4, +32 B (2 descriptor units) per 16 k
                            const uint64_t bj = b + (uint64_t)(((j / 4) * C::kBoxBytes + 32 * (j % 4)) >> 4);
                            ptx::mma_f16_ts(d, a + 8 * j, bj, idesc, (j == 0 && seg_start) ? 0u : 1u);
                        }
                        if (seg_end) ptx::mma_commit(ptx::smem_addr(&bar_dfull[db]));
                        ptx::mma_commit(ptx::smem_addr(&bar_empty[u]));
                        ptx::mma_commit(ptx::smem_addr(&bar_aempty[ts]));
                    }
                    __syncwarp();
                    if (seg_end) {
                        ++sg;
                        rem = gs;
                    } else {
                        --rem;
                    }
                }
            }
        } else {
            uint32_t acc = 0;
            // Segments of 16-k steps end at a group boundary or at the slab end; tracked incrementally.
            int64_t seg_next = (seg.k_lo / p.G + 1) * p.G;   // next group boundary after the slab start
            bool starts = true;
            for (int i = 0; i < nst; ++i) {
                const int s = i % AS, ts = i % kTmemStages;
                bool okw = ptx::mbar_wait(ptx::smem_addr(&bar_afull[ts]), (i / kTmemStages) & 1, &s_abort, p.wait_ns);
                okw = okw && ptx::mbar_wait(ptx::smem_addr(&bar_full[s]), (i / AS) & 1, &s_abort, p.wait_ns);
                if (!__all_sync(0xffffffffu, okw)) break;
                ptx::tc_fence_after();
                const uint32_t bbase = ptx::smem_addr(s_b + (size_t)s * C::kBStageBytes);
                bool ok = true;
#pragma unroll
                for (int j = 0; j < kMmaPerStage; ++j) {
                    const int64_t k = (st_lo + i) * kStageK + 16 * j;
                    const int db = sg % DB;
                    const bool ends = k + 16 == seg.k_hi || k + 16 == seg_next;
                    if (k + 16 == seg_next) seg_next += p.G;
                    if (starts) {
                        const bool okd = ptx::mbar_wait(ptx::smem_addr(&bar_dempty[db]), ((sg / DB) & 1) ^ 1,
                                                        &s_abort, p.wait_ns);
                        if (!__all_sync(0xffffffffu, okd)) {
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        acc = 0;
                    }
                    if (leader)
                        ptx::mma_f16_ts(tmem + (uint32_t)(C::kDCol + db * MN),
                                        tmem + (uint32_t)(ts * kAColsPerStage + 8 * j),
                                        kmajor_sw128_desc(bbase + (j / 4) * C::kBoxBytes + 32 * (j % 4)), idesc, acc);
                    acc = 1;
                    starts = ends;
                    if (ends) {
                        if (leader) ptx::mma_commit(ptx::smem_addr(&bar_dfull[db]));
                        ++sg;
                    }
                }
                if (leader) {
                    ptx::mma_commit(ptx::smem_addr(&bar_empty[s]));
                    ptx::mma_commit(ptx::smem_addr(&bar_aempty[ts]));
                }
                __syncwarp();
                if (!ok) break;
            }
        }
        // Wait for every MMA issued above before TMEM can be released.
        if (leader) ptx::mma_commit(ptx::smem_addr(&bar_drain));
        __syncwarp();
        volatile int dummy = 0;
        ptx::mbar_wait(ptx::smem_addr(&bar_drain), 0, &dummy, p.wait_ns);
    } else {
        // -------------------------------------------------------------- epilogue
        const int sub = warp & 3;                           // TMEM lanes 32 sub .. 32 sub + 31
        const int et = threadIdx.x - 32 * kEpiWarp0;        // index within the epilogue warps
        const int m0 = (et / 128) * EH;                     // my warpgroup's first accumulator column
        const int ncol = 32 * sub + 4 * (lane & 7) + (lane >> 3);
        const int64_t n = (int64_t)tile * kBlockN + ncol;
        const float fscale = (lane >> 3) & 1 ? 0.0625f : 1.0f;
        float tot[EH];
#pragma unroll
        for (int m = 0; m < EH; ++m) tot[m] = 0.f;
        int sg = 0;
        bool ok = true;
        // Segment ends in order (group boundaries, tracked incrementally).
        int64_t g_idx = seg.k_lo / p.G;                    // group of the current segment
        int64_t bound = (g_idx + 1) * p.G;                 // its end row (or the slab end)
        const int64_t g_last = (seg.k_hi - 1) / p.G;       // last group of the slab
        // Segments are consecutive groups. Their scales are loaded eight segments ahead into a ring
        // of raw fp16 bits and converted only when their segment is read. Converting at load time
        // made the thread wait for every load at once: a per-stage timeline on B200 (M = 32) showed
        // this epilogue as the slowest role, ~0.4-0.55 us per segment for 0.06 us of work, behind
        // scale loads that queue with the weight stream in DRAM for 1-4 us.
        constexpr int kSR = 8;
        auto scale_raw = [&](int64_t g) -> unsigned short {
            return g <= g_last ? __ldg(reinterpret_cast<const unsigned short*>(p.s) + g * p.N + n)
                               : (unsigned short)0;
        };
        unsigned short sr[kSR];
#pragma unroll
        for (int j = 0; j < kSR; ++j) sr[j] = scale_raw(g_idx + j);
        int64_t k_end = min(seg.k_hi, bound) - 16;
        while (k_end >= seg.k_lo && ok) {
            const int64_t k_next = k_end + 16 < seg.k_hi ? min(seg.k_hi, bound + p.G) - 16 : -1;
            const float sc = fscale * __half2float(__ushort_as_half(sr[0]));
#pragma unroll
            for (int j = 0; j < kSR - 1; ++j) sr[j] = sr[j + 1];
            sr[kSR - 1] = scale_raw(g_idx + kSR);
            const int db = sg % DB;
            const bool okw = ptx::mbar_wait(ptx::smem_addr(&bar_dfull[db]), (sg / DB) & 1, &s_abort, p.wait_ns);
            if (!__all_sync(0xffffffffu, okw)) {  // warp-uniform: tcgen05.ld is .sync.aligned
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(32 * sub) << 16) + (uint32_t)(C::kDCol + db * MN + m0);
            // Loads of 16 columns start on 16-column boundaries, of 8 on 8-column ones: a half of
            // MN = 48, 80 or 112 (24, 40 or 56 columns) reads its odd 8 columns with one x8 load,
            // first in the upper half (which starts 8 past a 16-column boundary), last in the lower.
            if (EH % 16 != 0 && m0 != 0) {
                uint32_t v[8];
                ptx::tmem_ld_32x32b_x8(taddr, v);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 8; ++q) tot[q] = fmaf(sc, __uint_as_float(v[q]), tot[q]);
            }
            const int c_off = (EH % 16 != 0 && m0 != 0) ? 8 : 0;
#pragma unroll
            for (int c0 = 0; c0 + 16 <= EH; c0 += 16) {
                uint32_t v[16];
                ptx::tmem_ld_32x32b_x16(taddr + c_off + c0, v);
                ptx::tmem_wait_ld();
                if (c_off) {
#pragma unroll
                    for (int q = 0; q < 16; ++q) tot[8 + c0 + q] = fmaf(sc, __uint_as_float(v[q]), tot[8 + c0 + q]);
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) tot[c0 + q] = fmaf(sc, __uint_as_float(v[q]), tot[c0 + q]);
                }
            }
            if (EH % 16 != 0 && m0 == 0) {
                uint32_t v[8];
                ptx::tmem_ld_32x32b_x8(taddr + (EH - 8), v);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 8; ++q) tot[EH - 8 + q] = fmaf(sc, __uint_as_float(v[q]), tot[EH - 8 + q]);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(ptx::smem_addr(&bar_dempty[db]));
            ++sg;
            k_end = k_next;
            ++g_idx;
            bound += p.G;
        }
        // One decision for all epilogue threads (a timeout seen by any of them,
        // or by another role, skips the output), so the named barriers below match.
        const bool bad = ptx::named_bar_or(1, kEpiThreads, !ok || s_abort);
        asm volatile("griddepcontrol.wait;" ::: "memory");   // before the first write
        if (!bad) {
            if (p.split == 1) {
                // The tile goes out through shared memory: every stage has been consumed (the last
                // group's accumulator is complete, so every MMA, and before them every dequantiser
                // read and every load, has finished), so the weight ring is idle. Each thread puts its
                // column there row-major, then whole rows leave as 16-byte stores. Measured on B200
                // (M = 128), one 2-byte store per row and thread took ~3.9 us at the end of the launch.
                const bool f32 = p.out.f != nullptr;
                const int esz = f32 ? 4 : 2;
                unsigned char* stg = s_w;
#pragma unroll
                for (int m = 0; m < EH; ++m) {
                    if (f32) reinterpret_cast<float*>(stg)[(m0 + m) * kBlockN + ncol] = tot[m];
                    else reinterpret_cast<__half*>(stg)[(m0 + m) * kBlockN + ncol] = __float2half_rn(tot[m]);
                }
                ptx::named_bar_sync(1, kEpiThreads);
                unsigned char* obase = f32 ? reinterpret_cast<unsigned char*>(p.out.f) : reinterpret_cast<unsigned char*>(p.out.h);
                const int64_t row_stride = p.N * esz, col0 = (int64_t)tile * kBlockN * esz;
                if (((reinterpret_cast<uintptr_t>(obase) | (uintptr_t)row_stride) & 15) == 0) {
                    const int cpr = kBlockN * esz / 16;   // 16-byte chunks per row of the tile
                    for (int c = et; c < p.mblk * cpr; c += kEpiThreads) {
                        const int r = c / cpr, q = c % cpr;
                        const uint4 v = *reinterpret_cast<const uint4*>(stg + r * kBlockN * esz + q * 16);
                        *reinterpret_cast<uint4*>(obase + r * row_stride + col0 + q * 16) = v;
                    }
                } else {
                    for (int c = et; c < p.mblk * kBlockN; c += kEpiThreads) {
                        const int r = c / kBlockN, q = c % kBlockN;
                        if (f32) p.out.f[(int64_t)r * p.N + (int64_t)tile * kBlockN + q] = reinterpret_cast<const float*>(stg)[c];
                        else p.out.h[(int64_t)r * p.N + (int64_t)tile * kBlockN + q] = reinterpret_cast<const __half*>(stg)[c];
                    }
                }
            } else {
#pragma unroll
                for (int m = 0; m < EH; ++m)
                    if (m0 + m < p.mblk) p.partials[((int64_t)blockIdx.y * p.mblk + m0 + m) * p.N + n] = tot[m];
                __threadfence();
                ptx::named_bar_sync(1, kEpiThreads);
                if (et == 0) {
                    const uint32_t ticket = atomicAdd(p.counters + tile, 1u);
                    s_last = (ticket == (uint32_t)p.split - 1);
                }
                ptx::named_bar_sync(1, kEpiThreads);
                if (s_last) {
                    // The last-arriving CTA adds the tile's partials in split order (0 + p0 + p1 + ...).
                    __threadfence();
                    if constexpr (EH <= 32) {
                        // The partials of one split for a block of 8 rows are loaded together, and
                        // the block is stored after the last split. Measured on B200 (K=N=4096,
                        // M=32, split 4): the row-by-row loop below, whose store keeps the next
                        // row's loads waiting, took ~11 us in these CTAs against ~2 us for the
                        // others; the call 19.4 -> 13.7 us. (Above 32 rows per warpgroup the blocks
                        // cost the kernel's main loops registers: M=128 26.8 -> 29.8 us unsplit.)
#pragma unroll
                        for (int c0 = 0; c0 < EH; c0 += 8) {
#pragma unroll
                            for (int m = c0; m < c0 + 8 && m < EH; ++m) tot[m] = 0.f;
                            for (int y = 0; y < p.split; ++y) {
                                const float* py = p.partials + ((int64_t)y * p.mblk + m0) * p.N + n;
#pragma unroll
                                for (int m = c0; m < c0 + 8 && m < EH; ++m)
                                    if (m0 + m < p.mblk) tot[m] += __ldcg(py + (int64_t)m * p.N);
                            }
#pragma unroll
                            for (int m = c0; m < c0 + 8 && m < EH; ++m)
                                if (m0 + m < p.mblk) p.out.put((int64_t)(m0 + m) * p.N + n, tot[m]);
                        }
                    } else {
                        for (int m = m0; m < min(m0 + EH, p.mblk); ++m) {
                            float a = 0.f;
                            for (int y = 0; y < p.split; ++y) a += __ldcg(p.partials + ((int64_t)y * p.mblk + m) * p.N + n);
                            p.out.put((int64_t)m * p.N + n, a);
                        }
                    }
                    if (et == 0) p.counters[tile] = 0u;
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (s_abort && threadIdx.x == 0 && p.status) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        atomicExch(p.status, (int)W4A16_ERR_TIMEOUT);
    }
    if (warp == kMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::kTmemCols);
    }
}

using TcFn = void (*)(CUtensorMap, CUtensorMap, TcArgs);

template <bool FAST>
TcFn select_tc_t(int mn) {
    switch (mn) {
        case 16: return tc_gemm_kernel<16, FAST>;
        case 32: return tc_gemm_kernel<32, FAST>;
        case 48: return tc_gemm_kernel<48, FAST>;
        case 64: return tc_gemm_kernel<64, FAST>;
        case 80: return tc_gemm_kernel<80, FAST>;
        case 96: return tc_gemm_kernel<96, FAST>;
        case 112: return tc_gemm_kernel<112, FAST>;
        default: return tc_gemm_kernel<128, FAST>;
    }
}
TcFn select_tc(int mn, bool fast) { return fast ? select_tc_t<true>(mn) : select_tc_t<false>(mn); }

size_t tc_smem(int mn) {
    switch (mn) {
        case 16: return TcCfg<16>::kSmemBytes;
        case 32: return TcCfg<32>::kSmemBytes;
        case 48: return TcCfg<48>::kSmemBytes;
        case 64: return TcCfg<64>::kSmemBytes;
        case 80: return TcCfg<80>::kSmemBytes;
        case 96: return TcCfg<96>::kSmemBytes;
        case 112: return TcCfg<112>::kSmemBytes;
        default: return TcCfg<128>::kSmemBytes;
    }
}

// Dynamic shared memory requested at launch. Shapes up to 32 rows ask for more than half of an
// SM's 228 KB so that each CTA has an SM to itself: measured on B200 (K=4096, N=14336, M=32),
// two CTAs per SM with the K range split in two ran 41.5 us against 31.8 us for 48 rows with one
// CTA per SM and no split.
size_t tc_launch_smem(int mn) { return mn <= 32 ? std::max<size_t>(tc_smem(mn), 116 * 1024) : tc_smem(mn); }

std::atomic<int> g_tc_occ[9];

int tc_ctas_per_sm(int mn) {
    int n = g_tc_occ[mn / 16].load(std::memory_order_relaxed);
    if (n > 0) return n;
    // Resident CTAs per SM from the three budgets the kernel draws on: shared
    // memory (228 KB per SM, 1 KB reserved per CTA), registers (64 K per SM)
    // and tensor memory (512 columns per SM).
    TcFn k = select_tc(mn, true);
    const size_t smem = tc_launch_smem(mn);
    cudaFuncAttributes fa{};
    int regs = 255;
    if (cudaFuncGetAttributes(&fa, k) == cudaSuccess && fa.numRegs > 0) regs = fa.numRegs;
    const int by_smem = (int)((228 * 1024) / (smem + fa.sharedSizeBytes + 1024));
    const int regs_per_warp = (regs + 7) / 8 * 8 * 32;  // allocation granularity: 8 registers per thread
    const int by_regs = 65536 / (regs_per_warp * (tc_threads(mn) / 32));
    const int dbufs = mn <= 32 ? 8 : mn <= 64 ? 4 : 2;   // TcCfg<MN>::kDBufs
    const int cols = kTmemStages * kAColsPerStage + dbufs * mn <= 256 ? 256 : 512;
    n = std::max(1, std::min(std::min(by_smem, by_regs), 512 / cols));
    g_tc_occ[mn / 16].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace

bool tc_supported(int64_t M, int64_t N, int64_t K, int32_t G, const void* a, const void* b) {
    (void)M; (void)G;
    return N % kBlockN == 0 && K % kStageK == 0 && (reinterpret_cast<uintptr_t>(a) % 16) == 0 &&
           (reinterpret_cast<uintptr_t>(b) % 16) == 0;
}

TcPlan plan_tc(int64_t M, int64_t N, int64_t K, int32_t G, int sm_count, int split_k_request) {
    (void)G;
    TcPlan pl{};
    pl.mblk_max = (int)std::min<int64_t>(M, 128);
    pl.mn = (int)((pl.mblk_max + 15) / 16 * 16);
    pl.n_tiles = (int)(N / kBlockN);
    const int64_t nst = K / kStageK;
    const int64_t slots = (int64_t)std::max(sm_count, 1) * tc_ctas_per_sm(pl.mn);
    // Pick the split that fills one wave best, counting the fp32 partials it writes and reads as
    // extra traffic against the packed weights. Only splits whose CTAs are all resident at once
    // are considered: measured on B200 (K=4096, N=28672, M=17, 224 column tiles), a 3-way split in
    // five waves, which this score rated level with no split, took 68.0 us against 36.5 us.
    const int64_t s_max = pl.n_tiles >= slots ? 1 : slots / std::max(pl.n_tiles, 1);
    double best = -1.0;
    int best_s = 1;
    for (int s = 1; s <= 16 && s <= nst && s <= s_max; ++s) {
        const int64_t ctas = (int64_t)pl.n_tiles * s;
        const double waves = (double)((ctas + slots - 1) / slots);
        const double fill = (double)ctas / (waves * slots);
        const double wbytes = (double)K * N / 2;
        const double pbytes = s > 1 ? 2.0 * s * pl.mblk_max * (double)N * 4 : 0.0;
        const double score = fill * wbytes / (wbytes + pbytes);
        if (score > best + 1e-9) {
            best = score;
            best_s = s;
        }
    }
    pl.split_k = split_k_request > 0 ? (int)std::min<int64_t>(split_k_request, nst) : best_s;
    pl.counters_off = kWsHeader;
    pl.partials_off = align_up(kWsHeader + (size_t)pl.n_tiles * 4, 256);
    pl.ws_bytes = pl.partials_off + (pl.split_k > 1 ? (size_t)pl.split_k * pl.mblk_max * (size_t)N * 4 : 0);
    return pl;
}

cudaError_t launch_tc(const __half* a, const uint32_t* b, const __half* s, const uint32_t* z, int64_t M, int64_t N,
                      int64_t K, int32_t G, int32_t zp_bias, OutPtr out, void* workspace, const TcPlan& pl,
                      const WaitPolicy& wp, cudaStream_t st) {
    // Tensor map over the activations [M, K] fp16: box 64 k x MN rows, 128-byte swizzle;
    // rows past M read as zero.
    CUtensorMap amap;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBoxK, (cuuint32_t)pl.mn};
    const cuuint32_t estr[2] = {1, 1};
    cudaError_t e = encode_tensor_map(&amap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void*)a, dims, strides, box, estr,
                                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    // Tensor map over the packed weights [K, N/8] int32: box 16 words x 64 rows, 64-byte swizzle.
    CUtensorMap wmap;
    const cuuint64_t wdims[2] = {(cuuint64_t)(N / 8), (cuuint64_t)K};
    const cuuint64_t wstrides[1] = {(cuuint64_t)(N / 8) * 4};
    const cuuint32_t wbox[2] = {(cuuint32_t)kTileWords, (cuuint32_t)kStageK};
    e = encode_tensor_map(&wmap, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, (void*)b, wdims, wstrides, wbox, estr,
                          CU_TENSOR_MAP_SWIZZLE_64B);
    if (e != cudaSuccess) return e;
    char* ws = static_cast<char*>(workspace);
    for (int64_t m0 = 0; m0 < M; m0 += 128) {
        TcArgs args;
        args.b = b;
        args.s = s;
        args.z = z;
        args.out = out.rows(m0, N);
        args.partials = reinterpret_cast<float*>(ws + pl.partials_off);
        args.counters = reinterpret_cast<uint32_t*>(ws + pl.counters_off);
        args.status = reinterpret_cast<int*>(ws);
        args.N = N;
        args.K = K;
        args.G = G;
        args.zp_bias = zp_bias;
        args.magic = 0x64006400u;
        args.split = pl.split_k;
        args.mblk = (int)std::min<int64_t>(128, M - m0);
        args.m0 = (int)m0;
        args.stall_loads = wp.stall_loads;
        args.wait_ns = wp.limit_ns;
        // Every row block uses the plan's MN (the largest); a short last block
        // leaves its padded rows to TMA's zero fill.
        TcFn k = select_tc(pl.mn, G % kStageK == 0);
        const size_t smem = tc_launch_smem(pl.mn);
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)pl.n_tiles, (unsigned)pl.split_k);
        cfg.blockDim = dim3(tc_threads(pl.mn));
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        // Later row blocks of one call read the same weights and write other rows: they may overlap
        // the block before them whenever the call may overlap its predecessor.
        cfg.numAttrs = wp.pdl ? 1 : 0;
        e = cudaLaunchKernelEx(&cfg, k, amap, wmap, args);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace w4a16
