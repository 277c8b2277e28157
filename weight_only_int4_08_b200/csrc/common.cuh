// Internal declarations shared by the library's translation units (not installed).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "w4a16.h"

namespace w4a16 {

// Workspace layout for the GEMM kernels. Byte offsets from the workspace base.
//   [0, 256)                 device status word (int32 at offset 0) + reserved
//   [256, 256 + tiles*4)     split-K arrival counters, one uint32 per column tile
//   [partials_offset, ...)   fp32 split-K partial sums
constexpr size_t kWsHeader = 256;
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Output of a GEMM launch: the layer's fp16 result (rounded to nearest even), or the
// fp32 sums themselves, unrounded, when the call computes one K-shard's share of a
// row-parallel layer whose shards are added up later (W4A16_OUT_F32).
struct OutPtr {
    __half* h;  // fp16 [M, N], or nullptr
    float* f;   // fp32 [M, N], or nullptr
    __device__ __forceinline__ void put(int64_t i, float v) const {
        if (f) f[i] = v;
        else h[i] = __float2half_rn(v);
    }
    OutPtr rows(int64_t m0, int64_t N) const { return {h ? h + m0 * N : nullptr, f ? f + m0 * N : nullptr}; }
};

// Device-side wait policy for the pipelined kernels: the limit on each wait,
// and (tests only) a switch that makes the load issuers issue nothing.
struct WaitPolicy {
    uint64_t limit_ns;
    int stall_loads;
    int pdl;  // launch with programmatic dependent launch (W4A16_LAUNCH_PDL)
};

struct GemvPlan {
    bool mma;         // tensor-instruction (mma.sync) inner loop, or the CUDA-core fp32 one
    bool tma;         // TMA-fed kernel (N % 32 == 0, 16-byte aligned weights) or plain loads
    int vec;          // int32 words per thread per row (4, 2 or 1)
    int m_rows;       // activation rows handled by one launch (1..8)
    int split_k;      // CTAs along K per column tile (stream-K GEMV: the grid size)
    int col_tiles;    // column tiles
    int cluster;      // mma GEMV: CTAs per thread-block cluster
    int cluster_tiles;  // mma GEMV: whole column tiles per cluster
    int warps;        // mma GEMV: warps per CTA
    int split_k_request;  // the caller's split_k option (0 = automatic)
    size_t ws_bytes;  // workspace bytes needed (0 when split_k == 1)
    size_t counters_off, partials_off;
};

// cuTensorMapEncodeTiled through the runtime's driver entry point (the library
// does not link libcuda, so it loads on machines without a driver).
cudaError_t encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, cuuint32_t rank, void* gaddr,
                              const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                              const cuuint32_t* estrides, CUtensorMapSwizzle swizzle);

// Record the text returned by w4a16_last_error() on the calling thread.
void set_last_error(const char* msg);

// SM count of the current device (cached per device).
int device_sm_count(int* err);

// max_vec: widest packed-word vector (4, 2, 1) the weight pointer's alignment allows;
// tma_ok: the caller allows the TMA-fed kernel.
GemvPlan plan_gemv(int64_t M, int64_t N, int64_t K, int32_t G, int split_k_request, int sm_count, int max_vec,
                   bool tma_ok);

// The stream-K mma.sync GEMV: N % 32 == 0, 16-byte aligned weights and activations,
// 8-byte aligned scales (z, the zeros, may be NULL; 4-byte alignment suffices).
bool gemv_mma_supported(int64_t N, int64_t K, const void* a, const void* b, const void* s, const void* z);
GemvPlan plan_gemv_mma(int64_t M, int64_t N, int64_t K, int32_t G, int split_k_request, int sm_count);
cudaError_t launch_gemv_mma(const __half* a, const uint32_t* b, const __half* s, const uint32_t* z, int64_t M,
                            int64_t N, int64_t K, int32_t G, int32_t zp_bias, OutPtr out, void* workspace,
                            const GemvPlan& plan, const WaitPolicy& wp, cudaStream_t st);

// Largest rows-per-CTA slab the GEMV stages in shared memory for an explicit split.
size_t gemv_smem_bytes(int64_t M, int64_t K, int split_k);

struct TcPlan {
    int mblk_max;     // activation rows per launch (<= 128)
    int mn;           // MMA N: rows padded to a multiple of 16
    int n_tiles;      // N / 128
    int split_k;      // CTAs along K per tile
    size_t ws_bytes;  // workspace bytes (status word + counters + partials)
    size_t counters_off, partials_off;
};

// The tensor-core kernel needs N % 128 == 0, K % 64 == 0 and 16-byte aligned A and weights.
bool tc_supported(int64_t M, int64_t N, int64_t K, int32_t G, const void* a, const void* b);
TcPlan plan_tc(int64_t M, int64_t N, int64_t K, int32_t G, int sm_count, int split_k_request);
cudaError_t launch_tc(const __half* a, const uint32_t* b, const __half* s, const uint32_t* z, int64_t M, int64_t N,
                      int64_t K, int32_t G, int32_t zp_bias, OutPtr out, void* workspace, const TcPlan& plan,
                      const WaitPolicy& wp, cudaStream_t st);

cudaError_t launch_repack(const uint32_t* ckpt, uint32_t* out, int64_t N, int64_t K, cudaStream_t st);

cudaError_t launch_ct_load(const uint32_t* ckpt, const uint16_t* s_ng, const uint32_t* z_n8g, uint32_t* b_kn8,
                           uint16_t* s_gn, uint32_t* z_gn8, int64_t N, int64_t K, int64_t ngroups, cudaStream_t st);

cudaError_t launch_gemv(const __half* a, const uint32_t* b, const __half* s, const uint32_t* z,
                        int64_t M, int64_t N, int64_t K, int32_t G, int32_t zp_bias, OutPtr out,
                        void* workspace, const GemvPlan& plan, const WaitPolicy& wp, cudaStream_t st);

// Sum of P fp32 [M, N] partials in fixed order, rounded once to fp16 (16-byte aligned
// pointers, M * N % 8 == 0).
constexpr int kMaxReduceParts = 16;
cudaError_t launch_reduce_partials(const float* const* parts, int P, int64_t M, int64_t N, __half* out, int sm_count,
                                   cudaStream_t st);

}  // namespace w4a16
