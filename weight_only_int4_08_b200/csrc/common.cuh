// Internal declarations shared by the library's translation units (not installed).
#pragma once

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

struct GemvPlan {
    int vec;          // int32 words per thread per row (4, 2 or 1)
    int m_rows;       // activation rows handled by one launch (1..8)
    int split_k;      // CTAs along K per column tile
    int col_tiles;    // CTAs along N
    size_t ws_bytes;  // workspace bytes needed (0 when split_k == 1)
    size_t counters_off, partials_off;
};

// SM count of the current device (cached per device).
int device_sm_count(int* err);

// max_vec: widest packed-word vector (4, 2, 1) the weight pointer's alignment allows.
GemvPlan plan_gemv(int64_t M, int64_t N, int64_t K, int32_t G, int split_k_request, int sm_count, int max_vec);

// Largest rows-per-CTA slab the GEMV stages in shared memory for an explicit split.
size_t gemv_smem_bytes(int64_t M, int64_t K, int split_k);

cudaError_t launch_repack(const uint32_t* ckpt, uint32_t* out, int64_t N, int64_t K, cudaStream_t st);

cudaError_t launch_gemv(const __half* a, const uint32_t* b, const __half* s, const uint32_t* z,
                        int64_t M, int64_t N, int64_t K, int32_t G, int32_t zp_bias, __half* out,
                        void* workspace, const GemvPlan& plan, cudaStream_t st);

}  // namespace w4a16
