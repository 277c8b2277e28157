// w4a16_reduce_partials: the closing step of a row-parallel (K-split) layer.
//
// Each shard of such a layer holds rows [k0, k1) of the packed weights and produces the
// fp32 sums of its slice of K (w4a16_gemm_ex with W4A16_OUT_F32). The layer's output is
// the sum of the shards' partials, rounded once to fp16:
//   out[i] = fp16( ((parts[0][i] + parts[1][i]) + parts[2][i]) + ... ),
// added in fp32 in that fixed order, so that every rank reducing the same partials gets
// the same bits whatever collective brought them together.
//
// The work is a pure stream: P * 4 bytes read and 2 bytes written per output element.
// Each thread takes 8 consecutive elements (two 16-byte loads per part, one 16-byte store);
// the grid is a multiple of the SM count, striding over the array. The partials are read
// once, with streaming loads (evict-first), so they do not push the next layer's weights
// out of L2. The part pointers may be peer mappings of other GPUs' memory (peer access or
// CUDA IPC): they are read with plain loads, never with TMA.
#include "common.cuh"

#include <algorithm>

namespace w4a16 {
namespace {

constexpr int kThreads = 256;
constexpr int kBlocksPerSm = 8;

struct ReduceArgs {
    const float4* parts[kMaxReduceParts];
    uint4* out;     // 8 fp16 per uint4
    int64_t n8;     // elements / 8
    int P;
};

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__global__ void __launch_bounds__(kThreads) reduce_partials_kernel(const __grid_constant__ ReduceArgs p) {
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < p.n8; i += stride) {
        float4 lo = __ldcs(p.parts[0] + 2 * i), hi = __ldcs(p.parts[0] + 2 * i + 1);
        for (int r = 1; r < p.P; ++r) {
            const float4 x = __ldcs(p.parts[r] + 2 * i), y = __ldcs(p.parts[r] + 2 * i + 1);
            lo.x += x.x; lo.y += x.y; lo.z += x.z; lo.w += x.w;
            hi.x += y.x; hi.y += y.y; hi.z += y.z; hi.w += y.w;
        }
        p.out[i] = make_uint4(pack_half2(lo.x, lo.y), pack_half2(lo.z, lo.w), pack_half2(hi.x, hi.y),
                              pack_half2(hi.z, hi.w));
    }
}

}  // namespace

cudaError_t launch_reduce_partials(const float* const* parts, int P, int64_t M, int64_t N, __half* out, int sm_count,
                                   cudaStream_t st) {
    ReduceArgs a{};
    for (int r = 0; r < P; ++r) a.parts[r] = reinterpret_cast<const float4*>(parts[r]);
    a.out = reinterpret_cast<uint4*>(out);
    a.n8 = M * N / 8;
    a.P = P;
    const int64_t need = (a.n8 + kThreads - 1) / kThreads;
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(need, (int64_t)sm_count * kBlocksPerSm));
    reduce_partials_kernel<<<blocks, kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace w4a16
