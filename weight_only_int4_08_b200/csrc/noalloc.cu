// w4a16_gemm_noalloc: the GEMV kernel family with its scratch memory (status
// word, split-K arrival counters and fp32 partials) taken from a fixed array
// inside this library instead of a caller-provided workspace. Which GEMV runs
// follows the library's GEMV rule: the mma.sync GEMV when N % 32 == 0 and the
// pointers are aligned, the CUDA-core split-K GEMV otherwise (or when forced).
//
// It serves callers that cannot allocate device memory for a workspace: code
// that must not call cudaMalloc because that call can synchronise the whole
// device in the middle of a latency-critical loop, and code embedded in a host
// program whose device memory is owned by someone else's allocator, so it
// has no buffer of its own to hand over.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds it (kScratchBytes) until the process exits. Host code cannot
// pass the array's name to a kernel (on the host it only stands for the
// symbol), so its device address is looked up once per device with
// cudaGetSymbolAddress and cached.
#include "common.cuh"

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <mutex>

namespace w4a16 {
namespace {

constexpr size_t kScratchBytes = 8u << 20;  // 8 MiB
constexpr int kMaxDev = 64;

__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::atomic<void*> g_scratch_ptr[kMaxDev];
std::mutex g_scratch_mu;

// Device address of g_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        p = g_scratch_ptr[dev].load(std::memory_order_acquire);
        if (!p) {
            e = cudaGetSymbolAddress(&p, g_scratch);
            if (e != cudaSuccess) return e;
            g_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return cudaSuccess;
}

w4a16_status fail(w4a16_status st, const char* msg) {
    set_last_error(msg);
    return st;
}

w4a16_status gemm_noalloc(const void* a, const void* b_packed, const void* scales, const void* qzeros, int64_t M,
                          int64_t N, int64_t K, int32_t group_size, int32_t zp_bias, void* out, void* stream,
                          const w4a16_gemm_options* user_opts) {
    w4a16_gemm_options opts{};
    if (user_opts) opts = *user_opts;
    // The GEMV family only: its scratch need is bounded by the fixed array for decode shapes.
    if (opts.kernel == W4A16_KERNEL_AUTO) opts.kernel = W4A16_KERNEL_GEMV;
    if (opts.kernel != W4A16_KERNEL_GEMV && opts.kernel != W4A16_KERNEL_GEMV_FMA)
        return fail(W4A16_ERR_INVALID_ARG, "invalid argument: the no-allocation GEMM runs the GEMV kernels only");
    // A rejected shape needs no scratch (the query returns 0) and is reported
    // by w4a16_gemm_ex below; pointer checks come before the scratch is touched.
    const uintptr_t ua = reinterpret_cast<uintptr_t>(a), ub = reinterpret_cast<uintptr_t>(b_packed);
    const uintptr_t us = reinterpret_cast<uintptr_t>(scales), uz = reinterpret_cast<uintptr_t>(qzeros);
    const uintptr_t uo = reinterpret_cast<uintptr_t>(out);
    if (!a || !b_packed || !scales || !out || (ua | us | uo) % 2 || ub % 4 || uz % 4 ||
        (!qzeros && (zp_bias < 0 || zp_bias > 15)))
        return fail(W4A16_ERR_INVALID_ARG,
                    "invalid argument: NULL or misaligned pointer, or zp_bias outside 0..15");
    const size_t need = w4a16_gemm_ex_workspace_bytes(M, N, K, group_size, &opts);
    if (need > kScratchBytes) {
        char msg[200];
        snprintf(msg, sizeof(msg), "invalid argument: this shape needs %zu bytes of scratch; the fixed array holds %zu",
                 need, kScratchBytes);
        return fail(W4A16_ERR_INVALID_ARG, msg);
    }
    void* scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) return fail(W4A16_ERR_CUDA, cudaGetErrorString(e));
    // The array keeps the previous call's contents. The split-K arrival counters
    // and the tagged partial words must start at zero: clear the part of the
    // array this call uses before every call (a successful call leaves it clean,
    // a call that timed out may not). The status word is left alone, so that a
    // timeout stays visible to w4a16_noalloc_status until it is read and cleared.
    if (need > kWsHeader) {
        e = cudaMemsetAsync(static_cast<char*>(scratch) + kWsHeader, 0, need - kWsHeader,
                            static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return fail(W4A16_ERR_CUDA, cudaGetErrorString(e));
    }
    return w4a16_gemm_ex(a, b_packed, scales, qzeros, M, N, K, group_size, zp_bias, out, scratch, kScratchBytes,
                         stream, &opts);
}

}  // namespace
}  // namespace w4a16

using namespace w4a16;

extern "C" {

w4a16_status w4a16_gemm_noalloc(const void* a, const void* b_packed, const void* scales, const void* qzeros,
                                int64_t M, int64_t N, int64_t K, int32_t group_size, int32_t zp_bias, void* out,
                                void* stream) {
    return gemm_noalloc(a, b_packed, scales, qzeros, M, N, K, group_size, zp_bias, out, stream, nullptr);
}

w4a16_status w4a16_gemm_noalloc_ex(const void* a, const void* b_packed, const void* scales, const void* qzeros,
                                   int64_t M, int64_t N, int64_t K, int32_t group_size, int32_t zp_bias, void* out,
                                   void* stream, const w4a16_gemm_options* opts) {
    return gemm_noalloc(a, b_packed, scales, qzeros, M, N, K, group_size, zp_bias, out, stream, opts);
}

w4a16_status w4a16_noalloc_status(int32_t clear, int32_t* status, void* stream) {
    if (!status) return fail(W4A16_ERR_INVALID_ARG, "invalid argument: NULL pointer");
    void* scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) return fail(W4A16_ERR_CUDA, cudaGetErrorString(e));
    return w4a16_workspace_status(scratch, clear, status, stream);
}

size_t w4a16_noalloc_scratch_bytes(void) { return kScratchBytes; }

}  // extern "C"
