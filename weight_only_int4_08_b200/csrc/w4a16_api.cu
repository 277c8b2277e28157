// C ABI of the W4A16 library: host-side argument checks, kernel selection and
// launch. Declarations and the full contract are in include/w4a16.h.
#include "common.cuh"

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>

namespace w4a16 {
namespace {

thread_local char g_last_error[256] = "";

void set_error(const char* fmt, const char* detail) {
    snprintf(g_last_error, sizeof(g_last_error), fmt, detail);
}

w4a16_status fail_arg(const char* why) {
    set_error("invalid argument: %s", why);
    return W4A16_ERR_INVALID_ARG;
}

w4a16_status fail_cuda(cudaError_t e) {
    set_error("CUDA error: %s", cudaGetErrorString(e));
    return W4A16_ERR_CUDA;
}

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];   // 0 = not cached yet
std::atomic<int> g_cc_major[kMaxDevices];

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void* p, size_t pn, const void* q, size_t qn) {
    if (!p || !q || pn == 0 || qn == 0) return false;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return a < b + qn && b < a + pn;
}

// Query (once per device) the SM count and compute-capability major.
cudaError_t device_info(int* sm_count, int* cc_major) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    int sms = g_sm_count[dev].load(std::memory_order_relaxed);
    int maj = g_cc_major[dev].load(std::memory_order_relaxed);
    if (sms == 0) {
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&maj, cudaDevAttrComputeCapabilityMajor, dev);
        if (e != cudaSuccess) return e;
        g_cc_major[dev].store(maj, std::memory_order_relaxed);
        g_sm_count[dev].store(sms, std::memory_order_relaxed);
    }
    *sm_count = sms;
    *cc_major = maj;
    return cudaSuccess;
}

constexpr int64_t kMaxDim = (int64_t)1 << 31;

// Shape rules shared by the GEMM entry points; returns nullptr when they hold.
const char* check_gemm_shape(int64_t M, int64_t N, int64_t K, int32_t G) {
    if (M < 1) return "M must be >= 1";
    if (N < 8 || N % 8) return "N must be a positive multiple of 8";
    if (G < 16 || G % 16) return "group_size must be a positive multiple of 16";
    if (K < G || K % G) return "K must be a positive multiple of group_size";
    if (M >= kMaxDim || N >= kMaxDim || K >= kMaxDim) return "dimension too large";
    return nullptr;
}

int max_vec_for(const void* b) {
    return aligned(b, 16) ? 4 : aligned(b, 8) ? 2 : 1;
}

struct Choice {
    int kernel;  // W4A16_KERNEL_GEMV or W4A16_KERNEL_TC
    GemvPlan gemv;
    TcPlan tc;
};

// Kernel table. M <= 16: the mma.sync GEMV (one launch; the CUDA-core GEMV when its
// alignment rules fail). Above 16 rows the GEMV needs a second launch that reads all the weights
// again, while the tensor-core GEMM reads them once: the GEMM, whenever the shape and pointers
// allow it (N % 128, K % 128, 16-byte aligned A and weights), the GEMV's row blocks otherwise.
// Null pointers (workspace query) count as aligned. Measured on B200, G=128, CUDA graphs with
// programmatic dependent launch, weights larger than L2 (GEMV / GEMM, us):
//   K=4096 N=6144:   M=16 11.1 / 12.5, M=17 18.8 / 13.2, M=24 20.7 / 13.4
//   K=4096 N=4096:   M=16  9.2 / 11.3, M=17 14.5 / 11.6, M=24 16.0 / 11.9
//   K=14336 N=4096:  M=16 15.7 / 19.7, M=17 27.6 / 20.8, M=24 29.8 / 20.9
//   K=4096 N=14336:  M=16 14.7 / 17.4, M=17 25.5 / 18.1, M=24 27.5 / 18.0
//   K=4096 N=28672:  M=16 30.9 / 34.8, M=17 61.3 / 36.4, M=32 63.5 / 36.4
constexpr int64_t kGemvOneLaunchM = 16;
bool auto_prefers_tc(int64_t M) { return M > kGemvOneLaunchM; }
Choice choose(int64_t M, int64_t N, int64_t K, int32_t G, const w4a16_gemm_options* opts, int sms,
              const void* a, const void* b, const void* s, const void* z) {
    Choice c{};
    const int req = opts ? opts->kernel : W4A16_KERNEL_AUTO;
    const bool tc_ok = tc_supported(M, N, K, G, a ? a : (const void*)16, b ? b : (const void*)16);
    if (req == W4A16_KERNEL_TC) c.kernel = W4A16_KERNEL_TC;
    else if (req == W4A16_KERNEL_GEMV || req == W4A16_KERNEL_GEMV_FMA) c.kernel = W4A16_KERNEL_GEMV;
    else c.kernel = (auto_prefers_tc(M) && tc_ok) ? W4A16_KERNEL_TC : W4A16_KERNEL_GEMV;
    const int split = opts ? opts->split_k : 0;
    if (c.kernel == W4A16_KERNEL_TC) {
        if (tc_ok) c.tc = plan_tc(M, N, K, G, sms, split);
    } else if (req != W4A16_KERNEL_GEMV_FMA &&
               gemv_mma_supported(N, K, a ? a : (const void*)16, b ? b : (const void*)16, s ? s : (const void*)16, z)) {
        c.gemv = plan_gemv_mma(M, N, K, G, split, sms);
    } else {
        c.gemv = plan_gemv(M, N, K, G, split, sms, b ? max_vec_for(b) : 4, true);
    }
    return c;
}

// Workspace that covers every plan this shape can take, whatever the alignment
// of the pointers turns out to be at launch.
size_t ws_bound(int64_t M, int64_t N, int64_t K, int32_t G, const w4a16_gemm_options* opts, int sms) {
    size_t ws = 0;
    const int req = opts ? opts->kernel : W4A16_KERNEL_AUTO;
    if (req != W4A16_KERNEL_TC) {
        const int split = opts ? opts->split_k : 0;
        for (int v : {4, 2, 1})
            for (bool tma : {true, false}) ws = std::max(ws, plan_gemv(M, N, K, G, split, sms, v, tma).ws_bytes);
        if (req != W4A16_KERNEL_GEMV_FMA && N % 32 == 0) ws = std::max(ws, plan_gemv_mma(M, N, K, G, split, sms).ws_bytes);
    }
    const bool tc_shape = tc_supported(M, N, K, G, (const void*)16, (const void*)16);
    if (tc_shape && (req == W4A16_KERNEL_TC || (req == W4A16_KERNEL_AUTO && auto_prefers_tc(M))))
        ws = std::max(ws, plan_tc(M, N, K, G, sms, opts ? opts->split_k : 0).ws_bytes);
    return ws;
}

}  // namespace

cudaError_t encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, cuuint32_t rank, void* gaddr,
                              const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                              const cuuint32_t* estrides, CUtensorMapSwizzle swizzle) {
    using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static std::atomic<EncodeFn> fn{nullptr};
    EncodeFn f = fn.load(std::memory_order_acquire);
    if (!f) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !p) return cudaErrorNotSupported;
        f = reinterpret_cast<EncodeFn>(p);
        fn.store(f, std::memory_order_release);
    }
    CUresult r = f(map, dtype, rank, gaddr, dims, strides, box, estrides, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

void set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

int device_sm_count(int* err) {
    int sms = 0, maj = 0;
    cudaError_t e = device_info(&sms, &maj);
    if (err) *err = (int)e;
    return sms;
}

}  // namespace w4a16

using namespace w4a16;

extern "C" {

const char* w4a16_status_string(w4a16_status s) {
    switch (s) {
        case W4A16_OK: return "ok";
        case W4A16_ERR_INVALID_ARG: return "invalid argument";
        case W4A16_ERR_UNSUPPORTED: return "unsupported";
        case W4A16_ERR_CUDA: return "CUDA error";
        case W4A16_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

const char* w4a16_last_error(void) { return g_last_error; }

w4a16_status w4a16_repack(const void* ckpt_nk8, void* out_kn8, int64_t N, int64_t K, void* stream) {
    g_last_error[0] = 0;
    if (!ckpt_nk8 || !out_kn8) return fail_arg("NULL pointer");
    if (N < 8 || N % 8) return fail_arg("N must be a positive multiple of 8");
    if (K < 8 || K % 8) return fail_arg("K must be a positive multiple of 8");
    if (N >= kMaxDim || K >= kMaxDim) return fail_arg("dimension too large");
    if (!aligned(ckpt_nk8, 4) || !aligned(out_kn8, 4)) return fail_arg("pointers must be 4-byte aligned");
    const size_t bytes = (size_t)N * (size_t)K / 2;
    if (overlaps(ckpt_nk8, bytes, out_kn8, bytes)) return fail_arg("input and output overlap");
    int sms = 0, maj = 0;
    cudaError_t e = device_info(&sms, &maj);
    if (e != cudaSuccess) return fail_cuda(e);
    if (maj != 10) {
        set_error("unsupported: %s", "this library is built for sm_100 (B200) devices");
        return W4A16_ERR_UNSUPPORTED;
    }
    e = launch_repack(static_cast<const uint32_t*>(ckpt_nk8), static_cast<uint32_t*>(out_kn8), N, K,
                      static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? W4A16_OK : fail_cuda(e);
}

w4a16_status w4a16_load_ct(const void* ckpt_nk8, const void* scale_ng, const void* zero_n8g, int64_t N, int64_t K,
                           int32_t group_size, void* out_kn8, void* scale_gn, void* zero_gn8, void* stream) {
    g_last_error[0] = 0;
    if (!ckpt_nk8 || !scale_ng || !out_kn8 || !scale_gn) return fail_arg("NULL pointer");
    if (zero_n8g && !zero_gn8) return fail_arg("NULL pointer: zero_gn8 is needed when zero_n8g is given");
    if (const char* why = check_gemm_shape(1, N, K, group_size)) return fail_arg(why);
    if (!aligned(ckpt_nk8, 4) || !aligned(out_kn8, 4)) return fail_arg("weight pointers must be 4-byte aligned");
    if (!aligned(scale_ng, 2) || !aligned(scale_gn, 2)) return fail_arg("scale pointers must be 2-byte aligned");
    if (zero_n8g && (!aligned(zero_n8g, 4) || !aligned(zero_gn8, 4)))
        return fail_arg("zero pointers must be 4-byte aligned");
    const int64_t ng = K / group_size;
    const size_t wb = (size_t)N * (size_t)K / 2, sb = (size_t)N * (size_t)ng * 2, zb = (size_t)N * (size_t)ng / 2;
    const void* ins[3] = {ckpt_nk8, scale_ng, zero_n8g};
    const size_t in_n[3] = {wb, sb, zb};
    const void* outs[3] = {out_kn8, scale_gn, zero_n8g ? zero_gn8 : nullptr};
    for (int i = 0; i < 3; ++i) {
        if (!outs[i]) continue;
        for (int j = 0; j < 3; ++j)
            if (ins[j] && overlaps(outs[i], in_n[i], ins[j], in_n[j])) return fail_arg("an output overlaps an input");
        for (int j = i + 1; j < 3; ++j)
            if (outs[j] && overlaps(outs[i], in_n[i], outs[j], in_n[j])) return fail_arg("outputs overlap");
    }
    int sms = 0, maj = 0;
    cudaError_t e = device_info(&sms, &maj);
    if (e != cudaSuccess) return fail_cuda(e);
    if (maj != 10) {
        set_error("unsupported: %s", "this library is built for sm_100 (B200) devices");
        return W4A16_ERR_UNSUPPORTED;
    }
    e = launch_ct_load(static_cast<const uint32_t*>(ckpt_nk8), static_cast<const uint16_t*>(scale_ng),
                       static_cast<const uint32_t*>(zero_n8g), static_cast<uint32_t*>(out_kn8),
                       static_cast<uint16_t*>(scale_gn), zero_n8g ? static_cast<uint32_t*>(zero_gn8) : nullptr, N, K,
                       ng, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? W4A16_OK : fail_cuda(e);
}

size_t w4a16_gemm_ex_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t group_size,
                                     const w4a16_gemm_options* opts) {
    if (check_gemm_shape(M, N, K, group_size)) return 0;
    int sms = 0, maj = 0;
    if (device_info(&sms, &maj) != cudaSuccess) return 0;
    return ws_bound(M, N, K, group_size, opts, sms);
}

w4a16_status w4a16_gemm_kernel_choice(int64_t M, int64_t N, int64_t K, int32_t group_size, const void* a,
                                      const void* b_packed, const void* scales, int32_t* kernel) {
    g_last_error[0] = 0;
    if (!kernel) return fail_arg("NULL pointer");
    if (const char* why = check_gemm_shape(M, N, K, group_size)) return fail_arg(why);
    const void* pa = a ? a : (const void*)16;
    const void* pb = b_packed ? b_packed : (const void*)16;
    const void* ps = scales ? scales : (const void*)16;
    // the same decisions as choose() and the launch path, without the device queries
    if (auto_prefers_tc(M) && tc_supported(M, N, K, group_size, pa, pb))
        *kernel = W4A16_KERNEL_TC;
    else
        *kernel = gemv_mma_supported(N, K, pa, pb, ps, nullptr) ? W4A16_KERNEL_GEMV : W4A16_KERNEL_GEMV_FMA;
    return W4A16_OK;
}

size_t w4a16_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t group_size) {
    return w4a16_gemm_ex_workspace_bytes(M, N, K, group_size, nullptr);
}

w4a16_status w4a16_gemm_ex(const void* a, const void* b_packed, const void* scales, const void* qzeros,
                           int64_t M, int64_t N, int64_t K, int32_t group_size, int32_t zp_bias,
                           void* out, void* workspace, size_t workspace_bytes, void* stream,
                           const w4a16_gemm_options* opts) {
    g_last_error[0] = 0;
    if (!a || !b_packed || !scales || !out) return fail_arg("NULL pointer");
    if (const char* why = check_gemm_shape(M, N, K, group_size)) return fail_arg(why);
    if (!qzeros && (zp_bias < 0 || zp_bias > 15)) return fail_arg("zp_bias must be in 0..15");
    if (opts && (opts->kernel < W4A16_KERNEL_AUTO || opts->kernel > W4A16_KERNEL_GEMV_FMA))
        return fail_arg("unknown kernel option");
    if (opts && (opts->split_k < 0 || opts->split_k > 1024)) return fail_arg("split_k must be in 0..1024");
    if (opts && (opts->debug_flags & ~(uint32_t)W4A16_DEBUG_STALL_LOADS)) return fail_arg("unknown debug flag");
    if (opts && (opts->launch_flags & ~(uint32_t)(W4A16_LAUNCH_PDL | W4A16_OUT_F32)))
        return fail_arg("unknown launch flag");
    const bool out_f32 = opts && (opts->launch_flags & W4A16_OUT_F32);
    if (!aligned(a, 2) || !aligned(scales, 2)) return fail_arg("fp16 pointers must be 2-byte aligned");
    if (!aligned(out, out_f32 ? 4 : 2)) return fail_arg(out_f32 ? "fp32 out must be 4-byte aligned" : "fp16 pointers must be 2-byte aligned");
    if (!aligned(b_packed, 4) || (qzeros && !aligned(qzeros, 4))) return fail_arg("int32 pointers must be 4-byte aligned");
    const size_t a_bytes = (size_t)M * K * 2, b_bytes = (size_t)K * N / 2, s_bytes = (size_t)(K / group_size) * N * 2;
    const size_t z_bytes = qzeros ? (size_t)(K / group_size) * N / 2 : 0, o_bytes = (size_t)M * N * (out_f32 ? 4 : 2);
    if (overlaps(out, o_bytes, a, a_bytes) || overlaps(out, o_bytes, b_packed, b_bytes) ||
        overlaps(out, o_bytes, scales, s_bytes) || overlaps(out, o_bytes, qzeros, z_bytes))
        return fail_arg("out overlaps an input");

    int sms = 0, maj = 0;
    cudaError_t e = device_info(&sms, &maj);
    if (e != cudaSuccess) return fail_cuda(e);
    if (maj != 10) {
        set_error("unsupported: %s", "this library is built for sm_100 (B200) devices");
        return W4A16_ERR_UNSUPPORTED;
    }
    Choice c = choose(M, N, K, group_size, opts, sms, a, b_packed, scales, qzeros);
    if (c.kernel == W4A16_KERNEL_TC && !tc_supported(M, N, K, group_size, a, b_packed)) {
        set_error("unsupported: %s", "tensor-core kernel needs N % 128 == 0, K % 128 == 0, 16-byte aligned a and b_packed");
        return W4A16_ERR_UNSUPPORTED;
    }
    // The documented contract: a workspace of at least what the size query advertises for these
    // arguments (a bound over the kernels the automatic choice may take), whatever this call uses.
    const size_t need = std::max(c.kernel == W4A16_KERNEL_TC ? c.tc.ws_bytes : c.gemv.ws_bytes,
                                 ws_bound(M, N, K, group_size, opts, sms));
    if (need > 0) {
        if (!workspace) return fail_arg("workspace required (see w4a16_gemm_workspace_bytes)");
        if (!aligned(workspace, 256)) return fail_arg("workspace must be 256-byte aligned");
        if (workspace_bytes < need) return fail_arg("workspace too small");
        if (overlaps(workspace, need, out, o_bytes) || overlaps(workspace, need, a, a_bytes) ||
            overlaps(workspace, need, b_packed, b_bytes) || overlaps(workspace, need, scales, s_bytes) ||
            overlaps(workspace, need, qzeros, z_bytes))
            return fail_arg("workspace overlaps an input or the output");
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    WaitPolicy wp;
    wp.limit_ns = (opts && opts->wait_limit_us) ? (uint64_t)opts->wait_limit_us * 1000ull : 2000000000ull;
    wp.stall_loads = (opts && (opts->debug_flags & W4A16_DEBUG_STALL_LOADS)) ? 1 : 0;
    wp.pdl = (opts && (opts->launch_flags & W4A16_LAUNCH_PDL)) ? 1 : 0;
    OutPtr o{out_f32 ? nullptr : static_cast<__half*>(out), out_f32 ? static_cast<float*>(out) : nullptr};
    if (c.kernel == W4A16_KERNEL_TC) {
        e = launch_tc(static_cast<const __half*>(a), static_cast<const uint32_t*>(b_packed),
                      static_cast<const __half*>(scales), static_cast<const uint32_t*>(qzeros), M, N, K, group_size,
                      zp_bias, o, workspace, c.tc, wp, st);
        return e == cudaSuccess ? W4A16_OK : fail_cuda(e);
    }
    if (c.gemv.mma) {
        e = launch_gemv_mma(static_cast<const __half*>(a), static_cast<const uint32_t*>(b_packed),
                            static_cast<const __half*>(scales), static_cast<const uint32_t*>(qzeros), M, N, K,
                            group_size, zp_bias, o, workspace, c.gemv, wp, st);
        return e == cudaSuccess ? W4A16_OK : fail_cuda(e);
    }
    if (gemv_smem_bytes(M, K, c.gemv.split_k) > 160 * 1024) return fail_arg("split_k too small for this K");
    e = launch_gemv(static_cast<const __half*>(a), static_cast<const uint32_t*>(b_packed),
                    static_cast<const __half*>(scales), static_cast<const uint32_t*>(qzeros), M, N, K,
                    group_size, zp_bias, o, workspace, c.gemv, wp, st);
    return e == cudaSuccess ? W4A16_OK : fail_cuda(e);
}

w4a16_status w4a16_gemm(const void* a, const void* b_packed, const void* scales, const void* qzeros,
                        int64_t M, int64_t N, int64_t K, int32_t group_size, int32_t zp_bias,
                        void* out, void* workspace, size_t workspace_bytes, void* stream) {
    return w4a16_gemm_ex(a, b_packed, scales, qzeros, M, N, K, group_size, zp_bias, out, workspace,
                         workspace_bytes, stream, nullptr);
}

w4a16_status w4a16_reduce_partials(const void* const* parts, int32_t P, int64_t M, int64_t N, void* out,
                                   void* stream) {
    g_last_error[0] = 0;
    if (!parts || !out) return fail_arg("NULL pointer");
    if (P < 1 || P > kMaxReduceParts) return fail_arg("P must be in 1..16");
    if (M < 1 || M >= kMaxDim) return fail_arg("M must be in 1..2^31-1");
    if (N < 8 || N % 8 || N >= kMaxDim) return fail_arg("N must be a positive multiple of 8");
    if (!aligned(out, 16)) return fail_arg("out must be 16-byte aligned");
    const size_t pb = (size_t)M * N * 4, ob = (size_t)M * N * 2;
    const float* fp[kMaxReduceParts];
    for (int r = 0; r < P; ++r) {
        if (!parts[r]) return fail_arg("NULL pointer in parts");
        if (!aligned(parts[r], 16)) return fail_arg("parts must be 16-byte aligned");
        if (overlaps(out, ob, parts[r], pb)) return fail_arg("out overlaps a part");
        fp[r] = static_cast<const float*>(parts[r]);
    }
    int sms = 0, maj = 0;
    cudaError_t e = device_info(&sms, &maj);
    if (e != cudaSuccess) return fail_cuda(e);
    if (maj != 10) {
        set_error("unsupported: %s", "this library is built for sm_100 (B200) devices");
        return W4A16_ERR_UNSUPPORTED;
    }
    e = launch_reduce_partials(fp, P, M, N, static_cast<__half*>(out), sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? W4A16_OK : fail_cuda(e);
}

w4a16_status w4a16_workspace_status(void* workspace, int32_t clear, int32_t* status, void* stream) {
    g_last_error[0] = 0;
    if (!workspace || !status) return fail_arg("NULL pointer");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && clear) {
        e = cudaMemsetAsync(workspace, 0, sizeof(int32_t), st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    if (e != cudaSuccess) return fail_cuda(e);
    *status = v;
    return W4A16_OK;
}

}  // extern "C"
