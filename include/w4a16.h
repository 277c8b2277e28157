/*
 * w4a16.h — C ABI of the B200 (sm_100a) weight-only int4 linear layer.
 *
 * The layer (vLLM PR #37352 analysis page, "[vllm] AMD ROCm을 위한 Triton 기반
 * W4A16 커널 도입", section "코드 분석 1. Triton 기반 GEMM 커널 구현 및 검증"):
 *
 *     out[M, N] = fp16( fp32(A[M, K]) @ W[K, N] ),   W[k, n] = (q[k, n] - z[k/G, n]) * s[k/G, n]
 *
 * with q the unsigned int4 weight, s the fp16 group scale, z the int4 zero point
 * (packed per group, or the constant zp_bias for symmetric quantisation) and an
 * fp32 accumulator.
 *
 * Data layouts (all dense, row-major, no padding between rows):
 *   A        fp16  [M, K]
 *   b_packed int32 [K, N/8]    word (k, c), nibble j (bits 4j..4j+3) = q[k, 8c + j]
 *   scales   fp16  [K/G, N]
 *   qzeros   int32 [K/G, N/8]  word (g, c), nibble j = z[g, 8c + j]
 *   out      fp16  [M, N]
 *   ckpt     int32 [N, K/8]    checkpoint layout: word (n, c), nibble j = q[8c + j, n]
 * Nibbles are unsigned (0..15). The nibble order inside a word is not printed on
 * the page; the order above (element 8c + j in nibble j) is the reading taken.
 *
 * Common rules for every entry point:
 *   - Every pointer argument is a DEVICE pointer (CUDA global memory) unless the
 *     comment says otherwise. The caller owns every buffer; the library never
 *     allocates, frees or retains a pointer after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Work is enqueued on it asynchronously; no entry point
 *     synchronises the device or the stream, except w4a16_workspace_status.
 *   - Arguments are checked on the host before any launch. A failed check
 *     returns W4A16_ERR_INVALID_ARG (or W4A16_ERR_UNSUPPORTED) and launches
 *     nothing. A launch failure returns W4A16_ERR_CUDA; the CUDA error text is
 *     then available from w4a16_last_error() on the calling thread.
 *   - The library is thread-safe. Its only global state is a per-device cache
 *     of device attributes (SM count).
 *   - The CUDA path is the only path: there is no CPU fallback.
 */
#ifndef W4A16_H_
#define W4A16_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define W4A16_API __attribute__((visibility("default")))
#else
#define W4A16_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W4A16_OK = 0,
    W4A16_ERR_INVALID_ARG = 1,   /* an argument failed a host-side check; nothing launched */
    W4A16_ERR_UNSUPPORTED = 2,   /* valid arguments this build cannot run (e.g. not an sm_100 device) */
    W4A16_ERR_CUDA = 3,          /* a CUDA call or launch failed; see w4a16_last_error() */
    W4A16_ERR_TIMEOUT = 4        /* a bounded device-side wait gave up (read via w4a16_workspace_status) */
} w4a16_status;

/*
 * w4a16_repack — checkpoint layout [N, K/8] to kernel layout [K, N/8], bit-exact.
 *
 * Cited operation: section "2. 가중치 레이아웃 재포장 (Weight Repacking)" of the
 * PR #37352 analysis page: the compressed-tensors checkpoint weight [N, K//8]
 * becomes the kernel's [K, N//8] after loading.
 *
 *   ckpt_nk8  const int32 [N, K/8], device, 4-byte aligned; read only.
 *   out_kn8   int32 [K, N/8], device, 4-byte aligned; fully overwritten.
 *             Must not overlap ckpt_nk8.
 *   N, K      N >= 8, K >= 8, N % 8 == 0, K % 8 == 0.
 * Errors: INVALID_ARG for a NULL pointer, a size rule broken, misalignment or
 * overlapping buffers; CUDA for a launch failure.
 */
W4A16_API w4a16_status w4a16_repack(const void* ckpt_nk8, void* out_kn8, int64_t N, int64_t K, void* stream);

/*
 * w4a16_load_ct — a whole layer from the checkpoint layout to the kernel layout in
 * one launch, bit-exact: the weight as w4a16_repack does it, the per-group scales
 * [N, K/G] -> [K/G, N] and the packed zeros [N/8, K/G] -> [K/G, N/8].
 *
 * Cited operation: section "2. 가중치 레이아웃 재포장 (Weight Repacking)" of the
 * PR #37352 analysis page: after loading, the layer's weight is [K, N//8] and its
 * scale [K//G, N]. The page gives the checkpoint layout of the weight only; the
 * scale and zero layouts on the checkpoint side are read as one row per output
 * channel (scales) and 8 output channels per int32 (zeros, nibble j of word
 * (c, g) = zero of channel 8c + j in group g, the kernel zeros' packing).
 *
 *   ckpt_nk8     const int32 [N, K/8], device, 4-byte aligned.
 *   scale_ng     const fp16 [N, K/G], device, 2-byte aligned.
 *   zero_n8g     const int32 [N/8, K/G], device, 4-byte aligned; or NULL for a
 *                symmetric layer (then zero_gn8 is not written and may be NULL).
 *   N, K, group_size  the w4a16_gemm shape rules for N, K and G.
 *   out_kn8      int32 [K, N/8], device, 4-byte aligned; fully overwritten.
 *   scale_gn     fp16 [K/G, N], device, 2-byte aligned; fully overwritten.
 *   zero_gn8     int32 [K/G, N/8], device, 4-byte aligned; fully overwritten
 *                when zero_n8g is given.
 *   stream       cudaStream_t as void*.
 * No output may overlap any input or another output.
 * Errors: INVALID_ARG for a NULL pointer, a size rule broken, misalignment or
 * overlapping buffers; UNSUPPORTED off sm_100; CUDA for a launch failure.
 */
W4A16_API w4a16_status w4a16_load_ct(const void* ckpt_nk8, const void* scale_ng, const void* zero_n8g, int64_t N,
                                     int64_t K, int32_t group_size, void* out_kn8, void* scale_gn, void* zero_gn8,
                                     void* stream);

/*
 * w4a16_gemm_kernel_choice — which kernel family w4a16_gemm runs for this shape and these
 * pointers (W4A16_KERNEL_GEMV, W4A16_KERNEL_TC or W4A16_KERNEL_GEMV_FMA, the CUDA-core GEMV).
 * Host only: no CUDA call, no device needed; the pointers are only checked for alignment and
 * may be NULL (a NULL pointer counts as aligned).
 *
 *   M, N, K, group_size  as for w4a16_gemm.
 *   a, b_packed, scales  the pointers w4a16_gemm would get, or NULL.
 *   kernel               out: one of the W4A16_KERNEL_* values above.
 * Errors: INVALID_ARG for a NULL `kernel` or a shape w4a16_gemm would reject.
 */
W4A16_API w4a16_status w4a16_gemm_kernel_choice(int64_t M, int64_t N, int64_t K, int32_t group_size, const void* a,
                                                const void* b_packed, const void* scales, int32_t* kernel);

/*
 * w4a16_gemm_workspace_bytes — bytes of device workspace w4a16_gemm needs for
 * this shape on the current device (0 when the shape needs none). Returns 0 for
 * shapes w4a16_gemm would reject. The value depends on the current device's SM
 * count; query it with the device current on which the GEMM will run.
 */
W4A16_API size_t w4a16_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t group_size);

/*
 * w4a16_gemm — out = fp16(fp32(A) @ ((q - z) * s)).
 *
 * Cited operation: the `_w4a16_reference` excerpt and the
 * `triton_w4a16_gemm(a, b_q, scales, qzeros, group_size, zp_bias)` call in
 * section "코드 분석 1" of the PR #37352 analysis page; the contiguity and
 * N % 8 checks follow section "3. 엄격한 데이터 정렬 및 연속성 보장".
 *
 *   a         const fp16 [M, K], device, 2-byte aligned.
 *   b_packed  const int32 [K, N/8], device, 4-byte aligned.
 *   scales    const fp16 [K/G, N], device, 2-byte aligned.
 *   qzeros    const int32 [K/G, N/8], device, 4-byte aligned; or NULL for the
 *             symmetric form, where every zero point is zp_bias. When qzeros is
 *             given, zp_bias is ignored.
 *   M, N, K   M >= 1, N >= 8, K >= group_size; N % 8 == 0; K % group_size == 0.
 *             M <= 16 runs the GEMV (warp mma.sync, one launch); larger M the
 *             tcgen05 tensor-core GEMM when its shape and alignment rules
 *             hold, otherwise the GEMV once per 16 rows.
 *   group_size G: G >= 16 and G % 16 == 0.
 *   zp_bias   0..15 when qzeros is NULL.
 *   out       fp16 [M, N], device, 2-byte aligned; fully overwritten; must not
 *             overlap any input.
 *   workspace device buffer of at least w4a16_gemm_workspace_bytes(M, N, K, G)
 *             bytes, 256-byte aligned, ZERO-FILLED BEFORE ITS FIRST USE. Every
 *             call leaves it as it found it (its counters are reset by the
 *             kernels), so one zero-fill serves any number of calls. Calls that
 *             share a workspace must be ordered (same stream, or events).
 *             May be NULL when the query returned 0.
 *   stream    cudaStream_t as void*.
 * Accumulation is fp32; the group scale is applied in fp32 after each group's
 * exact (q - z) * a partial sums; the result is rounded to fp16 to nearest even.
 * Repeated calls with the same inputs give bit-identical outputs (fixed
 * reduction order, no floating-point atomics).
 * Errors: INVALID_ARG for a NULL required pointer, a size rule broken, a short
 * or misaligned workspace or misaligned data; UNSUPPORTED when the current
 * device is not sm_100; CUDA for a launch failure.
 */
W4A16_API w4a16_status w4a16_gemm(const void* a, const void* b_packed, const void* scales, const void* qzeros,
                        int64_t M, int64_t N, int64_t K, int32_t group_size, int32_t zp_bias,
                        void* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Kernel selection for tests and measurement.
 *   kernel: W4A16_KERNEL_AUTO uses the same table as w4a16_gemm (GEMV for
 *     M <= 16; tensor cores otherwise
 *     when N % 128 == 0, K % 128 == 0 and a, b_packed are 16-byte aligned); GEMV forces the GEMV family (any M; larger
 *     M runs it once per block of 16 rows of A): its multiply-accumulate uses
 *     warp mma.sync when N % 32 == 0, a and b_packed are 16-byte and scales
 *     8-byte aligned, the CUDA-core fp32 loop (8-row blocks) otherwise;
 *     GEMV_FMA forces the CUDA-core fp32 loop;
 *     TC forces the tensor-core GEMM (any M; UNSUPPORTED when the shape or
 *     alignment rules above fail).
 *   split_k: 0 = automatic, else (1..1024) the number of K slices the kernel
 *     splits its work into: the tensor-core GEMM clamps it to K/128, the
 *     mma.sync GEMV to a thread-block cluster (at most 4 CTAs per column tile).
 *     The tensor-core GEMM's automatic split is one whose CTAs are all
 *     resident at once (none when the layer has as many 128-column tiles as
 *     the GPU has CTA slots); a requested split may take several waves.
 *   debug_flags: 0 in normal use. W4A16_DEBUG_STALL_LOADS makes the kernels'
 *     load issuers issue nothing, so every device-side wait runs out: the call
 *     then leaves W4A16_ERR_TIMEOUT in the workspace status word (read it with
 *     w4a16_workspace_status) and its output undefined. For testing the
 *     timeout path only.
 *   wait_limit_us: 0 = the default limit (2 s) on every device-side wait,
 *     else that many microseconds.
 *   launch_flags: 0, or a bit set of W4A16_LAUNCH_PDL and W4A16_OUT_F32.
 *     With W4A16_LAUNCH_PDL the mma.sync GEMV and the tensor-core GEMM are
 *     launched with programmatic dependent launch: a kernel may start while
 *     the kernel before it on the stream is still running, and streams its
 *     packed weights, scales and zeros right away; it waits for that kernel to
 *     finish (and its writes to be visible) before it reads A or writes out
 *     or the workspace. The caller guarantees that the preceding kernel does
 *     not write b_packed, scales or qzeros (a GEMM after another GEMM or an
 *     activation kernel qualifies; a GEMM right after the w4a16_repack that
 *     produced its weights does not). The CUDA-core GEMV ignores the flag.
 *     W4A16_OUT_F32 (any kernel): `out` is fp32 [M, N], 4-byte aligned, and
 *     receives the fp32 sums unrounded instead of their fp16 rounding. This is
 *     one K-shard's share of a row-parallel (K-split) layer: pass rows
 *     [k0, k1) of b_packed (k0, k1 multiples of G), rows [k0/G, k1/G) of
 *     scales and qzeros, and A's columns [k0, k1) as a contiguous
 *     [M, k1 - k0] array (the layout a column-parallel layer before it leaves
 *     on each rank), with K = k1 - k0; then add the shards' outputs in a
 *     fixed order and round once (w4a16_reduce_partials).
 */
enum { W4A16_KERNEL_AUTO = 0, W4A16_KERNEL_GEMV = 1, W4A16_KERNEL_TC = 2, W4A16_KERNEL_GEMV_FMA = 3 };
enum { W4A16_DEBUG_STALL_LOADS = 1 };
enum { W4A16_LAUNCH_PDL = 1, W4A16_OUT_F32 = 2 };
typedef struct {
    int32_t kernel;
    int32_t split_k;
    uint32_t debug_flags;
    uint32_t wait_limit_us;
    uint32_t launch_flags;
} w4a16_gemm_options;

/* Workspace bytes for w4a16_gemm_ex with these options (NULL opts = automatic). */
W4A16_API size_t w4a16_gemm_ex_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t group_size,
                                     const w4a16_gemm_options* opts);

/* w4a16_gemm with explicit kernel options (NULL opts = w4a16_gemm). Same contract. */
W4A16_API w4a16_status w4a16_gemm_ex(const void* a, const void* b_packed, const void* scales, const void* qzeros,
                           int64_t M, int64_t N, int64_t K, int32_t group_size, int32_t zp_bias,
                           void* out, void* workspace, size_t workspace_bytes, void* stream,
                           const w4a16_gemm_options* opts);

/*
 * w4a16_workspace_status — read the device status word kept at the start of a
 * GEMM workspace into *status (a w4a16_status value; W4A16_OK unless a bounded
 * device-side wait gave up). Synchronises `stream`. The word is sticky: pass
 * clear != 0 to reset it to W4A16_OK after reading.
 * Errors: INVALID_ARG for NULL pointers; CUDA for a failed copy.
 */
W4A16_API w4a16_status w4a16_workspace_status(void* workspace, int32_t clear, int32_t* status, void* stream);

/*
 * w4a16_reduce_partials — out = fp16(parts[0] + parts[1] + ... + parts[P-1]).
 *
 * Cited operation: the tensor-parallel layers of section "Arquitectura del
 * Sistema" of the kerneldigest.dev page on LLM inference with TP, where the
 * decode step ends each parallel layer with an all-reduce. A row-parallel
 * (K-split) layer's shards each produce an fp32 partial of the output
 * (w4a16_gemm_ex with W4A16_OUT_F32); the layer's output is their sum, rounded
 * once. This call is that sum and rounding, after the partials have been
 * brought together (an all-gather), or it rounds an all-reduced sum (P = 1).
 *
 *   parts  host array of P pointers to fp32 [M, N] device arrays, each 16-byte
 *          aligned. An array may be another GPU's memory mapped into this
 *          device's address space (peer access, CUDA IPC); it is read with
 *          plain loads. The caller orders the writes that produced the parts
 *          before this call (same stream, events, or a collective's completion).
 *   P      1..16 (P = 1 only rounds).
 *   M, N   M >= 1, N >= 8, N % 8 == 0.
 *   out    fp16 [M, N] device array, 16-byte aligned; fully overwritten; must
 *          not overlap any part.
 *   stream cudaStream_t as void*.
 * Every element is summed in fp32 in index order (((p0 + p1) + p2) + ...) and
 * rounded to fp16 to nearest even: ranks that reduce the same parts get
 * bit-identical outputs.
 * Errors: INVALID_ARG for a NULL pointer, P, M or N outside its range, a
 * misaligned pointer or an overlap; UNSUPPORTED when the current device is not
 * sm_100; CUDA for a launch failure.
 */
W4A16_API w4a16_status w4a16_reduce_partials(const void* const* parts, int32_t P, int64_t M, int64_t N, void* out,
                                             void* stream);

/*
 * w4a16_gemm_noalloc — w4a16_gemm for callers that cannot allocate device memory.
 *
 * The page has no counterpart: this entry point is an addition of this library.
 * Some callers cannot hand over a workspace: code that must not call cudaMalloc
 * because it can synchronise the whole device in the middle of a latency-
 * critical loop, or code embedded in a program whose device memory belongs to
 * another allocator. This variant runs the GEMV kernel family with its scratch
 * memory (status word, split-K arrival counters and fp32 partials) in a fixed
 * array compiled into the library (w4a16_noalloc_scratch_bytes() bytes, 8 MiB)
 * instead of a workspace. It allocates nothing and calls no allocating routine.
 * Which GEMV runs follows the GEMV rule of w4a16_gemm_ex: the warp mma.sync GEMV
 * (16 rows of A per launch) when N % 32 == 0, a and b_packed are 16-byte and
 * scales 8-byte aligned; otherwise the CUDA-core split-K GEMV (8 rows per
 * launch), whose arrival counters and partials live in the array.
 *
 *   Arguments a .. out and stream: as for w4a16_gemm (no workspace arguments).
 *   Limit: a shape whose GEMV scratch need exceeds the fixed array returns
 *     W4A16_ERR_INVALID_ARG ("needs N bytes of scratch...") and launches nothing.
 *   Every GPU that loads the library holds the array until the process exits.
 *   The first call on a device looks up the array's device address with that
 *     device current (cudaGetSymbolAddress) and caches it; make that first call
 *     before any stream capture.
 *   Each call first clears the part of the array it uses beyond the status
 *     word (split-K counters, partial sums) on `stream` (cudaMemsetAsync), then
 *     launches the kernel on `stream`. The status word is not cleared by calls:
 *     a device-side timeout stays recorded until w4a16_noalloc_status reads and
 *     clears it.
 *   All calls share the one array: calls that overlap on the GPU (different
 *     streams without ordering, or several host threads) race and give wrong
 *     results. Order them on one stream or with events.
 * Errors: as w4a16_gemm; CUDA when the address lookup or the clear fails.
 */
W4A16_API w4a16_status w4a16_gemm_noalloc(const void* a, const void* b_packed, const void* scales,
                                          const void* qzeros, int64_t M, int64_t N, int64_t K, int32_t group_size,
                                          int32_t zp_bias, void* out, void* stream);

/*
 * w4a16_gemm_noalloc with options (NULL opts = w4a16_gemm_noalloc). Same contract.
 * opts->kernel may be W4A16_KERNEL_AUTO or W4A16_KERNEL_GEMV (the GEMV rule above)
 * or W4A16_KERNEL_GEMV_FMA (the CUDA-core split-K GEMV); W4A16_KERNEL_TC returns
 * W4A16_ERR_INVALID_ARG. The other fields as for w4a16_gemm_ex.
 */
W4A16_API w4a16_status w4a16_gemm_noalloc_ex(const void* a, const void* b_packed, const void* scales,
                                             const void* qzeros, int64_t M, int64_t N, int64_t K,
                                             int32_t group_size, int32_t zp_bias, void* out, void* stream,
                                             const w4a16_gemm_options* opts);

/*
 * w4a16_noalloc_status — read the status word of the fixed scratch array of the
 * current device into *status (W4A16_OK, or W4A16_ERR_TIMEOUT when a bounded
 * device-side wait of a no-allocation call gave up; that call's output is then
 * undefined). Synchronises `stream`. Pass clear != 0 to reset the word to
 * W4A16_OK after reading.
 * Errors: INVALID_ARG for a NULL `status`; CUDA for a failed lookup or copy.
 */
W4A16_API w4a16_status w4a16_noalloc_status(int32_t clear, int32_t* status, void* stream);

/* Size in bytes of the fixed scratch array used by w4a16_gemm_noalloc. */
W4A16_API size_t w4a16_noalloc_scratch_bytes(void);

/* Static description of a status code. Never NULL. */
W4A16_API const char* w4a16_status_string(w4a16_status s);

/* Text of the last error on the calling thread ("" when none). Never NULL. */
W4A16_API const char* w4a16_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H_ */
