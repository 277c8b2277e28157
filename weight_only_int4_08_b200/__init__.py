"""B200 (sm_100a) weight-only int4 linear layer: thin Python binding of libw4a16.so.

The functions here only marshal arguments to the C ABI declared in
include/w4a16.h (same names); every step of the computation runs in the
library's CUDA kernels. PyTorch supplies device memory and the current stream.
There is no CPU fallback: importing this package fails if the library is not
built (``python -m weight_only_int4_08_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libw4a16.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m weight_only_int4_08_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

W4A16_OK, W4A16_ERR_INVALID_ARG, W4A16_ERR_UNSUPPORTED, W4A16_ERR_CUDA, W4A16_ERR_TIMEOUT = range(5)
KERNEL_AUTO, KERNEL_GEMV, KERNEL_TC, KERNEL_GEMV_FMA = 0, 1, 2, 3


class W4A16Options(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("split_k", ctypes.c_int32), ("debug_flags", ctypes.c_uint32),
                ("wait_limit_us", ctypes.c_uint32), ("launch_flags", ctypes.c_uint32)]


DEBUG_STALL_LOADS = 1
LAUNCH_PDL = 1
OUT_F32 = 2
MAX_REDUCE_PARTS = 16


_p, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
lib.w4a16_repack.argtypes = [_p, _p, _i64, _i64, _p]
lib.w4a16_repack.restype = ctypes.c_int
lib.w4a16_load_ct.argtypes = [_p, _p, _p, _i64, _i64, _i32, _p, _p, _p, _p]
lib.w4a16_load_ct.restype = ctypes.c_int
lib.w4a16_gemm_kernel_choice.argtypes = [_i64, _i64, _i64, _i32, _p, _p, _p, ctypes.POINTER(ctypes.c_int32)]
lib.w4a16_gemm_kernel_choice.restype = ctypes.c_int
lib.w4a16_gemm_workspace_bytes.argtypes = [_i64, _i64, _i64, _i32]
lib.w4a16_gemm_workspace_bytes.restype = _sz
lib.w4a16_gemm_ex_workspace_bytes.argtypes = [_i64, _i64, _i64, _i32, ctypes.POINTER(W4A16Options)]
lib.w4a16_gemm_ex_workspace_bytes.restype = _sz
lib.w4a16_gemm.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i32, _i32, _p, _p, _sz, _p]
lib.w4a16_gemm.restype = ctypes.c_int
lib.w4a16_gemm_ex.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i32, _i32, _p, _p, _sz, _p,
                              ctypes.POINTER(W4A16Options)]
lib.w4a16_gemm_ex.restype = ctypes.c_int
lib.w4a16_workspace_status.argtypes = [_p, _i32, ctypes.POINTER(ctypes.c_int32), _p]
lib.w4a16_workspace_status.restype = ctypes.c_int
lib.w4a16_gemm_noalloc.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i32, _i32, _p, _p]
lib.w4a16_gemm_noalloc.restype = ctypes.c_int
lib.w4a16_gemm_noalloc_ex.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i32, _i32, _p, _p,
                                      ctypes.POINTER(W4A16Options)]
lib.w4a16_gemm_noalloc_ex.restype = ctypes.c_int
lib.w4a16_noalloc_status.argtypes = [_i32, ctypes.POINTER(ctypes.c_int32), _p]
lib.w4a16_noalloc_status.restype = ctypes.c_int
lib.w4a16_noalloc_scratch_bytes.argtypes = []
lib.w4a16_noalloc_scratch_bytes.restype = _sz
lib.w4a16_reduce_partials.argtypes = [ctypes.POINTER(ctypes.c_void_p), _i32, _i64, _i64, _p, _p]
lib.w4a16_reduce_partials.restype = ctypes.c_int
lib.w4a16_status_string.argtypes = [ctypes.c_int]
lib.w4a16_status_string.restype = ctypes.c_char_p
lib.w4a16_last_error.argtypes = []
lib.w4a16_last_error.restype = ctypes.c_char_p

EXPORTED = ("w4a16_repack", "w4a16_load_ct", "w4a16_gemm_kernel_choice", "w4a16_gemm_workspace_bytes", "w4a16_gemm", "w4a16_gemm_ex_workspace_bytes",
            "w4a16_gemm_ex", "w4a16_workspace_status", "w4a16_status_string", "w4a16_last_error",
            "w4a16_gemm_noalloc", "w4a16_gemm_noalloc_ex", "w4a16_noalloc_status", "w4a16_noalloc_scratch_bytes",
            "w4a16_reduce_partials")


class W4A16Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.w4a16_last_error().decode() or lib.w4a16_status_string(status).decode()
        super().__init__(f"{where}: {lib.w4a16_status_string(status).decode()} ({msg})")


def _check(rc: int, where: str):
    if rc != W4A16_OK:
        raise W4A16Error(rc, where)


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, name, dtype):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtype:
        raise TypeError(f"{name} must have dtype in {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _opts(kernel, split_k, debug_flags=0, wait_limit_us=0, launch_flags=0):
    if kernel is None and not split_k and not debug_flags and not wait_limit_us and not launch_flags:
        return None
    return ctypes.byref(W4A16Options(int(kernel or KERNEL_AUTO), int(split_k or 0), int(debug_flags),
                                     int(wait_limit_us), int(launch_flags)))


def w4a16_status_string(status: int) -> str:
    return lib.w4a16_status_string(int(status)).decode()


def w4a16_gemm_kernel_choice(M: int, N: int, K: int, group_size: int, a=None, b_packed=None, scales=None) -> int:
    """The kernel family w4a16_gemm runs (KERNEL_GEMV, KERNEL_TC or KERNEL_GEMV_FMA); host only.
    Pointers may be given as tensors, integers or None (None counts as aligned)."""
    def ptr(x):
        if x is None:
            return None
        return ctypes.c_void_p(x.data_ptr() if isinstance(x, torch.Tensor) else int(x))
    k = ctypes.c_int32()
    _check(lib.w4a16_gemm_kernel_choice(M, N, K, group_size, ptr(a), ptr(b_packed), ptr(scales), ctypes.byref(k)),
           "w4a16_gemm_kernel_choice")
    return int(k.value)


def w4a16_gemm_workspace_bytes(M: int, N: int, K: int, group_size: int, kernel=None, split_k: int = 0) -> int:
    o = _opts(kernel, split_k)
    if o is None:
        return int(lib.w4a16_gemm_workspace_bytes(M, N, K, group_size))
    return int(lib.w4a16_gemm_ex_workspace_bytes(M, N, K, group_size, o))


def alloc_workspace(M: int, N: int, K: int, group_size: int, device=None, kernel=None, split_k: int = 0):
    """Zero-filled workspace for w4a16_gemm (reusable by every later call of that shape)."""
    n = w4a16_gemm_workspace_bytes(M, N, K, group_size, kernel, split_k)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def w4a16_repack(ckpt_nk8: torch.Tensor, N: int, K: int, out: torch.Tensor | None = None, stream=None):
    """Checkpoint [N, K/8] int32 -> kernel [K, N/8] int32 (bit-exact), on the GPU."""
    pc = _dev(ckpt_nk8, "ckpt_nk8", (torch.int32, torch.uint32))
    if ckpt_nk8.numel() != N * K // 8:
        raise ValueError("ckpt_nk8 must have N*K/8 elements")
    if out is None:
        out = torch.empty((K, N // 8), dtype=torch.int32, device=ckpt_nk8.device)
    po = _dev(out, "out", (torch.int32, torch.uint32))
    if out.numel() != N * K // 8:
        raise ValueError("out must have N*K/8 elements")
    _check(lib.w4a16_repack(pc, po, N, K, _stream_ptr(stream)), "w4a16_repack")
    return out


def w4a16_load_ct(ckpt_nk8: torch.Tensor, scale_ng: torch.Tensor, zero_n8g: torch.Tensor | None, N: int, K: int,
                  group_size: int, out=None, stream=None):
    """A checkpoint-layout layer -> the kernel layout in one launch (bit-exact).

    ckpt_nk8 int32 [N, K/8], scale_ng fp16 [N, K/G], zero_n8g int32 [N/8, K/G] or None.
    Returns (b_packed [K, N/8], scales [K/G, N], qzeros [K/G, N/8] or None); out, if
    given, is such a tuple of preallocated tensors."""
    G = group_size
    ng = K // G if G > 0 else 0
    pc = _dev(ckpt_nk8, "ckpt_nk8", (torch.int32, torch.uint32))
    ps = _dev(scale_ng, "scale_ng", (torch.float16,))
    pz = None if zero_n8g is None else _dev(zero_n8g, "zero_n8g", (torch.int32, torch.uint32))
    if ckpt_nk8.numel() != N * K // 8 or scale_ng.numel() != N * ng:
        raise ValueError("ckpt_nk8 must have N*K/8 elements and scale_ng N*(K/G)")
    if zero_n8g is not None and zero_n8g.numel() != (N // 8) * ng:
        raise ValueError("zero_n8g must have (N/8)*(K/G) elements")
    dev = ckpt_nk8.device
    if out is None:
        out = (torch.empty((K, N // 8), dtype=torch.int32, device=dev),
               torch.empty((ng, N), dtype=torch.float16, device=dev),
               None if zero_n8g is None else torch.empty((ng, N // 8), dtype=torch.int32, device=dev))
    b, s, z = out
    pb = _dev(b, "out[0]", (torch.int32, torch.uint32))
    pso = _dev(s, "out[1]", (torch.float16,))
    pzo = None if z is None else _dev(z, "out[2]", (torch.int32, torch.uint32))
    if b.numel() != N * K // 8 or s.numel() != N * ng or (z is not None and z.numel() != (N // 8) * ng):
        raise ValueError("out tensors have the wrong sizes")
    _check(lib.w4a16_load_ct(pc, ps, pz, N, K, G, pb, pso, pzo, _stream_ptr(stream)), "w4a16_load_ct")
    return b, s, (z if zero_n8g is not None else None)


def w4a16_gemm(a: torch.Tensor, b_packed: torch.Tensor, scales: torch.Tensor, qzeros: torch.Tensor | None,
               group_size: int, zp_bias: int = 8, out: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None, stream=None, kernel=None, split_k: int = 0,
               debug_flags: int = 0, wait_limit_us: int = 0, pdl: bool = False, out_f32: bool = False):
    """out[M, N] = fp16(fp32(a) @ ((q - z) * s)) on the GPU (see include/w4a16.h).

    pdl=True sets W4A16_LAUNCH_PDL: only when the kernel before this call on the stream does not
    write b_packed, scales or qzeros. out_f32=True sets W4A16_OUT_F32: `out` is fp32 and gets the
    sums unrounded (one K-shard's partial of a row-parallel layer; see w4a16_reduce_partials)."""
    pa = _dev(a, "a", (torch.float16,))
    pb = _dev(b_packed, "b_packed", (torch.int32, torch.uint32))
    ps = _dev(scales, "scales", (torch.float16,))
    pz = _dev(qzeros, "qzeros", (torch.int32, torch.uint32)) if qzeros is not None else None
    if a.dim() != 2 or b_packed.dim() != 2 or scales.dim() != 2:
        raise ValueError("a, b_packed and scales must be 2-D")
    M, K = a.shape
    N = b_packed.shape[1] * 8
    if b_packed.shape[0] != K:
        raise ValueError("b_packed must be [K, N/8]")
    if tuple(scales.shape) != (K // group_size, N):
        raise ValueError("scales must be [K/G, N]")
    if qzeros is not None and tuple(qzeros.shape) != (K // group_size, N // 8):
        raise ValueError("qzeros must be [K/G, N/8]")
    odt = torch.float32 if out_f32 else torch.float16
    if out is None:
        out = torch.empty((M, N), dtype=odt, device=a.device)
    po = _dev(out, "out", (odt,))
    if tuple(out.shape) != (M, N):
        raise ValueError("out must be [M, N]")
    if workspace is None:
        workspace = alloc_workspace(M, N, K, group_size, a.device, kernel, split_k)
    pw = _dev(workspace, "workspace", (torch.uint8,))
    o = _opts(kernel, split_k, debug_flags, wait_limit_us, (LAUNCH_PDL if pdl else 0) | (OUT_F32 if out_f32 else 0))
    args = (pa, pb, ps, pz, M, N, K, group_size, zp_bias, po, pw, workspace.numel(), _stream_ptr(stream))
    rc = lib.w4a16_gemm(*args) if o is None else lib.w4a16_gemm_ex(*args, o)
    _check(rc, "w4a16_gemm")
    return out


def w4a16_reduce_partials(parts, out: torch.Tensor | None = None, stream=None):
    """out[M, N] = fp16(parts[0] + parts[1] + ...), summed in fp32 in list order, on the GPU.

    parts: 1..16 fp32 CUDA tensors of one shape [M, N] (N % 8 == 0), each 16-byte aligned."""
    parts = list(parts)
    if not 1 <= len(parts) <= MAX_REDUCE_PARTS:
        raise ValueError(f"between 1 and {MAX_REDUCE_PARTS} parts are needed, got {len(parts)}")
    ptrs = [_dev(t, f"parts[{i}]", (torch.float32,)).value for i, t in enumerate(parts)]
    shape = tuple(parts[0].shape)
    if len(shape) != 2 or any(tuple(t.shape) != shape for t in parts):
        raise ValueError("parts must be 2-D tensors of one shape")
    M, N = shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=parts[0].device)
    po = _dev(out, "out", (torch.float16,))
    if tuple(out.shape) != (M, N):
        raise ValueError("out must be [M, N]")
    arr = (ctypes.c_void_p * len(ptrs))(*ptrs)
    _check(lib.w4a16_reduce_partials(arr, len(ptrs), M, N, po, _stream_ptr(stream)), "w4a16_reduce_partials")
    return out


def w4a16_gemm_noalloc(a: torch.Tensor, b_packed: torch.Tensor, scales: torch.Tensor, qzeros: torch.Tensor | None,
                       group_size: int, zp_bias: int = 8, out: torch.Tensor | None = None, stream=None):
    """w4a16_gemm without a workspace: scratch comes from the library's fixed array
    (for callers that cannot allocate device memory; see include/w4a16.h)."""
    pa = _dev(a, "a", (torch.float16,))
    pb = _dev(b_packed, "b_packed", (torch.int32, torch.uint32))
    ps = _dev(scales, "scales", (torch.float16,))
    pz = _dev(qzeros, "qzeros", (torch.int32, torch.uint32)) if qzeros is not None else None
    M, K = a.shape
    N = b_packed.shape[1] * 8
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=a.device)
    po = _dev(out, "out", (torch.float16,))
    _check(lib.w4a16_gemm_noalloc(pa, pb, ps, pz, M, N, K, group_size, zp_bias, po, _stream_ptr(stream)),
           "w4a16_gemm_noalloc")
    return out


def w4a16_noalloc_status(clear: bool = False, stream=None) -> int:
    """Status word of the no-allocation GEMM's fixed scratch array (synchronises the stream)."""
    v = ctypes.c_int32(-1)
    _check(lib.w4a16_noalloc_status(int(clear), ctypes.byref(v), _stream_ptr(stream)), "w4a16_noalloc_status")
    return int(v.value)


def w4a16_workspace_status(workspace: torch.Tensor, clear: bool = False, stream=None) -> int:
    """Device status word of a GEMM workspace (synchronises the stream)."""
    v = ctypes.c_int32(-1)
    _check(lib.w4a16_workspace_status(ctypes.c_void_p(workspace.data_ptr()), int(clear), ctypes.byref(v),
                                      _stream_ptr(stream)), "w4a16_workspace_status")
    return int(v.value)
