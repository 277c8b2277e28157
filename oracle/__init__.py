"""CPU oracle for the W4A16 linear layer (ctypes wrapper around w4a16_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()``
and by the cpu_baseline / reference leg of ``bench.py``. The product package
never imports it, and it imports nothing from the product package.

Every function takes and returns numpy arrays:
fp16 tensors travel as ``np.float16`` arrays (their bits are passed to C),
packed int4 tensors as ``np.int32`` or ``np.uint32`` arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4a16_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# -ffp-contract=off: the fp32 sum is product-then-add, as the page's test
# reference computes it; no fused multiply-add may be formed.
CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (plain C, single-threaded)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def load(path: str):
    """Load an oracle shared library from `path` and declare its signatures."""
    L = ctypes.CDLL(path)
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    L.oracle_half_to_float.argtypes = [ctypes.c_uint16]
    L.oracle_half_to_float.restype = ctypes.c_float
    L.oracle_float_to_half_rne.argtypes = [ctypes.c_float]
    L.oracle_float_to_half_rne.restype = ctypes.c_uint16
    for name in ("oracle_unpack_kn8", "oracle_pack_kn8"):
        getattr(L, name).argtypes = [p, i64, i64, p]
        getattr(L, name).restype = None
    for name in ("oracle_unpack_ct", "oracle_pack_ct"):
        getattr(L, name).argtypes = [p, i64, i64, p]
        getattr(L, name).restype = None
    L.oracle_repack.argtypes = [p, i64, i64, p]
    L.oracle_repack.restype = ctypes.c_int
    L.oracle_unrepack.argtypes = [p, i64, i64, p]
    L.oracle_unrepack.restype = ctypes.c_int
    L.oracle_ct_scales.argtypes = [p, i64, i64, p]
    L.oracle_ct_scales.restype = ctypes.c_int
    L.oracle_ct_zeros.argtypes = [p, i64, i64, p]
    L.oracle_ct_zeros.restype = ctypes.c_int
    L.oracle_gemm_cols.argtypes = [p, p, p, p, i64, i64, i64, i32, i32, p, i64, p, p]
    L.oracle_gemm_cols.restype = ctypes.c_int
    L.oracle_gemm.argtypes = [p, p, p, p, i64, i64, i64, i32, i32, p, p]
    L.oracle_gemm.restype = ctypes.c_int
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def _c(x, dtype):
    return np.ascontiguousarray(x).view(dtype) if x is not None else None


def half_to_float(bits: int) -> float:
    return float(lib().oracle_half_to_float(int(bits)))


def float_to_half_bits(x: float) -> int:
    return int(lib().oracle_float_to_half_rne(float(x)))


def unpack_kn8(b: np.ndarray, K: int, N: int) -> np.ndarray:
    b = _c(b, np.uint32)
    q = np.empty((K, N), np.uint8)
    lib().oracle_unpack_kn8(_ptr(b), K, N, _ptr(q))
    return q


def pack_kn8(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    K, N = q.shape
    b = np.empty((K, N // 8), np.uint32)
    lib().oracle_pack_kn8(_ptr(q), K, N, _ptr(b))
    return b


def unpack_ct(ckpt: np.ndarray, N: int, K: int) -> np.ndarray:
    ckpt = _c(ckpt, np.uint32)
    q = np.empty((K, N), np.uint8)
    lib().oracle_unpack_ct(_ptr(ckpt), N, K, _ptr(q))
    return q


def pack_ct(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    K, N = q.shape
    ckpt = np.empty((N, K // 8), np.uint32)
    lib().oracle_pack_ct(_ptr(q), N, K, _ptr(ckpt))
    return ckpt


def repack(ckpt: np.ndarray, N: int, K: int) -> np.ndarray:
    """Checkpoint [N, K/8] -> kernel [K, N/8] (uint32)."""
    ckpt = _c(ckpt, np.uint32)
    assert ckpt.size == N * K // 8
    out = np.empty((K, N // 8), np.uint32)
    rc = lib().oracle_repack(_ptr(ckpt), N, K, _ptr(out))
    if rc:
        raise ValueError(f"oracle_repack failed ({rc})")
    return out


def unrepack(b: np.ndarray, K: int, N: int) -> np.ndarray:
    """Kernel [K, N/8] -> checkpoint [N, K/8] (uint32); inverse of repack."""
    b = _c(b, np.uint32)
    out = np.empty((N, K // 8), np.uint32)
    rc = lib().oracle_unrepack(_ptr(b), K, N, _ptr(out))
    if rc:
        raise ValueError(f"oracle_unrepack failed ({rc})")
    return out


def ct_scales(s_ng: np.ndarray, N: int, ngroups: int) -> np.ndarray:
    """Checkpoint scales [N, K/G] -> kernel scales [K/G, N] (fp16 bits as uint16)."""
    s_ng = _c(s_ng, np.uint16)
    assert s_ng.size == N * ngroups
    out = np.empty((ngroups, N), np.uint16)
    rc = lib().oracle_ct_scales(_ptr(s_ng), N, ngroups, _ptr(out))
    if rc:
        raise ValueError(f"oracle_ct_scales failed ({rc})")
    return out


def ct_zeros(z_n8g: np.ndarray, N: int, ngroups: int) -> np.ndarray:
    """Checkpoint zeros [N/8, K/G] -> kernel zeros [K/G, N/8] (uint32)."""
    z_n8g = _c(z_n8g, np.uint32)
    assert z_n8g.size == (N // 8) * ngroups
    out = np.empty((ngroups, N // 8), np.uint32)
    rc = lib().oracle_ct_zeros(_ptr(z_n8g), N, ngroups, _ptr(out))
    if rc:
        raise ValueError(f"oracle_ct_zeros failed ({rc})")
    return out


def gemm(a, b, s, z, group_size: int, zp_bias: int = 8, cols=None, want_acc: bool = False):
    """out = fp16(fp32 a @ ((q - z) * s)), as the page's test reference computes it.

    a: fp16 [M, K]; b: packed [K, N/8]; s: fp16 [K/G, N]; z: packed [K/G, N/8] or None.
    cols: optional iterable of output columns (the result then has len(cols) columns).
    Returns the fp16 output, and the fp32 accumulator too when want_acc.
    """
    a = np.ascontiguousarray(a, dtype=np.float16)
    M, K = a.shape
    b = _c(b, np.uint32)
    N = b.shape[-1] * 8 if b.ndim == 2 else None
    assert b.shape == (K, N // 8), (b.shape, K, N)
    s = np.ascontiguousarray(s, dtype=np.float16)
    assert s.shape == (K // group_size, N)
    if z is not None:
        z = _c(z, np.uint32)
        assert z.shape == (K // group_size, N // 8)
    if cols is not None:
        cols = np.ascontiguousarray(np.asarray(cols, dtype=np.int64))
        ncols = int(cols.size)
    else:
        ncols = N
    acc = np.empty((M, ncols), np.float32)
    out = np.empty((M, ncols), np.float16)
    rc = lib().oracle_gemm_cols(_ptr(a.view(np.uint16)), _ptr(b), _ptr(s.view(np.uint16)), _ptr(z),
                                M, N, K, int(group_size), int(zp_bias),
                                _ptr(cols), ncols, _ptr(acc), _ptr(out.view(np.uint16)))
    if rc:
        raise ValueError(f"oracle_gemm failed ({rc})")
    return (out, acc) if want_acc else out
