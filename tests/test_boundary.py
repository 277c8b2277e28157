"""C-ABI boundary checks that need no GPU: the library loads, exports every symbol
include/w4a16.h declares, and rejects bad arguments on the host with a status
code before any CUDA call (nothing is launched)."""
import ctypes
import os
import re

import pytest

import weight_only_int4_08_b200 as w

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"W4A16_API\s+[\w\s\*]+?\b(w4a16_\w+)\s*\(", text))
    return names


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ("w4a16_repack", "w4a16_load_ct", "w4a16_gemm", "w4a16_gemm_workspace_bytes", "w4a16_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert names
    for n in names:
        assert hasattr(w.lib, n), n
    assert set(w.EXPORTED) == names


def test_status_strings():
    for code, text in [(0, "ok"), (1, "invalid argument"), (2, "unsupported"), (3, "CUDA error"),
                       (4, "device wait timed out"), (99, "unknown status")]:
        assert w.w4a16_status_string(code) == text


P = ctypes.c_void_p
GOOD = P(0x10000)        # well-aligned dummy addresses: never dereferenced on failure
GOOD2 = P(0x20000000)
GOOD3 = P(0x40000000)
OUT = P(0x60000000)


def gemm(a=GOOD, b=GOOD2, s=GOOD3, z=None, M=1, N=64, K=256, G=128, zp=8, out=OUT, ws=None, wsb=0):
    return w.lib.w4a16_gemm(a, b, s, z, M, N, K, G, zp, out, ws, wsb, None)


@pytest.mark.parametrize("kw,why", [
    (dict(a=None), "NULL pointer"),
    (dict(b=None), "NULL pointer"),
    (dict(s=None), "NULL pointer"),
    (dict(out=None), "NULL pointer"),
    (dict(M=0), "M must be"),
    (dict(M=-3), "M must be"),
    (dict(N=60), "N must be"),
    (dict(N=0), "N must be"),
    (dict(K=200), "K must be"),
    (dict(K=64), "K must be"),
    (dict(G=100), "group_size"),
    (dict(G=8, K=64), "group_size"),
    (dict(G=0), "group_size"),
    (dict(zp=16), "zp_bias"),
    (dict(zp=-1), "zp_bias"),
    (dict(a=P(0x10001)), "aligned"),
    (dict(b=P(0x20000002)), "aligned"),
    (dict(z=P(0x30000001)), "aligned"),
    (dict(out=P(0x10000)), "overlaps"),
    (dict(M=1 << 31), "too large"),
])
def test_gemm_rejects_bad_arguments_on_host(kw, why):
    rc = gemm(**kw)
    assert rc == w.W4A16_ERR_INVALID_ARG
    assert why in w.lib.w4a16_last_error().decode()


def test_zp_bias_not_checked_when_zeros_given():
    # with qzeros the zp_bias is ignored; the call then fails later (no GPU here), not on zp_bias
    gemm(z=P(0x30000000), zp=99)
    assert "zp_bias" not in w.lib.w4a16_last_error().decode()


@pytest.mark.parametrize("kw,why", [
    (dict(c=None), "NULL"), (dict(o=None), "NULL"),
    (dict(N=12), "N must be"), (dict(K=4), "K must be"), (dict(N=0), "N must be"),
    (dict(c=P(0x1002)), "aligned"), (dict(o=P(0x1000), c=P(0x1000)), "overlap"),
])
def test_repack_rejects_bad_arguments_on_host(kw, why):
    c = kw.get("c", P(0x1000))
    o = kw.get("o", P(0x80000000))
    rc = w.lib.w4a16_repack(c, o, kw.get("N", 64), kw.get("K", 64), None)
    assert rc == w.W4A16_ERR_INVALID_ARG
    assert why in w.lib.w4a16_last_error().decode()


def load_ct(c=P(0x1000), s=P(0x2000000), z=None, N=64, K=256, G=128, o=P(0x80000000), so=P(0x90000000),
            zo=None):
    return w.lib.w4a16_load_ct(c, s, z, N, K, G, o, so, zo, None)


@pytest.mark.parametrize("kw,why", [
    (dict(c=None), "NULL"), (dict(s=None), "NULL"), (dict(o=None), "NULL"), (dict(so=None), "NULL"),
    (dict(z=P(0x3000000)), "zero_gn8"),
    (dict(N=60), "N must be"), (dict(K=200), "K must be"), (dict(G=8, K=64), "group_size"),
    (dict(c=P(0x1002)), "aligned"), (dict(s=P(0x2000001)), "aligned"), (dict(so=P(0x90000001)), "aligned"),
    (dict(z=P(0x3000002), zo=P(0xA0000000)), "aligned"),
    (dict(o=P(0x1000)), "overlaps an input"),            # weight out on the checkpoint weight
    (dict(so=P(0x1000 + 64 * 256 // 2 - 2)), "overlaps an input"),   # scale out on the weight's last bytes
    (dict(z=P(0x3000000), zo=P(0x90000000)), "outputs overlap"),     # zero out on the scale out
])
def test_load_ct_rejects_bad_arguments_on_host(kw, why):
    rc = load_ct(**kw)
    assert rc == w.W4A16_ERR_INVALID_ARG
    assert why in w.lib.w4a16_last_error().decode()


def test_options_are_checked():
    o = w.W4A16Options(7, 0)
    rc = w.lib.w4a16_gemm_ex(GOOD, GOOD2, GOOD3, None, 1, 64, 256, 128, 8, OUT, None, 0, None, ctypes.byref(o))
    assert rc == w.W4A16_ERR_INVALID_ARG
    o = w.W4A16Options(1, 1025)
    rc = w.lib.w4a16_gemm_ex(GOOD, GOOD2, GOOD3, None, 1, 64, 256, 128, 8, OUT, None, 0, None, ctypes.byref(o))
    assert rc == w.W4A16_ERR_INVALID_ARG
    o = w.W4A16Options(0, 0, 0, 0, 4)   # an undefined launch flag
    rc = w.lib.w4a16_gemm_ex(GOOD, GOOD2, GOOD3, None, 1, 64, 256, 128, 8, OUT, None, 0, None, ctypes.byref(o))
    assert rc == w.W4A16_ERR_INVALID_ARG
    assert "launch flag" in w.lib.w4a16_last_error().decode()
    o = w.W4A16Options(0, 0, 4, 0, 0)   # an undefined debug flag
    rc = w.lib.w4a16_gemm_ex(GOOD, GOOD2, GOOD3, None, 1, 64, 256, 128, 8, OUT, None, 0, None, ctypes.byref(o))
    assert rc == w.W4A16_ERR_INVALID_ARG


def test_options_struct_matches_the_header():
    # field names and order of w4a16_gemm_options as include/w4a16.h declares them
    hdr = open(os.path.join(ROOT, "include", "w4a16.h")).read()
    body = re.search(r"typedef struct \{(.*?)\} w4a16_gemm_options;", hdr, re.S).group(1)
    fields = re.findall(r"(?:int32_t|uint32_t)\s+(\w+);", body)
    assert fields == [f for f, _ in w.W4A16Options._fields_]
    assert ctypes.sizeof(w.W4A16Options) == 4 * len(fields)


def test_workspace_query_rejects_bad_shapes():
    assert w.lib.w4a16_gemm_workspace_bytes(1, 60, 256, 128) == 0
    assert w.lib.w4a16_gemm_workspace_bytes(0, 64, 256, 128) == 0


def test_workspace_status_null_checks():
    v = ctypes.c_int32()
    assert w.lib.w4a16_workspace_status(None, 0, ctypes.byref(v), None) == w.W4A16_ERR_INVALID_ARG


def test_python_binding_requires_cuda_tensors():
    import torch
    a = torch.zeros(1, 256, dtype=torch.float16)
    with pytest.raises(TypeError):
        w.w4a16_gemm(a, torch.zeros(256, 8, dtype=torch.int32), torch.zeros(2, 64, dtype=torch.float16), None, 128)


KERNELS = {"GEMV": 1, "TC": 2, "GEMV_FMA": 3}


@pytest.mark.parametrize("M,N,K,G,ptrs,expect", [
    (1, 14336, 4096, 128, {}, "GEMV"),
    (16, 14336, 4096, 128, {}, "GEMV"),          # one GEMV launch
    (17, 14336, 4096, 128, {}, "TC"),            # above 16 rows: the GEMM whenever it can
    (32, 14336, 4096, 128, {}, "TC"),
    (16, 6144, 4096, 128, {}, "GEMV"),           # one GEMV launch
    (17, 6144, 4096, 128, {}, "TC"),
    (17, 4096, 4096, 128, {}, "TC"),
    (24, 4096, 14336, 128, {}, "TC"),
    (17, 4096, 8064, 128, {}, "TC"),             # 8064 = 63 x 128
    (16, 4096, 14336, 128, {}, "GEMV"),
    (33, 4096, 4096, 128, {}, "TC"),
    (64, 4096, 4160, 64, {}, "GEMV"),            # K % 128 != 0
    (64, 4128, 4096, 128, {}, "GEMV"),           # N % 128 != 0, N % 32 == 0
    (64, 4104, 4096, 128, {}, "GEMV_FMA"),       # N % 32 != 0
    (1, 14336, 4096, 128, {"a": 0x10008}, "GEMV_FMA"),        # activations only 8-byte aligned
    (64, 14336, 4096, 128, {"b": 0x20008}, "GEMV_FMA"),       # weights only 8-byte aligned
    (64, 14336, 4096, 128, {"a": 0x10008}, "GEMV_FMA"),
    (1, 14336, 4096, 128, {"s": 0x30004}, "GEMV_FMA"),        # scales only 4-byte aligned
    (64, 14336, 4096, 128, {"s": 0x30004}, "TC"),             # the GEMM reads scales per element
])
def test_kernel_choice_table(M, N, K, G, ptrs, expect):
    k = w.w4a16_gemm_kernel_choice(M, N, K, G, ptrs.get("a"), ptrs.get("b"), ptrs.get("s"))
    assert k == KERNELS[expect]


def test_kernel_choice_agrees_with_the_bench():
    import bench
    for M in (1, 8, 16, 17, 24, 25, 32, 33, 64, 128):
        for N in (4096, 6144, 12160, 12288, 14336, 28672):
            for K in (4096, 8064, 8192, 14336):
                k = w.w4a16_gemm_kernel_choice(M, N, K, 128)
                assert (k == KERNELS["TC"]) == bench.uses_tc(M, N, K), (M, N, K)


def test_kernel_choice_rejects_bad_arguments():
    v = ctypes.c_int32()
    assert w.lib.w4a16_gemm_kernel_choice(1, 64, 256, 128, None, None, None, None) == w.W4A16_ERR_INVALID_ARG
    assert w.lib.w4a16_gemm_kernel_choice(1, 60, 256, 128, None, None, None, ctypes.byref(v)) == w.W4A16_ERR_INVALID_ARG
    assert "N must be" in w.lib.w4a16_last_error().decode()


def test_noalloc_checks_on_host():
    """The no-allocation GEMM refuses bad arguments and the tensor-core kernel before any CUDA
    call (its scratch bound covers the GEMV family only); its status query needs a pointer."""
    v = ctypes.c_int32()
    assert w.lib.w4a16_noalloc_status(0, None, None) == w.W4A16_ERR_INVALID_ARG
    args = (GOOD, GOOD2, GOOD3, None, 1, 64, 256, 128, 8, OUT, None)
    assert w.lib.w4a16_gemm_noalloc(None, *args[1:]) == w.W4A16_ERR_INVALID_ARG
    assert w.lib.w4a16_gemm_noalloc(*args[:8], 16, *args[9:]) == w.W4A16_ERR_INVALID_ARG   # zp_bias > 15
    tc = w.W4A16Options(w.KERNEL_TC, 0, 0, 0, 0)
    assert w.lib.w4a16_gemm_noalloc_ex(*args, ctypes.byref(tc)) == w.W4A16_ERR_INVALID_ARG
    assert "GEMV kernels only" in w.lib.w4a16_last_error().decode()
    assert int(w.lib.w4a16_noalloc_scratch_bytes()) == 8 << 20
    del v


def test_fp32_output_alignment_is_checked():
    # W4A16_OUT_F32: the fp32 output needs 4-byte alignment (checked before any device query)
    o = w.W4A16Options(0, 0, 0, 0, w.OUT_F32)
    rc = w.lib.w4a16_gemm_ex(GOOD, GOOD2, GOOD3, None, 1, 64, 256, 128, 8, ctypes.c_void_p(OUT.value + 2), None, 0,
                             None, ctypes.byref(o))
    assert rc == w.W4A16_ERR_INVALID_ARG
    assert "fp32 out" in w.lib.w4a16_last_error().decode()


@pytest.mark.parametrize("P,M,N,part_off,out_off,why", [
    (0, 1, 8, 0, 0, "P must be"), (17, 1, 8, 0, 0, "P must be"), (1, 0, 8, 0, 0, "M must be"),
    (1, 1, 12, 0, 0, "N must be"), (1, 1, 8, 4, 0, "parts must be 16-byte aligned"),
    (1, 1, 8, 0, 8, "out must be 16-byte aligned"), (1, 1, 8, None, 0, "NULL pointer in parts"),
])
def test_reduce_partials_checks_on_host(P, M, N, part_off, out_off, why):
    base = 1 << 20
    ptrs = [None if part_off is None else base + 4096 * i + part_off for i in range(max(P, 1))]
    arr = (ctypes.c_void_p * len(ptrs))(*ptrs)
    rc = w.lib.w4a16_reduce_partials(arr, P, M, N, ctypes.c_void_p(base + (1 << 16) + out_off), None)
    assert rc == w.W4A16_ERR_INVALID_ARG
    assert why in w.lib.w4a16_last_error().decode()


def test_reduce_partials_rejects_overlap():
    base = 1 << 20
    arr = (ctypes.c_void_p * 2)(base, base + 4096)
    rc = w.lib.w4a16_reduce_partials(arr, 2, 4, 64, ctypes.c_void_p(base + 4096 + 512), None)
    assert rc == w.W4A16_ERR_INVALID_ARG and "overlaps" in w.lib.w4a16_last_error().decode()
