"""w4a16_gemm_noalloc: the GEMM for callers that cannot allocate device memory.

Such callers (code that must not call cudaMalloc in a latency-critical loop,
because it can synchronise the whole device, or code whose device memory
belongs to another allocator) get their scratch from a fixed array inside the
library. Through the C ABI, two calls in a row must match both w4a16_gemm and
the CPU oracle on the same inputs within the layer's tolerance
(|x - y| <= 1e-3 + 8e-3 |y|): on the decode shape and a small-batch asymmetric
shape (the mma.sync GEMV), and on a shape with N % 32 != 0 and 12 rows, which
runs the CUDA-core split-K GEMV in two row-block launches whose arrival
counters and fp32 partials live in the fixed array. A device-side timeout
must be visible through w4a16_noalloc_status, and an oversized shape is
refused with a clear error. Collected last on purpose (file name), so a
stop-at-first-failure run has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-3, 8e-3


@pytest.fixture(scope="module")
def w():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_int4_08_b200 as mod
    return mod


def _dev(x):
    x = np.ascontiguousarray(x)
    return torch.from_numpy(x if x.dtype == np.float16 else x.view(np.int32)).cuda()


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc_c_abi(w, a, b, s, z, G, zp, out, opts=None):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    M, K = a.shape
    N = b.shape[1] * 8
    args = (_ptr(a), _ptr(b), _ptr(s), _ptr(z), M, N, K, G, zp, _ptr(out), stream)
    if opts is None:
        return w.lib.w4a16_gemm_noalloc(*args)
    return w.lib.w4a16_gemm_noalloc_ex(*args, ctypes.byref(opts))


def _status(w, clear):
    v = ctypes.c_int32(-1)
    rc = w.lib.w4a16_noalloc_status(int(clear), ctypes.byref(v),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == w.W4A16_OK, w.lib.w4a16_last_error().decode()
    return int(v.value)


def _within(got, ref):
    return np.all(np.abs(got - ref) <= ATOL + RTOL * np.abs(ref))


CASES = {
    "decode_m1": lambda: synth.config2(),
    "asym_m4": lambda: synth.config3(4),
    # N % 32 != 0: the CUDA-core split-K GEMV, 8 rows per launch, partials in the fixed array
    "splitk_m12_n4104": lambda: synth.make_case(12, 4096, 4104, 128, sym=False, seed=21),
}


@pytest.mark.parametrize("case", list(CASES))
def test_noalloc_matches_gemm_and_oracle_twice(w, case):
    c = CASES[case]()
    M, K, N, G = c["M"], c["K"], c["N"], c["G"]
    if case.startswith("splitk"):
        # this shape really uses split-K scratch: counters and partials
        assert w.w4a16_gemm_kernel_choice(M, N, K, G) == w.KERNEL_GEMV_FMA
        assert w.w4a16_gemm_workspace_bytes(M, N, K, G) > 256
    a, b, s = _dev(c["a"]), _dev(c["b"]), _dev(c["s"])
    z = _dev(c["z"]) if c["z"] is not None else None
    via_gemm = w.w4a16_gemm(a, b, s, z, G, c["zp_bias"]).float().cpu().numpy()
    ref = oracle.gemm(c["a"], c["b"], c["s"], c["z"], G, c["zp_bias"]).astype(np.float32)
    assert _within(via_gemm, ref)
    for call in range(2):
        out = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        rc = _noalloc_c_abi(w, a, b, s, z, G, c["zp_bias"], out)
        assert rc == w.W4A16_OK, w.lib.w4a16_last_error().decode()
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        assert _within(got, via_gemm), f"call {call}: differs from w4a16_gemm"
        assert _within(got, ref), f"call {call}: differs from the oracle"
    assert _status(w, clear=False) == w.W4A16_OK


@pytest.mark.parametrize("kernel", ["GEMV", "GEMV_FMA"])
def test_noalloc_timeout_is_reported(w, kernel):
    """Every device-side wait of the call runs out (its loads are never issued): the
    fixed array's status word must say so until it is read and cleared, and the next
    call must be correct."""
    kid = w.KERNEL_GEMV if kernel == "GEMV" else w.KERNEL_GEMV_FMA
    c = synth.make_case(4, 1024, 1024, 128, sym=False, seed=11)
    a, b, s, z = _dev(c["a"]), _dev(c["b"]), _dev(c["s"]), _dev(c["z"])
    out = torch.empty((4, 1024), dtype=torch.float16, device="cuda")
    stall = w.W4A16Options(kid, 0, w.DEBUG_STALL_LOADS, 20000, 0)
    assert _noalloc_c_abi(w, a, b, s, z, 128, 0, out, stall) == w.W4A16_OK
    torch.cuda.synchronize()
    assert _status(w, clear=True) == w.W4A16_ERR_TIMEOUT
    assert _status(w, clear=False) == w.W4A16_OK
    ref = oracle.gemm(c["a"], c["b"], c["s"], c["z"], 128, 0).astype(np.float32)
    assert _noalloc_c_abi(w, a, b, s, z, 128, 0, out, w.W4A16Options(kid, 0, 0, 0, 0)) == w.W4A16_OK
    torch.cuda.synchronize()
    assert _within(out.float().cpu().numpy(), ref)
    assert _status(w, clear=False) == w.W4A16_OK


def test_noalloc_refuses_shapes_beyond_its_scratch(w):
    limit = int(w.lib.w4a16_noalloc_scratch_bytes())
    assert limit > 0
    # A very long K forces many split-K slabs, whose fp32 partials exceed the
    # fixed array. The buffers below are tiny: the call must be refused before
    # any launch, which the assertion on `need` guarantees first.
    M, K, N, G = 8, 1 << 20, 2048, 128
    need = w.w4a16_gemm_workspace_bytes(M, N, K, G, kernel=w.KERNEL_GEMV)
    assert need > limit
    a = torch.zeros((M, 16), dtype=torch.float16, device="cuda")
    b = torch.zeros((16, 8), dtype=torch.int32, device="cuda")       # never read: refused before launch
    s = torch.zeros((16, 8), dtype=torch.float16, device="cuda")
    out = torch.zeros((M, 8), dtype=torch.float16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = w.lib.w4a16_gemm_noalloc(ctypes.c_void_p(a.data_ptr()), ctypes.c_void_p(b.data_ptr()),
                                  ctypes.c_void_p(s.data_ptr()), None, M, N, K, G, 8,
                                  ctypes.c_void_p(out.data_ptr()), stream)
    assert rc == w.W4A16_ERR_INVALID_ARG
    assert "scratch" in w.lib.w4a16_last_error().decode()
