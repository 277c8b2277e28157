"""w4a16_gemm_noalloc: the GEMM for callers that cannot allocate device memory.

Such callers (code that must not call cudaMalloc in a latency-critical loop, or
code whose device memory belongs to another allocator) get their scratch from a
fixed array inside the library. This checks, through the C ABI, that two calls
in a row match w4a16_gemm on the same inputs within the layer's tolerance
(|x - y| <= 1e-3 + 8e-3 |y|), for a shape that needs split-K scratch and one
with zeros, and that an oversized shape is refused with a clear error.
Collected last on purpose (file name), so a stop-at-first-failure run has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

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


def _noalloc_c_abi(w, a, b, s, z, G, zp, out):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    M, K = a.shape
    N = b.shape[1] * 8
    return w.lib.w4a16_gemm_noalloc(ctypes.c_void_p(a.data_ptr()), ctypes.c_void_p(b.data_ptr()),
                                    ctypes.c_void_p(s.data_ptr()),
                                    ctypes.c_void_p(z.data_ptr()) if z is not None else None,
                                    M, N, K, G, zp, ctypes.c_void_p(out.data_ptr()), stream)


@pytest.mark.parametrize("case", ["decode_m1", "asym_m4"])
def test_noalloc_matches_gemm_twice(w, case):
    c = synth.config2() if case == "decode_m1" else synth.config3(4)
    a, b, s = _dev(c["a"]), _dev(c["b"]), _dev(c["s"])
    z = _dev(c["z"]) if c["z"] is not None else None
    ref = w.w4a16_gemm(a, b, s, z, c["G"], c["zp_bias"]).float()
    for call in range(2):
        out = torch.full((c["M"], c["N"]), float("nan"), dtype=torch.float16, device="cuda")
        rc = _noalloc_c_abi(w, a, b, s, z, c["G"], c["zp_bias"], out)
        assert rc == w.W4A16_OK, w.lib.w4a16_last_error().decode()
        torch.cuda.synchronize()
        got = out.float()
        assert torch.all(torch.abs(got - ref) <= ATOL + RTOL * torch.abs(ref)), f"call {call}"


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
