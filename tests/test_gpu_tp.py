"""Tensor-parallel shards of the layer on one GPU, through the C ABI, against the CPU oracle.

Column-parallel: each rank's column shard (b_packed[:, c0/8:c1/8], scales[:, c0:c1],
qzeros[:, c0/8:c1/8]) runs through w4a16_gemm like any layer; its output must match the
oracle's columns [c0, c1) of the whole layer within the layer's tolerance
(|x - y| <= 1e-3 + 8e-3 |y|), for the GEMV and the tensor-core GEMM.

Row-parallel: each K-shard runs with W4A16_OUT_F32 and writes fp32 partials, which must
match the oracle's fp32 sums over the same rows of K; w4a16_reduce_partials then adds the
shards' partials in rank order and rounds once. That must equal, bit for bit, the fp32
sum in the same order rounded to fp16 on the host (numpy: IEEE single additions and
round-to-nearest-even), and match the oracle on the whole layer within the tolerance.
The ranks of a real job would bring the partials together with a collective; here one
process holds every rank's shard (the collective logic is tested with gloo on CPU).
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


def _within(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return bool(np.all(np.abs(got - ref) <= ATOL + RTOL * np.abs(ref)))


def _dev(x):
    return None if x is None else torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _np(t):
    return None if t is None else t.cpu().numpy()


# (M, K, N, G, sym, world, unit): GEMV shapes (decode and small batch), a shape whose
# shards have N % 32 != 0 (the CUDA-core GEMV), and tensor-core shapes (M = 32, 64)
COLUMN_CASES = {
    "decode_m1_p2": (1, 4096, 14336, 128, False, 2, 128),
    "small_m4_p4": (4, 2048, 4096, 128, True, 4, 128),
    "ragged_m3_p3": (3, 1024, 1048, 64, False, 3, 8),
    "tc_m32_p2": (32, 1024, 8192, 128, False, 2, 128),
    "tc_m64_p4": (64, 2048, 4096, 128, True, 4, 128),
}


@pytest.mark.parametrize("case", list(COLUMN_CASES))
def test_column_shards_match_the_oracle(w, case):
    from weight_only_int4_08_b200 import tp
    M, K, N, G, sym, world, unit = COLUMN_CASES[case]
    c = synth.make_case(M, K, N, G, sym=sym, seed=101)
    a, b, s, z = _dev(c["a"]), _dev(c["b"]), _dev(c["s"]), _dev(c["z"])
    outs = []
    for r in range(world):
        sh = tp.column_shard(b, s, z, r, world, unit)
        out = tp.column_parallel_linear(a, sh, G, c["zp_bias"])
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        cols = np.arange(sh.hi - sh.lo)
        ref = oracle.gemm(c["a"], _np(sh.b_packed), _np(sh.scales), _np(sh.qzeros), G, c["zp_bias"],
                          cols=cols).astype(np.float32)
        assert _within(got, ref), f"rank {r}"
        outs.append(got)
    # the shards side by side are the whole layer
    full = oracle.gemm(c["a"], c["b"], c["s"], c["z"], G, c["zp_bias"]).astype(np.float32)
    assert _within(np.concatenate(outs, axis=1), full)


# (M, K, N, G, sym, world, kernel): each K-shard through the named kernel family
ROW_CASES = {
    "decode_m1_p2_gemv": (1, 4096, 14336, 128, False, 2, None),
    "decode_m1_p4_gemv": (1, 8192, 4096, 128, True, 4, None),
    "small_m16_p2_gemv": (16, 2048, 2048, 128, False, 2, None),
    "ragged_n_p2_fma": (5, 1024, 1000, 64, False, 2, None),
    "fma_forced_p3": (2, 768, 512, 128, True, 3, "fma"),
    "tc_m32_p2": (32, 2048, 8192, 128, False, 2, "tc"),
    "tc_m128_p2": (128, 1024, 4096, 128, True, 2, "tc"),
}


@pytest.mark.parametrize("case", list(ROW_CASES))
def test_row_shards_partials_and_reduction(w, case):
    from weight_only_int4_08_b200 import tp
    M, K, N, G, sym, world, kern = ROW_CASES[case]
    kernel = {None: None, "fma": w.KERNEL_GEMV_FMA, "tc": w.KERNEL_TC}[kern]
    c = synth.make_case(M, K, N, G, sym=sym, seed=202)
    a, b, s, z = _dev(c["a"]), _dev(c["b"]), _dev(c["s"]), _dev(c["z"])
    parts = []
    for r in range(world):
        sh = tp.row_shard(b, s, z, G, r, world)
        a_r = tp.row_shard_activations(a, sh)
        part = w.w4a16_gemm(a_r, sh.b_packed, sh.scales, sh.qzeros, G, c["zp_bias"], out_f32=True, kernel=kernel)
        assert part.dtype == torch.float32 and tuple(part.shape) == (M, N)
        torch.cuda.synchronize()
        _, ref_acc = oracle.gemm(_np(a_r), _np(sh.b_packed), _np(sh.scales), _np(sh.qzeros), G, c["zp_bias"],
                                 want_acc=True)
        assert _within(part.cpu().numpy(), ref_acc), f"rank {r}: fp32 partial"
        parts.append(part)
    out = tp.round_partials(parts)
    torch.cuda.synchronize()
    host = [p.cpu().numpy() for p in parts]
    expect = host[0].copy()
    for h in host[1:]:
        expect = expect + h
    assert np.array_equal(out.cpu().numpy().view(np.uint16), expect.astype(np.float16).view(np.uint16))
    full = oracle.gemm(c["a"], c["b"], c["s"], c["z"], G, c["zp_bias"]).astype(np.float32)
    assert _within(out.float().cpu().numpy(), full)


def test_row_parallel_linear_single_rank_is_the_layer(w):
    """With no process group (one rank), the row-parallel layer is the whole layer: fp32
    sums written unrounded, then rounded by the reduction kernel with P = 1."""
    from weight_only_int4_08_b200 import tp
    c = synth.config3(8)
    a, b, s, z = _dev(c["a"]), _dev(c["b"]), _dev(c["s"]), _dev(c["z"])
    sh = tp.row_shard(b, s, z, c["G"], 0, 1)
    out = tp.row_parallel_linear(a, sh, c["G"], c["zp_bias"])
    torch.cuda.synchronize()
    ref = oracle.gemm(c["a"], c["b"], c["s"], c["z"], c["G"], c["zp_bias"]).astype(np.float32)
    assert _within(out.float().cpu().numpy(), ref)


@pytest.mark.parametrize("P,M,N", [(1, 1, 8), (2, 3, 24), (4, 7, 4104), (16, 2, 2048), (8, 1, 14336)])
def test_reduce_partials_is_the_ordered_fp32_sum(w, P, M, N):
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([P, M, N])))
    host = [(g.standard_normal((M, N), dtype=np.float32) * np.float32(g.uniform(0.1, 3e3))).astype(np.float32)
            for _ in range(P)]
    parts = [torch.from_numpy(h).cuda() for h in host]
    out = w.w4a16_reduce_partials(parts)
    torch.cuda.synchronize()
    expect = host[0].copy()
    for h in host[1:]:
        expect = expect + h
    assert np.array_equal(out.cpu().numpy().view(np.uint16), expect.astype(np.float16).view(np.uint16))


def test_reduce_partials_rounding_edges(w):
    """Halfway cases round to even, values past the fp16 range become infinities, fp16
    subnormals are kept, signed zeros pass through; a NaN stays a NaN (its payload bits
    are not specified)."""
    v = np.array([1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 65504.0, 65520.0, -65520.0, 1e6,
                  2.0 ** -24, 3 * 2.0 ** -26, -0.0, np.nan, 2.0 ** -25, -(2.0 ** -25)], np.float32)
    host = np.zeros((1, 16), np.float32)
    host[0, :v.size] = v
    out = w.w4a16_reduce_partials([torch.from_numpy(host).cuda()])
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    with np.errstate(over="ignore"):
        expect = host.astype(np.float16)
    nan = np.isnan(expect)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got.view(np.uint16)[~nan], expect.view(np.uint16)[~nan])


def test_reduce_partials_checks_on_host(w):
    x = torch.zeros((2, 16), dtype=torch.float32, device="cuda")
    out = torch.empty((2, 16), dtype=torch.float16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    arr = lambda *ts: (ctypes.c_void_p * len(ts))(*[t if isinstance(t, int) else t.data_ptr() for t in ts])
    call = lambda parts, P, M, N, o: w.lib.w4a16_reduce_partials(parts, P, M, N, ctypes.c_void_p(o), stream)
    assert call(arr(x), 1, 2, 16, out.data_ptr()) == w.W4A16_OK
    assert call(arr(x), 0, 2, 16, out.data_ptr()) == w.W4A16_ERR_INVALID_ARG          # P = 0
    assert call(arr(*([x] * 17)), 17, 2, 16, out.data_ptr()) == w.W4A16_ERR_INVALID_ARG  # P > 16
    assert call(arr(x), 1, 2, 12, out.data_ptr()) == w.W4A16_ERR_INVALID_ARG         # N % 8
    assert call(arr(x), 1, 0, 16, out.data_ptr()) == w.W4A16_ERR_INVALID_ARG         # M = 0
    assert call(arr(x.data_ptr() + 4), 1, 1, 8, out.data_ptr()) == w.W4A16_ERR_INVALID_ARG  # part misaligned
    assert call(arr(x), 1, 1, 8, out.data_ptr() + 2) == w.W4A16_ERR_INVALID_ARG      # out misaligned
    assert call(arr(x), 1, 2, 16, x.data_ptr()) == w.W4A16_ERR_INVALID_ARG           # out overlaps a part
    assert call(arr(0), 1, 2, 16, out.data_ptr()) == w.W4A16_ERR_INVALID_ARG          # NULL part
    assert "invalid argument" in w.lib.w4a16_last_error().decode()
    torch.cuda.synchronize()


def test_fp32_output_is_checked_on_host(w):
    c = synth.make_case(1, 256, 64, 128, sym=True, seed=3)
    a, b, s = _dev(c["a"]), _dev(c["b"]), _dev(c["s"])
    buf = torch.zeros(65, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    opts = w.W4A16Options(0, 0, 0, 0, w.OUT_F32)
    ws = w.alloc_workspace(1, 64, 256, 128)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = w.lib.w4a16_gemm_ex(p(a), p(b), p(s), None, 1, 64, 256, 128, 8, ctypes.c_void_p(buf.data_ptr() + 2), p(ws),
                             ws.numel(), stream, ctypes.byref(opts))
    assert rc == w.W4A16_ERR_INVALID_ARG and "fp32 out" in w.lib.w4a16_last_error().decode()
    bad = w.W4A16Options(0, 0, 0, 0, 4)
    rc = w.lib.w4a16_gemm_ex(p(a), p(b), p(s), None, 1, 64, 256, 128, 8, p(buf), p(ws), ws.numel(), stream,
                             ctypes.byref(bad))
    assert rc == w.W4A16_ERR_INVALID_ARG
    # an fp32 output of M*N*4 bytes that would overlap the activations is refused
    rc = w.lib.w4a16_gemm_ex(p(a), p(b), p(s), None, 1, 64, 256, 128, 8, p(a), p(ws), ws.numel(), stream,
                             ctypes.byref(opts))
    assert rc == w.W4A16_ERR_INVALID_ARG
