"""Programmatic dependent launch (W4A16_LAUNCH_PDL) keeps every dependency.

With the flag, a GEMV or a tensor-core GEMM (48 and 200 rows: one and two row-block
launches) may start while the kernel before it is still running and
stream its weights early, but it must read its activations only after that
kernel has finished. A chain of layers where each call's input is the previous
call's output makes the dependency real: the chained outputs with the flag must
equal, bit for bit, the same chain without it (the kernels are deterministic),
both from eager launches and from a captured CUDA graph, and the first layer must
match the oracle within the layer's tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from test_gpu_parity import assert_close, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_int4_08_b200 as mod
    return mod


def _layers(n, K, G, sym, seed):
    out = []
    for i in range(n):
        g = np.random.default_rng(seed + i)
        c = synth.make_case(1, K, K, G, sym=sym, seed=seed + i, s_lo=0.001, s_hi=0.004)
        out.append((dev(c["b"]), dev(c["s"]), dev(c["z"]) if c["z"] is not None else None, c))
    return out


def _chain(w, x0, layers, G, pdl, outs):
    x = x0
    for (b, s, z, c), o in zip(layers, outs):
        w.w4a16_gemm(x, b, s, z, G, c["zp_bias"], out=o, pdl=pdl)
        x = o
    return outs


@pytest.mark.parametrize("M,sym", [(1, True), (4, False), (48, False), (200, True)])
def test_pdl_chain_matches_plain_chain(w, M, sym):
    K, G, n = 2048, 128, 6
    layers = _layers(n, K, G, sym, seed=40 + M)
    assert (w.w4a16_gemm_kernel_choice(M, K, K, G) == w.KERNEL_TC) == (M > 32)
    x0 = dev(synth.fp16_normal(np.random.default_rng(7), (M, K)))
    plain = _chain(w, x0, layers, G, False, [torch.empty((M, K), dtype=torch.float16, device="cuda") for _ in layers])
    fast = _chain(w, x0, layers, G, True, [torch.empty((M, K), dtype=torch.float16, device="cuda") for _ in layers])
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(plain, fast)):
        assert torch.equal(a, b), f"layer {i}"
    c0 = layers[0][3]
    ref = oracle.gemm(x0.cpu().numpy(), c0["b"], c0["s"], c0["z"], G, c0["zp_bias"])
    assert_close(plain[0], ref, "first layer vs oracle")


@pytest.mark.parametrize("M", [1, 48])
def test_pdl_chain_in_a_cuda_graph(w, M):
    K, G, n = 2048, 128, 6
    layers = _layers(n, K, G, True, seed=60)
    if M > 32:
        assert w.w4a16_gemm_kernel_choice(M, K, K, G) == w.KERNEL_TC
    x0 = dev(synth.fp16_normal(np.random.default_rng(8), (M, K)))
    plain = _chain(w, x0, layers, G, False, [torch.empty((M, K), dtype=torch.float16, device="cuda") for _ in layers])
    outs = [torch.empty((M, K), dtype=torch.float16, device="cuda") for _ in layers]
    _chain(w, x0, layers, G, True, outs)  # initialise outside the capture
    torch.cuda.synchronize()
    for o in outs:
        o.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _chain(w, x0, layers, G, True, outs)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(plain, outs)):
        assert torch.equal(a, b), f"layer {i}"
