"""GPU parity for the whole-layer checkpoint load (w4a16_load_ct, through the C ABI):
weight, scales and zeros must match the oracle's conversions bit for bit, on shapes
with ragged weight tiles (N not a multiple of 256, K/8 not a multiple of 32), ragged
scale/zero tiles (K/G not a multiple of 32, more than one column tile of groups),
both the symmetric and the asymmetric layer, the hand-computed worked example and the
batch-32 workload's layer (K=4096, N=14336, G=128) at full size. A GEMM run on the
loaded layer must then match the oracle on the oracle-converted layer.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import read_golden
from test_gpu_parity import ATOL, RTOL, assert_close, dev  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_int4_08_b200 as mod
    return mod


def _bits(t):
    return t.cpu().numpy().view(np.uint16 if t.dtype == torch.float16 else np.uint32)


def check_layer(w, K, N, G, sym, seed):
    c = synth.ct_checkpoint(K, N, G, sym=sym, seed=seed)
    b, s, z = w.w4a16_load_ct(dev(c["ckpt"]), dev(c["s_ng"]), None if sym else dev(c["z_n8g"]), N, K, G)
    torch.cuda.synchronize()
    ng = K // G
    assert np.array_equal(_bits(b), oracle.repack(c["ckpt"], N, K))
    assert np.array_equal(_bits(s), oracle.ct_scales(c["s_ng"].view(np.uint16), N, ng))
    if sym:
        assert z is None
    else:
        assert np.array_equal(_bits(z), oracle.ct_zeros(c["z_n8g"], N, ng))
    return c, (b, s, z)


@pytest.mark.parametrize("K,N,G", [(16, 8, 16), (128, 264, 16), (768, 520, 16), (512, 4104, 128),
                                   (2048, 96, 32), (1024, 2048, 1024), (4096, 1032, 64)])
@pytest.mark.parametrize("sym", [True, False])
def test_load_ct_bit_exact(w, K, N, G, sym):
    check_layer(w, K, N, G, sym, seed=40 + K % 97 + N % 13)


def test_load_ct_batch32_layer_full_size(w):
    check_layer(w, 4096, 14336, 128, False, seed=3)


def test_load_ct_worked_example(w):
    d = read_golden("worked_ct_load.txt")
    N, K, G = int(d["N"][0]), int(d["K"][0]), int(d["G"][0])
    h16 = lambda hs: np.array([int(h, 16) for h in hs], np.uint16)
    words = lambda hs: np.array([int(h, 16) for h in hs], np.uint32)
    s_ng = np.stack([h16(d[f"ct_scale_{n}"]) for n in range(N)])
    z_ct = np.stack([words(d[f"ct_zero_{c}"]) for c in range(N // 8)])
    ck = np.zeros((N, K // 8), np.uint32)
    b, s, z = w.w4a16_load_ct(dev(ck), torch.from_numpy(s_ng.view(np.float16)).cuda(), dev(z_ct), N, K, G)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(s), np.stack([h16(d[f"scale_{g}"]) for g in range(K // G)]))
    assert np.array_equal(_bits(z), np.stack([words(d[f"zero_{g}"]) for g in range(K // G)]))
    assert not _bits(b).any()


def test_load_ct_into_preallocated_outputs_then_gemm(w):
    K, N, G, M = 1024, 1032, 64, 5
    c = synth.ct_checkpoint(K, N, G, sym=False, seed=9)
    outs = (torch.full((K, N // 8), -1, dtype=torch.int32, device="cuda"),
            torch.full((K // G, N), 7.0, dtype=torch.float16, device="cuda"),
            torch.full((K // G, N // 8), -1, dtype=torch.int32, device="cuda"))
    b, s, z = w.w4a16_load_ct(dev(c["ckpt"]), dev(c["s_ng"]), dev(c["z_n8g"]), N, K, G, out=outs)
    assert b is outs[0] and s is outs[1] and z is outs[2]
    a = synth.fp16_normal(synth.rng(9, synth.T_A), (M, K))
    got = w.w4a16_gemm(dev(a), b, s, z, G)
    torch.cuda.synchronize()
    bk = oracle.repack(c["ckpt"], N, K)
    sk = oracle.ct_scales(c["s_ng"].view(np.uint16), N, K // G).view(np.float16)
    zk = oracle.ct_zeros(c["z_n8g"], N, K // G)
    assert_close(got, oracle.gemm(a, bk, sk, zk, G), "GEMM on the loaded layer")


def test_load_ct_on_a_side_stream(w):
    K, N, G = 512, 264, 32
    c = synth.ct_checkpoint(K, N, G, sym=True, seed=11)
    st = torch.cuda.Stream()
    ck, sn = dev(c["ckpt"]), dev(c["s_ng"])
    torch.cuda.synchronize()
    with torch.cuda.stream(st):
        b, s, _ = w.w4a16_load_ct(ck, sn, None, N, K, G, stream=st)
    st.synchronize()
    assert np.array_equal(_bits(b), oracle.repack(c["ckpt"], N, K))
    assert np.array_equal(_bits(s), oracle.ct_scales(c["s_ng"].view(np.uint16), N, K // G))
