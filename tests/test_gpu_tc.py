"""GPU parity of the tensor-core (tcgen05/TMEM) GEMM and the device-side timeout path.

The tensor-core kernel must satisfy |gpu - oracle| <= 1e-3 + 8e-3 |oracle| on the
batch workloads (M = 16 of the small-batch sweep, M = 32 with repack) and on
shapes that exercise every row-block size, group size and split. The timeout
tests make every device-side wait run out on purpose (the load issuers issue
nothing) and check that the status word reports it and the context stays usable.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from test_gpu_parity import assert_close, dev, ref, run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_int4_08_b200 as mod
    return mod


def test_config3_m16_auto_and_tensor_cores(w):
    c = synth.config3(16)
    assert_close(run(w, c), ref(c), "config3 M=16")
    assert_close(run(w, c, kernel=w.KERNEL_TC), ref(c), "config3 M=16 forced")


def test_config4_m32_tensor_cores(w):
    c = synth.config4()
    b_dev = w.w4a16_repack(dev(c["ckpt"]), c["N"], c["K"])
    c["b"] = oracle.repack(c["ckpt"], c["N"], c["K"])
    assert_close(run(w, c, b=b_dev, kernel=w.KERNEL_TC), ref(c), "config4 TC")


@pytest.mark.parametrize("M", [1, 5, 9, 17, 31, 33, 40, 48, 64, 72, 100, 112, 128, 129, 200])
def test_tc_row_blocks(w, M):
    c = synth.make_case(M, 512, 384, 128, sym=(M % 2 == 0), seed=100 + M)
    assert_close(run(w, c, kernel=w.KERNEL_TC), ref(c), f"TC M={M}")


@pytest.mark.parametrize("M", [64, 128, 256])
def test_tc_batch_layer_large_batches(w, M):
    """The batch-32 layer's shape (K=4096, N=14336, G=128, asymmetric) at 64, 128 and 256 rows,
    as the bench times it: every row against the oracle on sampled columns (one in each
    128-column tile, plus the first and the last column), which it computes one by one."""
    K, N = 4096, 14336
    c = synth.make_case(M, K, N, 128, sym=False, seed=3)
    g = np.random.default_rng(M)
    cols = np.unique(np.concatenate([np.arange(0, N, 128) + g.integers(0, 128, N // 128), [0, N - 1]]))
    out = run(w, c, kernel=w.KERNEL_TC).cpu().numpy()
    assert_close(out[:, cols], ref(c, cols=cols), f"TC M={M}")


def test_tc_batch_layer_256_rows_weights_from_dram(w):
    """256 rows of the batch layer with the weights, scales and zeros starting in DRAM: a fill of
    256 MB (twice the L2) after the operands are on the device evicts them, then one call runs its
    two 128-row launches back to back. Every row is checked against the oracle on sampled columns.
    Under ncu with --cache-control none this is the case that shows how many bytes a call reads
    from DRAM (the second launch finds the layer in L2)."""
    M, K, N = 256, 4096, 14336
    c = synth.make_case(M, K, N, 128, sym=False, seed=4)
    a, b, s, z = dev(c["a"]), dev(c["b"]), dev(c["s"]), dev(c["z"])
    out = torch.empty((M, N), dtype=torch.float16, device="cuda")
    ws = w.alloc_workspace(M, N, K, 128, kernel=w.KERNEL_TC)
    evict = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    evict.fill_(1)
    w.w4a16_gemm(a, b, s, z, 128, 0, out=out, workspace=ws, kernel=w.KERNEL_TC)
    torch.cuda.synchronize()
    del evict
    g = np.random.default_rng(256)
    cols = np.unique(np.concatenate([np.arange(0, N, 128) + g.integers(0, 128, N // 128), [0, N - 1]]))
    assert_close(out.cpu().numpy()[:, cols], ref(c, cols=cols), "TC M=256 from DRAM")


@pytest.mark.parametrize("M,N,K", [
    (17, 28672, 4096),    # 224 column tiles: more than one wave already on 148 SMs, no split
    (24, 28672, 4096),
    (32, 14336, 4096),    # 112 tiles: a split would need a second wave on 148 SMs
    (32, 4096, 14336),    # 32 tiles and a long K: a split that stays within one wave
])
def test_tc_automatic_split_stays_within_one_wave(w, M, N, K):
    """The automatic K split of the tensor-core GEMM is one whose CTAs are all resident at once
    (one CTA per SM at these row counts): its workspace holds fp32 partials only when two CTAs
    per column tile fit on the GPU, and then for a split that fits."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    tiles = N // 128
    ws = w.w4a16_gemm_workspace_bytes(M, N, K, 128, kernel=w.KERNEL_TC)
    split = ws // (M * N * 4)   # the partials hold split x M x N fp32 values (plus a small header)
    if 2 * tiles > sms:
        assert split == 0, (M, N, K, ws)
    else:
        assert 2 <= split and split * tiles <= sms, (M, N, K, ws, split)


@pytest.mark.parametrize("G", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("split", [1, 3])
def test_tc_group_sizes_and_splits(w, G, split):
    c = synth.make_case(24, 1024, 256, G, sym=False, seed=G + split)
    assert_close(run(w, c, kernel=w.KERNEL_TC, split_k=split), ref(c), f"TC G={G} split={split}")


@pytest.mark.parametrize("M", [32, 40, 72, 96, 104, 128])
@pytest.mark.parametrize("split", [2, 5, 7, 16])
def test_tc_splits(w, split, M):
    # From 32 rows up two epilogue warpgroups each reduce their half of the rows; at 40, 72 and
    # 104 rows (tile widths 48, 80, 112) the halves are 24, 40 and 56 columns wide.
    c = synth.make_case(M, 2048, 1024, 128, sym=True, seed=split)
    assert_close(run(w, c, kernel=w.KERNEL_TC, split_k=split), ref(c), f"TC split={split}")


def test_tc_q_equals_z_gives_exact_zero(w):
    K, N, G = 512, 256, 128
    g = np.random.default_rng(4)
    zq = synth.words_nibbles_in(g, (K // G, N // 8), 0, 15)
    c = dict(a=synth.fp16_normal(g, (20, K)), b=np.repeat(zq, G, axis=0),
             s=synth.fp16_uniform(g, (K // G, N), 0.01, 0.02), z=zq, G=G, zp_bias=0)
    assert torch.all(run(w, c, kernel=w.KERNEL_TC) == 0)


def test_tc_repeatable_and_workspace_restored(w):
    c = synth.make_case(32, 4096, 2048, 128, sym=False, seed=8)
    ws = w.alloc_workspace(32, 2048, 4096, 128, kernel=w.KERNEL_TC, split_k=4)
    o1 = run(w, c, kernel=w.KERNEL_TC, split_k=4, workspace=ws)
    o2 = run(w, c, kernel=w.KERNEL_TC, split_k=4, workspace=ws)
    assert torch.equal(o1, o2)
    assert int(ws[256:256 + 4 * (2048 // 128)].count_nonzero()) == 0
    assert w.w4a16_workspace_status(ws) == 0
    assert_close(o1, ref(c), "TC split 4")


def test_tc_rejects_unsupported_shapes(w):
    c = synth.make_case(16, 512, 136, 128, sym=True, seed=9)   # N % 128 != 0
    with pytest.raises(w.W4A16Error) as e:
        run(w, c, kernel=w.KERNEL_TC)
    assert e.value.status == w.W4A16_ERR_UNSUPPORTED
    # auto falls back to the GEMV row blocks for the same shape
    assert_close(run(w, c), ref(c), "auto fallback")


@pytest.mark.parametrize("kernel,M", [("TC", 32), ("GEMV", 1), ("GEMV", 4)])
def test_timeout_status_and_recovery(w, kernel, M):
    """Every device-side wait runs out (nothing is loaded): the kernel must report
    W4A16_ERR_TIMEOUT in the workspace status word, free its resources and leave
    the context usable for the next, normal call."""
    kid = w.KERNEL_TC if kernel == "TC" else w.KERNEL_GEMV
    c = synth.make_case(M, 1024, 1024, 128, sym=False, seed=11)
    ws = w.alloc_workspace(M, 1024, 1024, 128, kernel=kid)
    run(w, c, kernel=kid, workspace=ws, debug_flags=w.DEBUG_STALL_LOADS, wait_limit_us=20000)
    assert w.w4a16_workspace_status(ws, clear=True) == w.W4A16_ERR_TIMEOUT
    assert w.w4a16_workspace_status(ws) == 0
    # counters may be left mid-count by the aborted call: start from a clean workspace
    ws.zero_()
    assert_close(run(w, c, kernel=kid, workspace=ws), ref(c), f"after timeout ({kernel})")
