"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Repack must match bit-exactly; the GEMM must satisfy
|gpu - oracle| <= 1e-3 + 8e-3 * |oracle| elementwise (fp16 outputs compared as
floats; equal infinities match). Sizes cover several tiles plus ragged tails,
the five workloads at full size (the 32-layer stack on sampled columns), the
degenerate cases (q == z, K == G, N == 8) and every kernel/vector-width path.
"""
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


def dev(x):
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        return torch.from_numpy(x).cuda()
    return torch.from_numpy(x.view(np.int32)).cuda()


def assert_close(gpu, ref, what=""):
    g = gpu.float().cpu().numpy() if isinstance(gpu, torch.Tensor) else gpu.astype(np.float32)
    r = ref.astype(np.float32)
    both_inf = np.isinf(g) & np.isinf(r) & (np.sign(g) == np.sign(r))
    err = np.abs(g - r)
    ok = (err <= ATOL + RTOL * np.abs(r)) | both_inf
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        raise AssertionError(f"{what}: {int((~ok).sum())} of {ok.size} outside tolerance; first {idx.tolist()} "
                             f"gpu={[g[tuple(i)] for i in idx]} ref={[r[tuple(i)] for i in idx]}")


def run(w, case, b=None, **kw):
    a, s = dev(case["a"]), dev(case["s"])
    bb = b if b is not None else dev(case["b"])
    z = dev(case["z"]) if case["z"] is not None else None
    out = w.w4a16_gemm(a, bb, s, z, case["G"], case["zp_bias"], **kw)
    torch.cuda.synchronize()
    return out


def ref(case, cols=None):
    return oracle.gemm(case["a"], case["b"], case["s"], case["z"], case["G"], case["zp_bias"], cols=cols)


# ------------------------------------------------------------------ repack ----

@pytest.mark.parametrize("N,K", [(8, 8), (40, 24), (256, 256), (264, 520), (2056, 1032), (14336, 4096)])
def test_repack_bit_exact(w, N, K):
    g = np.random.default_rng(N * 7 + K)
    ck = synth.words_uniform(g, (N, K // 8))
    out = w.w4a16_repack(dev(ck), N, K)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint32), oracle.repack(ck, N, K))


def test_repack_worked_example(w):
    from conftest import read_golden
    d = read_golden("worked_repack.txt")
    ck = np.stack([np.array([int(h, 16) for h in d[f"ckpt_n{n}"]], np.uint32) for n in range(8)])
    out = w.w4a16_repack(dev(ck), 8, 16)
    expect = np.array([int(h, 16) for h in d["kernel"]], np.uint32).reshape(16, 1)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), expect)


# ---------------------------------------------------------- the workloads ----

def test_config1_tiny_symmetric(w):
    c = synth.config1()
    assert_close(run(w, c), ref(c), "config1")


def test_config2_decode_gemv(w):
    c = synth.config2()
    assert_close(run(w, c), ref(c), "config2")


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16])
def test_config3_small_batch_asym(w, M):
    c = synth.config3(M)
    assert_close(run(w, c), ref(c), f"config3 M={M}")


def test_config4_batch32_with_repack(w):
    c = synth.config4()
    b_dev = w.w4a16_repack(dev(c["ckpt"]), c["N"], c["K"])
    c["b"] = oracle.repack(c["ckpt"], c["N"], c["K"])
    assert np.array_equal(b_dev.cpu().numpy().view(np.uint32), c["b"])
    assert_close(run(w, c, b=b_dev), ref(c), "config4")


@pytest.mark.parametrize("M", [1, 32])
def test_config5_stack_sampled(w, M):
    g = np.random.default_rng(M)
    for layer in (0, 31):
        for idx in range(4):
            c = synth.config5_linear(layer, idx, M)
            cols = np.sort(g.choice(c["N"], 192, replace=False))
            out = run(w, c)
            assert_close(out[:, cols], ref(c, cols), f"config5 layer {layer} linear {idx} M={M}")


# ------------------------------------------------------------ edge cases ----

@pytest.mark.parametrize("M,K,N,G,sym", [
    (1, 16, 8, 16, True),        # smallest legal problem, K == G
    (3, 128, 8, 128, False),     # N == 8, K == G
    (5, 256, 40, 32, False),     # N % 16 != 0 -> one word per thread
    (7, 384, 48, 128, True),     # N % 32 != 0 -> two words per thread
    (2, 640, 520, 64, False),    # ragged column tile, odd group count
    (9, 512, 264, 128, True),    # M > 8 through the GEMV row blocks
    (15, 256, 136, 16, False),
    (33, 1024, 776, 128, False),
    (1, 4096, 4104, 128, False),  # 4104 = 16*256 + 8: one-word tail tile
    (5, 1024, 19968, 128, False),  # 156 column tiles, more than the SMs: the 4-warp GEMV
    (8, 512, 38912, 64, True),     # 304 tiles, G below the unit rows, 4-warp GEMV
    (1, 256, 19200, 128, True),    # 150 tiles: one tile per CTA, ragged last wave
])
def test_odd_shapes(w, M, K, N, G, sym):
    c = synth.make_case(M, K, N, G, sym=sym, seed=M + K + N)
    assert_close(run(w, c), ref(c), f"odd {M}x{K}x{N} G{G}")


@pytest.mark.parametrize("G", [16, 32, 48, 64, 80, 128, 192, 256])
@pytest.mark.parametrize("M", [1, 3, 12, 16])
def test_gemv_group_sizes(w, G, M):
    # groups that are and are not multiples of the 64-row load unit; K spans several groups
    c = synth.make_case(M, 8 * G, 384, G, sym=False, seed=G + M)
    assert_close(run(w, c, kernel=w.KERNEL_GEMV), ref(c), f"GEMV G={G} M={M}")


@pytest.mark.parametrize("M,K,N,G,sym", [
    (9, 512, 384, 64, False),      # one 16-row block, two batch tiles (the second partly empty)
    (13, 640, 544, 80, True),      # groups straddle the 64-row stages; ragged column tile
    (16, 1024, 256, 16, False),
    (17, 512, 384, 128, False),    # blocks of 16 and 1 rows (different stage heights)
    (40, 768, 256, 48, True),      # blocks of 16, 16 and 8 rows
])
def test_gemv_two_batch_tiles(w, M, K, N, G, sym):
    c = synth.make_case(M, K, N, G, sym=sym, seed=M * 31 + K)
    assert_close(run(w, c, kernel=w.KERNEL_GEMV), ref(c), f"GEMV {M}x{K}x{N} G{G}")


@pytest.mark.parametrize("MT", list(range(9, 17)))
def test_gemv_every_row_count_to_16(w, MT):
    c = synth.make_case(MT, 1024, 512, 128, sym=(MT % 2 == 0), seed=70 + MT)
    assert_close(run(w, c), ref(c), f"GEMV M={MT}")


@pytest.mark.parametrize("split", [1, 2, 3, 7, 33, 256])
def test_split_k_variants(w, split):
    c = synth.make_case(2, 2048, 1024, 128, sym=False, seed=21)
    assert_close(run(w, c, kernel=w.KERNEL_GEMV, split_k=split), ref(c), f"split {split}")


@pytest.mark.parametrize("offset_words", [1, 2, 3])
def test_misaligned_weights_take_narrow_path(w, offset_words):
    c = synth.make_case(1, 512, 512, 128, sym=False, seed=22)
    big = torch.zeros(c["b"].size + 8, dtype=torch.int32, device="cuda")
    big[offset_words:offset_words + c["b"].size] = dev(c["b"]).view(-1)
    b = big[offset_words:offset_words + c["b"].size].view(512, 64)
    assert_close(run(w, c, b=b), ref(c), f"offset {offset_words}")


def test_q_equals_z_gives_exact_zero(w):
    K, N, G = 512, 256, 128
    g = np.random.default_rng(3)
    zq = synth.words_nibbles_in(g, (K // G, N // 8), 0, 15)
    b = np.repeat(zq, G, axis=0)
    c = dict(a=synth.fp16_normal(g, (4, K)), b=b, s=synth.fp16_uniform(g, (K // G, N), 0.01, 0.02), z=zq,
             G=G, zp_bias=0)
    out = run(w, c)
    assert torch.all(out == 0)


def test_overflow_to_inf_matches(w):
    c = synth.make_case(1, 512, 64, 128, sym=True, seed=5)
    c["a"] = np.full((1, 512), 60000.0, np.float16)
    c["s"] = np.full((4, 64), 1.0, np.float16)
    assert_close(run(w, c), ref(c), "overflow")


def test_repeatable_and_workspace_restored(w):
    c = synth.config2()
    ws = w.alloc_workspace(1, c["N"], c["K"], c["G"])
    o1 = run(w, c, workspace=ws)
    o2 = run(w, c, workspace=ws)
    assert torch.equal(o1, o2)
    tiles = (c["N"] + 127) // 128                                # tiles are at least 128 columns wide
    assert int(ws[256:256 + 4 * tiles].count_nonzero()) == 0   # arrival counters back to zero
    assert w.w4a16_workspace_status(ws) == 0


def test_workspace_too_small_is_rejected(w):
    c = synth.config2()
    need = w.w4a16_gemm_workspace_bytes(1, c["N"], c["K"], c["G"])
    assert need > 0
    ws = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(w.W4A16Error) as e:
        run(w, c, workspace=ws)
    assert e.value.status == w.W4A16_ERR_INVALID_ARG


def test_runs_on_a_side_stream(w):
    c = synth.config1()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = run(w, c)
    s.synchronize()
    assert_close(out, ref(c), "side stream")
