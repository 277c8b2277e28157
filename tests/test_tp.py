"""Tensor-parallel sharding of the layer (weight_only_int4_08_b200.tp), host side, on CPU.

The shard bounds tile [0, extent) in whole units; a column shard's output is exactly the
full layer's columns (each output column depends on its own weights only), so the CPU
oracle on the shards, gathered, must equal the oracle on the whole layer bit for bit; a
row shard's fp32 partials, added and rounded once, must match the whole layer within the
layer's tolerance. Two `gloo` ranks (world size 2) run the same split and the collectives
(all-gather of column shards, all-gather and all-reduce of fp32 partials): both ranks must
end with the same bits, and those must match the oracle on the whole layer. The CUDA path
of the same functions is covered by tests/test_gpu_tp.py.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth
from weight_only_int4_08_b200 import tp

ATOL, RTOL = 1e-3, 8e-3


def _within(got, ref):
    return bool(np.all(np.abs(got.astype(np.float64) - ref) <= ATOL + RTOL * np.abs(ref.astype(np.float64))))


def _layer(M, K, N, G, sym, seed):
    c = synth.make_case(M, K, N, G, sym=sym, seed=seed)
    t = lambda x: None if x is None else torch.from_numpy(np.ascontiguousarray(x))
    return c, t(c["b"]), t(c["s"]), t(c["z"])


def _np(x):
    return None if x is None else x.numpy()


@pytest.mark.parametrize("extent,world,unit", [(4096, 2, 128), (14336, 4, 128), (40, 2, 8), (4104, 3, 8),
                                               (1024, 8, 128), (384, 3, 128)])
def test_split_bounds_tile_the_extent(extent, world, unit):
    b = [tp.split_bounds(extent, world, r, unit) for r in range(world)]
    assert b[0][0] == 0 and b[-1][1] == extent
    for (lo, hi), (lo2, _) in zip(b, b[1:]):
        assert hi == lo2
    widths = [hi - lo for lo, hi in b]
    assert all(w > 0 and w % unit == 0 and lo % unit == 0 for w, (lo, _) in zip(widths, b))
    assert max(widths) - min(widths) <= unit


def test_split_bounds_rejects_bad_splits():
    with pytest.raises(ValueError):
        tp.split_bounds(100, 2, 0, 8)       # not whole units
    with pytest.raises(ValueError):
        tp.split_bounds(16, 4, 0, 8)        # fewer units than ranks
    with pytest.raises(ValueError):
        tp.split_bounds(64, 2, 2, 8)        # rank outside the world
    _, b, s, z = _layer(1, 256, 64, 128, False, 1)
    with pytest.raises(ValueError):
        tp.row_shard(b, s, z, 128, 0, 2, unit=64)   # a group split over two ranks
    with pytest.raises(ValueError):
        tp.column_shard(b, s, z, 0, 2, unit=12)     # not whole packed words


@pytest.mark.parametrize("world,unit,sym", [(2, 8, False), (3, 8, True), (4, 16, False)])
def test_column_shards_concatenate_to_the_layer(world, unit, sym):
    M, K, N, G = 3, 256, 96, 64
    c, b, s, z = _layer(M, K, N, G, sym, 7)
    full = oracle.gemm(c["a"], c["b"], c["s"], c["z"], G, c["zp_bias"])
    outs = []
    for r in range(world):
        sh = tp.column_shard(b, s, z, r, world, unit)
        assert sh.b_packed.is_contiguous() and sh.scales.is_contiguous()
        assert sh.b_packed.shape == (K, (sh.hi - sh.lo) // 8) and sh.scales.shape == (K // G, sh.hi - sh.lo)
        outs.append(oracle.gemm(c["a"], _np(sh.b_packed), _np(sh.scales), _np(sh.qzeros), G, c["zp_bias"]))
    got = np.concatenate(outs, axis=1)
    assert np.array_equal(got.view(np.uint16), full.view(np.uint16))


@pytest.mark.parametrize("world,sym", [(2, False), (4, True), (3, False)])
def test_row_shards_add_up_to_the_layer(world, sym):
    M, K, N, G = 4, 768, 64, 64
    c, b, s, z = _layer(M, K, N, G, sym, 9)
    full, full_acc = oracle.gemm(c["a"], c["b"], c["s"], c["z"], G, c["zp_bias"], want_acc=True)
    a = torch.from_numpy(c["a"])
    total = np.zeros((M, N), np.float32)
    for r in range(world):
        sh = tp.row_shard(b, s, z, G, r, world)
        assert sh.lo % G == 0 and sh.hi % G == 0
        a_r = tp.row_shard_activations(a, sh)
        assert a_r.is_contiguous() and a_r.shape == (M, sh.hi - sh.lo)
        _, acc = oracle.gemm(a_r.numpy(), _np(sh.b_packed), _np(sh.scales), _np(sh.qzeros), G, c["zp_bias"],
                             want_acc=True)
        total = total + acc
    assert _within(total, full_acc)
    assert _within(total.astype(np.float16).astype(np.float32), full.astype(np.float32))


def _free_port():
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = {}
        # column-parallel, uneven shards (5 packed words over 2 ranks)
        M, K, N, G = 2, 256, 40, 64
        c, b, s, z = _layer(M, K, N, G, False, 31)
        sh = tp.column_shard(b, s, z, rank, world)
        mine = oracle.gemm(c["a"], _np(sh.b_packed), _np(sh.scales), _np(sh.qzeros), G, c["zp_bias"])
        got = tp.gather_columns(torch.from_numpy(mine), N)
        res["col"] = got.numpy().view(np.uint16).copy()
        res["col_ref"] = oracle.gemm(c["a"], c["b"], c["s"], c["z"], G, c["zp_bias"]).view(np.uint16)
        # row-parallel
        M, K, N, G = 3, 512, 48, 128
        c, b, s, z = _layer(M, K, N, G, True, 37)
        sh = tp.row_shard(b, s, z, G, rank, world)
        a_r = tp.row_shard_activations(torch.from_numpy(c["a"]), sh)
        _, acc = oracle.gemm(a_r.numpy(), _np(sh.b_packed), _np(sh.scales), _np(sh.qzeros), G, c["zp_bias"],
                             want_acc=True)
        parts = tp.collect_partials(torch.from_numpy(acc.copy()), mode="gather")
        res["parts"] = [p.numpy().copy() for p in parts]
        summed = tp.collect_partials(torch.from_numpy(acc.copy()), mode="sum")
        res["sum"] = summed[0].numpy().copy()
        res["row_ref"], res["row_ref_acc"] = oracle.gemm(c["a"], c["b"], c["s"], c["z"], G, c["zp_bias"],
                                                         want_acc=True)
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_tp_collectives_gloo_world_2():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    r0, r1 = out[0], out[1]
    # column shards gathered: the whole layer, bit for bit, on both ranks
    assert np.array_equal(r0["col"], r0["col_ref"]) and np.array_equal(r1["col"], r0["col_ref"])
    # all-gathered partials: the same list, in rank order, on both ranks
    assert len(r0["parts"]) == world
    for p0, p1 in zip(r0["parts"], r1["parts"]):
        assert np.array_equal(p0, p1)
    fixed_order = r0["parts"][0] + r0["parts"][1]
    # two fp32 addends: the all-reduce's sum has the same bits whatever its order
    assert np.array_equal(r0["sum"], fixed_order) and np.array_equal(r1["sum"], fixed_order)
    assert _within(fixed_order, r0["row_ref_acc"])
    assert _within(fixed_order.astype(np.float16).astype(np.float32), r0["row_ref"].astype(np.float32))
