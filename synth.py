"""Seeded synthetic inputs for the W4A16 linear layer.

This module only draws random numbers: it holds none of the layer's arithmetic
(no unpacking, dequantisation or matmul). The tests feed the same arrays to the
CPU oracle and to the CUDA library; bench.py uses it for its workloads.

Streams: numpy's PCG64 bit generator seeded from SeedSequence([seed, tensor_id]),
one independent stream per tensor. fp16 values are fp32 draws rounded to nearest
even once (numpy astype). Packed int4 words are built from independent draws,
so every nibble of every word is independently distributed:
  - uniform{0..15} nibbles: a uniformly random 32-bit word;
  - uniform{lo..hi} nibbles: eight independent draws per word.

Workload shapes and distributions follow the five configurations of the weight-only
int4 decode study (tiny GEMV, 8B MLP-up GEMV, small-batch sweep, batch-32 GEMM
with checkpoint repack, 32-layer decode-step linear stack).
"""
from __future__ import annotations

import numpy as np

# tensor ids: one stream each
T_A, T_B, T_S, T_Z, T_CKPT, T_CT_S, T_CT_Z = 1, 2, 3, 4, 5, 6, 7


def rng(seed: int, tensor_id: int, layer: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id, layer])))


def fp16_uniform(g: np.random.Generator, shape, lo: float, hi: float) -> np.ndarray:
    return g.uniform(lo, hi, size=shape).astype(np.float32).astype(np.float16)


def fp16_normal(g: np.random.Generator, shape) -> np.ndarray:
    return g.standard_normal(size=shape, dtype=np.float32).astype(np.float16)


def words_uniform(g: np.random.Generator, shape) -> np.ndarray:
    """int32 words whose 8 nibbles are independent uniform{0..15}."""
    return g.integers(0, 1 << 32, size=shape, dtype=np.uint32).view(np.int32)


def words_nibbles_in(g: np.random.Generator, shape, lo: int, hi: int) -> np.ndarray:
    """int32 words whose 8 nibbles are independent uniform{lo..hi} (inclusive)."""
    shape = tuple(shape) if isinstance(shape, (tuple, list)) else (shape,)
    d = g.integers(lo, hi + 1, size=shape + (8,), dtype=np.uint32)
    w = np.zeros(shape, np.uint32)
    for j in range(8):
        w |= d[..., j] << np.uint32(4 * j)
    return w.view(np.int32)


def make_case(M, K, N, G, *, sym: bool, seed: int, a_dist: str = "normal",
              s_lo: float = 0.002, s_hi: float = 0.02, zp_bias: int = 8,
              z_lo: int = 6, z_hi: int = 10, ckpt_layout: bool = False, layer: int = 0):
    """One W4A16 problem. Returns a dict of numpy arrays and sizes.

    b (kernel layout [K, N/8]) is drawn directly, or, with ckpt_layout, the
    checkpoint-layout weight ckpt [N, K/8] is drawn instead (b is then absent
    and must come from a repack)."""
    case = dict(M=M, K=K, N=N, G=G, zp_bias=zp_bias if sym else 0, sym=sym, seed=seed)
    ga = rng(seed, T_A, layer)
    case["a"] = fp16_uniform(ga, (M, K), -1.0, 1.0) if a_dist == "uniform" else fp16_normal(ga, (M, K))
    if ckpt_layout:
        case["ckpt"] = words_uniform(rng(seed, T_CKPT, layer), (N, K // 8))
    else:
        case["b"] = words_uniform(rng(seed, T_B, layer), (K, N // 8))
    case["s"] = fp16_uniform(rng(seed, T_S, layer), (K // G, N), s_lo, s_hi)
    case["z"] = None if sym else words_nibbles_in(rng(seed, T_Z, layer), (K // G, N // 8), z_lo, z_hi)
    return case


def ct_checkpoint(K, N, G, *, sym: bool, seed: int, s_lo: float = 0.002, s_hi: float = 0.02,
                  z_lo: int = 6, z_hi: int = 10):
    """A layer as the checkpoint stores it: weight [N, K/8], scales [N, K/G] fp16 and,
    unless sym, zeros [N/8, K/G] (8 output channels per int32)."""
    return dict(K=K, N=N, G=G, sym=sym, seed=seed,
                ckpt=words_uniform(rng(seed, T_CKPT), (N, K // 8)),
                s_ng=fp16_uniform(rng(seed, T_CT_S), (N, K // G), s_lo, s_hi),
                z_n8g=None if sym else words_nibbles_in(rng(seed, T_CT_Z), (N // 8, K // G), z_lo, z_hi))


# ---- the five workloads -----------------------------------------------------

def config1():
    """Tiny symmetric GEMV: M=1, K=N=512, G=128, zp_bias=8; A U[-1,1]; s U[0.005,0.02]; seed 0."""
    return make_case(1, 512, 512, 128, sym=True, seed=0, a_dist="uniform", s_lo=0.005, s_hi=0.02)


def config2():
    """Decode GEMV, 8B MLP-up shape: M=1, K=4096, N=14336, G=128, sym; A N(0,1); s U[0.002,0.02]; seed 1."""
    return make_case(1, 4096, 14336, 128, sym=True, seed=1)


def config3(M: int):
    """Small-batch asymmetric sweep: M in {1,2,4,8,16}, K=N=4096, G=128; zeros U{6..10}; seed 2."""
    return make_case(M, 4096, 4096, 128, sym=False, seed=2)


def config4():
    """Batch-32 GEMM with repack: M=32, K=4096, N=14336, G=128, asym; weight in checkpoint layout; seed 3."""
    return make_case(32, 4096, 14336, 128, sym=False, seed=3, ckpt_layout=True)


# 8B-shaped decoder layer (hidden 4096): (name, K, N)
LAYER_LINEARS = (("qkv", 4096, 6144), ("o", 4096, 4096), ("gate_up", 4096, 28672), ("down", 14336, 4096))
N_LAYERS = 32


def config5_linear(layer: int, idx: int, M: int):
    """Linear `idx` of decoder layer `layer` in the 32-layer stack; sym G=128; fresh N(0,1) input; seed 4."""
    _, K, N = LAYER_LINEARS[idx]
    return make_case(M, K, N, 128, sym=True, seed=4, layer=layer * 8 + idx)
