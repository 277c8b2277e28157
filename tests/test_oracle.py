"""Pins for the CPU oracle: it is checked against things other than itself.

- IEEE binary16 conversions against numpy's float16 (exhaustive decode, RNE encode);
- the hand-computed worked examples in tests/golden/ (GEMM closed form 1.5n - 7.25,
  repack hex words);
- brute force in float64 on tiny shapes covering every nibble value in every
  nibble position;
- invariants: q == z gives 0, zp_bias 8 == all-8 zeros, exact scale doubling,
  linearity in A, integer matmul special case (s = 1, z = 0) against numpy int64;
- repack: single-nibble tracking over every position, round trip, permutation;
- checkpoint scales/zeros: the hand-computed worked example, single-element
  tracking, the one-group special case (memory unchanged), and the dense
  dequantised weight computed straight from the checkpoint layout.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _words(hexes):
    return np.array([int(h, 16) for h in hexes], dtype=np.uint32)


# ---------------------------------------------------------------- fp16 ----

def test_half_decode_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([oracle.half_to_float(int(b)) for b in bits], dtype=np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_half_encode_rne():
    g = np.random.default_rng(123)
    vals = [g.standard_normal(20000).astype(np.float32) * np.float32(s) for s in (1e-6, 1e-3, 1.0, 300.0, 6e4)]
    h = np.arange(0, 0x7c00, 7, dtype=np.uint16).view(np.float16).astype(np.float32)
    # exact midpoints between adjacent halves (ties), and near-midpoints
    lo = np.arange(0, 0x7bff, 3, dtype=np.uint16)
    a = lo.view(np.float16).astype(np.float64)
    b = (lo + 1).view(np.float16).astype(np.float64)
    mid = ((a + b) / 2).astype(np.float32)
    special = np.array([0.0, -0.0, 65504.0, 65520.0, 65519.99, 7e4, -7e4, 2.0 ** -24, 2.0 ** -25,
                        2.0 ** -25 * 1.0000001, 2.0 ** -26, 6.1e-5, 1e-30, np.inf, -np.inf], np.float32)
    x = np.concatenate(vals + [h, -h, mid, -mid, np.nextafter(mid, np.float32(np.inf)), special])
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    got = np.array([oracle.float_to_half_bits(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got, ref)
    assert (oracle.float_to_half_bits(float("nan")) & 0x7c00) == 0x7c00


# ------------------------------------------------------- worked examples ----

def test_worked_gemm_symmetric_and_asymmetric(golden):
    d = golden("worked_gemm.txt")
    K, N, G = int(d["K"][0]), int(d["N"][0]), int(d["G"][0])
    b = _words(d["b_hex"]).reshape(K, N // 8)
    a = np.array([float(v) for v in d["a"]], np.float16).reshape(1, K)
    s = np.array([[float(d["s_group0"][0])] * N, [float(d["s_group1"][0])] * N], np.float16)
    expect = np.array([float(v) for v in d["out"]], np.float32)
    # closed form from the hand derivation
    assert np.array_equal(expect, 1.5 * np.arange(N) - 7.25)
    out = oracle.gemm(a, b, s, None, G, zp_bias=int(d["zp_bias"][0]))
    assert np.array_equal(out[0].astype(np.float32), expect)
    z = _words(d["qzeros_hex"]).reshape(K // G, N // 8)
    out2 = oracle.gemm(a, b, s, z, G, zp_bias=0)
    assert np.array_equal(out2[0].astype(np.float32), expect)
    # the packed words are q[k][n] = (k + n) mod 16
    q = oracle.unpack_kn8(b, K, N)
    kk, nn = np.meshgrid(np.arange(K), np.arange(N), indexing="ij")
    assert np.array_equal(q, (kk + nn) % 16)


def test_worked_repack(golden):
    d = golden("worked_repack.txt")
    K, N = int(d["K"][0]), int(d["N"][0])
    ckpt = np.stack([_words(d[f"ckpt_n{n}"]) for n in range(N)])
    expect = _words(d["kernel"]).reshape(K, N // 8)
    assert np.array_equal(oracle.repack(ckpt, N, K), expect)
    assert np.array_equal(oracle.unrepack(expect, K, N), ckpt)
    q = oracle.unpack_kn8(expect, K, N)
    kk, nn = np.meshgrid(np.arange(K), np.arange(N), indexing="ij")
    assert np.array_equal(q, (kk + 2 * nn) % 16)


# ------------------------------------------------------------ brute force ----

def _brute_f64(a, q, s, zfull, G):
    """Exact-ish float64 dense computation written without the oracle's code path."""
    M, K = a.shape
    N = q.shape[1]
    out = np.zeros((M, N), np.float64)
    for m in range(M):
        for n in range(N):
            tot = 0.0
            for k in range(K):
                g = k // G
                tot += float(a[m, k]) * (int(q[k, n]) - int(zfull[g, n])) * float(s[g, n])
            out[m, n] = tot
    return out


def _pack_rows(vals):
    """Pack an [R, C] array of nibbles 8 per word along C with Python ints (test-side)."""
    R, C = vals.shape
    w = np.zeros((R, C // 8), np.uint32)
    for r in range(R):
        for c in range(C // 8):
            x = 0
            for j in range(8):
                x |= int(vals[r, 8 * c + j]) << (4 * j)
            w[r, c] = x
    return w


@pytest.mark.parametrize("M,K,N,G", [(1, 8, 8, 8), (2, 16, 16, 8), (3, 32, 16, 16), (3, 32, 8, 8), (2, 16, 24, 16)])
@pytest.mark.parametrize("sym", [True, False])
def test_brute_force_tiny(M, K, N, G, sym):
    g = np.random.default_rng(1000 * M + 10 * K + N + G + sym)
    q = g.integers(0, 16, size=(K, N))
    # force coverage of every nibble value in every nibble position
    for j in range(min(8, N)):
        q[: min(K, 16), j] = (np.arange(min(K, 16)) + j) % 16
    zq = g.integers(0, 16, size=(K // G, N))
    zp = int(g.integers(0, 16))
    a = (g.standard_normal((M, K)) * 2).astype(np.float16)
    s = g.uniform(0.001, 0.05, size=(K // G, N)).astype(np.float16)
    b = _pack_rows(q)
    z = None if sym else _pack_rows(zq)
    zfull = np.full((K // G, N), zp) if sym else zq
    out, acc = oracle.gemm(a, b, s, z, G, zp_bias=zp, want_acc=True)
    ref = _brute_f64(a, q, s, zfull, G)
    # fp32 accumulation error bound: K * 2^-24 * sum |terms| (generous)
    bound = np.zeros_like(ref)
    for m in range(M):
        for n in range(N):
            bound[m, n] = sum(abs(float(a[m, k]) * (int(q[k, n]) - int(zfull[k // G, n])) * float(s[k // G, n]))
                              for k in range(K)) * K * 2.0 ** -23
    assert np.all(np.abs(acc.astype(np.float64) - ref) <= bound + 1e-30)
    # fp16 output within one fp16 ulp of the exact value, and equal to fp16(acc)
    r16 = ref.astype(np.float16).astype(np.float64)
    ulp = np.abs(np.nextafter(r16.astype(np.float16), np.float16(np.inf)).astype(np.float64) - r16)
    assert np.all(np.abs(out.astype(np.float64) - r16) <= ulp + 1e-12)
    assert np.array_equal(out.view(np.uint16), acc.astype(np.float16).view(np.uint16))


# ------------------------------------------------------------- invariants ----

def test_q_equals_z_gives_zero():
    g = np.random.default_rng(5)
    M, K, N, G = 3, 64, 32, 16
    zq = g.integers(0, 16, size=(K // G, N))
    q = np.repeat(zq, G, axis=0)
    b, z = _pack_rows(q), _pack_rows(zq)
    a = g.standard_normal((M, K)).astype(np.float16)
    s = g.uniform(0.01, 0.1, (K // G, N)).astype(np.float16)
    out, acc = oracle.gemm(a, b, s, z, G, want_acc=True)
    assert np.all(acc == 0.0) and np.all(out.astype(np.float32) == 0.0)
    # symmetric: q == zp_bias everywhere
    b8 = _pack_rows(np.full((K, N), 5))
    out8 = oracle.gemm(a, b8, s, None, G, zp_bias=5)
    assert np.all(out8.astype(np.float32) == 0.0)


def test_symmetric_equals_all_eight_zeros():
    c = synth.make_case(2, 256, 64, 64, sym=True, seed=9)
    z8 = np.full((256 // 64, 64 // 8), 0x88888888, np.uint32)
    o1 = oracle.gemm(c["a"], c["b"], c["s"], None, 64, zp_bias=8)
    o2 = oracle.gemm(c["a"], c["b"], c["s"], z8, 64, zp_bias=3)  # zp_bias ignored with zeros
    assert np.array_equal(o1.view(np.uint16), o2.view(np.uint16))


def test_scale_doubling_is_exact():
    c = synth.make_case(2, 256, 64, 128, sym=False, seed=10)
    _, acc1 = oracle.gemm(c["a"], c["b"], c["s"], c["z"], 128, want_acc=True)
    s2 = (c["s"].astype(np.float32) * 2).astype(np.float16)
    _, acc2 = oracle.gemm(c["a"], c["b"], s2, c["z"], 128, want_acc=True)
    assert np.array_equal(acc2, acc1 * 2)


def test_linearity_in_a():
    c = synth.make_case(2, 512, 64, 128, sym=False, seed=11)
    g = np.random.default_rng(12)
    # a1 + a2 exact in fp16: integers/4 in a small range
    a1 = (g.integers(-40, 40, (2, 512)) / 4).astype(np.float16)
    a2 = (g.integers(-40, 40, (2, 512)) / 4).astype(np.float16)
    a12 = (a1.astype(np.float32) + a2.astype(np.float32)).astype(np.float16)
    assert np.array_equal(a12.astype(np.float32), a1.astype(np.float32) + a2.astype(np.float32))
    _, r1 = oracle.gemm(a1, c["b"], c["s"], c["z"], 128, want_acc=True)
    _, r2 = oracle.gemm(a2, c["b"], c["s"], c["z"], 128, want_acc=True)
    _, r12 = oracle.gemm(a12, c["b"], c["s"], c["z"], 128, want_acc=True)
    mag = np.abs(r1) + np.abs(r2) + 1.0
    assert np.all(np.abs(r12 - (r1 + r2)) <= 1e-4 * mag)


def test_integer_matmul_special_case():
    """s = 1 and z = 0: the layer is a plain integer matmul a @ q (checked with numpy int64)."""
    g = np.random.default_rng(13)
    M, K, N, G = 4, 256, 48, 32
    q = g.integers(0, 16, size=(K, N))
    ai = g.integers(-8, 9, size=(M, K))
    a = ai.astype(np.float16)
    s = np.ones((K // G, N), np.float16)
    out, acc = oracle.gemm(a, _pack_rows(q), s, None, G, zp_bias=0, want_acc=True)
    ref = ai.astype(np.int64) @ q.astype(np.int64)
    assert np.array_equal(acc.astype(np.int64), ref)
    assert np.array_equal(out, ref.astype(np.float16))


def test_columns_subset_matches_full():
    c = synth.make_case(3, 512, 256, 128, sym=False, seed=14)
    full = oracle.gemm(c["a"], c["b"], c["s"], c["z"], 128)
    cols = [0, 7, 8, 100, 255, 31]
    sub = oracle.gemm(c["a"], c["b"], c["s"], c["z"], 128, cols=cols)
    assert np.array_equal(sub.view(np.uint16), full[:, cols].view(np.uint16))


# ---------------------------------------------------------------- packing ----

def test_pack_unpack_round_trip():
    g = np.random.default_rng(15)
    q = g.integers(0, 16, size=(24, 40)).astype(np.uint8)
    assert np.array_equal(oracle.unpack_kn8(oracle.pack_kn8(q), 24, 40), q)
    assert np.array_equal(oracle.unpack_ct(oracle.pack_ct(q), 40, 24), q)
    w = synth.words_uniform(g, (24, 5)).view(np.uint32)
    assert np.array_equal(oracle.pack_kn8(oracle.unpack_kn8(w, 24, 40)), w)
    # nibble j of word c is element 8c + j
    one = np.zeros((1, 16), np.uint8)
    one[0, 11] = 9
    assert oracle.pack_kn8(one)[0, 1] == 9 << (4 * 3)


def test_repack_tracks_every_single_nibble():
    K, N = 16, 16
    for k in range(K):
        for n in range(N):
            q = np.zeros((K, N), np.uint8)
            q[k, n] = 1 + (k + n) % 15
            ck = np.zeros((N, K // 8), np.uint32)
            ck[n, k // 8] = np.uint32(q[k, n]) << np.uint32(4 * (k % 8))   # checkpoint: along K
            kn = oracle.repack(ck, N, K)
            expect = np.zeros((K, N // 8), np.uint32)
            expect[k, n // 8] = np.uint32(q[k, n]) << np.uint32(4 * (n % 8))  # kernel: along N
            assert np.array_equal(kn, expect), (k, n)


def test_repack_round_trip_and_permutation():
    g = np.random.default_rng(16)
    for N, K in [(8, 8), (40, 24), (64, 128), (136, 72)]:
        ck = synth.words_uniform(g, (N, K // 8)).view(np.uint32)
        kn = oracle.repack(ck, N, K)
        assert kn.shape == (K, N // 8)
        assert np.array_equal(oracle.unrepack(kn, K, N), ck)
        nib = lambda w: np.sort(np.concatenate([(w >> np.uint32(4 * j)) & 15 for j in range(8)], axis=None))
        assert np.array_equal(nib(kn), nib(ck))


# ----------------------------------------------- checkpoint scales/zeros ----

def test_worked_ct_load(golden):
    d = golden("worked_ct_load.txt")
    N, K, G = int(d["N"][0]), int(d["K"][0]), int(d["G"][0])
    ng = K // G
    h16 = lambda hs: np.array([int(h, 16) for h in hs], np.uint16)
    s_ng = np.stack([h16(d[f"ct_scale_{n}"]) for n in range(N)])
    s_gn = np.stack([h16(d[f"scale_{g}"]) for g in range(ng)])
    z_ct = np.stack([_words(d[f"ct_zero_{c}"]) for c in range(N // 8)])
    z_gn = np.stack([_words(d[f"zero_{g}"]) for g in range(ng)])
    assert np.array_equal(oracle.ct_scales(s_ng, N, ng), s_gn)
    assert np.array_equal(oracle.ct_zeros(z_ct, N, ng), z_gn)
    # the fixture's own formula, read back through the kernel layout's unpacking
    z = oracle.unpack_kn8(z_gn, ng, N)
    gg, nn = np.meshgrid(np.arange(ng), np.arange(N), indexing="ij")
    assert np.array_equal(z, (3 * nn + 5 * gg) % 16)


def test_ct_load_tracks_every_single_element():
    N, ng = 16, 3
    for n in range(N):
        for g in range(ng):
            s = np.zeros((N, ng), np.uint16)
            s[n, g] = 0x3C00 + 7 * n + g
            expect = np.zeros((ng, N), np.uint16)
            expect[g, n] = s[n, g]
            assert np.array_equal(oracle.ct_scales(s, N, ng), expect), (n, g)
            v = np.uint32(1 + (n + g) % 15)
            z = np.zeros((N // 8, ng), np.uint32)
            z[n // 8, g] = v << np.uint32(4 * (n % 8))        # checkpoint: channel n in word n/8
            ez = np.zeros((ng, N // 8), np.uint32)
            ez[g, n // 8] = v << np.uint32(4 * (n % 8))       # kernel: row g, same nibble
            assert np.array_equal(oracle.ct_zeros(z, N, ng), ez), (n, g)


def test_ct_load_single_group_leaves_memory_unchanged():
    # K == G: [N, 1] and [1, N] (and [N/8, 1], [1, N/8]) are the same bytes
    g = np.random.default_rng(17)
    N = 40
    s = g.integers(0, 1 << 16, size=(N, 1), dtype=np.uint16)
    z = synth.words_uniform(g, (N // 8, 1)).view(np.uint32)
    assert np.array_equal(oracle.ct_scales(s, N, 1).ravel(), s.ravel())
    assert np.array_equal(oracle.ct_zeros(z, N, 1).ravel(), z.ravel())


@pytest.mark.parametrize("sym", [True, False])
def test_ct_load_preserves_the_dequantised_weight(sym):
    # W[k][n] = fp16((q - z) * s) taken straight from the checkpoint layout (element
    # by element, no oracle code) must equal the oracle GEMM of the identity matrix
    # on the converted layer.
    K, N, G = 48, 24, 16
    c = synth.ct_checkpoint(K, N, G, sym=sym, seed=5)
    ck, s_ng = c["ckpt"].view(np.uint32), c["s_ng"]
    z_ct = None if sym else c["z_n8g"].view(np.uint32)
    expect = np.zeros((K, N), np.float16)
    for k in range(K):
        for n in range(N):
            q = (int(ck[n, k // 8]) >> (4 * (k % 8))) & 15
            z = 8 if sym else (int(z_ct[n // 8, k // G]) >> (4 * (n % 8))) & 15
            expect[k, n] = np.float16(np.float32(q - z) * np.float32(s_ng[n, k // G]))
    b = oracle.repack(ck, N, K)
    s = oracle.ct_scales(s_ng.view(np.uint16), N, K // G).view(np.float16)
    zk = None if sym else oracle.ct_zeros(z_ct, N, K // G)
    eye = np.eye(K, dtype=np.float16)
    got = oracle.gemm(eye, b, s, zk, G, zp_bias=8)
    assert np.array_equal(got.astype(np.float32), expect.astype(np.float32))


def test_oracle_rejects_bad_sizes():
    with pytest.raises(ValueError):
        oracle.repack(np.zeros((4, 1), np.uint32), 4, 8)   # N % 8 != 0
