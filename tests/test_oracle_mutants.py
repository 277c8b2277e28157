"""Planted mistakes: each one is applied to a COPY of the oracle's C source, compiled
on the CPU, and must make at least one pin of test_oracle.py fail.

This shows the pins are strong enough to catch a dropped term, a wrong sign, a
wrong group or nibble index, a transposed repack, ignored zeros and a wrong
rounding mode.
"""
import os
import subprocess

import pytest

import oracle
import test_oracle as T
from conftest import read_golden

MUTANTS = {
    "sign_flip": ("w[k * ncols + i] = (float)(q - zz) * sc;", "w[k * ncols + i] = (float)(zz - q) * sc;"),
    "group_index": ("int64_t g = k / G;                                       /* step 3 */",
                    "int64_t g = k % (K / G);"),
    "nibble_order": ("int q = nibble(b[k * (N / 8) + n / 8], (int)(n % 8)); /* step 1 */",
                     "int q = nibble(b[k * (N / 8) + n / 8], (int)(7 - n % 8));"),
    "dropped_term": ("for (int64_t i = 0; i < ncols; ++i) row[i] = row[i] + ak * wk[i];",
                     "if (k + 1 < K) for (int64_t i = 0; i < ncols; ++i) row[i] = row[i] + ak * wk[i];"),
    "repack_transposed": ("q[k * N + n] = nibble(ckpt[n * (K / 8) + k / 8], (int)(k % 8));",
                          "q[k * N + n] = nibble(ckpt[n * (K / 8) + k / 8], (int)(7 - k % 8));"),
    "zeros_ignored": ("int zz = z ? nibble(z[g * (N / 8) + n / 8], (int)(n % 8)) : zp_bias;",
                      "int zz = zp_bias;"),
    "round_half_down": ("if (rem > halfway || (rem == halfway && (keep & 1))) keep += 1;",
                        "if (rem > halfway) keep += 1;"),
    "ct_zero_nibble": ("z[n * ngroups + g] = nibble(z_n8g[(n / 8) * ngroups + g], (int)(n % 8));",
                       "z[n * ngroups + g] = nibble(z_n8g[(n / 8) * ngroups + g], (int)(7 - n % 8));"),
    "ct_zero_word": ("z[n * ngroups + g] = nibble(z_n8g[(n / 8) * ngroups + g], (int)(n % 8));",
                     "z[n * ngroups + g] = nibble(z_n8g[(n / 8) + g * (N / 8)], (int)(n % 8));"),
    "ct_scales_untransposed": ("s_gn[g * N + n] = s_ng[n * ngroups + g];", "s_gn[g * N + n] = s_ng[g * N + n];"),
    "scale_of_wrong_group": ("float sc = oracle_half_to_float(s[g * N + n]);",
                             "float sc = oracle_half_to_float(s[n]);"),
}


def _pins():
    g = read_golden
    yield "half_encode", T.test_half_encode_rne
    yield "worked_gemm", lambda: T.test_worked_gemm_symmetric_and_asymmetric(g)
    yield "worked_repack", lambda: T.test_worked_repack(g)
    for args in [(3, 32, 16, 16), (2, 16, 24, 16)]:
        for sym in (True, False):
            yield f"brute{args}{sym}", (lambda a=args, s=sym: T.test_brute_force_tiny(*a, s))
    yield "q_eq_z", T.test_q_equals_z_gives_zero
    yield "integer_matmul", T.test_integer_matmul_special_case
    yield "repack_single", T.test_repack_tracks_every_single_nibble
    yield "worked_ct_load", lambda: T.test_worked_ct_load(g)
    yield "ct_single", T.test_ct_load_tracks_every_single_element
    for sym in (True, False):
        yield f"ct_dense{sym}", (lambda s=sym: T.test_ct_load_preserves_the_dequantised_weight(s))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = open(oracle._SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not found once"
    path_c = tmp_path / "mut.c"
    path_c.write_text(src.replace(old, new))
    so = str(tmp_path / "libmut.so")
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(path_c), "-o", so])
    saved = oracle._lib
    oracle._lib = oracle.load(so)
    caught = []
    try:
        for pin, fn in _pins():
            try:
                fn()
            except (AssertionError, ValueError):
                caught.append(pin)
    finally:
        oracle._lib = saved
    assert caught, f"no pin caught the planted mistake {name}"


def test_unmutated_passes_all_pins():
    for pin, fn in _pins():
        fn()
