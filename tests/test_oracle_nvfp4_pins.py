"""Pins of the oracle's NVFP4 decoding (reading R22): the format's value table,
a hand-worked row (tests/golden/nvfp4_example.json), and the factored form of a
score (sum over 16-element groups of scale x scale x the e2m1 dot product),
written out with explicit nibble loops, against the decoded dot product.  A
planted mistake (nibble order, group size, scale bias, the e2m1 subnormal)
fails at least one pin."""
import json
import math
import os

import numpy as np
import pytest

from oracle import msa_oracle as O

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "nvfp4_example.json")

# the sixteen e2m1 values in code order (the format's table)
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def test_e2m1_table():
    got = [O.e2m1_value(c) for c in range(16)]
    assert got == E2M1_TABLE
    assert [math.copysign(1, v) for v in got[8:]] == [-1.0] * 8


def test_ue4m3_points_and_nan():
    d = json.load(open(GOLD))
    for code, val in d["ue4m3_points"].items():
        assert O.ue4m3_value(int(code)) == val, code
    assert math.isnan(O.ue4m3_value(0x7F))
    assert math.isnan(O.ue4m3_value(0x80))
    # monotone over the valid codes: a larger code is a larger scale
    vals = [O.ue4m3_value(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))


def test_golden_row():
    d = json.load(open(GOLD))
    got = O.nvfp4_decode(np.array([d["codes"]], dtype=np.uint8),
                         np.array([d["scales"]], dtype=np.uint8))[0]
    np.testing.assert_array_equal(got, np.array(d["values"]))
    # the signed zeros are where the hand-worked row puts them
    assert [math.copysign(1, v) for v in got[[7, 15, 22]]] == [-1.0, 1.0, -1.0]


def _factored_score(qc, qs, kc, ks):
    """sum over groups g of scale_q[g] * scale_k[g] * sum_{j in g} e(q_j) e(k_j),
    element j read as nibble (j % 2) of byte j // 2, by explicit loops."""
    total = 0.0
    for g in range(len(qs)):
        part = 0.0
        for j in range(16 * g, 16 * g + 16):
            byte_q, hi = divmod(j, 2)
            nq = (int(qc[byte_q]) >> (4 * hi)) & 15
            nk = (int(kc[byte_q]) >> (4 * hi)) & 15
            part += O.e2m1_value(nq) * O.e2m1_value(nk)
        total += O.ue4m3_value(int(qs[g])) * O.ue4m3_value(int(ks[g])) * part
    return total


@pytest.mark.parametrize("di", [32, 64, 128])
def test_decoded_scores_equal_the_factored_form(di):
    rng = np.random.default_rng(di)
    n = 40
    qc = rng.integers(0, 256, (di // 2,), dtype=np.uint8)
    qs = rng.integers(0x20, 0x48, (di // 16,), dtype=np.uint8)
    kc = rng.integers(0, 256, (n, di // 2), dtype=np.uint8)
    ks = rng.integers(0x20, 0x48, (n, di // 16), dtype=np.uint8)
    q = O.nvfp4_decode(qc[None], qs[None])
    k = O.nvfp4_decode(kc, ks)
    s = O.index_scores_row(q, k, n - 1)[:, 0]
    want = np.array([_factored_score(qc, qs, kc[j], ks[j]) for j in range(n)])
    np.testing.assert_array_equal(s, want)  # dyadic values: exact in fp64


def _pins_pass():
    try:
        test_golden_row()
        for di in (32, 64, 128):
            test_decoded_scores_equal_the_factored_form(di)
        test_ue4m3_points_and_nan()
        test_e2m1_table()
    except AssertionError:
        return False
    return True


MUTANTS = ["nibble_order", "group_32", "scale_bias_8", "e2m1_subnormal_one"]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_planted_nvfp4_mistakes_are_caught(mutant, monkeypatch):
    if mutant == "nibble_order":
        real = O.nvfp4_decode

        def swapped(codes, scales):
            c = np.asarray(codes).astype(np.uint8)
            return real(((c & 15) << 4) | (c >> 4), scales)
        monkeypatch.setattr(O, "nvfp4_decode", swapped)
    elif mutant == "group_32":
        def g32(codes, scales):
            c = np.asarray(codes).astype(np.int64)
            sc = np.asarray(scales).astype(np.int64)
            d = c.shape[-1] * 2
            nib = np.empty(c.shape[:-1] + (d,), dtype=np.int64)
            nib[..., 0::2], nib[..., 1::2] = c & 15, (c >> 4) & 15
            e = np.array([O.e2m1_value(i) for i in range(16)])[nib]
            s = np.array([O.ue4m3_value(i) for i in range(256)])[sc]
            s32 = np.repeat(s[..., ::2], 32, axis=-1)[..., :d]
            return e * s32
        monkeypatch.setattr(O, "nvfp4_decode", g32)
    elif mutant == "scale_bias_8":
        real = O.ue4m3_value
        monkeypatch.setattr(O, "ue4m3_value", lambda c: real(c) / 2)
    elif mutant == "e2m1_subnormal_one":
        real = O.e2m1_value
        monkeypatch.setattr(O, "e2m1_value",
                            lambda c: (-1.0 if c & 8 else 1.0) if (c & 7) == 1 else real(c))
    assert not _pins_pass(), f"planted mistake '{mutant}' passed every pin"
