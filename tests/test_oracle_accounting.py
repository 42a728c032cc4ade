"""Pins for the storage accounting (CPU only).

BenQ: the card's bits/weight table (6.000 + 0.164 = 6.16) and its 28 GB -> 21 GB
packing remark.  MDBF: the page's b_eff, its inversion for the rank and the
b_max cap, checked against each other (b_max is b_eff at r = min(n, m)), against
bits counted in generated storage, and on the layer shapes the benchmarks use.
"""
import math
import warnings
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import accounting as acc

# 27B-class decoder layer (hidden 5120, intermediate 17408): (out, in) of q, k, v, o, gate, up, down
LAYER = [(5120, 5120), (1024, 5120), (1024, 5120), (5120, 5120), (17408, 5120), (17408, 5120), (5120, 17408)]


def test_benq_bits_per_weight_closed_form():
    assert acc.benq_bits_per_weight(5120) == pytest.approx(6.2)
    assert acc.benq_bits_per_weight(17408) == pytest.approx(6 + 1024 / 17408)
    assert acc.benq_bits_per_weight(17408) == pytest.approx(6.0588, abs=1e-4)


def test_benq_lut_share_matches_card_table():
    # parameter-weighted LUT share over a decoder layer's seven linears: the card prints 0.164
    # (amortised over 5120-17408 columns) for the whole model; the layer alone gives 0.1619
    params = sum(n * k for n, k in LAYER)
    lut_bits = sum(n * 64 * 16 for n, _ in LAYER)
    share = lut_bits / params
    assert share == pytest.approx(0.1619, abs=1e-4)
    assert abs(share - 0.164) < 0.003
    assert acc.benq_bits_per_weight(5120) - 6 >= share >= acc.benq_bits_per_weight(17408) - 6


def test_benq_packed_size_matches_card_28_to_21_gb():
    # the card: ~28 GB stored as raw uint8 codes, ~21 GB once packed to 6 bits
    assert acc.benq_packed_bytes_per_row(5120) / 5120 == 0.75
    assert 28 * 0.75 == 21
    w = synth.benq_weights(4, 512, seed=0)
    assert w.codes.shape == (4, acc.benq_packed_bytes_per_row(512))


def test_b_max_is_b_eff_at_full_rank():
    rng = np.random.default_rng(0)
    for _ in range(200):
        n, m = (int(v) for v in rng.integers(1, 20000, 2))
        P, l, sb = int(rng.integers(1, 3)), int(rng.integers(1, 17)), int(rng.integers(0, 33))
        assert acc.mdbf_b_max(n, m, P, l, sb) == acc.mdbf_b_eff(n, m, min(n, m), P, l, sb)


def test_halving_p_halves_the_ceiling():
    assert acc.mdbf_b_max(17408, 5120, 1, 4) * 2 == acc.mdbf_b_max(17408, 5120, 2, 4)


def test_square_layer_rank_2000_is_one_bit():
    # n = m = 4096, P = 1, l = 2, scale_bits = 16
    b = acc.mdbf_b_eff(4096, 4096, 2000, 1, 2, 16)
    assert b == Fraction(16774144, 16777216)
    assert float(b) == pytest.approx(0.999817, abs=1e-6)
    assert float(acc.mdbf_rank_real(4096, 4096, 1.0, 1, 2, 16)) == pytest.approx(2000.372, abs=1e-3)
    assert acc.mdbf_select_rank(4096, 4096, 1.0, 1, 2, 16) == (2000, False)
    assert acc.mdbf_b_max(4096, 4096, 1, 2) == Fraction(65, 32)          # 2.03125


def test_mlp_layers_at_one_and_a_half_bits():
    # gate/up (17408 x 5120) and down (5120 x 17408), P = 2, l = 4, target 1.5
    for n, m in ((17408, 5120), (5120, 17408)):
        r, clamped = acc.mdbf_select_rank(n, m, 1.5, 2, 4, 16)
        assert (r, clamped) == (2886, False)
        assert float(acc.mdbf_b_eff(n, m, r, 2, 4)) == pytest.approx(1.499558, abs=1e-6)
        assert float(acc.mdbf_b_max(n, m, 2, 4)) == pytest.approx(2.635294, abs=1e-6)


def test_rank_inversion_round_trip():
    rng = np.random.default_rng(1)
    for _ in range(300):
        n, m = (int(v) for v in rng.integers(64, 20000, 2))
        P, l, sb = int(rng.integers(1, 3)), int(rng.integers(1, 9)), int(rng.choice([0, 8, 16]))
        b = float(rng.uniform(0.3, 2.5))
        try:
            with warnings.catch_warnings():
                warnings.simplefilter("ignore")
                r, clamped = acc.mdbf_select_rank(n, m, b, P, l, sb)
        except ValueError:
            assert acc.mdbf_b_eff(n, m, 1, P, l, sb) > Fraction(b)
            continue
        if clamped:
            assert r == min(n, m) and acc.mdbf_b_max(n, m, P, l, sb) < Fraction(b)
        else:
            assert acc.mdbf_b_eff(n, m, r, P, l, sb) <= Fraction(b) < acc.mdbf_b_eff(n, m, r + 1, P, l, sb)


def test_target_above_b_max_is_clamped_with_warning():
    with pytest.warns(UserWarning, match="clamped"):
        r, clamped = acc.mdbf_select_rank(256, 4096, 2.5, 1, 2, 16)
    assert (r, clamped) == (256, True)
    assert float(acc.mdbf_b_max(256, 4096, 1, 2)) < 2.5


def test_scale_bits_zero_counts_signs_only():
    assert acc.mdbf_b_eff(300, 500, 40, 2, 4, 0) == Fraction(2 * 40 * 800, 300 * 500)


@pytest.mark.parametrize("shape", [(64, 96, 40, 2, 1), (128, 64, 24, 4, 2)])
def test_stored_bits_of_generated_layer_equal_b_eff(shape):
    n, m, r, l, P = shape
    paths = synth.mdbf_paths(P, n, m, r, l, seed=3, ldSA=r // 8, ldSB=m // 8)
    bits = 0
    for p in paths:
        bits += 8 * (p.S_A.nbytes + p.S_B.nbytes)
        bits += 8 * (p.A_amp.nbytes + p.B_amp.nbytes + p.Q_U.nbytes + p.Q_V.nbytes)
    assert Fraction(bits, n * m) == acc.mdbf_b_eff(n, m, r, P, l, 16)
    assert math.isclose(bits / (n * m), float(acc.mdbf_b_eff(n, m, r, P, l, 16)))
