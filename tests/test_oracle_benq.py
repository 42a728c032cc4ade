"""Pins for the BenQ oracle (CPU only).

Each test ties ``oracle.benq`` to something other than itself: a worked
example derived by hand from the BenQ card's definitions, an exhaustive
bijection with the (independent) generator packing, torch's gather (the card
defines decode as ``lut.gather(1, codes)``), or exact rational arithmetic.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth
from oracle import benq as ob


def _f32_of_bf16(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def test_unpack_matches_hand_worked_stream(golden):
    g = golden("benq_pack_example.txt")
    codes = np.array([int(c) for c in g["codes"]])
    packed = np.array([[int(b, 16) for b in g["bytes"]]], dtype=np.uint8)
    assert ob.unpack_codes(packed, 8).tolist() == [codes.tolist()]


def test_generator_pack_matches_hand_worked_stream(golden):
    g = golden("benq_pack_example.txt")
    codes = np.array([[int(c) for c in g["codes"]]], dtype=np.uint8)
    assert synth.pack_codes(codes).tolist() == [[int(b, 16) for b in g["bytes"]]]


def test_pack_unpack_bijection_all_code_groups():
    # every one of the 64^4 groups of four codes survives pack -> unpack
    c = np.arange(64 ** 4, dtype=np.int64)
    groups = np.stack([(c >> (6 * j)) & 63 for j in range(4)], axis=1).astype(np.uint8)
    packed = synth.pack_codes(groups.reshape(1, -1))
    back = ob.unpack_codes(packed, groups.size).reshape(-1, 4)
    assert np.array_equal(back, groups)


def test_unpack_pack_bijection_all_byte_triples():
    # every one of the 2^24 three-byte strings survives unpack -> pack
    v = np.arange(1 << 24, dtype=np.uint32)
    triples = np.stack([(v >> 8 * j) & 255 for j in range(3)], axis=1).astype(np.uint8)
    codes = ob.unpack_codes(triples.reshape(1, -1), 4 * (1 << 24))
    again = synth.pack_codes(codes.astype(np.uint8))
    assert np.array_equal(again.reshape(-1, 3), triples)


def test_unpack_ignores_bytes_past_the_row():
    rng = np.random.default_rng(0)
    packed = rng.integers(0, 256, size=(3, 24), dtype=np.uint8)
    wide = np.concatenate([packed, rng.integers(0, 256, size=(3, 16), dtype=np.uint8)], axis=1)
    assert np.array_equal(ob.unpack_codes(packed, 32), ob.unpack_codes(wide, 32))


def test_dequant_is_torch_gather():
    rng = np.random.default_rng(1)
    N, K = 37, 96
    codes = rng.integers(0, 64, size=(N, K), dtype=np.uint8)
    lut = rng.integers(0, 1 << 16, size=(N, 64), dtype=np.uint16)
    packed = synth.pack_codes(codes)
    ref = torch.gather(torch.from_numpy(lut.astype(np.int32)), 1, torch.from_numpy(codes.astype(np.int64)))
    assert np.array_equal(ob.dequant_bits(packed, lut, K), ref.numpy().astype(np.uint16))


def test_linear_hand_worked_example(golden):
    g = golden("benq_linear_example.txt")
    c = np.array([[int(v) for v in g["codes0"]], [int(v) for v in g["codes1"]]], dtype=np.uint8)
    lut0 = np.array([(2 * k - 63) / 32 for k in range(64)], dtype=np.float32)
    lut1 = np.array([-(2 * k - 63) / 64 for k in range(64)], dtype=np.float32)
    lut = synth.f32_to_bf16_bits(np.stack([lut0, lut1]))
    assert np.array_equal(_f32_of_bf16(lut), np.stack([lut0, lut1]))    # exact in bf16
    x = synth.f32_to_bf16_bits(np.array([[float(v) for v in g["x"]]], dtype=np.float32))
    y = ob.linear(synth.pack_codes(c), lut, x, 4)
    assert y.tolist() == [[float(v) for v in g["y"]]]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_linear_exact_rational_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    N, K, B = 3, 8, 2
    codes = rng.integers(0, 64, size=(N, K), dtype=np.uint8)
    lut = synth.f32_to_bf16_bits(rng.standard_normal((N, 64)).astype(np.float32))
    x = synth.f32_to_bf16_bits(rng.standard_normal((B, K)).astype(np.float32))
    y = ob.linear(synth.pack_codes(codes), lut, x, K)
    L = _f32_of_bf16(lut)
    X = _f32_of_bf16(x)
    for b in range(B):
        for n in range(N):
            exact = sum(Fraction(float(L[n, codes[n, k]])) * Fraction(float(X[b, k])) for k in range(K))
            bound = sum(abs(Fraction(float(L[n, codes[n, k]])) * Fraction(float(X[b, k]))) for k in range(K))
            assert abs(Fraction(y[b, n]) - exact) <= bound * Fraction(K, 2 ** 52)


def test_linear_row_subset_matches_full():
    w = synth.benq_weights(64, 128, seed=7)
    x = synth.activations(3, 128, seed=8)
    full = ob.linear(w.codes, w.lut, x, 128)
    rows = np.array([0, 5, 63, 17])
    assert np.array_equal(ob.linear(w.codes, w.lut, x, 128, rows=rows), full[:, rows])


# ---------------------------------------------------------------- gated MLP (gate, up) of the oracle

def test_silu_fixed_points_and_identities():
    # silu(0) = 0; silu(v) - silu(-v) = v (sigmoid(v) + sigmoid(-v) = 1); sigmoid(ln 3) = 3/4
    v = np.array([-30.0, -4.5, -1.0, -1e-3, 0.0, 1e-3, 0.7, 3.0, 40.0, 700.0])
    s = ob.silu(v)
    assert s[4] == 0.0
    assert np.allclose(s - ob.silu(-v), v, rtol=1e-15, atol=1e-15)
    assert abs(ob.silu(np.log(3.0)) - 0.75 * np.log(3.0)) < 1e-15
    # for large v the gate passes v through; for very negative v it vanishes from below
    assert ob.silu(700.0) == 700.0 and -1e-250 < ob.silu(-700.0) < 0.0
    # minimum of silu: v* solves 1 + v(1 - sigmoid(v)) = 0, v* ~ -1.2784645, silu(v*) ~ -0.2784645
    grid = np.linspace(-3, 0, 300001)
    assert abs(ob.silu(grid).min() - (-0.27846454276)) < 1e-9


def test_mlp_gate_up_exact_rational_brute_force():
    # tiny layer: h[b, n] = silu(sum_k Wg x) * sum_k Wu x with the sums in exact rationals and the
    # gate from the math library on the exact sum
    import math
    K, N = 8, 3
    wg = synth.benq_weights(N, K, seed=41)
    wu = synth.benq_weights(N, K, seed=42)
    x = synth.activations(2, K, seed=43)
    h = ob.mlp_gate_up(wg.codes, wg.lut, wu.codes, wu.lut, x, K)
    codes_g = ob.unpack_codes(wg.codes, K)
    codes_u = ob.unpack_codes(wu.codes, K)
    for b in range(2):
        for n in range(N):
            g = sum(Fraction(float(_f32_of_bf16(wg.lut[n, codes_g[n, k]]))) * Fraction(float(_f32_of_bf16(x[b, k])))
                    for k in range(K))
            u = sum(Fraction(float(_f32_of_bf16(wu.lut[n, codes_u[n, k]]))) * Fraction(float(_f32_of_bf16(x[b, k])))
                    for k in range(K))
            gf = float(g)
            ref = gf / (1.0 + math.exp(-gf)) * float(u)
            assert abs(h[b, n] - ref) <= 1e-15 * max(1.0, abs(ref))


def test_mlp_gate_up_row_subset_matches_full():
    K, N = 64, 40
    wg = synth.benq_weights(N, K, seed=51)
    wu = synth.benq_weights(N, K, seed=52)
    x = synth.activations(3, K, seed=53)
    full = ob.mlp_gate_up(wg.codes, wg.lut, wu.codes, wu.lut, x, K)
    rows = np.array([0, 7, 39])
    assert np.array_equal(ob.mlp_gate_up(wg.codes, wg.lut, wu.codes, wu.lut, x, K, rows=rows), full[:, rows])


# --------------------------------------------------------------------------- encoder of the oracle

def _bits(v):
    return synth.f32_to_bf16_bits(np.asarray(v, dtype=np.float32))


def test_encode_hand_worked_row():
    # one row, K = 8, dyadic values (exact at every step): max|w| = 3 -> shell width D = 3/32.
    # |w| / D: 3 -> 32 (tier 31), 0.0625 -> 0.67 (0), 0.25 -> 2.67 (2), 0 (0), 1 -> 10.67 (10),
    # 0.046875 -> 0.5 (0).  Levels: tier 31 = mean(3, 3) = 3, tier 2 = 0.25, tier 10 = 1, tier 0 =
    # mean(0.0625, 0, 0.046875) = 0.036458.. rounded to bf16, empty tiers at their shell midpoints
    # (t + 1/2) D, e.g. tier 5 = 0.515625 (exact in bf16).
    w = np.array([[3.0, 0.0625, -0.25, 0.0, 1.0, 0.25, -3.0, 0.046875]], dtype=np.float32)
    packed, lut = ob.encode(_bits(w))
    L = ob.bf16_to_f32(lut[0, 32:]).astype(np.float64)
    assert L[31] == 3.0 and L[2] == 0.25 and L[10] == 1.0 and L[5] == 0.515625 and L[1] == 0.140625
    assert L[0] == float(ob.bf16_to_f32(_bits(np.float32(0.109375 / 3)).reshape(1))[0])
    assert ob.unpack_codes(packed, 8)[0].tolist() == [63, 32, 29, 32, 42, 34, 0, 32]
    assert np.array_equal(lut[0, :32], lut[0, 32:][::-1] | np.uint16(0x8000))


def test_encode_exact_tie_takes_the_lower_level():
    # max|w| = 3 -> D = 3/32.  Tier 8 = [0.75, 0.84375) holds 0.75, 0.8125 and 0.828125, so its level
    # is their mean 51/64 = 0.796875; tier 7 is empty and sits at its midpoint 7.5 D = 45/64.  The
    # magnitude 0.75 is 3/64 from both levels (every value here is exact in bf16 and fp64): an exact
    # tie, which goes to the lower tier (code 32 + 7), not its own shell (32 + 8).  The other codes
    # are 63 (tier 31), 40, 40 and 32 for the zeros (tier 0, level 0).
    w = np.array([[3.0, 0.75, 0.8125, 0.828125, 0.0, 0.0, 0.0, 0.0]], dtype=np.float32)
    packed, lut = ob.encode(_bits(w))
    L = ob.bf16_to_f32(lut[0, 32:]).astype(np.float64)
    assert L[8] == 0.796875 and L[7] == 0.703125 and L[0] == 0.0 and L[31] == 3.0
    assert abs(0.75 - L[7]) == abs(0.75 - L[8])
    assert ob.unpack_codes(packed, 8)[0].tolist() == [63, 39, 40, 40, 32, 32, 32, 32]


def test_encode_table_is_sorted_and_codes_are_nearest():
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((6, 256)) * rng.uniform(0.01, 0.05, size=(6, 1))).astype(np.float32)
    wb = _bits(w)
    for iters in (0, 3):
        packed, lut = ob.encode(wb, iters)
        vals = ob.bf16_to_f32(lut).astype(np.float64)
        assert np.all(np.diff(vals, axis=1) >= 0)                         # ascending value
        assert np.all(vals[:, :32] <= 0) and np.all(vals[:, 32:] >= 0)
        W = ob.dequant(packed, lut, 256).astype(np.float64)
        a = ob.bf16_to_f32(wb).astype(np.float64)
        # every weight decodes to a level of its own sign at minimum distance among all 64 entries
        # whose sign matches (zero counts as non-negative)
        d = np.abs(a[:, :, None] - vals[:, None, :])
        sign_ok = np.where(a[:, :, None] < 0, vals[:, None, :] <= 0, vals[:, None, :] >= 0)
        dmin = np.where(sign_ok, d, np.inf).min(axis=2)
        assert np.array_equal(np.abs(a - W), dmin)


def test_lloyd_rounds_do_not_increase_the_error():
    # each Lloyd round (nearest assignment, then member means) cannot increase the squared error of
    # the magnitudes beyond what rounding the levels to bf16 adds back
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((4, 2048)) * 0.02).astype(np.float32)
    wb = _bits(w)
    a = np.abs(ob.bf16_to_f32(wb).astype(np.float64))
    errs = []
    for iters in range(4):
        packed, lut = ob.encode(wb, iters)
        errs.append(((np.abs(ob.dequant(packed, lut, 2048).astype(np.float64)) - a) ** 2).sum())
    assert errs[3] <= errs[0] * (1 + 1e-3)
    assert min(errs[1:]) < errs[0]


def test_encode_pack_matches_generator_packing():
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 64, size=(5, 64), dtype=np.uint8)
    assert np.array_equal(ob.pack(codes), synth.pack_codes(codes))
    assert np.array_equal(ob.unpack_codes(ob.pack(codes), 64), codes)


def test_encode_all_zero_row_and_signed_zero():
    wb = np.zeros((2, 8), dtype=np.uint16)
    wb[1, 3] = 0x8000                      # -0.0 counts as non-negative
    wb[1, 5] = _bits(np.array([0.5], dtype=np.float32))[0]
    packed, lut = ob.encode(wb)
    codes = ob.unpack_codes(packed, 8)
    assert codes[0].tolist() == [32] * 8 and np.all(lut[0, 32:] == 0)
    assert codes[1, 3] >= 32 and codes[1, 5] == 63
