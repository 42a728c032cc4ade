"""Planted mistakes in the oracle must each fail at least one pin (CPU only).

Each mutant replaces one oracle function with a plausible wrong version (bit
order, sign convention, dropped envelope term, transposed operand, off-by-one
in the accounting) and re-runs the pins; a mutant that no pin catches would
mean the pins do not actually constrain that part of the oracle.
"""
import numpy as np
import pytest

import tests.test_oracle_accounting as ta
import tests.test_oracle_benq as tb
import tests.test_oracle_mdbf as tm
from oracle import accounting as acc
from oracle import benq as ob
from oracle import mdbf as om
from tests.conftest import read_golden

_orig_unpack_codes = ob.unpack_codes
_orig_unpack_signs = om.unpack_signs
_orig_envelope = om.envelope


def _unpack_msb_first(packed, K):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    bits = np.unpackbits(packed[:, :6 * K // 8], axis=1, bitorder="little")
    fields = bits.reshape(packed.shape[0], K, 6).astype(np.int64)
    return fields @ np.array([32, 16, 8, 4, 2, 1])


def _unpack_big_endian_bytes(packed, K):
    p = np.ascontiguousarray(packed, dtype=np.uint8)[:, :3 * K // 4]
    p = p.reshape(p.shape[0], -1, 3)[:, :, ::-1].reshape(p.shape[0], -1)
    return _orig_unpack_codes(p, K)


def _dequant_reversed_table(packed, lut_bits, K):
    return np.take_along_axis(np.asarray(lut_bits, np.uint16), 63 - _orig_unpack_codes(packed, K), axis=1)


def _signs_flipped(packed, cols):
    return (-_orig_unpack_signs(packed, cols)).astype(np.int8)


def _signs_msb_first(packed, cols):
    bits = np.unpackbits(np.ascontiguousarray(packed, np.uint8), axis=1, bitorder="big")
    return (bits[:, :cols].astype(np.int8) * 2 - 1).astype(np.int8)


def _envelope_first_term_only(L, R):
    return _orig_envelope(L[:, :1], R[:, :1])


def _envelope_reversed_columns(L, R):
    return _orig_envelope(L, R[:, ::-1])


def _factors_swapped_qu_qv(path, n, m, r):
    F = (_orig_unpack_signs(path.S_A, r) * _orig_envelope(path.A_amp, path.Q_V)).astype(np.float32)
    G = (_orig_unpack_signs(path.S_B, m) * _orig_envelope(path.Q_U, path.B_amp)).astype(np.float32)
    return F, G


def _silu_sign_flipped(v):
    v = np.asarray(v, dtype=np.float64)
    return v / (1.0 + np.exp(np.clip(v, -700, 700)))     # v * sigmoid(-v)


def _mlp_gate_and_up_swapped(pg, lg, pu, lu, x, K, rows=None):
    return ob.silu(ob.linear(pu, lu, x, K, rows)) * ob.linear(pg, lg, x, K, rows)


_orig_shell_levels = ob._shell_levels


def _shell_levels_midpoints(a, tier, prev):
    return _orig_shell_levels(np.zeros_like(a), tier, prev) * 0 + prev      # ignores the members


def _encode_width_over_31(w_bits, lloyd_iters=0):
    w = ob.bf16_to_f32(np.asarray(w_bits, np.uint16)).astype(np.float64)
    scaled = ob._bf16_rne_of_f32((w * (32.0 / 31.0)).astype(np.float32))     # tiers of max/31 shells
    return _orig_encode(scaled, lloyd_iters)


_orig_encode = ob.encode


def _encode_signs_swapped(w_bits, lloyd_iters=0):
    packed, lut = _orig_encode(w_bits, lloyd_iters)          # 32 + t for w < 0, 31 - t for w >= 0
    K = 4 * packed.shape[1] // 3
    return ob.pack(63 - ob.unpack_codes(packed, K).astype(np.int64)), lut


def _nearest_upper_on_tie(a, levels):
    d = np.abs(a[:, None] - levels[None, :])
    return levels.shape[0] - 1 - np.argmin(d[:, ::-1], axis=1)   # the last (upper) index of a tie


def _b_eff_without_2r(n, m, r, P, l, scale_bits=16):
    from fractions import Fraction
    return Fraction(P * (r * (n + m) + scale_bits * l * (n + m)), n * m)


BENQ_PINS = [
    lambda: tb.test_unpack_matches_hand_worked_stream(read_golden),
    lambda: tb.test_linear_hand_worked_example(read_golden),
    tb.test_pack_unpack_bijection_all_code_groups,
    tb.test_dequant_is_torch_gather,
]
MDBF_PINS = [
    lambda: tm.test_sign_unpack_hand_worked(read_golden),
    lambda: tm.test_dequant_and_linear_hand_worked(read_golden),
    lambda: tm.test_dequant_exact_rational_dyadic((3, 4, 2, 2, 1)),
    lambda: tm.test_dequant_exact_rational_dyadic((2, 5, 3, 2, 2)),
]
MLP_PINS = [tb.test_silu_fixed_points_and_identities, tb.test_mlp_gate_up_exact_rational_brute_force]
ENC_PINS = [tb.test_encode_hand_worked_row, tb.test_encode_table_is_sorted_and_codes_are_nearest,
            tb.test_lloyd_rounds_do_not_increase_the_error, tb.test_encode_exact_tie_takes_the_lower_level]
ACC_PINS = [ta.test_square_layer_rank_2000_is_one_bit, ta.test_mlp_layers_at_one_and_a_half_bits,
            ta.test_b_max_is_b_eff_at_full_rank,
            lambda: ta.test_stored_bits_of_generated_layer_equal_b_eff((64, 96, 40, 2, 1))]

MUTANTS = [
    ("benq: 6-bit field read MSB first", ob, "unpack_codes", _unpack_msb_first, BENQ_PINS),
    ("benq: 3-byte group read big-endian", ob, "unpack_codes", _unpack_big_endian_bytes, BENQ_PINS),
    ("benq: table indexed from the top", ob, "dequant_bits", _dequant_reversed_table, BENQ_PINS),
    ("mdbf: bit 1 read as -1", om, "unpack_signs", _signs_flipped, MDBF_PINS),
    ("mdbf: signs packed MSB first", om, "unpack_signs", _signs_msb_first, MDBF_PINS),
    ("mdbf: envelope keeps only its first term", om, "envelope", _envelope_first_term_only, MDBF_PINS),
    ("mdbf: envelope columns misaligned", om, "envelope", _envelope_reversed_columns, MDBF_PINS),
    ("mdbf: Q_U and Q_V swapped", om, "factors", _factors_swapped_qu_qv, MDBF_PINS),
    ("accounting: b_eff without the 2r envelope term", acc, "mdbf_b_eff", _b_eff_without_2r, ACC_PINS),
    ("mlp: gate uses sigmoid(-v)", ob, "silu", _silu_sign_flipped, MLP_PINS),
    ("encoder: levels are shell midpoints, not member means", ob, "_shell_levels", _shell_levels_midpoints, ENC_PINS),
    ("encoder: shells of max/31", ob, "encode", _encode_width_over_31, ENC_PINS),
    ("encoder: code signs swapped", ob, "encode", _encode_signs_swapped, ENC_PINS),
    ("encoder: exact ties go to the upper level", ob, "_nearest", _nearest_upper_on_tie, ENC_PINS),
    ("mlp: gate applied to the up projection", ob, "mlp_gate_up", _mlp_gate_and_up_swapped, MLP_PINS),
]


@pytest.mark.parametrize("name,mod,attr,fn,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(monkeypatch, name, mod, attr, fn, pins):
    monkeypatch.setattr(mod, attr, fn)
    caught = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught >= 1, f"no pin catches: {name}"
