"""MDBF parity for batches past the decode kernels (l * B > 64): the tensor-core path.

y = X W^T with W = sum_p F_p G_p ("MDBF (Multi-Envelope Double Binary Factorization)",
section "Algorithm") evaluated as T = X G^T and Y = T F^T, with each factor element rebuilt in
fp16 inside the GEMM that consumes it.  Bar: max |y - y_ref| / max |y_ref| per batch row
<= 5e-3 against the oracle's fp64 result on the same seeded inputs, bf16 output equal to the
round-to-nearest-even of the fp32 output, and identical results from repeated calls.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import mdbf as om
from tests.qlhelpers import MDBF_TOL, bf16, f32_to_bf16_rne, max_rel, mdbf_dev_paths

pytestmark = pytest.mark.gpu


def _linear(ql, paths, n, m, r, l, xbits, ydtype=torch.float32):
    B = xbits.shape[0]
    dp = mdbf_dev_paths(paths)
    ws = torch.empty(ql.mdbf_workspace_bytes(len(paths), n, m, r, l, B), dtype=torch.uint8, device="cuda")
    y = torch.empty(B, n, dtype=ydtype, device="cuda")
    ql.mdbf_linear(dp, n, m, r, l, bf16(xbits), y, ws)
    ql.ql_check()
    return y


def _scaled_envelope(bits: np.ndarray, scale: float) -> np.ndarray:
    """fp16 envelope bits times a power of two (exact in fp16 for these magnitudes)."""
    v = bits.view(np.float16).astype(np.float32) * np.float32(scale)
    assert np.all(np.isfinite(v.astype(np.float16)))
    return v.astype(np.float16).view(np.uint16)


# (n, m, r, l, P, B): several 512 x 256 output tiles with ragged edges in every dimension, odd l
# (no paired envelope loads), l > 16 (two envelope chunks), three paths, more than one 512-row
# tile of tokens, the smallest layer the tensor cores take (n = m = r = 64) and the smallest
# batch past the decode kernels' limit.
SHAPES = [
    (1024, 1024, 512, 1, 1, 300),     # l = 1, P = 1 (DBF) on the tensor cores
    (512, 768, 256, 1, 2, 129),       # l = 1, P = 2 (LittleBit)
    (256, 512, 200, 4, 2, 40),
    (300, 200, 100, 3, 2, 70),
    (512, 1024, 256, 4, 1, 600),
    (1000, 777, 300, 2, 3, 97),
    (64, 64, 64, 17, 1, 8),
    (130, 70, 64, 32, 2, 3),
    (96, 1000, 95, 2, 1, 33),
]


@pytest.mark.parametrize("n,m,r,l,P,B", SHAPES)
def test_batched_shapes(ql, n, m, r, l, P, B):
    paths = synth.mdbf_paths(P, n, m, r, l, seed=7 * n + m + r)
    x = synth.activations(B, m, seed=B + n)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert max_rel(y, om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL
    yb = _linear(ql, paths, n, m, r, l, x, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(yb, f32_to_bf16_rne(y))


@pytest.mark.parametrize("n,m,r,l,P,B", [(40, 24, 20, 40, 1, 3), (70, 90, 50, 33, 2, 5), (5, 9, 3, 1, 1, 65),
                                         (63, 200, 63, 4, 2, 40), (100, 200, 63, 2, 1, 70), (256, 63, 32, 8, 2, 20)])
def test_batched_small_layers_run_in_batch_chunks(ql, n, m, r, l, P, B):
    # l > 32, or n, m or r below 64, with l * B > 64: the batch goes through the decode kernels
    # 64 / l rows at a time
    paths = synth.mdbf_paths(P, n, m, r, l, seed=n + l)
    x = synth.activations(B, m, seed=l)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert max_rel(y, om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL


def test_batched_repeated_calls_are_identical(ql):
    n, m, r, l, P, B = 2048, 1024, 700, 4, 2, 1100
    paths = synth.mdbf_paths(P, n, m, r, l, seed=99)
    x = synth.activations(B, m, seed=5)
    y0 = _linear(ql, paths, n, m, r, l, x)
    for _ in range(3):
        assert torch.equal(_linear(ql, paths, n, m, r, l, x), y0)
    sel = np.arange(0, B, 37)
    ref = om.linear_factored(paths, n, m, r, x[sel])
    assert max_rel(y0.cpu().numpy()[sel], ref) <= MDBF_TOL


def test_batched_activation_range(ql):
    # Rows whose bf16 values lie far outside fp16's range (1e6 and 1e-9 in magnitude), a zero row
    # and ordinary rows: each row is rescaled by a power of two before the fp16 contraction.
    n, m, r, l, P, B = 384, 640, 256, 4, 2, 24
    paths = synth.mdbf_paths(P, n, m, r, l, seed=21)
    xf = synth.bf16_bits_to_f32(synth.activations(B, m, seed=22)).astype(np.float32)
    xf[0] *= np.float32(2.0 ** 20)
    xf[1] *= np.float32(2.0 ** -30)
    xf[2] = 0.0
    xf[3, ::7] *= np.float32(2.0 ** 12)       # one row with a wide spread inside itself
    x = synth.f32_to_bf16_bits(xf)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert np.all(np.isfinite(y))
    assert np.all(y[2] == 0.0)
    keep = [b for b in range(B) if b != 2]
    assert max_rel(y[keep], om.linear_factored(paths, n, m, r, x[keep])) <= MDBF_TOL


def test_batched_large_envelopes(ql):
    # Envelopes 2^10 times larger push the bound on T' = X' G^T past fp16's range unless the
    # activations are scaled down as well (the e > 0 branch of the activation prep).
    n, m, r, l, P, B = 512, 4096, 512, 4, 2, 32
    paths = synth.mdbf_paths(P, n, m, r, l, seed=31)
    for p in paths:
        p.B_amp = _scaled_envelope(p.B_amp, 1024.0)
        p.Q_V = _scaled_envelope(p.Q_V, 4.0)
    x = synth.activations(B, m, seed=32)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert np.all(np.isfinite(y))
    assert max_rel(y, om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL


@pytest.mark.parametrize("which", ["G", "F", "both"])
def test_batched_factors_past_fp16_range(ql, which):
    # Envelopes 2^11 times larger put factor elements well past fp16's maximum (65504): G's when
    # Q_V and B_amp are scaled, F's when A_amp and Q_U are.  The tensor-core path rebuilds each
    # factor times a power of two chosen from the envelope maxima and scales the output back, so
    # the result still meets the tolerance (and the decode kernels, which have no such limit, are
    # not needed for it).
    n, m, r, l, P, B = 512, 1024, 384, 4, 2, 40      # l * B = 160: the tensor-core path
    paths = synth.mdbf_paths(P, n, m, r, l, seed=51)
    for p in paths:
        if which in ("G", "both"):
            p.Q_V = _scaled_envelope(p.Q_V, 2048.0)
            p.B_amp = _scaled_envelope(p.B_amp, 2048.0)
        if which in ("F", "both"):
            p.A_amp = _scaled_envelope(p.A_amp, 2048.0)
            p.Q_U = _scaled_envelope(p.Q_U, 2048.0)
    big = max(max(np.abs(F).max(), np.abs(G).max()) for F, G in (om.factors(p, n, m, r) for p in paths))
    assert big > 65504.0
    x = synth.activations(B, m, seed=52)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert np.all(np.isfinite(y))
    assert max_rel(y, om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL
    yb = _linear(ql, paths, n, m, r, l, x, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(yb, f32_to_bf16_rne(y))


@pytest.mark.parametrize("ldSA,ldSB", [(40, 128), (44, 132)])
def test_batched_narrow_sign_strides(ql, ldSA, ldSB):
    # strides that are multiples of 4 bytes but not of 16, the last 32-bit word of a row reaching
    # into its padding bytes
    n, m, r, l, P, B = 400, 1000, 300, 2, 2, 50
    paths = synth.mdbf_paths(P, n, m, r, l, seed=41, ldSA=ldSA, ldSB=ldSB)
    x = synth.activations(B, m, seed=42)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert max_rel(y, om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL


@pytest.mark.parametrize("n,m", [(17408, 5120), (5120, 17408)])
def test_batched_27b_mlp_sampled(ql, n, m):
    # The 27B-class MLP projections at P = 2, l = 4, rank 2886 (1.5 bits/weight) and a 2048-token
    # prefill batch, in the launch configuration the benchmark times; checked on sampled token
    # rows and output features spread over the tiles, the path boundary and the ragged edges.
    r, l, P, B = 2886, 4, 2, 2048
    paths = synth.mdbf_paths(P, n, m, r, l, seed=n // 7 + m)
    x = synth.activations(B, m, seed=m)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    rows_b = np.array([0, 1, 255, 256, 511, 512, 1023, 1500, 2046, 2047])
    rows_a = np.unique(np.concatenate([np.arange(0, n, n // 24), [1, 127, 128, 255, 256, n - 257, n - 2, n - 1]]))
    ref = om.linear_factored(paths, n, m, r, x[rows_b], rows=rows_a)
    assert max_rel(y[np.ix_(rows_b, rows_a)], ref) <= MDBF_TOL
