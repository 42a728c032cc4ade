"""Pins for the MDBF oracle (CPU only).

Ties ``oracle.mdbf`` to a worked layer derived by hand from the MDBF page's
"Algorithm" formulas, to exact rational arithmetic, to the degenerate
(l, P) = (1, 1) DBF form W = A diag(d) B and the (1, 2) LittleBit form the page
names, and to the agreement of two independent evaluation orders.
"""
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import mdbf as om


def _f16(vals):
    return np.array(vals, dtype=np.float16).view(np.uint16)


def _bf16(vals):
    return synth.f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


def _golden_path(g):
    return synth.MDBFPath(
        S_A=np.array([[int(b, 16)] for b in g["S_A_bytes"]], dtype=np.uint8),
        S_B=np.array([[int(b, 16)] for b in g["S_B_bytes"]], dtype=np.uint8),
        A_amp=_f16([float(v) for v in g["A_amp"]]).reshape(2, 2),
        B_amp=_f16([float(v) for v in g["B_amp"]]).reshape(3, 2),
        Q_U=_f16([float(v) for v in g["Q_U"]]).reshape(2, 2),
        Q_V=_f16([float(v) for v in g["Q_V"]]).reshape(2, 2),
    )


def test_sign_unpack_hand_worked(golden):
    g = golden("mdbf_sign_pack_example.txt")
    signs = [int(s) for s in g["signs"]]
    for key in ("bytes", "bytes_with_garbage_padding"):
        packed = np.array([[int(b, 16) for b in g[key]]], dtype=np.uint8)
        assert om.unpack_signs(packed, 10).tolist() == [signs]


def test_generator_sign_pack_hand_worked(golden):
    g = golden("mdbf_sign_pack_example.txt")
    bits = (np.array([[int(s) for s in g["signs"]]]) > 0).astype(np.uint8)
    assert synth.pack_signs(bits, 2).tolist() == [[int(b, 16) for b in g["bytes"]]]


def test_dequant_and_linear_hand_worked(golden):
    g = golden("mdbf_example.txt")
    path = _golden_path(g)
    W = om.dequant([path], 2, 3, 2)
    assert W.ravel().tolist() == [float(v) for v in g["W"]]
    x = _bf16([[float(v) for v in g["x"]]])
    y = [float(v) for v in g["y"]]
    assert om.linear_dense([path], 2, 3, 2, x).ravel().tolist() == y
    assert om.linear_factored([path], 2, 3, 2, x).ravel().tolist() == y
    F, G = om.factors(path, 2, 3, 2)
    assert F.tolist() == [[1.0, -2.25], [-0.5, -0.125]]
    assert G.tolist() == [[2.0, 1.0, -1.5], [0.0, 0.5, 0.25]]


def _exact_W(paths, n, m, r):
    """W with every operation in exact rationals, straight from the page's formulas."""
    W = [[Fraction(0)] * m for _ in range(n)]
    for p in paths:
        SA = om.unpack_signs(p.S_A, r)
        SB = om.unpack_signs(p.S_B, m)
        A = p.A_amp.view(np.float16)
        Bm = p.B_amp.view(np.float16)
        QU = p.Q_U.view(np.float16)
        QV = p.Q_V.view(np.float16)
        l = A.shape[1]
        F = [[int(SA[a, k]) * sum(Fraction(float(A[a, i])) * Fraction(float(QU[k, i])) for i in range(l))
              for k in range(r)] for a in range(n)]
        G = [[int(SB[k, j]) * sum(Fraction(float(QV[k, i])) * Fraction(float(Bm[j, i])) for i in range(l))
              for j in range(m)] for k in range(r)]
        for a in range(n):
            for j in range(m):
                W[a][j] += sum(F[a][k] * G[k][j] for k in range(r))
    return W


def _dyadic_path(rng, n, m, r, l):
    """Envelope values k/8, k in 1..8: every fp32 envelope sum and fp64 product sum is exact."""
    def env(shape):
        return _f16(rng.integers(1, 9, size=shape) / 8.0)
    return synth.MDBFPath(
        S_A=synth.pack_signs(rng.integers(0, 2, (n, r)), synth.default_ld(r), rng),
        S_B=synth.pack_signs(rng.integers(0, 2, (r, m)), synth.default_ld(m), rng),
        A_amp=env((n, l)), B_amp=env((m, l)), Q_U=env((r, l)), Q_V=env((r, l)))


@pytest.mark.parametrize("shape", [(3, 4, 2, 2, 1), (4, 3, 3, 1, 2), (2, 5, 3, 2, 2), (4, 4, 1, 3, 1)])
def test_dequant_exact_rational_dyadic(shape):
    n, m, r, l, P = shape
    rng = np.random.default_rng(sum(shape))
    paths = [_dyadic_path(rng, n, m, r, l) for _ in range(P)]
    W = om.dequant(paths, n, m, r)
    exact = _exact_W(paths, n, m, r)
    for a in range(n):
        for j in range(m):
            assert W[a, j] == np.float32(float(exact[a][j]))


@pytest.mark.parametrize("shape", [(3, 4, 2, 2, 1), (4, 3, 3, 2, 2), (2, 5, 3, 3, 2)])
def test_dequant_rational_random_fp16_within_rounding(shape):
    # general fp16 envelopes: the only rounding is fp32 in the l-sum and the final fp32 store
    n, m, r, l, P = shape
    paths = synth.mdbf_paths(P, n, m, r, l, seed=sum(shape))
    W = om.dequant(paths, n, m, r)
    exact = _exact_W(paths, n, m, r)
    absW = np.abs(om.dequant(paths, n, m, r, return_f64=True))
    for a in range(n):
        for j in range(m):
            err = abs(Fraction(float(W[a, j])) - exact[a][j])
            # |F||G| summed, times (2 l-sum roundings of 2^-24 each) plus one fp32 store rounding
            F_G = 0.0
            for p in paths:
                Fp, Gp = om.factors(p, n, m, r)
                F_G += float(np.abs(Fp[a]).astype(np.float64) @ np.abs(Gp[:, j]).astype(np.float64))
            assert err <= Fraction(F_G) * Fraction(2 * l + 1, 2 ** 23) + Fraction(float(absW[a, j])) / 2 ** 24


def test_dbf_degenerate_case_l1_p1():
    # (l, P) = (1, 1) is DBF: W = diag(a) S_A diag(q_u * q_v) S_B diag(b)
    rng = np.random.default_rng(5)
    n, m, r = 6, 9, 4
    path = _dyadic_path(rng, n, m, r, 1)
    a = path.A_amp.view(np.float16).astype(np.float64)[:, 0]
    b = path.B_amp.view(np.float16).astype(np.float64)[:, 0]
    d = (path.Q_U.view(np.float16).astype(np.float64) * path.Q_V.view(np.float16).astype(np.float64))[:, 0]
    SA = om.unpack_signs(path.S_A, r).astype(np.float64)
    SB = om.unpack_signs(path.S_B, m).astype(np.float64)
    dbf = np.diag(a) @ SA @ np.diag(d) @ SB @ np.diag(b)
    assert np.array_equal(om.dequant([path], n, m, r).astype(np.float64), dbf)
    # general fp16 values: agreement to fp64 rounding
    gpath = synth.mdbf_path(n, m, r, 1, seed=3)
    a = gpath.A_amp.view(np.float16).astype(np.float64)[:, 0]
    b = gpath.B_amp.view(np.float16).astype(np.float64)[:, 0]
    d = (gpath.Q_U.view(np.float16).astype(np.float64) * gpath.Q_V.view(np.float16).astype(np.float64))[:, 0]
    SA = om.unpack_signs(gpath.S_A, r).astype(np.float64)
    SB = om.unpack_signs(gpath.S_B, m).astype(np.float64)
    dbf = np.diag(a) @ SA @ np.diag(d) @ SB @ np.diag(b)
    W64 = om.dequant([gpath], n, m, r, return_f64=True)
    assert np.allclose(W64, dbf, rtol=1e-14, atol=0)


def test_littlebit_case_l1_p2_is_sum_of_two_dbf():
    rng = np.random.default_rng(6)
    n, m, r = 5, 7, 3
    paths = [_dyadic_path(rng, n, m, r, 1) for _ in range(2)]
    total = np.zeros((n, m))
    for p in paths:
        a = p.A_amp.view(np.float16).astype(np.float64)[:, 0]
        b = p.B_amp.view(np.float16).astype(np.float64)[:, 0]
        d = (p.Q_U.view(np.float16).astype(np.float64) * p.Q_V.view(np.float16).astype(np.float64))[:, 0]
        total += np.diag(a) @ om.unpack_signs(p.S_A, r) @ np.diag(d) @ om.unpack_signs(p.S_B, m) @ np.diag(b)
    assert np.array_equal(om.dequant(paths, n, m, r).astype(np.float64), total)


@pytest.mark.parametrize("shape", [(24, 40, 12, 2, 1), (40, 24, 20, 4, 2), (33, 17, 9, 3, 2)])
def test_factored_matches_materialised(shape):
    n, m, r, l, P = shape
    paths = synth.mdbf_paths(P, n, m, r, l, seed=n + m)
    x = synth.activations(3, m, seed=9)
    xf = om.bf16_to_f64(x)
    # W with fp64 envelopes, written out with matrix products straight from the page's formulas
    W_exact = np.zeros((n, m))
    for p in paths:
        f = lambda e: e.view(np.float16).astype(np.float64)
        F = om.unpack_signs(p.S_A, r) * (f(p.A_amp) @ f(p.Q_U).T)
        G = om.unpack_signs(p.S_B, m) * (f(p.Q_V) @ f(p.B_amp).T)
        W_exact += F @ G
    y_exact = xf @ W_exact.T
    yF = om.linear_factored(paths, n, m, r, x)
    scale = np.abs(y_exact).max()
    assert np.abs(yF - y_exact).max() <= 1e-12 * scale
    # the materialised oracle rounds envelopes and W to fp32: agreement to a few fp32 ulps
    yD = om.linear_dense(paths, n, m, r, x)
    assert np.abs(yD - y_exact).max() <= 1e-6 * scale
    rows = np.array([0, n - 1, n // 2])
    assert np.allclose(om.linear_factored(paths, n, m, r, x, rows=rows), yF[:, rows], rtol=0, atol=1e-13 * scale)


def test_dequant_at_matches_dequant_bit_exact():
    n, m, r, l, P = 30, 50, 20, 3, 2
    paths = synth.mdbf_paths(P, n, m, r, l, seed=11)
    W = om.dequant(paths, n, m, r)
    rng = np.random.default_rng(2)
    a = rng.integers(0, n, 64)
    j = rng.integers(0, m, 64)
    assert np.array_equal(om.dequant_at(paths, r, m, a, j), W[a, j])


def test_padding_bits_are_ignored():
    n, m, r, l = 8, 13, 5, 2
    p = synth.mdbf_path(n, m, r, l, seed=21)
    q = synth.MDBFPath(S_A=p.S_A.copy(), S_B=p.S_B.copy(), A_amp=p.A_amp, B_amp=p.B_amp, Q_U=p.Q_U, Q_V=p.Q_V)
    q.S_A[:, 0] ^= np.uint8(0xE0)          # bits 5..7 of byte 0 are columns >= r = 5
    q.S_A[:, 1:] ^= np.uint8(0xFF)
    q.S_B[:, 1] ^= np.uint8(0xE0)          # columns >= 13
    q.S_B[:, 2:] ^= np.uint8(0xFF)
    assert np.array_equal(om.dequant([p], n, m, r), om.dequant([q], n, m, r))
