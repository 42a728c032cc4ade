"""The seeded generators follow their stated rules (CPU only)."""
import numpy as np

import synth
from oracle import benq as ob


def _f(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 0.0], dtype=np.float32)
    out = _f(synth.f32_to_bf16_bits(vals))
    assert out.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5, 0.0]


def test_lut_rows_sorted_signed_and_mirrored():
    w = synth.benq_weights(300, 512, seed=0)
    L = _f(w.lut)
    assert (np.diff(L, axis=1) >= 0).all()
    assert (L[:, :32] <= 0).all() and (L[:, 32:] >= 0).all()
    assert np.array_equal(L[:, 31 - np.arange(32)], -L[:, 32 + np.arange(32)])


def test_codes_are_nearest_level_by_brute_force():
    N, K = 40, 256
    w = synth.benq_weights(N, K, seed=3)
    # regenerate the same raw weights with the generator's own stream to brute-force the assignment
    rng = synth._rng(3, 0)
    sigma = rng.uniform(0.01, 0.03, size=N).astype(np.float32)
    raw = rng.standard_normal((N, K), dtype=np.float32) * sigma[:, None]
    codes = ob.unpack_codes(w.codes, K)
    L = _f(w.lut).astype(np.float64)
    for n in range(N):
        lv = L[n, 32:]
        for k in range(K):
            v = float(raw[n, k])
            d = np.abs(abs(v) - lv)
            tier = int(np.flatnonzero(d == d.min())[0])
            want = 32 + tier if not (v < 0) else 31 - tier
            assert codes[n, k] == want


def test_generation_is_thread_count_independent():
    a = synth.benq_weights(600, 128, seed=5, threads=1)
    b = synth.benq_weights(600, 128, seed=5, threads=7)
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.lut, b.lut)
    p = synth.mdbf_path(600, 64, 32, 2, seed=1, threads=1)
    q = synth.mdbf_path(600, 64, 32, 2, seed=1, threads=5)
    assert np.array_equal(p.S_A, q.S_A) and np.array_equal(p.S_B, q.S_B)


def test_mdbf_envelopes_and_strides():
    p = synth.mdbf_path(100, 200, 50, 3, seed=2)
    assert p.S_A.shape == (100, 16) and p.S_B.shape == (50, 32)
    for e, shape in ((p.A_amp, (100, 3)), (p.B_amp, (200, 3)), (p.Q_U, (50, 3)), (p.Q_V, (50, 3))):
        v = e.view(np.float16).astype(np.float32)
        assert v.shape == shape and (v >= 0).all() and v.max() < 0.5
