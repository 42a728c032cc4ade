"""BenQ encoder on the GPU against the oracle's encoder: bit-exact codes and tables.

The inputs keep every row's nonzero magnitudes within a factor 2^30 of each other (the condition
under which the tier sums, and so the levels, do not depend on the order of addition).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import benq as ob
from tests.qlhelpers import bf16, dev

pytestmark = pytest.mark.gpu


def _weights(N, K, seed, scale=0.02):
    rng = np.random.default_rng(seed)
    sig = rng.uniform(0.5, 1.5, size=(N, 1)) * scale
    return synth.f32_to_bf16_bits((rng.standard_normal((N, K)) * sig).astype(np.float32))


def _encode(ql, wb, iters):
    N, K = wb.shape
    codes = torch.empty(N, 3 * K // 4, dtype=torch.uint8, device="cuda")
    lut = torch.empty(N, 64, dtype=torch.int16, device="cuda")
    ql.benq_encode(bf16(wb), codes, lut, lloyd_iters=iters)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), lut.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("N,K,iters", [(8, 64, 0), (33, 1000, 0), (33, 1000, 2), (256, 5120, 0), (64, 4096, 3),
                                       (5, 4, 1), (3, 20480, 1)])
def test_encode_bit_exact(ql, N, K, iters):
    wb = _weights(N, K, seed=N * 7 + K + iters)
    codes, lut = _encode(ql, wb, iters)
    oc, ol = ob.encode(wb, iters)
    assert np.array_equal(lut, ol)
    assert np.array_equal(codes, oc)


def test_encode_edge_rows(ql):
    K = 256
    wb = _weights(6, K, seed=1)
    wb[0] = 0                                       # all-zero row
    wb[1] = 0x8000                                  # all -0.0
    wb[2] = 0
    wb[2, 17] = synth.f32_to_bf16_bits(np.array([-0.75], np.float32))[0]   # a single nonzero
    wb[3, ::2] = 0                                  # half zeros
    wb[4] = wb[4, :1]                               # every entry equal: one tier holds the row
    wb[5, :128] = synth.f32_to_bf16_bits(np.full(128, 1e-3, np.float32))   # ties in a tier
    for iters in (0, 2):
        codes, lut = _encode(ql, wb, iters)
        oc, ol = ob.encode(wb, iters)
        assert np.array_equal(lut, ol) and np.array_equal(codes, oc)


def test_encode_exact_tie_row(ql):
    # 0.75 lies exactly halfway between the levels of tiers 7 (empty, its midpoint 45/64) and 8
    # (the mean 51/64 of 0.75, 0.8125, 0.828125) of a row with max 3: both sides take the lower
    # tier; repeated 32 times over a longer row, with the sign flipped on every other copy
    base = np.array([3.0, 0.75, 0.8125, 0.828125, 0.0, 0.0, 0.0, 0.0], dtype=np.float32)
    row = np.tile(base, 32) * np.repeat(np.array([1.0, -1.0] * 16, np.float32), 8)
    wb = synth.f32_to_bf16_bits(row.reshape(1, -1))
    codes, lut = _encode(ql, wb, 0)
    oc, ol = ob.encode(wb, 0)
    assert np.array_equal(lut, ol) and np.array_equal(codes, oc)
    assert ob.unpack_codes(codes, 256)[0, :8].tolist() == [63, 39, 40, 40, 32, 32, 32, 32]


def test_encode_27b_shape_sampled_rows(ql):
    # a 17408 x 5120 matrix in one launch; rows are independent, so sampled rows are checked against
    # the oracle run on those rows alone
    N, K = 17408, 5120
    wb = _weights(N, K, seed=99)
    codes, lut = _encode(ql, wb, 1)
    rows = np.unique(np.concatenate([np.arange(0, N, 271), [N - 1]]))
    oc, ol = ob.encode(wb[rows], 1)
    assert np.array_equal(lut[rows], ol) and np.array_equal(codes[rows], oc)


def test_encode_then_linear(ql):
    # the encoder's output is the storage benq_linear reads: the product equals the oracle's product
    # of the oracle's own encoding
    N, K = 512, 2048
    wb = _weights(N, K, seed=5)
    codes, lut = _encode(ql, wb, 2)
    x = synth.activations(1, K, seed=6)
    y = torch.empty(1, N, device="cuda")
    ql.benq_linear(dev(codes), torch.from_numpy(lut.view(np.int16)).cuda(), bf16(x), y)
    torch.cuda.synchronize()
    oc, ol = ob.encode(wb, 2)
    ref = ob.linear(oc, ol, x, K)
    yy = y.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(yy - ref)) <= 2e-3 * np.max(np.abs(ref))
