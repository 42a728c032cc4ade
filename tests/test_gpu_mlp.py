"""Gated MLP of two BenQ projections on the GPU, h = silu(x W_g^T) * (x W_u^T), against the oracle.

Bar: both projections are held to the BenQ bar (max |err| <= 2e-3 of the row's largest value), so
first-order propagation through h = silu(g) u bounds each output by
    |h - h_ref| <= 2e-3 (|silu'(g)| max|g| |u| + |silu(g)| max|u|)   (g, u, maxima from the oracle),
plus fp32 evaluation of the gate (a few ulps; values below fp32's normal range become 0).  The fused batch-1 kernel must also reproduce the separate
projections (its sums are the batch-1 GEMV's), and bf16 output must be the round-to-nearest-even of
the fp32 output.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import benq as ob
from tests.qlhelpers import BENQ_TOL, bf16, bits16, dev, f32_to_bf16_rne

pytestmark = pytest.mark.gpu


def _layers(N, K, seed):
    wg = synth.benq_weights(N, K, seed=seed)
    wu = synth.benq_weights(N, K, seed=seed + 1)
    return wg, wu


def _mlp(ql, wg, wu, x, dtype=torch.float32):
    B, K = x.shape
    N = wg.codes.shape[0]
    nws = ql.benq_mlp_workspace_bytes(B, N, K)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda") if nws else None
    h = torch.empty(B, N, dtype=dtype, device="cuda")
    ql.benq_mlp_gate_up(dev(wg.codes), bits16(wg.lut), dev(wu.codes), bits16(wu.lut), bf16(x), h, workspace=ws)
    ql.ql_check()
    return h


def _dsilu(v):
    s = 1.0 / (1.0 + np.exp(-np.clip(v, -700, 700)))
    return s * (1.0 + v * (1.0 - s))


def _check_against_oracle(h, wg, wu, x, K, rows=None):
    g = ob.linear(wg.codes, wg.lut, x, K, rows)
    u = ob.linear(wu.codes, wu.lut, x, K, rows)
    ref = ob.silu(g) * u
    gmax = np.abs(g).max(axis=1, keepdims=True)
    umax = np.abs(u).max(axis=1, keepdims=True)
    # + fp32 evaluation of the gate: a few ulps of h, and h below fp32's normal range flushes to 0
    bound = (BENQ_TOL * (np.abs(_dsilu(g)) * gmax * np.abs(u) + np.abs(ob.silu(g)) * umax) + 1e-6 * np.abs(ref)
             + np.finfo(np.float32).tiny)
    err = np.abs(np.asarray(h, dtype=np.float64) - ref)
    assert np.all(err <= bound), float((err / np.maximum(bound, 1e-300)).max())


@pytest.mark.parametrize("N,K", [(256, 1024), (1000, 2048), (34, 5120), (1024, 20480), (2, 1024), (6, 3072),
                                 (2050, 17408)])
def test_fused_decode_matches_oracle(ql, N, K):
    wg, wu = _layers(N, K, seed=N + K)
    x = synth.activations(1, K, seed=K)
    assert ql.benq_mlp_workspace_bytes(1, N, K) == 0          # the fused batch-1 kernel
    h = _mlp(ql, wg, wu, x).cpu().numpy()
    _check_against_oracle(h, wg, wu, x, K)
    hb = _mlp(ql, wg, wu, x, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(hb, f32_to_bf16_rne(h))


def test_fused_sums_equal_the_separate_projections(ql):
    # the fused kernel's g and u are the batch-1 GEMV's sums: h agrees with silu(g) * u formed from
    # benq_linear's own fp32 outputs to within the gate's few-ulp evaluation difference
    N, K = 2048, 4096
    wg, wu = _layers(N, K, seed=77)
    x = synth.activations(1, K, seed=78)
    h = _mlp(ql, wg, wu, x).cpu().numpy().astype(np.float64)
    g = torch.empty(1, N, device="cuda")
    u = torch.empty(1, N, device="cuda")
    ql.benq_linear(dev(wg.codes), bits16(wg.lut), bf16(x), g)
    ql.benq_linear(dev(wu.codes), bits16(wu.lut), bf16(x), u)
    torch.cuda.synchronize()
    gf = g.cpu().numpy().astype(np.float64)
    uf = u.cpu().numpy().astype(np.float64)
    ref = ob.silu(gf) * uf
    assert np.all(np.abs(h - ref) <= 4 * np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64) + 1e-30)


def test_gate_extremes(ql):
    # rows whose gate sums are large and negative (silu -> -0) or large and positive (silu -> g)
    N, K = 64, 1024
    wg, wu = _layers(N, K, seed=5)
    x = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(synth.activations(1, K, seed=6)) * np.float32(200.0))
    h = _mlp(ql, wg, wu, x).cpu().numpy()
    assert np.all(np.isfinite(h))
    _check_against_oracle(h, wg, wu, x, K)


@pytest.mark.parametrize("B,N,K", [(3, 300, 1000), (16, 512, 2048), (40, 512, 1024), (1, 300, 1000)])
def test_two_projection_path_matches_oracle(ql, B, N, K):
    # shapes the fused kernel does not take: GEMV batches, a tensor-core GEMM batch, and a batch-1
    # shape with K not a multiple of 1024
    wg, wu = _layers(N, K, seed=B * 1000 + N)
    x = synth.activations(B, K, seed=B + K)
    assert ql.benq_mlp_workspace_bytes(B, N, K) >= 2 * B * N * 4
    h = _mlp(ql, wg, wu, x).cpu().numpy()
    _check_against_oracle(h, wg, wu, x, K)
    hb = _mlp(ql, wg, wu, x, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(hb, f32_to_bf16_rne(h))


def test_27b_gate_up_sampled(ql):
    # the 27B-class gate/up projection pair (5120 -> 17408), batch 1, on sampled output features
    N, K = 17408, 5120
    wg, wu = _layers(N, K, seed=3001)
    x = synth.activations(1, K, seed=3002)
    h = _mlp(ql, wg, wu, x).cpu().numpy()
    rows = np.unique(np.concatenate([np.arange(0, N, 97), [1, 2, 3, N - 2, N - 1]]))
    _check_against_oracle(h[:, rows], wg, wu, x, K, rows=rows)
