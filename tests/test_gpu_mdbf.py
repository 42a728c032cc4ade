"""MDBF parity on the GPU: the C ABI against the CPU oracle on the same seeded inputs.

mdbf_dequant_debug must reproduce the oracle's W, F and G bit for bit;
mdbf_linear must be within 5e-3 (max |y - y_ref| / max |y_ref| per batch row,
fp32 output) of the oracle's fp64 result, and its bf16 output must be the
round-to-nearest-even of its own fp32 output.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import mdbf as om
from tests.qlhelpers import MDBF_TOL, bf16, dev, f32_to_bf16_rne, max_rel, mdbf_dev_paths

pytestmark = pytest.mark.gpu


def _linear(ql, paths, n, m, r, l, xbits, ydtype=torch.float32):
    B = xbits.shape[0]
    dp = mdbf_dev_paths(paths)
    ws = torch.empty(ql.mdbf_workspace_bytes(len(paths), n, m, r, l, B), dtype=torch.uint8, device="cuda")
    y = torch.empty(B, n, dtype=ydtype, device="cuda")
    ql.mdbf_linear(dp, n, m, r, l, bf16(xbits), y, ws)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("n,m,r,l,P", [(40, 24, 20, 4, 2), (64, 96, 33, 3, 2), (100, 37, 29, 1, 1),
                                       (128, 128, 64, 2, 1), (17, 300, 17, 2, 3), (512, 256, 200, 4, 2)])
def test_dequant_bit_exact(ql, n, m, r, l, P):
    paths = synth.mdbf_paths(P, n, m, r, l, seed=n + m + r)
    dp = mdbf_dev_paths(paths)
    W = torch.empty(n, m, device="cuda")
    F = torch.empty(P, n, r, device="cuda")
    G = torch.empty(P, r, m, device="cuda")
    ql.mdbf_dequant_debug(dp, n, m, r, l, W, F, G)
    torch.cuda.synchronize()
    assert np.array_equal(W.cpu().numpy().view(np.uint32), om.dequant(paths, n, m, r).view(np.uint32))
    for p in range(P):
        Fo, Go = om.factors(paths[p], n, m, r)
        assert np.array_equal(F[p].cpu().numpy().view(np.uint32), Fo.view(np.uint32))
        assert np.array_equal(G[p].cpu().numpy().view(np.uint32), Go.view(np.uint32))


def test_dequant_hand_worked_example(ql, golden):
    g = golden("mdbf_example.txt")
    f16 = lambda v: np.array([float(t) for t in v], dtype=np.float16).view(np.uint16)
    S_A = np.zeros((2, 4), np.uint8)
    S_A[:, 0] = [int(b, 16) for b in g["S_A_bytes"]]
    S_B = np.zeros((2, 4), np.uint8)
    S_B[:, 0] = [int(b, 16) for b in g["S_B_bytes"]]
    path = synth.MDBFPath(S_A=S_A, S_B=S_B, A_amp=f16(g["A_amp"]).reshape(2, 2), B_amp=f16(g["B_amp"]).reshape(3, 2),
                          Q_U=f16(g["Q_U"]).reshape(2, 2), Q_V=f16(g["Q_V"]).reshape(2, 2))
    W = torch.empty(2, 3, device="cuda")
    ql.mdbf_dequant_debug(mdbf_dev_paths([path]), 2, 3, 2, 2, W)
    x = synth.f32_to_bf16_bits(np.array([[float(v) for v in g["x"]]], dtype=np.float32))
    y = _linear(ql, [path], 2, 3, 2, 2, x)
    assert W.cpu().numpy().ravel().tolist() == [float(v) for v in g["W"]]
    assert np.allclose(y.cpu().numpy().ravel(), [float(v) for v in g["y"]], rtol=1e-6, atol=0)


@pytest.mark.parametrize("n,m,r,l,P,B", [(5, 7, 3, 1, 1, 1), (33, 65, 31, 2, 2, 3), (100, 40, 40, 4, 2, 16),
                                         (64, 64, 64, 8, 1, 8), (70, 90, 50, 3, 3, 5), (300, 200, 100, 1, 2, 1),
                                         (96, 1000, 95, 2, 1, 32), (1, 1, 1, 1, 1, 1),
                                         # l * B <= 4 with several token rows (the F stage's per-row
                                         # sums for each b), one and two paths, ragged n, m and r
                                         (130, 200, 64, 2, 2, 2), (77, 50, 40, 1, 2, 4), (4000, 300, 128, 1, 1, 3)])
def test_linear_shapes(ql, n, m, r, l, P, B):
    paths = synth.mdbf_paths(P, n, m, r, l, seed=3 * n + m)
    x = synth.activations(B, m, seed=B)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert max_rel(y, om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL
    yd = om.linear_dense(paths, n, m, r, x)
    assert max_rel(y, yd) <= MDBF_TOL
    yb = _linear(ql, paths, n, m, r, l, x, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(yb, f32_to_bf16_rne(y))


@pytest.mark.parametrize("B", [1, 16])
def test_linear_square_one_bit_layer(ql, B):
    # n = m = 4096, P = 1, l = 2, r = 2000 (b_eff ~ 1.0)
    n = m = 4096
    r, l = 2000, 2
    paths = synth.mdbf_paths(1, n, m, r, l, seed=3000)
    x = synth.activations(B, m, seed=3100 + B)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert max_rel(y, om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL


@pytest.mark.parametrize("P,B", [(1, 1), (1, 16), (2, 1), (2, 16)])
def test_linear_rank_one_envelopes(ql, P, B):
    # l = 1: the envelopes collapse to row and column scalings, W = sum_p diag(a) S_A diag(q_u q_v)
    # S_B diag(b) ("DBF" at P = 1, "LittleBit" at P = 2): the square one-bit layer at rank 2000
    n = m = 4096
    r, l = 2000, 1
    paths = synth.mdbf_paths(P, n, m, r, l, seed=3200 + P)
    x = synth.activations(B, m, seed=3300 + B)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert max_rel(y, om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL


@pytest.mark.parametrize("n,m", [(17408, 5120), (5120, 17408)])
def test_linear_mlp_shapes_sampled_rows(ql, n, m):
    # 27B-class gate/up and down at 1.5 bits/weight: P = 2, l = 4, r = 2886
    r, l, P = 2886, 4, 2
    paths = synth.mdbf_paths(P, n, m, r, l, seed=4000 + n // 1024)
    x = synth.activations(1, m, seed=4100)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    rows = np.r_[np.random.default_rng(2).choice(n, 256, replace=False), 0, n - 1]
    assert max_rel(y[:, rows], om.linear_factored(paths, n, m, r, x, rows=rows)) <= MDBF_TOL


@pytest.mark.parametrize("P", [1, 2])
def test_linear_more_g_blocks_than_sms(ql, P):
    # more 32-row blocks of S_B than SMs (the G stage then runs 16 warps per block), ragged r
    n, m, r, l, B = 5200, 4800, 4790 // P, 4, 1
    paths = synth.mdbf_paths(P, n, m, r, l, seed=4400 + P)
    x = synth.activations(B, m, seed=4500 + P)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert max_rel(y, om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL


def test_linear_is_deterministic(ql):
    paths = synth.mdbf_paths(2, 1024, 768, 300, 4, seed=8)
    x = synth.activations(2, 768, seed=9)
    a = _linear(ql, paths, 1024, 768, 300, 4, x)
    b = _linear(ql, paths, 1024, 768, 300, 4, x)
    assert torch.equal(a, b)


@pytest.mark.parametrize("B", [1, 2])
def test_linear_tall_layer_full_size_blocks(ql, B):
    # n >= 128 x 148 rows: the F stage runs 128-row blocks
    n, m, r, l, P = 20480, 1024, 256, 4, 2
    paths = synth.mdbf_paths(P, n, m, r, l, seed=5000 + B)
    x = synth.activations(B, m, seed=5100 + B)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    rows = np.r_[np.random.default_rng(4).choice(n, 256, replace=False), 0, 127, 128, n - 129, n - 1]
    assert max_rel(y[:, rows], om.linear_factored(paths, n, m, r, x, rows=rows)) <= MDBF_TOL


@pytest.mark.parametrize("n,P,l,B", [(4700, 2, 4, 1), (6000, 2, 2, 2), (9400, 1, 4, 1), (9500, 2, 1, 4)])
def test_linear_f_stage_row_blocks(ql, n, P, l, B):
    # the one-pass F stage takes 32-row CTAs while they fit in one round on 148 SMs (n = 4700), then
    # 64-row ones (n = 6000, a 48-row tail; n = 9400), then 128-row ones (n = 9500, a 28-row tail);
    # the results match the oracle and do not depend on the row count per CTA (bit-identical to a
    # two-layer call of the same layer, which halves the row count that fits)
    m, r = 640, 300
    paths = synth.mdbf_paths(P, n, m, r, l, seed=5250 + n + P)
    x = synth.activations(B, m, seed=5350 + B)
    y = _linear(ql, paths, n, m, r, l, x)
    assert max_rel(y.cpu().numpy(), om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL
    dp = mdbf_dev_paths(paths)
    ws = torch.empty(ql.mdbf_workspace_bytes(2 * P, n, m, r, l, B), dtype=torch.uint8, device="cuda")
    ys = [torch.empty(B, n, device="cuda") for _ in range(2)]
    ql.mdbf_linear_multi([dp, dp], n, m, r, l, bf16(x), ys, ws)
    torch.cuda.synchronize()
    assert torch.equal(ys[0], y) and torch.equal(ys[1], y)


@pytest.mark.parametrize("m,spread", [(8222, 3.0), (9000, 3.0), (8192, 0.0)])
def test_linear_s8_g_stage_group_scales(ql, m, spread):
    # the split G stage (m >= 8192) runs on the s8 MMA with z quantised per 128-column group and
    # vector: activations whose magnitudes span 10^(+-spread) across columns, a last group of one
    # partial word (8222 = 256 words + 30 columns), and an input with whole zero groups
    n, r, l, P, B = 700, 300, 4, 2, 1
    paths = synth.mdbf_paths(P, n, m, r, l, seed=5290 + m)
    xf = synth.bf16_bits_to_f32(synth.activations(B, m, seed=5390 + m))
    rng = np.random.default_rng(m)
    xf = xf * (10.0 ** rng.uniform(-spread, spread, size=(1, m))).astype(np.float32)
    if spread == 0.0:
        xf[:, 256:1024] = 0.0
    x = synth.f32_to_bf16_bits(xf.astype(np.float32))
    y = _linear(ql, paths, n, m, r, l, x)
    assert max_rel(y.cpu().numpy(), om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL


def test_linear_ring_g_three_stages(ql):
    # more than two 32-row G blocks per SM (4790 / 32 -> 150 per path, two paths) take the ring G
    # kernel with three stages (three CTAs per SM); its sums equal the four-stage kernel's
    n, m, r, l, P, B = 4800, 4800, 4790, 4, 2, 1
    paths = synth.mdbf_paths(P, n, m, r, l, seed=5270)
    x = synth.activations(B, m, seed=5370)
    y = _linear(ql, paths, n, m, r, l, x)
    assert max_rel(y.cpu().numpy(), om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL
    # the 27B-class gate and up projections in one call: 2 x 2 x 91 blocks, three stages; each
    # alone (182 blocks) keeps four
    n, m, r = 2900, 5120, 2886
    layers = [synth.mdbf_paths(P, n, m, r, l, seed=5280 + s) for s in range(2)]
    x = synth.activations(B, m, seed=5380)
    single = [_linear(ql, paths, n, m, r, l, x) for paths in layers]
    ws = torch.empty(ql.mdbf_workspace_bytes(2 * P, n, m, r, l, B), dtype=torch.uint8, device="cuda")
    ys = [torch.empty(B, n, device="cuda") for _ in range(2)]
    ql.mdbf_linear_multi([mdbf_dev_paths(p) for p in layers], n, m, r, l, bf16(x), ys, ws)
    torch.cuda.synchronize()
    assert torch.equal(ys[0], single[0]) and torch.equal(ys[1], single[1])
    assert max_rel(ys[1].cpu().numpy(), om.linear_factored(layers[1], n, m, r, x)) <= MDBF_TOL


@pytest.mark.parametrize("l,B", [(4, 4), (4, 8), (2, 16)])
def test_linear_wider_vector_blocks(ql, l, B):
    # l * B = 16, 32, 32: four and eight 8-column MMA blocks per word
    n, m, r, P = 700, 900, 300, 2
    paths = synth.mdbf_paths(P, n, m, r, l, seed=5200 + l * B)
    x = synth.activations(B, m, seed=5300 + B)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert max_rel(y, om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL


@pytest.mark.parametrize("B", [1, 3])
def test_linear_unaligned_sign_strides(ql, B):
    # row strides that are multiples of 4 but not of 16 take the kernels that read signs per lane
    n, m, r, l, P = 300, 200, 100, 2, 2
    ldSA, ldSB = 20, 28   # >= ceil(100/8) = 13 and >= ceil(200/8) = 25
    paths = synth.mdbf_paths(P, n, m, r, l, seed=5400 + B, ldSA=ldSA, ldSB=ldSB)
    assert paths[0].S_A.shape[1] == ldSA and paths[0].S_B.shape[1] == ldSB
    x = synth.activations(B, m, seed=5500 + B)
    y = _linear(ql, paths, n, m, r, l, x).cpu().numpy()
    assert max_rel(y, om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL


@pytest.mark.parametrize("n,m,r,l,P,B", [(1024, 8192, 512, 4, 1, 1), (900, 8000, 333, 2, 2, 1),
                                         (700, 6000, 300, 3, 2, 2), (640, 6144, 200, 1, 1, 1)])
def test_linear_long_sign_rows(ql, n, m, r, l, P, B):
    # few 32-row blocks of S_B with long rows (m up to 8192, ragged in m and r): each G-stage
    # warp runs many word groups through its shared-memory ring, with a partial last group
    paths = synth.mdbf_paths(P, n, m, r, l, seed=5600 + m + r)
    x = synth.activations(B, m, seed=5700 + B)
    y = _linear(ql, paths, n, m, r, l, x)
    assert max_rel(y.cpu().numpy(), om.linear_factored(paths, n, m, r, x)) <= MDBF_TOL
    for _ in range(2):
        assert torch.equal(_linear(ql, paths, n, m, r, l, x), y)


@pytest.mark.parametrize("n,m,r,l,P,B", [(700, 9000, 333, 2, 2, 2), (1100, 8192, 1000, 4, 1, 1), (200, 16400, 130, 1, 2, 4),
                                         # one, two and three vectors (l * B = 1, 2, 3)
                                         (600, 8200, 300, 1, 1, 1), (600, 8300, 300, 2, 2, 1), (600, 8192, 300, 3, 1, 1),
                                         # a rank below one 32-row word
                                         (100, 8500, 20, 4, 2, 1)])
def test_linear_split_g_stage(ql, n, m, r, l, P, B):
    # sign rows of 8192 columns or more run the G stage in split-K units (128 rows x a K slice, the
    # slices' partial sums added by the last unit of each row block): ragged m and r, one and two
    # paths, one to four vectors; a workspace full of stale bytes (arrival counts included) gives the
    # same result, and repeated calls are bit-identical whichever unit of a row block arrives last
    paths = synth.mdbf_paths(P, n, m, r, l, seed=5800 + m + r)
    xbits = synth.activations(B, m, seed=5900 + B)
    y = _linear(ql, paths, n, m, r, l, xbits)
    assert max_rel(y.cpu().numpy(), om.linear_factored(paths, n, m, r, xbits)) <= MDBF_TOL
    dp = mdbf_dev_paths(paths)
    ws = torch.full((ql.mdbf_workspace_bytes(P, n, m, r, l, B),), 0xA5, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        y2 = torch.empty(B, n, device="cuda")
        ql.mdbf_linear(dp, n, m, r, l, bf16(xbits), y2, ws)
        torch.cuda.synchronize()
        assert torch.equal(y2, y)


@pytest.mark.parametrize("S,P,n,m,r,l,B,aligned16,ydtype", [
    (2, 2, 2048, 1536, 700, 4, 1, True, torch.float32),     # one launch per stage, ring G stage
    (2, 2, 2048, 1536, 700, 4, 1, True, torch.bfloat16),
    (3, 1, 500, 300, 200, 2, 2, True, torch.float32),       # three layers, l * B = 4
    (4, 2, 400, 9000, 120, 1, 1, True, torch.float32),      # four layers, eight paths (the limits), split G
    (2, 2, 600, 9000, 300, 4, 1, True, torch.float32),      # long sign rows: split G stage
    (2, 2, 3000, 2000, 500, 2, 2, True, torch.float32),     # 64-row F blocks here, 32-row ones alone
    (2, 2, 300, 200, 100, 4, 2, True, torch.float32),       # l * B = 8: the layers one after another
    (2, 1, 300, 200, 100, 2, 1, False, torch.float32),      # 4-byte sign strides: one after another
    (2, 1, 256, 256, 128, 4, 20, True, torch.float32),      # l * B = 80: tensor-core GEMMs, in turn
])
def test_linear_multi_matches_each_layer(ql, S, P, n, m, r, l, B, aligned16, ydtype):
    # mdbf_linear_multi gives each layer exactly what mdbf_linear gives it (same kernels, same
    # arithmetic), whether the stages run once for all layers or the layers run in turn
    kw = {} if aligned16 else {"ldSA": 20, "ldSB": 28}
    layers = [synth.mdbf_paths(P, n, m, r, l, seed=6000 + 17 * s + m, **kw) for s in range(S)]
    xbits = synth.activations(B, m, seed=6100 + B)
    single = [_linear(ql, paths, n, m, r, l, xbits, ydtype) for paths in layers]
    dls = [mdbf_dev_paths(paths) for paths in layers]
    ws = torch.empty(ql.mdbf_workspace_bytes(S * P, n, m, r, l, B), dtype=torch.uint8, device="cuda")
    ys = [torch.empty(B, n, dtype=ydtype, device="cuda") for _ in range(S)]
    ql.mdbf_linear_multi(dls, n, m, r, l, bf16(xbits), ys, ws)
    torch.cuda.synchronize()
    for s in range(S):
        assert torch.equal(ys[s], single[s]), s
    # the same call with path arrays made once beforehand
    ys2 = [torch.empty(B, n, dtype=ydtype, device="cuda") for _ in range(S)]
    ql.mdbf_linear_multi([ql.mdbf_paths_c(d) for d in dls], n, m, r, l, bf16(xbits), ys2, ws)
    torch.cuda.synchronize()
    for s in range(S):
        assert torch.equal(ys2[s], single[s]), s
    if ydtype == torch.float32:
        assert max_rel(ys[-1].cpu().numpy(), om.linear_factored(layers[-1], n, m, r, xbits)) <= MDBF_TOL


def test_linear_multi_argument_errors(ql):
    paths = synth.mdbf_paths(1, 64, 64, 32, 2, seed=6200)
    dp = mdbf_dev_paths(paths)
    x = bf16(synth.activations(1, 64, seed=6201))
    ws = torch.empty(ql.mdbf_workspace_bytes(2, 64, 64, 32, 2, 1), dtype=torch.uint8, device="cuda")
    y = torch.empty(1, 64, device="cuda")
    with pytest.raises(ValueError):
        ql.mdbf_linear_multi([dp] * 5, 64, 64, 32, 2, x, [y] * 5, ws)                # more than 4 layers
    with pytest.raises(TypeError):
        ql.mdbf_linear_multi([dp, dp], 64, 64, 32, 2, x, [y, y.to(torch.bfloat16)], ws)   # mixed dtypes
    small = torch.empty(ql.mdbf_workspace_bytes(1, 64, 64, 32, 2, 1) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ql.QLinearError):
        ql.mdbf_linear_multi([dp, dp], 64, 64, 32, 2, x, [y, y.clone()], small)      # workspace for one layer
