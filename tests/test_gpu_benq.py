"""BenQ parity on the GPU: the C ABI against the CPU oracle on the same seeded inputs.

Debug dequantization must be bit-exact; benq_linear must be within 2e-3
(max |y - y_ref| / max |y_ref| per batch row, fp32 output) of the oracle's
fp64 result, and its bf16 output must be the round-to-nearest-even of its own
fp32 output.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import benq as ob
from tests.qlhelpers import BENQ_TOL, bf16, bits16, dev, f32_to_bf16_rne, max_rel

pytestmark = pytest.mark.gpu


def _linear(ql, w, xbits, ydtype=torch.float32):
    B = xbits.shape[0]
    y = torch.empty(B, w.N, dtype=ydtype, device="cuda")
    ql.benq_linear(dev(w.codes), bits16(w.lut), bf16(xbits), y)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("N,K", [(256, 512), (1, 4), (3, 8), (5, 100), (77, 1028), (40, 5120)])
def test_dequant_bit_exact(ql, N, K):
    w = synth.benq_weights(N, K, seed=N * 7 + K)
    W = torch.empty(N, K, dtype=torch.int16, device="cuda")
    ql.benq_dequant_debug(dev(w.codes), bits16(w.lut), W)
    torch.cuda.synchronize()
    assert np.array_equal(W.cpu().numpy().view(np.uint16), ob.dequant_bits(w.codes, w.lut, K))


def test_dequant_arbitrary_tables_bit_exact(ql):
    # tables need not be sorted or symmetric: random bit patterns (NaN/Inf included) must pass through
    rng = np.random.default_rng(3)
    N, K = 64, 256
    codes = rng.integers(0, 64, size=(N, K), dtype=np.uint8)
    lut = rng.integers(0, 1 << 16, size=(N, 64), dtype=np.uint16)
    packed = synth.pack_codes(codes)
    W = torch.empty(N, K, dtype=torch.int16, device="cuda")
    ql.benq_dequant_debug(dev(packed), bits16(lut), W)
    torch.cuda.synchronize()
    assert np.array_equal(W.cpu().numpy().view(np.uint16), ob.dequant_bits(packed, lut, K))


def test_dequant_full_size_sampled_rows(ql):
    N, K = 17408, 5120
    w = synth.benq_weights(N, K, seed=1001)
    W = torch.empty(N, K, dtype=torch.int16, device="cuda")
    ql.benq_dequant_debug(dev(w.codes), bits16(w.lut), W)
    torch.cuda.synchronize()
    rows = np.r_[np.random.default_rng(0).choice(N, 96, replace=False), N - 1]
    got = W[torch.from_numpy(rows).cuda()].cpu().numpy().view(np.uint16)
    assert np.array_equal(got, ob.dequant_bits(w.codes[rows], w.lut[rows], K))


@pytest.mark.parametrize("B", [1, 8])
def test_linear_small_layer(ql, B):
    # 256 out x 512 in, the small seeded layer
    w = synth.benq_weights(256, 512, seed=0)
    x = synth.activations(B, 512, seed=1)
    y = _linear(ql, w, x).cpu().numpy()
    assert max_rel(y, ob.linear(w.codes, w.lut, x, 512)) <= BENQ_TOL
    yb = _linear(ql, w, x, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(yb, f32_to_bf16_rne(y))


@pytest.mark.parametrize("N,K,B", [(8, 1024, 1), (64, 3072, 1), (40, 20480, 1), (7, 32, 1), (33, 1056, 3), (100, 2048, 16), (250, 5120, 2), (13, 96, 5),
                                   (129, 3072, 4), (65, 4096, 8), (31, 20480, 1), (2, 64, 16)])
def test_linear_fast_path_shapes(ql, N, K, B):
    w = synth.benq_weights(N, K, seed=N + K + B)
    x = synth.activations(B, K, seed=B)
    y = _linear(ql, w, x).cpu().numpy()
    assert max_rel(y, ob.linear(w.codes, w.lut, x, K)) <= BENQ_TOL


@pytest.mark.parametrize("N,K", [(2, 1024), (6, 1024), (10, 2048), (4098, 1024), (1026, 17408), (2050, 20480),
                                 (10242, 12288), (4096, 12288), (1032, 7168), (2052, 19456), (40, 8192)])
def test_linear_batch1_row_counts(ql, N, K):
    # batch 1 with few rows (fewer row tiles than SMs), N % 4 == 2, one warp per CTA (K = 1024), 20
    # warps (K = 20480) and CTAs that walk many row tiles (K = 12288, one CTA per SM); 7, 8, 12 and 19
    # warps per CTA with whole row tiles, and fewer row tiles than SMs
    w = synth.benq_weights(N, K, seed=N * 3 + K)
    x = synth.activations(1, K, seed=K + 1)
    y = _linear(ql, w, x).cpu().numpy()
    rows = np.arange(N) if N <= 4098 else np.r_[np.arange(0, N, 37), N - 2, N - 1]
    assert max_rel(y[:, rows], ob.linear(w.codes, w.lut, x, K, rows=rows)) <= BENQ_TOL
    yb = _linear(ql, w, x, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(yb, f32_to_bf16_rne(y))


@pytest.mark.parametrize("N,K,B", [(1, 4, 1), (10, 100, 1), (9, 36, 4), (17, 20484, 2), (5, 1000, 16)])
def test_linear_generic_path_shapes(ql, N, K, B):
    w = synth.benq_weights(N, K, seed=N * K + B)
    x = synth.activations(B, K, seed=B + 10)
    y = _linear(ql, w, x).cpu().numpy()
    assert max_rel(y, ob.linear(w.codes, w.lut, x, K)) <= BENQ_TOL


@pytest.mark.parametrize("N,K", [(17408, 5120), (5120, 17408)])
def test_linear_decode_shapes_full_size(ql, N, K):
    # the 27B-class gate/up and down projections at batch 1, sampled rows against the oracle
    w = synth.benq_weights(N, K, seed=1000 + N // 1024)
    x = synth.activations(1, K, seed=1100)
    y = _linear(ql, w, x).cpu().numpy()
    rows = np.r_[np.random.default_rng(1).choice(N, 512, replace=False), 0, N - 1]
    ref = ob.linear(w.codes, w.lut, x, K, rows=rows)
    assert max_rel(y[:, rows], ref) <= BENQ_TOL


def test_linear_is_deterministic(ql):
    w = synth.benq_weights(5120, 5120, seed=5)
    x = synth.activations(1, 5120, seed=6)
    a = _linear(ql, w, x)
    b = _linear(ql, w, x)
    assert torch.equal(a, b)


def test_linear_argument_errors(ql):
    w = synth.benq_weights(8, 64, seed=0)
    x = bf16(synth.activations(1, 64, seed=0))
    y = torch.empty(1, 8, device="cuda")
    codes, lut = dev(w.codes), bits16(w.lut)
    raw = ql.lib().benq_linear
    s = torch.cuda.current_stream().cuda_stream
    assert raw(codes.data_ptr(), lut.data_ptr(), x.data_ptr() + 2, y.data_ptr(), 0, 1, 8, 64, s) == ql.QL_ERR_ALIGNMENT
    assert raw(codes.data_ptr(), lut.data_ptr(), x.data_ptr(), y.data_ptr(), 0, 1, 8, 62, s) == ql.QL_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        ql.benq_linear(codes, lut, x, torch.empty(2, 8, device="cuda"))


@pytest.mark.parametrize("M,N,K", [(17, 256, 64), (32, 512, 320), (300, 256, 1024), (256, 768, 5120), (513, 1024, 2048)])
def test_gemm_shapes(ql, M, N, K):
    w = synth.benq_weights(N, K, seed=M + N + K)
    x = synth.activations(M, K, seed=M)
    y = _linear(ql, w, x).cpu().numpy()
    assert max_rel(y, ob.linear(w.codes, w.lut, x, K)) <= BENQ_TOL
    yb = _linear(ql, w, x, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(yb, f32_to_bf16_rne(y))


@pytest.mark.parametrize("N,K", [(17408, 5120), (5120, 17408)])
def test_gemm_prefill_shapes_sampled_columns(ql, N, K):
    # 2048-token prefill through the 27B-class gate/up and down projections, bf16 output
    w = synth.benq_weights(N, K, seed=2000 + N // 1024)
    x = synth.activations(2048, K, seed=2100)
    y32 = _linear(ql, w, x).cpu().numpy()
    yb = _linear(ql, w, x, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    cols = np.r_[np.random.default_rng(3).choice(N, 96, replace=False), 0, N - 1]
    ref = ob.linear(w.codes, w.lut, x, K, rows=cols)
    assert max_rel(y32[:, cols], ref) <= BENQ_TOL
    assert np.array_equal(yb, f32_to_bf16_rne(y32))


def _linear_ws(ql, w, xbits, ydtype=torch.float32):
    B = xbits.shape[0]
    nbytes = ql.benq_linear_workspace_bytes(B, w.N, xbits.shape[1])
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda") if nbytes else None
    y = torch.empty(B, w.N, dtype=ydtype, device="cuda")
    ql.benq_linear(dev(w.codes), bits16(w.lut), bf16(xbits), y, workspace=ws)
    torch.cuda.synchronize()
    return y, nbytes


@pytest.mark.parametrize("M,N,K", [(300, 1024, 1024), (1024, 768, 704), (2048, 512, 256)])
def test_gemm_split_last_wave(ql, M, N, K):
    # a single partial wave of pair tiles: every tile is split along K across idle SM pairs
    w = synth.benq_weights(N, K, seed=M + 3 * N + K)
    x = synth.activations(M, K, seed=M + 1)
    y, nbytes = _linear_ws(ql, w, x)
    assert nbytes > 0
    y = y.cpu().numpy()
    assert max_rel(y, ob.linear(w.codes, w.lut, x, K)) <= BENQ_TOL
    y_plain = _linear(ql, w, x).cpu().numpy()
    assert np.max(np.abs(y - y_plain)) <= 1e-5 * np.max(np.abs(y_plain))   # only the fp32 summation order differs
    yb, _ = _linear_ws(ql, w, x, torch.bfloat16)
    assert np.array_equal(yb.cpu().view(torch.int16).numpy().view(np.uint16), f32_to_bf16_rne(y))


def test_gemm_split_repeated_calls_are_identical(ql):
    # the per-tile counters are reset by the last part, so back-to-back calls on one workspace agree bit for bit
    M, N, K = 600, 1024, 2048
    w = synth.benq_weights(N, K, seed=77)
    xb = bf16(synth.activations(M, K, seed=78))
    codes, lut = dev(w.codes), bits16(w.lut)
    ws = torch.empty(ql.benq_linear_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    ys = [torch.empty(M, N, device="cuda") for _ in range(4)]
    for y in ys:
        ql.benq_linear(codes, lut, xb, y, workspace=ws)
    torch.cuda.synchronize()
    ql.ql_check()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])


def test_gemm_down_projection_split_sampled_columns(ql):
    # 2048 x 17408 -> 5120: 80 pair tiles, the last partial wave split along K
    N, K = 5120, 17408
    w = synth.benq_weights(N, K, seed=2000 + N // 1024)
    x = synth.activations(2048, K, seed=2100)
    y, nbytes = _linear_ws(ql, w, x)
    y = y.cpu().numpy()
    cols = np.r_[np.random.default_rng(5).choice(N, 64, replace=False), 0, N - 1]
    assert max_rel(y[:, cols], ob.linear(w.codes, w.lut, x, K, rows=cols)) <= BENQ_TOL


def test_workspace_arguments(ql):
    assert ql.benq_linear_workspace_bytes(16, 1024, 1024) == 0      # GEMV: no workspace
    codes = torch.zeros(256, 48, dtype=torch.uint8, device="cuda")
    lut = torch.zeros(256, 64, dtype=torch.int16, device="cuda")
    x = torch.zeros(32, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(32, 256, device="cuda")
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    raw = ql.lib().benq_linear_ws
    s = torch.cuda.current_stream().cuda_stream
    args = (codes.data_ptr(), lut.data_ptr(), x.data_ptr(), y.data_ptr(), 0, 32, 256, 64)
    assert raw(*args, ws.data_ptr(), 0, s) == ql.QL_ERR_INVALID_ARG
    assert raw(*args, None, 4096, s) == ql.QL_ERR_INVALID_ARG
    assert raw(*args, ws.data_ptr() + 16, 1024, s) == ql.QL_ERR_ALIGNMENT
    assert raw(*args, ws.data_ptr(), 4096, s) == ql.QL_OK     # too small for a split: whole tiles
    torch.cuda.synchronize()


@pytest.mark.parametrize("B,K,Ns", [(1, 5120, (5120, 1024, 1024)), (1, 2048, (8, 4, 100, 36)), (1, 1024, (4,)),
                                    (3, 2048, (64, 32)), (1, 1000, (16, 8)), (20, 512, (256, 512))])
def test_linear_multi_matches_each_layer(ql, B, K, Ns):
    # several layers that read the same x (the attention projections q, k, v of the 27B-class layer
    # first): every output equals benq_linear's result for that layer bit for bit, and the oracle's
    # within the bar; batch 1 with K % 1024 == 0 runs one launch, the other shapes one call per layer
    ws = [synth.benq_weights(N, K, seed=17 * N + K + i) for i, N in enumerate(Ns)]
    x = synth.activations(B, K, seed=K + B)
    xd = bf16(x)
    for dt in (torch.float32, torch.bfloat16):
        ys = [torch.full((B, w.N), float("nan"), dtype=dt, device="cuda") for w in ws]
        ql.benq_linear_multi([(dev(w.codes), bits16(w.lut), y) for w, y in zip(ws, ys)], xd)
        for w, y in zip(ws, ys):
            ref = torch.empty(B, w.N, dtype=dt, device="cuda")
            ql.benq_linear(dev(w.codes), bits16(w.lut), xd, ref)
            torch.cuda.synchronize()
            assert torch.equal(y, ref)
            if dt == torch.float32:
                assert max_rel(y.cpu().numpy(), ob.linear(w.codes, w.lut, x, K)) <= BENQ_TOL


def test_linear_multi_argument_errors(ql):
    w = synth.benq_weights(8, 1024, seed=3)
    x = bf16(synth.activations(1, 1024, seed=4))
    y = torch.empty(1, 8, device="cuda")
    with pytest.raises(ValueError):
        ql.benq_linear_multi([], x)
    with pytest.raises(ValueError):
        ql.benq_linear_multi([(dev(w.codes), bits16(w.lut), y)] * 5, x)
    arr = (ql.BenQLayerC * 1)()
    arr[0] = ql.BenQLayerC(dev(w.codes).data_ptr(), bits16(w.lut).data_ptr(), y.data_ptr() + 4, 8)
    s = torch.cuda.current_stream().cuda_stream
    assert ql.lib().benq_linear_multi(arr, 1, x.data_ptr(), ql.QL_OUT_F32, 1, 1024, s) == ql.QL_ERR_ALIGNMENT
    assert ql.lib().benq_linear_multi(arr, 0, x.data_ptr(), ql.QL_OUT_F32, 1, 1024, s) == ql.QL_ERR_INVALID_ARG


def test_linear_batch1_long_rows_are_deterministic(ql):
    # the warps' partial row sums are added in a fixed order
    w = synth.benq_weights(4096, 17408, seed=77)
    x = synth.activations(1, 17408, seed=78)
    a = _linear(ql, w, x)
    for _ in range(3):
        assert torch.equal(_linear(ql, w, x), a)
