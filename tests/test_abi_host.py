"""The C ABI loads, exports every declared entry point, and its host-only logic is right (CPU only).

No call here launches a kernel: argument errors are caught on the host before
any CUDA call, and the accounting functions are host code.
"""
import ctypes
import os
import re
import warnings
from fractions import Fraction

import numpy as np
import torch
import pytest

from oracle import accounting as acc

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "qlinear.h")


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"QL_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"benq_linear", "benq_dequant_debug", "mdbf_linear", "mdbf_dequant_debug",
            "mdbf_workspace_bytes", "ql_last_error"} <= names


def test_library_exports_every_declared_symbol(ql):
    lib = ql.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in ql._SIGNATURES, name


def test_benq_bits_per_weight_matches_oracle(ql):
    for K in (4, 512, 5120, 17408, 30000):
        assert ql.benq_bits_per_weight(K) == pytest.approx(acc.benq_bits_per_weight(K), rel=1e-15)


def test_mdbf_effective_bits_matches_oracle(ql):
    rng = np.random.default_rng(0)
    for _ in range(200):
        n, m = (int(v) for v in rng.integers(1, 20000, 2))
        r = int(rng.integers(1, min(n, m) + 1))
        P, l, sb = int(rng.integers(1, 3)), int(rng.integers(1, 9)), int(rng.choice([0, 8, 16]))
        assert ql.mdbf_effective_bits(n, m, r, P, l, sb) == pytest.approx(float(acc.mdbf_b_eff(n, m, r, P, l, sb)), rel=1e-13)


def test_mdbf_select_rank_matches_oracle(ql):
    assert ql.mdbf_select_rank(4096, 4096, 1, 2, 16, 1.0) == (2000, False)
    assert ql.mdbf_select_rank(17408, 5120, 2, 4, 16, 1.5) == (2886, False)
    assert ql.mdbf_select_rank(5120, 17408, 2, 4, 16, 1.5) == (2886, False)
    rng = np.random.default_rng(1)
    for _ in range(300):
        n, m = (int(v) for v in rng.integers(64, 20000, 2))
        P, l, sb = int(rng.integers(1, 3)), int(rng.integers(1, 9)), int(rng.choice([0, 8, 16]))
        b = float(rng.uniform(0.3, 2.5))
        rr = acc.mdbf_rank_real(n, m, b, P, l, sb)
        if abs(rr - round(rr)) < Fraction(1, 10 ** 6):
            continue            # a float evaluation may land either side of an exact integer
        try:
            with warnings.catch_warnings():
                warnings.simplefilter("ignore")
                want = acc.mdbf_select_rank(n, m, b, P, l, sb)
        except ValueError:
            with pytest.raises(ql.QLinearError):
                ql.mdbf_select_rank(n, m, P, l, sb, b)
            continue
        assert ql.mdbf_select_rank(n, m, P, l, sb, b) == want


def test_mdbf_workspace_bytes(ql):
    assert ql.mdbf_workspace_bytes(0, 1, 1, 1, 1, 1) == 0
    ws = ql.mdbf_workspace_bytes(2, 17408, 5120, 2886, 4, 1)
    assert ws >= 4 * 2 * 4 * (5120 + 2886) and ws % 256 == 0


def _raw(ql, name):
    return getattr(ql.lib(), name)


def test_benq_argument_errors_are_caught_on_the_host(ql):
    f = _raw(ql, "benq_linear")
    A = 1 << 20    # never dereferenced: every call below fails validation first
    assert f(None, A, A, A, 0, 1, 8, 8, None) == ql.QL_ERR_INVALID_ARG
    assert f(A, A, A, A, 0, 0, 8, 8, None) == ql.QL_ERR_INVALID_ARG
    assert f(A, A, A, A, 0, 1, 8, 6, None) == ql.QL_ERR_INVALID_ARG           # K % 4
    assert f(A, A, A + 2, A, 0, 1, 8, 8, None) == ql.QL_ERR_ALIGNMENT
    assert f(A, A, A, A, 7, 1, 8, 8, None) == ql.QL_ERR_INVALID_ARG           # y dtype
    assert f(A, A, A, A, 0, 32, 8, 40, None) == ql.QL_ERR_UNSUPPORTED         # GEMM needs K % 64
    assert b"K % 64" in _raw(ql, "ql_last_error")() or b"K %% 64" in _raw(ql, "ql_last_error")()
    g = _raw(ql, "benq_dequant_debug")
    assert g(A, A, None, 4, 8, None) == ql.QL_ERR_INVALID_ARG
    assert g(A, A, A, 4, 10, None) == ql.QL_ERR_INVALID_ARG


def test_multi_argument_errors_are_caught_on_the_host(ql):
    f = _raw(ql, "benq_linear_multi")
    A = 1 << 20    # never dereferenced: every call below fails validation first
    arr = (ql.BenQLayerC * 5)()
    for i in range(5):
        arr[i] = ql.BenQLayerC(A, A, A, 8)
    assert f(None, 1, A, 0, 1, 8, None) == ql.QL_ERR_INVALID_ARG              # no layers
    assert f(arr, 0, A, 0, 1, 8, None) == ql.QL_ERR_INVALID_ARG               # S < 1
    assert f(arr, 5, A, 0, 1, 8, None) == ql.QL_ERR_INVALID_ARG               # S > 4
    assert f(arr, 2, A, 0, 1, 6, None) == ql.QL_ERR_INVALID_ARG               # K % 4
    assert f(arr, 2, A + 2, 0, 1, 8, None) == ql.QL_ERR_ALIGNMENT             # x
    arr[1] = ql.BenQLayerC(A, A, A + 4, 8)
    assert f(arr, 2, A, 0, 1, 8, None) == ql.QL_ERR_ALIGNMENT                 # y of layer 1
    arr[1] = ql.BenQLayerC(A, None, A, 8)
    assert f(arr, 2, A, 0, 1, 8, None) == ql.QL_ERR_INVALID_ARG               # null table
    arr[1] = ql.BenQLayerC(A, A, A, 0)
    assert f(arr, 2, A, 0, 1, 8, None) == ql.QL_ERR_INVALID_ARG               # N
    arr[1] = ql.BenQLayerC(A, A, A, 8)
    assert f(arr, 2, A, 0, 32, 40, None) == ql.QL_ERR_UNSUPPORTED             # GEMM needs K % 64


def test_mlp_argument_errors_are_caught_on_the_host(ql):
    f = _raw(ql, "benq_mlp_gate_up")
    A = 1 << 20    # never dereferenced: every call below fails validation first
    assert ql.benq_mlp_workspace_bytes(1, 512, 1024) == 0                         # fused batch-1 kernel
    need = ql.benq_mlp_workspace_bytes(4, 512, 1024)
    assert need >= 2 * 4 * 512 * 4
    assert f(A, A, None, A, A, A, 0, 1, 512, 1024, None, 0, None) == ql.QL_ERR_INVALID_ARG
    assert f(A, A, A, A, A, A, 0, 1, 512, 1022, None, 0, None) == ql.QL_ERR_INVALID_ARG   # K % 4
    assert f(A, A, A + 4, A, A, A, 0, 1, 512, 1024, None, 0, None) == ql.QL_ERR_ALIGNMENT
    assert f(A, A, A, A, A, A, 5, 1, 512, 1024, None, 0, None) == ql.QL_ERR_INVALID_ARG     # h dtype
    assert f(A, A, A, A, A, A, 0, 4, 512, 1024, A, need - 256, None) == ql.QL_ERR_INVALID_ARG  # workspace
    assert f(A, A, A, A, A, A, 0, 4, 512, 1024, None, 0, None) == ql.QL_ERR_INVALID_ARG      # none given
    assert f(A, A, A, A, A, A, 0, 4, 512, 1024, A + 64, need, None) == ql.QL_ERR_ALIGNMENT   # ws 256
    assert f(A, A, A, A, A, A, 0, 32, 512, 1000, A, 1 << 30, None) == ql.QL_ERR_UNSUPPORTED  # GEMM K % 64


def _fake_paths(ql, P, ldSA=16, ldSB=16, base=1 << 20):
    arr = (ql.MDBFPathC * P)()
    for p in range(P):
        arr[p] = ql.MDBFPathC(base, base, ldSA, ldSB, base, base, base, base)
    return arr


def test_mdbf_argument_errors_are_caught_on_the_host(ql):
    f = _raw(ql, "mdbf_linear")
    A = 1 << 20
    ok = _fake_paths(ql, 1)
    ws = ql.mdbf_workspace_bytes(1, 64, 64, 32, 2, 1)
    assert f(None, 1, 64, 64, 32, 2, A, A, 0, 1, A, ws, None) == ql.QL_ERR_INVALID_ARG
    assert f(ok, 1, 64, 64, 65, 2, A, A, 0, 1, A, ws, None) == ql.QL_ERR_INVALID_ARG        # r > min(n, m)
    assert f(ok, 1, 64, 64, 32, 2, A, A, 0, 1, A, ws - 1, None) == ql.QL_ERR_INVALID_ARG    # workspace
    assert f(ok, 1, 64, 64, 32, 2, A, A, 0, 1, A + 16, ws, None) == ql.QL_ERR_ALIGNMENT     # workspace 256
    assert f(_fake_paths(ql, 1, ldSA=2), 1, 64, 64, 32, 2, A, A, 0, 1, A, ws, None) == ql.QL_ERR_INVALID_ARG
    assert f(_fake_paths(ql, 1, ldSB=10), 1, 64, 64, 32, 2, A, A, 0, 1, A, ws, None) == ql.QL_ERR_ALIGNMENT
    # l * B > 64 runs on the tensor cores: its workspace holds at least X' and T' in fp16
    # (B x m and B x r rounded up to 64 columns)
    big = ql.mdbf_workspace_bytes(1, 64, 64, 64, 8, 9)
    assert big >= 9 * 64 * 2 * 2 and big > ws
    assert f(ok, 1, 64, 64, 64, 8, A, A, 0, 9, A, big - 1, None) == ql.QL_ERR_INVALID_ARG  # workspace
    ws65 = ql.mdbf_workspace_bytes(1, 64, 64, 32, 65, 1)
    assert f(ok, 1, 64, 64, 32, 65, A, A, 0, 1, A, ws65, None) == ql.QL_ERR_UNSUPPORTED    # l > 64
    g = _raw(ql, "mdbf_dequant_debug")
    assert g(ok, 1, 64, 64, 32, 2, None, None, None, None) == ql.QL_ERR_INVALID_ARG


def test_mdbf_multi_argument_errors_are_caught_on_the_host(ql):
    f = _raw(ql, "mdbf_linear_multi")
    A = 1 << 20    # never dereferenced: every call below fails validation first
    ok = _fake_paths(ql, 8)
    ws = ql.mdbf_workspace_bytes(4, 64, 64, 32, 2, 1)
    ys = (ctypes.c_void_p * 4)(A, A, A, A)
    assert f(ok, 0, 2, 64, 64, 32, 2, A, ys, 0, 1, A, ws, None) == ql.QL_ERR_INVALID_ARG    # S < 1
    assert f(ok, 5, 1, 64, 64, 32, 2, A, ys, 0, 1, A, ws, None) == ql.QL_ERR_INVALID_ARG    # S > 4
    assert f(ok, 3, 3, 64, 64, 32, 2, A, ys, 0, 1, A, ws, None) == ql.QL_ERR_INVALID_ARG    # S * P > 8
    assert f(None, 2, 2, 64, 64, 32, 2, A, ys, 0, 1, A, ws, None) == ql.QL_ERR_INVALID_ARG  # no paths
    assert f(ok, 2, 2, 64, 64, 32, 2, A, None, 0, 1, A, ws, None) == ql.QL_ERR_INVALID_ARG  # no outputs
    assert f(ok, 2, 2, 64, 64, 32, 2, A, ys, 0, 1, A, ws - 1, None) == ql.QL_ERR_INVALID_ARG   # workspace
    assert f(ok, 2, 2, 64, 64, 32, 2, A + 1, ys, 0, 1, A, ws, None) == ql.QL_ERR_ALIGNMENT     # x
    bad = (ctypes.c_void_p * 2)(A, A + 2)
    assert f(ok, 2, 2, 64, 64, 32, 2, A, bad, 0, 1, A, ws, None) == ql.QL_ERR_ALIGNMENT        # y of layer 1
    none = (ctypes.c_void_p * 2)(A, None)
    assert f(ok, 2, 2, 64, 64, 32, 2, A, none, 0, 1, A, ws, None) == ql.QL_ERR_INVALID_ARG     # null y
    paths = _fake_paths(ql, 4)
    paths[3] = ql.MDBFPathC(A, A, 2, 16, A, A, A, A)
    assert f(paths, 2, 2, 64, 64, 32, 2, A, ys, 0, 1, A, ws, None) == ql.QL_ERR_INVALID_ARG    # stride of path 3


def test_binding_fails_loudly_without_the_library(ql, monkeypatch, tmp_path):
    monkeypatch.setattr(ql, "_lib", None)
    monkeypatch.setattr(ql, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        ql.benq_bits_per_weight(64)


def test_binding_refuses_host_tensors(ql):
    # the Python binding hands the library device addresses only: a host tensor is refused before
    # any call into the library could launch a kernel on it
    K, N = 8, 4
    codes = torch.zeros(N, 3 * K // 4, dtype=torch.uint8)
    lut = torch.zeros(N, 64, dtype=torch.bfloat16)
    x = torch.zeros(1, K, dtype=torch.bfloat16)
    y = torch.zeros(1, N)
    with pytest.raises(ValueError, match="CUDA tensors"):
        ql.benq_linear(codes, lut, x, y)
    with pytest.raises(ValueError, match="CUDA tensors"):
        ql.benq_mlp_gate_up(codes, lut, codes, lut, x, y)
    with pytest.raises(ValueError, match="CUDA tensors"):
        ql.mdbf_paths_c([{"S_A": codes, "S_B": codes, "A_amp": lut, "B_amp": lut, "Q_U": lut, "Q_V": lut}])
