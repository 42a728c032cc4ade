"""mdbf_linear_noalloc: the entry point for callers that cannot allocate device memory.

Some callers may not call cudaMalloc (allocator-internal code, real-time threads that must not
block in the driver, hosts with a memory budget fixed at start-up).  mdbf_linear_noalloc serves
them from a fixed scratch array compiled into the library.  This test calls it through the C ABI
on each of the paths its scratch feeds -- the batch decode kernels, the split G stage on long sign
rows, the envelope chunks of l > 32, and the tensor-core GEMMs whose split counters live in the
scratch -- twice in a row on different
inputs, so stale scratch from one call cannot leak into the next.  Each result is checked against
the oracle (within the MDBF tolerance) and against mdbf_linear, the workspace entry point (bit for
bit).  The file is collected last and passes alone or after the other tests.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import mdbf as om
from tests.qlhelpers import MDBF_TOL, bf16, max_rel, mdbf_dev_paths

pytestmark = pytest.mark.gpu

# (n, m, r, l, P, B, seed): decode kernels (l*B <= 64), envelope chunks (l > 32), the tensor
# cores (l*B > 64 with n, m, r >= 64) on a layer small enough for the array whose two K blocks per
# GEMM make both GEMMs split their last wave, so the split counters in the scratch are used, and
# the split s8 G stage (m >= 8192: quantised z, slice partials and arrival counts in the scratch)
PROBLEMS = [(1024, 768, 300, 4, 2, 3, 71), (640, 1280, 257, 2, 1, 16, 72),
            (256, 256, 128, 40, 1, 2, 74), (300, 128, 64, 4, 2, 20, 73), (256, 8192, 128, 4, 1, 1, 75)]


def _reference(ql, paths_c, n, m, r, l, x):
    B = x.shape[0]
    ws = torch.empty(ql.mdbf_workspace_bytes(len(paths_c), n, m, r, l, B), dtype=torch.uint8, device="cuda")
    y = torch.empty(B, n, device="cuda")
    ql.mdbf_linear(paths_c, n, m, r, l, x, y, ws)
    return y


def _noalloc_raw(ql, paths_c, n, m, r, l, x, y):
    f = ql.lib().mdbf_linear_noalloc
    return f(paths_c, len(paths_c), n, m, r, l, x.data_ptr(), y.data_ptr(), ql.QL_OUT_F32, x.shape[0],
             torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("n,m,r,l,P,B,seed", PROBLEMS)
def test_noalloc_matches_oracle_and_workspace_entry_on_two_calls(ql, n, m, r, l, P, B, seed):
    paths = synth.mdbf_paths(P, n, m, r, l, seed=seed)
    dp = mdbf_dev_paths(paths)
    pc = ql.mdbf_paths_c(dp)
    assert ql.mdbf_workspace_bytes(P, n, m, r, l, B) <= ql.mdbf_noalloc_scratch_bytes()
    for call in range(2):
        x_h = synth.activations(B, m, seed=seed + 1 + call)
        x = bf16(x_h)
        y = torch.full((B, n), float("nan"), device="cuda")
        assert _noalloc_raw(ql, pc, n, m, r, l, x, y) == ql.QL_OK
        y_ref = _reference(ql, pc, n, m, r, l, x)
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        assert np.isfinite(got).all()
        assert max_rel(got, om.linear_factored(paths, n, m, r, x_h)) <= MDBF_TOL
        assert torch.equal(y, y_ref)


def test_noalloc_rejects_sizes_beyond_the_scratch(ql):
    n = m = 4096
    r, l, P, B = 4096, 8, 8, 8                 # needs far more than the static array
    assert ql.mdbf_workspace_bytes(P, n, m, r, l, B) > ql.mdbf_noalloc_scratch_bytes()
    A = 1 << 20                                # never dereferenced: rejected before any launch
    arr = (ql.MDBFPathC * P)()
    for p in range(P):
        arr[p] = ql.MDBFPathC(A, A, 512, 512, A, A, A, A)
    status = ql.lib().mdbf_linear_noalloc(arr, P, n, m, r, l, A, A, ql.QL_OUT_F32, B, None)
    assert status == ql.QL_ERR_UNSUPPORTED
    assert b"scratch" in ql.lib().ql_last_error()
