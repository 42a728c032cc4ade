"""Back-to-back calls on one stream, each consuming the previous call's output.

Every kernel is launched with programmatic dependent launch: it may start while the kernel
before it in the stream is still running, reads only weights until it has waited for that
kernel, and reads activations or writes outputs only after the wait.  These chains feed each
output (bf16) straight into the next call with no host synchronisation, repeat the chain many
times back to back, and require the results to be bit-identical to the same chain run with
overlap disabled.  They also check that the switch reports and restores its setting.
"""
import numpy as np
import pytest
import torch

import synth
from tests.qlhelpers import bf16, bits16, dev, mdbf_dev_paths

pytestmark = pytest.mark.gpu


def _benq(N, K, seed):
    w = synth.benq_weights(N, K, seed=seed)
    return dev(w.codes), bits16(w.lut)


def _run(ql, chain, x0, reps, sync_each):
    outs = []
    for _ in range(reps):
        x = x0
        for f in chain:
            x = f(x)
            if sync_each:
                torch.cuda.synchronize()
        outs.append(x.clone())
    torch.cuda.synchronize()
    return outs


def _compare(ql, chain, x0, reps=8):
    prev = ql.ql_set_pdl(True)
    try:
        fast = _run(ql, chain, x0, reps, sync_each=False)
        ql.ql_set_pdl(False)
        slow = _run(ql, chain, x0, 1, sync_each=True)[0]
    finally:
        ql.ql_set_pdl(prev)
    assert torch.isfinite(slow.float()).all()
    for o in fast:
        assert torch.equal(o, slow)


def _benq_fn(ql, N, K, seed, B):
    codes, lut = _benq(N, K, seed)
    ys = [torch.empty(B, N, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    state = {"i": 0}

    def f(x):
        y = ys[state["i"] % 2]          # alternate output buffers so a write never lands on a buffer still being read
        state["i"] += 1
        ql.benq_linear(codes, lut, x, y)
        return y
    return f


def _mdbf_fn(ql, n, m, r, l, P, B, seed):
    paths = synth.mdbf_paths(P, n, m, r, l, seed=seed)
    dp = mdbf_dev_paths(paths)
    ws = torch.empty(ql.mdbf_workspace_bytes(P, n, m, r, l, B), dtype=torch.uint8, device="cuda")
    ys = [torch.empty(B, n, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    state = {"i": 0}

    def f(x):
        y = ys[state["i"] % 2]
        state["i"] += 1
        ql.mdbf_linear(dp, n, m, r, l, x, y, ws)
        return y
    return f


def test_decode_gemv_chain(ql):
    chain = [_benq_fn(ql, 4096, 1024, 901, 1), _benq_fn(ql, 1024, 4096, 902, 1), _benq_fn(ql, 2048, 1024, 903, 1)]
    _compare(ql, chain, bf16(synth.activations(1, 1024, seed=904)))


def test_small_batch_gemv_chain(ql):
    chain = [_benq_fn(ql, 1536, 2048, 911, 5), _benq_fn(ql, 2048, 1536, 912, 5)]
    _compare(ql, chain, bf16(synth.activations(5, 2048, seed=913)))


def test_prefill_gemm_chain(ql):
    chain = [_benq_fn(ql, 1024, 512, 921, 300), _benq_fn(ql, 512, 1024, 922, 300)]
    _compare(ql, chain, bf16(synth.activations(300, 512, seed=923)), reps=4)


def test_mdbf_chain(ql):
    chain = [_mdbf_fn(ql, 1024, 768, 300, 4, 2, 1, 931), _mdbf_fn(ql, 768, 1024, 300, 4, 2, 1, 932)]
    _compare(ql, chain, bf16(synth.activations(1, 768, seed=933)))


def test_mixed_chain(ql):
    chain = [_benq_fn(ql, 1024, 2048, 941, 2), _mdbf_fn(ql, 2048, 1024, 512, 4, 2, 2, 942),
             _benq_fn(ql, 1024, 2048, 943, 2)]
    _compare(ql, chain, bf16(synth.activations(2, 2048, seed=944)))


def test_batched_mdbf_chain(ql):
    # prefill-sized batches: BenQ GEMM -> MDBF on the tensor cores (4 launches per call, l = 4 with its
    # workspace column pairs; l = 6 on the warp-MMA decoders) -> BenQ GEMM
    chain = [_benq_fn(ql, 1024, 512, 951, 300), _mdbf_fn(ql, 768, 1024, 300, 4, 2, 300, 952),
             _mdbf_fn(ql, 512, 768, 256, 6, 2, 300, 953), _benq_fn(ql, 512, 512, 954, 300)]
    _compare(ql, chain, bf16(synth.activations(300, 512, seed=955)), reps=4)


def test_set_pdl_returns_previous(ql):
    prev = ql.ql_set_pdl(False)
    try:
        assert ql.ql_set_pdl(True) is False
        assert ql.ql_set_pdl(True) is True
    finally:
        ql.ql_set_pdl(prev)


def test_bounded_wait_runs_out_and_the_context_survives(ql):
    # a wait on a barrier that nothing arrives on gives up (~10 ms), the flag reaches ql_check, the
    # next check is clean, and the library keeps working on the same context
    ql.ql_check()
    ql.ql_selftest_timeout()
    with pytest.raises(ql.QLinearError) as e:
        ql.ql_check()
    assert e.value.status == ql.QL_ERR_TIMEOUT
    ql.ql_check()
    codes, lut = _benq(256, 1024, 961)
    x = bf16(synth.activations(1, 1024, seed=962))
    y = torch.empty(1, 256, device="cuda")
    ql.benq_linear(codes, lut, x, y)
    ql.ql_check()
    from oracle import benq as ob
    ref = ob.linear(codes.cpu().numpy(), lut.cpu().numpy().view(np.uint16), x.cpu().view(torch.int16).numpy().view(np.uint16), 1024)
    assert np.max(np.abs(y.cpu().numpy() - ref)) <= 2e-3 * np.max(np.abs(ref))
