"""bench.py's multi-rank path on CPU: two gloo ranks, as torchrun would start them.

Every rank must receive the slowest rank's time (the bench's max over ranks), and the whole-job
value must count every rank's bytes against that time (weak scaling).  The reference arm prints
on rank 0 only.
"""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(times[rank], world)
        out.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [3.25, 7.5]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 7.5, 1: 7.5}


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(4.0, 1) == 4.0


@pytest.mark.parametrize("world", [1, 2, 8])
def test_job_throughput_counts_every_rank(world):
    # 1 GB per step per rank, 10 steps in 100 ms -> 100 GB/s per rank
    assert bench.job_throughput(1e9, 10, 100.0, world) == pytest.approx(100.0 * world)


def test_reference_arm_prints_on_rank_zero_only(capsys):
    class A:
        workload, steps, warmup, gpus = "decode", 1, 0, 2
    bench.run_reference(A, rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_reference_arm_line_carries_the_contract_keys(capsys):
    # rank 0 prints one JSON line: the oracle timed on the host cores, with the keys the bench
    # contract asks of the reference arm
    class A:
        workload, steps, warmup, gpus = "decode", 1, 0, 1
    bench.run_reference(A, rank=0, world=1)
    lines = [s for s in capsys.readouterr().out.splitlines() if s.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["value"] > 0 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 1, 0) and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "decode" and d["data"] == "synthetic"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
