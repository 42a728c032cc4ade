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


def test_both_arms_print_the_same_config(capsys):
    # the reference arm's config is the GPU arm's (same workload keys, layers and L2 note)
    class A:
        workload, steps, warmup, gpus = "decode", 1, 0, 1
    bench.run_reference(A, rank=0, world=1)
    d = json.loads([s for s in capsys.readouterr().out.splitlines() if s.strip()][0])
    assert d["config"] == bench.line_config("decode", 1)
    assert d["config"]["layers"] == [L["label"] for L in bench.DECODE]


def test_alu_peak_is_the_fp32_lane_rate():
    # 148 SMs x 128 fp32 lanes x 1965 MHz, one add per lane per clock
    peaks = {"sm_max_mhz": 1965.0}
    assert bench.alu_peak_tadds(peaks) == pytest.approx(148 * 128 * 1965e6 / 1e12)


def test_mdbf_decode_roofline_is_the_larger_of_hbm_and_alu_time():
    peaks = {"hbm_gbs": 6551.0, "bf16_tflops": 1674.6, "sm_max_mhz": 1965.0, "source": "measured"}
    L = bench.L_mdbf(2, 17408, 5120, 2886, 4, 1, 1, "gate")     # the 27B MLP gate at batch 1
    adds = bench.mdbf_adds(17408, 5120, 2886, 4, 2, 1)
    assert adds == 2 * 4 * 1 * 2886 * (17408 + 5120)
    t_hbm = bench.layer_bytes(L) / (6551.0 * 1e3)
    t_alu = adds / (bench.alu_peak_tadds(peaks) * 1e6)
    assert t_alu > t_hbm                                          # signed adds bind at batch 1
    r = bench.roofline([L], 28.0, peaks)
    assert r["bound"] == "alu" and r["unit"] == "T add/s"
    assert r["frac"] == pytest.approx(max(t_hbm, t_alu) / 28.0)
    assert r["hbm_frac"] == pytest.approx(t_hbm / 28.0) and r["alu_frac"] == pytest.approx(t_alu / 28.0)


def test_gemv_and_gemm_rooflines():
    peaks = {"hbm_gbs": 6551.0, "bf16_tflops": 1674.6, "sm_max_mhz": 1965.0, "source": "measured"}
    r = bench.roofline(bench.DECODE, 40.0, peaks)
    byts = sum(bench.layer_bytes(L) for L in bench.DECODE)
    assert r["bound"] == "hbm" and r["frac"] == pytest.approx(byts / 40.0 / 1e3 / 6551.0)
    pre = bench.RECORDS["prefill"][0][1][0][1]
    r = bench.roofline(pre, 600.0, peaks)
    fl = sum(2.0 * L["B"] * L["N"] * L["K"] for L in pre)
    assert r["bound"] == "tensor" and r["frac"] == pytest.approx(fl / 600.0 / 1e6 / 1674.6)
    mixed = bench.layer_set(True, "mdbf")
    r = bench.roofline(mixed, 120.0, peaks)
    assert r["bound"] == "mixed"
    assert r["frac"] == pytest.approx(sum(bench.layer_ideal_us(L, peaks) for L in mixed) / 120.0)


def test_default_run_covers_every_configuration():
    recs = bench.line_config("all", 1)["records"]
    for key in ("cfg0_benq_256x512", "cfg1_decode_27b", "cfg2_prefill_m2048", "cfg3_mdbf_4096", "cfg4_layer_27b"):
        assert any(r.startswith(key + "/") for r in recs)
    # the 27B decoder layer: BenQ q/o 5120->5120, k/v 5120->1024, gate/up 5120->17408, down 17408->5120
    seven = bench.layer_set(True, "benq")
    assert [(L["N"], L["K"]) for L in seven] == [(5120, 5120), (1024, 5120), (1024, 5120), (5120, 5120),
                                                 (17408, 5120), (17408, 5120), (5120, 17408)]
    assert sum(bench.layer_weight_bytes(L) for L in seven) == pytest.approx(254.6e6, rel=1e-3)
