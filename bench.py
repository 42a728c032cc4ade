"""Benchmark of the weight-only quantized linear layers on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload decode|prefill|mdbf|mdbf_prefill|layer]
                    [--impl ours|reference]

Prints one JSON line.  Workloads (synthetic, seeded; shapes of a 27B-class
decoder layer, hidden 5120, intermediate 17408):

  decode   BenQ 6-bit decode GEMV at batch 1: gate/up 5120->17408 and down
           17408->5120 (one step = one pass of each).  Default.
  prefill  BenQ 6-bit prefill GEMM, 2048 tokens, same two shapes, bf16 output.
  mdbf     MDBF P=2, l=4 at 1.5 bits/weight (rank 2886), gate/up and down, batch 1.
  mdbf_prefill  the same MDBF layers at 2048 tokens (tensor-core path), bf16 output.
  layer    the full decoder-layer linear set at batch 1: BenQ q/k/v/o, gate and up in one
           call with the SiLU gate (benq_mlp_gate_up), down, plus MDBF gate/up/down.

Timing: W untimed warm-up steps, then exactly K steps between a barrier and a
device synchronize on both sides, CUDA events on the launching stream, the max
over ranks.  Weights rotate over enough device copies that every step reads
more than the 126 MB L2 before a copy is reused.  With N > 1 each rank runs an
independent replica of the workload (the layer has no data-path exchange), so
scaling is weak.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-linear GB/s & TFLOP/s vs B200 roofline; decode us per layer"
L2_BYTES = 126 * 1024 * 1024
HIDDEN, INTER = 5120, 17408
MLP_R, MLP_L, MLP_P = 2886, 4, 2


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def benq_bytes(N, K, B, out_bytes=4):
    """Algorithmic bytes of one BenQ call: packed codes, tables, activations, output."""
    return 0.75 * N * K + 128 * N + 2 * B * K + out_bytes * B * N


def mdbf_flops(n, m, r, P, B):
    """Algorithmic FLOPs of one batched MDBF call: the factored contraction, B x m x (P r) for
    T = X G^T and B x (P r) x n for Y = T F^T."""
    return 2.0 * B * P * r * (m + n)


def mdbf_bytes(n, m, r, l, P, B, out_bytes=4):
    """Algorithmic bytes of one MDBF call: both sign matrices, four fp16 envelopes, x and y."""
    signs = P * (n * ((r + 7) // 8) + r * ((m + 7) // 8))
    env = P * 2 * l * (n + m + 2 * r)
    return signs + env + 2 * B * m + out_bytes * B * n


# ---------------------------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _one(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        for bit, name in self.REASONS.items():
            if mask & bit:
                self.reasons.add(name)

    def _loop(self):
        while not self._stop.is_set():
            self._one()
            time.sleep(0.002)

    def __enter__(self):
        if self._nv:
            self._one()
            self._t = threading.Thread(target=self._loop, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._nv:
            self._stop.set()
            self._t.join()
            self._one()

    def summary(self):
        if not self._nv or not self.samples:
            return None
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------------- workloads

class Workload:
    """Device-resident inputs for one workload plus the calls of one step."""

    def __init__(self, name, ql, torch, copies_hint=None):
        import synth
        from tests.qlhelpers import bf16, bits16, dev, f16
        self.name, self.ql, self.torch = name, ql, torch
        self.calls = []          # (label, fn(copy_index), algorithmic bytes, flops)
        self.inputs_h = []       # host copies of step inputs (for the end-to-end number)
        self.outputs = []
        self.desc = {}
        cuda = torch.device("cuda")

        def benq_layer(N, K, B, seed, out_dtype=torch.float32, label=None):
            w = synth.benq_weights(N, K, seed=seed)
            codes, lut = dev(w.codes), bits16(w.lut)
            x_h = synth.activations(B, K, seed=seed + 500)
            x = bf16(x_h)
            y = torch.empty(B, N, dtype=out_dtype, device=cuda)
            nws = ql.benq_linear_workspace_bytes(B, N, K)
            ws = torch.empty(nws, dtype=torch.uint8, device=cuda) if nws else None
            return dict(kind="benq", N=N, K=K, B=B, codes=[codes], lut=[lut], x=x, x_h=x_h, y=y, ws=ws,
                        wbytes=codes.numel() + lut.numel() * 2, label=label or f"benq_{K}x{N}_b{B}")

        def benq_mlp_layer(N, K, seed, label):
            # gate and up of the same input in one call, h = silu(gate) * up (bf16 out)
            wg = synth.benq_weights(N, K, seed=seed)
            wu = synth.benq_weights(N, K, seed=seed + 1)
            x_h = synth.activations(1, K, seed=seed + 500)
            cg, lg, cu, lu = dev(wg.codes), bits16(wg.lut), dev(wu.codes), bits16(wu.lut)
            return dict(kind="benq_mlp", N=N, K=K, B=1, codes=[(cg, lg, cu, lu)], x=bf16(x_h), x_h=x_h,
                        y=torch.empty(1, N, dtype=torch.bfloat16, device=cuda), ws=None,
                        wbytes=2 * (cg.numel() + lg.numel() * 2), label=label)

        def mdbf_layer(n, m, B, seed, label=None, out_dtype=torch.float32):
            paths = synth.mdbf_paths(MLP_P, n, m, MLP_R, MLP_L, seed=seed)
            dps = [dict(S_A=dev(p.S_A), S_B=dev(p.S_B), A_amp=f16(p.A_amp), B_amp=f16(p.B_amp),
                        Q_U=f16(p.Q_U), Q_V=f16(p.Q_V)) for p in paths]
            x_h = synth.activations(B, m, seed=seed + 500)
            ws = torch.empty(ql.mdbf_workspace_bytes(MLP_P, n, m, MLP_R, MLP_L, B), dtype=torch.uint8, device=cuda)
            wbytes = sum(sum(t.numel() * t.element_size() for t in d.values()) for d in dps)
            return dict(kind="mdbf", n=n, m=m, B=B, paths=[dps], x=bf16(x_h), x_h=x_h,
                        y=torch.empty(B, n, dtype=out_dtype, device=cuda), ws=ws, wbytes=wbytes,
                        label=label or f"mdbf_{m}x{n}_b{B}")

        layers = []
        if name == "decode":
            layers = [benq_layer(INTER, HIDDEN, 1, 1001, label="benq_gate_up_5120x17408_b1"),
                      benq_layer(HIDDEN, INTER, 1, 1002, label="benq_down_17408x5120_b1")]
        elif name == "prefill":
            layers = [benq_layer(INTER, HIDDEN, 2048, 2001, torch.bfloat16, "benq_gemm_5120x17408_m2048"),
                      benq_layer(HIDDEN, INTER, 2048, 2002, torch.bfloat16, "benq_gemm_17408x5120_m2048")]
        elif name == "mdbf":
            layers = [mdbf_layer(INTER, HIDDEN, 1, 4001, "mdbf_gate_up_5120x17408_b1"),
                      mdbf_layer(HIDDEN, INTER, 1, 4002, "mdbf_down_17408x5120_b1")]
        elif name == "mdbf_prefill":
            layers = [mdbf_layer(INTER, HIDDEN, 2048, 6001, "mdbf_gemm_5120x17408_m2048", torch.bfloat16),
                      mdbf_layer(HIDDEN, INTER, 2048, 6002, "mdbf_gemm_17408x5120_m2048", torch.bfloat16)]
        elif name == "layer":
            layers = [benq_layer(HIDDEN, HIDDEN, 1, 5001, label="benq_q"),
                      benq_layer(1024, HIDDEN, 1, 5002, label="benq_k"),
                      benq_layer(1024, HIDDEN, 1, 5003, label="benq_v"),
                      benq_layer(HIDDEN, HIDDEN, 1, 5004, label="benq_o"),
                      benq_mlp_layer(INTER, HIDDEN, 5005, "benq_gate_up_silu"),
                      benq_layer(HIDDEN, INTER, 1, 5007, label="benq_down"),
                      mdbf_layer(INTER, HIDDEN, 1, 5008, "mdbf_gate"),
                      mdbf_layer(INTER, HIDDEN, 1, 5009, "mdbf_up"),
                      mdbf_layer(HIDDEN, INTER, 1, 5010, "mdbf_down")]
        else:
            raise SystemExit(f"unknown workload {name}")

        # rotate weight copies so that a copy is reused only after > 2 x L2 of other reads
        per_step = sum(L["wbytes"] for L in layers)
        self.copies = copies_hint or max(1, int(np.ceil(2 * L2_BYTES / per_step)) + 1)
        for L in layers:
            for _ in range(self.copies - 1):
                if L["kind"] == "benq":
                    L["codes"].append(L["codes"][0].clone())
                    L["lut"].append(L["lut"][0].clone())
                elif L["kind"] == "benq_mlp":
                    L["codes"].append(tuple(t.clone() for t in L["codes"][0]))
                else:
                    L["paths"].append([{k: v.clone() for k, v in d.items()} for d in L["paths"][0]])
        self.layers = layers
        self.working_set = per_step * self.copies

    def step_bytes(self):
        tot = 0.0
        for L in self.layers:
            ob = L["y"].element_size()
            if L["kind"] == "benq":
                tot += benq_bytes(L["N"], L["K"], L["B"], ob)
            elif L["kind"] == "benq_mlp":
                tot += 2 * benq_bytes(L["N"], L["K"], L["B"], 0) - 2 * L["B"] * L["K"] + ob * L["B"] * L["N"]
            else:
                tot += mdbf_bytes(L["n"], L["m"], MLP_R, MLP_L, MLP_P, L["B"], ob)
        return tot

    def step_flops(self):
        f = sum(2.0 * L["B"] * L["N"] * L["K"] for L in self.layers if L["kind"] == "benq")
        if self.name == "mdbf_prefill":
            f += sum(mdbf_flops(L["n"], L["m"], MLP_R, MLP_P, L["B"]) for L in self.layers if L["kind"] == "mdbf")
        return f

    def run_layer(self, L, c):
        ql = self.ql
        if L["kind"] == "benq":
            ql.benq_linear(L["codes"][c], L["lut"][c], L["x"], L["y"], workspace=L["ws"])
        elif L["kind"] == "benq_mlp":
            ql.benq_mlp_gate_up(*L["codes"][c], L["x"], L["y"])
        else:
            ql.mdbf_linear(L["paths"][c], L["n"], L["m"], MLP_R, MLP_L, L["x"], L["y"], L["ws"])

    def launches_per_step(self):
        # BenQ: one kernel; MDBF: pack, G stage, F stage, or for batches past the decode kernels
        # envelope prep, activation prep and the two GEMMs
        return sum(1 if L["kind"] in ("benq", "benq_mlp") else (4 if MLP_L * L["B"] > 64 else 3) for L in self.layers)


# the sources each kernel's DRAM-traffic figure depends on
_KERNEL_SOURCES = {
    "benq_gemv": ["benq_gemv.cu", "ql_device.cuh"],
    "benq_gemm": ["benq_gemm_sm100.cu", "pair_gemm.cuh", "sm100_ptx.cuh", "ql_device.cuh"],
    "mdbf_linear": ["mdbf.cu", "ql_device.cuh"],
    "mdbf_gemm": ["mdbf_gemm_sm100.cu", "pair_gemm.cuh", "sm100_ptx.cuh", "ql_device.cuh"],
}


def _kernel_source_sha(kernel_key):
    h = hashlib.sha256()
    d = os.path.join(ROOT, "quantized_linear_b200", "csrc")
    for f in _KERNEL_SOURCES[kernel_key]:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def _traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e or e.get("source_sha") != _kernel_source_sha(kernel_key):
        return None
    return e.get("dram_bytes_per_launch")


def oracle_samples(workload, rows=64, seed=0):
    """A bounded sample of the workload for the oracle: per shape, `rows` output rows with their
    inputs (generated once, outside any timing).  Returns [(label, run, algorithmic bytes)]."""
    import synth
    from oracle import benq as ob
    from oracle import mdbf as om
    rng = np.random.default_rng(seed)
    shapes = {"decode": [("benq", INTER, HIDDEN, 1), ("benq", HIDDEN, INTER, 1)],
              "prefill": [("benq", INTER, HIDDEN, 2048), ("benq", HIDDEN, INTER, 2048)],
              "mdbf": [("mdbf", INTER, HIDDEN, 1), ("mdbf", HIDDEN, INTER, 1)],
              "mdbf_prefill": [("mdbf", INTER, HIDDEN, 2048), ("mdbf", HIDDEN, INTER, 2048)],
              "layer": [("benq", INTER, HIDDEN, 1), ("mdbf", INTER, HIDDEN, 1)]}[workload]
    out = []
    for kind, N, K, B in shapes:
        if kind == "benq":
            bb = min(B, 16)   # prefill: a 16-row slice of the batch (the oracle's cost is linear in it)
            w = synth.benq_weights(rows, K, seed=int(rng.integers(1 << 30)))
            x = synth.activations(bb, K, seed=1)
            out.append((f"benq {rows} rows x K={K}, B={bb}", lambda w=w, x=x, K=K: ob.linear(w.codes, w.lut, x, K),
                        benq_bytes(rows, K, bb)))
        else:
            bb = min(B, 16)   # prefill: a 16-row slice of the batch (the oracle's cost is linear in it)
            paths = synth.mdbf_paths(MLP_P, N, K, MLP_R, MLP_L, seed=7)
            x = synth.activations(bb, K, seed=1)
            sel = np.sort(rng.choice(N, rows, replace=False))
            out.append((f"mdbf {rows} of {N} rows, m={K}, B={bb}",
                        lambda paths=paths, x=x, N=N, K=K, sel=sel: om.linear_factored(paths, N, K, MLP_R, x, rows=sel),
                        mdbf_bytes(rows, K, MLP_R, MLP_L, MLP_P, bb)))
    return out


def time_samples(samples, budget_s):
    """Runs the samples round-robin (single-threaded BLAS) until `budget_s` of oracle time; returns
    (bytes, seconds, runs)."""
    from threadpoolctl import threadpool_limits
    done, t_used, runs = 0.0, 0.0, 0
    with threadpool_limits(limits=1):
        while t_used < budget_s or runs == 0:
            for _, run, nbytes in samples:
                t0 = time.perf_counter()
                run()
                t_used += time.perf_counter() - t0
                done += nbytes
                runs += 1
    return done, t_used, runs


def cpu_baseline(workload, budget_s=10.0):
    """The oracle as it stands, on a bounded sample of the workload's rows, single-threaded BLAS."""
    samples = oracle_samples(workload)
    done, t_used, runs = time_samples(samples, budget_s)
    return {"value": done / t_used / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{runs} runs over {len(samples)} shapes ({samples[0][0]}; ...), {t_used:.1f} s of oracle time"}


def cublas_reference(torch, layers, steps, warmup=3):
    """Dense bf16 GEMMs of the prefill shapes through torch.matmul (cuBLAS) on random dense weights,
    timed the same way (device events, weights larger than L2): a reference point for the tensor-core
    rate at these shapes, not part of the measured path."""
    mats = [(torch.randn(L["B"], L["K"], device="cuda").to(torch.bfloat16),
             torch.randn(L["N"], L["K"], device="cuda").to(torch.bfloat16)) for L in layers]
    out = [torch.empty(L["B"], L["N"], device="cuda", dtype=torch.bfloat16) for L in layers]
    for _ in range(warmup):
        for (a, w), o in zip(mats, out):
            torch.matmul(a, w.t(), out=o)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record()
    for _ in range(steps):
        for (a, w), o in zip(mats, out):
            torch.matmul(a, w.t(), out=o)
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    flops = sum(2.0 * L["B"] * L["N"] * L["K"] for L in layers)
    del mats, out
    return {"us_per_step": 1e3 * ms, "tflops": flops / (ms / 1e3) / 1e12, "what": "torch.matmul bf16 (cuBLAS), same shapes, dense random weights"}


def max_over_ranks(value, world):
    """The largest of the ranks' `value` (a device time in ms), every rank getting the result.
    One rank returns its own value; otherwise an all-reduce on the process group (NCCL: a CUDA
    tensor, gloo: a CPU one)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_step, steps, ms, world):
    """Whole-job GB/s: every rank processes bytes_per_step per step (weak scaling), timed by the
    slowest rank's `ms` for `steps` steps."""
    return world * bytes_per_step * steps / (ms / 1e3) / 1e9


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step is one pass of the oracle over the sample
    (generated once), so the run's length is bounded by the sample, not by the weights' size."""
    if rank != 0:
        return
    samples = oracle_samples(args.workload)
    for _ in range(args.warmup):
        time_samples(samples, 0.0)
    done, t_used = 0.0, 0.0
    t0 = time.perf_counter()   # the timed steps only
    for _ in range(args.steps):
        d, t, _ = time_samples(samples, 0.0)
        done += d
        t_used += t
    t_steps = time.perf_counter() - t0
    v = done / t_used / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * t_steps / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "oracle": "CPU numpy, fp32 W materialised, fp64 contraction"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"one pass per step over {len(samples)} shapes: "
                                       + "; ".join(lbl for lbl, _, _ in samples)},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill", "mdbf", "mdbf_prefill", "layer"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    import quantized_linear_b200 as ql

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    wl = Workload(args.workload, ql, torch)
    stream = torch.cuda.current_stream()
    ncopy = wl.copies

    def step(i):
        c = i % ncopy
        for L in wl.layers:
            wl.run_layer(L, c)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # A decode step is launch-bound at this size, so it is replayed as a CUDA graph: one graph
    # per rotating weight copy, kernels chained by programmatic dependent launch.
    dom = [L for L in wl.layers if L["kind"] == ("benq" if args.workload in ("decode", "prefill", "layer") else "mdbf")]

    def capture(layers, copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for c in copies:
                for L in layers:
                    wl.run_layer(L, c)
        return g

    # one graph per rotation cycle (steps on copies 0 .. ncopy-1), as a model graph holds many
    # layers; single-step graphs cover a remainder so that exactly `steps` steps run
    def graph_set(layers):
        return {"cycle": capture(layers, range(ncopy)), "one": [capture(layers, [c]) for c in range(ncopy)]}

    graphs = graph_set(wl.layers)
    dom_graphs = graphs if len(dom) == len(wl.layers) else graph_set(dom)

    def replay(gs, steps):
        for _ in range(steps // ncopy):
            gs["cycle"].replay()
        for c in range(steps % ncopy):
            gs["one"][c].replay()

    def timed(gs, steps):
        """Replays `steps` steps between two events on the launching stream; returns
        milliseconds, the max over ranks."""
        replay(gs, max(args.warmup, ncopy))
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        start.record(stream)
        replay(gs, steps)
        stop.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return max_over_ranks(start.elapsed_time(stop), world)

    with ClockSampler(torch.cuda.current_device()) as clk:
        ms = timed(graphs, args.steps)
        # the dominant kernel's average duration: its own launches back to back, in the same
        # graphs when the step holds nothing else
        dom_ms = ms if dom_graphs is graphs else timed(dom_graphs, args.steps)
    ms_per_step = ms / args.steps
    step_bytes = wl.step_bytes()
    value = job_throughput(step_bytes, args.steps, ms, world)
    dom_launches = len(dom) * args.steps
    peaks = _peaks()
    if args.workload == "prefill":
        flops = sum(2.0 * L["B"] * L["N"] * L["K"] for L in dom) * args.steps
        achieved = flops / (dom_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": _traffic("benq_gemm"),
                "kernel": "benq_gemm_tcgen05", "avg_launch_us": 1e3 * dom_ms / dom_launches,
                "peak_source": peaks["source"] + " (burst)"}
    elif args.workload == "mdbf_prefill":
        # the whole call (envelope and activation prep plus both GEMMs) against the fp16 dense
        # peak, which equals the bf16 one; FLOPs are those of the factored contraction
        flops = sum(mdbf_flops(L["n"], L["m"], MLP_R, MLP_P, L["B"]) for L in dom) * args.steps
        achieved = flops / (dom_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": _traffic("mdbf_gemm"),
                "kernel": "mdbf_gemm_tcgen05 (2 GEMMs + 2 prep kernels per call)",
                "avg_launch_us": 1e3 * dom_ms / dom_launches, "peak_source": peaks["source"] + " (burst)"}
    else:
        kb = 0.0
        for L in dom:
            ob = L["y"].element_size()
            kb += (benq_bytes(L["N"], L["K"], L["B"], ob) if L["kind"] == "benq"
                   else mdbf_bytes(L["n"], L["m"], MLP_R, MLP_L, MLP_P, L["B"], ob))
        achieved = kb * args.steps / (dom_ms / 1e3) / 1e9
        kname = "benq_gemv" if dom[0]["kind"] == "benq" else "mdbf_linear"
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": _traffic(kname), "kernel": kname,
                "avg_launch_us": 1e3 * dom_ms / dom_launches, "peak_source": peaks["source"] + " (STREAM copy)"}

    # end to end through the public API: pinned host inputs in, results back to pinned host memory
    e2e = None
    try:
        xs_h = [torch.from_numpy(np.ascontiguousarray(L["x_h"]).view(np.int16)).view(torch.bfloat16).pin_memory()
                for L in wl.layers]
        ys_h = [torch.empty(L["y"].shape, dtype=L["y"].dtype).pin_memory() for L in wl.layers]
        h2d = sum(t.numel() * t.element_size() for t in xs_h)
        d2h = sum(t.numel() * t.element_size() for t in ys_h)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(args.steps):
            c = i % ncopy
            for L, xh, yh in zip(wl.layers, xs_h, ys_h):
                L["x"].copy_(xh, non_blocking=True)
                wl.run_layer(L, c)
                yh.copy_(L["y"], non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": job_throughput(step_bytes, args.steps, ems, world), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems / args.steps}
    except Exception as exc:  # pragma: no cover - reported, not hidden
        e2e = {"error": repr(exc)}

    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": {"mdbf": "u1+f16->f32", "mdbf_prefill": "u1+f16->f16 (fp32 accumulate)"}.get(args.workload,
                                                                                            "bf16xu6->f32"),
            "data": "synthetic",
            "config": {"workload": wl.name, "layers": [L["label"] for L in wl.layers],
                       "us_per_step": 1e3 * ms_per_step,
                       "algorithmic_bytes_per_step": step_bytes,
                       "tflops": (wl.step_flops() * args.steps / (ms / 1e3) / 1e12) if wl.step_flops() else None,
                       "l2": f"inputs larger than L2: {ncopy} rotating weight copies, "
                             f"{wl.working_set / 2**20:.0f} MiB working set vs 126 MiB L2",
                       "parallelism": f"replicas x{world}",
                       "launch": f"CUDA graphs of {ncopy} steps (one weight-copy rotation), kernels chained "
                                 "by programmatic dependent launch; e2e uses eager calls"},
            "roofline": roof, "e2e": e2e, "gpu_launches": wl.launches_per_step() * args.steps,
            "clocks": clk.summary()}
    if rank == 0 and world == 1 and args.workload == "prefill":
        line["config"]["cublas_bf16_same_shape"] = cublas_reference(torch, wl.layers, min(args.steps, 20))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs, dom_graphs
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
