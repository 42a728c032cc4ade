"""Benchmark of the weight-only quantized linear layers on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload all|small|decode|prefill|mdbf_square|mdbf_l1|layer|mdbf|mdbf_prefill]
                    [--impl ours|reference] [--no-cpu-baseline]

Prints one JSON line.  The default workload, ``all``, times every configuration of the
benchmark suite in one run; the line's headline (``value``, ``roofline``, ``e2e``) is the
27B-class BenQ decode GEMV and ``workloads`` holds one record per configuration:

  cfg0_benq_256x512   BenQ 6-bit 256 out x 512 in at batch 1 and 8 (launch-latency bound).
  cfg1_decode_27b     BenQ decode GEMV at batch 1: gate/up 5120->17408 and down 17408->5120.
  cfg2_prefill_m2048  BenQ prefill GEMM, 2048 tokens, the same two shapes, bf16 output.
  cfg3_mdbf_4096      MDBF n = m = 4096, P = 1, l = 2, rank 2000 (1.0 bit/weight), batch 1 and 16.
  cfg4_layer_27b      the decoder-layer linear set at batch 1 (q/o 5120->5120, k/v 5120->1024,
                      gate/up 5120->17408, down 17408->5120): BenQ on all seven; BenQ with gate and
                      up fused with the SiLU gate; MDBF (P = 2, l = 4, 1.5 bits/weight, rank 2886) on
                      gate/up/down; and BenQ attention with the MDBF MLP.  Each as a CUDA graph and
                      as separate launches.
  next1_mdbf_prefill  the MDBF MLP projections at 2048 tokens (tensor-core path), bf16 output.
  next4_mdbf_l1_4096  the square layer of cfg3 at l = 1: DBF (P = 1) and LittleBit (P = 2), batch 1 and 16.

The other workload names run one of these alone (``mdbf`` is the MDBF MLP of cfg4).

Timing: W untimed warm-up steps, then exactly K steps between a barrier and a device synchronize
on both sides, CUDA events on the launching stream, the max over ranks.  Workloads whose weights
exceed the L2 rotate over enough device copies that every step reads more than twice the 126 MB
L2 before a copy is reused; the small ones (cfg0, cfg3) write a 256 MiB buffer between steps and
time each step alone.  With N > 1 each rank runs an independent replica (the layer has no
data-path exchange), so scaling is weak.

Inputs: seeded and synthetic.  BenQ weights follow the generator recipe (per-row sigma ~
U(0.01, 0.03), w ~ N(0, sigma), 32 equal-width shells, member-mean levels, nearest-level codes)
with the draws made on the device by torch and the shells, levels and codes made by the
library's own encoder (``benq_encode``, bit-exact to the oracle's); MDBF weights and all
activations come from ``synth``.  The CPU baselines time the oracle on bounded samples made by
``synth``.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-linear GB/s & TFLOP/s vs B200 roofline; decode us per layer"
L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 256 * 1024 * 1024
HIDDEN, INTER = 5120, 17408
MLP_R, MLP_L, MLP_P = 2886, 4, 2         # MDBF at 1.5 bits/weight on the 27B MLP shapes
SQ_N, SQ_R, SQ_L, SQ_P = 4096, 2000, 2, 1  # MDBF square layer, rank 2000 (1.0 bit/weight)
DECODE_VLIM = 64                          # the MDBF decode kernels take l * B <= 64
SM_COUNT, FP32_LANES = 148, 128            # B200: SMs, fp32 lanes per SM


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


def alu_peak_tadds(peaks):
    """Signed fp32 adds per second of the whole part, in T/s: every SM's 128 fp32 lanes retire one
    add per clock at the maximum SM clock (148 x 128 x 1965 MHz = 37.2 T/s)."""
    return SM_COUNT * FP32_LANES * peaks["sm_max_mhz"] * 1e6 / 1e12


# ---------------------------------------------------------------------------------- algorithmic work

def benq_bytes(N, K, B, out_bytes=4):
    """Algorithmic bytes of one BenQ call: packed codes, tables, activations, output."""
    return 0.75 * N * K + 128 * N + 2 * B * K + out_bytes * B * N


def benq_weight_bytes(N, K):
    return 0.75 * N * K + 128 * N


def mdbf_flops(n, m, r, P, B):
    """Algorithmic FLOPs of one batched MDBF call: the factored contraction, B x m x (P r) for
    T = X G^T and B x (P r) x n for Y = T F^T."""
    return 2.0 * B * P * r * (m + n)


def mdbf_adds(n, m, r, l, P, B):
    """Signed adds of one MDBF call evaluated through the factors: the G stage sums l * B vectors
    over every sign of S_B (r x m), the F stage over every sign of S_A (n x r), per path."""
    return float(P) * l * B * r * (n + m)


def mdbf_weight_bytes(n, m, r, l, P):
    """Both packed sign matrices and the four fp16 envelopes of every path."""
    return P * (n * ((r + 7) // 8) + r * ((m + 7) // 8)) + P * 2 * l * (n + m + 2 * r)


def mdbf_bytes(n, m, r, l, P, B, out_bytes=4):
    """Algorithmic bytes of one MDBF call: both sign matrices, four fp16 envelopes, x and y."""
    return mdbf_weight_bytes(n, m, r, l, P) + 2 * B * m + out_bytes * B * n


# ---------------------------------------------------------------------------------- layer specs

def L_benq(N, K, B, seed, label, out="f32"):
    return dict(kind="benq", N=N, K=K, B=B, seed=seed, label=label, out=out)


def L_mlp(N, K, seed_g, seed_u, label):
    """Gate and up projections of the same x in one call, h = silu(gate) * up (bf16 out)."""
    return dict(kind="benq_mlp", N=N, K=K, B=1, seed=seed_g, seed_u=seed_u, label=label, out="bf16")


def L_multi(parts, K, label):
    """BenQ layers of the same K that read the same x, in one call (benq_linear_multi, batch 1);
    parts: [(N, seed, label)]."""
    return dict(kind="benq_multi", parts=parts, N=sum(p[0] for p in parts), K=K, B=1, seed=parts[0][1], label=label,
                out="f32")


def L_mdbf(P, n, m, r, l, B, seed, label, out="f32", group=None, group_skip=False):
    """An MDBF layer.  Layers with the same `group` read one x and run as one mdbf_linear_multi call,
    issued by the first of them (the others have `group_skip`)."""
    return dict(kind="mdbf", P=P, n=n, m=m, r=r, l=l, B=B, seed=seed, label=label, out=out, group=group,
                group_skip=group_skip)


# BenQ weight seeds: one matrix per shape and role, shared between the records that use it
SEED_GATE, SEED_DOWN, SEED_UP = 1001, 1002, 1003


def layer_set(attention, mlp):
    """One decoder layer's linears at batch 1: the BenQ attention projections (q, k, v, o) when
    `attention` ("fused": q, k and v in one call), then the MLP: "benq" (gate, up, down),
    "benq_fused" (gate and up in one call with the SiLU gate, then down), "mdbf" (gate, up, down
    in MDBF) or "mdbf_multi" (the MDBF gate and up in one mdbf_linear_multi call, then down)."""
    out = []
    if attention == "fused":
        out += [L_multi([(HIDDEN, 5001, "q"), (1024, 5002, "k"), (1024, 5003, "v")], HIDDEN, "benq_qkv"),
                L_benq(HIDDEN, HIDDEN, 1, 5004, "benq_o")]
    elif attention:
        out += [L_benq(HIDDEN, HIDDEN, 1, 5001, "benq_q"), L_benq(1024, HIDDEN, 1, 5002, "benq_k"),
                L_benq(1024, HIDDEN, 1, 5003, "benq_v"), L_benq(HIDDEN, HIDDEN, 1, 5004, "benq_o")]
    if mlp == "benq":
        out += [L_benq(INTER, HIDDEN, 1, SEED_GATE, "benq_gate"), L_benq(INTER, HIDDEN, 1, SEED_UP, "benq_up")]
    elif mlp == "benq_fused":
        out += [L_mlp(INTER, HIDDEN, SEED_GATE, SEED_UP, "benq_gate_up_silu")]
    if mlp in ("benq", "benq_fused"):
        out += [L_benq(HIDDEN, INTER, 1, SEED_DOWN, "benq_down")]
    if mlp == "mdbf":
        out += [L_mdbf(MLP_P, INTER, HIDDEN, MLP_R, MLP_L, 1, 5008, "mdbf_gate"),
                L_mdbf(MLP_P, INTER, HIDDEN, MLP_R, MLP_L, 1, 5009, "mdbf_up")]
    if mlp == "mdbf_multi":
        out += [L_mdbf(MLP_P, INTER, HIDDEN, MLP_R, MLP_L, 1, 5008, "mdbf_gate", group="gate_up"),
                L_mdbf(MLP_P, INTER, HIDDEN, MLP_R, MLP_L, 1, 5009, "mdbf_up", group="gate_up", group_skip=True)]
    if mlp in ("mdbf", "mdbf_multi"):
        out += [L_mdbf(MLP_P, HIDDEN, INTER, MLP_R, MLP_L, 1, 5010, "mdbf_down")]
    return out


DECODE = [L_benq(INTER, HIDDEN, 1, SEED_GATE, "benq_gate_up_5120x17408_b1"),
          L_benq(HIDDEN, INTER, 1, SEED_DOWN, "benq_down_17408x5120_b1")]

# workload -> [(record key, [(variant, layers, timing)])]; timing "rotate" (weights larger than
# L2, rotating copies) or "flush" (an L2 flush before each timed step)
RECORDS = {
    "small": [("cfg0_benq_256x512", [
        ("b1", [L_benq(256, 512, 1, 1, "benq_256x512_b1")], "flush"),
        ("b8", [L_benq(256, 512, 8, 2, "benq_256x512_b8")], "flush")])],
    "decode": [("cfg1_decode_27b", [("b1", DECODE, "rotate")])],
    "prefill": [("cfg2_prefill_m2048", [
        ("m2048", [L_benq(INTER, HIDDEN, 2048, SEED_GATE, "benq_gemm_5120x17408_m2048", "bf16"),
                   L_benq(HIDDEN, INTER, 2048, SEED_DOWN, "benq_gemm_17408x5120_m2048", "bf16")], "rotate")])],
    "mdbf_square": [("cfg3_mdbf_4096", [
        ("b1", [L_mdbf(SQ_P, SQ_N, SQ_N, SQ_R, SQ_L, 1, 3001, "mdbf_4096_r2000_b1")], "flush"),
        ("b16", [L_mdbf(SQ_P, SQ_N, SQ_N, SQ_R, SQ_L, 16, 3002, "mdbf_4096_r2000_b16")], "flush")])],
    "layer": [("cfg4_layer_27b", [
        ("benq_7_linears", layer_set(True, "benq"), "rotate"),
        ("benq_fused_mlp", layer_set(True, "benq_fused"), "rotate"),
        ("benq_4_launches", layer_set("fused", "benq_fused"), "rotate"),
        ("mdbf_mlp", layer_set(False, "mdbf"), "rotate"),
        ("mdbf_mlp_2_calls", layer_set(False, "mdbf_multi"), "rotate"),
        ("mixed_benq_attention_mdbf_mlp", layer_set(True, "mdbf"), "rotate"),
        ("mixed_5_calls", layer_set("fused", "mdbf_multi"), "rotate")])],
    "mdbf": [("cfg4_mdbf_mlp_27b", [("b1", layer_set(False, "mdbf"), "rotate")])],
    # the l = 1 cases (DBF at P = 1, LittleBit at P = 2) on the square layer, next to cfg3's l = 2
    "mdbf_l1": [("next4_mdbf_l1_4096", [
        ("dbf_b1", [L_mdbf(1, SQ_N, SQ_N, SQ_R, 1, 1, 3101, "mdbf_4096_r2000_l1_p1_b1")], "flush"),
        ("dbf_b16", [L_mdbf(1, SQ_N, SQ_N, SQ_R, 1, 16, 3102, "mdbf_4096_r2000_l1_p1_b16")], "flush"),
        ("littlebit_b1", [L_mdbf(2, SQ_N, SQ_N, SQ_R, 1, 1, 3103, "mdbf_4096_r2000_l1_p2_b1")], "flush"),
        ("littlebit_b16", [L_mdbf(2, SQ_N, SQ_N, SQ_R, 1, 16, 3104, "mdbf_4096_r2000_l1_p2_b16")], "flush")])],
    "mdbf_prefill": [("next1_mdbf_prefill_m2048", [
        ("m2048", [L_mdbf(MLP_P, INTER, HIDDEN, MLP_R, MLP_L, 2048, 6001, "mdbf_gemm_5120x17408_m2048", "bf16"),
                   L_mdbf(MLP_P, HIDDEN, INTER, MLP_R, MLP_L, 2048, 6002, "mdbf_gemm_17408x5120_m2048", "bf16")],
         "rotate")])],
}
ALL_ORDER = ["decode", "small", "prefill", "mdbf_square", "mdbf_l1", "layer", "mdbf_prefill"]
WORKLOADS = ["all"] + list(RECORDS)


def headline_workload(workload):
    return "decode" if workload == "all" else workload


def out_bytes(L):
    return 4 if L["out"] == "f32" else 2


def layer_bytes(L):
    if L["kind"] == "benq":
        return benq_bytes(L["N"], L["K"], L["B"], out_bytes(L))
    if L["kind"] == "benq_multi":   # x read once for all parts
        return benq_bytes(L["N"], L["K"], L["B"], out_bytes(L))
    if L["kind"] == "benq_mlp":
        return 2 * benq_weight_bytes(L["N"], L["K"]) + 2 * L["K"] + out_bytes(L) * L["N"]
    return mdbf_bytes(L["n"], L["m"], L["r"], L["l"], L["P"], L["B"], out_bytes(L))


def layer_weight_bytes(L):
    if L["kind"] in ("benq", "benq_multi"):
        return benq_weight_bytes(L["N"], L["K"])
    if L["kind"] == "benq_mlp":
        return 2 * benq_weight_bytes(L["N"], L["K"])
    return mdbf_weight_bytes(L["n"], L["m"], L["r"], L["l"], L["P"])


def layer_flops(L):
    if L["kind"] in ("benq", "benq_multi"):
        return 2.0 * L["B"] * L["N"] * L["K"]
    if L["kind"] == "benq_mlp":
        return 4.0 * L["N"] * L["K"]
    return mdbf_flops(L["n"], L["m"], L["r"], L["P"], L["B"])


def is_gemm(L):
    if L["kind"] in ("benq", "benq_multi"):
        return L["B"] > 16
    if L["kind"] == "mdbf":
        return L["l"] * L["B"] > DECODE_VLIM
    return False


def layer_launches(L):
    """Kernels of this library one call launches: BenQ one; MDBF decode pack z, G stage, F stage;
    MDBF batched envelope prep, activation prep and the two GEMMs."""
    if L["kind"] in ("benq", "benq_mlp", "benq_multi"):
        return 1
    if L.get("group_skip"):   # run by its group's first layer
        return 0
    return 4 if is_gemm(L) else 3


def layer_ideal_us(L, peaks):
    """The layer's roofline time: HBM time of its algorithmic bytes, tensor time of its FLOPs for the
    GEMMs, and for the MDBF decode the larger of its HBM and signed-add (ALU) times."""
    t_hbm = layer_bytes(L) / (peaks["hbm_gbs"] * 1e3)
    if is_gemm(L):
        return max(t_hbm, layer_flops(L) / (peaks["bf16_tflops"] * 1e6))
    if L["kind"] == "mdbf":
        return max(t_hbm, mdbf_adds(L["n"], L["m"], L["r"], L["l"], L["P"], L["B"]) / (alu_peak_tadds(peaks) * 1e6))
    return t_hbm


def copies_for(layers, timing):
    if timing == "flush":
        return 1
    per_step = sum(layer_weight_bytes(L) for L in layers)
    return max(1, int(np.ceil(2 * L2_BYTES / per_step)) + 1)


def l2_note(layers, timing):
    if timing == "flush":
        return f"L2 flushed: a {FLUSH_BYTES >> 20} MiB buffer is written before each timed step"
    c = copies_for(layers, timing)
    ws = c * sum(layer_weight_bytes(L) for L in layers)
    return f"inputs larger than L2: {c} rotating weight copies, {ws / 2**20:.0f} MiB working set vs 126 MiB L2"


def line_config(workload, world):
    """The line's `config` (the same for both arms: it depends on the workload only)."""
    wl = headline_workload(workload)
    key, variants = RECORDS[wl][0]
    name, layers, timing = variants[0]
    cfg = {"workload": workload, "headline": f"{key}/{name}", "layers": [L["label"] for L in layers],
           "l2": l2_note(layers, timing), "parallelism": f"replicas x{world}"}
    if workload == "all":
        cfg["records"] = [f"{k}/{v[0]}" for w in ALL_ORDER for k, vs in RECORDS[w] for v in vs]
    return cfg


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


# ---------------------------------------------------------------------------------------------- device inputs

# per-step copy bytes (in + out) from which the end-to-end steps overlap their copies with compute
E2E_OVERLAP_BYTES = 1 << 20


def packed_offsets(sizes, align=256):
    """Byte offsets of consecutive segments of the given sizes, each start aligned, and the total."""
    offs, o = [], 0
    for nb in sizes:
        offs.append(o)
        o += (nb + align - 1) // align * align
    return offs, max(o, align)


class Inputs:
    """Device-resident weights, activations and outputs of a list of layers, with rotating copies of
    the weights.  BenQ weights of one (N, K, seed) are made once and shared between records."""

    _benq_cache = {}

    def __init__(self, layers, copies, ql, torch):
        import synth
        from tests.qlhelpers import bf16, dev, f16
        self.layers, self.copies = [], copies
        cuda = torch.device("cuda")
        layers = [dict(L) for L in layers]
        for L in layers:
            L["x_h"] = synth.activations(L["B"], L["K"] if "K" in L else L["m"], seed=L["seed"] + 500)
        # The step's activations sit in one device buffer and its outputs in another (a 256-byte aligned
        # view per layer), so that the end-to-end step copies its inputs in and its results out with
        # one copy each.  Layers after the first of a group read the first one's x.
        own_x = [L for L in layers if not L.get("group_skip")]
        xoff, xbytes = packed_offsets([L["x_h"].size * 2 for L in own_x])
        self.xbuf = torch.empty(xbytes, dtype=torch.uint8, device=cuda)
        xh = np.zeros(xbytes, dtype=np.uint8)
        for L, o in zip(own_x, xoff):
            nb = L["x_h"].size * 2
            xh[o:o + nb] = np.ascontiguousarray(L["x_h"]).view(np.uint8).reshape(-1)
            L["x"] = self.xbuf[o:o + nb].view(torch.bfloat16).view(L["x_h"].shape)
            L["_xo"] = (o, nb)
        self.xbuf.copy_(torch.from_numpy(xh))
        self.x_host = xh
        odts = [torch.float32 if L["out"] == "f32" else torch.bfloat16 for L in layers]
        nouts = [L["N"] if "N" in L else L["n"] for L in layers]
        yoff, ybytes = packed_offsets([L["B"] * n * (4 if d == torch.float32 else 2) for L, n, d in zip(layers, nouts, odts)])
        self.ybuf = torch.empty(ybytes, dtype=torch.uint8, device=cuda)
        for L, o, n, d in zip(layers, yoff, nouts, odts):
            nb = L["B"] * n * (4 if d == torch.float32 else 2)
            L["y"] = self.ybuf[o:o + nb].view(d).view(L["B"], n)
            L["_yo"] = (o, nb)
        for L in layers:
            L["ws"] = None
            if L["kind"] == "benq":
                w0 = self.benq_device_weights(L["N"], L["K"], L["seed"], ql, torch)
                nws = ql.benq_linear_workspace_bytes(L["B"], L["N"], L["K"])
                L["ws"] = torch.empty(nws, dtype=torch.uint8, device=cuda) if nws else None
            elif L["kind"] == "benq_mlp":
                w0 = (self.benq_device_weights(L["N"], L["K"], L["seed"], ql, torch)
                      + self.benq_device_weights(L["N"], L["K"], L["seed_u"], ql, torch))
            elif L["kind"] == "benq_multi":
                # one output buffer, a contiguous view per part (batch 1, parts of 4k rows: 16-byte aligned)
                w0 = tuple(self.benq_device_weights(N, L["K"], sd, ql, torch) for N, sd, _ in L["parts"])
                offs = np.cumsum([0] + [N for N, _, _ in L["parts"]])
                L["_ys_offs"] = offs
                L["ys"] = [L["y"][:, offs[i]:offs[i + 1]] for i in range(len(L["parts"]))]
            else:
                paths = synth.mdbf_paths(L["P"], L["n"], L["m"], L["r"], L["l"], seed=L["seed"])
                w0 = [dict(S_A=dev(p.S_A), S_B=dev(p.S_B), A_amp=f16(p.A_amp), B_amp=f16(p.B_amp),
                           Q_U=f16(p.Q_U), Q_V=f16(p.Q_V)) for p in paths]
                L["ws"] = torch.empty(ql.mdbf_workspace_bytes(L["P"], L["n"], L["m"], L["r"], L["l"], L["B"]),
                                      dtype=torch.uint8, device=cuda)
            L["w"] = [w0] + [self.clone(w0) for _ in range(copies - 1)]
            if L["kind"] not in ("benq", "benq_mlp", "benq_multi"):
                L["wc"] = [ql.mdbf_paths_c(w) for w in L["w"]]   # path arrays made once, not per call
            self.layers.append(L)
        # layers of one group read the first one's x; its workspace serves all of their paths
        for L in self.layers:
            if L.get("group") and not L.get("group_skip"):
                members = [M for M in self.layers if M.get("group") == L["group"]]
                for M in members[1:]:
                    M["x"] = L["x"]
                L["group_members"] = members
                L["ws"] = torch.empty(ql.mdbf_workspace_bytes(len(members) * L["P"], L["n"], L["m"], L["r"], L["l"],
                                                              L["B"]), dtype=torch.uint8, device=cuda)

    def views(self, torch, xbuf, ybuf):
        """Every layer's x, y (and ys) as views of the given activation and output buffers, at this
        record's offsets; group members read their first member's x."""
        vs = []
        for L in self.layers:
            o, nb = L["_yo"]
            v = {"y": ybuf[o:o + nb].view(L["y"].dtype).view(L["y"].shape)}
            if "_xo" in L:
                o, nb = L["_xo"]
                v["x"] = xbuf[o:o + nb].view(torch.bfloat16).view(L["x"].shape)
            if "_ys_offs" in L:
                offs = L["_ys_offs"]
                v["ys"] = [v["y"][:, offs[i]:offs[i + 1]] for i in range(len(offs) - 1)]
            vs.append(v)
        index = {id(L): i for i, L in enumerate(self.layers)}
        for L, v in zip(self.layers, vs):
            for M in L.get("group_members", [])[1:]:
                vs[index[id(M)]]["x"] = v["x"]
        return vs

    def use(self, vs):
        for L, v in zip(self.layers, vs):
            L.update(v)

    @classmethod
    def benq_device_weights(cls, N, K, seed, ql, torch):
        key = (N, K, seed)
        if key not in cls._benq_cache:
            g = torch.Generator(device="cuda")
            g.manual_seed(seed)
            sigma = torch.rand(N, 1, generator=g, device="cuda") * 0.02 + 0.01
            w = (torch.randn(N, K, generator=g, device="cuda") * sigma).to(torch.bfloat16)
            codes = torch.empty(N, 3 * K // 4, dtype=torch.uint8, device="cuda")
            lut = torch.empty(N, 64, dtype=torch.int16, device="cuda")
            ql.benq_encode(w, codes, lut, lloyd_iters=0)
            del w, sigma
            cls._benq_cache[key] = (codes, lut)
        return cls._benq_cache[key]

    @staticmethod
    def clone(w):
        if isinstance(w, tuple):
            return tuple(tuple(u.clone() for u in t) if isinstance(t, tuple) else t.clone() for t in w)
        return [{k: v.clone() for k, v in d.items()} for d in w]

    def run(self, ql, L, c):
        w = L["w"][c]
        if L["kind"] == "benq":
            ql.benq_linear(w[0], w[1], L["x"], L["y"], workspace=L["ws"])
        elif L["kind"] == "benq_mlp":
            ql.benq_mlp_gate_up(*w, L["x"], L["y"])
        elif L["kind"] == "benq_multi":
            ql.benq_linear_multi([(c, t, y) for (c, t), y in zip(w, L["ys"])], L["x"])
        elif L.get("group_skip"):
            return
        elif "group_members" in L:
            ms = L["group_members"]
            ql.mdbf_linear_multi([M["wc"][c] for M in ms], L["n"], L["m"], L["r"], L["l"], L["x"],
                                 [M["y"] for M in ms], L["ws"])
        else:
            ql.mdbf_linear(L["wc"][c], L["n"], L["m"], L["r"], L["l"], L["x"], L["y"], L["ws"])


# ---------------------------------------------------------------------------------------------- timing

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


class Timer:
    """Runs a record's steps (graph replays or eager calls) and times them on the launching stream."""

    def __init__(self, ql, torch, world, warmup):
        self.ql, self.torch, self.world, self.warmup = ql, torch, world, warmup
        self.stream = torch.cuda.current_stream()
        self._flush = None

    def sync_all(self):
        import torch.distributed as dist
        if self.world > 1:
            dist.barrier()
        self.torch.cuda.synchronize()

    def capture(self, inp, layers, copies):
        g = self.torch.cuda.CUDAGraph()
        with self.torch.cuda.graph(g, capture_error_mode="thread_local"):
            for c in copies:
                for L in layers:
                    inp.run(self.ql, L, c)
        return g

    def graphs(self, inp, layers, steps):
        """Graphs of one rotation of the weight copies, of each single copy, and of the `steps` timed
        steps in one piece (copies in turn), so that the timed region holds no graph boundary."""
        n = inp.copies
        return {"cycle": self.capture(inp, layers, range(n)), "one": [self.capture(inp, layers, [c]) for c in range(n)],
                "all": self.capture(inp, layers, [i % n for i in range(steps)]) if steps else None}

    def replay(self, gs, steps, n):
        for _ in range(steps // n):
            gs["cycle"].replay()
        for c in range(steps % n):
            gs["one"][c].replay()

    def flush(self):
        if self._flush is None:
            self._flush = self.torch.empty(FLUSH_BYTES, dtype=self.torch.uint8, device="cuda")
        self._flush.fill_(1)

    def time_graph(self, inp, gs, steps, timing):
        """Milliseconds for `steps` graph-replayed steps (max over ranks)."""
        torch, n = self.torch, inp.copies
        self.replay(gs, max(self.warmup, n), n)
        if timing == "rotate":
            gs["all"].replay()   # the first replay of a graph also uploads it
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            self.sync_all()
            a.record(self.stream)
            gs["all"].replay()
            b.record(self.stream)
            self.sync_all()
            return max_over_ranks(a.elapsed_time(b), self.world)
        gs["one"][0].replay()
        ev = []
        self.sync_all()
        for _ in range(steps):
            self.flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(self.stream)
            gs["one"][0].replay()
            b.record(self.stream)
            ev.append((a, b))
        self.sync_all()
        return max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), self.world)

    def time_eager(self, inp, layers, steps, timing):
        """Milliseconds for `steps` steps of separate launches (no graph)."""
        torch, n = self.torch, inp.copies
        for i in range(self.warmup):
            for L in layers:
                inp.run(self.ql, L, i % n)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        self.sync_all()
        if timing == "flush":
            tot = 0.0
            for i in range(steps):
                self.flush()
                a.record(self.stream)
                for L in layers:
                    inp.run(self.ql, L, 0)
                b.record(self.stream)
                b.synchronize()
                tot += a.elapsed_time(b)
            self.sync_all()
            return max_over_ranks(tot, self.world)
        a.record(self.stream)
        for i in range(steps):
            for L in layers:
                inp.run(self.ql, L, i % n)
        b.record(self.stream)
        self.sync_all()
        return max_over_ranks(a.elapsed_time(b), self.world)

    def time_e2e(self, inp, layers, steps):
        """The same steps through the public API with every step's inputs copied in from pinned host
        memory and its results copied back (eager calls; one copy each way, the layers' activations
        and outputs being views of one buffer each); returns (ms, h2d bytes, d2h bytes) per run.

        Steps whose copies reach E2E_OVERLAP_BYTES alternate between two sets of device buffers, so
        that step i's copy in (on a copy stream) overlaps step i-1's kernels and its copy out (on
        another) overlaps step i+1's: a buffer is refilled only after the kernels two steps back
        have read it, and an output buffer is rewritten only after its previous copy out.  Smaller
        steps run on one stream, where the events and stream switches would cost more host time
        than the overlap saves.  The last step's copied-back outputs are checked against a plain
        call of the same step."""
        torch, n = self.torch, inp.copies
        if inp.xbuf.numel() + inp.ybuf.numel() < E2E_OVERLAP_BYTES:
            x_h = torch.from_numpy(inp.x_host).pin_memory()
            y_h = torch.empty(inp.ybuf.numel(), dtype=torch.uint8).pin_memory()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            self.sync_all()
            a.record(self.stream)
            for i in range(steps):
                inp.xbuf.copy_(x_h, non_blocking=True)
                for L in layers:
                    inp.run(self.ql, L, i % n)
                y_h.copy_(inp.ybuf, non_blocking=True)
            b.record(self.stream)
            self.sync_all()
            self.check_e2e(inp, layers, y_h.clone())
            return max_over_ranks(a.elapsed_time(b), self.world), x_h.numel(), y_h.numel()
        xb = [inp.xbuf, torch.empty_like(inp.xbuf)]
        yb = [inp.ybuf, torch.empty_like(inp.ybuf)]
        sets = [inp.views(torch, xb[k], yb[k]) for k in range(2)]
        x_h = torch.from_numpy(inp.x_host).pin_memory()
        y_h = [torch.empty(inp.ybuf.numel(), dtype=torch.uint8).pin_memory() for _ in range(2)]
        main, cin, cout = self.stream, torch.cuda.Stream(), torch.cuda.Stream()
        read = [None, None]       # the kernels that last read activation buffer k
        back = [None, None]       # the last copy out of output buffer k
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        self.sync_all()
        a.record(main)
        cin.wait_event(a)
        for i in range(steps):
            k = i % 2
            if read[k] is not None:
                cin.wait_event(read[k])
            with torch.cuda.stream(cin):
                xb[k].copy_(x_h, non_blocking=True)
            e_in = torch.cuda.Event()
            e_in.record(cin)
            main.wait_event(e_in)
            if back[k] is not None:
                main.wait_event(back[k])
            inp.use(sets[k])
            for L in layers:
                inp.run(self.ql, L, i % n)
            read[k] = torch.cuda.Event()
            read[k].record(main)
            cout.wait_event(read[k])
            with torch.cuda.stream(cout):
                y_h[k].copy_(yb[k], non_blocking=True)
            back[k] = torch.cuda.Event()
            back[k].record(cout)
        for e in back:
            if e is not None:
                main.wait_event(e)
        b.record(main)
        self.sync_all()
        last = y_h[(steps - 1) % 2].clone()
        inp.use(sets[0])
        self.check_e2e(inp, layers, last)
        return max_over_ranks(a.elapsed_time(b), self.world), x_h.numel(), y_h[0].numel()

    def check_e2e(self, inp, layers, copied):
        """The outputs an end-to-end step copied back equal those of a plain call of the step."""
        for L in layers:
            inp.run(self.ql, L, 0)
        self.torch.cuda.synchronize()
        if not self.torch.equal(copied, inp.ybuf.cpu()):
            raise RuntimeError("end-to-end step: the copied-back outputs differ from a plain call's")


# ---------------------------------------------------------------------------------------------- records

# the sources each kernel's DRAM-traffic figure depends on
_KERNEL_SOURCES = {
    "benq_gemv": ["benq_gemv.cu", "ql_device.cuh"],
    "benq_gemm": ["benq_gemm_sm100.cu", "pair_gemm.cuh", "sm100_ptx.cuh", "ql_device.cuh"],
    "mdbf_linear": ["mdbf.cu", "ql_device.cuh"],
    "mdbf_gemm": ["mdbf_gemm_sm100.cu", "pair_gemm.cuh", "sm100_ptx.cuh", "ql_device.cuh"],
}


_COMMENT = re.compile(r"/\*.*?\*/|//[^\n]*", re.S)


def _kernel_source_sha(kernel_key):
    """Hash of the code (comments and trailing blanks removed) of the sources a kernel's traffic
    figure depends on: a comment edit leaves the figure valid, any code change voids it."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "quantized_linear_b200", "csrc")
    for f in _KERNEL_SOURCES[kernel_key]:
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            code = _COMMENT.sub("", fh.read())
        code = "\n".join(line.rstrip() for line in code.splitlines() if line.strip())
        h.update(f.encode() + code.encode())
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


def kernel_name(L):
    if L["kind"] in ("benq", "benq_mlp", "benq_multi"):
        return "benq_gemm" if is_gemm(L) else "benq_gemv"
    return "mdbf_gemm" if is_gemm(L) else "mdbf_linear"


def roofline(layers, us, peaks):
    """Roofline of one step of `layers` taking `us` microseconds.

    Homogeneous steps report their own bound: GB/s against the measured copy bandwidth (BenQ
    GEMV), TFLOP/s against the measured bf16 peak (the GEMMs), and for the MDBF decode kernels the
    larger of the HBM and ALU (signed-add) times, with both fractions.  A step that mixes bounds
    reports the sum of its layers' roofline times against the measured time."""
    ideal = sum(layer_ideal_us(L, peaks) for L in layers)
    byts = sum(layer_bytes(L) for L in layers)
    kinds = {kernel_name(L) for L in layers}
    kname = kinds.pop() if len(kinds) == 1 else "mixed"
    hbm = {"bound": "hbm", "achieved": byts / us / 1e3, "peak": peaks["hbm_gbs"], "unit": "GB/s",
           "peak_source": peaks["source"] + " (STREAM copy)"}
    if kname in ("benq_gemm", "mdbf_gemm"):
        fl = sum(layer_flops(L) for L in layers)
        r = {"bound": "tensor", "achieved": fl / us / 1e6, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
             "peak_source": peaks["source"] + " (burst)"}
    elif kname == "mdbf_linear":
        adds = sum(mdbf_adds(L["n"], L["m"], L["r"], L["l"], L["P"], L["B"]) for L in layers)
        t_hbm = byts / (peaks["hbm_gbs"] * 1e3)
        t_alu = adds / (alu_peak_tadds(peaks) * 1e6)
        r = dict(hbm) if t_hbm >= t_alu else {
            "bound": "alu", "achieved": adds / us / 1e6, "peak": alu_peak_tadds(peaks), "unit": "T add/s",
            "peak_source": "derived: 148 SMs x 128 fp32 lanes x max SM clock, one add per lane per clock"}
        r.update(hbm_us=t_hbm, alu_us=t_alu, hbm_frac=t_hbm / us, alu_frac=t_alu / us,
                 hbm_achieved_gbs=byts / us / 1e3)
    elif kname == "mixed":
        r = {"bound": "mixed", "achieved": byts / us / 1e3, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "peak_source": peaks["source"] + " (STREAM copy); frac = sum of the layers' roofline times / time"}
    else:
        r = hbm
    r.update(frac=(ideal / us) if kname in ("mixed", "mdbf_linear") else r["achieved"] / r["peak"],
             ideal_us=ideal, kernel=kname, traffic=None if kname == "mixed" else _traffic(kname))
    return r


def cublas_reference(torch, layers, steps, warmup=3):
    """Dense bf16 GEMMs of the same shapes through torch.matmul (cuBLAS) on random dense weights,
    timed the same way (device events, weights larger than L2): a reference point for the
    tensor-core rate at these shapes, not part of the measured path."""
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
    return {"us_per_step": 1e3 * ms, "tflops": flops / (ms / 1e3) / 1e12,
            "what": "torch.matmul bf16 (cuBLAS), same shapes, dense random weights"}


def measure_variant(timer, layers, timing, steps, peaks, eager=False):
    inp = Inputs(layers, copies_for(layers, timing), timer.ql, timer.torch)
    for L in inp.layers:   # first calls outside any capture (kernel attributes, tensor maps)
        inp.run(timer.ql, L, 0)
    timer.torch.cuda.synchronize()
    gs = timer.graphs(inp, inp.layers, steps if timing == "rotate" else 0)
    ms = timer.time_graph(inp, gs, steps, timing)
    us = 1e3 * ms / steps
    byts = sum(layer_bytes(L) for L in layers)
    rec = {"us": us, "layers": [L["label"] for L in layers], "algorithmic_bytes": byts,
           "gbs": byts / us / 1e3, "launches_per_step": sum(layer_launches(L) for L in layers),
           "roofline": roofline(layers, us, peaks), "l2": l2_note(layers, timing),
           "launch": "CUDA graph, kernels chained by programmatic dependent launch"}
    fl = sum(layer_flops(L) for L in layers)
    if any(is_gemm(L) for L in layers):
        rec["tflops"] = fl / us / 1e6
    if eager:
        ems = timer.time_eager(inp, inp.layers, steps, timing)
        rec["us_separate_launches"] = 1e3 * ems / steps
    if all(L["kind"] == "benq" and is_gemm(L) for L in layers) and timer.world == 1:
        rec["cublas_bf16_same_shape"] = cublas_reference(timer.torch, layers, min(steps, 20))
    ems, h2d, d2h = timer.time_e2e(inp, inp.layers, steps)
    rec["e2e"] = {"value": byts * steps / (ems / 1e3) / 1e9, "unit": "GB/s", "us": 1e3 * ems / steps,
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    del gs
    return rec, inp


# ---------------------------------------------------------------------------------------------- CPU oracle

def oracle_sample(layers, rows=64, seed=0):
    """A bounded sample of a step for the oracle: per layer, `rows` output rows (all of them when the
    layer has fewer) with their inputs, and at most 16 token rows of a batch; generated once,
    outside any timing.  Returns [(label, run, algorithmic bytes, flops)]."""
    import synth
    from oracle import benq as ob
    from oracle import mdbf as om
    rng = np.random.default_rng(seed)
    out = []
    for L in layers:
        bb = min(L["B"], 16)
        if L["kind"] in ("benq", "benq_mlp", "benq_multi"):
            N, K = L["N"], L["K"]
            rr = min(rows, N)
            w = synth.benq_weights(rr, K, seed=int(rng.integers(1 << 30)))
            x = synth.activations(bb, K, seed=1)
            if L["kind"] != "benq_mlp":
                run = (lambda w=w, x=x, K=K: ob.linear(w.codes, w.lut, x, K))
                out.append((f"benq {rr} of {N} rows x K={K}, B={bb}", run, benq_bytes(rr, K, bb), 2.0 * bb * rr * K))
            else:
                wu = synth.benq_weights(rr, K, seed=int(rng.integers(1 << 30)))
                run = (lambda w=w, wu=wu, x=x, K=K: ob.mlp_gate_up(w.codes, w.lut, wu.codes, wu.lut, x, K))
                out.append((f"benq gate/up {rr} of {N} rows x K={K}", run,
                            2 * benq_weight_bytes(rr, K) + 2 * K + 4 * rr, 4.0 * rr * K))
        else:
            n, m, r, l, P = L["n"], L["m"], L["r"], L["l"], L["P"]
            rr = min(rows, n)
            paths = synth.mdbf_paths(P, n, m, r, l, seed=7)
            x = synth.activations(bb, m, seed=1)
            sel = np.sort(rng.choice(n, rr, replace=False))
            run = (lambda paths=paths, x=x, n=n, m=m, r=r, sel=sel: om.linear_factored(paths, n, m, r, x, rows=sel))
            out.append((f"mdbf {rr} of {n} rows, m={m}, r={r}, l={l}, P={P}, B={bb}", run,
                        mdbf_bytes(rr, m, r, l, P, bb), mdbf_flops(rr, m, r, P, bb)))
    return out


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def time_sample(sample, budget_s, threads):
    """Runs the sample (every entry once per pass) until `budget_s` seconds of oracle time have been
    spent, with BLAS limited to `threads` threads (None: the library's default, all cores).  Returns
    (bytes, flops, seconds, passes, threads used)."""
    from threadpoolctl import threadpool_limits
    done_b, done_f, t_used, passes = 0.0, 0.0, 0.0, 0
    with threadpool_limits(limits=threads):
        used = _blas_threads()
        while t_used < budget_s or passes == 0:
            for _, run, nb, nf in sample:
                t0 = time.perf_counter()
                run()
                t_used += time.perf_counter() - t0
                done_b += nb
                done_f += nf
            passes += 1
    return done_b, done_f, t_used, passes, used


def cpu_baseline(layers, budget_s, unit):
    """The oracle as it stands on a bounded sample of the step: one thread, and all cores."""
    sample = oracle_sample(layers)
    res = {"kind": "oracle", "unit": unit, "os_cpu_count": os.cpu_count(),
           "affinity_cores": len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else None}
    for tag, threads in (("", 1), ("all_cores_", None)):
        b, f, t, passes, used = time_sample(sample, budget_s, threads)
        v = b / t / 1e9 if unit == "GB/s" else f / t / 1e12
        res[tag + "value"] = v
        res[tag + "cores"] = used
        res[tag + "sample"] = (f"{passes} passes over {len(sample)} layers ({sample[0][0]}; ...), "
                               f"{t:.1f} s of oracle time")
    return res


# ---------------------------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    """The oracle as the reference arm: each step is one pass of the oracle over the headline's sample
    (generated once), so the run's length is bounded by the sample, not by the weights' size; the
    other records of the workload get a bounded single-threaded timing each."""
    if rank != 0:
        return
    from threadpoolctl import threadpool_limits
    wl = headline_workload(args.workload)
    key, variants = RECORDS[wl][0]
    sample = oracle_sample(variants[0][1])
    unit = "TFLOP/s" if any(is_gemm(L) for L in variants[0][1]) else "GB/s"
    for _ in range(args.warmup):
        time_sample(sample, 0.0, 1)
    done_b, done_f, t_used = 0.0, 0.0, 0.0
    t0 = time.perf_counter()   # the timed steps only
    with threadpool_limits(limits=1):
        for _ in range(args.steps):
            b, f, t, _, _ = time_sample(sample, 0.0, 1)
            done_b += b
            done_f += f
            t_used += t
    t_steps = time.perf_counter() - t0
    v = done_b / t_used / 1e9 if unit == "GB/s" else done_f / t_used / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * t_steps / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": line_config(args.workload, world),
            "cpu_baseline": {"value": v, "unit": unit, "cores": 1, "kind": "oracle",
                             "os_cpu_count": os.cpu_count(),
                             "sample": f"one pass per step over {len(sample)} layers: "
                                       + "; ".join(s[0] for s in sample)},
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if args.workload == "all":
        recs = {}
        for w in ALL_ORDER:
            for k, vs in RECORDS[w]:
                for name, layers, _ in vs:
                    u = "TFLOP/s" if any(is_gemm(L) for L in layers) else "GB/s"
                    s = oracle_sample(layers)
                    b, f, t, passes, _ = time_sample(s, getattr(args, "ref_budget", 1.0), 1)
                    recs[f"{k}/{name}"] = {"value": b / t / 1e9 if u == "GB/s" else f / t / 1e12, "unit": u,
                                           "cores": 1, "sample": f"{passes} passes over {len(s)} layers"}
        line["workloads"] = recs
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="all", choices=WORKLOADS)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=1.5, help="seconds of oracle time per record and thread setting")
    ap.add_argument("--cpu-budget-headline", type=float, default=10.0,
                    help="seconds of oracle time per thread setting for the headline record")
    ap.add_argument("--ref-budget", type=float, default=1.0, help=argparse.SUPPRESS)
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

    peaks = _peaks()
    timer = Timer(ql, torch, world, args.warmup)
    order = ALL_ORDER if args.workload == "all" else [args.workload]
    records, head = {}, None
    with ClockSampler(torch.cuda.current_device()) as clk:
        for w in order:
            for key, variants in RECORDS[w]:
                rec = {}
                for name, layers, timing in variants:
                    r, inp = measure_variant(timer, layers, timing, args.steps, peaks, eager=(w == "layer"))
                    rec[name] = r
                    if head is None:
                        head = (key, name, layers, r)
                    del inp
                records[key] = rec
                torch.cuda.empty_cache()

    key, name, layers, hr = head
    ms = hr["us"] * args.steps / 1e3
    step_bytes = hr["algorithmic_bytes"]
    value = job_throughput(step_bytes, args.steps, ms, world)
    roof = dict(hr["roofline"])
    roof["avg_launch_us"] = hr["us"] / len(layers)
    headline_gemm = any(is_gemm(L) for L in layers)

    # CPU baselines (rank 0, one GPU only): the oracle on bounded samples, after all GPU timing
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        for w in order:
            for k, variants in RECORDS[w]:
                for vname, vlayers, _ in variants:
                    unit = "TFLOP/s" if any(is_gemm(L) for L in vlayers) else "GB/s"
                    budget = args.cpu_budget_headline if (k, vname) == (key, name) else args.cpu_budget
                    records[k][vname]["cpu_baseline"] = cpu_baseline(vlayers, budget, unit)

    e2e = hr["e2e"]
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": "u1+f16->f32" if layers[0]["kind"] == "mdbf" else "bf16xu6->f32",
            "data": "synthetic (seeded; BenQ codes made on the device by benq_encode, see the docstring)",
            "config": line_config(args.workload, world),
            "roofline": roof,
            "e2e": {"value": job_throughput(step_bytes, args.steps, e2e["us"] * args.steps / 1e3, world),
                    "unit": "GB/s", "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                    "d2h_bytes_per_step": e2e["d2h_bytes_per_step"], "ms_per_step": e2e["us"] / 1e3},
            "gpu_launches": hr["launches_per_step"] * args.steps,
            "clocks": clk.summary()}
    if headline_gemm:
        line["unit_note"] = "value is GB/s of algorithmic bytes; roofline is TFLOP/s"
    if "cpu_baseline" in hr:
        cb = hr["cpu_baseline"]
        line["cpu_baseline"] = {"value": cb["value"], "unit": cb["unit"], "cores": cb["cores"], "kind": "oracle",
                                "sample": cb["sample"], "all_cores_value": cb["all_cores_value"],
                                "all_cores": cb["all_cores_cores"], "os_cpu_count": cb["os_cpu_count"],
                                "affinity_cores": cb["affinity_cores"]}
    if args.workload in ("all", "layer"):
        lay = records.get("cfg4_layer_27b")
        if lay:
            line["decode_us_per_layer"] = {k: v["us"] for k, v in lay.items()}
    line["workloads"] = records
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
