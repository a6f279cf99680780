#!/usr/bin/env python
"""Benchmark of the Sparse-BitNet BitLinear forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|decode_entropy|prefill|qwen05b|layer_small]
                    [--only]

One step is one pass of the whole path over one batch of synthetic input.
The headline workload (default: decode) is the decode GEMV sweep:
sbn_quantize_weights on the latent weights W [6912, 2560] bf16 ~ N(0, 0.02)
(the dynamic 6:8 mask is recomputed every forward), then sbn_bitlinear_x
(activation quantization fused into the contraction) for T = 1, 4 and 16
tokens. With N = 1 and without --only, the same JSON line also carries, under
"workloads", every other configuration of the method's workloads, each with
its own roofline, CPU baseline and end-to-end figure:

* prefill      T = 4096 through (K, N_out) = (2560, 6912) and (6912, 2560) at
               2:4: quantize_weights, then quantize_acts + bitlinear per layer;
* qwen05b      the 24-layer Qwen2.5-0.5B-shaped stack (168 projections, hidden
               896, intermediate 4864), T = 2048, 6:8, weights packed once,
               quantize_acts + bitlinear per projection; tokens/s;
* ffn3b        the 3B-scale FFN sweep: gate (K 2048, N_out 11008) and down
               (K 11008, N_out 2048), T in {1, 64, 512, 8192} x n:m in
               {2:4, 4:8, 6:8, 8:16, 8:8}; each entry's contraction and
               activation quantization timed, and sbn_quantize_weights (the
               per-step dynamic mask) timed separately per pattern;
* layer_small  T = 16, K = N_out = 256, 2:4: latency of the three calls.

Timing. Every step is a captured CUDA graph. Steps rotate over R copies of
their inputs, with R such that the inputs of R steps exceed 3x the L2 cache
(queried from the device), so no step finds another step's inputs in L2.
The timed region is P passes of K graph replays, each pass bracketed by a
barrier and a synchronize and timed with CUDA events on the graph's stream;
the reported step time is the median pass (the max over ranks of each pass
for N > 1). Per-call durations come from per-kind graphs that launch every
call of one kind back to back over all R slots (events around the whole
replay, not around each call: an event pair around a single launch costs
several microseconds of its own); the kind with the largest time per step is
the dominant kernel, whose algorithmic bytes or operations over its measured
duration give the roofline line. The clocks are sampled during the timed
region. `e2e` times the same step through the public binding from pinned
host buffers (inputs copied in, outputs copied out, every step).

The reference arm (--impl reference) is the CPU oracle, timed on the host
cores with BLAS limited to one thread, on a bounded sample of the same
workload. For N > 1 every rank runs its own independent layer (weak
scaling, no collective on the data path); rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "BitLinear TOPS (prefill) and weight GB/s (decode) vs B200 roofline; tokens/s"
L2_FALLBACK_BYTES = 126 * 1024 * 1024
DATA_DESC = "synthetic (seeded: W ~ N(0,0.02) bf16, X ~ N(0,1) bf16)"
DTYPE = "int8xternary->int32, bf16 io"


# ---------------------------------------------------------------------------
# workloads: shapes and algorithmic bytes / ops
# ---------------------------------------------------------------------------

def codes_row_bytes(k, n, m):
    kept = k * n // m
    return ((kept + 3) // 4 + 15) // 16 * 16


def meta_row_bytes(k, n, m):
    return 0 if n == m else (k // 8 + 15) // 16 * 16


def packed_bytes(n_out, k, n, m):
    return n_out * (codes_row_bytes(k, n, m) + meta_row_bytes(k, n, m))


def qw_bytes(n_out, k, n, m):
    """sbn_quantize_weights: bf16 W read once + packed codes/meta + gamma."""
    return 2 * n_out * k + packed_bytes(n_out, k, n, m) + 4


def qa_bytes(t, k):
    """sbn_quantize_acts: bf16 X read + int8 Xq + fp32 scales."""
    return 3 * t * k + 4 * t


def bl_bytes(t, k, n_out, n, m):
    """sbn_bitlinear: packed W + Xq + scales + gamma + bf16 Y."""
    return packed_bytes(n_out, k, n, m) + t * k + 4 * t + 4 + 2 * t * n_out


def blx_bytes(t, k, n_out, n, m):
    """sbn_bitlinear_x (act-quant fused into the contraction): bf16 X + packed W
    + gamma + bf16 Y (the INT8 activations stay on chip)."""
    return 2 * t * k + packed_bytes(n_out, k, n, m) + 4 + 2 * t * n_out


def entropy_bytes(n_out, k, n, m):
    """Entropy-tight packed weights (one word of ceil(log2(C(m,n) 3^n)) bits per group)."""
    bits = (math.comb(m, n) * 3 ** n - 1).bit_length()
    return n_out * ((((k // m) * bits + 7) // 8 + 15) // 16 * 16)


def pe_bytes(n_out, k, n, m):
    """sbn_pack_entropy: canonical packed weights read, entropy-tight written."""
    return packed_bytes(n_out, k, n, m) + entropy_bytes(n_out, k, n, m)


def ble_bytes(t, k, n_out, n, m):
    """sbn_bitlinear_entropy: entropy-tight W + Xq + scales + gamma + bf16 Y."""
    return entropy_bytes(n_out, k, n, m) + t * k + 4 * t + 4 + 2 * t * n_out


def blex_bytes(t, k, n_out, n, m):
    """sbn_bitlinear_entropy_x (act-quant fused): bf16 X + entropy-tight W +
    gamma + bf16 Y."""
    return 2 * t * k + entropy_bytes(n_out, k, n, m) + 4 + 2 * t * n_out


def bl_ops(t, k, n_out, n, m):
    """Algorithmic ops (2 per kept multiply-add)."""
    return 2 * t * k * n_out * n // m


def _qwen_layers():
    from sparse_linear_layers_fwd_b200 import synth
    return [(n_out, k, 6, 8, [2048]) for _layer in range(24) for (_p, k, n_out) in synth.QWEN05B_PROJ]


WORKLOADS = {
    # name: list of layers (n_out, k, n, m, [token counts]) in one step; mode:
    # "fused" (sbn_bitlinear_x), "split" (quantize_acts + bitlinear),
    # "entropy" (pack_entropy + bitlinear_entropy_x); qw: the step quantizes
    # the latent weights (else they are packed once, outside the step)
    "decode": dict(desc="decode GEMV sweep: K=2560, N_out=6912, 6:8, T in {1,4,16}; value = "
                        "algorithmic bytes of the step / step time; activation quantization "
                        "fused into the contraction (sbn_bitlinear_x)",
                   unit="GB/s", mode="fused", qw=True, layers=[(6912, 2560, 6, 8, [1, 4, 16])]),
    "decode_entropy": dict(desc="decode GEMV sweep over entropy-tight weights: K=2560, N_out=6912, "
                                "6:8, T in {1,4,16}; each step packs the quantized layer into the "
                                "entropy-tight format (1.875 bit/weight) and contracts from it",
                           unit="GB/s", mode="entropy", qw=True, layers=[(6912, 2560, 6, 8, [1, 4, 16])]),
    "prefill": dict(desc="prefill GEMM: T=4096, (K,N_out)=(2560,6912) and (6912,2560), 2:4; value = "
                         "algorithmic ops (2 per kept multiply-add) of the step / step time",
                    unit="TOPS", mode="split", qw=True,
                    layers=[(6912, 2560, 2, 4, [4096]), (2560, 6912, 2, 4, [4096])]),
    "qwen05b": dict(desc="24-layer Qwen2.5-0.5B-shaped stack: 168 BitLinear projections (hidden 896, "
                         "intermediate 4864), T=2048, 6:8, weights packed once; per projection "
                         "quantize_acts + bitlinear; value = tokens / step time",
                    unit="tokens/s", mode="split", qw=False, layers=None),
    "layer_small": dict(desc="single BitLinear T=16, K=N_out=256, 2:4: latency of quantize_weights + "
                             "quantize_acts + bitlinear",
                        unit="us", mode="split", qw=True, layers=[(256, 256, 2, 4, [16])]),
}
EXTRA_WORKLOADS = ["prefill", "qwen05b", "ffn3b", "layer_small", "backward"]


def workload_layers(workload):
    layers = WORKLOADS[workload]["layers"]
    return _qwen_layers() if layers is None else layers


def is_fused(workload: str) -> bool:
    """Whether the workload's steps use sbn_bitlinear_x (act-quant fused)."""
    return WORKLOADS[workload]["mode"] == "fused"


def workload_mode(workload: str):
    """"fused", "entropy" or "split" (quantize_acts + bitlinear)."""
    return WORKLOADS[workload]["mode"]


def act_bytes(t, k, n_out, n, m, mode):
    """Bytes of one token set after the weights are packed."""
    if mode is True or mode == "fused":
        return blx_bytes(t, k, n_out, n, m)
    if mode == "entropy":
        return blex_bytes(t, k, n_out, n, m)
    return qa_bytes(t, k) + bl_bytes(t, k, n_out, n, m)


def step_bytes(layers, mode=False, qw=True):
    b = 0
    for (n_out, k, n, m, ts) in layers:
        if qw:
            b += qw_bytes(n_out, k, n, m)
        if mode == "entropy":
            b += pe_bytes(n_out, k, n, m)
        for t in ts:
            b += act_bytes(t, k, n_out, n, m, mode)
    return b


def step_tokens(layers):
    return sum(sum(ts) for (_, _, _, _, ts) in layers)


def step_ops(layers):
    return sum(bl_ops(t, k, n_out, n, m) for (n_out, k, n, m, ts) in layers for t in ts)


def step_units(workload, layers):
    """Units of one step in the workload's unit (GB, T-ops, tokens or a step)."""
    unit = WORKLOADS[workload]["unit"]
    if unit == "TOPS":
        return step_ops(layers) / 1e12
    if unit == "tokens/s":
        return layers[0][4][0]          # one pass of T tokens through the stack
    if unit == "us":
        return 1.0
    w = WORKLOADS[workload]
    return step_bytes(layers, w["mode"], w["qw"]) / 1e9


def rate(workload, layers, steps, world, ms):
    """Whole-job value: units of all ranks over the slowest rank's time (for
    "us", the step latency instead)."""
    if WORKLOADS[workload]["unit"] == "us":
        return ms * 1e3 / steps
    return step_units(workload, layers) * steps * world / (ms * 1e-3)


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank contributes its own and gets the max."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(workload: str, steps: int, world: int, ms_max: float) -> float:
    """Units processed by all ranks (weak scaling: each rank runs a full step
    on its own layer) over the slowest rank's time, in the workload's unit."""
    return rate(workload, workload_layers(workload), steps, world, ms_max)


# the calls of one step, in order: (kind, layer, token count)
def step_calls(workload, layers=None):
    layers = layers if layers is not None else workload_layers(workload)
    w = WORKLOADS[workload]
    calls = []
    for li, (n_out, k, n, m, ts) in enumerate(layers):
        if w["qw"]:
            calls.append(("quantize_weights", li, None))
        if w["mode"] == "entropy":
            calls.append(("pack_entropy", li, None))
        for t in ts:
            if w["mode"] == "entropy":
                calls.append(("bitlinear_entropy_x", li, t))
            elif w["mode"] == "fused":
                calls.append(("bitlinear_x", li, t))
            else:
                calls.append(("quantize_acts", li, t))
                calls.append(("bitlinear", li, t))
    return calls


def call_bytes(kind, layer, t):
    n_out, k, n, m, _ = layer
    return {"quantize_weights": lambda: qw_bytes(n_out, k, n, m),
            "pack_entropy": lambda: pe_bytes(n_out, k, n, m),
            "quantize_acts": lambda: qa_bytes(t, k),
            "bitlinear": lambda: bl_bytes(t, k, n_out, n, m),
            "bitlinear_x": lambda: blx_bytes(t, k, n_out, n, m),
            "bitlinear_entropy_x": lambda: blex_bytes(t, k, n_out, n, m)}[kind]()


def call_ops(kind, layer, t):
    n_out, k, n, m, _ = layer
    return bl_ops(t, k, n_out, n, m) if kind.startswith("bitlinear") else 0


def call_launches(kind, t):
    """Kernels of one call: the contraction over T > 16 tokens adds the weight expansion."""
    return 2 if kind == "bitlinear" and t > 16 else 1


def tensor_bound(kind, t):
    return kind == "bitlinear" and t is not None and t > 16


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# device sources each call's kernels are built from: a recorded DRAM figure
# stays valid while these files are unchanged
TRAFFIC_FILES = {
    "quantize_weights": ["qw_stream.cuh", "qw_fused.cuh", "qw.cuh", "async.cuh", "common.cuh"],
    "quantize_acts": ["qa.cuh", "common.cuh"],
    "bitlinear_x": ["bl_gemv.cuh", "bl_decode.cuh", "expand.cuh", "qa.cuh", "async.cuh", "common.cuh"],
    "bitlinear": ["bl_tc2.cuh", "bl_tc_sp.cuh", "bl_tc.cuh", "expand_dense.cuh", "expand.cuh", "async.cuh",
                  "common.cuh"],
    "bitlinear_entropy_x": ["bl_decode_ent.cuh", "bl_decode_res.cuh", "bl_decode.cuh", "entropy.cuh",
                            "expand.cuh", "qa.cuh", "common.cuh"],
    "pack_entropy": ["entropy_pack.cuh", "entropy.cuh", "common.cuh"],
}


def kernel_source_sha(call=None):
    """Hash of the device sources of a call's kernels (all of csrc/ if unknown)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_linear_layers_fwd_b200", "csrc")
    files = TRAFFIC_FILES.get(call) or sorted(os.listdir(csrc))
    for f in sorted(files):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, workload):
    """Per-launch DRAM bytes from a committed ncu summary, if the call's kernel
    sources have not changed since it was captured; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel_key}@{workload}")
    if not e or e.get("source_sha") != kernel_source_sha(kernel_key):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.gpu = gpu_index
        self.period = period_ms
        self.proc = None

    def start(self):
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period)],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [ln.strip().split(",") for ln in self.out.read().splitlines() if ln.strip()]
        os.unlink(self.out.name)
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm, mx = float(r[1]), float(r[2])
            except (ValueError, IndexError):
                continue
            sms.append(sm)
            maxes.append(mx)
            for nm, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxes),
                "reasons": sorted(reasons), "samples": len(sms)}


def oracle_threads_one():
    """Context that limits BLAS to one thread (the oracle's numpy code is
    otherwise single-threaded), so that the CPU baseline's core count is
    exactly 1."""
    try:
        import threadpoolctl
        return threadpoolctl.threadpool_limits(limits=1)
    except Exception:  # noqa: BLE001
        import contextlib
        return contextlib.nullcontext()


# ---------------------------------------------------------------------------
# CPU oracle legs (the only places bench.py runs oracle/)
# ---------------------------------------------------------------------------

def oracle_step(layers_data, rows, mode="split"):
    """One step of the oracle on the first `rows` output features of every
    layer: quantize_weights, then quantize_acts + contraction per token set.
    mode "entropy": the weights are packed into the entropy-tight format and
    the contraction reads them back from it, as the GPU step does."""
    import oracle
    for (w, xs, n, m) in layers_data:
        ws = w[:rows]
        cb, mb, gamma, mask, dense = oracle.quantize_weights(ws, n, m)
        if mode == "entropy":
            ent = oracle.entropy_pack(mask, dense, n, m)
            dense, _ = oracle.entropy_unpack(ent, ws.shape[1], n, m)
        for x in xs:
            q, s = oracle.quantize_acts(x)
            acc = oracle.bitlinear_acc(q, dense)
            oracle.dequant_bf16(acc, s, gamma)


def make_layers_data(workload, rank=0, layers=None, first=None):
    """Seeded inputs of the workload's layers (the first `first` layers only
    when given): (w bits, [x bits per token set], n, m)."""
    from sparse_linear_layers_fwd_b200 import synth
    layers = layers if layers is not None else workload_layers(workload)
    out = []
    for li, (n_out, k, n, m, ts) in enumerate(layers[:first] if first else layers):
        tag = f"bench_{workload}_{li}_r{rank}"
        w = synth.latent_weights(n_out, k, seed=0, tag=tag)
        if workload == "qwen05b":
            xs = [synth.activations(t, k, seed=0, tag=f"{tag}_t{t}",
                                    heavy_tail_channels=synth.qwen_heavy_channels(k)) for t in ts]
        elif workload == "layer_small":
            xs = [synth.activations(t, k, seed=0, tag=f"{tag}_t{t}", outlier_channels=2) for t in ts]
        else:
            xs = [synth.activations(t, k, seed=0, tag=f"{tag}_t{t}") for t in ts]
        out.append((w, xs, n, m))
    return out


def oracle_sample(workload, layers, data, target_s, max_frac=1.0):
    """Time the oracle on a sample sized for about target_s seconds: a
    fraction of the output rows of every layer in `data` (a prefix of the
    workload's layers). Returns (seconds, fraction of one step's work done,
    description)."""
    mode = workload_mode(workload)
    frac = min(max_frac, 0.01)

    def run(f):
        t0 = time.perf_counter()
        for (w, xs, n, m), l in zip(data, layers):
            oracle_step([(w, xs, n, m)], max(1, int(l[0] * f)), mode)
        return time.perf_counter() - t0

    dt = run(frac)
    frac = min(max_frac, frac * max(1.0, target_s / max(dt, 1e-3)))
    dt = run(frac)
    # work done relative to one full step: the contraction ops (or bytes) of
    # the sampled rows of the sampled layers
    def work(ls, f):
        if WORKLOADS[workload]["unit"] in ("TOPS", "tokens/s"):
            return sum(bl_ops(t, k, max(1, int(n_out * f)), n, m) for (n_out, k, n, m, ts) in ls for t in ts)
        return step_bytes([(max(1, int(l[0] * f)),) + tuple(l[1:]) for l in ls], mode,
                          WORKLOADS[workload]["qw"])
    done = work(layers[:len(data)], frac) / work(workload_layers(workload), 1.0)
    desc = (f"{frac:.3f} of the output features of {len(data)} of {len(workload_layers(workload))} "
            f"layer(s), full K and all token sets; one pass, {dt:.1f} s")
    return dt, done, desc


def cpu_baseline(workload, target_s=10.0, first=None):
    layers = workload_layers(workload)
    data = make_layers_data(workload, 0, first=first)
    with oracle_threads_one():
        dt, done, desc = oracle_sample(workload, layers, data, target_s)
    unit = WORKLOADS[workload]["unit"]
    if unit == "us":
        value = dt / done * 1e6
    else:
        value = step_units(workload, layers) * done / dt
    return {"value": round(value, 6), "unit": unit, "cores": 1, "kind": "oracle", "sample": desc}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def l2_bytes(dev):
    import torch
    try:
        return int(torch.cuda.get_device_properties(dev).L2_cache_size) or L2_FALLBACK_BYTES
    except Exception:  # noqa: BLE001
        return L2_FALLBACK_BYTES


def to_dev(bits, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


class Engine:
    """Slots of device buffers of one workload and the calls of its steps."""

    def __init__(self, workload, layers, data, dev, stream, rotations):
        import torch
        from sparse_linear_layers_fwd_b200 import sbn
        self.sbn = sbn
        self.workload = workload
        self.w = WORKLOADS[workload]
        self.layers = layers
        self.dev = dev
        self.stream = stream
        self.calls = step_calls(workload, layers)
        base = []
        for (w, xs, n, m), (n_out, k, _, _, ts) in zip(data, layers):
            base.append((to_dev(w, dev), [to_dev(x, dev) for x in xs]))
        self.slots = []
        ws_of = {}
        for r in range(rotations):
            sl = []
            for li, ((wd, xds), (n_out, k, n, m, ts)) in enumerate(zip(base, layers)):
                L = dict(n=n, m=m)
                L["w"] = wd if r == 0 else wd.clone()
                L["xs"] = [x if r == 0 else x.clone() for x in xds]
                L["pw"] = sbn.alloc_packed(n_out, k, n, m, dev)
                L["ws"] = torch.empty(sbn.workspace_bytes(n_out, k), dtype=torch.uint8, device=dev)
                L["qs"] = [(torch.empty((t, k), dtype=torch.int8, device=dev),
                            torch.empty((t,), dtype=torch.float32, device=dev)) for t in ts]
                L["ys"] = [torch.empty((t, n_out), dtype=torch.bfloat16, device=dev) for t in ts]
                # the contraction's workspace is written and read within one
                # call, so one per shape serves every slot
                L["bws"] = ws_of.setdefault((n_out, k), torch.empty(
                    (max(1, max(max(sbn.bitlinear_workspace_bytes(t, k, n_out),
                                    sbn.bitlinear_x_workspace_bytes(t, k, n_out)) for t in ts)),),
                    dtype=torch.uint8, device=dev))
                L["ent"] = (torch.empty((n_out, sbn.entropy_row_bytes(k, n, m)), dtype=torch.uint8, device=dev)
                            if self.w["mode"] == "entropy" else None)
                sl.append(L)
            self.slots.append(sl)
        if not self.w["qw"]:
            # weights packed once, outside the timed steps
            with torch.cuda.stream(stream):
                for sl in self.slots:
                    for L in sl:
                        sbn.quantize_weights(L["w"], L["n"], L["m"], out=L["pw"], workspace=L["ws"],
                                             stream=stream)
            stream.synchronize()

    def enqueue(self, call, r):
        kind, li, t = call
        sbn, st = self.sbn, self.stream
        L = self.slots[r][li]
        ti = None if t is None else self.layers[li][4].index(t)
        if kind == "quantize_weights":
            sbn.quantize_weights(L["w"], L["n"], L["m"], out=L["pw"], workspace=L["ws"], stream=st)
        elif kind == "pack_entropy":
            sbn.pack_entropy(L["pw"], out=L["ent"], stream=st)
        elif kind == "bitlinear_entropy_x":
            sbn.bitlinear_entropy_x(L["xs"][ti], L["ent"], L["pw"], out=L["ys"][ti], workspace=False, stream=st)
        elif kind == "bitlinear_x":
            sbn.bitlinear_x(L["xs"][ti], L["pw"], out=L["ys"][ti], workspace=L["bws"], stream=st)
        elif kind == "quantize_acts":
            q, s = L["qs"][ti]
            sbn.quantize_acts(L["xs"][ti], out_q=q, out_s=s, stream=st)
        elif kind == "bitlinear":
            q, s = L["qs"][ti]
            sbn.bitlinear(q, s, L["pw"], out=L["ys"][ti], workspace=L["bws"], stream=st)
        else:
            raise ValueError(kind)

    def graph(self, calls_of_slot):
        """One CUDA graph over all slots: calls_of_slot(r) enqueued for r = 0..R-1."""
        import torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            for r in range(len(self.slots)):
                for c in calls_of_slot(r):
                    self.enqueue(c, r)
        return g

    def step_graphs(self):
        import torch
        gs = []
        for r in range(len(self.slots)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                for c in self.calls:
                    self.enqueue(c, r)
            gs.append(g)
        return gs


def replay_ms(g, stream, reps, warmup=2):
    """Mean milliseconds of one replay of graph g (events around reps replays)."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g.replay()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    stream.synchronize()
    return e0.elapsed_time(e1) / reps


def rotations_for(layers, workload, l2):
    """Slots so that the inputs of R steps exceed 3x L2, at most 96."""
    w = WORKLOADS[workload]
    per_step = sum((2 * n_out * k if w["qw"] else packed_bytes(n_out, k, n, m)) + sum(2 * t * k for t in ts)
                   for (n_out, k, n, m, ts) in layers)
    return int(min(96, max(2, math.ceil(3 * l2 / per_step))))


def kind_breakdown(eng, kinds, peaks, reps):
    """Per kind: mean duration of one launch in back-to-back per-kind graphs
    over all slots, its time per step and its achieved rate."""
    out = {}
    R = len(eng.slots)
    for kind in kinds:
        cs = [c for c in eng.calls if c[0] == kind]
        g = eng.graph(lambda r: cs)
        ms = replay_ms(g, eng.stream, reps)
        del g
        per_step_us = ms * 1e3 / R
        nbytes = sum(call_bytes(c[0], eng.layers[c[1]], c[2]) for c in cs)
        nops = sum(call_ops(c[0], eng.layers[c[1]], c[2]) for c in cs)
        e = {"calls_per_step": len(cs), "us_per_step": round(per_step_us, 3),
             "us_per_call": round(per_step_us / len(cs), 3),
             "GB/s": round(nbytes / (per_step_us * 1e-6) / 1e9, 1),
             "hbm_frac": round(nbytes / (per_step_us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)}
        if nops:
            e["TOPS"] = round(nops / (per_step_us * 1e-6) / 1e12, 3)
        out[kind] = e
    return out


def roofline_of(workload, eng, kind, per_kind, peaks, i8_peak):
    cs = [c for c in eng.calls if c[0] == kind]
    us = per_kind[kind]["us_per_step"]
    tensor = all(tensor_bound(c[0], c[2]) for c in cs)
    launches = sum(call_launches(c[0], c[2]) for c in cs)
    if tensor:
        ops = sum(call_ops(c[0], eng.layers[c[1]], c[2]) for c in cs)
        dense = sum(2 * c[2] * eng.layers[c[1]][1] * eng.layers[c[1]][0] for c in cs)
        achieved = ops / (us * 1e-6) / 1e12
        patterns = {(eng.layers[c[1]][2], eng.layers[c[1]][3]) for c in cs}
        peak, src, logical = i8_peak.for_patterns(patterns)
        return {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TOPS",
                "frac": round(achieved / peak, 4), "traffic": ncu_traffic(kind, workload), "kernel": kind,
                "ops_per_launch": ops // len(cs), "launch_us": round(us / len(cs), 3),
                "launches_per_call": launches // len(cs), "peak_source": src,
                "dense_equivalent_frac": round(dense / (us * 1e-6) / 1e12 / logical, 4)}
    nbytes = sum(call_bytes(c[0], eng.layers[c[1]], c[2]) for c in cs)
    achieved = nbytes / (us * 1e-6) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": ncu_traffic(kind, workload),
            "kernel": kind, "bytes_per_launch": nbytes // len(cs), "launch_us": round(us / len(cs), 3),
            "peak_source": f"{peaks['source']} hbm_gbs (MEASURED_PEAKS.json)"
            if peaks["source"] == "measured" else "fallback 6650 GB/s"}


def measure_i8_peak(stream, iters=32768, reps=5):
    """The INT8 dense rate of the tensor pipe, measured in this run: one CTA
    per SM issuing back-to-back tcgen05.mma kind::i8 (128 x 256 x 32, the
    prefill contraction's instruction and tile) with no loads, timed with CUDA
    events; the best of `reps` launches. Returns TOP/s."""
    import torch
    from sparse_linear_layers_fwd_b200 import sbn
    with torch.cuda.stream(stream):
        sbn.probe_i8_mma(iters, stream=stream)   # warm-up
    stream.synchronize()
    best = float("inf")
    ctas = 0
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            ctas = sbn.probe_i8_mma(iters, stream=stream)
            e1.record(stream)
        stream.synchronize()
        best = min(best, e0.elapsed_time(e1))
    assert sbn.get_device_error() == 0
    return ctas * iters * 2 * 128 * 256 * 32 / (best * 1e-3) / 1e12


def measure_i8_sparse_peak(stream, iters=32768, reps=5):
    """The sparse INT8 rate of the tensor pipe, measured in this run: CTA pairs
    issuing back-to-back tcgen05.mma.sp.cta_group::2 kind::i8 (256 x 224 x 64
    logical positions, the 2:4 prefill contraction's instruction and tile)
    with no loads; the best of `reps` launches. Returns logical TOP/s (2 per
    multiply-add of all positions; half of them are products of kept
    weights)."""
    import torch
    from sparse_linear_layers_fwd_b200 import sbn
    with torch.cuda.stream(stream):
        sbn.probe_i8_sparse_mma(iters, stream=stream)   # warm-up
    stream.synchronize()
    best = float("inf")
    pairs = 0
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            pairs = sbn.probe_i8_sparse_mma(iters, stream=stream)
            e1.record(stream)
        stream.synchronize()
        best = min(best, e0.elapsed_time(e1))
    assert sbn.get_device_error() == 0
    return pairs * iters * 2 * 256 * 224 * 64 / (best * 1e-3) / 1e12


class I8Peaks:
    """The tensor peaks a prefill contraction is measured against, in
    algorithmic operations (2 per multiply-add of a kept weight):
    - dense patterns run the dense INT8 MMA on expanded weights: the dense
      probe's rate (else 2x the measured bf16 figure, labelled derived);
    - 2:4 runs the sparse MMA, which multiplies only the kept half: half the
      sparse probe's logical rate (else the dense figure, labelled so)."""

    def __init__(self, peaks, dense_measured=None, sparse_logical=None):
        if dense_measured:
            self.dense = (dense_measured, "measured in this run: in-tree tcgen05 kind::i8 probe (sbn_probe_i8_mma)")
        else:
            self.dense = (2.0 * peaks["bf16_tflops"], f"derived: 2 x {peaks['source']} bf16_tflops "
                          f"{peaks['bf16_tflops']} (nominal int8 : bf16 ratio)")
        self.sparse_logical = sparse_logical
        if sparse_logical:
            self.sparse = (sparse_logical / 2.0, "measured in this run: half the logical rate of the in-tree "
                           "tcgen05.mma.sp kind::i8 probe on CTA pairs (sbn_probe_i8_sparse_mma); 2:4 "
                           "multiplies only the kept half")
        else:
            self.sparse = (self.dense[0], "sparse probe unavailable: dense figure " + self.dense[1])

    def for_patterns(self, patterns):
        """(peak, source, logical peak) for contractions of these (n, m)."""
        if patterns and all(nm == (2, 4) for nm in patterns):
            return self.sparse[0], self.sparse[1], 2.0 * self.sparse[0]
        return self.dense[0], self.dense[1], self.dense[0]


def run_workload(workload, args, rank, world, dev, stream, peaks, i8_peak_src, headline):
    """Measure one workload on this rank; returns its JSON entry (rank 0)."""
    import torch
    import torch.distributed as dist
    layers = workload_layers(workload)
    data = make_layers_data(workload, rank)
    l2 = l2_bytes(dev)
    R = rotations_for(layers, workload, l2)
    eng = Engine(workload, layers, data, dev, stream, R)
    with torch.cuda.stream(stream):
        for c in eng.calls:
            eng.enqueue(c, 0)        # loads the kernels before capture
    stream.synchronize()
    graphs = eng.step_graphs()
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, R)):
            graphs[i % R].replay()
    stream.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    steps = args.steps
    passes = args.passes
    clocks = ClockSampler(dev.index if dev.index is not None else 0) if headline else None
    if clocks:
        clocks.start()
    pass_ms = []
    for _ in range(passes):
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(steps):
                graphs[i % R].replay()
            e1.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        barrier()
        pass_ms.append(max_over_ranks(e0.elapsed_time(e1), world, dev))
    clk = clocks.stop() if clocks else None
    ms = statistics.median(pass_ms)
    graphs.clear()

    kinds = list(dict.fromkeys(c[0] for c in eng.calls))
    per_kind = kind_breakdown(eng, kinds, peaks, reps=max(3, args.kernel_reps))
    dom = max(per_kind, key=lambda k: per_kind[k]["us_per_step"])
    roof = roofline_of(workload, eng, dom, per_kind, peaks, i8_peak_src)
    launches = sum(call_launches(c[0], c[2]) for c in eng.calls)
    unit = WORKLOADS[workload]["unit"]
    e2e = run_e2e(workload, eng, data, dev, stream, world, steps=max(3, min(steps, args.e2e_steps)))
    entry = {
        "metric": METRIC, "value": round(rate(workload, layers, steps, world, ms), 3), "unit": unit,
        "higher_is_better": unit != "us", "ms_per_step": round(ms / steps, 5),
        "passes_ms_per_step": [round(p / steps, 5) for p in pass_ms],
        "config": {"workload": workload, "desc": WORKLOADS[workload]["desc"],
                   "bytes_per_step": step_bytes(layers, WORKLOADS[workload]["mode"], WORKLOADS[workload]["qw"]),
                   "tokens_per_step": step_tokens(layers), "ops_per_step": step_ops(layers),
                   "l2": f"inputs rotated over {R} copies (> 3x the {l2 // (1 << 20)} MiB L2) between steps",
                   "parallelism": f"replicas x{world} (independent layers per rank)"},
        "tokens_per_s": round(step_tokens(layers) * steps * world / (ms * 1e-3), 1),
        "roofline": roof, "breakdown": per_kind,
        "breakdown_note": "per kind: back-to-back launches of every call of that kind over all rotation "
                          "slots in one graph, events around the whole replay",
        "e2e": e2e, "gpu_launches": launches * steps, "clocks": clk,
    }
    del eng
    torch.cuda.empty_cache()
    return entry


def run_e2e(workload, eng, data, dev, stream, world, steps):
    """The step through the public binding from pinned host buffers: H2D of the
    step's inputs, the calls, D2H of its outputs, every step."""
    import torch
    import torch.distributed as dist
    sbn = eng.sbn
    w = WORKLOADS[workload]
    layers = eng.layers
    host = []
    for (wb, xs, n, m) in data:
        hw = (torch.from_numpy(np.ascontiguousarray(wb).view(np.int16)).view(torch.bfloat16).pin_memory()
              if w["qw"] else torch.empty((wb.shape[0], 0), dtype=torch.bfloat16))
        hxs = [torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).pin_memory()
               for x in xs]
        host.append((hw, hxs, n, m))
    ys_host = [[torch.empty((x.shape[0], h[0].shape[0]), dtype=torch.bfloat16).pin_memory() for x in h[1]]
               for h in host]
    L0 = eng.slots[0]
    h2d = sum((h[0].numel() * 2 if w["qw"] else 0) + sum(x.numel() * 2 for x in h[1]) for h in host)
    d2h = sum(y.numel() * 2 for ys in ys_host for y in ys)

    def step():
        for li, (hw, hxs, n, m) in enumerate(host):
            L = L0[li]
            if w["qw"]:
                L["w"].copy_(hw, non_blocking=True)
                sbn.quantize_weights(L["w"], n, m, out=L["pw"], workspace=L["ws"], stream=stream)
            ent = sbn.pack_entropy(L["pw"], out=L["ent"], stream=stream) if w["mode"] == "entropy" else None
            for j, hx in enumerate(hxs):
                L["xs"][j].copy_(hx, non_blocking=True)
                if w["mode"] == "entropy":
                    y = sbn.bitlinear_entropy_x(L["xs"][j], ent, L["pw"], out=L["ys"][j], workspace=False,
                                                stream=stream)
                elif w["mode"] == "fused":
                    y = sbn.bitlinear_x(L["xs"][j], L["pw"], out=L["ys"][j], workspace=L["bws"], stream=stream)
                else:
                    q, s = L["qs"][j]
                    sbn.quantize_acts(L["xs"][j], out_q=q, out_s=s, stream=stream)
                    y = sbn.bitlinear(q, s, L["pw"], out=L["ys"][j], workspace=L["bws"], stream=stream)
                ys_host[li][j].copy_(y, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(2):
            step()
    stream.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
    stream.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return {"value": round(rate(workload, layers, steps, world, ms), 3), "unit": WORKLOADS[workload]["unit"],
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 4)}


# ---------------------------------------------------------------------------
# the 3B-scale pattern sweep
# ---------------------------------------------------------------------------

def run_backward(args, dev, stream, peaks):
    """The straight-through backward of the prefill up-projection (T = 4096,
    K = 2560, N_out = 6912, 2:4): sbn_bitlinear_grad_x and sbn_bitlinear_grad_w,
    each timed back to back over rotated copies of its inputs (more than 3x L2)
    in one graph. value = 2 * T * K * N_out flops per call, both calls, over
    their summed time; the roofline divides by the measured bf16 tensor peak."""
    import torch
    from sparse_linear_layers_fwd_b200 import sbn, synth
    l2 = l2_bytes(dev)
    t, k, n_out, n, m = 4096, 2560, 6912, 2, 4
    w = to_dev(synth.latent_weights(n_out, k, seed=0, tag="bench_bwd"), dev)
    x = to_dev(synth.activations(t, k, seed=0, tag="bench_bwd_x"), dev)
    dy0 = to_dev(synth.activations(t, n_out, seed=0, tag="bench_bwd_dy"), dev)
    pw = sbn.quantize_weights(w, n, m)
    xq, xs = sbn.quantize_acts(x)
    R = int(min(16, max(2, math.ceil(3 * l2 / (2 * t * n_out)))))
    dys = [dy0] + [dy0.clone() for _ in range(R - 1)]
    dxs = [torch.empty((t, k), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    dws = [torch.empty((n_out, k), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    with torch.cuda.stream(stream):
        for i in range(R):
            sbn.bitlinear_grad_x(dys[i], pw, out=dxs[i], stream=stream)
            sbn.bitlinear_grad_w(dys[i], xq, xs, out=dws[i], stream=stream)
    stream.synchronize()
    gx, gw = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(gx, stream=stream):
        for i in range(R):
            sbn.bitlinear_grad_x(dys[i], pw, out=dxs[i], stream=stream)
    with torch.cuda.graph(gw, stream=stream):
        for i in range(R):
            sbn.bitlinear_grad_w(dys[i], xq, xs, out=dws[i], stream=stream)
    reps = max(3, args.kernel_reps)
    dx_us = replay_ms(gx, stream, reps) * 1e3 / R
    dw_us = replay_ms(gw, stream, reps) * 1e3 / R
    del gx, gw
    assert sbn.get_device_error() == 0
    flops = 2 * t * k * n_out
    peak = peaks["bf16_tflops"]
    tf_x, tf_w = flops / (dx_us * 1e-6) / 1e12, flops / (dw_us * 1e-6) / 1e12
    value = 2 * flops / ((dx_us + dw_us) * 1e-6) / 1e12
    dom, dom_us, dom_tf = ("grad_w", dw_us, tf_w) if dw_us >= dx_us else ("grad_x", dx_us, tf_x)
    return {"metric": "straight-through backward TFLOP/s (dX and dW of one layer)", "value": round(value, 2),
            "unit": "TFLOP/s", "higher_is_better": True,
            "config": {"workload": "backward",
                       "desc": "dX = gamma dY C and dW = dY^T Xd of the prefill up-projection: T=4096, K=2560, "
                               "N_out=6912, 2:4; 2*T*K*N_out flops per call (pruned positions of C included)",
                       "l2": f"dY rotated over {R} copies (> 3x L2)"},
            "calls": {"grad_x": {"us_per_call": round(dx_us, 3), "TFLOP/s": round(tf_x, 2)},
                      "grad_w": {"us_per_call": round(dw_us, 3), "TFLOP/s": round(tf_w, 2),
                                 "note": "two bf16 MMAs per step (the scaled dY split into hi and lo parts)"}},
            "roofline": {"bound": "tensor", "achieved": round(dom_tf, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(dom_tf / peak, 4), "traffic": None, "kernel": dom,
                         "launch_us": round(dom_us, 3),
                         "peak_source": f"{peaks['source']} bf16_tflops (MEASURED_PEAKS.json)"}}


def run_ffn3b(args, dev, stream, peaks, i8_peak_src, with_cpu):
    """Per pattern: sbn_quantize_weights of gate and down (the per-step dynamic
    mask, timed separately); per (pattern, projection, T): quantize_acts and
    bitlinear, each timed back to back over rotated copies of its inputs."""
    import torch
    from sparse_linear_layers_fwd_b200 import sbn, synth
    l2 = l2_bytes(dev)
    projs = [("gate", 2048, 11008), ("down", 11008, 2048)]
    entries, qw_entries = [], []
    tot_ops, tot_us = 0, 0.0
    for (pn, k, n_out) in projs:
        wbits = synth.latent_weights(n_out, k, seed=0, tag=f"bench_ffn3b_{pn}")
        wd = to_dev(wbits, dev)
        xs_dev = {t: to_dev(synth.activations(t, k, seed=0, tag=f"bench_ffn3b_{pn}_t{t}"), dev)
                  for t in synth.FFN3B_TOKENS}
        ws = torch.empty(sbn.workspace_bytes(n_out, k), dtype=torch.uint8, device=dev)
        for (n, m) in synth.FFN3B_PATTERNS:
            # quantize_weights: rotated latent copies
            Rw = int(min(24, max(2, math.ceil(3 * l2 / (2 * n_out * k)))))
            wcopies = [wd] + [wd.clone() for _ in range(Rw - 1)]
            pws = [sbn.alloc_packed(n_out, k, n, m, dev) for _ in range(Rw)]
            with torch.cuda.stream(stream):
                for i in range(Rw):
                    sbn.quantize_weights(wcopies[i], n, m, out=pws[i], workspace=ws, stream=stream)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(Rw):
                    sbn.quantize_weights(wcopies[i], n, m, out=pws[i], workspace=ws, stream=stream)
            us = replay_ms(g, stream, max(3, args.kernel_reps)) * 1e3 / Rw
            del g
            qb = qw_bytes(n_out, k, n, m)
            qw_entries.append({"proj": pn, "pattern": f"{n}:{m}", "us": round(us, 3),
                               "GB/s": round(qb / (us * 1e-6) / 1e9, 1),
                               "hbm_frac": round(qb / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)})
            del wcopies
            for t in synth.FFN3B_TOKENS:
                x = xs_dev[t]
                per = bl_bytes(t, k, n_out, n, m)
                R = int(min(48, max(1, math.ceil(3 * l2 / per))))
                pw_r = [pws[i % Rw] for i in range(R)]
                xq = [torch.empty((t, k), dtype=torch.int8, device=dev) for _ in range(R)]
                xsc = [torch.empty((t,), dtype=torch.float32, device=dev) for _ in range(R)]
                ys = [torch.empty((t, n_out), dtype=torch.bfloat16, device=dev) for _ in range(R)]
                xcopies = [x] + [x.clone() for _ in range(R - 1)]
                bws = torch.empty((max(1, sbn.bitlinear_workspace_bytes(t, k, n_out)),), dtype=torch.uint8,
                                  device=dev)
                with torch.cuda.stream(stream):
                    for i in range(R):
                        sbn.quantize_acts(xcopies[i], out_q=xq[i], out_s=xsc[i], stream=stream)
                        sbn.bitlinear(xq[i], xsc[i], pw_r[i], out=ys[i], workspace=bws, stream=stream)
                stream.synchronize()
                ga, gb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
                with torch.cuda.graph(ga, stream=stream):
                    for i in range(R):
                        sbn.quantize_acts(xcopies[i], out_q=xq[i], out_s=xsc[i], stream=stream)
                with torch.cuda.graph(gb, stream=stream):
                    for i in range(R):
                        sbn.bitlinear(xq[i], xsc[i], pw_r[i], out=ys[i], workspace=bws, stream=stream)
                reps = max(3, args.kernel_reps if t < 8192 else 3)
                qa_us = replay_ms(ga, stream, reps) * 1e3 / R
                bl_us = replay_ms(gb, stream, reps) * 1e3 / R
                del ga, gb
                ops = bl_ops(t, k, n_out, n, m)
                tot_ops += ops
                tot_us += bl_us
                e = {"proj": pn, "pattern": f"{n}:{m}", "T": t, "bitlinear_us": round(bl_us, 3),
                     "TOPS": round(ops / (bl_us * 1e-6) / 1e12, 3),
                     "weight_GB/s": round(packed_bytes(n_out, k, n, m) / (bl_us * 1e-6) / 1e9, 1),
                     "quantize_acts_us": round(qa_us, 3)}
                if t > 16:
                    peak, _src, _lg = i8_peak_src.for_patterns({(n, m)})
                    e["bound"] = "tensor"
                    e["frac"] = round(ops / (bl_us * 1e-6) / 1e12 / peak, 4)
                else:
                    e["bound"] = "hbm"
                    e["frac"] = round(per / (bl_us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)
                entries.append(e)
                del xq, xsc, ys, xcopies, bws, pw_r
            del pws
        del wd, xs_dev
        torch.cuda.empty_cache()
    tops = tot_ops / (tot_us * 1e-6) / 1e12
    big = [e for e in entries if e["T"] >= 512]
    dom = max(big, key=lambda e: e["bitlinear_us"])
    peak, src, _lg = i8_peak_src.for_patterns({tuple(int(v) for v in dom["pattern"].split(":"))})
    out = {"metric": METRIC, "value": round(tops, 3), "unit": "TOPS", "higher_is_better": True,
           "config": {"workload": "ffn3b",
                      "desc": "3B-scale FFN sweep: gate (K=2048, N_out=11008) and down (K=11008, N_out=2048), "
                              "T in {1,64,512,8192} x n:m in {2:4,4:8,6:8,8:16,8:8}; value = algorithmic ops "
                              "of every contraction / their summed times; quantize_weights timed separately",
                      "l2": "each entry rotated over enough input copies to exceed 3x L2"},
           "roofline": {"bound": "tensor", "achieved": dom["TOPS"], "peak": round(peak, 1), "unit": "TOPS",
                        "frac": dom["frac"], "traffic": None, "kernel": "bitlinear",
                        "entry": f"{dom['proj']} {dom['pattern']} T={dom['T']}", "peak_source": src},
           "sweep": entries, "quantize_weights": qw_entries}
    if with_cpu:
        out["cpu_baseline"] = ffn3b_cpu_baseline()
    out["e2e"] = None
    out["e2e_note"] = "per-entry kernel timings only; end-to-end figures are given for the other workloads"
    return out


def ffn3b_cpu_baseline(target_s=8.0):
    """The oracle on a row sample of the 6:8 gate projection at T = 64 (TOPS)."""
    import oracle
    from sparse_linear_layers_fwd_b200 import synth
    w = synth.latent_weights(11008, 2048, seed=0, tag="bench_ffn3b_gate")
    x = synth.activations(64, 2048, seed=0, tag="bench_ffn3b_gate_t64")
    with oracle_threads_one():
        rows = 16
        t0 = time.perf_counter()
        oracle_step([(w, [x], 6, 8)], rows)
        dt = time.perf_counter() - t0
        rows = int(min(11008, max(16, rows * target_s / max(dt, 1e-3))))
        t0 = time.perf_counter()
        oracle_step([(w, [x], 6, 8)], rows)
        dt = time.perf_counter() - t0
    ops = bl_ops(64, 2048, rows, 6, 8)
    return {"value": round(ops / dt / 1e12, 9), "unit": "TOPS", "cores": 1, "kind": "oracle",
            "sample": f"gate projection 6:8, T=64, {rows} of 11008 output features; quantize_weights + "
                      f"quantize_acts + contraction; one pass, {dt:.1f} s"}


# ---------------------------------------------------------------------------
# driver
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    import torch
    from sparse_linear_layers_fwd_b200 import sbn
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    sbn.lib()
    stream = torch.cuda.Stream(device=dev)
    peaks = load_peaks()
    i8_measured = sp_measured = None
    try:
        i8_measured = measure_i8_peak(stream)
    except Exception as ex:  # noqa: BLE001
        print(f"i8 probe unavailable: {ex}", file=sys.stderr)
    try:
        sp_measured = measure_i8_sparse_peak(stream)
    except Exception as ex:  # noqa: BLE001
        print(f"sparse i8 probe unavailable: {ex}", file=sys.stderr)
    i8 = I8Peaks(peaks, i8_measured, sp_measured)
    head = run_workload(args.workload, args, rank, world, dev, stream, peaks, i8, headline=True)
    extras = {}
    if world == 1 and not args.only:
        for wl in EXTRA_WORKLOADS:
            if wl == args.workload:
                continue
            try:
                if wl == "ffn3b":
                    extras[wl] = run_ffn3b(args, dev, stream, peaks, i8, with_cpu=not args.no_cpu_baseline)
                elif wl == "backward":
                    extras[wl] = run_backward(args, dev, stream, peaks)
                else:
                    e = run_workload(wl, args, rank, world, dev, stream, peaks, i8, headline=False)
                    if not args.no_cpu_baseline:
                        e["cpu_baseline"] = cpu_baseline(wl, target_s=args.cpu_seconds / 2,
                                                         first=7 if wl == "qwen05b" else None)
                    extras[wl] = e
            except torch.cuda.OutOfMemoryError as ex:  # noqa: PERF203
                extras[wl] = {"error": f"out of device memory: {ex}"[:200]}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, target_s=args.cpu_seconds)
    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": head["higher_is_better"], "scaling": "weak", "vs_baseline": None,
            "dtype": DTYPE, "data": DATA_DESC, "config": head["config"],
            "passes_ms_per_step": head["passes_ms_per_step"], "tokens_per_s": head["tokens_per_s"],
            "roofline": head["roofline"], "breakdown": head["breakdown"],
            "breakdown_note": head["breakdown_note"], "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"], "clocks": head["clocks"], "cpu_baseline": cpu,
            "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"],
                      "i8_tops": round(i8.dense[0], 1), "i8_source": i8.dense[1],
                      "i8_sparse_tops_logical": round(i8.sparse_logical, 1) if i8.sparse_logical else None,
                      "i8_sparse_tops_algorithmic": round(i8.sparse[0], 1), "i8_sparse_source": i8.sparse[1]},
        }
        if extras:
            line["workloads"] = extras
        print(json.dumps(line), flush=True)


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm, on the same config, metric and
    unit: every step is the same bounded sample of the workload."""
    if rank != 0:
        return
    workload = args.workload
    layers = workload_layers(workload)
    mode = workload_mode(workload)
    data = make_layers_data(workload, 0, first=7 if workload == "qwen05b" else None)
    per_step = max(0.01, args.reference_seconds / max(1, args.steps + args.warmup))
    with oracle_threads_one():
        _dt, done, desc = oracle_sample(workload, layers, data, per_step)   # sizes the sample
        frac = desc_frac(desc)
        for _ in range(args.warmup):
            oracle_sample_step(workload, layers, data, frac)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle_sample_step(workload, layers, data, frac)
        dt = time.perf_counter() - t0
    unit = WORKLOADS[workload]["unit"]
    if unit == "us":
        value = dt / args.steps / done * 1e6
    else:
        value = step_units(workload, layers) * done * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": unit != "us",
        "scaling": "weak", "vs_baseline": None, "dtype": DTYPE, "data": DATA_DESC,
        "config": {"workload": workload, "desc": WORKLOADS[workload]["desc"],
                   "bytes_per_step": step_bytes(layers, mode, WORKLOADS[workload]["qw"]),
                   "tokens_per_step": step_tokens(layers), "ops_per_step": step_ops(layers),
                   "l2": "host CPU (no GPU L2)", "parallelism": f"replicas x{world} (independent layers per rank)"},
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": 1, "kind": "oracle",
                         "sample": "each step: " + desc},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def desc_frac(desc):
    return float(desc.split(" ", 1)[0])


def oracle_sample_step(workload, layers, data, frac):
    mode = workload_mode(workload)
    for (w, xs, n, m), l in zip(data, layers):
        oracle_step([(w, xs, n, m)], max(1, int(l[0] * frac)), mode)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--passes", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode")
    ap.add_argument("--only", action="store_true", help="the headline workload only")
    ap.add_argument("--kernel-reps", type=int, default=20)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-seconds", type=float, default=60.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
