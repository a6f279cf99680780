#!/usr/bin/env python
"""Benchmark of the Sparse-BitNet BitLinear forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill|decode_entropy]

One step is one pass of the whole path over one batch of synthetic input:
sbn_quantize_weights on the latent weights (the dynamic N:M mask is
recomputed every forward), then, for every token set, the activation
quantization and the contraction: sbn_bitlinear_x (fused) for the decode
workload, sbn_quantize_acts + sbn_bitlinear for prefill. The default workload
is the decode GEMV sweep: W [6912, 2560] bf16 ~ N(0, 0.02), 6:8, activations
of T = 1, 4 and 16 tokens. The prefill workload is T = 4096 through
(K, N_out) = (2560, 6912) and (6912, 2560) at 2:4. decode_entropy is the
decode sweep over the entropy-tight weight format (sbn_pack_entropy +
sbn_bitlinear_entropy_x). The other shapes of the pages' workloads are
covered by the parity tests.

Timing: each step is a captured CUDA graph; steps rotate over enough
distinct copies of the inputs and outputs that their total exceeds 3x the
L2 cache, so no step reads another step's data from L2. An untimed
calibration replay with events around every call gives the per-call
breakdown; the timed replays bracket only the dominant call. The timed region is
K graph replays bracketed by barrier + synchronize, timed with CUDA events;
for N > 1 the max over ranks is taken and every rank runs its own
independent layer (weak scaling, no collective on the data path).

Rank 0 prints one JSON line.
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
L2_BYTES = 126 * 1024 * 1024


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


WORKLOADS = {
    # name: list of layers (n_out, k, n, m, [token counts]) in one step
    "decode": dict(desc="decode GEMV sweep: K=2560, N_out=6912, 6:8, T in {1,4,16}; value = "
                        "algorithmic bytes of the step / step time; activation quantization "
                        "fused into the contraction (sbn_bitlinear_x)",
                   unit="GB/s", fused=True, layers=[(6912, 2560, 6, 8, [1, 4, 16])]),
    "decode_entropy": dict(desc="decode GEMV sweep over entropy-tight weights: K=2560, N_out=6912, "
                                "6:8, T in {1,4,16}; each step packs the quantized layer into the "
                                "entropy-tight format (1.875 bit/weight) and contracts from it",
                           unit="GB/s", mode="entropy", layers=[(6912, 2560, 6, 8, [1, 4, 16])]),
    "prefill": dict(desc="prefill GEMM: T=4096, (K,N_out)=(2560,6912) and (6912,2560), 2:4; value = "
                         "algorithmic ops (2 per kept multiply-add) of the step / step time",
                    unit="TOPS", layers=[(6912, 2560, 2, 4, [4096]), (2560, 6912, 2, 4, [4096])]),
}


def act_bytes(t, k, n_out, n, m, mode):
    """Bytes of one token set after the weights are packed (mode: True or
    "fused", False or "split", "entropy")."""
    if mode is True or mode == "fused":
        return blx_bytes(t, k, n_out, n, m)
    if mode == "entropy":
        return blex_bytes(t, k, n_out, n, m)
    return qa_bytes(t, k) + bl_bytes(t, k, n_out, n, m)


def step_bytes(layers, mode=False):
    b = 0
    for (n_out, k, n, m, ts) in layers:
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


# ---------------------------------------------------------------------------
# across ranks (one process per GPU, each on its own independent layer)
# ---------------------------------------------------------------------------

def is_fused(workload: str) -> bool:
    """Whether the workload's steps use sbn_bitlinear_x (act-quant fused)."""
    return bool(WORKLOADS[workload].get("fused", False))


def workload_mode(workload: str):
    """"fused", "entropy" or "split" (quantize_acts + bitlinear)."""
    w = WORKLOADS[workload]
    return w.get("mode", "fused" if w.get("fused") else "split")


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
    layers = WORKLOADS[workload]["layers"]
    if WORKLOADS[workload]["unit"] == "TOPS":
        return step_ops(layers) * steps * world / (ms_max * 1e-3) / 1e12
    return step_bytes(layers, workload_mode(workload)) * steps * world / (ms_max * 1e-3) / 1e9


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
    "quantize_weights": ["qw_fused.cuh", "qw.cuh", "async.cuh", "common.cuh"],
    "bitlinear_x": ["bl_decode_res.cuh", "bl_decode.cuh", "expand.cuh", "qa.cuh", "common.cuh"],
    "bitlinear": ["bl_tc.cuh", "expand_dense.cuh", "expand.cuh", "async.cuh", "common.cuh"],
    "bitlinear_entropy": ["bl_decode_ent.cuh", "bl_decode_res.cuh", "bl_decode.cuh", "entropy.cuh",
                          "expand.cuh", "common.cuh"],
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
        self.t0 = self.t1 = None

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

    def mark(self, which):
        setattr(self, which, time.time())

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


def cores_used():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        blas = max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
        return int(blas)
    except Exception:  # noqa: BLE001
        return 1


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


def oracle_sample_bytes(layers, rows_frac, fused=False):
    tot = 0
    for (n_out, k, n, m, ts) in layers:
        r = max(1, int(n_out * rows_frac))
        tot += qw_bytes(r, k, n, m)
        for t in ts:
            tot += act_bytes(t, k, r, n, m, fused)
        if fused == "entropy":
            tot += pe_bytes(r, k, n, m)
    return tot


def oracle_sample_metric(workload, layers, rows_frac):
    """The sample's amount of work in the workload's unit (GB or T-ops)."""
    if WORKLOADS[workload]["unit"] == "TOPS":
        tot = 0
        for (n_out, k, n, m, ts) in layers:
            r = max(1, int(n_out * rows_frac))
            tot += sum(bl_ops(t, k, r, n, m) for t in ts)
        return tot / 1e12
    return oracle_sample_bytes(layers, rows_frac, workload_mode(workload)) / 1e9


def make_layers_data(workload, rank=0):
    from sparse_linear_layers_fwd_b200 import synth
    out = []
    for li, (n_out, k, n, m, ts) in enumerate(WORKLOADS[workload]["layers"]):
        tag = f"bench_{workload}_{li}_r{rank}"
        w = synth.latent_weights(n_out, k, seed=0, tag=tag)
        xs = [synth.activations(t, k, seed=0, tag=f"{tag}_t{t}") for t in ts]
        out.append((w, xs, n, m))
    return out


def run_oracle_timed(layers, data, target_s, max_frac=1.0, mode="split"):
    """Time the oracle on a row sample sized for about target_s seconds."""
    frac = min(max_frac, 0.02)
    rows_of = lambda f: [max(1, int(l[0] * f)) for l in layers]  # noqa: E731
    t0 = time.perf_counter()
    for (w, xs, n, m), r in zip(data, rows_of(frac)):
        oracle_step([(w, xs, n, m)], r, mode)
    dt = time.perf_counter() - t0
    frac = min(max_frac, frac * max(1.0, target_s / max(dt, 1e-3)))
    t0 = time.perf_counter()
    for (w, xs, n, m), r in zip(data, rows_of(frac)):
        oracle_step([(w, xs, n, m)], r, mode)
    dt = time.perf_counter() - t0
    return frac, dt


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from sparse_linear_layers_fwd_b200 import sbn

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    sbn.lib()
    layers = WORKLOADS[args.workload]["layers"]
    data = make_layers_data(args.workload, rank)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    in_bytes = sum(w.nbytes + sum(x.nbytes for x in xs) for (w, xs, _, _) in data)
    R = max(2, math.ceil(3 * L2_BYTES / in_bytes))
    stream = torch.cuda.Stream(device=dev)

    # R rotation slots of inputs, packed weights, activations and outputs
    slots = []
    layer_bws = {}
    for _ in range(R):
        sl = []
        for (w, xs, n, m), (n_out, k, _, _, ts) in zip(data, layers):
            wd = to_dev(w)
            xds = [to_dev(x) for x in xs]
            pw = sbn.alloc_packed(n_out, k, n, m, dev)
            ws = torch.empty(sbn.workspace_bytes(n_out, k), dtype=torch.uint8, device=dev)
            qs = [(torch.empty((t, k), dtype=torch.int8, device=dev),
                   torch.empty((t,), dtype=torch.float32, device=dev)) for t in ts]
            ys = [torch.empty((t, n_out), dtype=torch.bfloat16, device=dev) for t in ts]
            # the contraction's workspace (expanded weights, T > 16); written
            # and read within one call, so one per layer serves every slot
            bws = layer_bws.setdefault((n_out, k), torch.empty(
                (max(1, max(max(sbn.bitlinear_workspace_bytes(t, k, n_out),
                                sbn.bitlinear_x_workspace_bytes(t, k, n_out)) for t in ts)),),
                dtype=torch.uint8, device=dev))
            ent = (torch.empty((n_out, sbn.entropy_row_bytes(k, n, m)), dtype=torch.uint8, device=dev)
                   if workload_mode(args.workload) == "entropy" else None)
            sl.append(dict(w=wd, xs=xds, pw=pw, ws=ws, bws=bws, qs=qs, ys=ys, n=n, m=m, ent=ent))
        slots.append(sl)

    # per-call events inside each slot's graph: names of the calls in order
    fused = is_fused(args.workload)
    mode = workload_mode(args.workload)
    call_names = []
    for li, (n_out, k, n, m, ts) in enumerate(layers):
        call_names.append(("quantize_weights", li, None))
        if mode == "entropy":
            call_names.append(("pack_entropy", li, None))
        for t in ts:
            if mode == "entropy":
                call_names.append(("bitlinear_entropy_x", li, t))
            elif fused:
                call_names.append(("bitlinear_x", li, t))
            else:
                call_names.append(("quantize_acts", li, t))
                call_names.append(("bitlinear", li, t))

    def enqueue_step(sl, evs=None):
        i = 0
        for li, L in enumerate(sl):
            if evs and evs[i]: evs[i][0].record(stream)
            sbn.quantize_weights(L["w"], L["n"], L["m"], out=L["pw"], workspace=L["ws"], stream=stream)
            if evs and evs[i]: evs[i][1].record(stream)
            i += 1
            if mode == "entropy":
                if evs and evs[i]: evs[i][0].record(stream)
                sbn.pack_entropy(L["pw"], out=L["ent"], stream=stream)
                if evs and evs[i]: evs[i][1].record(stream)
                i += 1
            for x, (q, s), y in zip(L["xs"], L["qs"], L["ys"]):
                if mode == "entropy":
                    if evs and evs[i]: evs[i][0].record(stream)
                    sbn.bitlinear_entropy_x(x, L["ent"], L["pw"], out=y, workspace=False, stream=stream)
                    if evs and evs[i]: evs[i][1].record(stream)
                    i += 1
                    continue
                if fused:
                    if evs and evs[i]: evs[i][0].record(stream)
                    sbn.bitlinear_x(x, L["pw"], out=y, workspace=L["bws"], stream=stream)
                    if evs and evs[i]: evs[i][1].record(stream)
                    i += 1
                    continue
                if evs and evs[i]: evs[i][0].record(stream)
                sbn.quantize_acts(x, out_q=q, out_s=s, stream=stream)
                if evs and evs[i]: evs[i][1].record(stream)
                i += 1
                if evs and evs[i]: evs[i][0].record(stream)
                sbn.bitlinear(q, s, L["pw"], out=y, workspace=L["bws"], stream=stream)
                if evs and evs[i]: evs[i][1].record(stream)
                i += 1

    def capture(which):
        """One graph per slot; events around the calls `which` selects."""
        gs, evss = [], []
        for r in range(R):
            evs = [(torch.cuda.Event(enable_timing=True, external=True),
                    torch.cuda.Event(enable_timing=True, external=True)) if which(c) else None
                   for c in call_names]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                enqueue_step(slots[r], evs)
            gs.append(g)
            evss.append(evs)
        return gs, evss

    with torch.cuda.stream(stream):
        enqueue_step(slots[0])  # load kernels before capture
    stream.synchronize()
    # calibration graphs: every call bracketed by events (per-call breakdown)
    cal_graphs, cal_events = capture(lambda c: True)
    # our kernels per step: quantize_weights 1 per layer; quantize_acts 1 and
    # bitlinear 1 (+1 weight expansion when T > 16) per token set
    # (fused: one kernel per token set for T <= 16)
    # (entropy: + 1 pack per layer, then one fused entropy contraction per token set)
    launches_per_step = sum(1 + (1 if mode == "entropy" else 0)
                            + sum((1 if mode == "entropy" else
                                   1 if fused and t <= 16 else 2 + (1 if t > 16 else 0))
                                  for t in ts)
                            for (_, _, _, _, ts) in layers)

    def barrier():
        if world > 1:
            dist.barrier()

    # warm-up, then one calibration replay per slot (untimed)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            cal_graphs[i % R].replay()
        for r in range(R):
            cal_graphs[r].replay()
    stream.synchronize()
    per_call = {}
    for r in range(R):
        for (name, li, t), ab in zip(call_names, cal_events[r]):
            per_call.setdefault((name, li, t), []).append(ab[0].elapsed_time(ab[1]))
    cal_totals = {}
    for (name, li, t), v in per_call.items():
        cal_totals[name] = cal_totals.get(name, 0.0) + statistics.mean(v)
    dom = max(cal_totals, key=cal_totals.get)
    # timed graphs: events only around the dominant call (its live launch
    # durations for the roofline), so the other calls run back to back
    graphs, slot_events = capture(lambda c: c[0] == dom)
    with torch.cuda.stream(stream):
        for r in range(R):
            graphs[r].replay()
    stream.synchronize()

    clocks = ClockSampler(local_rank)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for i in range(args.steps):
            graphs[i % R].replay()
        ev1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1)

    # the dominant call's durations in the last timed replay of every slot
    used = min(R, args.steps)
    dom_calls = {}
    for r in range(used):
        for (name, li, t), ab in zip(call_names, slot_events[r]):
            if ab:
                dom_calls.setdefault((name, li, t), []).append(ab[0].elapsed_time(ab[1]))

    ms = max_over_ranks(ms, world, dev)

    sb = step_bytes(layers, mode)
    ms_per_step = ms / args.steps
    value = whole_job_value(args.workload, args.steps, world, ms)

    # dominant call (by total time in a calibration step): its time per step
    # in the timed region
    dom_ms = sum(statistics.mean(v) for v in dom_calls.values())
    peaks = load_peaks()
    n_dom_launches = len([c for c in call_names if c[0] == dom])
    traffic = ncu_traffic(dom, args.workload)
    tensor_bound = dom == "bitlinear" and min(t for (_, _, _, _, ts) in layers for t in ts) > 16
    if tensor_bound:
        # contraction on the tensor cores: algorithmic ops (2 per kept
        # multiply-add) against the INT8 peak = measured bf16 peak x 2 (the
        # nominal int8 : bf16 ratio of 4.5 : 2.25 POPS)
        dom_ops = sum(bl_ops(t, k, n_out, n, m) for (n_out, k, n, m, ts) in layers for t in ts)
        achieved = dom_ops / (dom_ms * 1e-3) / 1e12
        peak = 2.0 * peaks["bf16_tflops"]
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1),
                    "unit": "TOPS", "frac": round(achieved / peak, 4), "traffic": traffic,
                    "kernel": dom, "ops_per_launch": dom_ops // n_dom_launches,
                    "launch_us": round(dom_ms * 1e3 / n_dom_launches, 3),
                    "peak_source": f"2 x {peaks['source']} bf16_tflops {peaks['bf16_tflops']} "
                                   f"(MEASURED_PEAKS.json; int8 = 2 x bf16 nominal)",
                    "dense_equivalent_frac": round(
                        sum(2 * t * k * n_out for (n_out, k, n, m, ts) in layers for t in ts)
                        / (dom_ms * 1e-3) / 1e12 / peak, 4)}
    else:
        if dom == "quantize_weights":
            dom_bytes = sum(qw_bytes(n_out, k, n, m) for (n_out, k, n, m, ts) in layers)
        elif dom == "quantize_acts":
            dom_bytes = sum(qa_bytes(t, k) for (n_out, k, n, m, ts) in layers for t in ts)
        elif dom == "bitlinear_x":
            dom_bytes = sum(blx_bytes(t, k, n_out, n, m) for (n_out, k, n, m, ts) in layers for t in ts)
        elif dom == "bitlinear_entropy":
            dom_bytes = sum(ble_bytes(t, k, n_out, n, m) for (n_out, k, n, m, ts) in layers for t in ts)
        elif dom == "bitlinear_entropy_x":
            dom_bytes = sum(blex_bytes(t, k, n_out, n, m) for (n_out, k, n, m, ts) in layers for t in ts)
        elif dom == "pack_entropy":
            dom_bytes = sum(pe_bytes(n_out, k, n, m) for (n_out, k, n, m, ts) in layers)
        else:
            dom_bytes = sum(bl_bytes(t, k, n_out, n, m) for (n_out, k, n, m, ts) in layers for t in ts)
        achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                    "traffic": traffic, "kernel": dom,
                    "bytes_per_launch": dom_bytes // n_dom_launches,
                    "launch_us": round(dom_ms * 1e3 / n_dom_launches, 3),
                    "peak_source": f"{peaks['source']} hbm_gbs (MEASURED_PEAKS.json)"
                    if peaks["source"] == "measured" else "fallback 6650 GB/s"}
    breakdown = {}
    for (name, li, t), v in per_call.items():
        key = f"{name}[L{li}]" + (f"[T={t}]" if t else "")
        n_out, k, n, m, _ = layers[li]
        us = statistics.mean(v) * 1e3
        if name == "quantize_weights":
            b = qw_bytes(n_out, k, n, m)
        elif name == "quantize_acts":
            b = qa_bytes(t, k)
        elif name == "bitlinear_x":
            b = blx_bytes(t, k, n_out, n, m)
        elif name == "bitlinear_entropy":
            b = ble_bytes(t, k, n_out, n, m)
        elif name == "bitlinear_entropy_x":
            b = blex_bytes(t, k, n_out, n, m)
        elif name == "pack_entropy":
            b = pe_bytes(n_out, k, n, m)
        else:
            b = bl_bytes(t, k, n_out, n, m)
        e = {"us": round(us, 3), "GB/s": round(b / (us * 1e-6) / 1e9, 1),
             "hbm_frac": round(b / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)}
        if name in ("bitlinear", "bitlinear_x", "bitlinear_entropy", "bitlinear_entropy_x"):
            wb = (entropy_bytes(n_out, k, n, m) if name.startswith("bitlinear_entropy")
                  else packed_bytes(n_out, k, n, m))
            e["weight_GB/s"] = round(wb / (us * 1e-6) / 1e9, 1)
            ops = bl_ops(t, k, n_out, n, m)
            e["TOPS"] = round(ops / (us * 1e-6) / 1e12, 3)
            e["dense_eq_TOPS"] = round(2 * t * k * n_out / (us * 1e-6) / 1e12, 3)
            e["tokens_per_s"] = round(t / (us * 1e-6), 1)
        breakdown[key] = e

    # ---- end to end through the public API with pinned host buffers ----
    e2e = run_e2e(args, data, layers, dev, stream, world)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N=1 only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        frac, dt = run_oracle_timed(layers, data, target_s=args.cpu_seconds, mode=workload_mode(args.workload))
        cpu = {"value": round(oracle_sample_metric(args.workload, layers, frac) / dt, 6),
               "unit": WORKLOADS[args.workload]["unit"], "cores": cores_used(),
               "kind": "oracle",
               "sample": f"{frac:.3f} of the output features of every layer, full K and all "
                         f"token sets; one pass, {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": WORKLOADS[args.workload]["unit"],
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8xternary->int32, bf16 io",
            "data": "synthetic (seeded: W ~ N(0,0.02) bf16, X ~ N(0,1) bf16)",
            "config": {"workload": args.workload, "desc": WORKLOADS[args.workload]["desc"],
                       "bytes_per_step": sb, "tokens_per_step": step_tokens(layers),
                       "ops_per_step": step_ops(layers),
                       "l2": f"inputs rotated over {R} copies (> 3x L2) between steps",
                       "parallelism": f"replicas x{world} (independent layers per rank)"},
            "tokens_per_s": round(step_tokens(layers) * args.steps * world / (ms * 1e-3), 1),
            "roofline": roofline, "breakdown": breakdown,
            "breakdown_note": "per-call means from one untimed replay per rotation slot with "
                              "events around every call; the timed replays bracket only the "
                              "dominant call (roofline.launch_us)",
            "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "clocks": clk, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    graphs.clear()


def run_e2e(args, data, layers, dev, stream, world):
    import torch
    import torch.distributed as dist
    from sparse_linear_layers_fwd_b200 import sbn

    host = []
    for (w, xs, n, m) in data:
        hw = torch.from_numpy(np.ascontiguousarray(w).view(np.int16)).view(torch.bfloat16).pin_memory()
        hxs = [torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).pin_memory()
               for x in xs]
        host.append((hw, hxs, n, m))
    dw = [torch.empty(h[0].shape, dtype=torch.bfloat16, device=dev) for h in host]
    dxs = [[torch.empty(x.shape, dtype=torch.bfloat16, device=dev) for x in h[1]] for h in host]
    ys_host = [[torch.empty((x.shape[0], h[0].shape[0]), dtype=torch.bfloat16).pin_memory()
                for x in h[1]] for h in host]
    h2d = sum(h[0].numel() * 2 + sum(x.numel() * 2 for x in h[1]) for h in host)
    d2h = sum(y.numel() * 2 for ys in ys_host for y in ys)
    ws = [torch.empty(sbn.workspace_bytes(*h[0].shape), dtype=torch.uint8, device=dev) for h in host]
    pws = [sbn.alloc_packed(h[0].shape[0], h[0].shape[1], h[2], h[3], dev) for h in host]

    fused = is_fused(args.workload)
    mode = workload_mode(args.workload)

    def step():
        for li, (hw, hxs, n, m) in enumerate(host):
            dw[li].copy_(hw, non_blocking=True)
            sbn.quantize_weights(dw[li], n, m, out=pws[li], workspace=ws[li], stream=stream)
            ent = sbn.pack_entropy(pws[li], stream=stream) if mode == "entropy" else None
            for j, hx in enumerate(hxs):
                dxs[li][j].copy_(hx, non_blocking=True)
                if mode == "entropy":
                    y = sbn.bitlinear_entropy_x(dxs[li][j], ent, pws[li], workspace=False, stream=stream)
                elif fused:
                    y = sbn.bitlinear_x(dxs[li][j], pws[li], stream=stream)
                else:
                    q, s = sbn.quantize_acts(dxs[li][j], stream=stream)
                    y = sbn.bitlinear(q, s, pws[li], stream=stream)
                ys_host[li][j].copy_(y, non_blocking=True)

    steps = max(3, min(args.steps, args.e2e_steps))
    with torch.cuda.stream(stream):
        for _ in range(max(3, min(args.warmup, 10))):
            step()
    stream.synchronize()
    if world > 1:
        dist.barrier()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
    stream.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    ev = whole_job_value(args.workload, steps, world, ms)
    return {"value": round(ev, 3), "unit": WORKLOADS[args.workload]["unit"],
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 4)}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle as it stands
# ---------------------------------------------------------------------------

def run_reference(args, rank, world):
    if rank != 0:
        return
    layers = WORKLOADS[args.workload]["layers"]
    data = make_layers_data(args.workload, 0)
    total_steps = args.steps + args.warmup
    per_step = max(0.01, args.reference_seconds / max(1, total_steps))
    mode = workload_mode(args.workload)
    frac, _ = run_oracle_timed(layers, data, target_s=per_step, mode=mode)
    rows = [max(1, int(l[0] * frac)) for l in layers]
    for _ in range(args.warmup):
        for d, r in zip(data, rows):
            oracle_step([d], r, mode)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for d, r in zip(data, rows):
            oracle_step([d], r, mode)
    dt = time.perf_counter() - t0
    value = oracle_sample_metric(args.workload, layers, frac) * args.steps / dt
    unit = WORKLOADS[args.workload]["unit"]
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8xternary->int32, bf16 io",
        "data": "synthetic (seeded: W ~ N(0,0.02) bf16, X ~ N(0,1) bf16)",
        "config": {"workload": args.workload, "desc": WORKLOADS[args.workload]["desc"],
                   "bytes_per_step": step_bytes(layers, workload_mode(args.workload)),
                   "tokens_per_step": step_tokens(layers)},
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": cores_used(),
                         "kind": "oracle",
                         "sample": f"each step: {frac:.3f} of the output features of every "
                                   f"layer, full K, all token sets"},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-seconds", type=float, default=90.0)
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
