#!/usr/bin/env python3
"""Benchmark of the quantized-state decode step on B200.

One step = one decode token for every head of every request of the workload: a single
stq_decode_step over 2304 heads x 70 requests (48 layers x 48 heads of 128 x 128 states, mixed
4/6/8-bit codes with 1.4% FP16 pivot heads), reading and writing the packed state in place.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Under torchrun (N > 1) every rank runs its own 70 requests on its own GPU (weak scaling; the
(request, head) tiles are independent, so no data-path collective exists); the timed region is
bracketed by a barrier and a device synchronize, and the reported time is the max over ranks.
Rank 0 prints one JSON line. `--impl reference` times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-state head-steps/sec and achieved HBM GB/s (% roofline) at batch 70"
DEFAULT_WORKLOAD = "full2304_b70_mixed"
LIFETIME_WORKLOAD = "full2304_b70_lifetime"  # same workload, lifetime-aware widths
TOKENS_CYCLED = 8
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
DECODE_SOURCES = ("quantized_linear_attention_stq_b200/csrc/decode_d128.cu",
                  "quantized_linear_attention_stq_b200/csrc/stq_internal.cuh")
TRAFFIC_FILE = "profiles/decode_d128_full2304_b70.md"


# ------------------------------------------------------------------------------------------------
# distributed plumbing (host logic; covered by gloo tests on CPU)
# ------------------------------------------------------------------------------------------------

def dist_env():
    """(rank, world, local_rank) from the torchrun environment (1 process if absent)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def request_offset(rank: int, batch: int) -> int:
    """First request index of a rank: every rank owns its own `batch` requests."""
    return rank * batch


def reduce_max(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier(device_ids=[device.index] if device is not None and device.type == "cuda" else None)


# ------------------------------------------------------------------------------------------------
# small helpers
# ------------------------------------------------------------------------------------------------

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "of measured"
    return FALLBACK_HBM_GBS, "of fallback"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s of a kernel timed alone (the burst figure)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "of measured"
    return FALLBACK_BF16_TFLOPS, "of fallback"


# Dense contractions of one 64-token chunk of one 128 x 128 head in the UT form, as multiply-adds
# x 2: [K;Q]K^T (128 x 64 x 128), [K;Q] S0 (128 x 128 x 128), T R' and P U (64 x 128 x 64 each),
# K^T U (128 x 128 x 64). The bf16 operand splits make the tensor cores issue about four times this.
PREFILL_FLOPS_PER_CHUNK_HEAD = 2 * (128 * 64 * 128 + 128 * 128 * 128 + 2 * 64 * 128 * 64 + 128 * 128 * 64)


def decode_source_hash() -> str:
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this source."""
    path = os.path.join(ROOT, TRAFFIC_FILE)
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.strip().startswith(("traffic_bytes_per_step", "kernel_source_sha256")):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256") != decode_source_hash():
        return None
    try:
        return float(vals["traffic_bytes_per_step"])
    except (KeyError, ValueError):
        return None


def step_traffic(args):
    """The committed capture's DRAM bytes per step, for the step it was taken on (the default
    workload at its own batch, fp32 scales, the one-pass fit) and the current decode source; None
    for any other configuration."""
    if args.workload != DEFAULT_WORKLOAD or args.batch or args.scale_dtype != "f32" or args.fit_rounds != 0:
        return None
    return profiled_traffic()


# fp32 lane operations on the FMA pipe that one state element needs in this formulation of the
# decode step: code unpack 1, the k and q column sums 2, the update 2, the column energy 1, the
# column rescale 1, the rounding 1 (FP16 pivots: column sums 2, update 2)
FMA_OPS_PER_ELEMENT = {4: 8, 6: 8, 8: 8, 16: 4}
FP32_LANES_PER_SM = 128


def clocks_sm_mhz(summary) -> float:
    v = summary.get("sm_mhz") if isinstance(summary, dict) else None
    return float(v) if v else 1965.0


def alu_roofline(bits, B: int, step_s: float, sm_mhz: float) -> dict:
    """The FMA-pipe co-bound of the decode step: algorithmic fp32 lane operations per step over
    the step time, against 148 SMs x 128 fp32 lanes x the SM clock sampled during the run."""
    ops = sum(FMA_OPS_PER_ELEMENT[b] for b in bits) * 128 * 128 * B
    peak = 148 * FP32_LANES_PER_SM * sm_mhz * 1e6 / 1e12
    achieved = ops / step_s / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Tlane-op/s", "frac": achieved / peak,
            "ops_per_step": ops, "note": "fp32 lane operations on the FMA pipe; peak = 148 SMs x 128 lanes x clock"}


class ClockSampler:
    """nvidia-smi clock / throttle sampling around the timed region."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self, t0: float, t1: float):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        inside = [r for r in rows if t0 - 0.15 <= r[0] <= t1 + 0.15]
        used = inside or sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:3]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in used for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in used), "sm_max_mhz": max(r[2] for r in used),
                "reasons": reasons, "samples": len(used), "samples_inside_timed_region": len(inside)}


# ------------------------------------------------------------------------------------------------
# CPU oracle timing (the reported CPU baseline and the reference arm)
# ------------------------------------------------------------------------------------------------

def _oracle_worker(args):
    """Runs in a spawned process: decode `reps` passes over a list of tiles with the oracle."""
    tiles, reps = args
    sys.path.insert(0, ROOT)
    import oracle as orc

    orc.lib()
    blocks = [t["block"] for t in tiles]
    t0 = time.perf_counter()
    n = 0
    for _ in range(reps):
        for i, t in enumerate(tiles):
            res = orc.decode_step(t["bits"], t["gate"], blocks[i], t["q"], t["k"], t["v"], t["beta"], t["alpha"],
                                  t["w"], t["d"], t["d"])
            blocks[i] = res["block"]
            n += 1
    return n, time.perf_counter() - t0


def oracle_sample_tiles(workload_name: str, n_tiles: int, seed_offset: int = 0):
    """A bounded sample of the workload's tiles (same width mix and input distributions)."""
    import numpy as np
    import oracle as orc
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl = wlm.WORKLOADS[workload_name]
    bits_all = wlm.head_bits(wl)
    rng = np.random.default_rng(1234 + seed_offset)
    heads = rng.choice(len(bits_all), size=n_tiles, replace=False)
    # with room for it, make sure every width of the workload appears (a single-tile sample keeps
    # its random draw, so that samples over many processes follow the workload's width mix)
    widths = sorted(set(bits_all))
    if n_tiles >= len(widths):
        for slot, b in enumerate(widths):
            if not any(bits_all[h] == b for h in heads):
                heads[slot] = bits_all.index(b)
    small = wlm.scaled(wl, batch=1, heads=len(heads), outliers=wl.outliers)
    S0 = wlm.initial_state(small, 0).double().numpy()
    w_all = wlm.impact_weights(wl).double().numpy()
    inp = wlm.decode_inputs(small, 0)
    alpha = wlm.gate_values(wl).double().numpy()  # [H] or [H, d]
    tiles = []
    for i, h in enumerate(heads):
        b = int(bits_all[h])
        blk, _, _, _ = orc.quantize(b, S0[i], w_all[h])
        tiles.append(dict(bits=b, gate=wl.gate, d=wl.d, block=blk, w=w_all[h], q=inp["q"][0, i].double().numpy(),
                          k=inp["k"][0, i].double().numpy(), v=inp["v"][0, i].double().numpy(),
                          beta=float(inp["beta"][0, i]), alpha=alpha[h]))
    return tiles


# Tiles per oracle process: the bounded sample both the CPU baseline and the reference arm step.
ORACLE_TILES_PER_WORKER = 16


def time_oracle(workload_name: str, workers: int, tiles_per_worker: int, reps: int):
    """Run the oracle on `workers` spawned processes; returns (head-steps/s, cores, sample text)."""
    import multiprocessing as mp

    samples = [oracle_sample_tiles(workload_name, tiles_per_worker, seed_offset=k) for k in range(workers)]
    ctx = mp.get_context("spawn")
    with ctx.Pool(workers) as pool:
        pool.map(_oracle_worker, [(s[:1], 1) for s in samples])  # warm the workers (load + build)
        t0 = time.perf_counter()
        res = pool.map(_oracle_worker, [(s, reps) for s in samples])
        wall = time.perf_counter() - t0
    n = sum(r[0] for r in res)
    widths = sorted({t["bits"] for s in samples for t in s})
    d = samples[0][0]["d"]
    sample = (f"{n} head-steps: {workers} processes x {tiles_per_worker} sampled {d}x{d} tiles of "
              f"{workload_name} (widths {widths}) x {reps} decode steps; fp64 C oracle")
    return n / wall, workers, sample


def cpu_baseline(workload_name: str, reps: int) -> dict:
    """The oracle's rate on one core (one process) and on all host cores (one process per core,
    disjoint tile samples), over the same kind of sample."""
    rate1, _, sample1 = time_oracle(workload_name, 1, ORACLE_TILES_PER_WORKER, reps)
    workers = oracle_workers()
    rate, cores, sample = time_oracle(workload_name, workers, ORACLE_TILES_PER_WORKER, reps)
    return {"value": rate, "unit": "head-steps/s", "cores": cores, "kind": "oracle", "sample": sample,
            "single_core": {"value": rate1, "unit": "head-steps/s", "cores": 1, "sample": sample1}}


def oracle_workers():
    return max(1, min(os.cpu_count() or 1, 32))


# ------------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------------

def per_layer_graph_leg(stq, lay, pool, slots, toks, w, status, dev, steps: int, warmup: int, heads_per_layer: int = 48):
    """The serving shape of a decode token: one stq_decode_step per layer (48 heads each), all
    layers of a token captured in one CUDA graph and replayed; inputs resident in HBM."""
    import torch

    B, H, d = toks[0]["q"].shape
    L = H // heads_per_layer

    def part(x, lo):
        return x[:, lo:lo + heads_per_layer].contiguous()

    per_tok = [[{n: part(x[n], heads_per_layer * l) for n in x} for l in range(L)] for x in toks]
    w_l = [w[heads_per_layer * l:heads_per_layer * (l + 1)].contiguous() for l in range(L)]
    o_l = [torch.empty(B, heads_per_layer, d, dtype=torch.float32, device=dev) for _ in range(L)]
    graphs = []
    cap = torch.cuda.Stream(dev)
    for t in range(len(toks)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for l in range(L):
                x = per_tok[t][l]
                stq.decode_step(lay, pool, slots, x["q"], x["k"], x["v"], x["beta"], x["alpha"], w_l[l], o_l[l],
                                head_begin=heads_per_layer * l, status=status)
        graphs.append(g)
    stream = torch.cuda.current_stream(dev)
    for t in range(warmup):
        graphs[t % len(graphs)].replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for t in range(steps):
        graphs[t % len(graphs)].replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    del graphs, per_tok
    return {"layers": L, "heads_per_layer": heads_per_layer, "ms_per_token": ms,
            "head_steps_per_s": B * H / (ms / 1e3), "steps": steps,
            "note": "one stq_decode_step per layer, a token's layers captured in one CUDA graph"}


def init_dequant_leg(stq, wlm, wl, lay, w, dev, requests: int = 10, reps: int = 5) -> dict:
    """stq_init_state and stq_dequantize over `requests` requests of the workload (all heads), timed
    as whole calls with inputs resident in HBM. Algorithmic bytes: the fp32 states read (init) or
    written (dequantize) plus the packed blocks written or read."""
    import torch

    H, d = wl.heads, wl.d
    slots = torch.arange(requests, dtype=torch.int32, device=dev)
    S0 = torch.stack([wlm.initial_state(wl, r, dev) for r in range(requests)])
    out = torch.empty_like(S0)
    pool = lay.alloc_pool(requests, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    packed = requests * sum(lay.head_bytes(h) for h in range(H))
    dense = S0.numel() * 4
    res = {}
    for name, call in (("init", lambda: stq.init_state(lay, pool, slots, S0, w, status=status, stream=stream)),
                       ("dequantize", lambda: stq.dequantize(lay, pool, slots, out, status=status, stream=stream))):
        call()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            call()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / reps
        gbs = (packed + dense) / (ms / 1e3) / 1e9
        peak, kind = measured_peaks()
        res[name] = {"ms_per_call": ms, "bytes_per_call": packed + dense, "achieved_gbs": gbs, "frac": gbs / peak,
                     "peak_kind": kind}
    if status.item() != 0:
        raise RuntimeError(f"device status after the init/dequantize leg: {stq.status_flags(status)}")
    del S0, out, pool
    res["requests"] = requests
    res["kernels"] = ("init_d128_kernel (persistent, streaming; pivot heads: init_kernel) / "
                      "dequant_kernel (one CTA per tile)")
    return res


def prefill_leg(dev, steps: int = 3, warmup: int = 1, T: int = 8192, fit_rounds: int = 0) -> dict:
    """The chunked-prefill workload (16 requests x 16 heads, 6-bit, an 8192-token prompt in 64-token
    chunks, bf16 inputs) timed as whole stq_prefill_chunk calls, inputs resident in HBM."""
    import torch

    import quantized_linear_attention_stq_b200 as stq
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl = wlm.WORKLOADS["prefill16_b16_6bit"]
    B, H, d, C = wl.batch, wl.heads, wl.d, 64
    bits = wlm.head_bits(wl)
    lay = stq.Layout(bits, d, gate=wl.gate, in_dtype=wl.in_dtype, fit_rounds=fit_rounds)
    pool = lay.alloc_pool(B, dev)
    slots = torch.arange(B, dtype=torch.int32, device=dev)
    w = wlm.impact_weights(wl, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stq.init_state(lay, pool, slots, torch.stack([wlm.initial_state(wl, r, dev) for r in range(B)]), w,
                   status=status)
    inp = wlm.prefill_inputs(wl, 0, T, dev)
    o = torch.empty(B, H, T, d, dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, stq.prefill_workspace_bytes(lay, B, T, C)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call():
        stq.prefill_chunk(lay, pool, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], w, o, chunk=C,
                          workspace=ws, status=status, stream=stream)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for k in range(steps):
        call()
        ev[k + 1].record(stream)
    torch.cuda.synchronize(dev)
    if status.item() != 0:
        raise RuntimeError(f"device status after prefill: {stq.status_flags(status)}")
    ms = ev[0].elapsed_time(ev[-1]) / steps
    in_bytes = B * H * T * (3 * d * 2 + 8)  # q, k, v bf16 + beta, alpha
    out_bytes = B * H * T * d * 4             # o fp32
    state_bytes = 2 * B * sum(lay.head_bytes(h) for h in range(H))  # read at the start, written at the end
    nbytes = in_bytes + out_bytes + state_bytes
    peak, kind = measured_peaks()
    achieved = nbytes / (ms / 1e3) / 1e9
    flops = B * H * (T // C) * PREFILL_FLOPS_PER_CHUNK_HEAD
    tpeak, tkind = measured_tensor_peak()
    tflops = flops / (ms / 1e3) / 1e12
    del inp, o, pool
    return {"workload": "prefill16_b16_6bit", "prompt_tokens": T, "chunk": C, "requests": B, "heads": H,
            "ms_per_call": ms, "head_tokens_per_s": B * H * T / (ms / 1e3), "tokens_per_s": B * T / (ms / 1e3),
            "calls": steps, "fit_rounds": fit_rounds,
            "kernel": (f"ut_inputs_kernel + ut_state_kernel<6> + ut_readout_kernel per segment of up to 32 chunks "
                       f"(tcgen05, workspace of {ws.numel()} bytes)") if stq.prefill_workspace_bytes(lay, B, T, C)
                      else "prefill_wy_kernel<6> (tcgen05, one launch)" if fit_rounds <= 1 else "prefill_seq_kernel",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "peak_kind": kind, "bytes_per_call": nbytes},
            "tensor_roofline": {"bound": "tensor", "achieved": tflops, "peak": tpeak, "unit": "TFLOP/s",
                                "frac": tflops / tpeak, "peak_kind": tkind, "flops_per_call": flops,
                                "note": "algorithmic FLOPs of the five dense contractions per chunk and head"}}


L2_BYTES = 126 * 2 ** 20


def _decode_generation(stq, wlm, wl, lay, pool, slots, w, dev, steps: int, tok0: int = 0) -> dict:
    """Time `steps` decode steps of one generation on `pool` (inputs of 8 tokens cycled, resident
    in HBM): one CUDA event pair around the whole generation, launches included. Reports whether
    the state stayed finite instead of failing on the device status."""
    import torch

    B, H, d = wl.batch, wl.heads, wl.d
    toks = [wlm.decode_inputs(wl, tok0 + t, dev) for t in range(TOKENS_CYCLED)]
    o = torch.empty(B, H, d, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for t in range(steps):
        x = toks[t % TOKENS_CYCLED]
        stq.decode_step(lay, pool, slots, x["q"], x["k"], x["v"], x["beta"], x["alpha"], w, o, status=status,
                        stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    pool_bytes = B * sum(lay.head_bytes(h) for h in range(H))
    state_bytes = 2 * pool_bytes
    gbs = state_bytes / (ms / 1e3) / 1e9
    flags = stq.status_flags(status)
    return {"steps": steps, "ms_per_step": ms, "head_steps_per_s": B * H / (ms / 1e3),
            "tokens_per_s": B / (ms / 1e3), "state_bytes_per_step": state_bytes, "state_gbs": gbs,
            "gbs_kind": ("effective: the whole pool stays in the 126 MB L2" if pool_bytes <= L2_BYTES
                         else "HBM: the pool exceeds the L2"),
            "finite": "non-finite state, scale or output" not in flags, "status": flags}


def config_leg(stq, wlm, name: str, dev, fit_rounds: int = 0, steps: int = 0, warmup: int = 3) -> dict:
    """One of the workloads' own decode configurations: the workload's requests and heads, a full
    generation of its stated length (or `steps`), after `warmup` untimed steps from the same
    initial pool."""
    import torch

    wl = wlm.WORKLOADS[name]
    B, H, d = wl.batch, wl.heads, wl.d
    bits = wlm.head_bits(wl)
    lay = stq.Layout(bits, d, gate=wl.gate, in_dtype=wl.in_dtype, fit_rounds=fit_rounds)
    pool = lay.alloc_pool(B, dev)
    slots = torch.arange(B, dtype=torch.int32, device=dev)
    w = wlm.impact_weights(wl, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    stq.init_state(lay, pool, slots, torch.stack([wlm.initial_state(wl, r, dev) for r in range(B)]), w, status=st)
    pristine = pool.clone()
    _decode_generation(stq, wlm, wl, lay, pool, slots, w, dev, warmup)
    pool.copy_(pristine)
    res = _decode_generation(stq, wlm, wl, lay, pool, slots, w, dev, steps or wl.steps)
    res.update({"workload": name, "requests": B, "heads": H, "d_k": d, "d_v": d,
                "widths": {str(b): bits.count(b) for b in sorted(set(bits))}, "in_dtype": str(wl.in_dtype),
                "gate": ("scalar", "channel", "channel_decay_first")[wl.gate], "fit_rounds": fit_rounds})
    del pool, pristine
    return res


def prefill_then_decode_leg(stq, wlm, dev, decode_steps: int = 0) -> dict:
    """The prefill workload end to end: the 8192-token prompt in 64-token chunks (one
    stq_prefill_chunk call), then its stated decode generation on the same pool."""
    import torch

    wl = wlm.WORKLOADS["prefill16_b16_6bit"]
    B, H, d, T, C = wl.batch, wl.heads, wl.d, wl.prompt, wl.chunk
    bits = wlm.head_bits(wl)
    lay = stq.Layout(bits, d, gate=wl.gate, in_dtype=wl.in_dtype)
    pool = lay.alloc_pool(B, dev)
    slots = torch.arange(B, dtype=torch.int32, device=dev)
    w = wlm.impact_weights(wl, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    stq.init_state(lay, pool, slots, torch.stack([wlm.initial_state(wl, r, dev) for r in range(B)]), w, status=st)
    inp = wlm.prefill_inputs(wl, 0, T, dev)
    o = torch.empty(B, H, T, d, dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, stq.prefill_workspace_bytes(lay, B, T, C)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # one untimed call on a copy of the pool (first-call setup), then the timed call on the pool
    scratch = pool.clone()
    stq.prefill_chunk(lay, scratch, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], w, o, chunk=C,
                      workspace=ws, stream=stream)
    del scratch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    stq.prefill_chunk(lay, pool, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], w, o, chunk=C,
                      workspace=ws, status=st, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    pre_ms = e0.elapsed_time(e1)
    del inp, o, ws
    dec = _decode_generation(stq, wlm, wl, lay, pool, slots, w, dev, decode_steps or wl.steps, tok0=T)
    return {"workload": "prefill16_b16_6bit", "requests": B, "heads": H, "d_k": d, "prompt_tokens": T, "chunk": C,
            "prefill_ms": pre_ms, "prefill_tokens_per_s": B * T / (pre_ms / 1e3),
            "prefill_finite": "non-finite state, scale or output" not in stq.status_flags(st),
            "decode": dec}


def config_legs(dev, steps: int = 0, warmup: int = 3) -> dict:
    """Every configuration of the workload set besides the headline step (which the main line
    measures): the small parity case, one 48-head layer at batch 8, the channel-gate workload over
    its 2048-step generation (one-pass fit and one refit round), and prefill then decode."""
    import quantized_linear_attention_stq_b200 as stq
    from quantized_linear_attention_stq_b200 import workloads as wlm

    out = {}
    out["pr1_d16_6bit"] = config_leg(stq, wlm, "pr1_d16_6bit", dev, steps=steps, warmup=warmup)
    out["layer48_b8_4bit"] = config_leg(stq, wlm, "layer48_b8_4bit", dev, steps=steps, warmup=warmup)
    out["channel32_b128_4bit"] = config_leg(stq, wlm, "channel32_b128_4bit", dev, steps=steps, warmup=warmup)
    out["channel32_b128_4bit_fit1"] = config_leg(stq, wlm, "channel32_b128_4bit", dev, fit_rounds=1, steps=steps,
                                                 warmup=warmup)
    out["prefill16_b16_6bit"] = prefill_then_decode_leg(stq, wlm, dev, decode_steps=steps)
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    import quantized_linear_attention_stq_b200 as stq
    from quantized_linear_attention_stq_b200 import workloads as wlm

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    lifetime = args.workload == LIFETIME_WORKLOAD
    wl = wlm.WORKLOADS[DEFAULT_WORKLOAD if lifetime else args.workload]
    if args.batch:
        wl = wlm.scaled(wl, batch=args.batch)
    B, H, d = wl.batch, wl.heads, wl.d
    bits = wlm.head_bits(wl)
    if lifetime:
        # the same requests, inputs and byte budget, with widths from the lifetime-aware allocation
        # calibrated on four other requests' states
        import numpy as np

        from quantized_linear_attention_stq_b200 import calibrate

        w_cal = wlm.impact_weights(wl, dev)
        S_cal = torch.stack([wlm.initial_state(wl, 100 + r, dev) for r in range(4)])
        bits = calibrate.lifetime_widths(S_cal, w_cal, np.log(wlm.gate_values(wl).double().numpy()),
                                         stq.Layout(bits, d).bytes_per_request, bits.count(16))
        del S_cal
    scale_dtype = torch.bfloat16 if args.scale_dtype == "bf16" else torch.float32
    lay = stq.Layout(bits, d, gate=wl.gate, in_dtype=wl.in_dtype, scale_dtype=scale_dtype,
                     fit_rounds=args.fit_rounds)
    pool = lay.alloc_pool(B, dev)
    slots = torch.arange(B, dtype=torch.int32, device=dev)
    w = wlm.impact_weights(wl, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    r0 = request_offset(rank, B)
    chunk = 10
    for b0 in range(0, B, chunk):
        nb = min(chunk, B - b0)
        S0 = torch.stack([wlm.initial_state(wl, r0 + b0 + i, dev) for i in range(nb)])
        stq.init_state(lay, pool, slots[b0:b0 + nb].clone(), S0, w, status=status)
        del S0
    # realised outlier ratios of the initial states (first request, first 64 heads)
    S0s = wlm.initial_state(wl, r0, dev)[:64].double()
    row_rms = S0s.pow(2).mean(dim=2).sqrt()
    col_rms = S0s.pow(2).mean(dim=1).sqrt()
    row_ratio = float((row_rms.max(dim=1).values / row_rms.median(dim=1).values).median())
    col_ratio = float((col_rms.max(dim=1).values / col_rms.median(dim=1).values).median())
    del S0s
    toks = [wlm.decode_inputs(wl, 1000 * rank + t, dev) for t in range(TOKENS_CYCLED)]
    o = torch.empty(B, H, d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    # the workload is a generation of wl.steps tokens; longer runs restart it from the initial
    # pool (a device copy between generations, outside the per-step timings)
    pristine = pool.clone()
    gen = max(1, wl.steps)
    torch.cuda.synchronize(dev)

    def step(t):
        x = toks[t % TOKENS_CYCLED]
        stq.decode_step(lay, pool, slots, x["q"], x["k"], x["v"], x["beta"], x["alpha"], w, o, status=status,
                        stream=stream)

    for t in range(args.warmup):
        step(t)
    torch.cuda.synchronize(dev)
    if status.item() != 0:
        raise RuntimeError(f"device status after warm-up: {stq.status_flags(status)}")
    pool.copy_(pristine)

    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(dev)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    for t in range(args.steps):
        if t > 0 and t % gen == 0:
            pool.copy_(pristine, non_blocking=True)
        ev0[t].record(stream)
        step(t)
        ev1[t].record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier(dev)
    time.sleep(0.3)
    clocks.stop()
    per_step = [ev0[i].elapsed_time(ev1[i]) for i in range(args.steps)]
    total_ms = sum(per_step)
    total_ms_max = reduce_max(total_ms, dev)
    if status.item() != 0:
        raise RuntimeError(f"device status after timing: {stq.status_flags(status)}")

    graph_leg = None
    if world == 1 and H % 48 == 0 and args.workload in (DEFAULT_WORKLOAD, LIFETIME_WORKLOAD):
        pool.copy_(pristine)
        graph_leg = per_layer_graph_leg(stq, lay, pool, slots, toks, w, status, dev, min(args.steps, gen), 5)
        if status.item() != 0:
            raise RuntimeError(f"device status after the per-layer graph leg: {stq.status_flags(status)}")
    pool.copy_(pristine)
    init_leg = None
    if world == 1:
        init_leg = init_dequant_leg(stq, wlm, wl, lay, w, dev)

    # end to end through the public API with host buffers: every step copies its inputs from pinned
    # host memory and reads its readout back; copies run on their own streams (double-buffered
    # device inputs and readouts) so that step t+1's upload and step t-1's download overlap step t
    e2e_steps = max(1, min(args.steps, 50, gen))
    host_in = [{n: x.cpu().pin_memory() for n, x in toks[t].items()} for t in range(min(TOKENS_CYCLED, e2e_steps))]
    dev_in = [{n: torch.empty_like(x) for n, x in toks[0].items()} for _ in range(2)]
    dev_o = [torch.empty(B, H, d, dtype=torch.float32, device=dev) for _ in range(2)]
    host_o = [torch.empty(B, H, d, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d_bytes = sum(x.numel() * x.element_size() for x in host_in[0].values())
    d2h_bytes = host_o[0].numel() * host_o[0].element_size()
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    up_done = [torch.cuda.Event() for _ in range(2)]
    step_done = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pool.copy_(pristine)
    barrier(dev)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    s_up.wait_stream(stream)
    s_down.wait_stream(stream)
    for t in range(e2e_steps):
        k = t % 2
        src = host_in[t % len(host_in)]
        with torch.cuda.stream(s_up):
            if t >= 2:
                s_up.wait_event(step_done[k])  # step t-2 has read this input buffer
            for n in dev_in[k]:
                dev_in[k][n].copy_(src[n], non_blocking=True)
            up_done[k].record(s_up)
        stream.wait_event(up_done[k])
        if t >= 2:
            stream.wait_event(down_done[k])  # readout t-2 has left this buffer
        x = dev_in[k]
        stq.decode_step(lay, pool, slots, x["q"], x["k"], x["v"], x["beta"], x["alpha"], w, dev_o[k],
                        status=status, stream=stream)
        step_done[k].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(step_done[k])
            host_o[k].copy_(dev_o[k], non_blocking=True)
            down_done[k].record(s_down)
    stream.wait_stream(s_down)
    stream.wait_stream(s_up)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev)
    if status.item() != 0:
        raise RuntimeError(f"device status after the end-to-end leg: {stq.status_flags(status)}")

    # figures
    clocks_summary = clocks.summary(t_wall0, t_wall1)
    state_bytes = 2 * sum(lay.head_bytes(h) for h in range(H)) * B  # read + write, one launch
    io_bytes = B * H * (3 * d * (2 if wl.in_dtype == torch.bfloat16 else 4) + 4 * d + 8)
    # the d = 128 decode: one launch for the FP16 pivots, then one per width when every width has
    # at least 8192 tiles, else one for all widths; together they move `state_bytes`
    coded = [b for b in set(bits) if b != 16]
    per_width = all(bits.count(b) * B >= 8192 for b in coded)
    launches_per_step = (16 in bits) + (len(coded) if per_width else 1)
    step_s_local = total_ms / 1e3 / args.steps
    achieved = state_bytes / step_s_local / 1e9
    peak, peak_kind = measured_peaks()
    step_s = total_ms_max / 1e3 / args.steps
    head_steps = B * H * world
    result = {
        "metric": METRIC,
        "value": head_steps / step_s,
        "unit": "head-steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": args.workload, "batch_per_gpu": B, "heads": H, "d_k": d, "d_v": d,
                   "widths": {str(b): bits.count(b) for b in sorted(set(bits))}, "in_dtype": str(wl.in_dtype),
                   "gate": "scalar" if wl.gate == 0 else "channel", "tokens_cycled": TOKENS_CYCLED,
                   "scale_dtype": args.scale_dtype, "fit_rounds": args.fit_rounds,
                   "l2": "no flush: the 2.0 GB state pool read+written per step exceeds the 126 MB L2",
                   "generation_tokens": gen,
                   "timing": "CUDA events around each step; the pool restarts from its initial state every "
                             "generation_tokens steps, between steps and outside the timings",
                   "parallelism": f"dp{world} (independent requests per GPU)",
                   "s0_row_max_to_median": round(row_ratio, 2), "s0_col_max_to_median": round(col_ratio, 2)},
        "tokens_per_s": B * world / step_s,
        "state_gbs": state_bytes / step_s / 1e9,
        "state_plus_io_gbs": (state_bytes + io_bytes * launches_per_step) / step_s / 1e9,
        "step_ms_median": statistics.median(per_step),
        "step_ms_min": min(per_step),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind, "traffic": step_traffic(args),
                     "bytes_per_step": state_bytes, "launches_per_step": launches_per_step,
                     "kernel": ("decode_d128_kernel<width> (pivots, then one launch per width)" if per_width
                                else "decode_d128_kernel<width> (pivots, then one launch for all widths)"),
                     "kernel_source_sha256": decode_source_hash()},
        "e2e": {"value": head_steps / (e2e_ms / 1e3 / e2e_steps), "unit": "head-steps/s",
                "copies": "uploads and readouts on their own streams, overlapping the neighbouring steps",
                "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes, "steps": e2e_steps},
        "alu_roofline": alu_roofline(bits, B, step_s_local, clocks_sm_mhz(clocks_summary)),
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clocks_summary,
        "gpu": torch.cuda.get_device_name(dev),
    }
    if graph_leg is not None:
        result["per_layer_graph"] = graph_leg
    if init_leg is not None:
        result["init_dequantize"] = init_leg
    if lifetime:
        result["config"]["widths_from"] = "lifetime-aware allocation (stq_allocate_widths), same byte budget"
    if world == 1 and not args.no_prefill:
        result["prefill"] = prefill_leg(dev, T=args.prefill_tokens, fit_rounds=args.fit_rounds)
    if world == 1 and not args.no_configs and args.workload == DEFAULT_WORKLOAD:
        result["configs"] = config_legs(dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not lifetime:
        result["cpu_baseline"] = cpu_baseline(args.workload, 20)
    elif rank == 0:
        result["cpu_baseline"] = None
    if world > 1:
        dist.barrier(device_ids=[dev.index])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    workers = oracle_workers()
    # one step = one decode step of ORACLE_TILES_PER_WORKER sampled tiles per worker (the CPU
    # baseline's sample); all steps run back to back inside the workers
    rate, cores, sample = time_oracle(args.workload, workers, ORACLE_TILES_PER_WORKER, max(1, args.steps))
    result = {
        "metric": METRIC,
        "impl": "reference",
        "value": rate,
        "unit": "head-steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": workers * ORACLE_TILES_PER_WORKER / rate * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.workload, "note": "CPU oracle on the host cores; bounded sample per step"},
        "cpu_baseline": {"value": rate, "unit": "head-steps/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": rate, "unit": "head-steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(result), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=512)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workload configurations")
    ap.add_argument("--configs-only", action="store_true",
                    help="run only the other workload configurations (each for --steps decode steps when "
                         "given explicitly, else its own generation length; profiling)")
    ap.add_argument("--no-prefill", action="store_true", help="skip the chunked-prefill leg")
    ap.add_argument("--prefill-only", action="store_true", help="run only the chunked-prefill leg (profiling)")
    ap.add_argument("--init-only", action="store_true",
                    help="run only the init / dequantize leg, over --batch requests (default 10; profiling)")
    ap.add_argument("--prefill-tokens", type=int, default=8192, help="prompt length of the prefill leg")
    ap.add_argument("--batch", type=int, default=0, help="requests per GPU (default: the workload's)")
    ap.add_argument("--scale-dtype", choices=("f32", "bf16"), default="f32",
                    help="storage of the row and column scales (bf16: the 16-bit scale format)")
    ap.add_argument("--fit-rounds", type=int, default=0,
                    help="rounds of the impact-weighted joint scale refinement (runs on the plain kernels)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.configs_only:
        import torch

        dev = torch.device("cuda", torch.cuda.current_device())
        steps = args.steps if any(a.startswith("--steps") for a in (argv if argv is not None else sys.argv[1:])) else 0
        print(json.dumps({"configs": config_legs(dev, steps=steps, warmup=args.warmup)}), flush=True)
    elif args.prefill_only:
        import torch

        dev = torch.device("cuda", torch.cuda.current_device())
        print(json.dumps({"prefill": prefill_leg(dev, steps=args.steps, warmup=args.warmup, T=args.prefill_tokens,
                                                 fit_rounds=args.fit_rounds)}),
              flush=True)
    elif args.init_only:
        import torch

        import quantized_linear_attention_stq_b200 as stq
        from quantized_linear_attention_stq_b200 import workloads as wlm

        dev = torch.device("cuda", torch.cuda.current_device())
        wl = wlm.WORKLOADS[args.workload]
        lay = stq.Layout(wlm.head_bits(wl), wl.d, gate=wl.gate, in_dtype=wl.in_dtype,
                         scale_dtype=torch.bfloat16 if args.scale_dtype == "bf16" else torch.float32,
                         fit_rounds=args.fit_rounds)
        leg = init_dequant_leg(stq, wlm, wl, lay, wlm.impact_weights(wl, dev), dev, requests=args.batch or 10,
                               reps=args.steps)
        print(json.dumps({"init_dequantize": leg}), flush=True)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
