#!/usr/bin/env python
"""Benchmark of the single-GPU Ulysses attention layer (sm_100a).

One step = the whole hot path over one batch of the workload:
  seq->head(Q, K, V) -> attention forward -> head->seq(O)
  seq->head(dO) -> attention backward -> head->seq(dQ, dK, dV)
  token-weighted cross-entropy aggregated over the P shards.
Default workload: the Qwen3-4B-shaped layer at n = 65536 (B=1, P=4 logical
ranks, 32 query / 8 KV heads, head_dim 128, bf16, causal, vocab 8192).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` is whole-job tokens/s with inputs
resident in HBM (CUDA events on the launch stream, max over ranks); `e2e`
repeats the step through the same C ABI with pinned host buffers, the
host->device copies of the step's inputs and the device->host copies of its
outputs inside the timed region.  Every GPU runs an independent replica
(different seed): the path has no data-path collective, so scaling is weak.
`--impl reference` times the CPU oracle (the plain fp64 reference
implementation) on a bounded sample of the same workload.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from long_context_sequence_all_b200.workloads import WORKLOADS, make_inputs, to_natural  # noqa: E402

METRIC = "Ulysses attn layer tokens/s + TFLOP/s (frac BF16 peak); permute GB/s (frac HBM)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0   # B200 dense bf16 (data-sheet figure, without sparsity)
CLOCK_FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
                "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ----------------------------------------------------------------- workload

def causal_pairs(inp) -> float:
    """Unmasked (query, key) pairs of one head: n(n+1)/2 causal, n^2 full,
    sum over documents of L(L+1)/2 for the doc-causal mask."""
    n = inp["n"]
    if inp["mask"] == 0:
        return float(n) * n
    if inp["mask"] == 1:
        return n * (n + 1) / 2.0
    cu = inp["cu_seqlens"].tolist()
    return float(sum((b - a) * (b - a + 1) / 2.0 for a, b in zip(cu[:-1], cu[1:])))


MASK_NAMES = {0: "full (no mask)", 1: "causal", 2: "doc-causal (packed documents)"}


def workload_label(w, inp) -> str:
    """The workload in words: shapes, input dtype, mask and the passes of one step."""
    loss = f" + CE loss V={w.vocab}" if "logits" in inp else ""
    return (f"{w.name}: Qwen3-4B-shaped Ulysses attention layer, B={w.B} n={inp['n']} P={w.P} H={w.H} "
            f"G={w.G} d={w.d} bf16 {MASK_NAMES[inp['mask']]} fwd+bwd{loss}")


def algorithmic_work(inp):
    """Algorithmic flops / bytes of each kernel per launch (see the design notes)."""
    B, H, G, d, n = inp["B"], inp["H"], inp["G"], inp["d"], inp["n"]
    pairs = causal_pairs(inp)
    qb = B * n * H * d * 2
    kvb = B * n * G * d * 2
    n_pad = (n + 127) // 128 * 128
    w = {
        "attn_fwd_sm100": ("flops", 4.0 * B * H * d * pairs),
        "attn_bwd_sm100": ("flops", 10.0 * B * H * d * pairs),   # S, dP, dV, dK, dQ in one pass
        "attn_dkdv_sm100": ("flops", 8.0 * B * H * d * pairs),   # deterministic path: S, dP, dV, dK
        "attn_dq_sm100": ("flops", 2.0 * B * H * d * pairs),     # deterministic path: dQ (S, dP recomputed)
        # reads O, dO, LSE; writes D and LSE log2(e); zeroes the fp32 dQ accumulator
        "attn_bwd_stats": ("bytes", 2.0 * qb + 3 * B * n * H * 4 + B * H * n_pad * d * 4.0),
        # reads the fp32 dQ accumulator, writes dQ (bf16, seq layout)
        "attn_dq_convert": ("bytes", B * H * n * d * 4.0 + qb),
    }
    if "logits" in inp:
        valid = int((inp["labels"] != -100).sum())
        w["loss_partial"] = ("bytes", valid * inp["vocab"] * 2.0 + inp["labels"].numel() * 4)
    # permutations: one read + one write of every element, per step (the
    # head->seq direction is done by the attention kernels' epilogues)
    w["seq_to_head"] = ("bytes_step", 2.0 * (qb + 2 * kvb + qb))    # Q, K, V, dO
    w["head_to_seq"] = ("bytes_step", 2.0 * (qb + qb + 2 * kvb))    # O, dQ, dK, dV (when run separately)
    return w, pairs


# ------------------------------------------------------------- GPU ("ours")

class Layer:
    """Device buffers and one step of the layer through the C ABI."""

    def __init__(self, inp, dev):
        from long_context_sequence_all_b200 import ulysses as U
        self.U = U
        self.inp = inp
        self.P = inp["P"]
        self.mask = inp["mask"]
        f = lambda x: x.to(dev, non_blocking=False)
        self.q, self.k, self.v, self.do = (f(inp[x]) for x in ("q", "k", "v", "do"))
        self.cu = None if inp["cu_seqlens"] is None else f(inp["cu_seqlens"])
        self.logits = f(inp["logits"]) if "logits" in inp else None
        self.labels = f(inp["labels"]) if "labels" in inp else None
        P = self.P
        self.qh = U.ulysses_seq_to_head(self.q, P)
        self.kh = U.ulysses_seq_to_head(self.k, P)
        self.vh = U.ulysses_seq_to_head(self.v, P)
        self.doh = U.ulysses_seq_to_head(self.do, P)
        # the layer's outputs O, dQ, dK, dV go straight to the seq layout (the
        # second all-to-all in the attention kernels' epilogues)
        self.o, self.lse = U.ulysses_attn_fwd(self.qh, self.kh, self.vh, mask=self.mask, cu_seqlens=self.cu,
                                              out_seq_layout=True)
        desc = U._desc_from(self.qh, self.kh, self.mask, self.cu, 0.0, out_seq_layout=True)
        self.ws = torch.empty(max(256, U.ulysses_attn_bwd_workspace_size(desc)), dtype=torch.uint8, device=dev)
        self.dq, self.dk, self.dv = (torch.empty_like(x) for x in (self.q, self.k, self.v))
        if self.logits is not None:
            T, V = self.logits.shape
            self.S = torch.empty(P, dtype=torch.float32, device=dev)
            self.C = torch.empty(P, dtype=torch.int64, device=dev)
            self.L = torch.empty(1, dtype=torch.float32, device=dev)
            self.lws = torch.empty(max(256, U.ulysses_loss_workspace_size(P, T, V)), dtype=torch.uint8, device=dev)
            self.dlogits = torch.empty_like(self.logits)
            self.lbws = torch.empty(max(256, U.ulysses_loss_bwd_workspace_size(P, T, V)), dtype=torch.uint8,
                                    device=dev)

    def loss_bwd(self):
        """The loss with its gradient dL/dlogits (the step after the layer's
        loss in training; measured on its own, not part of the layer step)."""
        self.U.ulysses_loss_aggregate_bwd(self.logits, self.labels, self.P, dlogits=self.dlogits,
                                          shard_sum=self.S, shard_count=self.C, loss=self.L,
                                          workspace=self.lbws)

    def fwd_step(self):
        """The forward half alone: seq->head(Q, K, V) in one launch, attention
        forward writing O in the seq layout."""
        U, P = self.U, self.P
        U.ulysses_seq_to_head_batch([self.q, self.k, self.v], P, outs=[self.qh, self.kh, self.vh])
        U.ulysses_attn_fwd(self.qh, self.kh, self.vh, mask=self.mask, cu_seqlens=self.cu, o=self.o, lse=self.lse,
                           out_seq_layout=True)

    def step(self):
        U, P = self.U, self.P
        U.ulysses_seq_to_head_batch([self.q, self.k, self.v], P, outs=[self.qh, self.kh, self.vh])
        U.ulysses_attn_fwd(self.qh, self.kh, self.vh, mask=self.mask, cu_seqlens=self.cu, o=self.o, lse=self.lse,
                           out_seq_layout=True)
        U.ulysses_seq_to_head(self.do, P, out=self.doh)
        U.ulysses_attn_bwd(self.qh, self.kh, self.vh, self.o, self.lse, self.doh, mask=self.mask,
                           cu_seqlens=self.cu, dq=self.dq, dk=self.dk, dv=self.dv, workspace=self.ws,
                           out_seq_layout=True)
        if self.logits is not None:
            U.ulysses_loss_aggregate(self.logits, self.labels, P, shard_sum=self.S, shard_count=self.C,
                                     loss=self.L, workspace=self.lws)


class HostIO:
    """End-to-end arm: every step copies its inputs from pinned host memory to
    the device, runs the layer through the C ABI and copies its results back.
    The steps are pipelined the way a training loop prefetches its next batch:
    two device buffer sets (two layers) alternate, the host-to-device and
    device-to-host copies run on their own streams (the copy engines work
    beside the kernels), and events keep each set's inputs until the compute
    that reads them is done and its outputs until they have been copied out."""

    def __init__(self, layers):
        self.layers = layers
        L = layers[0]
        host_in = {"q": L.inp["q"], "k": L.inp["k"], "v": L.inp["v"], "do": L.inp["do"]}
        if L.logits is not None:
            host_in.update(logits=L.inp["logits"], labels=L.inp["labels"])
        self.host_in = {k: v.pin_memory() for k, v in host_in.items()}
        outs = ["o", "dq", "dk", "dv"] + (["L", "S", "C"] if L.logits is not None else [])
        self.out_names = outs
        self.host_out = {k: torch.empty(getattr(L, k).shape, dtype=getattr(L, k).dtype, pin_memory=True)
                         for k in outs}
        self.h2d = sum(h.numel() * h.element_size() for h in self.host_in.values())
        self.d2h = sum(h.numel() * h.element_size() for h in self.host_out.values())
        self.s_in, self.s_out = torch.cuda.Stream(), torch.cuda.Stream()
        n = len(layers)
        self.in_done = [torch.cuda.Event() for _ in range(n)]
        self.comp_done = [torch.cuda.Event() for _ in range(n)]
        self.out_done = [torch.cuda.Event() for _ in range(n)]
        self.used = [False] * n
        self.k = 0

    def step(self):
        b = self.k % len(self.layers)
        L = self.layers[b]
        comp = torch.cuda.current_stream()
        with torch.cuda.stream(self.s_in):
            if self.used[b]:
                self.s_in.wait_event(self.comp_done[b])      # the set's last compute read its inputs
            for name, h in self.host_in.items():
                getattr(L, name).copy_(h, non_blocking=True)
            self.in_done[b].record(self.s_in)
        comp.wait_event(self.in_done[b])
        if self.used[b]:
            comp.wait_event(self.out_done[b])                # its last outputs have left the device
        L.step()
        self.comp_done[b].record(comp)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.comp_done[b])
            for name in self.out_names:
                self.host_out[name].copy_(getattr(L, name), non_blocking=True)
            self.out_done[b].record(self.s_out)
        self.used[b] = True
        self.k += 1

    def drain(self):
        """Make the current stream wait for every copy issued so far."""
        comp = torch.cuda.current_stream()
        for b in range(len(self.layers)):
            if self.used[b]:
                comp.wait_event(self.out_done[b])


class ClockSampler:
    """nvidia-smi samples (every 200 ms) of the SM clock and throttle reasons."""

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(CLOCK_FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < len(CLOCK_FIELDS):
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kernel: str) -> str:
    files = {"attn_fwd_sm100": "attn_fwd_sm100.cu", "attn_dkdv_sm100": "attn_bwd_sm100.cu",
             "attn_bwd_sm100": "attn_bwd_fused_sm100.cu", "attn_dq_convert": "attn_bwd_fused_sm100.cu",
             "attn_dq_sm100": "attn_bwd_sm100.cu", "seq_to_head": "permute.cu", "head_to_seq": "permute.cu",
             "loss_partial": "loss.cu", "attn_bwd_stats": "attn_bwd_sm100.cu"}
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "long_context_sequence_all_b200", "csrc")
    for f in [files.get(kernel, ""), "sm100.cuh", "common.cuh"]:
        p = os.path.join(csrc, f)
        if f and os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def dram_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, or None
    when there is none or the kernel's source changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        d = json.load(open(p))
        e = d[workload][kernel]
        if e.get("source_hash") != kernel_source_hash(kernel):
            return None
        return float(e["bytes_per_launch"])
    except (OSError, KeyError, ValueError, TypeError):
        return None


def run_ours(args, rank, world, dev):
    from long_context_sequence_all_b200 import build, ulysses as U
    build.build()
    U.lib()
    w = WORKLOADS[args.workload]
    inp = make_inputs(w, seed=rank_seed(w, rank))
    work, pairs = algorithmic_work(inp)
    layer = Layer(inp, dev)
    U.ulysses_read_error()
    for _ in range(args.warmup):
        layer.step()
    torch.cuda.synchronize()
    err = U.ulysses_read_error()
    if err:
        raise RuntimeError(f"device error word {err:#x} after warm-up")

    stream = torch.cuda.current_stream()
    gpu_index = _gpu_index(dev)
    n0 = U.ulysses_launch_count()
    U.ulysses_profile_enable(True)
    with ClockSampler(gpu_index) as clk:
        _barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            layer.step()
        e1.record(stream)
        torch.cuda.synchronize()
        _barrier(world)
    prof = U.ulysses_profile_read()
    U.ulysses_profile_enable(False)
    launches = U.ulysses_launch_count() - n0
    ms = e0.elapsed_time(e1) / args.steps
    ms_max = _max_over_ranks(ms, world, dev)
    err = U.ulysses_read_error()
    if err:
        raise RuntimeError(f"device error word {err:#x} in the timed region")

    # end to end through the same C ABI with pinned host buffers (two
    # alternating device buffer sets; every step's copies are in the timed region)
    io = HostIO([layer, Layer(inp, dev)])
    for _ in range(2):
        io.step()
    io.drain()
    torch.cuda.synchronize()
    _barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    io.s_in.wait_event(e0)
    for _ in range(args.steps):
        io.step()
    io.drain()
    e1.record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)

    # the forward half alone (seq->head(Q,K,V), attention forward, head->seq(O)),
    # this rank's device time; a failure here only records the error
    fwd_only = None
    try:
        for _ in range(2):
            layer.fwd_step()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            layer.fwd_step()
        e1.record(stream)
        torch.cuda.synchronize()
        fms = e0.elapsed_time(e1) / args.steps
        fwd_only = {"ms_per_step": fms, "tokens_per_s": inp["B"] * inp["n"] / (fms / 1e3),
                    "note": "seq->head(Q,K,V) + attention forward + head->seq(O); this rank alone"}
    except Exception as exc:  # noqa: BLE001 -- a side figure never breaks the bench line
        fwd_only = {"error": str(exc)[:200]}

    # the deterministic (atomic-free, two-pass) backward on the same inputs, for
    # comparison with the fused pass the step uses
    det_bwd = None
    try:
        def det():
            U.ulysses_attn_bwd(layer.qh, layer.kh, layer.vh, layer.o, layer.lse, layer.doh, mask=layer.mask,
                               cu_seqlens=layer.cu, dq=layer.dq, dk=layer.dk, dv=layer.dv, workspace=layer.ws,
                               out_seq_layout=True, deterministic=True)
        det()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            det()
        e1.record(stream)
        torch.cuda.synchronize()
        dms = e0.elapsed_time(e1) / args.steps
        det_bwd = {"ms_per_call": dms,
                   "tflops": 10.0 * inp["B"] * inp["H"] * inp["d"] * pairs / (dms / 1e3) / 1e12,
                   "note": "statistics + dK/dV pass + dQ pass (S and dP formed twice), bitwise repeatable"}
    except Exception as exc:  # noqa: BLE001 -- a side figure never breaks the bench line
        det_bwd = {"error": str(exc)[:200]}

    # the fused loss + gradient, timed on its own (it follows the layer's loss
    # in training and is not part of the layer step)
    loss_bwd = None
    if layer.logits is not None:
        layer.loss_bwd()
        torch.cuda.synchronize()
        U.ulysses_profile_enable(True)
        for _ in range(args.steps):
            layer.loss_bwd()
        torch.cuda.synchronize()
        lprof = U.ulysses_profile_read()
        U.ulysses_profile_enable(False)
        if "loss_fwd_bwd" in lprof:
            tot, cnt = lprof["loss_fwd_bwd"]
            T, V = layer.logits.shape
            nbytes = 2.0 * T * V * layer.logits.element_size() + 2.0 * T * 4
            loss_bwd = {"ms_per_launch": tot / cnt, "gbs": nbytes / (tot / cnt / 1e3) / 1e9,
                        "note": "logits read once, dlogits written once; timed outside the layer step"}
        if U.ulysses_read_error():
            raise RuntimeError("device error word set by the loss gradient")

    tokens = inp["B"] * inp["n"]
    value = job_throughput(tokens, world, ms_max)
    peaks, peak_src = load_peaks()
    side = side_kernels(inp, dev, args.steps, peaks)
    kernels = {}
    for name, (tot_ms, cnt) in prof.items():
        per_launch = tot_ms / cnt
        k = {"launches_per_step": cnt / args.steps, "ms_per_launch": per_launch,
             "ms_per_step": tot_ms / args.steps}
        if name in work:
            kind, amount = work[name]
            if kind == "flops":
                k["tflops"] = amount / (per_launch / 1e3) / 1e12
                k["frac_bf16_sustained"] = k["tflops"] / peaks["bf16_tflops_sustained"]
                k["frac_bf16_burst"] = k["tflops"] / peaks["bf16_tflops"]
                k["frac_bf16_nominal"] = k["tflops"] / NOMINAL_BF16_TFLOPS
            elif kind == "bytes":
                k["gbs"] = amount / (per_launch / 1e3) / 1e9
                k["frac_hbm"] = k["gbs"] / peaks["hbm_gbs"]
            else:  # bytes per step over all launches of the kernel
                k["gbs"] = amount / (tot_ms / args.steps / 1e3) / 1e9
                k["frac_hbm"] = k["gbs"] / peaks["hbm_gbs"]
        kernels[name] = k
    if loss_bwd is not None:
        loss_bwd["frac_hbm"] = loss_bwd["gbs"] / peaks["hbm_gbs"]
    dominant = max(kernels, key=lambda n: kernels[n]["ms_per_step"])
    dk = kernels[dominant]
    kind, amount = work.get(dominant, ("flops", float("nan")))
    if kind == "flops":
        # the peak for a kernel timed inside a long step is the sustained GEMM
        # rate; the burst and nominal fractions are given beside it, labelled
        roof = {"kernel": dominant, "bound": "tensor", "achieved": dk["tflops"],
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                "frac": dk["tflops"] / peaks["bf16_tflops_sustained"],
                "frac_of_burst": {"peak": peaks["bf16_tflops"], "frac": dk["tflops"] / peaks["bf16_tflops"]},
                "frac_of_nominal": {"peak": NOMINAL_BF16_TFLOPS, "frac": dk["tflops"] / NOMINAL_BF16_TFLOPS}}
    else:
        roof = {"kernel": dominant, "bound": "hbm", "achieved": dk["gbs"], "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": dk["gbs"] / peaks["hbm_gbs"]}
    roof["peak_source"] = f"{peak_src} ({'bf16_tflops_sustained' if kind == 'flops' else 'hbm_gbs'})"
    roof["traffic"] = dram_traffic(dominant, args.workload)
    attn_ms = sum(kernels[k]["ms_per_step"] for k in kernels if k.startswith("attn_"))
    fwd_fl = 4.0 * inp["B"] * inp["H"] * inp["d"] * pairs
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1)/sqrt(128) Q/K/V, N(0,1) dO and logits, uniform labels)",
        "config": {"workload": workload_label(w, inp),
                   "global_batch": inp["B"] * world, "seq_len": inp["n"],
                   "parallelism": f"P={w.P} logical Ulysses ranks per GPU; {world} independent replica(s)",
                   "l2": _l2_note(inp)},
        "attn_tflops": (fwd_fl * 3.5) / (attn_ms / 1e3) / 1e12,
        "attn_fwd_tflops": kernels.get("attn_fwd_sm100", {}).get("tflops"),
        "attn_bwd_tflops": (10.0 * inp["B"] * inp["H"] * inp["d"] * pairs) /
                           (sum(kernels[k]["ms_per_step"] for k in ("attn_bwd_sm100", "attn_dkdv_sm100",
                                                                   "attn_dq_sm100", "attn_bwd_stats",
                                                                   "attn_dq_convert") if k in kernels) / 1e3) / 1e12,
        "permute_gbs": {"seq_to_head": kernels.get("seq_to_head", {}).get("gbs"),
                        "head_to_seq": side.get("head_to_seq", {}).get("gbs")},
        "roofline": roof,
        "kernels": kernels,
        "forward_only": fwd_only,
        "deterministic_backward": det_bwd,
        "loss_grad": loss_bwd,
        "side_kernels": side,
        "gpu_launches": launches,
        "e2e": {"value": job_throughput(tokens, world, e2e_ms), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": io.h2d, "d2h_bytes_per_step": io.d2h},
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inp, budget_s=args.cpu_budget)
    return line


def side_kernels(inp, dev, steps: int, peaks) -> dict:
    """Kernels outside the layer step, each timed on its own at the workload's
    sizes (CUDA events on the launching stream, via the library's profiler):
    the KV-head copies used when there are fewer KV heads than ranks (this K
    split over 2G ranks, so every KV head goes to two ranks, and the summing
    reverse of its gradient), and the label shift before sharding."""
    from long_context_sequence_all_b200 import ulysses as U
    B, n, G, d = inp["B"], inp["n"], inp["G"], inp["d"]
    eb = inp["k"].element_size()
    out = {}

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        U.ulysses_profile_enable(True)
        for _ in range(steps):
            fn()
        torch.cuda.synchronize()
        prof = U.ulysses_profile_read()
        U.ulysses_profile_enable(False)
        if U.ulysses_read_error():
            raise RuntimeError("device error word set by a side kernel")
        return prof

    def entry(prof, name, nbytes, note):
        tot, cnt = prof[name]
        gbs = nbytes / (tot / cnt / 1e3) / 1e9
        return {"ms_per_launch": tot / cnt, "gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                "bytes_per_launch": nbytes, "note": note}

    # the second all-to-all as its own kernel (the layer step folds it into the
    # attention epilogues): O-sized head layout -> seq layout
    P = inp["P"]
    q_dev = inp["q"].to(dev)
    qh = U.ulysses_seq_to_head(q_dev, P)
    back = torch.empty_like(q_dev)
    prof = timed(lambda: U.ulysses_head_to_seq(qh, P, out=back))
    qbytes = q_dev.numel() * q_dev.element_size()
    out["head_to_seq"] = entry(prof, "head_to_seq", 2.0 * qbytes,
                               "O-sized tensor, head layout -> seq layout (one read, one write)")
    if not torch.equal(back, q_dev):
        raise RuntimeError("head_to_seq(seq_to_head(Q)) != Q")
    del q_dev, qh, back
    P2 = 2 * G
    if n % P2 == 0:
        k2 = to_natural(inp["k"]).reshape(B, P2, n // P2, G, d).transpose(0, 1).contiguous().to(dev)
        rep = torch.empty((P2, B, 1, n, d), dtype=k2.dtype, device=dev)
        back = torch.empty_like(k2)
        prof = timed(lambda: (U.ulysses_kv_seq_to_head_replicated(k2, P2, out=rep),
                              U.ulysses_kv_head_to_seq_reduce(rep, P2, G, out=back)))
        small, big = B * n * G * d * eb, B * n * P2 * d * eb
        note = f"K of this workload over P={P2} ranks (G={G}: two copies per KV head)"
        out["kv_seq_to_head_rep"] = entry(prof, "kv_seq_to_head_rep", small + big, note)
        out["kv_head_to_seq_sum"] = entry(prof, "kv_head_to_seq_sum", big + small, note)
        del k2, rep, back
    # the projections either side of the attention (synthetic weights of the
    # Qwen3-4B shapes: hidden 2560), each a tcgen05 GEMM with an all-to-all
    # folded in; timed alone, so against the burst bf16 peak
    P, H, hidden = inp["P"], inp["H"], 2560
    if G % P == 0:
        x = torch.randn((P, B, n // P, hidden), device=dev).to(torch.bfloat16)
        w = (torch.randn(((H + 2 * G) * d, hidden), device=dev) / hidden ** 0.5).to(torch.bfloat16)
        tab = U.ulysses_rope_table(n, d, 1.0e6, device=dev)
        qb = torch.empty((P, B, H // P, n, d), dtype=torch.bfloat16, device=dev)
        kb = torch.empty((P, B, G // P, n, d), dtype=torch.bfloat16, device=dev)
        vb = torch.empty_like(kb)
        prof = timed(lambda: U.ulysses_qkv_proj_rope(x, w, P, H, G, tab, q=qb, k=kb, v=vb))
        wo = (torch.randn((hidden, H * d), device=dev) / (H * d) ** 0.5).to(torch.bfloat16)
        yb = torch.empty((P, B, n // P, hidden), dtype=torch.bfloat16, device=dev)
        prof2 = timed(lambda: U.ulysses_o_proj(qb, wo, P, y=yb))
        # the projections' backward (synthetic output gradients)
        dx = torch.empty_like(x)
        dwq = torch.empty(w.shape, dtype=torch.float32, device=dev)
        ws = torch.empty(B * n * (H + 2 * G) * d * 2 + 256, dtype=torch.uint8, device=dev)
        prof3 = timed(lambda: U.ulysses_qkv_proj_rope_bwd(x, w, P, H, G, tab, qb, kb, vb, dx=dx, dw=dwq, workspace=ws))
        o_seq = torch.randn((P, B, n // P, H, d), device=dev).to(torch.bfloat16)
        dyo = torch.randn((P, B, n // P, hidden), device=dev).to(torch.bfloat16)
        do_h = torch.empty_like(qb)
        dwo = torch.empty(wo.shape, dtype=torch.float32, device=dev)
        prof4 = timed(lambda: U.ulysses_o_proj_bwd(o_seq, wo, dyo, P, do=do_h, dw_o=dwo))
        fq, fo = 2.0 * B * n * (H + 2 * G) * d * hidden, 2.0 * B * n * hidden * H * d
        for name, pr, fl, note in (
                ("qkv_proj_sm100", prof, fq,
                 f"[Q K V] = X W^T, rotary positions, written in the head layout; hidden={hidden}"),
                ("o_proj_sm100", prof2, fo,
                 f"Y = O W_o^T read from the head layout, written in the seq layout; hidden={hidden}"),
                ("qkv_proj_dx_sm100", prof3, fq, "dX = dY W (dY: head layout back to tokens, rotated by -pos)"),
                ("qkv_proj_dw_sm100", prof3, fq, "dW = dY^T X over all tokens, fp32"),
                ("o_proj_do_sm100", prof4, fo, "dO = dY W_o, written in the head layout"),
                ("o_proj_dw_sm100", prof4, fo, "dW_o = dY^T O over all tokens, fp32")):
            tot, cnt = pr[name]
            tf = fl / (tot / cnt / 1e3) / 1e12
            out[name] = {"ms_per_launch": tot / cnt, "tflops": tf, "frac_bf16": tf / peaks["bf16_tflops"],
                         "flops_per_launch": fl, "note": note}
        tot, cnt = prof3["qkv_dy"]
        dyb = B * n * (H + 2 * G) * d * 2.0 * 2
        out["qkv_dy"] = {"ms_per_launch": tot / cnt, "gbs": dyb / (tot / cnt / 1e3) / 1e9,
                         "frac_hbm": dyb / (tot / cnt / 1e3) / 1e9 / peaks["hbm_gbs"],
                         "note": "dQ, dK, dV read from the head layout, dY written in token order (rotated)"}
        del x, w, tab, qb, kb, vb, wo, yb, dx, dwq, ws, o_seq, dyo, do_h, dwo
    ids = torch.randint(0, 151936, (B, n), dtype=torch.int32, device=dev)
    lab = torch.empty((inp["P"], B, n // inp["P"]), dtype=torch.int32, device=dev)
    cu = inp["cu_seqlens"].to(dev) if inp["cu_seqlens"] is not None else None
    prof = timed(lambda: U.ulysses_shift_labels(ids, inp["P"], cu_seqlens=cu, valid_len=inp["real_tokens"],
                                                out=lab))
    out["shift_labels"] = entry(prof, "shift_labels", 2.0 * B * n * 4,
                                "int32 ids read once, labels written once")
    return out


def _l2_note(inp):
    qmib = inp["q"].numel() * inp["q"].element_size() / 2 ** 20
    if qmib * 2 ** 20 > 126e6:
        return f"no flush needed: the inputs (Q alone {qmib:.0f} MiB) exceed the 126 MB L2"
    return f"no flush: inputs (Q {qmib:.0f} MiB) smaller than L2; numbers include L2 reuse across steps"


def _gpu_index(dev):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    idx = dev.index or 0
    if vis:
        parts = [p for p in vis.split(",") if p.strip()]
        if idx < len(parts) and parts[idx].strip().isdigit():
            return int(parts[idx])
    return idx


def _barrier(world):
    if world > 1:
        torch.distributed.barrier()


def _max_over_ranks(x, world, dev):
    """Largest value of x over the ranks (the job is as slow as its slowest
    replica).  dev: the device the collective's tensor lives on (cuda for
    NCCL, cpu for gloo)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(w, rank: int) -> int:
    """Seed of the replica on `rank`: every GPU draws its own batch."""
    return 1000 + w.index + 7919 * rank


def job_throughput(tokens_per_replica: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: every replica processes its own batch, the job
    takes as long as the slowest one."""
    return world * tokens_per_replica / (ms_max / 1e3)


# ------------------------------------------------------ CPU oracle timings

def cpu_step_sample(inp, rows_per_head: int, token_frac: float):
    """Time the oracle on a bounded sample of one step and extrapolate to the
    whole step: `rows_per_head` uniformly spaced query rows of every head
    (forward, dQ and their dK/dV terms: all the attention work of those rows)
    and a `token_frac` fraction of the tokens for the two all-to-alls and the
    loss.  Returns (extrapolated seconds for the full step, seconds the
    sample took, description)."""
    import oracle
    P, B, n, H, G, d = inp["P"], inp["B"], inp["n"], inp["H"], inp["G"], inp["d"]
    group = H // G
    f32 = lambda t: t.to(torch.float32).numpy()
    spent = 0.0
    # all-to-alls on a token subset (same P and heads), both directions
    s_sub = max(1, int(round(n // P * token_frac)))
    frac_perm = s_sub / (n // P)
    t_perm = 0.0
    for x, heads in ((inp["q"], H), (inp["k"], G), (inp["v"], G), (inp["do"], H)):
        sub = np.ascontiguousarray(x[:, :, :s_sub].contiguous().view(torch.int16).numpy())
        t0 = time.perf_counter()
        h = oracle.seq_to_head(sub, B, s_sub * P, P, heads)
        oracle.head_to_seq(h, B, s_sub * P, P, heads)           # O, dQ, dK, dV come back
        t_perm += time.perf_counter() - t0
    spent += t_perm
    t_perm /= frac_perm
    # loss on a token subset
    t_loss = 0.0
    if "logits" in inp:
        T = inp["logits"].shape[0]
        tsub = max(P, int(round(T * token_frac)) // P * P)
        z = f32(inp["logits"][:tsub])
        y = inp["labels"][:tsub].numpy()
        t0 = time.perf_counter()
        oracle.loss_aggregate(z, y, P)
        dt = time.perf_counter() - t0
        spent += dt
        t_loss = dt * T / tsub
    # attention: uniformly spaced rows of every head
    qn, kn, vn, don = (to_natural(inp[x])[0] for x in ("q", "k", "v", "do"))
    rows = np.unique(np.linspace(0, n - 1, rows_per_head).astype(np.int32))
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy()
    t_attn = 0.0
    for g in range(G):
        kg, vg = f32(kn[:, g].contiguous()), f32(vn[:, g].contiguous())
        dk = np.zeros((n, d)); dv = np.zeros((n, d))
        for h in range(g * group, (g + 1) * group):
            qg, dg = f32(qn[:, h].contiguous()), f32(don[:, h].contiguous())
            t0 = time.perf_counter()
            oracle.head_rows_step(qg, kg, vg, dg, rows, mask=inp["mask"], cu_seqlens=cu, dk=dk, dv=dv)
            t_attn += time.perf_counter() - t0
    spent += t_attn
    desc = (f"{rows.size} uniformly spaced query rows of each of the {H} heads (forward, dQ and their "
            f"dK/dV terms: {rows.size}/{n} of the attention work) and {token_frac:.4g} of the tokens for "
            f"the all-to-alls and the loss, each extrapolated linearly to the full step; "
            f"the sample took {spent:.1f} s")
    return t_perm + t_loss + t_attn * n / rows.size, spent, desc


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def _rows_for(inp, budget_s, token_frac):
    """Rows per head so that one sample takes about budget_s seconds."""
    _, spent, _ = cpu_step_sample(inp, rows_per_head=2, token_frac=token_frac)
    return int(max(2, min(1024, 2 * budget_s / max(1e-6, spent))))


def cpu_baseline(inp, budget_s: float = 20.0):
    rows = _rows_for(inp, budget_s, token_frac=1 / 64)
    t_full, spent, desc = cpu_step_sample(inp, rows_per_head=rows, token_frac=1 / 64)
    tokens = inp["B"] * inp["n"]
    return {"value": tokens / t_full, "unit": "tokens/s", "cores": _cores(), "kind": "oracle",
            "sample": desc, "step_s_extrapolated": t_full}


def run_reference(args, rank, world):
    """The CPU oracle, as it stands, on this machine's host cores: every step is a
    bounded sample of the workload, extrapolated to the whole step."""
    if rank != 0:
        return None
    w = WORKLOADS[args.workload]
    inp = make_inputs(w)
    per_step = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    rows = _rows_for(inp, per_step, token_frac=1 / 256)
    for _ in range(args.warmup):
        cpu_step_sample(inp, rows_per_head=rows, token_frac=1 / 256)
    ts, desc = [], ""
    for _ in range(args.steps):
        t, _, desc = cpu_step_sample(inp, rows_per_head=rows, token_frac=1 / 256)
        ts.append(t)
    step_s = statistics.median(ts)
    tokens = inp["B"] * inp["n"]
    value = tokens / step_s
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded inputs as the GPU arm)",
        "config": {"workload": workload_label(w, inp),
                   "global_batch": inp["B"], "seq_len": inp["n"], "parallelism": "CPU oracle (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": _cores(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------- main

KERNEL_ONLY = ("attn_fwd", "attn_bwd", "attn_bwd_deterministic", "seq_to_head", "head_to_seq", "loss", "loss_bwd")


def run_kernel_only(args, dev):
    """One entry point of the layer, alone, `steps` times on the workload's
    operands (no other kernel of the step runs), for profiling a single kernel
    with few launches before it; prints its CUDA-event time per call.  Not a
    bench line."""
    from long_context_sequence_all_b200 import build, ulysses as U
    build.build()
    w = WORKLOADS[args.workload]
    inp = make_inputs(w, seed=rank_seed(w, 0))
    layer = Layer(inp, dev)
    P, U_ = layer.P, U
    calls = {
        "attn_fwd": lambda: U_.ulysses_attn_fwd(layer.qh, layer.kh, layer.vh, mask=layer.mask, cu_seqlens=layer.cu,
                                                o=layer.o, lse=layer.lse, out_seq_layout=True),
        "attn_bwd": lambda: U_.ulysses_attn_bwd(layer.qh, layer.kh, layer.vh, layer.o, layer.lse, layer.doh,
                                                mask=layer.mask, cu_seqlens=layer.cu, dq=layer.dq, dk=layer.dk,
                                                dv=layer.dv, workspace=layer.ws, out_seq_layout=True),
        "attn_bwd_deterministic": lambda: U_.ulysses_attn_bwd(
            layer.qh, layer.kh, layer.vh, layer.o, layer.lse, layer.doh, mask=layer.mask, cu_seqlens=layer.cu,
            dq=layer.dq, dk=layer.dk, dv=layer.dv, workspace=layer.ws, out_seq_layout=True, deterministic=True),
        "seq_to_head": lambda: U_.ulysses_seq_to_head_batch([layer.q, layer.k, layer.v], P,
                                                            outs=[layer.qh, layer.kh, layer.vh]),
        "head_to_seq": lambda: U_.ulysses_head_to_seq_batch([layer.qh, layer.kh, layer.vh], P,
                                                            outs=[layer.q, layer.k, layer.v]),
        "loss": lambda: U_.ulysses_loss_aggregate(layer.logits, layer.labels, P, shard_sum=layer.S,
                                                  shard_count=layer.C, loss=layer.L, workspace=layer.lws),
        "loss_bwd": layer.loss_bwd,
    }
    fn = calls[args.kernel_only]
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    e0.record(stream)
    for _ in range(args.steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    if U.ulysses_read_error():
        raise RuntimeError("device error word set")
    print(json.dumps({"kernel_only": args.kernel_only, "workload": args.workload, "calls": args.steps,
                      "ms_per_call": e0.elapsed_time(e1) / args.steps}), flush=True)


def _free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_command(gpus: int, argv) -> list:
    """The command that runs this benchmark as `gpus` ranks, one per GPU of
    this node (torch.distributed.run on 127.0.0.1), under a hard time limit."""
    return ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1", f"--master-port={_free_port()}",
            os.path.abspath(__file__), *argv]


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen64k", choices=sorted(k for k in WORKLOADS if k != "tiny_f32"))
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-only", choices=KERNEL_ONLY, default=None,
                    help="run one entry point alone (for profiling); prints its time per call, not a bench line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "ours" and args.gpus != world:
        if world == 1 and args.gpus > 1 and "LOCAL_RANK" not in os.environ:
            # started directly with --gpus N: run the same command as N ranks
            raise SystemExit(subprocess.call(launch_command(args.gpus, sys.argv[1:])))
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.kernel_only:
        run_kernel_only(args, dev)
        return
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=dev)
    try:
        line = run_ours(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
