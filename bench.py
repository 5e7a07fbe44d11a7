#!/usr/bin/env python
"""Benchmark of the FP4 attention hot path on B200.

One step = the whole hot path on one batch of synthetic input: the quantise
prologue (smooth K + Hadamard + NVFP4 pack of Q and K) followed by the FP4
attention forward, on the 15-second-clip workload (B=1, H=48, N=109568,
d=128, non-causal).  Inputs are resident in HBM when timing starts; every
input tensor (1.35 GB each) is larger than the 126 MB L2, so no flush is
needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs its own replica
of the workload (no data-path collective; weak scaling) and the time is the
max over ranks.  ``--impl reference`` times the CPU oracle (as it stands) on
the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_precision_b200 import synth  # noqa: E402

METRIC = "FP4-attn TFLOPS @N=109k,d=128 (% composite roofline); quantize GB/s"
UNIT = "TFLOP/s"
WORKLOAD = "clip15s"
PROLOGUE_BYTES_PER_ELEMENT = 5.125  # Q,K bf16 read (2+2) + codes (0.5+0.5) + scales (1/16+1/16)
L2_BYTES = 126 * 2 ** 20  # B200 L2
# The pages' own figures for this path, with their hardware: context for the
# numbers above, not a target (the pages give no kernel-level throughput).
PAGES_CONTEXT = {
    "source": 'FastVideo "Pika H3 Flex in FastVideo", sections "TL;DR" and "FP4 attention"',
    "nvfp4_model_480p_5s_clip": {"value": 5.8, "unit": "s end to end", "hardware": "1x GB200"},
    "fp4_attention_768p_15s_clip": {"bf16_attention_s": 101.8, "fp4_attention_s": 85.3, "change": "-16%",
                                    "unit": "s end to end", "hardware": "1x GB200"},
    "fused_transform": {"value": "under 1 ms per attention call", "hardware": "GB200"},
}
# ncu DRAM bytes (read + write) per launch, keyed by the sha256 prefix of the
# kernel source they were measured on (comments and blank space removed) and
# the workload; a changed kernel reports null until it is profiled again
# (profiles/ holds the commands).  The 15-second
# clip's figures are the eight-head capture (clip15s_8heads, the same head
# length, a few GB on the device) times six: heads are independent and the
# traffic of a launch grows with their number.
ATTN_TRAFFIC_BYTES = {
    ("05cb295263156a8d", "clip15s_8heads"): 0.4297e9 + 0.2081e9,
    ("05cb295263156a8d", "clip15s"): 6 * (0.4297e9 + 0.2081e9),
}
PROLOGUE_TRAFFIC_BYTES = {
    ("403b668cf754852d", "clip15s_8heads"): 0.5990e9 + 0.0756e9,
    ("403b668cf754852d", "clip15s"): 6 * (0.5990e9 + 0.0756e9),
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def attention_flops(B, H, N, D=128):
    return 4.0 * B * H * N * N * D


def source_hash(path):
    """sha256 prefix of a kernel source with its comments and blank space
    removed: the counters stay attached to the code they were taken on, not
    to its comments."""
    with open(path, encoding="utf-8") as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = " ".join(text.split())
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sustained=d["bf16_tflops_sustained"],
                    sm_mhz=(d.get("clocks_under_load") or {}).get("sm_mhz_median"), source="measured")
    # the profiling recipe's fallback: the sustained figure settles near 1.4 PF at about 1.3 GHz
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, sm_mhz=1300.0, source="fallback")


def composite_peak(bf16_tflops):
    """Peak of a contraction doing half its FLOPs on FP4 (4x the BF16 rate,
    the nominal dense ratio) and half on BF16: 2 / (1/P_fp4 + 1/P_bf16)."""
    p4 = 4.0 * bf16_tflops
    return 2.0 / (1.0 / p4 + 1.0 / bf16_tflops)


# ---------------------------------------------------------------- clocks ----

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    QUERY = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            pass
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits", "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid if self.uuid.startswith("GPU-") else "GPU-" + self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.strip().split(", ") for r in self.file.read().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 10:
                continue
            try:
                sm.append(float(r[2]))
                mx.append(float(r[3]))
            except ValueError:
                continue
            for name, val in zip(names, r[6:10]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ distributed ----

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------- CPU baseline -----

def cpu_sample(w, target_s=12.0, max_rows=4096):
    """Time the oracle (as it stands) on one head of the workload: its prologue
    and the attention of R query rows against all N keys, R sized for about
    target_s seconds.  Returns dict with TFLOP/s of the attention sample."""
    import oracle
    d = synth.generate(w, ("q", "k", "v"), heads=[0])
    qb, kb, vb = (synth.bf16_bits(d[t]) for t in "qkv")
    t0 = time.perf_counter()
    codes = oracle.quantize_qk(qb, kb)
    t_pro = time.perf_counter() - t0
    qh = oracle.dequant(codes["q_codes"][0, 0], codes["q_scales"][0, 0])
    kh = oracle.dequant(codes["k_codes"][0, 0], codes["k_scales"][0, 0])
    rows = synth.sample_rows(w.N, 32, seed=w.seed)
    t0 = time.perf_counter()
    oracle.attention_head(qh, kh, vb[0, 0], rows=rows)
    t_probe = time.perf_counter() - t0
    R = int(min(max_rows, max(32, 32 * target_s / max(t_probe, 1e-3))))
    rows = synth.sample_rows(w.N, R, seed=w.seed)
    t0 = time.perf_counter()
    oracle.attention_head(qh, kh, vb[0, 0], rows=rows)
    t_att = time.perf_counter() - t0
    flops = 4.0 * R * w.N * 128
    return dict(value=flops / t_att / 1e12, unit=UNIT, cores=oracle.num_threads(), kind="oracle",
                sample=(f"head 0 of {w.name}: fp64 attention of {R} query rows against all {w.N} keys "
                        f"({t_att:.1f} s); oracle prologue of that head's Q and K took {t_pro:.2f} s "
                        f"({PROLOGUE_BYTES_PER_ELEMENT * w.N * 128 / t_pro / 1e9:.3f} GB/s)"),
                prologue_gbs=PROLOGUE_BYTES_PER_ELEMENT * w.N * 128 / t_pro / 1e9)


def run_reference(args, rank, world):
    """The oracle arm: each step is a bounded sample of the workload on the host cores."""
    if rank != 0:
        return
    import oracle
    w = synth.WORKLOADS[args.workload]
    d = synth.generate(w, ("q", "k", "v"), heads=[0])
    qb, kb, vb = (synth.bf16_bits(d[t]) for t in "qkv")
    codes = oracle.quantize_qk(qb, kb)
    qh = oracle.dequant(codes["q_codes"][0, 0], codes["q_scales"][0, 0])
    kh = oracle.dequant(codes["k_codes"][0, 0], codes["k_scales"][0, 0])
    R = args.ref_rows
    rows = synth.sample_rows(w.N, R, seed=w.seed)

    def step():
        c = oracle.quantize_qk(qb[:, :, :4096], kb[:, :, :4096])  # prologue on a slice of the head
        oracle.attention_head(qh, kh, vb[0, 0], rows=rows)
        return c

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    flops = 4.0 * R * w.N * 128
    value = flops / dt / 1e12
    sample = (f"per step: oracle prologue of 4096 rows of head 0 plus fp64 attention of {R} query rows of "
              f"head 0 of {w.name} against all {w.N} keys")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": 128, "causal": False,
                   "parallelism": f"replicas{world}", "l2": "inputs larger than L2"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- our arm ------

def run_ours(args, rank, world, local):
    from nvfp4_precision_b200 import fp4attn as fa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS[args.workload]
    B, H, N = w.B, w.H, w.N
    t0 = time.perf_counter()
    host = synth.generate(w)
    log(f"[rank {rank}] inputs generated in {time.perf_counter() - t0:.1f} s: {w.describe()}")
    q, k, v = (host[t].to(dev) for t in "qkv")
    out = dict(q_codes=torch.empty((B, H, N, 64), dtype=torch.uint8, device=dev),
               q_scales=torch.empty((B, H, N, 8), dtype=torch.uint8, device=dev),
               k_codes=torch.empty((B, H, N, 64), dtype=torch.uint8, device=dev),
               k_scales=torch.empty((B, H, N, 8), dtype=torch.uint8, device=dev),
               k_mean=torch.empty((B, H, 128), dtype=torch.float32, device=dev))
    o = torch.empty_like(v)
    ws = fa.new_workspace(B, H, N, dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 2  # the fused prologue, the attention

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        fa.fp4attn_quantize_qk(q, k, flags=0, out=out, workspace=ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        fa.fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v, o=o,
                           workspace=ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = fa.fp4attn_read_status(ws)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {fa.status_string(st)}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    # inputs smaller than L2 (the small workloads): write a buffer twice the L2
    # size between timed steps and time each step by its own events
    small = min(t.numel() * t.element_size() for t in (q, k, v)) < L2_BYTES
    l2_flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if small else None
    l2_note = ("inputs smaller than L2: L2 flushed between steps (a write of twice its size)" if small
               else "inputs larger than L2 (no flush needed)")
    sampler = ClockSampler(local) if not args.no_clocks else None
    barrier(world)
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.5)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        if l2_flush is not None:
            l2_flush.zero_()  # outside the step's events
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    barrier(world)
    if l2_flush is None:
        ms_step = start.elapsed_time(end) / args.steps
    else:
        ms_step = statistics.mean(e[0].elapsed_time(e[2]) for e in evs)
        del l2_flush
    ms_pro = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    ms_att = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    ms_step_max = max_over_ranks(ms_step, world, dev)
    ms_pro_max = max_over_ranks(ms_pro, world, dev)
    ms_att_max = max_over_ranks(ms_att, world, dev)
    st = fa.fp4attn_read_status(ws)
    if st != 0:
        raise RuntimeError(f"device status after timing: {fa.status_string(st)}")

    F = attention_flops(B, H, N)
    value = world * F / (ms_step_max * 1e-3) / 1e12
    peaks = measured_peaks()
    # The sustained cuBLAS figure was taken under the power cap at a lower SM
    # clock than this kernel runs at; tensor throughput scales with the SM
    # clock, so the peak is put on this run's clock (median of the samples
    # taken during the timed region).
    p_comp_measured = composite_peak(peaks["bf16_sustained"])
    clock_ratio = None
    if clocks and clocks.get("sm_mhz") and peaks.get("sm_mhz"):
        clock_ratio = clocks["sm_mhz"] / peaks["sm_mhz"]
    p_comp = p_comp_measured * (clock_ratio if clock_ratio else 1.0)
    att_tflops = F / (ms_att_max * 1e-3) / 1e12
    pro_bytes = PROLOGUE_BYTES_PER_ELEMENT * B * H * N * 128
    pro_gbs = pro_bytes / (ms_pro_max * 1e-3) / 1e9
    # ---- the BF16-QK attention on the same inputs (outside the timed step) ----
    bf16qk = None
    if not args.no_bf16qk:
        o2 = torch.empty_like(v)
        fa.fp4attn_forward_bf16qk(q, k, v, o=o2, workspace=ws, stream=stream)
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        for e in bev:
            e[0].record(stream)
            fa.fp4attn_forward_bf16qk(q, k, v, o=o2, workspace=ws, stream=stream)
            e[1].record(stream)
        torch.cuda.synchronize(dev)
        st = fa.fp4attn_read_status(ws)
        if st != 0:
            raise RuntimeError(f"device status after the BF16-QK attention: {fa.status_string(st)}")
        ms_b = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in bev), world, dev)
        tf_b = F / (ms_b * 1e-3) / 1e12
        bf16qk = {"ms": ms_b, "tflops": tf_b, "frac_bf16_sustained": tf_b / peaks["bf16_sustained"],
                  "fp4_speedup": ms_b / ms_att_max}
        del o2

    # ---- general forms (outside the timed step): the dynamic global scale and
    # the [B,N,H,128] layout a QKV projection writes ----
    general = None
    if not args.no_general:
        reps = max(2, min(args.steps, 3))
        gq = torch.empty(1, dtype=torch.float32, device=dev)
        gk = torch.empty(1, dtype=torch.float32, device=dev)

        def dyn():
            fa.fp4attn_quantize_qk(q, k, gq, gk, out=out, workspace=ws, stream=stream, dynamic_gscale=True)

        dyn()
        dev_ = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        for e in dev_:
            e[0].record(stream)
            dyn()
            e[1].record(stream)
        torch.cuda.synchronize(dev)
        ms_dyn = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in dev_), world, dev)
        qt, kt, vt = (x.transpose(1, 2).contiguous().transpose(1, 2) for x in (q, k, v))
        ot = torch.empty((B, N, H, 128), dtype=torch.bfloat16, device=dev).transpose(1, 2)

        def bnhd_step():
            fa.fp4attn_quantize_qk(qt, kt, flags=0, out=out, workspace=ws, stream=stream)
            fa.fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], vt, o=ot,
                               workspace=ws, stream=stream)

        bnhd_step()
        tev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        for e in tev:
            e[0].record(stream)
            bnhd_step()
            e[1].record(stream)
        torch.cuda.synchronize(dev)
        st = fa.fp4attn_read_status(ws)
        if st != 0:
            raise RuntimeError(f"device status after the general forms: {fa.status_string(st)}")
        ms_t = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in tev), world, dev)
        # the prologue on the heavy-tailed stress tensors of the same shape
        # (Student-t(3) values, outlier channels x50: every block scale in use)
        ws_ = synth.WORKLOADS["prologue_stress"]
        ms_stress = None
        if (ws_.B, ws_.H, ws_.N) == (B, H, N):
            hs = synth.generate(ws_, ("q", "k"))
            qs_, ks_ = hs["q"].to(dev), hs["k"].to(dev)
            fa.fp4attn_quantize_qk(qs_, ks_, flags=0, out=out, workspace=ws, stream=stream)
            sev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
            for e in sev:
                e[0].record(stream)
                fa.fp4attn_quantize_qk(qs_, ks_, flags=0, out=out, workspace=ws, stream=stream)
                e[1].record(stream)
            torch.cuda.synchronize(dev)
            st = fa.fp4attn_read_status(ws)
            if st != 0:
                raise RuntimeError(f"device status after the stress prologue: {fa.status_string(st)}")
            ms_stress = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in sev), world, dev)
            del qs_, ks_, hs
        general = {"quantize_stress_ms": ms_stress,
                   "quantize_stress_gbs": None if ms_stress is None else pro_bytes / (ms_stress * 1e-3) / 1e9,
                   "quantize_dynamic_g_ms": ms_dyn,
                   "quantize_dynamic_g_gbs": pro_bytes / (ms_dyn * 1e-3) / 1e9,
                   "bnhd_layout_step_ms": ms_t, "bnhd_layout_tflops": F / (ms_t * 1e-3) / 1e12}
        del qt, kt, vt, ot

    # ---- training-time backward (straight-through), outside the timed step:
    # this step's NVFP4 codes, O and lse, a random dO ----
    training = None
    if not args.no_train:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        fa.fp4attn_quantize_qk(q, k, flags=0, out=out, workspace=ws, stream=stream)
        fa.fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v, o=o, lse=lse,
                           workspace=ws, stream=stream)
        cq = (out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"])
        g = torch.Generator(device=dev).manual_seed(17)
        dout = torch.randn((B, H, N, 128), generator=g, device=dev).to(torch.bfloat16)
        bws = torch.empty(fa.fp4attn_backward_workspace_bytes(B, H, N), dtype=torch.uint8, device=dev)
        fa.fp4attn_backward(*cq, v, o, dout, lse, workspace=bws, stream=stream)
        reps = 2
        tev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        for e in tev:
            e[0].record(stream)
            fa.fp4attn_backward(*cq, v, o, dout, lse, workspace=bws, stream=stream)
            e[1].record(stream)
        torch.cuda.synchronize(dev)
        st = fa.fp4attn_read_status(bws)
        if st != 0:
            raise RuntimeError(f"device status after the backward: {fa.status_string(st)}")
        ms_bw = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in tev), world, dev)
        f_bw = 2.5 * F  # five N x N x d products against the forward's two
        training = {"backward_ms": ms_bw, "backward_tflops": f_bw / (ms_bw * 1e-3) / 1e12,
                    "frac_bf16_sustained": f_bw / (ms_bw * 1e-3) / 1e12 / peaks["bf16_sustained"],
                    "launches": 6}
        del dout, bws

    # ---- the tensor-core rates behind the composite roofline (context for
    # its nominal FP4:BF16 ratio of 4): block-scaled FP4 and BF16 MMAs back to
    # back on every SM, operands resident, outside the timed step ----
    rates = None
    if not args.no_rates:
        fa.fp4attn_probe_mma_rate(0, reps=4000, stream=stream)  # warm-up
        r4 = fa.fp4attn_probe_mma_rate(0, reps=40000, stream=stream)
        r16 = fa.fp4attn_probe_mma_rate(1, reps=10000, stream=stream)
        rates = {"fp4_tflops": r4["tflops"], "bf16_tflops": r16["tflops"],
                 "fp4_flop_per_clk_sm": r4["flop_per_clk_sm"], "bf16_flop_per_clk_sm": r16["flop_per_clk_sm"],
                 "fp4_to_bf16_per_clock": r4["flop_per_clk_sm"] / r16["flop_per_clk_sm"],
                 "sm_mhz": [r4["sm_mhz"], r16["sm_mhz"]],
                 "what": ("tcgen05 kind::mxf4nvf4 M128 N256 K64 and kind::f16 M128 N256 K16, back to back "
                          "on every SM, operands in shared memory and TMEM")}

    csrc = os.path.join(ROOT, "nvfp4_precision_b200", "csrc")
    traffic = ATTN_TRAFFIC_BYTES.get((source_hash(os.path.join(csrc, "attention.cu")), args.workload))
    pro_traffic = PROLOGUE_TRAFFIC_BYTES.get((source_hash(os.path.join(csrc, "prologue.cu")), args.workload))

    # ---- end to end through the public API: pinned host inputs in, O out ----
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (host[t].pin_memory() for t in "qkv")
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        step()  # the whole-tensor result the pipelined steps must reproduce
        o_ref = o.clone()
        # Pipelined over chunks of heads (heads are independent): the inputs of
        # chunk c+1 cross PCIe on one copy stream while chunk c is quantised and
        # attended, and chunk c's output goes back on a second copy stream (PCIe
        # is full duplex).  Chunks alternate between two compute streams (each
        # with its own workspace), so a chunk's kernels start on the SMs that the
        # previous chunk's last wave leaves idle.  One head per chunk (measured:
        # 12 chunks on one compute stream 219.5 ms per step, 24 on two 213.3,
        # 48 on two 212.2).
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        cstreams = (stream, torch.cuda.Stream(dev))
        wss = (ws, fa.new_workspace(B, H, N, dev))
        nchunk = H if B == 1 else 1  # head slices of a B=1 tensor are contiguous
        edges = [(H * i) // nchunk for i in range(nchunk + 1)]
        chunks = [(a, b) for a, b in zip(edges[:-1], edges[1:]) if b > a]
        ev_in = [torch.cuda.Event() for _ in chunks]
        ev_out = [torch.cuda.Event() for _ in chunks]
        code_keys = ("q_codes", "q_scales", "k_codes", "k_scales", "k_mean")

        def e2e_step():
            # the previous step no longer reads q, k, v (stream waited for all of it)
            for st_ in (h2d, d2h, cstreams[1]):
                st_.wait_stream(stream)
            with torch.cuda.stream(h2d):
                for i, (a, b) in enumerate(chunks):
                    for dst, src in ((q, hq), (k, hk), (v, hv)):
                        dst[:, a:b].copy_(src[:, a:b], non_blocking=True)
                    ev_in[i].record(h2d)
            for i, (a, b) in enumerate(chunks):
                cs, w_ = cstreams[i % 2], wss[i % 2]
                cs.wait_event(ev_in[i])
                co = {key: out[key][:, a:b] for key in code_keys}
                fa.fp4attn_quantize_qk(q[:, a:b], k[:, a:b], flags=0, out=co, workspace=w_, stream=cs)
                fa.fp4attn_forward(co["q_codes"], co["q_scales"], co["k_codes"], co["k_scales"], v[:, a:b],
                                   o=o[:, a:b], workspace=w_, stream=cs)
                ev_out[i].record(cs)
                d2h.wait_event(ev_out[i])
                with torch.cuda.stream(d2h):
                    ho[:, a:b].copy_(o[:, a:b], non_blocking=True)
            stream.wait_stream(d2h)
            stream.wait_stream(cstreams[1])

        e2e_step()
        torch.cuda.synchronize(dev)
        barrier(world)
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e2.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = max_over_ranks(s2.elapsed_time(e2) / args.e2e_steps, world, dev)
        st = max(fa.fp4attn_read_status(w_) for w_ in wss)
        if st != 0:
            raise RuntimeError(f"device status after the end-to-end steps: {fa.status_string(st)}")
        if not torch.equal(ho.to(dev), o_ref):
            raise RuntimeError("the pipelined end-to-end output differs from the whole-tensor step")
        del o_ref
        e2e = {"value": world * F / (ms_e2e * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": int(q.numel() * 2 * 3), "d2h_bytes_per_step": int(o.numel() * 2),
               "ms_per_step": ms_e2e, "pipeline": f"{len(chunks)} chunks of heads on 2 compute streams, copies overlapping compute"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_sample(w)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp4(e2m1,ue4m3)xbf16->f32", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": 128, "causal": False,
                       "parallelism": f"replicas{world}", "l2": l2_note,
                       "step": "quantize prologue + attention forward"},
            "attention": {"ms": ms_att_max, "tflops": att_tflops,
                          "frac_composite_measured_at_run_clock": att_tflops / p_comp,
                          "frac_composite_measured_sustained": att_tflops / p_comp_measured,
                          "frac_composite_nominal": att_tflops / composite_peak(2250.0)},
            "quantize": {"ms": ms_pro_max, "gbs": pro_gbs, "frac_hbm": pro_gbs / peaks["hbm_gbs"],
                         "algorithmic_bytes": pro_bytes, "dram_bytes": pro_traffic,
                         "dram_gbs": None if pro_traffic is None else pro_traffic / (ms_pro_max * 1e-3) / 1e9},
            "bf16qk_attention": bf16qk,
            "general_forms": general,
            "training_backward": training,
            "roofline": {"bound": "tensor", "achieved": att_tflops, "peak": p_comp, "unit": "TFLOP/s",
                         "frac": att_tflops / p_comp, "traffic": traffic,
                         "peak_note": (f"composite FP4/BF16 peak 2/(1/P4 + 1/P16) from the {peaks['source']} "
                                       f"sustained bf16 {peaks['bf16_sustained']} TFLOP/s at {peaks['sm_mhz']} MHz, "
                                       f"x nominal FP4:BF16 ratio 4"
                                       + (f", scaled to this run's median SM clock {clocks['sm_mhz']} MHz"
                                          if clock_ratio else ", no clock samples: unscaled"))},
            "tensor_rates": rates,
            "clocks": clocks,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "cpu_baseline": cpu,
            "pages_context": PAGES_CONTEXT,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--ref-rows", type=int, default=256)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-bf16qk", action="store_true", help="skip timing the BF16-QK attention")
    ap.add_argument("--no-train", action="store_true", help="skip timing the training-time backward")
    ap.add_argument("--no-rates", action="store_true", help="skip the tensor-core rate probe")
    ap.add_argument("--no-general", action="store_true",
                    help="skip timing the dynamic-scale prologue and the [B,N,H,128] layout")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        # the oracle arm runs on rank 0's host cores only; other ranks exit at once
        if int(os.environ.get("RANK", "0")) == 0:
            run_reference(args, 0, int(os.environ.get("WORLD_SIZE", "1")))
        return
    rank, world, local = dist_init()
    try:
        run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
