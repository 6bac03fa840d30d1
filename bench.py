#!/usr/bin/env python
"""Benchmark: jagged HSTU attention forward + backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload fixed8192|zipf|long|tiny] [--cp-C 2 4 8] [--no-cp] [--no-e2e]
                    [--no-norm-gate]

One step = one pass of the attention hot path over one synthetic jagged
batch (by default the fixed-length workload: 16 sequences of 8192 tokens as
jagged offsets, 8 heads of 64, the largest single-GPU forward+backward
configuration): the forward kernel (tile lookup on the device offsets, S = Q K^T,
bias gather, SiLU, mask, P V) and the backward kernel (dQ, dK, dV, dw_pos,
dw_ts).  Inputs are resident in HBM when the timed region starts; the L2 is
flushed (a 256 MiB write) before every timed step, outside the step's CUDA
events.  The load-balanced mini-chunk pairing path (reorder q/k/v/ts,
attention on the paired buffers, restore) is measured separately on the
paired workload for C = 2, 4 and 8 and reported under "cp_path"; the target-aware forward
(M-FALCON ranking: a user history followed by a microbatch of candidates that
attend the history and themselves only) on its ranking workload under
"targets_path"; the post-attention norm gate (y = LayerNorm(O) * U and its
backward) on the headline workload's output shape under "norm_gate_path", and
Stochastic Length (selection at alpha = 1.6 and the row gather of q, k, v and
timestamps) on the headline batch under "stochastic_length_path".

With N > 1 (torchrun) every rank runs its own batch of the same recipe
(seed offset by the rank): weak scaling with no data-path collective; the
timed region is bracketed by barriers and the slowest rank's time is used.

--impl reference times the fp64 CPU oracle (the reference for this build) on
a bounded sample of the same workload on the host cores, rank 0 only.
"""
from __future__ import annotations

import argparse
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

import workloads  # noqa: E402

METRIC = "jagged HSTU attn fwd+bwd effective TFLOP/s & tokens/s, % bf16 tensor peak (1 B200)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DESCRIPTIONS = {
    "tiny": "B=4, L~U{16..128}, H=2, d=32, Exp(3600 s) gaps, P=256, NB=128, seed 0",
    "zipf": "B=32, L=clip(Zipf(1.2),256,3072), H=4, d=128, Exp(600 s) gaps, P=3072, NB=128",
    "fixed8192": "B=16, L=8192 as jagged offsets, H=8, d=64, Exp(60 s) gaps, P=3072, NB=128",
    "long": "B=8, L~U{4096..16384}, H=4, d=128, LogNormal(6,2) s gaps, P=3072, NB=128",
}
SEEDS = {"tiny": 0, "zipf": 1, "fixed8192": 2, "long": 3}


KERNEL_SOURCES = {
    "hstu_bwd_kernel": "attn_bwd.cu",
    "hstu_fwd_kernel": "attn_fwd.cu",
    "cp_permute_kernel": "cp_reorder.cu",
    "norm_gate_fwd_kernel": "norm_gate.cu",
    "norm_gate_bwd_kernel": "norm_gate.cu",
}


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch (read + write) from the committed ncu record in
    profiles/dram_traffic.txt, or None when there is no record for this
    kernel and workload or the kernel's sources changed since the capture."""
    import hashlib
    try:
        lines = open(os.path.join(ROOT, "profiles", "dram_traffic.txt")).read().splitlines()
    except OSError:
        return None
    csrc = os.path.join(ROOT, "jagged_hstu_attention_attn_b200", "csrc")
    m = hashlib.sha256()
    try:
        for f in (KERNEL_SOURCES[kernel], "common.cuh", "internal.h"):
            with open(os.path.join(csrc, f), "rb") as fh:
                m.update(fh.read())
    except (KeyError, OSError):
        return None
    digest = m.hexdigest()[:16]
    for line in lines:
        parts = line.split()
        if not parts or parts[0].startswith("#") or len(parts) < 5:
            continue
        if parts[0] == kernel and parts[1] == workload and parts[2] == digest:
            return int(parts[3]) + int(parts[4])
    return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def make_workload(name, rank=0, with_dout=True):
    fn = workloads.WORKLOADS[name]
    return fn(seed=SEEDS[name] + 1000 * rank, with_dout=with_dout)


def max_over_ranks(values, device=None):
    """Element-wise maximum over all ranks (torch.distributed initialised)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def weak_scaling_rate(world, steps, units_per_step, max_total_ms):
    """Whole-job throughput: units every rank processed / the slowest rank's time."""
    return world * steps * units_per_step / (max_total_ms * 1e-3)


def flops_fwd(batch):
    return 4.0 * batch.d * batch.num_heads * batch.causal_pairs()


def flops_bwd(batch):
    return 10.0 * batch.d * batch.num_heads * batch.causal_pairs()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        # the raw samples (the JSON line carries their summary)
        out_dir = os.environ.get("HSTU_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_dev{device_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["sampler unavailable"],
                    "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower() in ("active", "1"):
                        reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# the native (CUDA) arm
# ---------------------------------------------------------------------------

def run_native(args):
    import torch
    import torch.distributed as dist
    import jagged_hstu_attention_attn_b200 as hstu

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()

    batch = make_workload(args.workload, rank)
    B, T, H, D = batch.B, batch.T, batch.num_heads, batch.d
    max_len = int(batch.lengths.max())
    as_bf16 = lambda bits: torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    host = {
        "q": as_bf16(batch.q).pin_memory(), "k": as_bf16(batch.k).pin_memory(),
        "v": as_bf16(batch.v).pin_memory(), "dout": as_bf16(batch.dout).pin_memory(),
        "offsets": torch.from_numpy(batch.offsets.copy()).pin_memory(),
        "ts": torch.from_numpy(batch.timestamps.copy()).pin_memory(),
        "w_pos": torch.from_numpy(batch.w_pos.copy()).pin_memory(),
        "w_ts": torch.from_numpy(batch.w_ts.copy()).pin_memory(),
    }
    d = {k_: v_.to(dev, non_blocking=False) for k_, v_ in host.items()}
    out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    dq = torch.empty_like(d["q"]); dk = torch.empty_like(d["k"]); dv = torch.empty_like(d["v"])
    dwp = torch.empty_like(d["w_pos"]); dwt = torch.empty_like(d["w_ts"])
    ws = torch.empty(hstu.hstu_jagged_attn_bwd_workspace_bytes(T, H, D), dtype=torch.uint8,
                     device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def fwd():
        hstu.hstu_jagged_attn_fwd(d["q"], d["k"], d["v"], d["offsets"], d["ts"], d["w_pos"],
                                  d["w_ts"], scale=batch.scale, max_seq_len=max_len, out=out,
                                  dev_status=status)

    def bwd():
        hstu.hstu_jagged_attn_bwd(d["q"], d["k"], d["v"], d["offsets"], d["ts"], d["w_pos"],
                                  d["w_ts"], d["dout"], scale=batch.scale, max_seq_len=max_len,
                                  dq=dq, dk=dk, dv=dv, dw_pos=dwp, dw_ts=dwt, workspace=ws,
                                  dev_status=status)

    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} after warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device())
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    launches0 = hstu.hstu_kernel_launches()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)       # evict the inputs from L2 (outside the step's events)
        ev[i][0].record()
        fwd()
        ev[i][1].record()
        bwd()
        ev[i][2].record()
    torch.cuda.synchronize()
    launches = hstu.hstu_kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    fwd_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]
    bwd_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(args.steps)]
    total_ms = sum(fwd_ms) + sum(bwd_ms)
    if world > 1:
        total_ms, fwd_sum, bwd_sum = max_over_ranks([total_ms, sum(fwd_ms), sum(bwd_ms)], dev)
    else:
        fwd_sum, bwd_sum = sum(fwd_ms), sum(bwd_ms)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the timed region")

    f_fwd, f_bwd = flops_fwd(batch), flops_bwd(batch)
    step_ms = total_ms / args.steps
    tflops = weak_scaling_rate(world, args.steps, f_fwd + f_bwd, total_ms) / 1e12
    tokens_s = weak_scaling_rate(world, args.steps, T, total_ms)
    fwd_avg, bwd_avg = fwd_sum / args.steps, bwd_sum / args.steps
    dom = "bwd" if bwd_avg >= fwd_avg else "fwd"
    dom_flops, dom_ms = (f_bwd, bwd_avg) if dom == "bwd" else (f_fwd, fwd_avg)
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    dom_kernel = "hstu_bwd_kernel" if dom == "bwd" else "hstu_fwd_kernel"
    traffic = recorded_traffic(dom_kernel, args.workload) if world == 1 else None
    roofline = {
        "kernel": "hstu_bwd_kernel (+dq convert)" if dom == "bwd" else "hstu_fwd_kernel",
        "bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
        "peak_source": f"{peak_src} bf16 dense burst (MEASURED_PEAKS.json)"
        if peak_src == "measured" else "fallback 1.59 PFLOP/s",
        "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
        "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum, "
                        "profiles/dram_traffic.txt)",
        "algorithmic_flops_per_launch": dom_flops,
    }

    f_achieved = f_fwd / (fwd_avg * 1e-3) / 1e12
    fwd_roofline = {
        "kernel": "hstu_fwd_kernel", "bound": "tensor", "achieved": round(f_achieved, 2),
        "peak": peak, "unit": "TFLOP/s", "frac": round(f_achieved / peak, 4),
        "traffic": recorded_traffic("hstu_fwd_kernel", args.workload) if world == 1 else None,
        "algorithmic_flops_per_launch": f_fwd,
        "target": "forward >= 50% of the bf16 dense peak on the fixed 8192-length workload",
    }

    # ---------------------------------------------------------------- e2e
    # Every step copies all of its inputs host -> device and all of its
    # outputs device -> host (pinned buffers).  Three streams and two device
    # sets overlap step i's inputs, step i - 1's compute and step i - 2's
    # outputs, as a training input pipeline would; the timed region runs from
    # the first input copy to the last output copy.
    e2e = None
    if not args.no_e2e:
        hout = [{n: torch.empty(t_.shape, dtype=t_.dtype).pin_memory()
                 for n, t_ in (("out", out), ("dq", dq), ("dk", dk), ("dv", dv),
                               ("dw_pos", dwp), ("dw_ts", dwt))} for _ in range(2)]
        h2d = sum(t_.numel() * t_.element_size() for t_ in host.values())
        d2h = sum(t_.numel() * t_.element_size() for t_ in hout[0].values())
        sets = [{"in": d, "out": {"out": out, "dq": dq, "dk": dk, "dv": dv, "dw_pos": dwp,
                                   "dw_ts": dwt}}]
        sets.append({"in": {k_: torch.empty_like(v_) for k_, v_ in d.items()},
                     "out": {k_: torch.empty_like(v_) for k_, v_ in sets[0]["out"].items()}})
        ws2 = torch.empty_like(ws)
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        s_comp = torch.cuda.current_stream()
        n_e2e = max(3, min(args.steps, 20))
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            b = i % 2
            di, do_ = sets[b]["in"], sets[b]["out"]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[b])     # step i - 2 has read this input set
                for n_, t_ in host.items():
                    di[n_].copy_(t_, non_blocking=True)
                ev_in[b].record(s_in)
            s_comp.wait_event(ev_in[b])
            if i >= 2:
                s_comp.wait_event(ev_out[b])        # step i - 2's outputs are copied out
            hstu.hstu_jagged_attn_fwd(di["q"], di["k"], di["v"], di["offsets"], di["ts"],
                                      di["w_pos"], di["w_ts"], scale=batch.scale,
                                      max_seq_len=max_len, out=do_["out"], dev_status=status,
                                      stream=s_comp)
            hstu.hstu_jagged_attn_bwd(di["q"], di["k"], di["v"], di["offsets"], di["ts"],
                                      di["w_pos"], di["w_ts"], di["dout"], scale=batch.scale,
                                      max_seq_len=max_len, dq=do_["dq"], dk=do_["dk"],
                                      dv=do_["dv"], dw_pos=do_["dw_pos"], dw_ts=do_["dw_ts"],
                                      workspace=ws if b == 0 else ws2, dev_status=status,
                                      stream=s_comp)
            ev_comp[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                for n_, t_ in hout[b].items():
                    t_.copy_(do_[n_], non_blocking=True)
                ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_in.wait_stream(s_comp)
        e0.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        s_out.wait_stream(s_in)
        s_out.wait_stream(s_comp)
        e1.record(s_out)
        torch.cuda.synchronize()
        e_ms = e0.elapsed_time(e1)
        if world > 1:
            e_ms = max_over_ranks([e_ms], dev)[0]
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item())} in the e2e run")
        e2e = {"value": round(world * n_e2e * (f_fwd + f_bwd) / (e_ms * 1e-3) / 1e12, 3),
               "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "tokens_per_s": round(world * n_e2e * T / (e_ms * 1e-3), 1),
               "ms_per_step": round(e_ms / n_e2e, 4), "steps": n_e2e,
               "note": "pinned host buffers; every step copies all inputs H2D and O, dQ, dK, dV, "
                       "dw_pos, dw_ts D2H, on their own streams overlapping the neighbouring "
                       "steps' compute (two device sets); timed from the first input copy to "
                       "the last output copy"}

    # ---------------------------------------------------------------- cp path
    cp = None
    if not args.no_cp:
        cp = {f"C={C}": measure_cp_path(torch, hstu, dev, rank, peaks, peak_src, args, C)
              for C in args.cp_C}

    # ---------------------------------------------------------------- targets path
    tg = None
    if not args.no_cp:
        tg = measure_targets_path(torch, hstu, dev, rank, peaks, peak_src, args)

    # ---------------------------------------------------------------- norm gate
    ng = None
    if not args.no_norm_gate:
        ng = measure_norm_gate(torch, hstu, dev, rank, peaks, peak_src, args, T, H * D)

    # ---------------------------------------------------------------- stochastic length
    slp = None
    if not args.no_norm_gate:
        slp = measure_stochastic_length(torch, hstu, dev, rank, peaks, peak_src, args, batch)

    # ---------------------------------------------------------------- cpu baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(batch, budget_s=args.cpu_budget)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": round(tflops, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded workloads module; no dataset)",
        "config": {"workload": f"{args.workload}: {DESCRIPTIONS[args.workload]}", "B": B, "T": T,
                   "H": H, "d": D, "P": batch.P, "NB": batch.NB, "max_seq_len": max_len,
                   "causal_pairs_per_head": batch.causal_pairs(),
                   "l2": "flushed before every timed step (256 MiB write, outside the events)",
                   "parallelism": f"{world} independent replica(s), one batch per rank"},
        "tokens_per_s": round(tokens_s, 1),
        "pct_bf16_peak": round(100.0 * tflops / world / peak, 2),
        "fwd_ms": round(fwd_avg, 4), "bwd_ms": round(bwd_avg, 4),
        "fwd_tflops": round(f_fwd / (fwd_avg * 1e-3) / 1e12, 2),
        "bwd_tflops": round(f_bwd / (bwd_avg * 1e-3) / 1e12, 2),
        "roofline": roofline, "fwd_roofline": fwd_roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches),
        "clocks": clk, "cp_path": cp, "targets_path": tg, "norm_gate_path": ng,
        "stochastic_length_path": slp,
    }
    return line


def measure_targets_path(torch, hstu, dev, rank, peaks, peak_src, args):
    """Target-aware forward on the ranking workload: every user's history
    followed by a microbatch of candidates (history causal; each candidate
    attends the history and itself)."""
    batch = workloads.mfalcon(seed=6 + 1000 * rank, with_dout=False)
    nt_np = batch.meta["num_targets"]
    as_bf16 = lambda bits: torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    q, k, v = (as_bf16(x).to(dev) for x in (batch.q, batch.k, batch.v))
    off = torch.from_numpy(batch.offsets.copy()).to(dev)
    ts = torch.from_numpy(batch.timestamps.copy()).to(dev)
    nt = torch.from_numpy(nt_np.copy()).to(dev)
    wp = torch.from_numpy(batch.w_pos.copy()).to(dev)
    wt = torch.from_numpy(batch.w_ts.copy()).to(dev)
    out = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    max_len = int(batch.lengths.max())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    T, H, D = q.shape

    max_nt = int(nt_np.max())

    def step_full():
        hstu.hstu_jagged_attn_fwd_targets(q, k, v, off, nt, ts, wp, wt, scale=batch.scale,
                                          max_seq_len=max_len, out=out, dev_status=status)

    def step_cand():
        hstu.hstu_jagged_attn_fwd_candidates(q, k, v, off, nt, ts, wp, wt, scale=batch.scale,
                                             max_seq_len=max_len, max_targets=max_nt, out=out,
                                             dev_status=status)

    def timed(step):
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        times = []
        for _ in range(max(3, min(args.steps, 10))):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            step()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        if int(status.item()) != 0:
            raise RuntimeError(f"targets path device status {int(status.item())}")
        return statistics.median(times)

    ms = timed(step_full)
    ms_c = timed(step_cand)
    lh = batch.lengths - nt_np
    # history pairs (causal) + every candidate's history keys and itself
    cand_pairs = float(np.sum(nt_np * (lh + 1)))
    pairs = float(np.sum(lh * (lh + 1) // 2)) + cand_pairs
    flops = 4.0 * D * H * pairs
    flops_c = 4.0 * D * H * cand_pairs
    tf = flops / (ms * 1e-3) / 1e12
    tf_c = flops_c / (ms_c * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    ncand = float(np.sum(nt_np))
    return {
        "workload": f"mfalcon: B={batch.B} users, history L_h~U{{1024..3072}}, b_m="
                    f"{int(nt_np[0])} candidates each, H={H}, d={D}, Exp(600 s) gaps, P=3072",
        "T": T, "pairs_per_head": pairs, "fwd_ms": round(ms, 4), "tflops": round(tf, 2),
        "frac_bf16_peak": round(tf / peak, 4),
        "candidates_per_s": round(ncand / (ms * 1e-3), 1),
        "candidates_only": {
            "note": "scores each user's microbatch against its cached history: candidate rows "
                    "only, history key tiles plus each candidate's own key",
            "pairs_per_head": cand_pairs, "fwd_ms": round(ms_c, 4), "tflops": round(tf_c, 2),
            "frac_bf16_peak": round(tf_c / peak, 4),
            "candidates_per_s": round(ncand / (ms_c * 1e-3), 1)},
    }


def measure_norm_gate(torch, hstu, dev, rank, peaks, peak_src, args, T, N):
    """The layer's step after attention, y = LayerNorm(O) * U over each
    token's N = H*d features, and its backward, on the headline workload's
    output shape [T, N].  Both are streams over HBM: the forward reads O and U
    and writes Y (6 bytes per element), the backward reads O, U, dY and writes
    dO, dU (10 bytes per element).  Timing inputs are drawn on the device
    (torch.randn, seeded); parity is the tests' job."""
    g = torch.Generator(device=dev)
    g.manual_seed(8 + 1000 * rank)
    o, u, dy = (torch.randn((T, N), generator=g, device=dev).to(torch.bfloat16)
                for _ in range(3))
    y, d_o, d_u = (torch.empty_like(o) for _ in range(3))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        hstu.hstu_norm_gate_fwd(o, u, out=y)
        hstu.hstu_norm_gate_bwd(o, u, dy, d_o=d_o, d_u=d_u)
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 20))
    tf, tb = [], []
    for _ in range(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        flush.fill_(1)
        evs[0].record()
        hstu.hstu_norm_gate_fwd(o, u, out=y)
        evs[1].record()
        flush.fill_(2)
        evs[2].record()
        hstu.hstu_norm_gate_bwd(o, u, dy, d_o=d_o, d_u=d_u)
        evs[3].record()
        torch.cuda.synchronize()
        tf.append(evs[0].elapsed_time(evs[1]))
        tb.append(evs[2].elapsed_time(evs[3]))
    f_ms, b_ms = statistics.median(tf), statistics.median(tb)
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    fb, bb = 6.0 * T * N, 10.0 * T * N
    f_gbs, b_gbs = fb / (f_ms * 1e-3) / 1e9, bb / (b_ms * 1e-3) / 1e9
    line = lambda kern, ms, gbs, nbytes: {
        "kernel": kern, "bound": "hbm", "ms": round(ms, 4), "achieved": round(gbs, 1),
        "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
        "algorithmic_bytes_per_launch": nbytes, "traffic": recorded_traffic(kern, "fixed8192"),
        "peak_source": f"{peak_src} copy bandwidth"}
    return {
        "workload": f"the headline workload's attention output: T={T} tokens x N={N} "
                    f"features (bf16), gate and output gradient of the same shape",
        "fwd": line("norm_gate_fwd_kernel", f_ms, f_gbs, fb),
        "bwd": line("norm_gate_bwd_kernel", b_ms, b_gbs, bb),
        "l2": "flushed before each timed launch (256 MiB write, outside the events)",
    }


def measure_stochastic_length(torch, hstu, dev, rank, peaks, peak_src, args, batch, alpha=1.6):
    """Stochastic Length on the headline batch: select (L = floor(N^(alpha/2))
    for N = the batch's longest sequence) and gather q, k, v and the
    timestamps into the shorter batch in one launch.  The gather is a stream over HBM:
    per selected row, its bytes read and written plus its 4-byte index."""
    L = hstu.sl_target_length(int(batch.lengths.max()), alpha)
    u_tok, u_seq = workloads.sl_draws(batch.T, batch.B, 12 + 1000 * rank)
    as_i32 = lambda a: torch.from_numpy(a.view(np.int32).copy()).to(dev)
    ut, us = as_i32(u_tok), as_i32(u_seq)
    off = torch.from_numpy(batch.offsets.copy()).to(dev)
    as_bf16 = lambda bits: torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    q, k, v = (as_bf16(x).to(dev) for x in (batch.q, batch.k, batch.v))
    ts = torch.from_numpy(batch.timestamps.copy()).to(dev)
    dst_off = torch.empty(batch.B + 1, dtype=torch.int64, device=dev)
    rows = torch.empty(batch.T, dtype=torch.int32, device=dev)
    outs = [torch.empty_like(x) for x in (q, k, v, ts)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step(evs=None):
        rec = (lambda i: evs[i].record()) if evs else (lambda i: None)
        rec(0)
        hstu.hstu_sl_select(off, ut, us, L, dst_offsets=dst_off, src_rows=rows)
        rec(1)
        hstu.hstu_gather_rows_multi((q, k, v, ts), rows, dst_off[batch.B:], outs=outs)
        rec(2)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    n_out = int(dst_off[batch.B].item())
    n = max(3, min(args.steps, 10))
    t_sel, t_gat = [], []
    for _ in range(n):
        flush.fill_(1)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        step(evs)
        torch.cuda.synchronize()
        t_sel.append(evs[0].elapsed_time(evs[1]))
        t_gat.append(evs[1].elapsed_time(evs[2]))
    sel_ms, gat_ms = statistics.median(t_sel), statistics.median(t_gat)
    row_bytes = sum(x[0].numel() * x.element_size() for x in (q, k, v, ts))
    gbytes = n_out * (2.0 * row_bytes + 4 * 4)
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    gbs = gbytes / (gat_ms * 1e-3) / 1e9
    return {
        "workload": f"the headline batch (T={batch.T}), alpha={alpha}: L={L}",
        "L": L, "rows_in": batch.T, "rows_out": n_out,
        "sparsity": round(1.0 - n_out / batch.T, 4),
        "select_ms": round(sel_ms, 4), "gather_ms": round(gat_ms, 4),
        "gather_roofline": {"kernel": "gather_rows_multi_kernel (q, k, v, timestamps, one launch)",
                            "bound": "hbm",
                            "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                            "frac": round(gbs / hbm, 4), "algorithmic_bytes": gbytes,
                            "peak_source": f"{peak_src} copy bandwidth"},
        "l2": "flushed before each timed step (256 MiB write, outside the events)",
    }


def measure_cp_path(torch, hstu, dev, rank, peaks, peak_src, args, C):
    """Reorder q, k, v, ts into the paired layout, attend on it, restore O."""
    batch = workloads.paired(C, seed=4 + 1000 * rank, with_dout=False)
    as_bf16 = lambda bits: torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    q, k, v = (as_bf16(x).to(dev) for x in (batch.q, batch.k, batch.v))
    off = torch.from_numpy(batch.offsets.copy()).to(dev)
    ts = torch.from_numpy(batch.timestamps.copy()).to(dev)
    wp = torch.from_numpy(batch.w_pos.copy()).to(dev)
    wt = torch.from_numpy(batch.w_ts.copy()).to(dev)
    T, H, D = q.shape
    pq, pk, pv, pts = (torch.empty_like(x) for x in (q, k, v, ts))
    pout = torch.empty_like(q)
    out = torch.empty_like(q)
    dst_off = torch.empty(C * batch.B + 1, dtype=torch.int64, device=dev)
    gpos = torch.empty(T, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    max_len = int(batch.lengths.max())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step(evs=None):
        rec = (lambda i: evs[i].record()) if evs else (lambda i: None)
        rec(0)
        hstu.hstu_cp_reorder(q, off, C, dst=pq, dst_offsets=dst_off, global_pos=gpos,
                             dev_status=status)
        rec(4)
        hstu.hstu_cp_reorder(k, off, C, dst=pk, want_maps=False, dev_status=status)
        rec(5)
        hstu.hstu_cp_reorder(v, off, C, dst=pv, want_maps=False, dev_status=status)
        rec(6)
        hstu.hstu_cp_reorder(ts, off, C, dst=pts, want_maps=False, dev_status=status)
        rec(1)
        hstu.hstu_cp_paired_attn_fwd(pq, pk, pv, off, pts, C, wp, wt, scale=batch.scale,
                                     max_seq_len=max_len, out=pout, dev_status=status)
        rec(2)
        hstu.hstu_cp_restore(pout, off, C, dst=out, dev_status=status)
        rec(3)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 10))
    times = []
    for _ in range(n):
        flush.fill_(1)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
        step(evs)
        torch.cuda.synchronize()
        # whole reorder, attention, restore; then the k and v reorder launches
        # alone (events right around each launch) for the kernel's roofline
        times.append([evs[0].elapsed_time(evs[1]), evs[1].elapsed_time(evs[2]),
                      evs[2].elapsed_time(evs[3]), evs[4].elapsed_time(evs[5]),
                      evs[5].elapsed_time(evs[6])])
    if int(status.item()) != 0:
        raise RuntimeError(f"cp path device status {int(status.item())}")
    re_ms, at_ms, rs_ms, k_ms, v_ms = (statistics.median(x) for x in zip(*times))
    launch_ms = 0.5 * (k_ms + v_ms)   # one q/k/v reorder launch
    row_qkv = H * D * 2
    reorder_bytes = 2.0 * T * (3 * row_qkv + 8) + 4.0 * T + 8.0 * (C * batch.B + 1)
    restore_bytes = 2.0 * T * row_qkv
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    f_attn = 4.0 * D * H * batch.causal_pairs()
    re_gbs = reorder_bytes / (re_ms * 1e-3) / 1e9
    rs_gbs = restore_bytes / (rs_ms * 1e-3) / 1e9
    launch_bytes = 2.0 * T * row_qkv   # one tensor read and written
    launch_gbs = launch_bytes / (launch_ms * 1e-3) / 1e9
    return {
        "workload": f"paired C={C}: B={batch.B}, L~U{{1024..16384}} rounded up to 2C, H={H}, "
                    f"d={D}, Exp(600 s) gaps, P=3072",
        "T": T, "C": C,
        "reorder_ms": round(re_ms, 4), "reorder_GBps": round(re_gbs, 1),
        "reorder_frac_hbm": round(re_gbs / hbm, 4),
        "reorder_frac_nominal_8TBps": round(re_gbs / 8000.0, 4),
        "paired_attn_ms": round(at_ms, 4),
        "paired_attn_tflops": round(f_attn / (at_ms * 1e-3) / 1e12, 2),
        "restore_ms": round(rs_ms, 4), "restore_GBps": round(rs_gbs, 1),
        "roofline": {"kernel": "cp_permute_kernel (one q/k/v reorder launch)", "bound": "hbm",
                     "achieved": round(launch_gbs, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(launch_gbs / hbm, 4), "launch_ms": round(launch_ms, 4),
                     "traffic": recorded_traffic("cp_permute_kernel", f"paired_c{C}"),
                     "traffic_unit": "bytes per launch of the q/k/v reorder (ncu dram bytes)",
                     "algorithmic_bytes_per_launch": launch_bytes,
                     "algorithmic_bytes_per_step": reorder_bytes,
                     "peak_source": f"{peak_src} copy bandwidth"},
    }


# ---------------------------------------------------------------------------
# the oracle on the host cores
# ---------------------------------------------------------------------------

def _oracle_sample(batch, budget_s):
    """A sample of (sequence, head) units whose fp64 fwd+bwd takes about
    budget_s seconds: whole sequences (all heads) in drawing order while they
    fit, else one sequence with as many of its heads as fit (at least one)."""
    import oracle
    # calibrate on the shortest sequence, one head
    order = np.argsort(batch.lengths, kind="stable")
    probe = batch.subset([int(order[0])]).head_subset([0])
    q, k, v, dout = oracle.batch_inputs(probe)
    t0 = time.perf_counter()
    oracle.fwd(q, k, v, probe.offsets, probe.timestamps, probe.w_pos, probe.w_ts,
               probe.num_heads, probe.d, probe.scale)
    oracle.bwd(q, k, v, probe.offsets, probe.timestamps, probe.w_pos, probe.w_ts,
               probe.num_heads, probe.d, probe.scale, dout)
    dt = max(time.perf_counter() - t0, 1e-4)
    rate = probe.causal_pairs() / dt          # (pair, head) units per second
    target = rate * budget_s
    H = batch.num_heads
    picked, acc = [], 0
    for idx in range(batch.B):                # in drawing order: a fair mix of lengths
        L = int(batch.lengths[idx])
        pairs = H * L * (L + 1) // 2
        if picked and acc + pairs > target:
            continue
        picked.append(idx)
        acc += pairs
        if acc >= 0.8 * target:
            break
    sub = batch.subset(picked)
    if len(picked) == 1 and acc > 1.25 * target and H > 1:
        L = int(batch.lengths[picked[0]])
        nh = int(max(1, min(H, target // max(1, L * (L + 1) // 2))))
        sub = sub.head_subset(list(range(nh)))
        return sub, f"sequence {picked[0]}, heads 0..{nh - 1} of {H}"
    return sub, f"{len(picked)} of {batch.B} sequences (all {H} heads)"


def time_oracle(sub):
    import oracle
    q, k, v, dout = oracle.batch_inputs(sub)
    t0 = time.perf_counter()
    oracle.fwd(q, k, v, sub.offsets, sub.timestamps, sub.w_pos, sub.w_ts, sub.num_heads, sub.d,
               sub.scale)
    oracle.bwd(q, k, v, sub.offsets, sub.timestamps, sub.w_pos, sub.w_ts, sub.num_heads, sub.d,
               sub.scale, dout)
    return time.perf_counter() - t0


def cpu_baseline(batch, budget_s=15.0):
    import oracle
    sub, what = _oracle_sample(batch, budget_s)
    secs = time_oracle(sub)
    flops = flops_fwd(sub) + flops_bwd(sub)
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.get_threads(),
            "kind": "oracle",
            "sample": f"fp64 C oracle fwd+bwd on {what} (T={sub.T}, {sub.causal_pairs()} "
                      f"causal pairs per head), {secs:.2f} s wall",
            "tokens_per_s": round(sub.T / secs, 2), "seconds": round(secs, 3)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import oracle
    batch = make_workload(args.workload, 0)
    budget = max(1.0, min(args.cpu_budget, 150.0 / max(1, args.steps + args.warmup)))
    sub, what = _oracle_sample(batch, budget)
    for _ in range(args.warmup):
        time_oracle(sub)
    secs = [time_oracle(sub) for _ in range(args.steps)]
    total = sum(secs)
    flops = flops_fwd(sub) + flops_bwd(sub)
    value = args.steps * flops / total / 1e12
    cores = oracle.get_threads()
    sample = (f"fp64 C oracle fwd+bwd on {what} (T={sub.T}) of the {args.workload} "
              f"workload per step")
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded workloads module; no dataset)", "impl": "reference",
            "config": {"workload": f"{args.workload}: {DESCRIPTIONS[args.workload]}",
                       "sample_T": sub.T, "sample": what},
            "tokens_per_s": round(args.steps * sub.T / total, 2),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=sorted(workloads.WORKLOADS), default="fixed8192")
    ap.add_argument("--cp-C", type=int, nargs="+", default=[2, 4, 8])
    ap.add_argument("--no-cp", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-norm-gate", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    line = run_reference(args) if args.impl == "reference" else run_native(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
