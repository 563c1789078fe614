"""Benchmark: fwd+bwd tokens/s of tiled causal linear attention over the
length sweep (H=32, d=e=128, bf16, 65,536 tokens per batch at
(B,L) in {(16,4K),(8,8K),(4,16K),(2,32K),(1,64K)}), on one B200 per rank.

One step = forward + backward at every sweep point (5 x 65,536 tokens,
32 heads each).  Inputs (512 MiB per tensor) are larger than L2, so no L2
flush is needed between steps.  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl la2|reference]

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the only other code path this script runs).
Multi-GPU (torchrun): every rank runs the whole sweep on its own GPU with no
collective on the data path (weak scaling); timing is the max over ranks.
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
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "fwd+bwd tokens/s vs L (H=32,d=e=128,bf16); % of bf16 tensor-core peak"
SWEEP = [(16, 4096), (8, 8192), (4, 16384), (2, 32768), (1, 65536)]
H, D, E = 32, 128, 128
TOKENS = 65536
# Algorithmic work per token per head (d = e = 128, bf16 I/O):
#   bytes each kernel must move: forward reads q,k,v and writes o; the dQ
#   kernel reads k,v,dO and writes dq; the dV kernel reads k,q,dO and writes
#   dv; the dK kernel reads v,dO,q and writes dk (the portable dK/dV kernel
#   reads q,k,v,dO and writes dk,dv).  The whole fwd+bwd needs at least 2,816 B.
#   The paired dV/dK launch (tc_dkdv) reads k,q,dO,v once and writes dk,dv.
BYTES_PER_TH = {"tc_fwd": 1024, "simt_fwd": 1024, "tc_dq": 1024, "simt_dq": 1024,
                "tc_dv": 1024, "tc_dk": 1024, "tc_dkdv": 1536, "simt_dkdv": 1536}
FWD_BWD_MIN_BYTES = 2816
# method flops per token-head, intra part over the causal triangle at a
# fixed C = 64 accounting: fwd (C+1)(d+e) + 4de, bwd (C+1)(3d+2e) + 10de
ALG_FLOPS_PER_TH = 65 * (D + E) + 4 * D * E + 65 * (3 * D + 2 * E) + 10 * D * E


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"la2_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
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
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        busy = [s for s in sm if mx and s > 0.3 * max(mx)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------ distributed
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of every rank's value (timings: the job is as slow as its
    slowest rank).  NCCL reduces a device tensor, gloo a host one."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processed `units_per_rank` units in
    at most `ms_max` milliseconds."""
    return world * units_per_rank / (ms_max / 1e3)


# ------------------------------------------------------------- workloads
def make_sweep_inputs(dev):
    from causal_linear_attention_fwd_b200 import inputs
    x = inputs.make_inputs(1, H, TOKENS, D, E, dtype=torch.bfloat16, device=dev, seed=0)
    lam = inputs.decay_lambdas(H, dev)
    return x, lam


def sweep_views(x, Bn, L):
    return {n: t.view(Bn, H, L, t.shape[-1]) for n, t in x.items()}


# The sources each kernel family's code comes from: a captured DRAM-traffic
# figure stays valid while these files are unchanged, whatever else changes.
SOURCE_GROUPS = {
    "tc": ("la2_tc.cuh", "la2_sm100.cuh", "la2_common.cuh"),
    "decode": ("la2_decode.cuh", "la2_common.cuh"),
    "fmap": ("la2_fmap.cuh", "la2_common.cuh"),
}


def group_of(kernel: str) -> str:
    if kernel.startswith("tc_"):
        return "tc"
    if kernel.startswith("decode"):
        return "decode"
    if kernel.startswith("feature_map"):
        return "fmap"
    return "other"


def kernel_source_hash(group: str = "tc"):
    """sha256 prefix of the sources of one kernel family."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "causal_linear_attention_fwd_b200", "csrc")
    for f in SOURCE_GROUPS[group]:
        h.update(f.encode())
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, units: int):
    """dram bytes per launch from the committed ncu summary, if it was taken
    on the current sources of the kernel's family; scaled to `units`
    token-heads."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    k = j.get("kernels", {}).get(kernel)
    group = group_of(kernel)
    if not k or group not in SOURCE_GROUPS:
        return None
    if j.get("source_hashes", {}).get(group) != kernel_source_hash(group):
        return None
    return k["dram_bytes_per_token_head"] * units


def cpu_baseline(x, lam, target_s=30.0):
    """The fp64 oracle (as it stands) on host cores on a bounded sample of the
    sweep workload: whole (b,h) sequences of the L=4096 sweep point, fwd+bwd
    (all 512 of them -- the whole sweep point -- when that fits in about
    `target_s` seconds, else as many as do)."""
    import oracle
    orc = oracle.load()
    xs = sweep_views(x, 16, 4096)
    lam_h = lam.double().cpu().numpy()
    threads = orc.num_threads()
    total = 16 * H

    def run(nh):
        flat = {n: t.view(total, 4096, t.shape[-1])[:nh].float().cpu().numpy()[None]
                for n, t in xs.items()}
        lh = np.array([lam_h[i % H] for i in range(nh)])
        t0 = time.perf_counter()
        orc.forward(flat["q"], flat["k"], flat["v"], lh)
        orc.backward(flat["q"], flat["k"], flat["v"], lh, flat["dO"])
        return time.perf_counter() - t0

    nh = min(total, max(1, threads))
    probe = run(nh)
    per_wave = probe  # one head per thread
    waves_fit = max(1, int(target_s / max(per_wave, 1e-6)))
    nh2 = min(total, waves_fit * max(1, threads))
    if nh2 > nh:
        nh, elapsed = nh2, run(nh2)
    else:
        elapsed = probe
    token_heads = nh * 4096
    return {"value": token_heads / H / elapsed, "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": f"fwd+bwd of {nh} of the 512 whole (b,h) sequences of the L=4096 sweep "
                      f"point ({token_heads} token-heads; tokens/s counts 32 heads per token) "
                      f"in {elapsed:.2f} s"}


# ------------------------------------------------------------------- main
def run_la2(args, world, rank, local):
    import causal_linear_attention_fwd_b200 as la2
    dev = torch.device("cuda", local)
    pk = peaks()
    x, lam = make_sweep_inputs(dev)
    outs = {n: torch.empty_like(x[src]) for n, src in
            (("o", "v"), ("dq", "q"), ("dk", "k"), ("dv", "v"))}
    stream = torch.cuda.current_stream()
    ws_need = max(la2.workspace_size(1, Bn, H, L, D, E, torch.bfloat16) for Bn, L in SWEEP)
    ws = torch.empty(max(ws_need, 16), dtype=torch.uint8, device=dev)

    def one_shape(Bn, L, xin=None, oo=None):
        # a training step: the backward reuses the chunk states the forward
        # left in the shared workspace
        xv = sweep_views(xin or x, Bn, L)
        ov = sweep_views(oo or outs, Bn, L)
        la2.forward(xv["q"], xv["k"], xv["v"], lam, out=ov["o"], workspace=ws)
        la2.backward(xv["q"], xv["k"], xv["v"], lam, xv["dO"],
                     outs=(ov["dq"], ov["dk"], ov["dv"]), workspace=ws,
                     reuse_forward_states=ws_need > 0)

    for _ in range(args.warmup):
        for Bn, L in SWEEP:
            one_shape(Bn, L)
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0

    clocks = ClockSampler(local)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(SWEEP) + 1)]
          for _ in range(args.steps)]
    la2.profile_enable(True)
    la2.profile_report()  # clear
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        ev[s][0].record(stream)
        for i, (Bn, L) in enumerate(SWEEP):
            one_shape(Bn, L)
            ev[s][i + 1].record(stream)
    t_stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    prof = la2.profile_report()
    la2.profile_enable(False)
    assert la2.last_device_error() == 0
    ms_local = t_start.elapsed_time(t_stop)
    ms = max_over_ranks(ms_local, world)
    per_shape = [sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps)) / args.steps
                 for i in range(len(SWEEP))]

    tokens_step = TOKENS * len(SWEEP)
    value = weak_scaling_value(tokens_step * args.steps, world, ms)
    sweep = [{"B": Bn, "L": L, "tokens_per_s": TOKENS / (t / 1e3), "ms": t}
             for (Bn, L), t in zip(SWEEP, per_shape)]
    rates = [s["tokens_per_s"] for s in sweep]
    th_per_launch = TOKENS * H

    # dominant kernel and its roofline
    launches = sum(v["launches"] for v in prof.values())
    top = max(prof.items(), key=lambda kv: kv[1]["ms"]) if prof else None
    roof = None
    if top:
        name, rec = top
        avg_ms = rec["ms"] / rec["launches"]
        bpt = BYTES_PER_TH.get(name)
        if bpt:
            alg = bpt * th_per_launch
            ach = alg / (avg_ms / 1e3) / 1e9
            tr = traffic_for(name, th_per_launch)
            roof = {"kernel": name, "bound": "hbm", "achieved": round(ach, 1),
                    "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(ach / pk["hbm_gbs"], 4),
                    "traffic": tr, "alg_bytes_per_launch": alg, "avg_launch_ms": avg_ms,
                    "peak_source": pk["source"] + " (hbm_gbs, STREAM-style copy)"}
    tc_tflops = ALG_FLOPS_PER_TH * H * value / world / 1e12 if world else 0
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "length sweep fwd+bwd, H=32, d=e=128, bf16, 65,536 tokens/batch",
                   "sweep": [[b, l] for b, l in SWEEP], "global_batch_tokens": TOKENS * world,
                   "heads": H, "d": D, "e": E, "decay": "lambda_h = 1 - 2^-(5+8h/H)",
                   "l2": "inputs 512 MiB per tensor, larger than L2; no flush",
                   "parallelism": f"replicas x{world} (independent sequences per GPU)"},
        "sweep": sweep, "sweep_spread": max(rates) / min(rates),
        "roofline": roof,
        "tensor": {"alg_flops_per_token_head": ALG_FLOPS_PER_TH,
                   "achieved_tflops_per_gpu": round(tc_tflops, 2),
                   "frac_of_bf16_peak": round(tc_tflops / pk["bf16_tflops_sustained"], 4),
                   "peak": pk["bf16_tflops_sustained"], "peak_source": pk["source"] + " sustained"},
        "hbm_frac_fwd_bwd_min": round(FWD_BWD_MIN_BYTES * H * value / world / 1e9 / pk["hbm_gbs"], 4),
        "kernels": prof, "gpu_launches": launches, "clocks": clk,
    }

    # end to end through the public API with host buffers (pinned), copies timed
    if not args.no_e2e:
        line["e2e"] = run_e2e(args, la2, lam, ws, dev, world)
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(x, lam)
    elif rank == 0:
        line["cpu_baseline"] = None
    return line


def run_e2e(args, la2, lam, ws, dev, world):
    """End to end through the public API with host buffers: every step copies
    each sweep point's q,k,v,dO from pinned host memory to the device, runs
    forward + backward, and copies o,dq,dk,dv back.  Copies run on their own
    streams, double-buffered, so the next point's upload and the previous
    point's download overlap the current point's kernels."""
    from causal_linear_attention_fwd_b200 import inputs
    hx = inputs.make_inputs(1, H, TOKENS, D, E, dtype=torch.bfloat16, device="cpu", seed=0)
    hin = {n: t.pin_memory() for n, t in hx.items()}
    hout = {n: torch.empty(hin[s].shape, dtype=torch.bfloat16).pin_memory()
            for n, s in (("o", "v"), ("dq", "q"), ("dk", "k"), ("dv", "v"))}
    din = [{n: torch.empty_like(t, device=dev) for n, t in hin.items()} for _ in range(2)]
    dout = [{n: torch.empty_like(t, device=dev) for n, t in hout.items()} for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    comp = torch.cuda.current_stream()
    bi = sum(t.numel() * t.element_size() for t in hin.values()) * len(SWEEP)
    bo = sum(t.numel() * t.element_size() for t in hout.values()) * len(SWEEP)
    # per device buffer: the compute that last read its inputs and the
    # download that last read its outputs; a buffer is refilled only after
    # both, so uploads and downloads stream across step boundaries too
    last_done, last_out = [None, None], [None, None]

    def step():
        for i, (Bn, L) in enumerate(SWEEP):
            buf = i % 2
            ev_in, ev_done, ev_out = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
            with torch.cuda.stream(s_in):
                if last_done[buf] is not None:
                    s_in.wait_event(last_done[buf])  # the buffer's inputs consumed
                for name in din[buf]:
                    din[buf][name].copy_(hin[name], non_blocking=True)
                ev_in.record(s_in)
            comp.wait_event(ev_in)
            if last_out[buf] is not None:
                comp.wait_event(last_out[buf])  # the buffer's outputs downloaded
            xv = sweep_views(din[buf], Bn, L)
            ov = sweep_views(dout[buf], Bn, L)
            la2.forward(xv["q"], xv["k"], xv["v"], lam, out=ov["o"], workspace=ws)
            la2.backward(xv["q"], xv["k"], xv["v"], lam, xv["dO"],
                         outs=(ov["dq"], ov["dk"], ov["dv"]), workspace=ws,
                         reuse_forward_states=ws.numel() > 16)
            ev_done.record(comp)
            last_done[buf] = ev_done
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done)
                for name in hout:
                    hout[name].copy_(dout[buf][name], non_blocking=True)
                ev_out.record(s_out)
            last_out[buf] = ev_out

    def drain():  # every download of the steps so far has landed in host memory
        for e in last_out:
            if e is not None:
                comp.wait_event(e)

    for _ in range(min(args.warmup, 3)):
        step()
    drain()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 5))
    barrier(world)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(comp)
    for _ in range(steps):
        step()
    drain()
    b.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world)
    return {"value": round(world * TOKENS * len(SWEEP) * steps / (ms / 1e3), 1),
            "unit": "tokens/s", "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
            "steps": steps,
            "note": "pinned host q,k,v,dO -> device, fwd+bwd, o,dq,dk,dv -> host every step; "
                    "copies double-buffered on their own streams, overlapping the kernels "
                    "and streaming across steps; timed from the first upload to the last "
                    "download"}


def run_reference(args, world, rank):
    """The oracle on host cores: each step is one bounded sample."""
    if rank != 0:
        return None
    from causal_linear_attention_fwd_b200 import inputs
    import oracle
    orc = oracle.load()
    lam = inputs.decay_lambdas(H, "cpu").double().numpy()
    nh = max(1, orc.num_threads())
    L = 4096
    x = inputs.make_inputs(1, nh, L, D, E, dtype=torch.bfloat16, device="cpu", seed=0)
    h = {n: t.float().numpy() for n, t in x.items()}
    lh = np.array([lam[i % H] for i in range(nh)])

    def step():
        orc.forward(h["q"], h["k"], h["v"], lh)
        orc.backward(h["q"], h["k"], h["v"], lh, h["dO"])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    sec = time.perf_counter() - t0
    value = nh * L * args.steps / H / sec
    return {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "length sweep fwd+bwd, H=32, d=e=128, bf16 inputs; "
                                   f"each step = {nh} (b,h) sequences at L={L}",
                       "heads": H, "d": D, "e": E},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": nh,
                             "kind": "oracle",
                             "sample": f"{nh} whole (b,h) sequences of L={L}, fwd+bwd, per step"},
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def _common(world, steps, warmup, value, unit, metric, workload_cfg, ms, extra):
    line = {"metric": metric, "value": round(value, 1), "unit": unit, "n_gpus": world,
            "steps": steps, "warmup": warmup, "ms_per_step": ms / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "data": "synthetic", "config": workload_cfg}
    line.update(extra)
    return line


def run_long(args, world, rank, local):
    """B=1, H=64, L=1,048,576 forward only (secondary workload)."""
    import causal_linear_attention_fwd_b200 as la2
    from causal_linear_attention_fwd_b200 import inputs
    dev = torch.device("cuda", local)
    pk = peaks()
    Bn, Hh, L = 1, 64, 1 << 20
    x = inputs.make_inputs(Bn, Hh, L, D, E, dtype=torch.bfloat16, device=dev, seed=0,
                           with_dO=False)
    lam = inputs.decay_lambdas(Hh, dev)
    o = torch.empty_like(x["v"])
    ws_n = la2.workspace_size(0, Bn, Hh, L, D, E, torch.bfloat16)
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        la2.forward(x["q"], x["k"], x["v"], lam, out=o, workspace=ws)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    la2.profile_enable(True)
    la2.profile_report()
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        la2.forward(x["q"], x["k"], x["v"], lam, out=o, workspace=ws)
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    prof = la2.profile_report()
    la2.profile_enable(False)
    assert la2.last_device_error() == 0
    ms = max_over_ranks(a.elapsed_time(b), world)
    value = world * L * args.steps / (ms / 1e3)
    top = max(prof.items(), key=lambda kv: kv[1]["ms"])
    name, rec = top
    avg = rec["ms"] / rec["launches"]
    roof = None
    if name in BYTES_PER_TH:
        alg = 1024 * Hh * L
        ach = alg / (avg / 1e3) / 1e9
        roof = {"kernel": name, "bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": round(ach / pk["hbm_gbs"], 4),
                "traffic": traffic_for(name, Hh * L), "alg_bytes_per_launch": alg,
                "avg_launch_ms": avg}
    extra_cpu = {}
    if rank == 0 and world == 1 and not args.no_cpu:
        # the oracle on 16 heads x the first 65,536 rows (a quarter of the
        # heads, 1/16 of the length): token-heads per second / 64 heads
        import oracle
        orc = oracle.load()
        sl = {n: x[n][:, :16, :65536].float().cpu().numpy() for n in ("q", "k", "v")}
        t0 = time.perf_counter()
        orc.forward(sl["q"], sl["k"], sl["v"], lam[:16].double().cpu().numpy())
        dt = time.perf_counter() - t0
        extra_cpu = {"cpu_baseline": {
            "value": round(16 * 65536 / 64 / dt, 1), "unit": "tokens/s", "cores": orc.num_threads(),
            "kind": "oracle",
            "sample": "forward of 16 of the 64 heads over the first 65,536 of 1,048,576 rows "
                      f"({dt:.1f} s); token-heads/s divided by 64 heads, i.e. extrapolated to "
                      "the full configuration at the same rate per token-head"}}
    return _common(world, args.steps, args.warmup, value, "tokens/s",
                   "long-context forward tokens/s (B=1,H=64,L=1M,d=e=128,bf16)",
                   {"workload": "long-context forward, B=1, H=64, L=1,048,576, d=e=128, bf16",
                    "l2": "inputs 16 GiB per tensor, larger than L2; no flush"}, ms,
                   {"dtype": "bf16", "roofline": roof, "kernels": prof,
                    "gpu_launches": sum(v["launches"] for v in prof.values()), "clocks": clk,
                    "hbm_frac_fwd_min": round(1024 * Hh * value / world / 1e9 / pk["hbm_gbs"], 4),
                    **extra_cpu})


def run_varlen(args, world, rank, local):
    """Packed variable-length batch, 65,536 rows per head slab, H=32,
    d=e=128, bf16, fwd+bwd (secondary workload)."""
    import causal_linear_attention_fwd_b200 as la2
    from causal_linear_attention_fwd_b200 import inputs
    dev = torch.device("cuda", local)
    pk = peaks()
    Hh, T = H, TOKENS
    lens = inputs.varlen_lengths(T, seed=0)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int64, device=dev)
    x = inputs.make_inputs(1, Hh, T, D, E, dtype=torch.bfloat16, device=dev, seed=0)
    x = {n: t[0] for n, t in x.items()}
    lam = inputs.decay_lambdas(Hh, dev)
    o = torch.empty_like(x["v"])
    outs = (torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"]))

    def step():
        la2.forward_varlen(x["q"], x["k"], x["v"], lam, cu, out=o)
        la2.backward_varlen(x["q"], x["k"], x["v"], lam, cu, x["dO"], outs=outs)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    clocks = ClockSampler(local)
    la2.profile_enable(True)
    la2.profile_report()
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        step()
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    prof = la2.profile_report()
    la2.profile_enable(False)
    assert la2.last_device_error() == 0
    ms = max_over_ranks(a.elapsed_time(b), world)
    value = world * T * args.steps / (ms / 1e3)
    name, rec = max(prof.items(), key=lambda kv: kv[1]["ms"])
    avg = rec["ms"] / rec["launches"]
    alg = 1024 * Hh * T
    ach = alg / (avg / 1e3) / 1e9
    roof = {"kernel": name, "bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
            "unit": "GB/s", "frac": round(ach / pk["hbm_gbs"], 4),
            "traffic": traffic_for(name + "_packed", Hh * T),
            "alg_bytes_per_launch": alg, "avg_launch_ms": avg}
    extra_cpu = {}
    if rank == 0 and world == 1 and not args.no_cpu:
        # the oracle, fwd+bwd, every head, on the documents in batch order
        # until 8,192 rows (copied to the host before the clock starts)
        import oracle
        orc = oracle.load()
        lam_h = lam.double().cpu().numpy()
        offs = np.concatenate([[0], np.cumsum(lens)])
        docs, rows = [], 0
        for n in range(len(lens)):
            if rows >= 8192:
                break
            a_, b_ = int(offs[n]), int(offs[n + 1])
            docs.append({k: x[k][:, a_:b_].float().cpu().numpy()[None] for k in ("q", "k", "v", "dO")})
            rows += b_ - a_
        t0 = time.perf_counter()
        for sl in docs:
            orc.forward(sl["q"], sl["k"], sl["v"], lam_h)
            orc.backward(sl["q"], sl["k"], sl["v"], lam_h, sl["dO"])
        dt = time.perf_counter() - t0
        extra_cpu = {"cpu_baseline": {
            "value": round(rows / dt, 1), "unit": "tokens/s", "cores": orc.num_threads(),
            "kind": "oracle",
            "sample": f"fwd+bwd of the first {len(docs)} documents ({rows} rows x 32 heads, "
                      f"{dt:.2f} s)"}}
    return _common(world, args.steps, args.warmup, value, "tokens/s",
                   "packed varlen fwd+bwd tokens/s (H=32, d=e=128, bf16)",
                   {"workload": f"packed variable-length batch, {len(lens)} sequences "
                                f"(log-uniform 64..8192 rows, seed 0, longest {max(lens)}), "
                                f"65,536 rows per head, H=32, d=e=128, bf16, fwd+bwd",
                    "l2": "inputs 512 MiB per tensor, larger than L2; no flush"}, ms,
                   {"dtype": "bf16", "roofline": roof, "kernels": prof,
                    "gpu_launches": sum(v["launches"] for v in prof.values()), "clocks": clk,
                    "sequences": len(lens), **extra_cpu})


def run_decode(args, world, rank, local):
    """Recurrent decode, batch 256, H=64, d=e=128, fp32 state; one step of
    this workload = `--decode-steps` consecutive tokens per request replayed
    from a CUDA graph, `--decode-tokens` T of them per call (T = 1: one
    la2_decode_step per token; T > 1: la2_decode_tokens, the state read and
    written once per T tokens) (secondary workload)."""
    import causal_linear_attention_fwd_b200 as la2
    from causal_linear_attention_fwd_b200 import inputs
    dev = torch.device("cuda", local)
    pk = peaks()
    Bn, Hh, n, T = 256, 64, args.decode_steps, args.decode_tokens
    assert n % T == 0, "--decode-steps must be a multiple of --decode-tokens"
    calls = n // T
    lam = inputs.decay_lambdas(Hh, dev)
    kv = inputs.decode_state0(Bn, Hh, D, E, device=dev, seed=0)
    gen = inputs.DecodeStream(Bn, Hh, D, E, device=dev, seed=0)
    toks = [gen.next() for _ in range(n)]
    # the oracle's sample: requests 0..3 (all 64 heads), every step
    samp = [tuple(a[:4].float().cpu().numpy() for a in toks[t]) for t in range(n)]
    if T > 1:  # [B,H,T,d|e] per call
        toks = [tuple(torch.stack([toks[c * T + t][i] for t in range(T)], dim=2).contiguous()
                      for i in range(3)) for c in range(calls)]
    outs = torch.empty((calls, Bn, Hh, T, E) if T > 1 else (n, Bn, Hh, E), dtype=torch.bfloat16,
                       device=dev)

    def call(c, stream):
        if T > 1:
            la2.decode_tokens(*toks[c], lam, kv, out=outs[c], stream=stream)
        else:
            la2.decode_step(*toks[c], lam, kv, out=outs[c], stream=stream)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for c in range(min(calls, 8)):  # eager warm-up launches
            call(c, s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for c in range(calls):
            call(c, s)
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    a.record(cur)
    for _ in range(args.steps):
        g.replay()
    b.record(cur)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = max_over_ranks(a.elapsed_time(b), world)
    value = world * Bn * n * args.steps / (ms / 1e3)
    per_launch_ms = ms / (calls * args.steps)
    bytes_launch = Bn * Hh * (2 * D * E * 4 + T * (2 * D + 2 * E) * 2)
    ach = bytes_launch / (per_launch_ms / 1e3) / 1e9
    roof = {"kernel": "decode_step", "bound": "hbm", "achieved": round(ach, 1),
            "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(ach / pk["hbm_gbs"], 4),
            "traffic": traffic_for("decode_step", Bn * Hh), "alg_bytes_per_launch": bytes_launch,
            "avg_launch_ms": per_launch_ms,
            "note": f"launch time = graph replay time / launches ({calls} launches per replay)"}
    what = ("one decode step per call" if T == 1 else
            f"{T} tokens per call (la2_decode_tokens)")
    extra = {"dtype": "f32", "roofline": roof, "gpu_launches": calls * args.steps, "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu:
        import oracle
        orc = oracle.load()
        st = kv[:4].double().cpu().numpy().copy()
        lam_h = lam.double().cpu().numpy()
        t0 = time.perf_counter()
        for qt, kt, vt in samp:
            orc.decode_step(qt, kt, vt, lam_h, st)
        dt = time.perf_counter() - t0
        extra["cpu_baseline"] = {
            "value": round(4 * len(samp) / dt, 1), "unit": "tokens/s", "cores": orc.num_threads(),
            "kind": "oracle",
            "sample": f"{len(samp)} decode steps of 4 of the 256 requests (64 heads each, fp64 "
                      f"state) ({dt:.2f} s); the same rate per request-token as the full batch"}
    line = _common(world, args.steps, args.warmup, value, "tokens/s",
                   "decode tokens/s (batch 256, H=64, d=e=128, fp32 state); % of HBM bandwidth",
                   {"workload": f"recurrent decode, batch 256, H=64, d=e=128, fp32 state "
                                f"(1 GiB), {n} tokens per request per graph replay, {what}",
                    "l2": "state 1 GiB, larger than L2; no flush"}, ms, extra)
    del g
    return line


def run_dlambda(args, world, rank, local):
    """Gradient with respect to the decay, la2_backward_dlambda, on the
    B=4, H=16, L=2048 training shape (bf16 inputs, fp32-FMA arithmetic)
    (secondary workload)."""
    import causal_linear_attention_fwd_b200 as la2
    from causal_linear_attention_fwd_b200 import inputs
    dev = torch.device("cuda", local)
    Bn, Hh, L = 4, 16, 2048
    x = inputs.make_inputs(Bn, Hh, L, D, E, dtype=torch.bfloat16, device=dev, seed=0)
    lam = inputs.decay_lambdas(Hh, dev)
    ws_n = la2.workspace_size(la2.LA2_OP_DLAMBDA, Bn, Hh, L, D, E, torch.bfloat16)
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        la2.dlambda(x["q"], x["k"], x["v"], lam, x["dO"], workspace=ws)
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    clocks = ClockSampler(local)
    la2.profile_enable(True)
    la2.profile_report()
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        la2.dlambda(x["q"], x["k"], x["v"], lam, x["dO"], workspace=ws)
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    prof = la2.profile_report()
    la2.profile_enable(False)
    assert la2.last_device_error() == 0
    ms = max_over_ranks(a.elapsed_time(b), world)
    value = world * Bn * L * args.steps / (ms / 1e3)
    name, rec = max(prof.items(), key=lambda kv: kv[1]["ms"])
    avg = rec["ms"] / rec["launches"]
    pk = peaks()
    tensor = name.startswith("tc_")
    if tensor:
        # tensor-core form (C = 128 rows, two CTAs per chunk, one per half
        # of e): the MMA flops it executes per token-head -- S = Q K^T by
        # both CTAs (2 x 2 C d), G = dO V^T in halves (2 C e), Q KV and Q W
        # and the KV and W updates each as a bf16 pair of products (4 x 4 d e)
        fl_th = 4 * 128 * D + 2 * 128 * E + 16 * D * E
        alg = fl_th * Bn * Hh * L
        ach = alg / (avg / 1e3) / 1e12
        roof = {"kernel": name, "bound": "tensor", "achieved": round(ach, 2),
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(ach / pk["bf16_tflops"], 4), "traffic": None,
                "alg_flops_per_launch": alg, "avg_launch_ms": avg,
                "peak_source": pk["source"] + " (bf16_tflops, burst: a kernel timed alone)",
                "note": "executed MMA flops of the tensor-core form (operand pairs counted twice)"}
    else:
        # fp32 FMA work of the block schedule per token-head (C = 32 rows): the
        # state terms q KV and q W, the updates of KV and W (2 d e flops each),
        # and the block's own pairs, (C-1)/2 of them per row at 2 (d + e) flops
        fl_th = 8 * D * E + (32 - 1) * (D + E)
        alg = fl_th * Bn * Hh * L
        ach = alg / (avg / 1e3) / 1e12
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mhz = float(json.load(f).get("sm_max_mhz", 1965.0))
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        peak = sms * 128 * 2 * mhz * 1e6 / 1e12  # fp32 lanes x FMA x max SM clock
        roof = {"kernel": name, "bound": "alu", "achieved": round(ach, 2), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": None,
                "alg_flops_per_launch": alg, "avg_launch_ms": avg,
                "peak_source": f"{sms} SMs x 128 fp32 lanes x 2 flops x {mhz:.0f} MHz (max SM clock)"}
    extra = {"dtype": "bf16" if tensor else "f32", "roofline": roof, "kernels": prof,
             "gpu_launches": sum(v["launches"] for v in prof.values()), "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu:
        import oracle
        orc = oracle.load()
        h = {n: t[:1].double().cpu().numpy() for n, t in x.items()}
        t0 = time.perf_counter()
        orc.dlambda(h["q"], h["k"], h["v"], lam.double().cpu().numpy(), h["dO"])
        dt = time.perf_counter() - t0
        extra["cpu_baseline"] = {"value": round(L / dt, 1), "unit": "tokens/s",
                                 "cores": orc.num_threads(), "kind": "oracle",
                                 "sample": f"one batch row (16 heads x {L} rows) of the workload"}
    return _common(world, args.steps, args.warmup, value, "tokens/s",
                   "dlambda tokens/s (B=4,H=16,L=2048,d=e=128, bf16 inputs)",
                   {"workload": "gradient w.r.t. the decay, B=4, H=16, L=2,048, d=e=128, bf16 "
                                "inputs",
                    "l2": "inputs 32 MiB (fit in L2); the pass is arithmetic-bound"}, ms, extra)


# The feature map's streaming passes per token-head (d = 128, bf16): the map
# reads q, k and writes phi_q, phi_k (4 x 256 B); its gradient reads q, k,
# dphi_q, dphi_k and writes dq, dk (6 x 256 B).
FMAP_BYTES_PER_TH = {"feature_map": 4 * 2 * D, "feature_map_grad": 6 * 2 * D}


def hbm_roofline(name, rec, bytes_per_th, th_per_launch, pk, traffic=None):
    avg = rec["ms"] / rec["launches"]
    alg = bytes_per_th * th_per_launch
    ach = alg / (avg / 1e3) / 1e9
    return {"kernel": name, "bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
            "unit": "GB/s", "frac": round(ach / pk["hbm_gbs"], 4), "traffic": traffic,
            "alg_bytes_per_launch": alg, "avg_launch_ms": avg,
            "peak_source": pk["source"] + " (hbm_gbs, STREAM-style copy)"}


def run_fmap(args, world, rank, local):
    """A training step with the feature map phi(x) = elu(x) + 1 on q and k:
    the map, the attention forward and backward on the mapped inputs, and the
    map's chain rule, on the B=8, H=32, L=8,192 sweep point (secondary
    workload)."""
    import causal_linear_attention_fwd_b200 as la2
    from causal_linear_attention_fwd_b200 import inputs
    dev = torch.device("cuda", local)
    pk = peaks()
    Bn, L = 8, 8192
    if args.tokens:  # profiling aid: fewer batch rows of the same length
        Bn = max(1, args.tokens // L)
    x = inputs.make_inputs(Bn, H, L, D, E, dtype=torch.bfloat16, device=dev, seed=0)
    lam = inputs.decay_lambdas(H, dev)
    buf = {n: torch.empty_like(x[src]) for n, src in
           (("pq", "q"), ("pk", "k"), ("o", "v"), ("gq", "q"), ("gk", "k"), ("dv", "v"))}
    ws_n = la2.workspace_size(la2.LA2_OP_BACKWARD, Bn, H, L, D, E, torch.bfloat16)
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)

    def step():
        la2.feature_map(x["q"], x["k"], out=(buf["pq"], buf["pk"]))
        la2.forward(buf["pq"], buf["pk"], x["v"], lam, out=buf["o"], workspace=ws)
        la2.backward(buf["pq"], buf["pk"], x["v"], lam, x["dO"],
                     outs=(buf["gq"], buf["gk"], buf["dv"]), workspace=ws,
                     reuse_forward_states=ws_n > 0)
        # dq, dk in place over the attention's gradients
        la2.feature_map_backward(x["q"], x["k"], buf["gq"], buf["gk"], out=(buf["gq"], buf["gk"]))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    clocks = ClockSampler(local)
    la2.profile_enable(True)
    la2.profile_report()
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        step()
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    prof = la2.profile_report()
    la2.profile_enable(False)
    assert la2.last_device_error() == 0
    ms = max_over_ranks(a.elapsed_time(b), world)
    value = world * Bn * L * args.steps / (ms / 1e3)
    th = Bn * L * H
    # the dominant kernel, among the attention passes and the map's two
    name, rec = max(prof.items(), key=lambda kv: kv[1]["ms"])
    bpt = {**BYTES_PER_TH, **FMAP_BYTES_PER_TH}.get(name)
    roof = hbm_roofline(name, rec, bpt, th, pk, traffic_for(name, th)) if bpt else None
    fmap_roof = {n: hbm_roofline(n, prof[n], bpt, th, pk)
                 for n, bpt in FMAP_BYTES_PER_TH.items() if n in prof}
    extra = {"dtype": "bf16", "roofline": roof, "roofline_feature_map": fmap_roof,
             "kernels": prof, "gpu_launches": sum(v["launches"] for v in prof.values()),
             "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu:
        import oracle
        orc = oracle.load()
        h = {n: t[:1].float().cpu().numpy() for n, t in x.items()}
        lam_h = lam.double().cpu().numpy()
        t0 = time.perf_counter()
        fq, fk = orc.feature_map(h["q"]), orc.feature_map(h["k"])
        orc.forward(fq, fk, h["v"], lam_h)
        g = orc.backward(fq, fk, h["v"], lam_h, h["dO"])
        orc.feature_map_grad(h["q"], g[0])
        orc.feature_map_grad(h["k"], g[1])
        dt = time.perf_counter() - t0
        extra["cpu_baseline"] = {"value": round(L / dt, 1), "unit": "tokens/s",
                                 "cores": orc.num_threads(), "kind": "oracle",
                                 "sample": f"one batch row ({H} heads x {L} rows) of the workload"}
    return _common(world, args.steps, args.warmup, value, "tokens/s",
                   f"fwd+bwd tokens/s with the elu+1 feature map (B={Bn},H={H},L={L},d=e=128,bf16)",
                   {"workload": "training step with the feature map phi(x) = elu(x) + 1 on q "
                                f"and k, B={Bn}, H={H}, L={L:,}, d=e=128, bf16",
                    "l2": f"inputs {Bn * H * L * D * 2 >> 20} MiB per tensor, larger than L2; "
                          "no flush"}, ms, extra)


def run_subrecords(args, world, rank, local):
    """The two other spec workloads, measured in the same run as the
    sweep: the long-context forward (B=1, H=64, L=1M) and recurrent decode
    (batch 256, H=64, 1,024 steps of one token).  Each is the line its own
    --workload run prints, with --sub-steps timed steps; the sweep's buffers
    are released first."""
    import copy
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    sub = copy.copy(args)
    sub.steps = args.sub_steps
    sub.warmup = 3
    out = {}
    out["long_context"] = run_long(sub, world, rank, local)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    sub.decode_tokens = 1
    out["decode"] = run_decode(sub, world, rank, local)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="la2", choices=["la2", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--workload", default="sweep",
                    choices=["sweep", "long", "decode", "varlen", "dlambda", "fmap"],
                    help="sweep (the metric; default), long (1M-token forward), decode, "
                         "varlen (packed variable-length fwd+bwd), dlambda (decay gradient), "
                         "fmap (fwd+bwd with the elu+1 feature map)")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--decode-tokens", type=int, default=1,
                    help="decode workload: tokens per request per call (1 = decode_step)")
    ap.add_argument("--no-sub", action="store_true",
                    help="sweep workload: skip the long-context forward and decode "
                         "sub-records that the default line carries")
    ap.add_argument("--sub-steps", type=int, default=5,
                    help="timed steps of each sub-record (decode: graph replays of "
                         "--decode-steps tokens)")
    ap.add_argument("--bwd-form", type=int, default=None,
                    help="profiling aid: LA2_OPT_BWD_FORM for the run (0 paired dV/dK "
                         "launch, the library's default; 1 two separate passes)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="profiling aid: tokens per sweep batch (default 65,536; with --only, "
                         "B*L must equal it), or per batch of --workload fmap (rows of 8,192); "
                         "smaller batches keep ncu captures small")
    ap.add_argument("--only", default=None,
                    help="B:L -- time a single sweep point instead of the whole sweep "
                         "(profiling aid; not the metric)")
    args = ap.parse_args()
    global SWEEP, TOKENS
    if args.tokens and args.workload == "sweep":
        assert args.only, "--tokens is a profiling aid: give the point with --only B:L"
        TOKENS = args.tokens
    if args.only:
        b_, l_ = (int(x) for x in args.only.split(":"))
        assert b_ * l_ == TOKENS, "--only must keep the batch's tokens (65,536 unless --tokens)"
        SWEEP = [(b_, l_)]
    args.warmup = max(args.warmup, 3) if args.impl == "la2" else args.warmup
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup(args.gpus)
    if args.bwd_form is not None:
        import causal_linear_attention_fwd_b200 as la2
        la2.set_option(la2.LA2_OPT_BWD_FORM, args.bwd_form)
    try:
        fn = {"sweep": run_la2, "long": run_long, "decode": run_decode,
              "varlen": run_varlen, "dlambda": run_dlambda, "fmap": run_fmap}[args.workload]
        line = fn(args, world, rank, local)
        if args.workload == "sweep" and not args.no_sub and not args.only:
            line["subrecords"] = run_subrecords(args, world, rank, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
