"""Benchmark of the exact-attention library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--legs all|none]

Prints ONE JSON line (rank 0).  The headline workload is the forward pass at
the pages' 4,096-token example: B=4, H=16, L=4096, d=128, causal, Q ~ 4 N(0,1)
(peaky rows), bf16 inputs, fp32 O + LSE.  A step is one fa_forward over that
batch; `value` is algorithmic TFLOP/s (4 B H L^2 d, halved for causal) of all
ranks' work divided by the slowest rank's time.  The other measured paths of
the library -- the training forward+backward at L=8192, the 65,536-token
forward and the split-KV decode -- are reported under "legs", each with its
own roofline.

Multi-GPU: the path does not shard (each GPU is an independent replica); the
ranks only share a barrier and a max-over-ranks of the timings.
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
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

HEADLINE = "fwd_L4096_peaky"
METRIC = "attention fwd/bwd TFLOP/s and % of bf16 tensor peak; decode HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16, datasheet
NOMINAL_HBM_GBS = 8000.0


# ----------------------------------------------------------------------------- host helpers
def attn_flops(B, H, Lq, Lk, d, causal, backward=False):
    f = 4.0 * B * H * Lq * Lk * d
    if causal:
        f *= 0.5
    if backward:
        f *= 2.5
    return f


def blocksparse_pairs(mask, Lq, Lk, causal, block=128):
    """Permitted (query, key) pairs under a block mask ([..., Tq, Tk], nonzero = permitted)
    ANDed with the length bound and the bottom-right causal mask, summed over the mask's
    leading dimensions: the algorithmic work of a block-sparse forward is 4 d FLOP per pair."""
    import numpy as np

    m = np.asarray(mask) != 0
    tq, tk = m.shape[-2], m.shape[-1]
    rows = np.arange(tq * block)[:, None]          # query row, padded to whole blocks
    c0 = np.arange(tk)[None, :] * block             # first key of each key block
    c1 = np.minimum(c0 + block, Lk)                 # one past its last key
    hi = np.minimum(c1, rows + (Lk - Lq) + 1) if causal else np.broadcast_to(c1, (rows.shape[0], tk))
    per_row = np.clip(hi - c0, 0, None) * (rows < Lq)  # [rows, tk] keys of each block per row
    per_block = per_row.reshape(tq, block, tk).sum(1)  # [tq, tk]
    return float((m * per_block).sum())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            m = json.load(fh)
        return {k: float(m[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# Source files whose state a recorded ncu capture of each kernel family depends on:
# the kernel file, the PTX helpers, the shared internal header and the host API
# (tile maps, unit orders and launch shapes are set there).
KERNEL_SOURCES = {
    "fa_fwd_kernel": ["fwd_sm100.cu", "ptx.cuh", "fa_internal.h", "api.cu"],
    "fa_fwd256_kernel": ["fwd256_sm100.cu", "ptx.cuh", "fa_internal.h", "api.cu"],
    "fa_bwd": ["bwd_sm100.cu", "ptx.cuh", "fa_internal.h", "api.cu"],
    "fa_bwd256": ["bwd256_sm100.cu", "bwd_sm100.cu", "ptx.cuh", "fa_internal.h", "api.cu"],
    "fa_decode": ["decode_sm100.cu", "ptx.cuh", "fa_internal.h", "api.cu"],
    "fa_decode_paged": ["decode_paged_mma.cu", "decode_sm100.cu", "ptx.cuh", "fa_internal.h", "api.cu"],
}


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "exact_io_aware_94_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload, algorithmic_bytes=None):
    """DRAM bytes (read + write) per launch from a committed ncu summary, if the
    kernel's sources are unchanged since the capture.  A record taken on a smaller
    case of the same kernel stores its traffic/algorithmic ratio instead, which is
    applied to this workload's algorithmic bytes."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh)
    except (OSError, ValueError):
        return None
    e = rec.get(kernel, {}).get(workload)
    if not e or e.get("source_hash") != kernel_source_hash(KERNEL_SOURCES[kernel]):
        return None
    if "bytes_per_launch" in e:
        return e["bytes_per_launch"]
    if "traffic_over_algorithmic" in e and algorithmic_bytes:
        return int(round(e["traffic_over_algorithmic"] * algorithmic_bytes))
    return None


def reduce_max(value, dist=None, device=None):
    """Max over ranks of a float (the slowest rank's time)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value, dist=None, device=None):
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.QUERY, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.25)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)
        return False

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = []
        mx = None
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU baseline (oracle)
def oracle_forward_sample(workload, budget_s, seed=0):
    """Time the oracle on a bounded sample of the forward workload's rows.

    Returns (tflops, seconds, threads, description).  Each sampled row is a
    complete output row (exact: rows are independent)."""
    import numpy as np

    import oracle
    from exact_io_aware_94_b200.inputs import WORKLOADS, attention_inputs

    w = WORKLOADS[workload]
    B, H, L, d, causal = w["B"], w["H"], w["L"], w["d"], w["causal"]
    # one head's inputs suffice for a row sample; same shapes and value distribution
    inp = attention_inputs(1, 1, L, L, d, seed=w["seed"], q_scale=w["q_scale"])
    rng = np.random.default_rng(seed)
    scale = 1.0 / math.sqrt(d)

    def run(n):
        rows = rng.integers(0, L, size=n)
        flops = sum(4.0 * d * oracle.permitted_keys(int(i), L, L, causal) for i in rows)
        t0 = time.perf_counter()
        oracle.forward_rows(inp.q, inp.k, inp.v, rows, scale, causal)
        return flops, time.perf_counter() - t0

    n = 64
    f, t = run(n)
    while t < budget_s / 8 and n < 1 << 20:
        n *= 2
        f, t = run(n)
    if t < budget_s / 2:
        n = max(n, int(n * (budget_s / 2) / max(t, 1e-6)))
        f, t = run(n)
    desc = "%d random query rows of one head of %s (B=%d H=%d L=%d d=%d causal=%s), %.1f s" % (
        n, workload, B, H, L, d, causal, t)
    return f / t / 1e12, t, oracle.num_threads(), desc


def oracle_tiny_full():
    """Time the oracle on the whole tiny forward (B=1 H=2 L=256 d=64, non-causal):
    returns (tflops, seconds)."""
    import oracle
    from exact_io_aware_94_b200.inputs import WORKLOADS, attention_inputs

    w = WORKLOADS["tiny_fwd"]
    B, H, L, d = w["B"], w["H"], w["L"], w["d"]
    inp = attention_inputs(B, H, L, L, d, seed=w["seed"])
    flops = attn_flops(B, H, L, L, d, w["causal"])
    reps, t = 0, 0.0
    t0 = time.perf_counter()
    while t < 0.5:
        oracle.forward(inp.q, inp.k, inp.v, 1.0 / math.sqrt(d), w["causal"])
        reps += 1
        t = time.perf_counter() - t0
    return flops * reps / t / 1e12, t / reps


def cpu_baseline(budget_s):
    """The oracle on the host cores (all of them, then one): the headline workload's
    row sample, and the whole tiny forward."""
    import oracle

    tf, _, cores, desc = oracle_forward_sample(HEADLINE, budget_s)
    out = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}
    tiny_tf, tiny_s = oracle_tiny_full()
    out["tiny_fwd_full"] = {"TFLOP/s": tiny_tf, "s_per_call": tiny_s, "cores": cores}
    oracle.set_num_threads(1)
    try:
        tf1, _, _, desc1 = oracle_forward_sample(HEADLINE, budget_s / 4)
        tiny_tf1, tiny_s1 = oracle_tiny_full()
    finally:
        oracle.set_num_threads(cores)
    out["single_core"] = {"cores": 1, HEADLINE: {"TFLOP/s": tf1, "sample": desc1},
                          "tiny_fwd_full": {"TFLOP/s": tiny_tf1, "s_per_call": tiny_s1}}
    return out


# ----------------------------------------------------------------------------- GPU timing
def time_steps(fn, steps, warmup, stream, dist=None, device=None):
    """Warm up, then time exactly `steps` calls between barrier+synchronize pairs with
    CUDA events on the launching stream; returns the max-over-ranks total seconds."""
    import torch

    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if dist is not None and dist.is_initialized():
        dist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    if dist is not None and dist.is_initialized():
        dist.barrier()
    torch.cuda.synchronize()
    return reduce_max(start.elapsed_time(end) / 1e3, dist, device)


def run_ours(args, dist, rank, world, device):
    import torch

    import exact_io_aware_94_b200 as fa
    from exact_io_aware_94_b200.inputs import WORKLOADS

    peaks, peak_kind = load_peaks()
    stream = torch.cuda.current_stream(device)
    w = WORKLOADS[HEADLINE]
    B, H, L, d, causal = w["B"], w["H"], w["L"], w["d"], w["causal"]
    gen = torch.Generator(device=device).manual_seed(w["seed"] + 1000 * rank)
    # seeded synthetic inputs of the workload's shape and distribution, resident in HBM
    q = (torch.randn(B, H, L, d, generator=gen, device=device) * w["q_scale"]).to(torch.bfloat16)
    k = torch.randn(B, H, L, d, generator=gen, device=device).to(torch.bfloat16)
    v = torch.randn(B, H, L, d, generator=gen, device=device).to(torch.bfloat16)
    o = torch.empty(B, H, L, d, dtype=torch.float32, device=device)
    lse = torch.empty(B, H, L, dtype=torch.float32, device=device)
    scale = 1.0 / math.sqrt(d)

    def step():
        rc = fa.fa_forward(q, k, v, o, lse, B, H, L, L, d, scale, causal, fa.FA_DT_F32, stream)
        if rc != fa.FA_OK:
            raise fa.FAError(rc, "fa_forward")

    flops = attn_flops(B, H, L, L, d, causal)
    with ClockSampler(torch.cuda.current_device()) as clk:
        secs = time_steps(step, args.steps, args.warmup, stream, dist, device)
    status = fa.fa_check_status(stream)
    if status != fa.FA_OK:
        raise fa.FAError(status, "device status after the timed region")
    ms_per_step = secs / args.steps * 1e3
    value = reduce_sum(flops * args.steps, dist, device) / secs / 1e12
    achieved = flops / (secs / args.steps) / 1e12  # the step is one launch of the forward kernel
    roof = {"kernel": "fa_fwd_kernel<128>", "bound": "tensor", "achieved": round(achieved, 1),
            "peak": peaks["bf16_tflops"], "peak_kind": peak_kind + " burst bf16 (cuBLAS 8192^3)",
            "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
            "frac_of_nominal_2250": round(achieved / NOMINAL_BF16_TFLOPS, 4),
            "traffic": recorded_traffic("fa_fwd_kernel", HEADLINE),
            "algorithmic_flops_per_launch": flops}

    # ---- end to end through the public API: every step copies its Q/K/V in from pinned host
    # memory and its O/LSE out to pinned host memory.  Steps are pipelined as a serving loop
    # would run them: two device buffer sets and three streams, so the host->device copy of
    # step i+1 and the device->host copy of step i-1 overlap the forward of step i.
    qh = q.cpu().pin_memory()
    kh = k.cpu().pin_memory()
    vh = v.cpu().pin_memory()
    sets = [(q, k, v, o, lse), tuple(torch.empty_like(t) for t in (q, k, v, o, lse))]
    outs = [(torch.empty(o.shape, dtype=o.dtype).pin_memory(), torch.empty(lse.shape, dtype=lse.dtype).pin_memory())
            for _ in range(2)]
    s_in = torch.cuda.Stream(device)
    s_out = torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_fwd = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        """n pipelined steps; device seconds from the first copy in to the last copy out."""
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(s_in)
        for i in range(n):
            b = i % 2
            qd, kd, vd, od, ld = sets[b]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_fwd[b])  # step i-2's forward has read this set's inputs
                qd.copy_(qh, non_blocking=True)
                kd.copy_(kh, non_blocking=True)
                vd.copy_(vh, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # step i-2's results have left this set's outputs
            rc = fa.fa_forward(qd, kd, vd, od, ld, B, H, L, L, d, scale, causal, fa.FA_DT_F32, stream)
            if rc != fa.FA_OK:
                raise fa.FAError(rc, "fa_forward")
            ev_fwd[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_fwd[b])
                outs[b][0].copy_(od, non_blocking=True)
                outs[b][1].copy_(ld, non_blocking=True)
                ev_out[b].record(s_out)
        end.record(s_out)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / 1e3

    e2e_steps = max(2, min(args.steps, 20))
    e2e_run(max(2, args.warmup))
    if dist is not None and dist.is_initialized():
        dist.barrier()
    e2e_secs = reduce_max(e2e_run(e2e_steps), dist, device)
    e2e_value = reduce_sum(flops * e2e_steps, dist, device) / e2e_secs / 1e12
    h2d = 3 * q.numel() * q.element_size()
    d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()

    legs = {}
    launches = args.steps  # fa_forward launches exactly one kernel per call
    if args.legs == "all":
        del qh, kh, vh, outs, sets
        legs = run_legs(args, fa, torch, device, stream, peaks, peak_kind, rank, dist)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, Q x4), generated on device",
        "config": {"workload": HEADLINE + ": forward, B=4 H=16 Lq=Lk=4096 d=128 causal, Q~4N(0,1), O fp32 + LSE",
                   "global_batch": B * world, "seq_len": L, "parallelism": "replicas%d" % world,
                   "l2": "inputs larger than L2 (192 MiB of Q/K/V per replica vs 126 MB L2)"},
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "path": "each step: pinned host Q/K/V -> device (copy stream), fa_forward (compute stream), O/LSE -> pinned host (second copy stream); two device buffer sets, so the copies of neighbouring steps overlap the forward"},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "legs": legs,
    }
    if rank == 0 and world == 1 and args.cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.cpu_budget)
    return out


def run_legs(args, fa, torch, device, stream, peaks, peak_kind, rank, dist):
    from exact_io_aware_94_b200.inputs import WORKLOADS, blocksparse_mask

    legs = {}
    steps = max(3, min(args.steps, 20))
    warm = max(3, args.warmup)

    # the tiny forward (B=1 H=2 L=256 d=64, non-causal): latency-bound, so no roofline
    w = WORKLOADS["tiny_fwd"]
    B, H, L, d = w["B"], w["H"], w["L"], w["d"]
    gen = torch.Generator(device=device).manual_seed(w["seed"] + 1000 * rank)
    q, k, v = (torch.randn(B, H, L, d, generator=gen, device=device).to(torch.bfloat16) for _ in range(3))
    o = torch.empty(B, H, L, d, dtype=torch.float32, device=device)
    lse = torch.empty(B, H, L, dtype=torch.float32, device=device)

    def fwd_tiny():
        rc = fa.fa_forward(q, k, v, o, lse, B, H, L, L, d, 1.0 / math.sqrt(d), 0, fa.FA_DT_F32, stream)
        assert rc == fa.FA_OK

    t_t = time_steps(fwd_tiny, steps, warm, stream, dist, device) / steps
    legs["tiny_fwd"] = {"ms": round(t_t * 1e3, 5), "us": round(t_t * 1e6, 2),
                        "TFLOP/s": round(attn_flops(B, H, L, L, d, False) / t_t / 1e12, 3), "launches": 1,
                        "note": "latency-bound (4 units on 148 SMs): time reported, no roofline target",
                        "l2": "inputs 192 KB, L2-resident between calls"}
    del q, k, v, o, lse

    # training forward + backward at L = 8192
    w = WORKLOADS["train_L8192"]
    B, H, L, d = w["B"], w["H"], w["L"], w["d"]
    gen = torch.Generator(device=device).manual_seed(w["seed"] + 1000 * rank)
    q, k, v, g = (torch.randn(B, H, L, d, generator=gen, device=device).to(torch.bfloat16) for _ in range(4))
    o = torch.empty(B, H, L, d, dtype=torch.float32, device=device)
    lse = torch.empty(B, H, L, dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = fa.workspace(fa.fa_backward_workspace_size(B, H, L, L, d), device)
    scale = 1.0 / math.sqrt(d)

    def fwd():
        rc = fa.fa_forward(q, k, v, o, lse, B, H, L, L, d, scale, 1, fa.FA_DT_F32, stream)
        assert rc == fa.FA_OK

    def bwd():
        rc = fa.fa_backward(q, k, v, o, g, lse, dq, dk, dv, B, H, L, L, d, scale, 1, fa.FA_DT_F32, ws,
                            ws.numel(), stream)
        assert rc == fa.FA_OK

    ff = attn_flops(B, H, L, L, d, True)
    fb = attn_flops(B, H, L, L, d, True, backward=True)
    t_f = time_steps(fwd, steps, warm, stream, dist, device) / steps
    t_b = time_steps(bwd, steps, warm, stream, dist, device) / steps
    legs["train_L8192_fwd"] = {"ms": round(t_f * 1e3, 4), "TFLOP/s": round(ff / t_f / 1e12, 1),
                               "frac_of_peak": round(ff / t_f / 1e12 / peaks["bf16_tflops"], 4), "launches": 1}
    legs["train_L8192_bwd"] = {"ms": round(t_b * 1e3, 4), "TFLOP/s": round(fb / t_b / 1e12, 1),
                               "frac_of_peak": round(fb / t_b / 1e12 / peaks["bf16_tflops"], 4),
                               "launches": 3, "kernels": "fa_bwd_dot + fa_bwd_dkdv + fa_bwd_dq",
                               "flops_convention": "2.5 x forward (5 GEMMs); the kernels run 7",
                               "traffic": recorded_traffic("fa_bwd", "train_L8192")}
    del q, k, v, g, o, lse, dq, dk, dv, ws

    # 65,536-token forward
    w = WORKLOADS["long_L65536"]
    B, H, L, d = w["B"], w["H"], w["L"], w["d"]
    q, k, v = (torch.randn(B, H, L, d, generator=gen, device=device).to(torch.bfloat16) for _ in range(3))
    o = torch.empty(B, H, L, d, dtype=torch.float32, device=device)
    lse = torch.empty(B, H, L, dtype=torch.float32, device=device)

    def fwd_long():
        rc = fa.fa_forward(q, k, v, o, lse, B, H, L, L, d, scale, 1, fa.FA_DT_F32, stream)
        assert rc == fa.FA_OK

    fl = attn_flops(B, H, L, L, d, True)
    t_l = time_steps(fwd_long, max(3, steps // 4), 3, stream, dist, device) / max(3, steps // 4)
    legs["long_L65536_fwd"] = {"ms": round(t_l * 1e3, 4), "TFLOP/s": round(fl / t_l / 1e12, 1),
                               "frac_of_peak": round(fl / t_l / 1e12 / peaks["bf16_tflops"], 4), "launches": 1}
    del q, k, v, o, lse

    # head dimension 256 (one 128-row Q tile per unit, 64-key K/V tiles)
    w = WORKLOADS["fwd_d256_L4096"]
    B, H, L, d = w["B"], w["H"], w["L"], w["d"]
    q, k, v = (torch.randn(B, H, L, d, generator=gen, device=device).to(torch.bfloat16) for _ in range(3))
    o = torch.empty(B, H, L, d, dtype=torch.float32, device=device)
    lse = torch.empty(B, H, L, dtype=torch.float32, device=device)

    def fwd_d256():
        rc = fa.fa_forward(q, k, v, o, lse, B, H, L, L, d, 1.0 / math.sqrt(d), 1, fa.FA_DT_F32, stream)
        assert rc == fa.FA_OK

    f256 = attn_flops(B, H, L, L, d, True)
    t_256 = time_steps(fwd_d256, steps, warm, stream, dist, device) / steps
    legs["fwd_d256_L4096"] = {"ms": round(t_256 * 1e3, 4), "TFLOP/s": round(f256 / t_256 / 1e12, 1),
                              "frac_of_peak": round(f256 / t_256 / 1e12 / peaks["bf16_tflops"], 4), "launches": 1,
                              "kernel": "fa_fwd256_kernel",
                              "traffic": recorded_traffic("fa_fwd256_kernel", "fwd_d256_L4096"),
                              "config": "B4 H16 L4096 d256 causal, O fp32 + LSE"}
    g256 = torch.randn(B, H, L, d, generator=gen, device=device).to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = fa.workspace(fa.fa_backward_workspace_size(B, H, L, L, d), device)

    def bwd_d256():
        rc = fa.fa_backward(q, k, v, o, g256, lse, dq, dk, dv, B, H, L, L, d, 1.0 / math.sqrt(d), 1, fa.FA_DT_F32,
                            ws, ws.numel(), stream)
        assert rc == fa.FA_OK

    fb256 = attn_flops(B, H, L, L, d, True, backward=True)
    t_b256 = time_steps(bwd_d256, steps, warm, stream, dist, device) / steps
    legs["bwd_d256_L4096"] = {"ms": round(t_b256 * 1e3, 4), "TFLOP/s": round(fb256 / t_b256 / 1e12, 1),
                              "frac_of_peak": round(fb256 / t_b256 / 1e12 / peaks["bf16_tflops"], 4),
                              "launches": 3, "kernels": "fa_bwd_dot + fa_bwd_dkdv256 + fa_bwd_dq256",
                              "traffic": recorded_traffic("fa_bwd256", "bwd_d256_L4096"),
                              "flops_convention": "2.5 x forward (5 GEMMs); the kernels run 9 (dK/dV halves "
                                                  "recompute S^T and dP^T; dQ recomputes S and dP)",
                              "config": "B4 H16 L4096 d256 causal"}
    del q, k, v, o, lse, g256, dq, dk, dv, ws

    # decode over a 32,768-slot cache
    w = WORKLOADS["decode_cap32768"]
    B, H, cap, d = w["B"], w["H"], w["cap"], w["d"]
    cg = torch.Generator("cpu").manual_seed(w["seed"])
    lens = torch.randint(w["len_lo"], w["len_hi"] + 1, (B,), generator=cg).to(torch.int32)
    kc = torch.randn(B, H, cap, d, generator=gen, device=device).to(torch.bfloat16)
    vc = torch.randn(B, H, cap, d, generator=gen, device=device).to(torch.bfloat16)
    qd = torch.randn(B, H, d, generator=gen, device=device).to(torch.bfloat16)
    lens_d = lens.to(device)
    od = torch.empty(B, H, d, dtype=torch.float32, device=device)
    ld = torch.empty(B, H, dtype=torch.float32, device=device)
    wsd = fa.workspace(fa.fa_decode_workspace_size(B, H, cap, d), device)

    def dec():
        rc = fa.fa_decode(qd, kc, vc, lens_d, od, ld, B, H, cap, d, scale, fa.FA_DT_F32, wsd, wsd.numel(), stream)
        assert rc == fa.FA_OK

    nbytes = int(lens.sum()) * H * d * 2 * 2
    t_d = time_steps(dec, steps, warm, stream, dist, device) / steps
    legs["decode_cap32768"] = {"ms": round(t_d * 1e3, 4), "GB/s": round(nbytes / t_d / 1e9, 1),
                               "kv_bytes": nbytes,
                               "frac_of_peak": round(nbytes / t_d / 1e9 / peaks["hbm_gbs"], 4),
                               "frac_of_nominal_8000": round(nbytes / t_d / 1e9 / NOMINAL_HBM_GBS, 4),
                               "launches": 3, "kernels": "fa_decode_plan + fa_decode_split + fa_decode_combine",
                               "l2": "caches 2 x 16 GiB, far larger than L2",
                               "traffic": recorded_traffic("fa_decode", "decode_cap32768", nbytes)}
    del kc, vc

    # packed prefill batch of sequences of different lengths (causal)
    w = WORKLOADS["prefill_varlen"]
    Bv, Hv, dv_ = w["B"], w["H"], w["d"]
    cg = torch.Generator("cpu").manual_seed(w["seed"])
    lens_v = torch.randint(w["len_lo"], w["len_hi"] + 1, (Bv,), generator=cg).to(torch.int32)
    cu = torch.zeros(Bv + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lens_v, 0)
    tot = int(cu[-1])
    qv, kv_, vv = (torch.randn(tot, Hv, dv_, generator=gen, device=device).to(torch.bfloat16) for _ in range(3))
    ov = torch.empty(tot, Hv, dv_, dtype=torch.float32, device=device)
    lv = torch.empty(Hv, tot, dtype=torch.float32, device=device)
    cu_d = cu.to(device)
    mx = int(lens_v.max())
    sc_v = 1.0 / math.sqrt(dv_)

    def fwd_varlen():
        rc = fa.fa_forward_varlen(qv, kv_, vv, ov, lv, cu_d, cu_d, Bv, Hv, tot, tot, mx, dv_, sc_v, 1, fa.FA_DT_F32,
                                  stream)
        assert rc == fa.FA_OK

    fv = sum(attn_flops(1, Hv, int(n), int(n), dv_, True) for n in lens_v)
    # algorithmic bytes: Q, K, V in (bf16), O (fp32) and LSE out
    bytes_v = tot * Hv * dv_ * (3 * 2 + 4) + tot * Hv * 4
    t_v = time_steps(fwd_varlen, steps, warm, stream, dist, device) / steps
    legs["prefill_varlen"] = {"ms": round(t_v * 1e3, 4), "TFLOP/s": round(fv / t_v / 1e12, 1),
                              "frac_of_peak": round(fv / t_v / 1e12 / peaks["bf16_tflops"], 4), "launches": 1,
                              "kernel": "fa_fwd_kernel (packed)",
                              "traffic": recorded_traffic("fa_fwd_kernel", "prefill_varlen", bytes_v),
                              "config": "16 causal sequences, lengths U[512, 8192] (%d tokens), H16 d128, packed"
                                        % tot}
    del qv, kv_, vv, ov, lv

    # causal prefill under a block-sparse mask (sink + local window + 10% random blocks, per head)
    w = WORKLOADS["prefill_blocksparse"]
    Bs, Hs, Ls, ds = w["B"], w["H"], w["L"], w["d"]
    mask = blocksparse_mask(Hs, Ls, Ls, seed=w["seed"], sink=w["sink"], window=w["window"], p_random=w["p_random"])
    qs, ks, vs = (torch.randn(Bs, Hs, Ls, ds, generator=gen, device=device).to(torch.bfloat16) for _ in range(3))
    os_ = torch.empty(Bs, Hs, Ls, ds, dtype=torch.float32, device=device)
    ls_ = torch.empty(Bs, Hs, Ls, dtype=torch.float32, device=device)
    mask_d = mask.to(device)
    tq = mask.shape[1]
    wss = fa.workspace(fa.fa_forward_blocksparse_workspace_size(Bs, Hs, Ls, Ls), device)
    sc_s = 1.0 / math.sqrt(ds)

    def fwd_blocksparse():
        rc = fa.fa_forward_blocksparse(qs, ks, vs, os_, ls_, mask_d, 0, tq * tq, Bs, Hs, Ls, Ls, ds, sc_s, 1,
                                       fa.FA_DT_F32, wss, wss.numel(), stream)
        assert rc == fa.FA_OK

    # algorithmic work: 4 d FLOP per permitted (query, key) pair (the mask is shared by the batch)
    pairs = Bs * blocksparse_pairs(mask.numpy(), Ls, Ls, True)
    fs = 4.0 * ds * pairs
    density = pairs / (Bs * Hs * Ls * (Ls + 1) / 2)
    t_s = time_steps(fwd_blocksparse, steps, warm, stream, dist, device) / steps
    legs["prefill_blocksparse"] = {"ms": round(t_s * 1e3, 4), "TFLOP/s": round(fs / t_s / 1e12, 1),
                                   "frac_of_peak": round(fs / t_s / 1e12 / peaks["bf16_tflops"], 4),
                                   "launches": 2, "kernels": "fa_bsparse_plan + fa_fwd_kernel (block-sparse)",
                                   "permitted_fraction_of_causal": round(density, 4),
                                   "traffic": recorded_traffic("fa_fwd_kernel", "prefill_blocksparse"),
                                   "config": "B2 H16 L16384 d128 causal; per-head block mask: sink block, window "
                                             "of 8 key blocks, 10% of other blocks below the diagonal; TFLOP/s "
                                             "counts permitted pairs only"}
    del qs, ks, vs, os_, ls_

    # paged cache with grouped heads: same batch and lengths, 8 KV heads for 32 query heads
    w = WORKLOADS["decode_paged_gqa"]
    B, H, Hkv, ps, nblk, d = w["B"], w["H"], w["Hkv"], w["page_size"], w["max_blocks"], w["d"]
    cg = torch.Generator("cpu").manual_seed(w["seed"])
    lens = torch.randint(w["len_lo"], w["len_hi"] + 1, (B,), generator=cg).to(torch.int32)
    used = [(int(n) + ps - 1) // ps for n in lens]
    num_pages = sum(used)
    perm = torch.randperm(num_pages, generator=cg).to(torch.int32)
    table = torch.zeros(B, nblk, dtype=torch.int32)
    at = 0
    for b in range(B):
        table[b, : used[b]] = perm[at:at + used[b]]
        at += used[b]
    kp = torch.randn(num_pages, Hkv, ps, d, generator=gen, device=device).to(torch.bfloat16)
    vp = torch.randn(num_pages, Hkv, ps, d, generator=gen, device=device).to(torch.bfloat16)
    qp = torch.randn(B, H, d, generator=gen, device=device).to(torch.bfloat16)
    table_d, lens_p = table.to(device), lens.to(device)
    op = torch.empty(B, H, d, dtype=torch.float32, device=device)
    lp = torch.empty(B, H, dtype=torch.float32, device=device)
    wsp = fa.workspace(fa.fa_decode_paged_workspace_size(B, H, nblk, ps, d), device)

    def dec_paged():
        rc = fa.fa_decode_paged(qp, kp, vp, table_d, lens_p, op, lp, B, H, Hkv, num_pages, ps, nblk, d, scale,
                                fa.FA_DT_F32, wsp, wsp.numel(), stream)
        assert rc == fa.FA_OK

    nbytes = int(lens.sum()) * Hkv * d * 2 * 2
    t_p = time_steps(dec_paged, steps, warm, stream, dist, device) / steps
    legs["decode_paged_gqa"] = {"ms": round(t_p * 1e3, 4), "GB/s": round(nbytes / t_p / 1e9, 1),
                                "kv_bytes": nbytes,
                                "frac_of_peak": round(nbytes / t_p / 1e9 / peaks["hbm_gbs"], 4),
                                "frac_of_nominal_8000": round(nbytes / t_p / 1e9 / NOMINAL_HBM_GBS, 4),
                                "launches": 3,
                                "kernels": "fa_decode_plan + fa_decode_paged_mma + fa_decode_combine",
                                "traffic": recorded_traffic("fa_decode_paged", "decode_paged_gqa", nbytes),
                                "config": "B64 H32 Hkv8 (groups of 4) d128, 64-token pages in shuffled order, "
                                          "lengths U[1024, 32768]",
                                "l2": "pages 2 x %.1f GiB, far larger than L2" % (kp.numel() * 2 / 2 ** 30)}
    del kp, vp
    status = fa.fa_check_status(stream)
    if status != fa.FA_OK:
        raise fa.FAError(status, "device status after the legs")
    return legs


def run_profile_case(args, device):
    """One path of the library, W + K calls on seeded device inputs, for a profiler
    (ncu) to capture; prints a single status line.  fwd: the headline forward;
    bwd: forward then backward at the 8,192-token training shape; decode_small:
    decode at B=16 H=32 cap=8192 (1 GiB of cache, small enough to capture);
    varlen_small: packed causal forward of 8 sequences of 512..4,096 tokens;
    fwd256: the d = 256 forward at B=4 H=16 L=4,096;
    decode_paged_small: paged, grouped-head decode at B=16 H=32 Hkv=8;
    blocksparse_small: block-sparse causal forward at B=2 H=16 L=8192 with the
    benchmark's mask recipe (192 MiB of Q/K/V, more than L2); blocksparse: the same at
    the benchmark's B=2 H=16 L=16384; bwd256: forward then backward at B=4 H=16
    L=4,096 d=256."""
    import torch

    import exact_io_aware_94_b200 as fa
    from exact_io_aware_94_b200.inputs import WORKLOADS

    gen = torch.Generator(device=device).manual_seed(11)
    stream = torch.cuda.current_stream(device)
    calls = args.warmup + args.steps
    if args.profile_case in ("fwd", "bwd"):
        w = WORKLOADS[HEADLINE if args.profile_case == "fwd" else "train_L8192"]
        B, H, L, d = w["B"], w["H"], w["L"], w["d"]
        q = (torch.randn(B, H, L, d, generator=gen, device=device) * w["q_scale"]).to(torch.bfloat16)
        k, v, g = (torch.randn(B, H, L, d, generator=gen, device=device).to(torch.bfloat16) for _ in range(3))
        o, lse = fa.forward(q, k, v, causal=True, stream=stream)
        if args.profile_case == "fwd":
            for _ in range(calls):
                fa.forward(q, k, v, causal=True, out=o, lse=lse, stream=stream)
        else:
            ws = fa.workspace(fa.fa_backward_workspace_size(B, H, L, L, d), device)
            for _ in range(calls):
                fa.backward(q, k, v, o, g, lse, causal=True, ws=ws, stream=stream)
        nbytes = 0
    elif args.profile_case == "fwd256":
        # head dimension 256: the d = 256 forward at B4 H16 L4096 causal (384 MiB of Q/K/V)
        w = WORKLOADS["fwd_d256_L4096"]
        B, H, L, d = w["B"], w["H"], w["L"], w["d"]
        q, k, v = (torch.randn(B, H, L, d, generator=gen, device=device).to(torch.bfloat16) for _ in range(3))
        o, lse = fa.forward(q, k, v, causal=True, stream=stream)
        for _ in range(calls):
            fa.forward(q, k, v, causal=True, out=o, lse=lse, stream=stream)
        nbytes = 0
    elif args.profile_case == "varlen_small":
        # 8 causal sequences of 512..4,096 tokens, H16 d128 (about 1 GB on the device)
        lens = torch.randint(512, 4097, (8,), generator=torch.Generator().manual_seed(7)).to(torch.int32)
        cu = torch.zeros(9, dtype=torch.int32)
        cu[1:] = torch.cumsum(lens, 0)
        tot, H, d = int(cu[-1]), 16, 128
        q, k, v = (torch.randn(tot, H, d, generator=gen, device=device).to(torch.bfloat16) for _ in range(3))
        cu_d = cu.to(device)
        for _ in range(calls):
            fa.forward_varlen(q, k, v, cu_d, cu_d, int(lens.max()), causal=True, stream=stream)
        nbytes = 0
    elif args.profile_case == "bwd256":
        w = WORKLOADS["fwd_d256_L4096"]
        B, H, L, d = w["B"], w["H"], w["L"], w["d"]
        q, k, v, g = (torch.randn(B, H, L, d, generator=gen, device=device).to(torch.bfloat16) for _ in range(4))
        o, lse = fa.forward(q, k, v, causal=True, stream=stream)
        ws = fa.workspace(fa.fa_backward_workspace_size(B, H, L, L, d), device)
        for _ in range(calls):
            fa.backward(q, k, v, o, g, lse, causal=True, ws=ws, stream=stream)
        nbytes = 0
    elif args.profile_case in ("blocksparse_small", "blocksparse"):
        from exact_io_aware_94_b200.inputs import blocksparse_mask

        w = WORKLOADS["prefill_blocksparse"]
        B, H, L, d = (2, 16, 8192, 128) if args.profile_case == "blocksparse_small" else (w["B"], w["H"], w["L"], w["d"])
        q, k, v = (torch.randn(B, H, L, d, generator=gen, device=device).to(torch.bfloat16) for _ in range(3))
        mask = blocksparse_mask(H, L, L, seed=w["seed"], sink=w["sink"], window=w["window"],
                                p_random=w["p_random"]).to(device)
        ws = fa.workspace(fa.fa_forward_blocksparse_workspace_size(B, H, L, L), device)
        for _ in range(calls):
            fa.forward_blocksparse(q, k, v, mask, causal=True, ws=ws, stream=stream)
        nbytes = 0
    elif args.profile_case == "decode_paged_small":
        # paged, grouped heads: B16 H32 Hkv8 d128, 64-token pages, lengths U[1024, 8192]
        B, H, Hkv, ps, nblk, d = 16, 32, 8, 64, 128, 128
        cg = torch.Generator().manual_seed(6)
        lens = torch.randint(1024, nblk * ps + 1, (B,), generator=cg).to(torch.int32)
        used = [(int(n) + ps - 1) // ps for n in lens]
        npg = sum(used)
        perm = torch.randperm(npg, generator=cg).to(torch.int32)
        table = torch.zeros(B, nblk, dtype=torch.int32)
        at = 0
        for b in range(B):
            table[b, : used[b]] = perm[at:at + used[b]]
            at += used[b]
        kp, vp = (torch.randn(npg, Hkv, ps, d, generator=gen, device=device).to(torch.bfloat16) for _ in range(2))
        qd = torch.randn(B, H, d, generator=gen, device=device).to(torch.bfloat16)
        ws = fa.workspace(fa.fa_decode_paged_workspace_size(B, H, nblk, ps, d), device)
        t_d, l_d = table.to(device), lens.to(device)
        for _ in range(calls):
            fa.decode_paged(qd, kp, vp, t_d, l_d, ws=ws, stream=stream)
        nbytes = int(lens.sum()) * Hkv * d * 2 * 2
    else:
        B, H, cap, d = 16, 32, 8192, 128
        kc, vc = (torch.randn(B, H, cap, d, generator=gen, device=device).to(torch.bfloat16) for _ in range(2))
        qd = torch.randn(B, H, d, generator=gen, device=device).to(torch.bfloat16)
        lens = torch.randint(1024, cap + 1, (B,), generator=torch.Generator().manual_seed(5)).to(torch.int32)
        ws = fa.workspace(fa.fa_decode_workspace_size(B, H, cap, d), device)
        lens_d = lens.to(device)
        for _ in range(calls):
            fa.decode(qd, kc, vc, lens_d, ws=ws, stream=stream)
        nbytes = int(lens.sum()) * H * d * 2 * 2
    torch.cuda.synchronize()
    status = fa.fa_check_status(stream)
    print(json.dumps({"profile_case": args.profile_case, "calls": calls, "status": status,
                      "algorithmic_kv_bytes_per_call": nbytes}), flush=True)
    return 0 if status == fa.FA_OK else 1


def run_reference(args, rank):
    """The oracle, as it stands, on the host cores: bounded samples of the same workload."""
    if rank != 0:
        return None
    vals = []
    secs = []
    desc = ""
    cores = 0
    for _ in range(args.warmup):
        oracle_forward_sample(HEADLINE, 1.0)
    for _ in range(args.steps):
        tf, s, cores, desc = oracle_forward_sample(HEADLINE, args.ref_budget)
        vals.append(tf)
        secs.append(s)
    value = statistics.median(vals)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.median(secs), 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16, Q x4)",
        "config": {"workload": HEADLINE + ": forward, B=4 H=16 Lq=Lk=4096 d=128 causal, Q~4N(0,1)",
                   "global_batch": 4, "seq_len": 4096, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--legs", choices=["all", "none"], default="all")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=5.0, help="seconds of oracle work per reference step")
    ap.add_argument("--profile-case", choices=["fwd", "bwd", "decode_small", "varlen_small", "decode_paged_small",
                                                    "blocksparse_small", "blocksparse", "fwd256", "bwd256"],
                    default=None,
                    help="run only this path W+K times for a profiler; no benchmark line")
    args = ap.parse_args(argv)
    if args.impl == "ours" and args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if args.profile_case:
        return run_profile_case(args, device)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    try:
        out = run_ours(args, dist if world > 1 else None, rank, world, device)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
