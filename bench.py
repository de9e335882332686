#!/usr/bin/env python
"""Benchmark of exact tiled attention on B200.

One step = forward + backward (O, LSE, dQ, dK, dV) of the dense causal
prefill workload B=4, H=16, S=2048, D=128 (bf16, i.i.d. N(0,1) synthetic
inputs), i.e. every row of the hot path: tile staging, QK^T, masking, online
softmax, exact rescale, PV, epilogue, backward preprocess, backward main,
dQ convert, on the persistent LPT schedule.  The metric is algorithmic
TFLOP/s: forward 4*B*H*S^2*D/2 (causal), backward 2.5x that.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs N independent replicas (one process per GPU, launched with
torch.distributed.run); the work does not shard, so scaling is weak and the
value is the sum over ranks of the work divided by the slowest rank's time.
Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle on
a bounded sample of the same workload instead.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd & bwd TFLOP/s (bf16, causal, D=128) and % of B200 dense BF16 peak"
WORKLOAD = dict(workload="dense_prefill_B4_H16_S2048_D128_causal_fwd+bwd", batch_per_gpu=4, heads=16,
                seq_len=2048, head_dim=128, causal=True)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def fwd_flops(B, H, Sq, Sk, D, causal):
    return 4.0 * B * H * Sq * Sk * D * (0.5 if causal else 1.0)


def window_pairs(Sq, Sk, left, right, causal):
    """Number of (query, key) pairs a bottom-right aligned window (and causal mask) keeps."""
    import numpy as np
    i = np.arange(Sq, dtype=np.int64)
    off = Sk - Sq
    lo = np.zeros(Sq, dtype=np.int64) if left < 0 else np.maximum(i + off - left, 0)
    r = 0 if causal else right
    hi = np.full(Sq, Sk - 1, dtype=np.int64) if (r < 0 and not causal) else np.minimum(i + off + max(r, 0), Sk - 1)
    return int(np.maximum(hi - lo + 1, 0).sum())


def max_over_ranks(value, world, device="cpu"):
    """The slowest rank's figure; every rank takes part in the same collective (no-op for one rank)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(step_flops, world, ms_per_step):
    """Whole-job throughput of `world` replicas that each did one step in (at most) ms_per_step."""
    return world * step_flops / (ms_per_step * 1e-3) / 1e12


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


def traffic_record(kernel_name, source_file):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "roofline_traffic.txt")
    try:
        sha = hashlib.sha256(open(os.path.join(ROOT, source_file), "rb").read()).hexdigest()[:16]
        for line in open(path):
            f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
            if f.get("kernel") == kernel_name and f.get("source_sha") == sha:
                return float(f["bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpus):
        self.gpus = gpus
        self.proc = None
        self.out = os.path.join("/tmp", f"fa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", ",".join(str(g) for g in self.gpus)],
                                         stdout=open(self.out, "w"), stderr=subprocess.DEVNULL)
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
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.out):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                for n, v in zip(names, f[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
            os.remove(self.out)
        except Exception:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


_CPU_WORKLOAD = []


def cpu_oracle_sample(budget_s=12.0, max_heads=64, prefix=None):
    """Time the fp64 oracle on whole (batch, head) problems of the workload until budget_s is spent."""
    import oracle
    from exact_tiled_attention_41_b200 import workloads as W

    if not _CPU_WORKLOAD:
        _CPU_WORKLOAD.append(W.dense_prefill(seed=0))
    w = _CPU_WORKLOAD[0]
    t = w.tensors
    S = prefix or w.meta["Sq"]
    q = t["q"][:, :S].double().numpy()
    k = t["k"][:, :S].double().numpy()
    v = t["v"][:, :S].double().numpy()
    do = t["do"][:, :S].double().numpy()
    mask = oracle.allowed_mask(S, S, True)
    flops, heads = 0.0, 0
    t0 = time.perf_counter()
    for h in range(max_heads):
        b, hh = divmod(h, w.meta["Hq"])
        oracle.head_forward(q[b, :, hh], k[b, :, hh], v[b, :, hh], w.scale, mask)
        oracle.head_backward(q[b, :, hh], k[b, :, hh], v[b, :, hh], do[b, :, hh], w.scale, mask)
        flops += 3.5 * fwd_flops(1, 1, S, S, 128, True)
        heads += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return flops, dt, heads, S


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"), default=0)
        if n:
            return n
    except Exception:
        pass
    return os.cpu_count()


# ---------------------------------------------------------------------------------------------- reference arm


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    # each step: fp64 oracle forward + backward of one (batch, head) problem on the first `prefix`
    # tokens of the causal workload (rows there see exactly the same keys as in the full problem)
    prefix = 512 if (args.steps + args.warmup) <= 400 else 256
    for _ in range(args.warmup):
        cpu_oracle_sample(budget_s=0.0, max_heads=1, prefix=prefix)
    tot_flops, tot_dt = 0.0, 0.0
    for _ in range(args.steps):
        f, dt, _, _ = cpu_oracle_sample(budget_s=0.0, max_heads=1, prefix=prefix)
        tot_flops += f
        tot_dt += dt
    value = tot_flops / tot_dt / 1e12
    cores = cpu_threads()
    sample = f"per step: fp64 oracle fwd+bwd of one (batch, head) causal problem on the first {prefix} tokens"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(WORKLOAD, parallelism="replicas"),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------- our arm


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from exact_tiled_attention_41_b200 import abi, attention as A, workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    abi.load()
    pk, pk_kind = peaks()

    w = W.dense_prefill(seed=rank)
    B, S, H, D = 4, 2048, 16, 128
    t = {n: x.to(dev) for n, x in w.tensors.items()}
    q, k, v, do = t["q"], t["k"], t["v"], t["do"]
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = abi.fa_bwd_workspace_size(B, H, H, S, S, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)   # > 126 MB L2
    stream = torch.cuda.current_stream()
    scale = w.scale
    ff = fwd_flops(B, H, S, S, D, True)
    step_flops = 3.5 * ff

    det = 1 if args.deterministic else 0

    def step():
        st = abi.fa_fwd(q, k, v, out, lse, B, H, H, S, S, D, scale, 1, None, 0, stream)
        st |= abi.fa_bwd_ex(q, k, v, out, do, lse, dq, dk, dv, B, H, H, S, S, D, scale, 1, -1, -1, det, ws, ws_bytes,
                            stream)
        return st

    for _ in range(args.warmup):
        flush.zero_()
        if step() != 0:
            raise RuntimeError("launch failed in warm-up")
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    sampler = ClockSampler(list(range(world)) if world > 1 else [local_rank]) if local_rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    abi.fa_profile_begin(1)
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    abi.fa_profile_begin(0)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    _, n_f, ms_f = abi.fa_profile_read(abi.FA_KERNEL_FWD)
    _, n_b, ms_b = abi.fa_profile_read(abi.FA_KERNEL_BWD)
    _, n_q, ms_q = abi.fa_profile_read(abi.FA_KERNEL_BWD_DQ)   # deterministic backward only
    _, n_ba, ms_ba = abi.fa_profile_read(abi.FA_KERNEL_BWD_ALL)   # whole backward: preprocess + main + dQ
    total_ms = max_over_ranks(total_ms, world, dev)
    if abi.fa_get_device_status() != 0:
        raise RuntimeError("a kernel reported a device-side timeout during the timed region")
    ms_per_step = total_ms / args.steps
    value = aggregate_tflops(step_flops, world, ms_per_step)

    # ----------------------------------------------------------------- end to end through the public API
    # Each step copies its inputs from pinned host memory, runs the forward and backward through the
    # torch-level API and copies every result back.  Three streams (copy in, compute, copy out) with
    # two buffer sets: step i's results go out while step i+1's inputs come in (the two directions of
    # the host link are independent); every dependency is an event.
    e2e_steps = min(args.steps, 30)
    pin = {n: x.cpu().pin_memory() for n, x in w.tensors.items()}
    names_out = ("out", "lse", "dq", "dk", "dv")
    shapes_out = {"out": (q.shape, q.dtype), "lse": (lse.shape, lse.dtype), "dq": (q.shape, q.dtype),
                  "dk": (k.shape, k.dtype), "dv": (v.shape, v.dtype)}
    host_out = [{n: torch.empty(sh, dtype=dt, pin_memory=True) for n, (sh, dt) in shapes_out.items()}
                for _ in range(2)]
    dev_in = [{n: torch.empty_like(x, device=dev) for n, x in pin.items()} for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x in pin.values())
    d2h = sum(x.numel() * x.element_size() for x in host_out[0].values())
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    started = [False, False]

    def e2e_step(i):
        b_ = i % 2
        x = dev_in[b_]
        with torch.cuda.stream(s_in):
            if started[b_]:
                s_in.wait_event(ev_cmp[b_])          # the compute of step i-2 has read this buffer set
            for n, src in pin.items():
                x[n].copy_(src, non_blocking=True)
            ev_in[b_].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[b_])
            o_, l_ = A.flash_attn_func(x["q"], x["k"], x["v"], scale, True)
            g = A.flash_attn_backward(x["do"], x["q"], x["k"], x["v"], o_, l_, scale, True,
                                      deterministic=bool(det))
            outs = (o_, l_) + tuple(g)
            for t_ in outs:
                t_.record_stream(s_out)              # the allocator keeps them until the copy-out is done
            ev_cmp[b_].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b_])
            for n, t_ in zip(names_out, outs):
                host_out[b_][n].copy_(t_, non_blocking=True)
        started[b_] = True

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(e2e_steps):
        e2e_step(3 + i)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    e2e_value = aggregate_tflops(step_flops, world, e2e_ms)

    extras = {}
    if world == 1 and not args.no_extras:
        extras = measure_extras(torch, abi, A, W, dev, pk)

    if rank != 0:
        return 0
    peak_t = pk["bf16_tflops"]
    bwd_ms = ms_b / max(n_b, 1) + (ms_q / max(n_q, 1) if det else 0.0)
    fwd_ms = ms_f / max(n_f, 1)
    bwd_tf = 2.5 * ff / (bwd_ms * 1e-3) / 1e12
    fwd_tf = ff / (fwd_ms * 1e-3) / 1e12
    bwd_all_ms = ms_ba / max(n_ba, 1)
    bwd_all_tf = 2.5 * ff / (bwd_all_ms * 1e-3) / 1e12
    traffic = None if det else traffic_record("bwd_kernel", "exact_tiled_attention_41_b200/csrc/bwd.cu")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(WORKLOAD, global_batch=4 * world, parallelism="replicas" if world > 1 else "single",
                       l2="flushed before every step (256 MiB write, outside the per-step events)",
                       **({"backward": "deterministic"} if det else {})),
        "roofline": {"bound": "tensor",
                     "kernel": "bwd_kernel + dq_kernel (deterministic backward)" if det else "bwd_kernel (backward main)",
                     "achieved": bwd_tf,
                     "peak": peak_t, "unit": "TFLOP/s", "frac": bwd_tf / peak_t, "traffic": traffic,
                     "peak_source": f"{pk_kind} bf16_tflops (burst)",
                     "algorithmic_flops_per_launch": 2.5 * ff, "avg_launch_ms": bwd_ms, "launches": n_b,
                     "whole_backward": {"launches": "preprocess + main + dQ " + ("pass" if det else "convert"),
                                        "achieved": bwd_all_tf, "frac": bwd_all_tf / peak_t,
                                        "avg_ms": bwd_all_ms, "calls": n_ba}},
        "parts": {
            "fwd_kernel": {"tflops": fwd_tf, "avg_launch_ms": fwd_ms, "launches": n_f,
                           "frac_of_measured_peak": fwd_tf / peak_t, "frac_of_spec_2250": fwd_tf / 2250.0},
            "bwd_kernel": {"tflops": bwd_tf, "avg_launch_ms": bwd_ms, "launches": n_b,
                           "frac_of_measured_peak": bwd_tf / peak_t, "frac_of_spec_2250": bwd_tf / 2250.0},
            "bwd_total": {"tflops": bwd_all_tf, "avg_ms": bwd_all_ms, "calls": n_ba,
                          "frac_of_measured_peak": bwd_all_tf / peak_t, "frac_of_spec_2250": bwd_all_tf / 2250.0,
                          "what": "preprocess + main + dQ " + ("pass" if det else "convert")},
            "step_frac_of_measured_peak": value / world / peak_t,
        },
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms,
                "api": "attention.flash_attn_func + flash_attn_backward, pinned host buffers; copy-in, compute and "
                       "copy-out on three streams, two buffer sets (step i's results leave while step i+1's "
                       "inputs arrive)"},
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
    }
    if extras:
        line["extras"] = extras
    if world == 1 and not args.no_cpu_baseline:
        f, dt, heads, Sx = cpu_oracle_sample(budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                                "sample": f"fp64 oracle fwd+bwd of {heads} whole (batch, head) problems of the "
                                          f"workload (S={Sx}), {dt:.1f} s"}
    print(json.dumps(line), flush=True)
    return 0


def measure_extras(torch, abi, A, W, dev, pk):
    """Other workloads, timed with CUDA events on the launching stream (not part of the step)."""
    res = {}
    stream = torch.cuda.current_stream()

    def timed(fn, iters):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(iters):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    # long-context GQA: B=2, Hq=32, Hkv=8, S=8192, D=128, causal (inputs > L2)
    w = W.gqa_long(seed=0)
    t = {n: x.to(dev) for n, x in w.tensors.items()}
    B, S, Hq, Hkv, D = 2, 8192, 32, 8, 128
    out = torch.empty_like(t["q"])
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(t["q"]), torch.empty_like(t["k"]), torch.empty_like(t["v"])
    nb = abi.fa_bwd_workspace_size(B, Hq, Hkv, S, S, D)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)
    ff = fwd_flops(B, Hq, S, S, D, True)
    fms = timed(lambda: abi.fa_fwd(t["q"], t["k"], t["v"], out, lse, B, Hq, Hkv, S, S, D, w.scale, 1, None, 0,
                                   stream), 5)
    bms = timed(lambda: abi.fa_bwd(t["q"], t["k"], t["v"], out, t["do"], lse, dq, dk, dv, B, Hq, Hkv, S, S, D,
                                   w.scale, 1, ws, nb, stream), 3)
    # the same backward with deterministic dq (query-tile-stationary pass, fixed summation order)
    dms = timed(lambda: abi.fa_bwd_ex(t["q"], t["k"], t["v"], out, t["do"], lse, dq, dk, dv, B, Hq, Hkv, S, S, D,
                                      w.scale, 1, -1, -1, 1, ws, nb, stream), 3)
    res["gqa_long_B2_Hq32_Hkv8_S8192_D128_causal"] = {
        "fwd_ms": fms, "fwd_tflops": ff / fms / 1e9, "bwd_ms": bms, "bwd_tflops": 2.5 * ff / bms / 1e9,
        "fwd_frac_of_measured_peak": ff / fms / 1e9 / pk["bf16_tflops"],
        "bwd_frac_of_measured_peak": 2.5 * ff / bms / 1e9 / pk["bf16_tflops"],
        "bwd_deterministic_ms": dms, "bwd_deterministic_tflops": 2.5 * ff / dms / 1e9}
    # sliding window of 4096 keys (causal): FLOPs of the pairs the window keeps
    wf = 4.0 * B * Hq * D * window_pairs(S, S, 4096, 0, True)
    wfms = timed(lambda: abi.fa_fwd_ex(t["q"], t["k"], t["v"], out, lse, B, Hq, Hkv, S, S, D, w.scale, 1, 4096, 0,
                                       None, 0, stream), 5)
    wbms = timed(lambda: abi.fa_bwd_ex(t["q"], t["k"], t["v"], out, t["do"], lse, dq, dk, dv, B, Hq, Hkv, S, S, D,
                                       w.scale, 1, 4096, 0, 0, ws, nb, stream), 3)
    res["gqa_long_B2_Hq32_Hkv8_S8192_D128_causal_window4096"] = {
        "fwd_ms": wfms, "fwd_tflops": wf / wfms / 1e9, "bwd_ms": wbms, "bwd_tflops": 2.5 * wf / wbms / 1e9,
        "fwd_frac_of_measured_peak": wf / wfms / 1e9 / pk["bf16_tflops"],
        "bwd_frac_of_measured_peak": 2.5 * wf / wbms / 1e9 / pk["bf16_tflops"]}
    del t, out, lse, dq, dk, dv, ws

    # varlen packed batch, D = 64 and 256 (forward and backward)
    for D in (64, 256):
        w = W.varlen_packed(D, seed=0)
        t = {n: x.to(dev) for n, x in w.tensors.items()}
        m = w.meta
        lens = (w.tensors["cu_q"][1:] - w.tensors["cu_q"][:-1]).tolist()
        ff = 4.0 * 0.5 * m["Hq"] * D * sum(L * L for L in lens)
        out = torch.empty_like(t["q"])
        lse = torch.empty((m["Hq"], m["total_q"]), dtype=torch.float32, device=dev)
        fnb = abi.fa_varlen_fwd_workspace_size(16, m["total_q"], m["total_k"], 16, 16, D)
        fws = torch.empty(fnb, dtype=torch.uint8, device=dev)    # the forward's dynamic schedule
        fms = timed(lambda: abi.fa_varlen_fwd(t["q"], t["k"], t["v"], out, lse, t["cu_q"], t["cu_k"], 16, m["max_q"],
                                              m["max_k"], m["total_q"], m["total_k"], 16, 16, D, w.scale, 1, fws,
                                              fnb, stream), 5)
        r = {"fwd_ms": fms, "fwd_tflops": ff / fms / 1e9, "total_tokens": m["total_q"]}
        dq, dk, dv = torch.empty_like(t["q"]), torch.empty_like(t["k"]), torch.empty_like(t["v"])
        nb = abi.fa_varlen_bwd_workspace_size(16, m["total_q"], m["total_k"], 16, 16, D)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        bms = timed(lambda: abi.fa_varlen_bwd(t["q"], t["k"], t["v"], out, t["do"], lse, dq, dk, dv, t["cu_q"],
                                              t["cu_k"], 16, m["max_q"], m["max_k"], m["total_q"], m["total_k"], 16,
                                              16, D, w.scale, 1, ws, nb, stream), 3)
        r.update(bwd_ms=bms, bwd_tflops=2.5 * ff / bms / 1e9)
        res[f"varlen_16seq_H16_D{D}_causal"] = r
        del t

    # KV-cache decode: B=64, Hq=32, Hkv=8, cache lengths U[1024, 16384], capacity 16384, D=128
    w = W.decode(seed=0, nan_guard=False, device=str(dev))
    t = w.tensors
    lens = t["cache_seqlens"].to(dev)
    B, Hq, Hkv, D, cap = 64, 32, 8, 128, 16384
    out = torch.empty_like(t["q"])
    lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=dev)
    nb = abi.fa_fwd_kvcache_workspace_size(B, Hq, Hkv, 1, cap, D, 0)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)
    kv_bytes = float(w.tensors["cache_seqlens"].sum().item()) * Hkv * D * 2 * 2
    alg_bytes = kv_bytes + 2 * t["q"].numel() * 2
    dec = lambda: abi.fa_fwd_kvcache(t["q"], t["k_cache"], t["v_cache"], lens, out, lse, B, Hq, Hkv, 1, cap, D,
                                     w.scale, 0, 0, ws, nb, stream)
    dms = timed(dec, 10)
    # the split kernel alone, from the library's own events (a separate pass: the events around it
    # serialize the launches, which the call above does not)
    abi.fa_profile_begin(1)
    timed(dec, 10)
    abi.fa_profile_begin(0)
    _, n_s, ms_s = abi.fa_profile_read(abi.FA_KERNEL_DECODE)
    split_ms = ms_s / max(n_s, 1)
    res["decode_B64_Hq32_Hkv8_cap16384_D128"] = {
        "ms": dms, "gbs": alg_bytes / dms / 1e6, "frac_of_measured_hbm": alg_bytes / dms / 1e6 / pk["hbm_gbs"],
        "split_kernel_ms": split_ms, "split_kernel_gbs": kv_bytes / split_ms / 1e6,
        "algorithmic_bytes": alg_bytes}

    # the same cache in pages of 256 keys behind a random block table
    page = 256
    nps = cap // page
    gperm = torch.Generator("cpu").manual_seed(1)
    table = torch.randperm(B * nps, generator=gperm).reshape(B, nps).to(torch.int32).to(dev)
    kp = torch.empty((B * nps, page, Hkv, D), dtype=torch.bfloat16, device=dev)
    vp = torch.empty_like(kp)
    kp[table.flatten().long()] = t["k_cache"].view(B * nps, page, Hkv, D)
    vp[table.flatten().long()] = t["v_cache"].view(B * nps, page, Hkv, D)
    del t["k_cache"], t["v_cache"]
    nbp = abi.fa_fwd_kvcache_ex_workspace_size(B, Hq, Hkv, 1, D, page, nps, 0)
    wsp = torch.empty(nbp, dtype=torch.uint8, device=dev)
    pms = timed(lambda: abi.fa_fwd_kvcache_ex(t["q"], kp, vp, lens, None, None, 0, None, table, nps, B * nps, page,
                                              out, lse, B, Hq, Hkv, 1, D, w.scale, 0, -1, -1, 0, wsp, nbp, stream), 10)
    res["decode_paged256_B64_Hq32_Hkv8_cap16384_D128"] = {
        "ms": pms, "gbs": alg_bytes / pms / 1e6, "frac_of_measured_hbm": alg_bytes / pms / 1e6 / pk["hbm_gbs"]}

    # four new tokens per row (speculative-decoding shape), appended in place, causal
    sn = 4
    g4 = torch.Generator(str(dev)).manual_seed(2)
    q4 = torch.randn((B, sn, Hq, D), generator=g4, device=dev).to(torch.bfloat16)
    kn = torch.randn((B, sn, Hkv, D), generator=g4, device=dev).to(torch.bfloat16)
    vn = torch.randn((B, sn, Hkv, D), generator=g4, device=dev).to(torch.bfloat16)
    lens4 = torch.clamp(lens, max=cap - sn)
    out4 = torch.empty_like(q4)
    lse4 = torch.empty((B, Hq, sn), dtype=torch.float32, device=dev)
    nb4 = abi.fa_fwd_kvcache_ex_workspace_size(B, Hq, Hkv, sn, D, page, nps, 0)
    ws4 = torch.empty(nb4, dtype=torch.uint8, device=dev)
    ams = timed(lambda: abi.fa_fwd_kvcache_ex(q4, kp, vp, lens4, kn, vn, sn, None, table, nps, B * nps, page, out4,
                                              lse4, B, Hq, Hkv, sn, D, w.scale, 1, -1, -1, 0, ws4, nb4, stream), 10)
    a_bytes = (float(lens4.sum().item()) + B * sn) * Hkv * D * 2 * 2 + 2 * q4.numel() * 2 + 2 * kn.numel() * 2 * 2
    res["decode_append4_causal_paged256_B64_Hq32_Hkv8_D128"] = {
        "ms": ams, "gbs": a_bytes / ams / 1e6, "frac_of_measured_hbm": a_bytes / ams / 1e6 / pk["hbm_gbs"]}
    del t, w, kp, vp, wsp, ws4

    # merging four partial results of the long-context GQA output (B=2, S=8192, H=32, D=128, bf16)
    C, Bm, Sm, Hm, Dm = 4, 2, 8192, 32, 128
    gm = torch.Generator(str(dev)).manual_seed(3)
    o_parts = torch.randn((C, Bm, Sm, Hm, Dm), generator=gm, device=dev).to(torch.bfloat16)
    l_parts = torch.randn((C, Bm, Hm, Sm), generator=gm, device=dev)
    o_m = torch.empty((Bm, Sm, Hm, Dm), dtype=torch.bfloat16, device=dev)
    l_m = torch.empty((Bm, Hm, Sm), dtype=torch.float32, device=dev)
    mms = timed(lambda: abi.fa_merge_lse(o_parts, l_parts, C, Bm, Sm, Hm, Dm, 0, o_m, l_m, 0, stream), 10)
    m_bytes = (C + 1) * (o_m.numel() * 2 + l_m.numel() * 4)
    res["merge_lse_4parts_B2_S8192_H32_D128"] = {
        "ms": mms, "gbs": m_bytes / mms / 1e6, "frac_of_measured_hbm": m_bytes / mms / 1e6 / pk["hbm_gbs"]}
    del o_parts, l_parts, o_m, l_m
    torch.cuda.empty_cache()
    return res


def w_scale(D):
    return 1.0 / math.sqrt(D)


def run_profile_case(args):
    """One mid-size case of a single path, for an ncu capture: inputs larger than L2 but under a GB."""
    import torch
    from exact_tiled_attention_41_b200 import abi
    from exact_tiled_attention_41_b200 import workloads as W
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    if args.profile_case == "decode":
        # B=64, Hq=32, Hkv=8, D=128, cache lengths uniform in [1024, 2048], capacity 2048 (537 MB of cache)
        B, Hq, Hkv, D, cap = 64, 32, 8, 128, 2048
        w = W.kvcache(B, Hq, Hkv, D, cap, 1024, 2048, seed=0, nan_guard=False, device=str(dev))
        t = w.tensors
        lens = t["cache_seqlens"].to(dev)
        out = torch.empty_like(t["q"])
        lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=dev)
        nb = abi.fa_fwd_kvcache_workspace_size(B, Hq, Hkv, 1, cap, D, 0)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        nbytes = float(t["cache_seqlens"].sum().item()) * Hkv * D * 2 * 2 + 2 * t["q"].numel() * 2
        fn = lambda: abi.fa_fwd_kvcache(t["q"], t["k_cache"], t["v_cache"], lens, out, lse, B, Hq, Hkv, 1, cap, D,
                                        w.scale, 0, 0, ws, nb, stream)
        name = "decode_B64_Hq32_Hkv8_cap2048_D128"
    elif args.profile_case in ("varlen64", "varlen256"):
        # the varlen packed workload (16 sequences, L ~ U[128, 4096], H = 16, causal): forward + backward
        D = 64 if args.profile_case == "varlen64" else 256
        w = W.varlen_packed(D, seed=0)
        t = {n: x.to(dev) for n, x in w.tensors.items()}
        m = w.meta
        n, T, H = m["num_seqs"], m["total_q"], m["Hq"]
        out = torch.empty_like(t["q"])
        lse = torch.empty((H, T), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(t["q"]), torch.empty_like(t["k"]), torch.empty_like(t["v"])
        nb = abi.fa_varlen_bwd_workspace_size(n, T, T, H, H, D)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        lens = (t["cu_q"][1:] - t["cu_q"][:-1]).cpu().double()
        nbytes = 3.5 * float((4.0 * H * D * lens * lens * 0.5).sum())    # algorithmic FLOPs (fwd + bwd)

        fws = torch.empty(256, dtype=torch.uint8, device=dev)    # the forward's dynamic schedule

        def fn():
            st = abi.fa_varlen_fwd(t["q"], t["k"], t["v"], out, lse, t["cu_q"], t["cu_k"], n, m["max_q"], m["max_k"],
                                   T, T, H, H, D, w.scale, 1, fws, 256, stream)
            return st | abi.fa_varlen_bwd(t["q"], t["k"], t["v"], out, t["do"], lse, dq, dk, dv, t["cu_q"], t["cu_k"],
                                          n, m["max_q"], m["max_k"], T, T, H, H, D, w.scale, 1, ws, nb, stream)
        name = f"varlen_16seq_L128-4096_H16_D{D}_causal_fwd+bwd"
    elif args.profile_case in ("append", "decode256"):
        # paged cache, B=64, Hq=32, Hkv=8, lengths uniform in [1024, 2048], pages of 256 keys; "append" adds 4
        # causal query tokens whose k / v are written into the cache first, "decode256" is one token at D = 256
        D = 128 if args.profile_case == "append" else 256
        Sq = 4 if args.profile_case == "append" else 1
        B, Hq, Hkv, cap, page = 64, 32, 8, 2304, 256
        g = torch.Generator("cpu").manual_seed(5)
        lens_l = torch.randint(1024, 2049, (B,), generator=g).tolist()
        gd = torch.Generator(str(dev)).manual_seed(5)
        nblk = B * cap // page
        perm = torch.randperm(nblk, generator=g).reshape(B, cap // page).to(torch.int32).to(dev)
        kc = torch.randn((nblk, page, Hkv, D), generator=gd, device=dev).to(torch.bfloat16)
        vc = torch.randn((nblk, page, Hkv, D), generator=gd, device=dev).to(torch.bfloat16)
        q_ = torch.randn((B, Sq, Hq, D), generator=gd, device=dev).to(torch.bfloat16)
        kn = torch.randn((B, Sq, Hkv, D), generator=gd, device=dev).to(torch.bfloat16) if Sq > 1 else None
        vn = torch.randn((B, Sq, Hkv, D), generator=gd, device=dev).to(torch.bfloat16) if Sq > 1 else None
        lens = torch.tensor(lens_l, dtype=torch.int32, device=dev)
        out = torch.empty_like(q_)
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev)
        nb = abi.fa_fwd_kvcache_ex_workspace_size(B, Hq, Hkv, Sq, D, page, cap // page, 0)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        keys = float(sum(lens_l)) + (B * Sq if Sq > 1 else 0)
        nbytes = keys * Hkv * D * 2 * 2 + 2 * q_.numel() * 2 + (2 * 2 * B * Sq * Hkv * D * 2 if Sq > 1 else 0)
        # the appended rows land at the same positions every call (cache_seqlens is not advanced)
        fn = lambda: abi.fa_fwd_kvcache_ex(q_, kc, vc, lens, kn, vn, Sq if Sq > 1 else 0, None, perm, cap // page, nblk,
                                           page, out, lse, B, Hq, Hkv, Sq, D, w_scale(D), 1, -1, -1, 0, ws, nb,
                                           stream)
        name = (f"decode_append4_paged256_B64_Hq32_Hkv8_L1024-2048_D{D}" if Sq > 1
                else f"decode_paged256_B64_Hq32_Hkv8_L1024-2048_D{D}")
    else:
        C, B, S, H, D = 4, 2, 8192, 32, 128
        g = torch.Generator(str(dev)).manual_seed(3)
        o_parts = torch.randn((C, B, S, H, D), generator=g, device=dev).to(torch.bfloat16)
        l_parts = torch.randn((C, B, H, S), generator=g, device=dev)
        o_m = torch.empty((B, S, H, D), dtype=torch.bfloat16, device=dev)
        l_m = torch.empty((B, H, S), dtype=torch.float32, device=dev)
        nbytes = (C + 1) * (o_m.numel() * 2 + l_m.numel() * 4)
        fn = lambda: abi.fa_merge_lse(o_parts, l_parts, C, B, S, H, D, 0, o_m, l_m, 0, stream)
        name = "merge_lse_4parts_B2_S8192_H32_D128"
    for _ in range(args.warmup):
        if fn() != 0:
            raise RuntimeError(f"{name}: the call failed")
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / max(args.steps, 1)
    if args.profile_case.startswith("varlen"):
        print(json.dumps({"profile_case": name, "ms": ms, "tflops": nbytes / ms / 1e9, "algorithmic_flops": nbytes}))
    else:
        print(json.dumps({"profile_case": name, "ms": ms, "gbs": nbytes / ms / 1e6, "algorithmic_bytes": nbytes}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--deterministic", action="store_true",
                    help="time the step with the deterministic backward (dq from the query-tile-stationary pass)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--profile-case", choices=["decode", "merge", "varlen64", "varlen256", "append", "decode256"],
                    default=None,
                    help="run only a mid-size case of one path (inputs > L2, < 1 GB), e.g. under ncu, and print its time")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.profile_case is not None:
        return run_profile_case(args)
    if args.impl == "reference":
        return run_reference(args, rank, world)
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
