#!/usr/bin/env python
"""Decode-step benchmark of the compressed-KV attention library.

Workload (default): the Llama-3.1-8B-shaped layer at 32K context -- batch 8,
32 query / 8 KV heads, head dim 128, 32768 cached tokens per row, per-KV-head
K rank 32 / V rank 48 INT4 latents (groups of 32, fp16 scale + zero), keys
stored pre-RoPE (theta 500000).  One step = one kvc_decode_attn call (the whole
hot path: split-T fused decode + split combine with the up-projection) over
the batch.  Inputs are seeded synthetic codes resident in HBM; consecutive
steps rotate over several cache copies whose total exceeds the 126 MB L2, so
every step streams its compressed bytes from HBM.

Metric: decode step time and achieved HBM GB/s on the compressed bytes the
step must read (value = GB/s, whole job; us_per_step alongside).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvc|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs its own replica of
the workload (the path shards by batch row and KV head with no exchange), and
value = bytes of all ranks / max-over-ranks time.
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

L2_BYTES = 126 * 1024 * 1024
METRIC = "decode step µs & achieved HBM GB/s vs ~8 TB/s, Llama-8B shape, 32K ctx"
WORKLOAD = "c2"
WORKLOAD_NAME = "llama3.1-8b-layer-32k-ctx-int4-lowrank-k32-v48-prerope"
NOMINAL_HBM_GBS = 8000.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="kvc", choices=["kvc", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    return ap.parse_args()


# --------------------------------------------------------------------------- helpers


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def profiled_traffic(version):
    """dram bytes per launch of the hot kernel from the committed ncu summary,
    if it was taken on the current kernel version."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel_version") != version:
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", str(self.gpu_id)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.1)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        os.unlink(self.path)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if "Active" in v and "Not" not in v:
                        reasons.add(n)
            except (ValueError, IndexError):
                pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- workload


def build_workload(torch, kvc, synth, device, n_copies=None, seed_offset=0):
    c = synth.config(WORKLOAD)
    lay = kvc.Layout(kvc.desc_from_config(c))
    a = synth.lowrank_cache(c, rng=np.random.default_rng(c["seed"] + seed_offset))
    step_bytes = lay.step_bytes(c["T"])
    if n_copies is None:
        n_copies = max(2, math.ceil(3 * L2_BYTES / step_bytes) + 1)
    first = kvc.Cache(lay, device=device, fill=a)
    first.n_tokens = c["T"]
    caches = [first]
    for _ in range(n_copies - 1):
        cc = kvc.Cache(lay, device=device)
        for k, t in first.bufs.items():
            cc.bufs[k].copy_(t)
        cc.n_tokens = c["T"]
        caches.append(cc)
    q = torch.from_numpy(a["q"].view(np.int16)).to(device).view(torch.bfloat16)
    return c, lay, caches, q, a


def dense_step(torch, kvc, synth, device, steps, warmup):
    """The same decode step on a dense bf16 cache (same library and GPU)."""
    c = synth.config(WORKLOAD)
    dc = dict(kind="dense", B=c["B"], Hq=c["Hq"], Hkv=c["Hkv"], d=c["d"], T=c["T"])
    lay = kvc.Layout(kvc.desc_from_config(dc))
    cache = kvc.Cache(lay, device=device)
    g = torch.Generator(device=device)
    g.manual_seed(7)
    for k in ("k_dense", "v_dense"):
        cache.bufs[k].view(torch.bfloat16).copy_(
            torch.randn(cache.bufs[k].numel() // 2, device=device, generator=g).to(torch.bfloat16))
    cache.n_tokens = c["T"]
    q = torch.randn(c["B"], c["Hq"], c["d"], device=device, generator=g).to(torch.bfloat16)
    out = torch.empty(q.shape, device=device)
    ws = torch.empty(lay.workspace_bytes(c["T"]), dtype=torch.uint8, device=device)
    for _ in range(warmup):
        kvc.decode(lay, cache, q, out, ws)
    torch.cuda.synchronize()
    n = max(3, min(steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        kvc.decode(lay, cache, q, out, ws)     # 1.07 GB per step: larger than L2
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / n
    byts = lay.step_bytes(c["T"])
    return {"us_per_step": round(us, 2), "bytes_per_step": byts, "GB/s": round(byts / us / 1e3, 1)}


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:
        return 1


def _oracle_unit(a, c, b, h, n_tok):
    """Oracle decode of one (batch row, KV head) unit over its first n_tok tokens."""
    from oracle import kvc_oracle as O

    sub = {n: a[n][[b]][:, [h]] for n in ("lk_codes", "lk_sz", "lv_codes", "lv_sz")}
    sub["q"] = a["q"][[b]][:, h * 4:(h + 1) * 4]
    sub["bk"], sub["bv"] = a["bk"][[h]], a["bv"][[h]]
    return O.decode_from_storage(dict(c, B=1, Hkv=1, Hq=4), sub, n_tok)


def _unit_bytes(c, n_tok):
    from oracle import kvc_oracle as O

    return O.lowrank_bytes_per_token_head(c["rk"], c["rv"], c["bits"], c["g"]) * n_tok


def cpu_oracle_rate(a, c, seconds):
    """Time the fp64 oracle on a bounded sample of the workload: whole
    (batch row, KV head) units at the full context, until `seconds` elapse."""
    done, t0 = 0, time.perf_counter()
    units = [(b, h) for b in range(c["B"]) for h in range(c["Hkv"])]
    while True:
        b, h = units[done % len(units)]
        _oracle_unit(a, c, b, h, c["T"])
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    gbs = done * _unit_bytes(c, c["T"]) / el / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": _oracle_threads(), "kind": "oracle",
            "sample": f"{done} unit decodes cycling over the {len(units)} (batch row, KV head) units at T={c['T']} "
                      f"({done * _unit_bytes(c, c['T'])} compressed bytes) in {el:.1f} s, "
                      f"fp64 numpy"}


# --------------------------------------------------------------------------- arms


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle on the host cores (rank 0 only).
    Each step is a bounded sample of the workload: the first n tokens of one
    (batch row, KV head) unit, n sized so that the whole run stays near two
    minutes; the rate is in the workload's unit (compressed GB/s)."""
    if rank != 0:
        return
    from rank_bit_kv_b200 import synth

    c = synth.config(WORKLOAD)
    a = synth.lowrank_cache(c)
    t0 = time.perf_counter()
    _oracle_unit(a, c, 0, 0, 4096)
    per_tok = (time.perf_counter() - t0) / 4096
    budget = 120.0 / max(1, args.steps + args.warmup)
    n_tok = int(min(c["T"], max(256, budget / per_tok)))
    units = [(b, h) for b in range(c["B"]) for h in range(c["Hkv"])]
    for i in range(args.warmup):
        _oracle_unit(a, c, *units[i % len(units)], n_tok)
    t0 = time.perf_counter()
    for i in range(args.steps):
        _oracle_unit(a, c, *units[i % len(units)], n_tok)
    el = time.perf_counter() - t0
    gbs = args.steps * _unit_bytes(c, n_tok) / el / 1e9
    full_step = _unit_bytes(c, c["T"]) * c["B"] * c["Hkv"]
    us = full_step / (gbs * 1e9) * 1e6
    cb = {"value": round(gbs, 5), "unit": "GB/s", "cores": _oracle_threads(), "kind": "oracle",
          "sample": f"per step: first {n_tok} of {c['T']} tokens of one (batch row, KV head) "
                    f"unit ({_unit_bytes(c, n_tok)} compressed bytes), fp64 numpy"}
    line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 5), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(us / 1e3, 3), "us_per_step": round(us, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(c, "n/a (host)"),
            "cpu_baseline": cb,
            "e2e": {"value": round(gbs, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(torch, dist, value, device):
    """The slowest rank's time: every rank passes its own device-timed value."""
    if not dist:
        return value
    tt = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_rate(world, step_bytes, steps, ms):
    """Whole-job compressed GB/s: the bytes of all ranks' replicas over the
    max-over-ranks time."""
    return world * step_bytes * steps / (ms / 1e3) / 1e9


def workload_config(c, l2):
    return {"workload": WORKLOAD_NAME, "batch": c["B"], "q_heads": c["Hq"], "kv_heads": c["Hkv"],
            "head_dim": c["d"], "context": c["T"], "rank_k": c["rk"], "rank_v": c["rv"],
            "latent_bits": c["bits"], "group": c["g"], "rope_theta": c["theta"],
            "keys": "pre-RoPE", "l2": l2}


def run_kvc(args, rank, world, torch, dist):
    from rank_bit_kv_b200 import kvc, synth

    device = torch.device("cuda", torch.cuda.current_device())
    c, lay, caches, q, a = build_workload(torch, kvc, synth, device, seed_offset=rank)
    T = c["T"]
    step_bytes = lay.step_bytes(T)
    out = torch.empty(q.shape, device=device)
    ws = torch.empty(lay.workspace_bytes(T), dtype=torch.uint8, device=device)
    n = len(caches)
    K, W = args.steps, args.warmup
    launches = lay.decode_launches(T)
    stream = torch.cuda.current_stream()

    for i in range(W):
        kvc.decode(lay, caches[i % n], q, out, ws)
    torch.cuda.synchronize()

    # hot-kernel events, recorded by the library around the split-T kernel
    ev = [(kvc.RawEvent(), kvc.RawEvent()) for _ in range(K)]
    props = torch.cuda.get_device_properties(device)
    sampler = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else
                           torch.cuda.current_device())
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(K):
        kvc.decode(lay, caches[i % n], q, out, ws, events=ev[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1)
    hot_us = statistics.mean(e[0].elapsed_ms(e[1]) for e in ev) * 1e3
    ms = max_over_ranks(torch, dist, ms, device)
    ms_per_step = ms / K
    value = job_rate(world, step_bytes, K, ms)

    # end to end through the C ABI with host buffers: q in, output out, each step
    q_host = q.cpu().pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    q_dev = torch.empty_like(q)
    for i in range(W):
        q_dev.copy_(q_host, non_blocking=True)
        kvc.decode(lay, caches[i % n], q_dev, out, ws)
        out_host.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    t0.record(stream)
    for i in range(K):
        q_dev.copy_(q_host, non_blocking=True)
        kvc.decode(lay, caches[i % n], q_dev, out, ws)
        out_host.copy_(out, non_blocking=True)
    t1.record(stream)
    torch.cuda.synchronize()
    ems = t0.elapsed_time(t1)
    ems = max_over_ranks(torch, dist, ems, device)
    e2e = {"value": round(job_rate(world, step_bytes, K, ems), 1), "unit": "GB/s",
           "us_per_step": round(ems * 1e3 / K, 2),
           "h2d_bytes_per_step": int(q.numel() * q.element_size()),
           "d2h_bytes_per_step": int(out.numel() * out.element_size())}

    dense = None
    if not args.no_dense:
        dense = dense_step(torch, kvc, synth, device, K, 3)

    if rank != 0:
        return
    peak, peak_kind = measured_peaks()
    achieved = step_bytes / (hot_us * 1e-6) / 1e9
    version = kvc.lib().kvc_version().decode()
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} copy bandwidth",
            "traffic": profiled_traffic(version), "kernel": "split-T fused decode",
            "kernel_us": round(hot_us, 2), "bytes_per_launch": step_bytes,
            "frac_of_nominal_8TBps": round(achieved / NOMINAL_HBM_GBS, 4)}
    cpu = None
    if not args.no_cpu_baseline and world >= 1:
        cpu = cpu_oracle_rate(a, c, args.cpu_seconds)
    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": round(ms_per_step, 5),
            "us_per_step": round(ms_per_step * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic",
            "config": workload_config(c, f"{n} rotating cache copies of {step_bytes} B "
                                         f"({n * step_bytes} B > 126 MiB L2)"),
            "bytes_per_step": step_bytes, "gpu_launches": K * launches,
            "kernel_version": version, "clocks": clocks, "roofline": roof, "e2e": e2e,
            "dense_bf16_same_step": dense, "cpu_baseline": cpu}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import torch

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_mod

        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    try:
        run_kvc(args, rank, world, torch, dist)
    finally:
        if dist:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
