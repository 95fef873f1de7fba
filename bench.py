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
    ap.add_argument("--no-others", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    return ap.parse_args()


# --------------------------------------------------------------------------- helpers


def measured_peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, which): the driver's measured peaks, else
    the fallback figures of earlier measurements on this hardware."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


def profiled_traffic(version):
    """dram bytes per launch of the hot kernel from the committed ncu summary,
    if it was taken on the revision of that kernel the library reports."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel_revision", "\0") not in version:
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


OTHER_WORKLOADS = {
    "c3": "block-shared latent, 4 layers x 32 q heads, latent 512 INT4/g64 sym, B=4, T=65536",
    "c4": "variable rank per token {4..64}, ragged INT4 records, B=1, T=131072",
    "c5": "low rank K32/V64 INT4 + 2-bit rotated residual, 16-token pages, B=16, T=65536, "
          "one kvc_append of a new token per step then decode",
}


def other_workloads(torch, kvc, synth, device, steps, peak_gbs, peak_tflops):
    """The other configured workloads, each timed the same way: a 512 MiB
    write flushes L2 before every step; CUDA events around the step (for C5
    the append of one new token at slot T-1 of every row, then the decode),
    and in a second pass of as many steps events recorded by the library
    around the split-T kernel; medians over the steps."""
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    n = max(5, min(steps, 20))
    res = {}
    for name, what in OTHER_WORKLOADS.items():
        c = synth.config(name)
        lay = kvc.Layout(kvc.desc_from_config(c))
        fill = (synth.block_shared_cache(c) if name == "c3" else
                synth.varrate_cache(c) if name == "c4" else synth.lowrank_cache(c))
        cache = kvc.Cache(lay, device=device, fill=fill)
        cache.n_tokens = c["T"]
        q = torch.from_numpy(np.ascontiguousarray(fill["q"]).view(np.int16)).to(device).view(
            torch.bfloat16)
        del fill
        out = torch.empty(q.shape, device=device)
        ws = torch.empty(lay.workspace_bytes(c["T"]), dtype=torch.uint8, device=device)
        app = None
        if name == "c5":
            kn, vn = synth.new_tokens(c, 1)
            app = (torch.from_numpy(kn.view(np.int16)).to(device).view(torch.bfloat16),
                   torch.from_numpy(vn.view(np.int16)).to(device).view(torch.bfloat16),
                   torch.full((c["B"],), c["T"] - 1, dtype=torch.int32, device=device))

        def step(ev=None):
            if app is not None:
                kvc.append(lay, cache, app[0], app[1], app[2], 1)
            kvc.decode(lay, cache, q, out, ws, events=ev)

        for _ in range(3):
            step()
        torch.cuda.synchronize()
        evs = [(kvc.RawEvent(), kvc.RawEvent()) for _ in range(n)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        st_us, k_us = [], []
        for i in range(n):              # the step, uninstrumented
            flush.fill_(i & 255)
            e0.record()
            step()
            e1.record()
            torch.cuda.synchronize()
            st_us.append(e0.elapsed_time(e1) * 1e3)
        for i in range(n):              # the split-T kernel, between the library's events
            flush.fill_(i & 255)
            step(evs[i])
            torch.cuda.synchronize()
            k_us.append(evs[i][0].elapsed_ms(evs[i][1]) * 1e3)
        byts = lay.step_bytes(c["T"])
        su, ku = statistics.median(st_us), statistics.median(k_us)
        r = {"what": what, "steps": n, "step_us": round(su, 2), "kernel_us": round(ku, 2),
             "bytes_per_step": byts, "step_GBps": round(byts / su / 1e3, 1),
             "kernel_GBps": round(byts / ku / 1e3, 1),
             "kernel_frac_of_measured_hbm": round(byts / ku / 1e3 / peak_gbs, 4),
             "finite": bool(torch.isfinite(out).all().item()),
             "launches_per_step": lay.decode_launches(c["T"]) + (1 if app is not None else 0)}
        if name == "c3":
            flops = 2 * 2 * c["L"] * c["Hq"] * c["D"] * c["T"] * c["B"]
            r["flops_per_step"] = flops
            r["kernel_TFLOPs"] = round(flops / ku / 1e6, 1)
            r["kernel_frac_of_measured_bf16"] = round(flops / ku / 1e6 / peak_tflops, 4)
            r["bound"] = "tensor"
        else:
            r["bound"] = "hbm"
        res[name] = r
        del cache, q, out, ws, app
        torch.cuda.empty_cache()
    del flush
    torch.cuda.empty_cache()
    return res


def producer_workloads(torch, kvc, synth, device, steps):
    """The steps around decode, timed with CUDA events (L2 flushed before each
    repetition): bulk prefill compression at the Llama-3.1-8B layer's size
    (randomized-SVD factor fit of K and V, then one kvc_append of every prefill
    token), the variable-rate producer at its workload's size (window salience
    of 32 queries per head, ranks by the configured mix), and the joint
    rank / residual-bit allocation (host) over 64 cells."""
    import time as _time

    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    n = max(3, min(steps, 5))
    res = {}

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        fn()
        torch.cuda.synchronize()
        for i in range(n):
            flush.fill_(i & 255)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        return statistics.median(ts)

    # ---- prefill compression, C2 shape (8 rows x 32768 tokens x 8 KV heads)
    c = synth.config("c2")
    # 4096 seeded prefill tokens per row, repeated along the context on the device
    # (the generator's cost stays small; sizes and spectrum are the workload's)
    kb, vb = synth.prefill_kv(c, 4096)
    reps = c["T"] // 4096
    kd = torch.from_numpy(kb.view(np.int16)).to(device).view(torch.bfloat16).repeat(1, 1, reps, 1)
    vd = torch.from_numpy(vb.view(np.int16)).to(device).view(torch.bfloat16).repeat(1, 1, reps, 1)
    del kb, vb
    omk = torch.from_numpy(synth.gaussian_test_matrix(c["Hkv"], 128, 48, 1)).to(device)
    omv = torch.from_numpy(synth.gaussian_test_matrix(c["Hkv"], 128, 64, 2)).to(device)
    lay = kvc.Layout(kvc.desc_from_config(c))
    cache = kvc.Cache(lay, device=device)
    pos = torch.zeros(c["B"], dtype=torch.int32, device=device)

    def fit():
        bk, _ = kvc.fit_factors(kd, omk, c["rk"], 2, with_sigma2=False)
        bv, _ = kvc.fit_factors(vd, omv, c["rv"], 2, with_sigma2=False)
        cache.bufs["bk"].copy_(bk.view(torch.uint8).reshape(-1))
        cache.bufs["bv"].copy_(bv.view(torch.uint8).reshape(-1))

    def app():
        kvc.append(lay, cache, kd, vd, pos, c["T"])

    fit_us = timed(fit)
    app_us = timed(app)
    in_bytes = 2 * kd.numel() * 2
    res["prefill_c2"] = {
        "what": "factor fit (randomized SVD, rank 32 / 48, sketch 48 / 64, 2 power iterations) "
                "of K and V, then kvc_append of all 32768 tokens of 8 rows",
        "fit_us": round(fit_us, 1), "append_us": round(app_us, 1),
        "tokens": c["B"] * c["T"], "bf16_input_bytes": in_bytes,
        "fit_GBps": round(in_bytes / fit_us / 1e3, 1),
        "append_GBps_in": round(in_bytes / app_us / 1e3, 1)}
    del kd, vd, cache
    torch.cuda.empty_cache()

    # ---- variable-rate producer, C4 shape (1 row x 131072 tokens)
    c4 = synth.config("c4")
    kb, _ = synth.prefill_kv(c4, 8192)
    kd = torch.from_numpy(kb.view(np.int16)).to(device).view(torch.bfloat16).repeat(
        1, 1, c4["T"] // 8192, 1)
    del kb
    qw = torch.randn(1, 32, 32, 128, device=device).to(torch.bfloat16)
    T = c4["T"]
    counts = [int(T * f) for f in (0.05, 0.10, 0.20, 0.25)]
    out = {}

    def sal():
        out["s"] = kvc.window_salience(qw, kd)
        out["r"] = kvc.ranks_by_salience(out["s"], [64, 32, 16, 8, 4], counts)

    sal_us = timed(sal)
    res["salience_ranks_c4"] = {
        "what": "window salience (32 query heads x 32 window queries over 131072 keys, "
                "two tensor-core passes) + ranks by the {5,10,20,25,40} % mix",
        "us": round(sal_us, 1), "keys_bytes": kd.numel() * 2,
        "GBps_keys_per_pass": round(2 * kd.numel() * 2 / sal_us / 1e3, 1)}
    del kd
    torch.cuda.empty_cache()

    # ---- joint rank / residual-bit allocation (host), 64 cells x 15 options
    rng = np.random.default_rng(0)
    spectra = np.exp(-rng.uniform(0.02, 0.08, (64, 1)) * np.arange(128)[None])
    opts = [(r, b) for r in (8, 16, 32, 48, 64) for b in (0, 2, 4)]
    t0 = _time.perf_counter()
    B_, D_ = kvc.rank_bit_tables(spectra, np.full(64, 32768 * 8), np.full(64, 8), opts, 128, 0.006,
                                 {0: 1.0, 2: 0.12, 4: 0.01})
    ch, lam = kvc.allocate_rank_bits(B_, D_, B_.min(1).sum() + 0.4 * (B_.max(1).sum() - B_.min(1).sum()))
    res["allocator_host"] = {"cells": 64, "options": len(opts),
                             "us": round((_time.perf_counter() - t0) * 1e6, 1)}
    del flush
    torch.cuda.empty_cache()
    return res


def _oracle_threads():
    """BLAS threads numpy would use (the oracle's matrix products)."""
    try:
        from threadpoolctl import threadpool_info
        return max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:
        return 1


def _cpu_model():
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.startswith("Model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def _oracle_slice(a, c, n_tok):
    """The fp64 oracle on the whole batch (all rows and KV heads) over the first
    n_tok tokens of every row: the workload's step on a shorter context."""
    from oracle import kvc_oracle as O

    return O.decode_from_storage(c, a, n_tok)


def _slice_bytes(c, n_tok):
    from oracle import kvc_oracle as O

    per = O.lowrank_bytes_per_token_head(c["rk"], c["rv"], c["bits"], c["g"])
    return per * n_tok * c["B"] * c["Hkv"]


def _sized_slice(a, c, seconds):
    """Tokens per row such that one whole-batch oracle call takes about
    `seconds` (calibrated on a 1024-token call), a multiple of 256."""
    t0 = time.perf_counter()
    _oracle_slice(a, c, 1024)
    per_tok = (time.perf_counter() - t0) / 1024
    n = int(seconds / max(per_tok, 1e-9)) // 256 * 256
    return int(min(c["T"], max(256, n)))


def _time_slices(a, c, n_tok, seconds):
    done, t0 = 0, time.perf_counter()
    while True:
        _oracle_slice(a, c, n_tok)
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            return done, el


def cpu_oracle_rate(a, c, seconds):
    """The fp64 oracle, as it stands, on a bounded sample of the workload: the
    whole batch (all 64 (row, KV head) units) over the first n tokens of every
    row, repeated for about `seconds`, once with numpy's default threads and
    once limited to one thread."""
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        threadpool_limits = None
    n_tok = _sized_slice(a, c, seconds / 4)
    done, el = _time_slices(a, c, n_tok, seconds / 2)
    gbs = done * _slice_bytes(c, n_tok) / el / 1e9
    one = None
    if threadpool_limits is not None:
        with threadpool_limits(1):
            d1, e1 = _time_slices(a, c, n_tok, seconds / 2)
        one = round(d1 * _slice_bytes(c, n_tok) / e1 / 1e9, 5)
    return {"value": round(gbs, 5), "unit": "GB/s", "cores": _oracle_threads(), "kind": "oracle",
            "value_1_core": one, "host_cpus": os.cpu_count(), "cpu_model": _cpu_model(),
            "sample": f"{done} whole-batch oracle calls over the first {n_tok} of {c['T']} "
                      f"tokens of all {c['B'] * c['Hkv']} (row, KV head) units "
                      f"({_slice_bytes(c, n_tok)} compressed bytes each) in {el:.1f} s, fp64 "
                      f"numpy; the oracle's numpy calls use up to `cores` BLAS threads, "
                      f"value_1_core limits them to one"}


# --------------------------------------------------------------------------- arms


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle, as it stands, on the host cores
    (rank 0 only; other ranks exit without work).  Each step is the whole
    batch -- every (batch row, KV head) unit -- over the first n tokens of
    every row, n sized so that the --warmup + --steps calls end within about
    three minutes (the full 32K context when the host is fast enough).
    ms_per_step is the measured time of that call; value is its compressed
    bytes over that time (GB/s, the workload's unit)."""
    if rank != 0:
        return
    from rank_bit_kv_b200 import synth

    c = synth.config(WORKLOAD)
    a = synth.lowrank_cache(c)
    n_tok = _sized_slice(a, c, 150.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        _oracle_slice(a, c, n_tok)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_slice(a, c, n_tok)
    el = time.perf_counter() - t0
    per_step = _slice_bytes(c, n_tok)
    gbs = args.steps * per_step / el / 1e9
    ms = el / args.steps * 1e3
    cb = {"value": round(gbs, 5), "unit": "GB/s", "cores": _oracle_threads(), "kind": "oracle",
          "host_cpus": os.cpu_count(), "cpu_model": _cpu_model(),
          "sample": f"per step: all {c['B'] * c['Hkv']} (row, KV head) units over the first "
                    f"{n_tok} of {c['T']} tokens of every row ({per_step} compressed bytes), "
                    f"fp64 numpy"}
    line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 5), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "us_per_step": round(ms * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(c),
            "tokens_per_row_per_step": n_tok, "bytes_per_step": per_step,
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


def workload_config(c):
    return {"workload": WORKLOAD_NAME, "batch": c["B"], "q_heads": c["Hq"], "kv_heads": c["Hkv"],
            "head_dim": c["d"], "context": c["T"], "rank_k": c["rk"], "rank_v": c["rv"],
            "latent_bits": c["bits"], "group": c["g"], "rope_theta": c["theta"],
            "keys": "pre-RoPE",
            "l2": "inputs larger than L2: consecutive GPU steps rotate over cache copies "
                  "whose total exceeds the 126 MB L2"}


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
    # the timed steps carry no instrumentation: an event between the split-T
    # kernel and the combine would cost the combine its programmatic early launch
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(K):
        kvc.decode(lay, caches[i % n], q, out, ws)
    t1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    # the hot kernel's duration: K more steps, the library recording events
    # around the split-T kernel of each (same caches, same order)
    torch.cuda.synchronize()
    for i in range(K):
        kvc.decode(lay, caches[i % n], q, out, ws, events=ev[i])
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    hot_us = statistics.mean(e[0].elapsed_ms(e[1]) for e in ev) * 1e3
    ms = max_over_ranks(torch, dist, ms, device)
    ms_per_step = ms / K
    value = job_rate(world, step_bytes, K, ms)

    # end to end through the C ABI with host buffers: every step copies its q in
    # from pinned host memory, decodes, and copies its output out to pinned host
    # memory, one after the other on the decode's stream
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
           "d2h_bytes_per_step": int(out.numel() * out.element_size()),
           "copies": "serial: q in, decode, output out, every step on one stream"}

    # the same copies on a second stream with two device buffers each, as a
    # serving loop would run them: step i + 1's q arrives and step i's output
    # leaves while the neighbouring step decodes (all inside the timed region;
    # the last output is waited for before the end event)
    cs = torch.cuda.Stream(device=device)
    q_hp = [q.cpu().pin_memory() for _ in range(2)]
    out_hp = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    q_dv = [torch.empty_like(q) for _ in range(2)]
    out_dv = [torch.empty_like(out) for _ in range(2)]
    ev_h2d = [torch.cuda.Event() for _ in range(2)]
    ev_dec = [torch.cuda.Event() for _ in range(2)]
    ev_d2h = [torch.cuda.Event() for _ in range(2)]

    def pipelined_steps(steps, start_event=None):
        with torch.cuda.stream(cs):
            if start_event is not None:
                cs.wait_event(start_event)
            q_dv[0].copy_(q_hp[0], non_blocking=True)
            ev_h2d[0].record(cs)
        for i in range(steps):
            k = i & 1
            if i + 1 < steps:   # the next q; its buffer's last reader (decode i - 1) precedes on cs
                with torch.cuda.stream(cs):
                    q_dv[k ^ 1].copy_(q_hp[k ^ 1], non_blocking=True)
                    ev_h2d[k ^ 1].record(cs)
            stream.wait_event(ev_h2d[k])
            if i >= 2:
                stream.wait_event(ev_d2h[k])   # out_dv[k] copied out by step i - 2
            kvc.decode(lay, caches[i % n], q_dv[k], out_dv[k], ws)
            ev_dec[k].record(stream)
            with torch.cuda.stream(cs):
                cs.wait_event(ev_dec[k])
                out_hp[k].copy_(out_dv[k], non_blocking=True)
                ev_d2h[k].record(cs)
        for k in range(min(steps, 2)):
            stream.wait_event(ev_d2h[k])

    pipelined_steps(W)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    t0.record(stream)
    pipelined_steps(K, t0)
    t1.record(stream)
    torch.cuda.synchronize()
    pms = max_over_ranks(torch, dist, t0.elapsed_time(t1), device)
    e2e_pipelined = {"value": round(job_rate(world, step_bytes, K, pms), 1), "unit": "GB/s",
                     "us_per_step": round(pms * 1e3 / K, 2),
                     "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                     "d2h_bytes_per_step": e2e["d2h_bytes_per_step"],
                     "copies": "a second stream, two device buffers each: step i+1's q in and "
                               "step i's output out overlap the neighbouring decodes"}

    dense = None
    if not args.no_dense:
        dense = dense_step(torch, kvc, synth, device, K, 3)
    others = None
    if not args.no_others:
        others = other_workloads(torch, kvc, synth, device, K, measured_peaks()[0],
                                 measured_peaks()[1])
        others.update(producer_workloads(torch, kvc, synth, device, K))

    if rank != 0:
        return
    peak, peak_tf, peak_kind = measured_peaks()
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
            "scaling": "weak", "vs_baseline": None, "dtype": "f16 operands, f32 accumulate",
            "data": "synthetic",
            "config": workload_config(c),
            "cache_copies": {"n": n, "bytes_each": step_bytes, "total": n * step_bytes},
            "bytes_per_step": step_bytes, "gpu_launches": K * launches,
            "kernel_version": version, "clocks": clocks, "roofline": roof, "e2e": e2e,
            "e2e_pipelined": e2e_pipelined,
            "dense_bf16_same_step": dense, "workloads": others, "cpu_baseline": cpu}
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
