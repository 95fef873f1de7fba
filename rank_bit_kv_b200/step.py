"""Run (and time) the decode step of a named synthetic workload.

    python -m rank_bit_kv_b200.step c5 [--batch B] [--steps N] [--time] [--append]

Builds the seeded synthetic cache of the workload (optionally with a smaller
batch), then calls kvc_decode_attn N times on the current CUDA device.  With
--time it flushes L2 (a 512 MiB write) before every call and prints medians
over the calls, from CUDA events: the whole step (query projection, split-T
kernel, combine) timed without instrumentation, then, in a second pass with
the library recording events around the split-T kernel, that kernel and the
parts of the instrumented step before and after it; with the compressed bytes
the step reads.  Without --time it only runs the calls (the form used under a
profiler).
With --append (low-rank layouts) every step first appends one new token to
slot T - 1 of every row with kvc_append, as the C5 workload's step does.
"""

from __future__ import annotations

import argparse
import json
import statistics


def _cache(kvc, synth, c):
    lay = kvc.Layout(kvc.desc_from_config(c))
    if c["kind"] == "varrate":
        fill = synth.varrate_cache(c)
    elif c["kind"] == "block_shared":
        fill = synth.block_shared_cache(c)
    else:
        fill = synth.lowrank_cache(c)
    cache = kvc.Cache(lay, fill=fill)
    cache.n_tokens = c["T"]
    return lay, cache, fill


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("config", choices=["c1", "c2", "c3", "c4", "c5"])
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--time", action="store_true")
    ap.add_argument("--rope-kernel", type=int, default=0,
                    help="pre-RoPE layouts: 0 / 1 warp-level mma.sync kernel, 2 tcgen05 warpgroup kernel")
    ap.add_argument("--append", action="store_true",
                    help="low-rank layouts: one kvc_append of a new token per step")
    ap.add_argument("--varrate-kernel", type=int, default=0,
                    help="variable-rate layout: 0 lane-per-head kernel, 1 tensor-core kernel")
    args = ap.parse_args(argv)

    import numpy as np
    import torch

    from rank_bit_kv_b200 import kvc, synth

    over = {} if args.batch is None else {"B": args.batch}
    kvc.lib().kvc_select_rope_kernel(args.rope_kernel)
    kvc.lib().kvc_select_varrate_kernel(args.varrate_kernel)
    c = synth.config(args.config, **over)
    lay, cache, fill = _cache(kvc, synth, c)
    q = torch.from_numpy(np.ascontiguousarray(fill["q"]).view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty(q.shape, device="cuda")
    ws = torch.zeros(lay.workspace_bytes(c["T"]), dtype=torch.uint8, device="cuda")
    app = None
    if args.append and c["kind"] == "lowrank":
        kn, vn = synth.new_tokens(c, 1)
        app = (torch.from_numpy(kn.view(np.int16)).cuda().view(torch.bfloat16),
               torch.from_numpy(vn.view(np.int16)).cuda().view(torch.bfloat16),
               torch.full((c["B"],), c["T"] - 1, dtype=torch.int32, device="cuda"))

    def step(events=None):
        if app is not None:
            kvc.append(lay, cache, app[0], app[1], app[2], 1)
        kvc.decode(lay, cache, q, out, ws, events=events)

    if not args.time:
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize()
        print(json.dumps({"config": args.config, "batch": c["B"], "steps": args.steps,
                          "finite": bool(torch.isfinite(out).all().item()),
                          "err_word": int(ws[:4].view(torch.int32).item())}))
        return
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    step_us, kern_us, pre_us, post_us = [], [], [], []
    for _ in range(args.steps):         # the step, uninstrumented
        flush.zero_()
        e0, e1 = kvc.RawEvent(), kvc.RawEvent()
        e0.record()
        step()
        e1.record()
        torch.cuda.synchronize()
        step_us.append(e0.elapsed_ms(e1) * 1e3)
    for _ in range(args.steps):         # the split-T kernel between the library's events
        flush.zero_()
        ev = (kvc.RawEvent(), kvc.RawEvent())
        e0, e1 = kvc.RawEvent(), kvc.RawEvent()
        e0.record()
        step(ev)
        e1.record()
        torch.cuda.synchronize()
        kern_us.append(ev[0].elapsed_ms(ev[1]) * 1e3)
        pre_us.append(e0.elapsed_ms(ev[0]) * 1e3)
        post_us.append(ev[1].elapsed_ms(e1) * 1e3)
    nbytes = lay.step_bytes(c["T"])
    st, kt = statistics.median(step_us), statistics.median(kern_us)
    print(json.dumps({"config": args.config, "batch": c["B"], "context": c["T"],
                      "bytes_per_step": nbytes, "step_us": round(st, 2),
                      "split_kernel_us": round(kt, 2), "step_gbs": round(nbytes / st / 1e3, 1),
                      "before_split_us": round(statistics.median(pre_us), 2),
                      "after_split_us": round(statistics.median(post_us), 2),
                      "split_kernel_gbs": round(nbytes / kt / 1e3, 1),
                      "finite": bool(torch.isfinite(out).all().item()),
                      "err_word": int(ws[:4].view(torch.int32).item()),
                      "kernel_version": kvc.lib().kvc_version().decode()}))


if __name__ == "__main__":
    main()
