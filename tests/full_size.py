"""Oracle outputs of whole batch rows at the full workload sizes, computed in a
process pool so that every row of a full-size decode can be compared.

The pool uses the `spawn` start method (a process forked from one that has a
CUDA context can hang), and each worker rebuilds the seeded synthetic arrays
itself from the workload name and variant instead of receiving gigabytes of
pickled cache, then runs the fp64 oracle on its share of the rows.

Variants:
  uniform   the seeded integer codes of ``synth`` (uniform codes, scales and
            zeros in the range of quantized N(0,1) groups);
  gaussian  codes produced from N(0,1) latents by the oracle's INT4 quantizer
            (the configurations' "values ~N(0,1) before quantization"), and for
            the residual layout 2-bit codes of N(0, 0.1^2) rotated residuals by
            the oracle's 2-bit quantizer.
"""

from __future__ import annotations

import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np

_CACHE = {}


def _quantize_chunked(lat, g, out_codes, out_sz):
    """Quantize [..., T, r] latents in chunks of tokens into packed codes and
    (scale, zero) pairs (the oracle's quantizer; chunking only bounds memory)."""
    from oracle import kvc_oracle as O

    T = lat.shape[-2]
    step = 4096
    for t0 in range(0, T, step):
        sl = lat[..., t0:t0 + step, :]
        codes, s, z = O.quantize_int4_asym(sl, g)
        out_codes[..., t0:t0 + step, :] = O.pack_int4(codes)
        out_sz[..., t0:t0 + step, :, :] = np.stack([s, z], -1).astype(np.float16)


def _to_pages(x, page_table, P):
    """[B, Hkv, T, ...] logical rows -> [n_pages, Hkv, P, ...] physical rows."""
    B, Hkv, T = x.shape[:3]
    n_pages = page_table.size
    out = np.empty((n_pages, Hkv, P) + x.shape[3:], dtype=x.dtype)
    for b in range(B):
        for j in range(T // P):
            out[page_table[b, j]] = x[b, :, j * P:(j + 1) * P]
    return out


def build_arrays(name, variant, over=None):
    """The storage arrays of workload `name` (see module docstring)."""
    from oracle import kvc_oracle as O
    from rank_bit_kv_b200 import synth

    c = synth.config(name, **(over or {}))
    a = synth.lowrank_cache(c)
    if variant == "uniform":
        return c, a
    assert variant == "gaussian", variant
    lk, lv = synth.gaussian_latents(c, c["T"])
    P = c["page"]
    for comp, lat, r in (("lk", lk, c["rk"]), ("lv", lv, c["rv"])):
        codes = np.empty(lat.shape[:-1] + (r // 2,), np.uint8)
        sz = np.empty(lat.shape[:-1] + (O.n_groups(r, c["g"]), 2), np.float16)
        _quantize_chunked(lat, c["g"], codes, sz)
        del lat
        if P:
            codes, sz = _to_pages(codes, a["page_table"], P), _to_pages(sz, a["page_table"], P)
        a[f"{comp}_codes"], a[f"{comp}_sz"] = codes, sz
    del lk, lv
    if c["resid"]:
        rng = np.random.default_rng(c["seed"] + 3000)
        for comp in ("rk", "rv"):
            lead = a[f"{comp}_scale"].shape
            codes = np.empty(lead + (c["d"] // 4,), np.uint8)
            scale = np.empty(lead, np.float16)
            n = lead[0]
            for p0 in range(0, n, 8192):
                y = 0.1 * rng.standard_normal((min(8192, n - p0),) + lead[1:] + (c["d"],))
                cc, ss = O.quantize_resid2(y)
                codes[p0:p0 + len(y)] = O.pack_int2(cc)
                scale[p0:p0 + len(y)] = ss.astype(np.float16)
            a[f"{comp}_codes"], a[f"{comp}_scale"] = codes, scale
    return c, a


def row_arrays(c, a, b):
    """The arrays of batch row b alone (a one-row workload)."""
    sub = dict(a)
    sub["q"] = a["q"][[b]]
    if c["page"]:
        sub["page_table"] = a["page_table"][[b]]
    else:
        for k in ("lk_codes", "lk_sz", "lv_codes", "lv_sz", "rk_codes", "rk_scale",
                  "rv_codes", "rv_scale"):
            if k in a:
                sub[k] = a[k][[b]]
    return sub


def _rows_worker(name, variant, over, rows, threads):
    try:
        from threadpoolctl import threadpool_limits

        threadpool_limits(threads)
    except ImportError:
        pass
    from oracle import kvc_oracle as O

    key = (name, variant, tuple(sorted((over or {}).items())))
    if key not in _CACHE:
        _CACHE.clear()
        _CACHE[key] = build_arrays(name, variant, over)
    c, a = _CACHE[key]
    return {b: O.decode_from_storage(dict(c, B=1), row_arrays(c, a, b), c["T"])[0]
            for b in rows}


def submit_rows(name, variant, rows, over=None, workers=None):
    """Start the oracle on every row in `rows`; returns (executor, futures).
    Collect with `collect`.  Started before the GPU work so that the two overlap."""
    ncpu = os.cpu_count() or 1
    workers = workers or max(1, min(len(rows), ncpu // 4, 8))
    threads = max(1, ncpu // workers)
    chunks = [rows[i::workers] for i in range(workers)]
    ex = cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn"))
    futs = [ex.submit(_rows_worker, name, variant, over, ch, threads) for ch in chunks if ch]
    return ex, futs


def collect(ex, futs):
    out = {}
    try:
        for f in futs:
            out.update(f.result())
    finally:
        ex.shutdown()
    return out
