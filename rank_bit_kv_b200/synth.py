"""Seeded synthetic inputs shared by the tests and the benchmark.

This module only draws random numbers and lays them out in the cache's
storage format.  It holds none of the method's arithmetic: no projection,
quantization, reconstruction, rotation or attention.  Quantized caches are
drawn directly as integer codes with per-group fp16 scales and zeros (the
"identical seeded integer codes" that both the CUDA path and the oracle read);
tests that want codes produced from Gaussian latents quantize the raw draws
returned by ``gaussian_latents`` with the oracle's quantizer.

Shapes follow the Llama-3.1-8B-class long-context workloads of the pages
(32 query / 8 KV heads, head dim 128, contexts 32K-128K); no dataset is used.
"""

from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------
# workload table
# --------------------------------------------------------------------------

CONFIGS = {
    # tiny single-head check: fp16 latents, no quantization, no RoPE
    "c1": dict(kind="lowrank", B=1, Hq=4, Hkv=1, d=64, T=512, rk=16, rv=24, bits=16,
               g=32, rope=0, resid=0, page=0, seed=0),
    # Llama-3.1-8B-shaped layer at 32K context, INT4 latents, keys pre-RoPE
    "c2": dict(kind="lowrank", B=8, Hq=32, Hkv=8, d=128, T=32768, rk=32, rv=48, bits=4,
               g=32, rope=1, theta=500000.0, resid=0, page=0, seed=1),
    # block-shared latent for 4 layers, symmetric INT4 per 64
    "c3": dict(kind="block_shared", L=4, B=4, Hq=32, Hkv=8, d=128, T=65536, D=512, g=64,
               seed=2),
    # per-token variable rank, ragged records
    "c4": dict(kind="varrate", B=1, Hq=32, Hkv=8, d=128, T=131072, rmax=64, g=32, seed=3,
               ranks=(4, 8, 16, 32, 64), probs=(0.4, 0.25, 0.2, 0.1, 0.05)),
    # low rank + 2-bit Hadamard-rotated residual, 16-token pages, shuffled table
    "c5": dict(kind="lowrank", B=16, Hq=32, Hkv=8, d=128, T=65536, rk=32, rv=64, bits=4,
               g=32, rope=0, resid=2, page=16, seed=4),
}


def config(name, **over):
    c = dict(CONFIGS[name])
    c.update(over)
    return c


# --------------------------------------------------------------------------
# primitive draws
# --------------------------------------------------------------------------


def to_bf16_bits(x):
    """float -> bf16 bit patterns (uint16), round to nearest even."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(u):
    return (np.asarray(u, np.uint16).astype(np.uint32) << 16).view(np.float32)


def orthonormal_rows(rng, r, d):
    """r x d factor with orthonormal rows (QR of an N(0,1) d x r matrix), as fp16."""
    a = rng.standard_normal((d, r))
    qm, _ = np.linalg.qr(a)
    return qm.T.astype(np.float16)


def uniform_codes(rng, shape):
    """Uniform random bytes: every packed INT4 / INT2 code uniform over its range."""
    return rng.integers(0, 256, size=shape, dtype=np.uint8)


def int4_scale_zero(rng, shape):
    """fp16 (scale, zero) pairs [..., 2] spanning roughly the range of an N(0,1)
    group of 32: values code*s + z lie in about [-2.3, 2.5]."""
    s = rng.uniform(0.22, 0.32, size=shape)
    z = rng.uniform(-2.4, -1.6, size=shape)
    return np.stack([s, z], axis=-1).astype(np.float16)


def signs(rng, n):
    return rng.choice(np.array([-1, 1], dtype=np.int8), size=n)


def n_groups(n, g):
    return (n + g - 1) // g


def varrate_record_bytes(r, n_kv_heads, g=32):
    """Bytes of one token's ragged record: per KV head r/2 code bytes then
    ceil(r/g) fp16 (scale, zero) pairs."""
    return n_kv_heads * (r // 2 + 4 * n_groups(r, g))


# --------------------------------------------------------------------------
# low-rank caches (configs c1, c2, c5)
# --------------------------------------------------------------------------


def lowrank_cache(c, T=None, capacity=None, rng=None):
    """Storage arrays of a low-rank cache holding T tokens (slots 0..T-1).

    Returns a dict of numpy arrays in device layout:
      q        uint16 (bf16) [B, Hq, d]
      bk, bv   fp16 [Hkv, r, d]   (orthonormal rows)
      lk_codes / lv_codes : INT4 -> uint8 [rows, r/2]; fp16 latents -> fp16 [rows, r]
      lk_sz / lv_sz       : fp16 [rows, nG, 2] (scale, zero)     (INT4 only)
      rk_codes / rv_codes : uint8 [rows, d/4]; rk_scale / rv_scale fp16 [rows]
      signs_k / signs_v   : int8 [d]
      page_table          : int32 [B, capacity/P]  (paged layouts)
    where rows is B*Hkv*capacity for contiguous layouts ([B, Hkv, capacity])
    and n_pages*Hkv*P for paged ones ([n_pages, Hkv, P]).
    """
    rng = rng or np.random.default_rng(c["seed"])
    T = c["T"] if T is None else T
    cap = capacity or T
    B, Hq, Hkv, d, rk, rv = c["B"], c["Hq"], c["Hkv"], c["d"], c["rk"], c["rv"]
    P = c["page"]
    if P:
        cap = -(-cap // P) * P
    out = {}
    out["q"] = to_bf16_bits(rng.standard_normal((B, Hq, d)))
    if c["bits"] == 16:
        out["lk_codes"] = (rng.standard_normal((B, Hkv, cap, rk)) / np.sqrt(rk)).astype(np.float16)
        out["lv_codes"] = (rng.standard_normal((B, Hkv, cap, rv)) / np.sqrt(rv)).astype(np.float16)
    out["bk"] = np.stack([orthonormal_rows(rng, rk, d) for _ in range(Hkv)])
    out["bv"] = np.stack([orthonormal_rows(rng, rv, d) for _ in range(Hkv)])
    if P:
        n_pages = B * cap // P
        lead = (n_pages, Hkv, P)
        out["page_table"] = rng.permutation(n_pages).astype(np.int32).reshape(B, cap // P)
    else:
        lead = (B, Hkv, cap)
    if c["bits"] == 4:
        out["lk_codes"] = uniform_codes(rng, lead + (rk // 2,))
        out["lk_sz"] = int4_scale_zero(rng, lead + (n_groups(rk, c["g"]),))
        out["lv_codes"] = uniform_codes(rng, lead + (rv // 2,))
        out["lv_sz"] = int4_scale_zero(rng, lead + (n_groups(rv, c["g"]),))
    if c["resid"]:
        out["rk_codes"] = uniform_codes(rng, lead + (d // 4,))
        out["rv_codes"] = uniform_codes(rng, lead + (d // 4,))
        out["rk_scale"] = rng.uniform(0.14, 0.20, size=lead).astype(np.float16)
        out["rv_scale"] = rng.uniform(0.14, 0.20, size=lead).astype(np.float16)
        out["signs_k"] = signs(rng, d)
        out["signs_v"] = signs(rng, d)
    return out


def gaussian_latents(c, T, rng=None):
    """Raw N(0,1) latent draws [B, Hkv, T, r] (float32) for K and V, for tests
    that quantize real Gaussian latents with the oracle's quantizer."""
    rng = rng or np.random.default_rng(c["seed"] + 1000)
    B, Hkv = c["B"], c["Hkv"]
    lk = rng.standard_normal((B, Hkv, T, c["rk"])).astype(np.float32)
    lv = rng.standard_normal((B, Hkv, T, c["rv"])).astype(np.float32)
    return lk, lv


def new_tokens(c, n_new=1, rng=None, n_layers=None):
    """Pre-RoPE keys and values of new tokens, N(0,1) bf16 [B, Hkv, n_new, d]
    (with a leading layer axis when n_layers is given)."""
    rng = rng or np.random.default_rng(c["seed"] + 2000)
    shape = (c["B"], c["Hkv"], n_new, c["d"])
    if n_layers:
        shape = (n_layers,) + shape
    return (to_bf16_bits(rng.standard_normal(shape)),
            to_bf16_bits(rng.standard_normal(shape)))


# --------------------------------------------------------------------------
# dense bf16 cache (baseline on the same library)
# --------------------------------------------------------------------------


def dense_cache(B, Hq, Hkv, d, T, seed, n_layers=1, capacity=None):
    rng = np.random.default_rng(seed)
    cap = capacity or T
    shape = (n_layers, B, Hkv, cap, d) if n_layers > 1 else (B, Hkv, cap, d)
    qshape = (n_layers, B, Hq, d) if n_layers > 1 else (B, Hq, d)
    return dict(q=to_bf16_bits(rng.standard_normal(qshape)),
                k_dense=to_bf16_bits(rng.standard_normal(shape)),
                v_dense=to_bf16_bits(rng.standard_normal(shape)))


# --------------------------------------------------------------------------
# block-shared latent (config c3)
# --------------------------------------------------------------------------


def block_shared_cache(c, T=None, capacity=None, rng=None):
    """q uint16 [L, B, Hq, d]; codes uint8 [B, cap, D * bits / 8]; scales fp16
    [B, cap, D/g] (scaled so that the latent's spread is the same at every
    width); wk, wv fp16 [L, D, Hkv*d] ~ N(0, 1/D); with c['vbits'] > 0 a value
    latent lv_codes / lv_sz at that width."""
    rng = rng or np.random.default_rng(c["seed"])
    T = c["T"] if T is None else T
    cap = capacity or T
    L, B, Hq, Hkv, d, D, g = c["L"], c["B"], c["Hq"], c["Hkv"], c["d"], c["D"], c["g"]
    bits, vbits = c.get("bits", 4), c.get("vbits", 0)
    out = dict(
        q=to_bf16_bits(rng.standard_normal((L, B, Hq, d))),
        wk=(rng.standard_normal((L, D, Hkv * d)) / np.sqrt(D)).astype(np.float16),
        wv=(rng.standard_normal((L, D, Hkv * d)) / np.sqrt(D)).astype(np.float16),
        lk_codes=uniform_codes(rng, (B, cap, D * bits // 8)),
        lk_sz=(rng.uniform(0.30, 0.45, size=(B, cap, D // g)) * 8 / 2 ** (bits - 1)).astype(np.float16),
    )
    if vbits:
        out["lv_codes"] = uniform_codes(rng, (B, cap, D * vbits // 8))
        out["lv_sz"] = (rng.uniform(0.30, 0.45, size=(B, cap, D // g)) * 8 / 2 ** (vbits - 1)).astype(np.float16)
    return out


# --------------------------------------------------------------------------
# variable-rate ragged records (config c4)
# --------------------------------------------------------------------------


def varrate_cache(c, T=None, capacity=None, rng=None, ranks=None):
    """Ragged INT4 records with per-token ranks drawn from c['ranks'] with
    probabilities c['probs'] (independently for K and V; never zero).

    Returns q, bk, bv [Hkv, rmax, d], rank_k / rank_v uint8 [B, cap],
    offset_k / offset_v int32 [B, cap + 1] (byte offsets, offset[0] = 0, only
    the first T + 1 entries meaningful), kstream / vstream uint8 [B, stream_cap].
    """
    rng = rng or np.random.default_rng(c["seed"])
    T = c["T"] if T is None else T
    cap = capacity or T
    B, Hq, Hkv, d, rmax, g = c["B"], c["Hq"], c["Hkv"], c["d"], c["rmax"], c["g"]
    out = dict(q=to_bf16_bits(rng.standard_normal((B, Hq, d))))
    out["bk"] = np.stack([orthonormal_rows(rng, rmax, d) for _ in range(Hkv)])
    out["bv"] = np.stack([orthonormal_rows(rng, rmax, d) for _ in range(Hkv)])
    choices = np.asarray(c["ranks"], dtype=np.int64)
    stream_cap = cap * varrate_record_bytes(rmax, Hkv, g)
    for comp in ("k", "v"):
        if ranks is not None:
            r = np.asarray(ranks[comp], dtype=np.int64)
        else:
            r = rng.choice(choices, size=(B, T), p=np.asarray(c["probs"]))
        rank = np.zeros((B, cap), dtype=np.uint8)
        rank[:, :T] = r
        sizes = np.zeros((B, cap), dtype=np.int64)
        for rv in choices:
            sizes[:, :T][r == rv] = varrate_record_bytes(int(rv), Hkv, g)
        off = np.zeros((B, cap + 1), dtype=np.int64)
        off[:, 1:] = np.cumsum(sizes, axis=1)
        stream = uniform_codes(rng, (B, stream_cap))
        # overwrite every (scale, zero) slot with plausible fp16 values
        for b in range(B):
            for rv in choices:
                tok = np.nonzero(r[b] == rv)[0]
                if tok.size == 0:
                    continue
                rr, ng = int(rv), n_groups(int(rv), g)
                per_head = rr // 2 + 4 * ng
                base = (off[b, tok][:, None] + np.arange(Hkv)[None, :] * per_head + rr // 2)
                idx = base[..., None] + np.arange(4 * ng)
                raw = np.ascontiguousarray(int4_scale_zero(rng, base.shape + (ng,)))
                stream[b, idx.reshape(-1)] = raw.view(np.uint8).reshape(-1)
        out[f"rank_{comp}"] = rank
        out[f"offset_{comp}"] = off.astype(np.int32)
        out[f"{comp}stream"] = stream
    return out


# --------------------------------------------------------------------------
# prefill keys / values and test matrices for the factor fit
# --------------------------------------------------------------------------


def prefill_kv(c, T, rng=None, decay=0.06, noise=0.02):
    """Pre-RoPE keys and values of a prefill, bf16 bits [B, Hkv, T, d]: per KV
    head a random orthonormal basis with an exponentially decaying spectrum
    (component i scaled by exp(-decay * i), as the low effective rank of cached
    keys and values), plus a small isotropic part."""
    rng = rng or np.random.default_rng(c["seed"] + 4000)
    B, Hkv, d = c["B"], c["Hkv"], c["d"]
    out = []
    for _ in range(2):
        x = np.empty((B, Hkv, T, d), np.float32)
        scale = np.exp(-decay * np.arange(d))
        for h in range(Hkv):
            basis, _ = np.linalg.qr(rng.standard_normal((d, d)))
            z = rng.standard_normal((B, T, d)) * scale
            x[:, h] = (z @ basis.T + noise * rng.standard_normal((B, T, d))).astype(np.float32)
        out.append(to_bf16_bits(x))
    return out[0], out[1]


def gaussian_test_matrix(n_heads, d, k, seed):
    """N(0, 1) test matrices [n_heads, d, k] (fp32) of the randomized range finder."""
    return np.random.default_rng(seed).standard_normal((n_heads, d, k)).astype(np.float32)
