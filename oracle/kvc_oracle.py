"""Plain fp64 CPU oracle for single-token decode attention over a compressed KV cache.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package's smoke entry and the
CPU-baseline / reference legs of the benchmark import this module.  The library
(its CUDA kernels and C ABI) never calls it, and it imports nothing from the
library: the two share no code, tables or constants.

What is computed, and where it comes from (the five web pages on low-rank and
low-bit KV caches):

* Each KV head stores its keys and values as a token latent L (T x r) times a
  small factor B (r x d): "BELT Connects KV-Cache Compression to Faster
  Long-Context Decoding", section 2 ("Learned rank allocation replaces a
  uniform compression budget") and section 3 (low rank combined with
  quantization).
* The latent is stored as INT4 codes with a per-group scale and offset.  The
  quantizer is the min/max uniform rule of the worked example on the page
  "BellowsKV Architecture: Block-Shared Cache Latents, Outlier-Free Low-Bit
  Storage, and Single-Decision Eviction ..." (section "Worked Example: Why the
  Latent Quantizes Flat"): the range between a group's smallest and largest
  value is cut into 2^bits - 1 equal steps, every value is replaced by its
  nearest step counted from the minimum, ties going to the even step (the
  rounding of the example's language).
* Block-shared latents: one latent per block of n layers, every layer
  reconstructing its own keys and values through its own up-projection; the
  latent is quantized with one scale per group of adjacent coordinates and no
  rotation (same BellowsKV page, sections "Share the Input, Not the Cache" and
  "Three Measurements, Three Operators").
* Keys are stored before RoPE and rotated on reconstruction ("JoLT: Near-Lossless
  KV Cache Compression", section "Key findings": decomposing K after RoPE costs
  extra error, so the method works pre-RoPE).
* A rotated low-bit quantizer stores the truncation residual ("A JoLT for the
  KV cache ...", Abstract).  The rotation is an orthonormal signed Walsh-Hadamard
  transform built with the Sylvester recursion of the BellowsKV worked example.
* Per-token variable rank, no token ever at rank zero ("VarRate: Training-Free
  Variable-Rate KV Cache Compression for Long-Context LLMs", sections
  "Principles" and "Method").
* Attention itself is the textbook single-query softmax attention: the method
  reaches exactly (up to rounding order) the result of dense attention over the
  dequantized, reconstructed cache, so the oracle is that definition written out:
  dequantize -> reconstruct dense K/V -> RoPE -> softmax(q k^T * scale) v.

Readings taken where the pages are silent:
  - scale/zero are fp16; the zero is a float offset (the group minimum), and the
    fp16-rounded scale and zero are the ones used to compute the codes;
  - INT4 packing: element 2i is the low nibble of byte i, 2i+1 the high nibble;
    2-bit packing: element 4i+k sits in bits 2k..2k+1 of byte i;
  - a partial last group is allowed;
  - symmetric block-shared INT4: s = max|x| / 7, code = round(x / s) + 8;
  - 2-bit residual: s = max|y| / 1.5, code = floor(y / s) + 2 clamped to 0..3,
    levels (code - 1.5) * s; residual taken against the dequantized latent;
  - RoPE pairs (i, i + d/2) ("rotate half"), frequencies theta^(-2i/d), key
    position = slot index, no frequency scaling;
  - GQA: query head h reads KV head h // (Hq / Hkv).

Every function works in float64 unless it says otherwise.
"""

from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------


def fp16_rn(x):
    """Round float64 values to the nearest fp16 value (ties to even); return float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def f16_to_f64(a):
    """fp16 storage (np.float16 array) -> float64."""
    return np.asarray(a, dtype=np.float16).astype(np.float64)


def bf16_bits_to_f64(u16):
    """bf16 values given as their uint16 bit patterns -> float64 (exact)."""
    u = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# packing
# ----------------------------------------------------------------------------


def unpack_int4(codes, n):
    """uint8 [..., n/2] -> int64 [..., n]; element 2i = low nibble of byte i."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    out = np.empty(c.shape[:-1] + (2 * c.shape[-1],), dtype=np.int64)
    out[..., 0::2] = c & 0xF
    out[..., 1::2] = c >> 4
    return out[..., :n]


def pack_int4(c):
    """int [..., n] (n even, values 0..15) -> uint8 [..., n/2]."""
    c = np.asarray(c, dtype=np.int64)
    assert c.shape[-1] % 2 == 0
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_int2(codes, n):
    """uint8 [..., n/4] -> int64 [..., n]; element 4i+k = bits 2k..2k+1 of byte i."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    out = np.empty(c.shape[:-1] + (4 * c.shape[-1],), dtype=np.int64)
    for k in range(4):
        out[..., k::4] = (c >> (2 * k)) & 0x3
    return out[..., :n]


def pack_int2(c):
    """int [..., n] (n % 4 == 0, values 0..3) -> uint8 [..., n/4]."""
    c = np.asarray(c, dtype=np.int64)
    assert c.shape[-1] % 4 == 0
    out = np.zeros(c.shape[:-1] + (c.shape[-1] // 4,), dtype=np.int64)
    for k in range(4):
        out |= c[..., k::4] << (2 * k)
    return out.astype(np.uint8)


def n_groups(n, g):
    return (n + g - 1) // g


# ----------------------------------------------------------------------------
# quantizers (BellowsKV page, "Worked Example: Why the Latent Quantizes Flat")
# ----------------------------------------------------------------------------


def quantize_int4_asym(x, g):
    """Group-wise asymmetric INT4 of the last axis.

    Per group of g consecutive values (the last group may be shorter):
      lo, hi = min, max;  z = fp16(lo);  s = fp16((hi - lo) / 15);
      code = clamp(round_half_even((x - z) / s), 0, 15)   (code = 0 when s == 0).
    Returns (codes int64 [..., n], scale f64 [..., nG], zero f64 [..., nG]); the
    scale and zero are exactly representable in fp16.
    """
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    ng = n_groups(n, g)
    codes = np.empty(x.shape, dtype=np.int64)
    s_out = np.empty(x.shape[:-1] + (ng,), dtype=np.float64)
    z_out = np.empty(x.shape[:-1] + (ng,), dtype=np.float64)
    for j in range(ng):
        sl = x[..., j * g : min((j + 1) * g, n)]
        lo = sl.min(axis=-1)
        hi = sl.max(axis=-1)
        z = fp16_rn(lo)
        s = fp16_rn((hi - lo) / 15.0)
        safe = np.where(s > 0, s, 1.0)
        c = np.rint((sl - z[..., None]) / safe[..., None])
        c = np.clip(c, 0, 15)
        c = np.where((s > 0)[..., None], c, 0)
        codes[..., j * g : min((j + 1) * g, n)] = c.astype(np.int64)
        s_out[..., j] = s
        z_out[..., j] = z
    return codes, s_out, z_out


def dequant_int4_asym(codes, scale, zero, g):
    """x_hat = code * s + z with (s, z) of the element's group."""
    c = np.asarray(codes, dtype=np.float64)
    n = c.shape[-1]
    grp = np.arange(n) // g
    return c * np.asarray(scale, np.float64)[..., grp] + np.asarray(zero, np.float64)[..., grp]


def quantize_int4_sym(x, g):
    """Group-wise symmetric INT4 (scale only, no rotation; BellowsKV-Quant).

    Per group: s = fp16(max|x| / 7); code = clamp(round_half_even(x / s), -7, 7) + 8
    (offset binary, code 8 is zero; code = 8 when s == 0).
    """
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    ng = n_groups(n, g)
    codes = np.empty(x.shape, dtype=np.int64)
    s_out = np.empty(x.shape[:-1] + (ng,), dtype=np.float64)
    for j in range(ng):
        sl = x[..., j * g : min((j + 1) * g, n)]
        s = fp16_rn(np.abs(sl).max(axis=-1) / 7.0)
        safe = np.where(s > 0, s, 1.0)
        c = np.clip(np.rint(sl / safe[..., None]), -7, 7) + 8
        c = np.where((s > 0)[..., None], c, 8)
        codes[..., j * g : min((j + 1) * g, n)] = c.astype(np.int64)
        s_out[..., j] = s
    return codes, s_out


def quantize_sym(x, g, bits):
    """Group-wise symmetric quantizer of width `bits` (BellowsKV-Quant at the
    page's other operating points: INT8, INT3 and a 2-bit value latent).

    Per group: s = fp16(max|x| / (2^(bits-1) - 1)); code = clamp(round_half_even
    (x / s), -(2^(bits-1) - 1), 2^(bits-1) - 1) + 2^(bits-1) (offset binary);
    code = 2^(bits-1) when s == 0.  bits = 4 is quantize_int4_sym."""
    x = np.asarray(x, dtype=np.float64)
    qmax, off = 2 ** (bits - 1) - 1, 2 ** (bits - 1)
    n = x.shape[-1]
    ng = n_groups(n, g)
    codes = np.empty(x.shape, dtype=np.int64)
    s_out = np.empty(x.shape[:-1] + (ng,), dtype=np.float64)
    for j in range(ng):
        sl = x[..., j * g : min((j + 1) * g, n)]
        s = fp16_rn(np.abs(sl).max(axis=-1) / qmax)
        safe = np.where(s > 0, s, 1.0)
        c = np.clip(np.rint(sl / safe[..., None]), -qmax, qmax) + off
        c = np.where((s > 0)[..., None], c, off)
        codes[..., j * g : min((j + 1) * g, n)] = c.astype(np.int64)
        s_out[..., j] = s
    return codes, s_out


def dequant_sym(codes, scale, g, bits):
    """x_hat = (code - 2^(bits-1)) * s."""
    c = np.asarray(codes, dtype=np.float64)
    grp = np.arange(c.shape[-1]) // g
    return (c - 2.0 ** (bits - 1)) * np.asarray(scale, np.float64)[..., grp]


def pack_bits(c, bits):
    """Codes [..., n] -> bytes [..., n * bits / 8]: element i in bits
    [bits i, bits i + bits) of the little-endian bit stream (n * bits % 8 == 0)."""
    c = np.asarray(c, dtype=np.int64)
    n = c.shape[-1]
    out = np.zeros(c.shape[:-1] + (n * bits // 8,), dtype=np.uint8)
    for i in range(n):
        for k in range(bits):
            bit = (c[..., i] >> k) & 1
            pos = bits * i + k
            out[..., pos // 8] |= (bit << (pos % 8)).astype(np.uint8)
    return out


def unpack_bits(codes, n, bits):
    """Inverse of pack_bits: bytes [..., n * bits / 8] -> codes [..., n]."""
    b = np.asarray(codes, dtype=np.int64)
    out = np.zeros(b.shape[:-1] + (n,), dtype=np.int64)
    for i in range(n):
        for k in range(bits):
            pos = bits * i + k
            out[..., i] |= ((b[..., pos // 8] >> (pos % 8)) & 1) << k
    return out


def dequant_int4_sym(codes, scale, g):
    """x_hat = (code - 8) * s."""
    c = np.asarray(codes, dtype=np.float64)
    grp = np.arange(c.shape[-1]) // g
    return (c - 8.0) * np.asarray(scale, np.float64)[..., grp]


def quantize_resid2(y):
    """Per-vector 2-bit mid-rise quantizer of the rotated residual.

    s = fp16(max|y| / 1.5); code = clamp(floor(y / s) + 2, 0, 3); levels
    (code - 1.5) * s, i.e. {-1.5, -0.5, 0.5, 1.5} * s.  When s == 0 every code is 2.
    """
    y = np.asarray(y, dtype=np.float64)
    s = fp16_rn(np.abs(y).max(axis=-1) / 1.5)
    safe = np.where(s > 0, s, 1.0)
    c = np.clip(np.floor(y / safe[..., None]) + 2, 0, 3)
    c = np.where((s > 0)[..., None], c, 2)
    return c.astype(np.int64), s


def dequant_resid2(codes, scale):
    """y_hat = (code - 1.5) * s."""
    return (np.asarray(codes, np.float64) - 1.5) * np.asarray(scale, np.float64)[..., None]


# ----------------------------------------------------------------------------
# rotation of the residual: orthonormal signed Walsh-Hadamard
# ----------------------------------------------------------------------------


def sylvester_hadamard(n):
    """H_1 = [1]; H_2m = [[H, H], [H, -H]] (the BellowsKV worked example's recursion)."""
    assert n >= 1 and (n & (n - 1)) == 0
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def residual_rotation(signs):
    """Q = H D / sqrt(n) with D = diag(signs); Q is orthonormal.  y = Q e."""
    signs = np.asarray(signs, dtype=np.float64)
    n = signs.shape[0]
    return sylvester_hadamard(n) * signs[None, :] / math.sqrt(n)


# ----------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------


def rope_rotate_half(x, positions, theta):
    """Rotate x [..., T, d] at integer positions [T]: pairs (i, i + d/2),
    angle = pos * theta^(-2i/d)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    i = np.arange(h, dtype=np.float64)
    omega = float(theta) ** (-2.0 * i / d)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * omega[None, :]
    c, s = np.cos(ang), np.sin(ang)
    lo, hi = x[..., :h], x[..., h:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------


def softmax_attention(q, K, V, scale):
    """Textbook single-query attention.  q [d], K [T, d], V [T, dv].
    Returns (o [dv], p [T])."""
    s = scale * (K @ q)
    p = np.exp(s - s.max())
    p = p / p.sum()
    return p @ V, p


def gqa_decode(q, K, V, scale):
    """q [Hq, d], K [Hkv, T, d], V [Hkv, T, dv] -> o [Hq, dv]; head h reads KV head h // G."""
    hq, hkv = q.shape[0], K.shape[0]
    grp = hq // hkv
    out = np.empty((hq, V.shape[-1]), dtype=np.float64)
    for h in range(hq):
        out[h], _ = softmax_attention(q[h], K[h // grp], V[h // grp], scale)
    return out


# ----------------------------------------------------------------------------
# reconstruction of dense K / V from the stored factors
# ----------------------------------------------------------------------------


def reconstruct_lowrank(lat, factor, resid=None, signs=None):
    """k_t = l_t B  (+ Q^T y_t when a rotated residual is stored).

    lat [T, r], factor [r, d], resid [T, d] (the dequantized rotated residual y_hat).
    """
    k = np.asarray(lat, np.float64) @ np.asarray(factor, np.float64)
    if resid is not None:
        q = residual_rotation(signs)
        k = k + np.asarray(resid, np.float64) @ q  # rows of (Q^T y)^T = y^T Q
    return k


def decode_lowrank(q, lat_k, lat_v, bk, bv, scale, *, rope_theta=None,
                   res_k=None, res_v=None, signs_k=None, signs_v=None):
    """Single-token decode over a low-rank cache given dequantized latents.

    q [B, Hq, d]; lat_k [B, Hkv, T, rK]; lat_v [B, Hkv, T, rV]; bk [Hkv, rK, d];
    bv [Hkv, rV, d]; optional residuals res_k/res_v [B, Hkv, T, d].
    Returns o [B, Hq, d].
    """
    bsz, hkv, T = lat_k.shape[:3]
    out = np.empty((bsz, q.shape[1], bv.shape[-1]), dtype=np.float64)
    for b in range(bsz):
        K = np.empty((hkv, T, bk.shape[-1]))
        V = np.empty((hkv, T, bv.shape[-1]))
        for g in range(hkv):
            K[g] = reconstruct_lowrank(lat_k[b, g], bk[g],
                                       None if res_k is None else res_k[b, g], signs_k)
            V[g] = reconstruct_lowrank(lat_v[b, g], bv[g],
                                       None if res_v is None else res_v[b, g], signs_v)
            if rope_theta is not None:
                K[g] = rope_rotate_half(K[g], np.arange(T), rope_theta)
        out[b] = gqa_decode(q[b], K, V, scale)
    return out


def decode_dense(q, K, V, scale):
    """q [B, Hq, d]; K, V [B, Hkv, T, d] -> [B, Hq, d]."""
    return np.stack([gqa_decode(q[b], K[b], V[b], scale) for b in range(q.shape[0])])


def decode_varrate(q, lat_k, lat_v, rank_k, rank_v, bk, bv, scale):
    """Per-token variable rank.  lat_* [B, Hkv, T, rmax] (entries beyond the
    token's rank are ignored), rank_* [B, T] (every rank >= 1), factors
    [Hkv, rmax, d] truncated to the token's first r rows:
    k_t = lat_t[:r_t] Bk[:r_t]."""
    bsz, hkv, T, _ = lat_k.shape
    d = bk.shape[-1]
    out = np.empty((bsz, q.shape[1], bv.shape[-1]))
    for b in range(bsz):
        rk = np.asarray(rank_k)[b, :T].astype(np.int64)
        rv = np.asarray(rank_v)[b, :T].astype(np.int64)
        assert (rk >= 1).all() and (rv >= 1).all(), "a token is never at rank zero"
        K = np.empty((hkv, T, d))
        V = np.empty((hkv, T, bv.shape[-1]))
        for g in range(hkv):
            for r in np.unique(rk):
                tok = np.nonzero(rk == r)[0]
                K[g, tok] = lat_k[b, g][tok][:, :r] @ bk[g, :r]
            for r in np.unique(rv):
                tok = np.nonzero(rv == r)[0]
                V[g, tok] = lat_v[b, g][tok][:, :r] @ bv[g, :r]
        out[b] = gqa_decode(q[b], K, V, scale)
    return out


def decode_block_shared(q, latent, wk, wv, n_kv_heads, scale, latent_v=None):
    """One latent per block of layers.  q [L, B, Hq, d]; latent [B, T, D];
    wk, wv [L, D, Hkv*d].  Layer l reconstructs K_l = latent W_k^l and
    V_l = latent W_v^l (latent_v W_v^l when a separate value latent is given),
    then runs GQA attention.  Returns [L, B, Hq, d]."""
    lat_v = latent if latent_v is None else latent_v
    nl, bsz, hq, d = q.shape
    out = np.empty((nl, bsz, hq, d))
    for l in range(nl):
        for b in range(bsz):
            K = (latent[b] @ wk[l]).reshape(-1, n_kv_heads, d).transpose(1, 0, 2)
            V = (lat_v[b] @ wv[l]).reshape(-1, n_kv_heads, d).transpose(1, 0, 2)
            out[l, b] = gqa_decode(q[l, b], K, V, scale)
    return out


# ----------------------------------------------------------------------------
# reading the stored formats
# ----------------------------------------------------------------------------


def read_int4_latent(codes, sz, r, g):
    """codes uint8 [..., r/2]; sz fp16 [..., nG, 2] holding (scale, zero) -> f64 [..., r]."""
    sz = f16_to_f64(sz)
    return dequant_int4_asym(unpack_int4(codes, r), sz[..., 0], sz[..., 1], g)


def read_resid2(codes, scale, n=128):
    """codes uint8 [..., n/4]; scale fp16 [...] -> f64 [..., n]."""
    return dequant_resid2(unpack_int2(codes, n), f16_to_f64(scale))


def gather_pages(pool, page_table, n_tokens, page_size):
    """Paged storage: pool [NP, Hkv, P, ...]; page_table [B, >= ceil(T/P)] int ->
    [B, Hkv, T, ...] in logical token order (token t lives in slot t % P of
    physical page page_table[b, t // P])."""
    pool = np.asarray(pool)
    pt = np.asarray(page_table)
    t = np.arange(n_tokens)
    phys = pt[:, t // page_size]                       # [B, T]
    g = pool[phys, :, t[None, :] % page_size]          # [B, T, Hkv, ...]
    return np.moveaxis(g, 2, 1)


def read_varrate_records(stream, offsets, ranks, n_kv_heads, n_tokens, rmax, g):
    """Ragged per-token records.  For batch row b and token t the record is
    stream[b, offsets[b, t] : offsets[b, t + 1]], holding for each KV head in
    turn: r/2 code bytes, then ceil(r/g) (scale, zero) fp16 pairs, r = ranks[b, t].
    Returns dequantized latents [B, Hkv, T, rmax], zero beyond each token's rank.
    (Tokens are handled in groups of equal rank; each group is read the same way.)"""
    stream = np.asarray(stream, dtype=np.uint8)
    offsets = np.asarray(offsets, dtype=np.int64)
    ranks = np.asarray(ranks)[:, :n_tokens].astype(np.int64)
    bsz = stream.shape[0]
    out = np.zeros((bsz, n_kv_heads, n_tokens, rmax))
    for b in range(bsz):
        sizes = offsets[b, 1 : n_tokens + 1] - offsets[b, :n_tokens]
        for r in np.unique(ranks[b]):
            r = int(r)
            ng = n_groups(r, g)
            per_head = r // 2 + 4 * ng
            tok = np.nonzero(ranks[b] == r)[0]
            assert (sizes[tok] == n_kv_heads * per_head).all(), "record length mismatch"
            for h in range(n_kv_heads):
                start = offsets[b, tok] + h * per_head               # [n]
                codes = stream[b][start[:, None] + np.arange(r // 2)]
                szb = stream[b][start[:, None] + r // 2 + np.arange(4 * ng)]
                sz = np.ascontiguousarray(szb).view(np.float16).reshape(len(tok), ng, 2)
                out[b, h, tok, :r] = read_int4_latent(codes, sz, r, g)
    return out


# ----------------------------------------------------------------------------
# append: project one new token onto the latent and quantize it
# ----------------------------------------------------------------------------


def append_lowrank(x, factor, g, *, signs=None):
    """x [..., d] (pre-RoPE key or value), factor [r, d].

    l = x B^T (the coefficients on the factor's rows), quantized group-wise INT4.
    With a rotated residual: e = x - l_hat B (against the dequantized latent),
    y = Q e, 2-bit quantized with one fp16 scale per token.
    Returns dict(codes, scale, zero[, rcodes, rscale]) with unpacked integer codes.
    """
    x = np.asarray(x, np.float64)
    B = np.asarray(factor, np.float64)
    lat = x @ B.T
    codes, s, z = quantize_int4_asym(lat, g)
    out = dict(codes=codes, scale=s, zero=z, lat=lat)
    if signs is not None:
        lhat = dequant_int4_asym(codes, s, z, g)
        e = x - lhat @ B
        y = e @ residual_rotation(signs).T
        rc, rs = quantize_resid2(y)
        out.update(rcodes=rc, rscale=rs, y=y)
    return out


# ----------------------------------------------------------------------------
# byte closed forms (per token and KV head unless stated)
# ----------------------------------------------------------------------------


def latent_bytes(r, bits, g, has_zero=True):
    """Stored bytes for one latent row: codes plus per-group fp16 scale (+ zero)."""
    if bits == 16:
        return 2 * r
    return (r * bits + 7) // 8 + n_groups(r, g) * (2 + (2 if has_zero else 0))


def lowrank_bytes_per_token_head(rk, rv, bits, g, resid_bits=0, d=128):
    b = latent_bytes(rk, bits, g) + latent_bytes(rv, bits, g)
    if resid_bits:
        b += 2 * ((d * resid_bits + 7) // 8 + 2)
    return b


def dense_bytes_per_token(n_layers, n_kv_heads, head_dim, elt_bytes=2):
    """Dense K+V cache bytes per token across all layers."""
    return n_layers * n_kv_heads * head_dim * 2 * elt_bytes


# ----------------------------------------------------------------------------
# decode straight from the storage arrays (the layout the library documents)
# ----------------------------------------------------------------------------


def _scale(desc):
    s = desc.get("scale")
    return float(s) if s else 1.0 / math.sqrt(desc["d"])


def _lowrank_component(arrays, name, desc, n_tokens):
    a = arrays[name]
    if desc.get("page"):
        return gather_pages(a, arrays["page_table"], n_tokens, desc["page"])
    return np.asarray(a)[:, :, :n_tokens]


def decode_from_storage(desc, arrays, n_tokens):
    """Oracle decode of a cache given in the library's storage format.

    desc: dict with kind ('lowrank' | 'varrate' | 'block_shared' | 'dense') and
    the shape fields used by the synthetic generator; arrays: dict of numpy
    arrays as the generator lays them out.  Returns float64 output
    [B, Hq, d] ([L, B, Hq, d] for block_shared / layered dense).
    """
    kind = desc["kind"]
    scale = _scale(desc)
    q = bf16_bits_to_f64(arrays["q"])
    if kind == "lowrank":
        rk, rv, g = desc["rk"], desc["rv"], desc.get("g", 32)
        lk = _lowrank_component(arrays, "lk_codes", desc, n_tokens)
        lv = _lowrank_component(arrays, "lv_codes", desc, n_tokens)
        if desc["bits"] == 16:
            lat_k, lat_v = f16_to_f64(lk), f16_to_f64(lv)
        else:
            lat_k = read_int4_latent(lk, _lowrank_component(arrays, "lk_sz", desc, n_tokens), rk, g)
            lat_v = read_int4_latent(lv, _lowrank_component(arrays, "lv_sz", desc, n_tokens), rv, g)
        res = {}
        if desc.get("resid"):
            for c in ("k", "v"):
                res[c] = read_resid2(_lowrank_component(arrays, f"r{c}_codes", desc, n_tokens),
                                     _lowrank_component(arrays, f"r{c}_scale", desc, n_tokens),
                                     desc["d"])
        return decode_lowrank(
            q, lat_k, lat_v, f16_to_f64(arrays["bk"]), f16_to_f64(arrays["bv"]), scale,
            rope_theta=desc.get("theta") if desc.get("rope") else None,
            res_k=res.get("k"), res_v=res.get("v"),
            signs_k=arrays.get("signs_k"), signs_v=arrays.get("signs_v"))
    if kind == "varrate":
        g, rmax, hkv = desc.get("g", 32), desc["rmax"], desc["Hkv"]
        lat_k = read_varrate_records(arrays["kstream"], arrays["offset_k"], arrays["rank_k"],
                                     hkv, n_tokens, rmax, g)
        lat_v = read_varrate_records(arrays["vstream"], arrays["offset_v"], arrays["rank_v"],
                                     hkv, n_tokens, rmax, g)
        return decode_varrate(q, lat_k, lat_v, arrays["rank_k"], arrays["rank_v"],
                              f16_to_f64(arrays["bk"]), f16_to_f64(arrays["bv"]), scale)
    if kind == "block_shared":
        D, g = desc["D"], desc["g"]
        bits, vbits = desc.get("bits", 4), desc.get("vbits", 0)

        def latent_of(codes_name, sz_name, b):
            codes = unpack_bits(np.asarray(arrays[codes_name])[:, :n_tokens], D, b)
            return dequant_sym(codes, f16_to_f64(np.asarray(arrays[sz_name])[:, :n_tokens]), g, b)

        lat = latent_of("lk_codes", "lk_sz", bits)
        lat_v = latent_of("lv_codes", "lv_sz", vbits) if vbits else None
        wk, wv = f16_to_f64(arrays["wk"]), f16_to_f64(arrays["wv"])
        layer = desc.get("layer", 0)
        if layer:                      # one layer of the block: q [B, Hq, d]
            return decode_block_shared(q[None], lat, wk[layer - 1:layer], wv[layer - 1:layer],
                                       desc["Hkv"], scale, latent_v=lat_v)[0]
        return decode_block_shared(q, lat, wk, wv, desc["Hkv"], scale, latent_v=lat_v)
    if kind == "dense":
        K = bf16_bits_to_f64(arrays["k_dense"])[..., :n_tokens, :]
        V = bf16_bits_to_f64(arrays["v_dense"])[..., :n_tokens, :]
        if q.ndim == 4:
            return np.stack([decode_dense(q[l], K[l], V[l], scale) for l in range(q.shape[0])])
        return decode_dense(q, K, V, scale)
    raise ValueError(kind)
