"""Pins of the fp64 oracle against things other than itself: library routines,
closed forms, printed numbers of the pages, invariants and brute force.

Every function of the oracle used by the parity tests is checked here so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand)
fails at least one test.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import kvc_oracle as O
from rank_bit_kv_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sdpa(q, K, V, scale):
    """Independent dense attention: torch's scaled_dot_product_attention in fp64."""
    qt = torch.tensor(q).reshape(1, 1, 1, -1)
    kt = torch.tensor(K)[None, None]
    vt = torch.tensor(V)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return o.reshape(-1).numpy()


def gqa_sdpa(q, K, V, scale):
    hq, hkv = q.shape[0], K.shape[0]
    return np.stack([sdpa(q[h], K[h // (hq // hkv)], V[h // (hq // hkv)], scale) for h in range(hq)])


def rand_orthogonal(rng, n):
    qm, r = np.linalg.qr(rng.standard_normal((n, n)))
    return qm * np.sign(np.diag(r))[None, :]


# ---------------------------------------------------------------- attention


@pytest.mark.parametrize("T", [1, 7, 64])
def test_full_rank_no_quant_equals_dense_attention(T):
    """Full rank and no quantization: the low-rank decode is plain dense attention."""
    rng = np.random.default_rng(10 + T)
    B, Hq, Hkv, d = 2, 4, 2, 64
    q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, Hkv, T, d))
    V = rng.standard_normal((B, Hkv, T, d))
    bk = np.stack([rand_orthogonal(rng, d) for _ in range(Hkv)])
    bv = np.stack([rand_orthogonal(rng, d) for _ in range(Hkv)])
    lat_k = np.einsum("bgtd,grd->bgtr", K, bk)       # L = K B^T (B orthogonal)
    lat_v = np.einsum("bgtd,grd->bgtr", V, bv)
    scale = 1 / math.sqrt(d)
    o = O.decode_lowrank(q, lat_k, lat_v, bk, bv, scale)
    ref = np.stack([gqa_sdpa(q[b], K[b], V[b], scale) for b in range(B)])
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_constant_values_give_constant_output():
    rng = np.random.default_rng(1)
    B, Hq, Hkv, d, T, rk, rv = 1, 4, 1, 128, 50, 8, 12
    lat_v = np.repeat(rng.standard_normal((B, Hkv, 1, rv)), T, axis=2)
    bv = rng.standard_normal((Hkv, rv, d))
    o = O.decode_lowrank(rng.standard_normal((B, Hq, d)) * 5, rng.standard_normal((B, Hkv, T, rk)),
                         lat_v, rng.standard_normal((Hkv, rk, d)), bv, 0.3, rope_theta=500000.0)
    v = lat_v[0, 0, 0] @ bv[0]
    for h in range(Hq):
        np.testing.assert_allclose(o[0, h], v, rtol=0, atol=1e-12)


def test_weights_sum_to_one_and_nonnegative():
    rng = np.random.default_rng(2)
    for T in (1, 3, 1000):
        _, p = O.softmax_attention(rng.standard_normal(16) * 10, rng.standard_normal((T, 16)),
                                   rng.standard_normal((T, 3)), 0.25)
        assert abs(p.sum() - 1) < 1e-12 and (p >= 0).all()


def test_single_token_returns_its_value():
    rng = np.random.default_rng(3)
    V = rng.standard_normal((1, 5))
    o, p = O.softmax_attention(rng.standard_normal(8), rng.standard_normal((1, 8)), V, 1.0)
    np.testing.assert_array_equal(o, V[0])
    assert p[0] == 1.0


def test_identical_keys_average_values():
    rng = np.random.default_rng(4)
    K = np.repeat(rng.standard_normal((1, 8)), 9, axis=0)
    V = rng.standard_normal((9, 3))
    o, p = O.softmax_attention(rng.standard_normal(8), K, V, 0.7)
    np.testing.assert_allclose(p, np.full(9, 1 / 9), rtol=0, atol=1e-15)
    np.testing.assert_allclose(o, V.mean(0), rtol=0, atol=1e-12)


def test_needle_selects_its_value():
    rng = np.random.default_rng(5)
    d, T, j = 16, 200, 117
    q = rng.standard_normal(d)
    K = rng.standard_normal((T, d)) * 0.1
    K[j] = q * 60 / (q @ q)        # scale * (q.k_j - max other) >= 40
    V = rng.standard_normal((T, 4))
    o, _ = O.softmax_attention(q, K, V, 1.0)
    np.testing.assert_allclose(o, V[j], rtol=1e-12, atol=1e-12)


def test_gqa_head_mapping():
    """Head h must read KV head h // G (consecutive grouping)."""
    rng = np.random.default_rng(6)
    q = rng.standard_normal((8, 4))
    K = rng.standard_normal((2, 5, 4))
    V = np.stack([np.zeros((5, 1)), np.ones((5, 1))])   # KV head 0 -> 0, head 1 -> 1
    o = O.gqa_decode(q, K, V, 1.0)
    np.testing.assert_allclose(o[:, 0], [0, 0, 0, 0, 1, 1, 1, 1], rtol=0, atol=1e-15)


# ---------------------------------------------------------------- RoPE


def test_rope_position_zero_is_identity_and_norm_preserving():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 128))
    np.testing.assert_array_equal(O.rope_rotate_half(x[:1], [0], 500000.0), x[:1])
    y = O.rope_rotate_half(x, np.arange(5) * 1000 + 3, 500000.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


def test_rope_matches_complex_rotation():
    """Independent formulation: pair (i, i+64) as the complex number x_i + 1j x_{i+64}
    multiplied by exp(1j * pos * theta^(-2i/d))."""
    rng = np.random.default_rng(8)
    d, theta = 128, 500000.0
    x = rng.standard_normal((6, d))
    pos = np.array([0, 1, 17, 4095, 32767, 131071])
    z = x[:, : d // 2] + 1j * x[:, d // 2 :]
    w = np.exp(1j * np.outer(pos, [theta ** (-2 * i / d) for i in range(d // 2)]))
    zr = z * w
    ref = np.concatenate([zr.real, zr.imag], axis=1)
    # fp64 angle rounding at position 131071 is ~1e-11 rad, hence 1e-10
    np.testing.assert_allclose(O.rope_rotate_half(x, pos, theta), ref, rtol=0, atol=1e-10)


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(9)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for m, n, delta in [(5, 100, 1000), (0, 31, 20000)]:
        a = O.rope_rotate_half(q[None], [m], 5e5)[0] @ O.rope_rotate_half(k[None], [n], 5e5)[0]
        b = (O.rope_rotate_half(q[None], [m + delta], 5e5)[0]
             @ O.rope_rotate_half(k[None], [n + delta], 5e5)[0])
        assert abs(a - b) < 1e-10


# ---------------------------------------------------------------- Hadamard residual


def test_sylvester_matches_scipy_and_is_orthogonal():
    for n in (1, 2, 16, 128):
        h = O.sylvester_hadamard(n)
        np.testing.assert_array_equal(h, scipy.linalg.hadamard(n))
        np.testing.assert_array_equal(h @ h.T, n * np.eye(n))


def test_residual_rotation_orthonormal_and_basis_image():
    rng = np.random.default_rng(11)
    s = synth.signs(rng, 128)
    Q = O.residual_rotation(s)
    np.testing.assert_allclose(Q @ Q.T, np.eye(128), atol=1e-14)
    e0 = np.zeros(128)
    e0[0] = 1
    np.testing.assert_allclose(Q @ e0, np.full(128, s[0] / math.sqrt(128)), atol=1e-15)


def test_residual_reconstruction_adds_rotated_back_residual():
    """k = l B + Q^T y: with y = Q e exactly, the residual term restores e."""
    rng = np.random.default_rng(12)
    s = synth.signs(rng, 128)
    Q = scipy.linalg.hadamard(128) * s[None, :] / math.sqrt(128)   # built independently
    lat, B = rng.standard_normal((3, 8)), rng.standard_normal((8, 128))
    e = rng.standard_normal((3, 128))
    y = e @ Q.T
    np.testing.assert_allclose(O.reconstruct_lowrank(lat, B, y, s), lat @ B + e, atol=1e-12)


def test_residual_off_equals_plain_lowrank():
    rng = np.random.default_rng(13)
    B, Hq, Hkv, d, T = 1, 8, 2, 128, 33
    args = (rng.standard_normal((B, Hq, d)), rng.standard_normal((B, Hkv, T, 4)),
            rng.standard_normal((B, Hkv, T, 6)), rng.standard_normal((Hkv, 4, d)),
            rng.standard_normal((Hkv, 6, d)), 0.1)
    z = np.zeros((B, Hkv, T, d))
    sg = synth.signs(rng, d)
    np.testing.assert_array_equal(
        O.decode_lowrank(*args, res_k=z, res_v=z, signs_k=sg, signs_v=sg), O.decode_lowrank(*args))


# ---------------------------------------------------------------- quantizers


def test_int4_asym_matches_page_formula_on_fp16_exact_groups():
    """When lo and (hi-lo)/15 are already fp16 values the codes and the
    dequantized values are exactly the worked example's rule (BellowsKV page,
    "Worked Example: Why the Latent Quantizes Flat"): the nearest of the
    fifteen equal steps above the minimum, ties to the even step -- evaluated
    here in exact rational arithmetic, independently of the oracle's floats."""
    from fractions import Fraction
    rng = np.random.default_rng(14)
    for _ in range(200):
        lo = float(np.float16(rng.uniform(-3, 0)))
        s = float(np.float16(rng.uniform(0.01, 0.5)))
        hi = lo + 15 * s
        if float(np.float16((hi - lo) / 15)) != s:
            continue
        x = np.concatenate([[lo, hi], rng.uniform(lo, hi, 30)])
        codes, sc, zc = O.quantize_int4_asym(x, 32)
        assert sc[0] == s and zc[0] == lo
        steps = [round(Fraction(v) / Fraction(s) - Fraction(lo) / Fraction(s)) for v in x]
        page = [float(Fraction(lo) + k * Fraction(s)) for k in steps]
        np.testing.assert_array_equal(codes * s + lo, page)
        np.testing.assert_array_equal(O.dequant_int4_asym(codes, sc, zc, 32), page)
        assert codes[0] == 0 and codes[1] == 15


def test_int4_asym_rounds_half_to_even_and_bounds_error():
    x = np.array([0.0, 15.0, 2.5, 3.5, 4.5, 7.0])       # lo = 0, s = 1 exactly
    codes, s, z = O.quantize_int4_asym(x, 32)
    np.testing.assert_array_equal(codes, [0, 15, 2, 4, 4, 7])
    rng = np.random.default_rng(15)
    x = rng.standard_normal((100, 48))
    codes, s, z = O.quantize_int4_asym(x, 32)            # groups of 32 + 16 (partial)
    assert s.shape == (100, 2) and codes.min() >= 0 and codes.max() <= 15
    xh = O.dequant_int4_asym(codes, s, z, 32)
    grp = np.arange(48) // 32
    err = np.abs(x - xh)
    # half a step, plus the fp16 rounding of z and of the step count
    bound = s[:, grp] / 2 + np.abs(z[:, grp]) * 2 ** -11 + 15 * s[:, grp] * 2 ** -11 + 1e-12
    assert (err <= bound).all()


def test_int4_sym_offset_binary():
    x = np.array([-7.0, 7.0, 0.0, 3.49, -3.5, 1.5] + [0.0] * 58)
    codes, s = O.quantize_int4_sym(x, 64)
    assert s[0] == 1.0
    np.testing.assert_array_equal(codes[:6], [1, 15, 8, 11, 4, 10])
    np.testing.assert_array_equal(O.dequant_int4_sym(codes, s, 64)[:6], [-7, 7, 0, 3, -4, 2])
    codes, s = O.quantize_int4_sym(np.zeros(64), 64)
    assert s[0] == 0 and (codes == 8).all()


def test_resid2_levels_and_boundaries():
    y = np.array([-1.5, -1.0, -0.999, -0.2, 0.0, 0.2, 0.999, 1.0, 1.5, 0.7])
    c, s = O.quantize_resid2(y)
    assert s == 1.0
    np.testing.assert_array_equal(c, [0, 1, 1, 1, 2, 2, 2, 3, 3, 2])
    np.testing.assert_array_equal(O.dequant_resid2(c, s), [-1.5, -.5, -.5, -.5, .5, .5, .5, 1.5, 1.5, .5])
    c, s = O.quantize_resid2(np.zeros(128))
    assert s == 0 and (c == 2).all()


def test_packing_byte_layout():
    np.testing.assert_array_equal(O.unpack_int4(np.array([0x3A, 0xF0], np.uint8), 4), [0xA, 0x3, 0, 0xF])
    np.testing.assert_array_equal(O.unpack_int2(np.array([0b11100100], np.uint8), 4), [0, 1, 2, 3])
    rng = np.random.default_rng(16)
    c4 = rng.integers(0, 16, (5, 48))
    c2 = rng.integers(0, 4, (5, 128))
    np.testing.assert_array_equal(O.unpack_int4(O.pack_int4(c4), 48), c4)
    np.testing.assert_array_equal(O.unpack_int2(O.pack_int2(c2), 128), c2)


def test_append_projection_and_residual_target():
    """Append: l = x B^T; the residual is taken against the dequantized latent."""
    rng = np.random.default_rng(17)
    B = synth.orthonormal_rows(rng, 32, 128).astype(np.float64)
    x = rng.standard_normal(128)
    sg = synth.signs(rng, 128)
    r = O.append_lowrank(x, B, 32, signs=sg)
    np.testing.assert_allclose(r["lat"], np.einsum("rd,d->r", B, x), atol=1e-12)
    lhat = r["codes"] * r["scale"][0] + r["zero"][0]
    Q = scipy.linalg.hadamard(128) * sg[None, :] / math.sqrt(128)
    np.testing.assert_allclose(r["y"], Q @ (x - lhat @ B), atol=1e-12)


# ---------------------------------------------------------------- layouts


def test_varrate_full_rank_equals_uniform_and_truncation_is_zero_padding():
    rng = np.random.default_rng(18)
    B, Hq, Hkv, d, T, rmax = 1, 8, 2, 32, 20, 16
    q = rng.standard_normal((B, Hq, d))
    lk, lv = rng.standard_normal((B, Hkv, T, rmax)), rng.standard_normal((B, Hkv, T, rmax))
    bk, bv = rng.standard_normal((Hkv, rmax, d)), rng.standard_normal((Hkv, rmax, d))
    full = np.full((B, T), rmax)
    np.testing.assert_allclose(O.decode_varrate(q, lk, lv, full, full, bk, bv, 0.2),
                               O.decode_lowrank(q, lk, lv, bk, bv, 0.2), atol=1e-12)
    rk = rng.choice([4, 8, 16], (B, T))
    rv = rng.choice([4, 8, 16], (B, T))
    mk = np.arange(rmax)[None, None, None, :] < rk[:, None, :, None]
    mv = np.arange(rmax)[None, None, None, :] < rv[:, None, :, None]
    np.testing.assert_allclose(O.decode_varrate(q, lk, lv, rk, rv, bk, bv, 0.2),
                               O.decode_lowrank(q, lk * mk, lv * mv, bk, bv, 0.2), atol=1e-12)


def test_varrate_record_parsing_round_trip():
    c = synth.config("c4", B=2, Hkv=2, Hq=4, d=32, T=40, rmax=64)
    a = synth.varrate_cache(c)
    lat = O.read_varrate_records(a["kstream"], a["offset_k"], a["rank_k"], 2, 40, 64, 32)
    b, t, h = 1, 17, 1
    r = int(a["rank_k"][b, t])
    per_head = r // 2 + 4 * ((r + 31) // 32)
    pos = int(a["offset_k"][b, t]) + h * per_head
    codes = a["kstream"][b, pos:pos + r // 2]
    sz = a["kstream"][b, pos + r // 2:pos + per_head].view(np.float16).astype(np.float64)
    manual = [((codes[i // 2] >> (4 * (i % 2))) & 15) * sz[2 * (i // 32)] + sz[2 * (i // 32) + 1]
              for i in range(r)]
    np.testing.assert_array_equal(lat[b, h, t, :r], manual)
    assert (lat[b, h, t, r:] == 0).all()
    sizes = np.diff(a["offset_k"][:, :41].astype(np.int64), axis=1)
    expect = np.vectorize(lambda rr: 2 * (rr // 2 + 4 * ((rr + 31) // 32)))(a["rank_k"][:, :40])
    np.testing.assert_array_equal(sizes, expect)


def test_paging_permutation_invariance():
    c = synth.config("c5", B=2, Hkv=2, Hq=8, T=64)
    a = synth.lowrank_cache(c)
    desc = dict(c, kind="lowrank")
    o1 = O.decode_from_storage(desc, a, 64)
    # move every page to a new physical slot, permuting the table the same way
    rng = np.random.default_rng(19)
    perm = rng.permutation(a["lk_codes"].shape[0])
    inv = np.argsort(perm)
    b = dict(a)
    for k in ("lk_codes", "lk_sz", "lv_codes", "lv_sz", "rk_codes", "rv_codes", "rk_scale", "rv_scale"):
        b[k] = a[k][perm]
    b["page_table"] = inv[a["page_table"]].astype(np.int32)
    np.testing.assert_array_equal(O.decode_from_storage(desc, b, 64), o1)


def test_block_shared_equals_per_layer_dense_attention():
    c = synth.config("c3", L=2, B=2, Hq=8, Hkv=2, d=16, D=32, g=16, T=24)
    a = synth.block_shared_cache(c)
    desc = dict(c, kind="block_shared")
    o = O.decode_from_storage(desc, a, 24)
    codes = np.stack([(a["lk_codes"] & 15), a["lk_codes"] >> 4], -1).reshape(2, 24, 32).astype(float)
    lat = (codes - 8) * np.repeat(a["lk_sz"].astype(np.float64), 16, axis=-1)
    q = synth.bf16_bits_to_f32(a["q"]).astype(np.float64)
    for l in range(2):
        for b in range(2):
            K = (lat[b] @ a["wk"][l].astype(np.float64)).reshape(24, 2, 16).transpose(1, 0, 2)
            V = (lat[b] @ a["wv"][l].astype(np.float64)).reshape(24, 2, 16).transpose(1, 0, 2)
            np.testing.assert_allclose(o[l, b], gqa_sdpa(q[l, b], K, V, 0.25), atol=1e-12)


def test_lowrank_storage_decode_matches_sdpa_brute_force():
    """Storage path (INT4 + residual + pages + RoPE) against explicit loops and SDPA."""
    c = synth.config("c5", B=1, Hkv=2, Hq=4, T=32, rope=1, theta=500000.0)
    a = synth.lowrank_cache(c)
    desc = dict(c, kind="lowrank")
    o = O.decode_from_storage(desc, a, 32)
    d = 128
    Q = scipy.linalg.hadamard(d)
    q = synth.bf16_bits_to_f32(a["q"]).astype(np.float64)
    for g in range(2):
        K = np.zeros((32, d))
        V = np.zeros((32, d))
        for t in range(32):
            pg, sl = a["page_table"][0, t // 16], t % 16
            for comp, out, fac, r, sg in (("k", K, a["bk"], 32, a["signs_k"]), ("v", V, a["bv"], 64, a["signs_v"])):
                codes = a[f"l{comp}_codes"][pg, g, sl]
                sz = a[f"l{comp}_sz"][pg, g, sl].astype(np.float64)
                lat = np.array([((codes[i // 2] >> (4 * (i % 2))) & 15) * sz[i // 32, 0] + sz[i // 32, 1]
                                for i in range(r)])
                rc = a[f"r{comp}_codes"][pg, g, sl]
                rs = float(a[f"r{comp}_scale"][pg, g, sl])
                y = np.array([(((rc[i // 4] >> (2 * (i % 4))) & 3) - 1.5) * rs for i in range(d)])
                out[t] = lat @ fac[g].astype(np.float64) + (sg * (Q @ y)) / math.sqrt(d)
            # RoPE by complex multiplication
            z = K[t, :64] + 1j * K[t, 64:]
            z = z * np.exp(1j * t * 500000.0 ** (-2 * np.arange(64) / 128))
            K[t] = np.concatenate([z.real, z.imag])
        for h in range(2):
            np.testing.assert_allclose(o[0, 2 * g + h], sdpa(q[0, 2 * g + h], K, V, 1 / math.sqrt(d)),
                                       atol=1e-12)


# ---------------------------------------------------------------- bytes


def test_llama_cache_arithmetic_from_the_page():
    gold = json.load(open(os.path.join(GOLDEN, "llama31_8b_cache_arithmetic.json")))
    m, p = gold["model"], gold["printed"]
    per_tok = O.dense_bytes_per_token(m["layers"], m["kv_heads"], m["head_dim"], m["bytes_per_elt"])
    assert per_tok == 131072
    assert round(per_tok * 128000 / 1e9, 1) == p["gb_per_sequence"]
    assert round(8 * per_tok * 128000 / 1e9) == p["gb_batch_of_8"]
    assert round(8 * per_tok * 128000 / 1e9 / p["ratio"], 1) == p["gb_at_13_8x"]
    assert m["q_heads"] // m["kv_heads"] == p["gqa_shrink"]


def test_belt_ratio_arithmetic():
    gold = json.load(open(os.path.join(GOLDEN, "belt_compression_arithmetic.json")))["printed"]
    low_rank = 1 / (1 - gold["low_rank_reduction"])
    assert abs(low_rank - 10 / 3) < 1e-12
    assert abs(gold["overall_ratio"] / low_rank - 5.34) < 0.01   # quantization's share


@pytest.mark.parametrize("name,per_unit,total", [
    ("c1", 80, 40960),
    ("c2", 52, 109051904),
    ("c5", 128, 1073741824),
])
def test_lowrank_bytes_closed_form(name, per_unit, total):
    c = synth.config(name)
    bits = c["bits"]
    b = O.lowrank_bytes_per_token_head(c["rk"], c["rv"], bits, c["g"], c["resid"], c["d"])
    assert b == per_unit
    assert b * c["B"] * c["Hkv"] * c["T"] == total
    a = synth.lowrank_cache(c, T=16)
    stored = sum(a[k].nbytes for k in ("lk_codes", "lk_sz", "lv_codes", "lv_sz", "rk_codes",
                                       "rk_scale", "rv_codes", "rv_scale") if k in a)
    assert stored == b * c["B"] * c["Hkv"] * 16


def test_block_shared_and_varrate_bytes():
    c = synth.config("c3")
    assert O.latent_bytes(c["D"], 4, c["g"], has_zero=False) == 272
    assert 272 * c["B"] * c["T"] == 71303168
    # varrate: f(r) = r/2 + 4*ceil(r/32) per head, 10 bytes of metadata per token
    f = {r: O.latent_bytes(r, 4, 32) for r in (4, 8, 16, 32, 64)}
    assert f == {4: 6, 8: 8, 16: 12, 32: 20, 64: 40}
    c4 = synth.config("c4")
    ef = sum(p * f[r] for r, p in zip(c4["ranks"], c4["probs"]))
    assert abs(ef - 10.8) < 1e-12
    expected = c4["T"] * (8 * 2 * ef + 10)
    assert abs(expected - 23.96e6) / 23.96e6 < 2e-3
