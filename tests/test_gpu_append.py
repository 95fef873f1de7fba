"""GPU append parity: codes written by the append kernel against the reference
quantizer, bit-exact except where the fp32 pre-quantization value lies within
1e-5 (in code units) of a rounding boundary; a group whose fp64 min or step
lies within 1e-5 relative of an fp16 rounding boundary is excluded whole (its
stored scale / zero may legitimately differ by one fp16 ulp)."""

import numpy as np
import pytest
import torch

from oracle import kvc_oracle as O
from rank_bit_kv_b200 import kvc, synth

pytestmark = pytest.mark.gpu
EPS = 1e-5


def near_fp16_boundary(x):
    x = np.asarray(x, np.float64)
    return O.fp16_rn(x * (1 + EPS) + EPS * 1e-3) != O.fp16_rn(x * (1 - EPS) - EPS * 1e-3)


def asym_masks(lat, g):
    """(group_ok [.., nG], elem_ok [.., r]) for the INT4 asymmetric quantizer."""
    n = lat.shape[-1]
    ng = O.n_groups(n, g)
    codes, s, z = O.quantize_int4_asym(lat, g)
    gok = np.ones(lat.shape[:-1] + (ng,), bool)
    eok = np.ones(lat.shape, bool)
    for j in range(ng):
        sl = lat[..., j * g:min((j + 1) * g, n)]
        lo, hi = sl.min(-1), sl.max(-1)
        gok[..., j] = ~(near_fp16_boundary(lo) | near_fp16_boundary((hi - lo) / 15))
        t = (sl - z[..., j, None]) / np.where(s[..., j, None] > 0, s[..., j, None], 1)
        eok[..., j * g:min((j + 1) * g, n)] = np.abs(t - np.floor(t) - 0.5) > EPS
    return codes, s, z, gok, eok


def to_dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def fetch(cache, name, dtype, shape):
    return cache.bufs[name].cpu().numpy().view(dtype).reshape(shape)


def check_int4(got_codes, got_sz, lat, g, what):
    codes, s, z, gok, eok = asym_masks(lat, g)
    gcodes = O.unpack_int4(got_codes, lat.shape[-1])
    gs = got_sz[..., 0].astype(np.float64)
    gz = got_sz[..., 1].astype(np.float64)
    grp = np.arange(lat.shape[-1]) // g
    ok = gok[..., grp] & eok
    assert (gs[gok] == s[gok]).all() and (gz[gok] == z[gok]).all(), f"{what}: scale/zero"
    bad = (gcodes != codes) & ok
    assert not bad.any(), f"{what}: {bad.sum()} code mismatches"
    COMPARED.append(ok.mean())
    return ok, codes, s, z


COMPARED = []


@pytest.fixture(autouse=True)
def _compared_fraction():
    """Most codes must actually be compared: about 3% of fp16 values lie within
    1e-5 relative of a rounding midpoint, so a few percent of groups drop out."""
    COMPARED.clear()
    yield
    if COMPARED:
        frac = float(np.mean(COMPARED))
        assert frac > 0.75, f"only {frac:.2%} of codes compared"


@pytest.mark.parametrize("name,n_new", [("c2", 5), ("c5", 3)])
def test_lowrank_append_bit_exact(name, n_new):
    c = synth.config(name, B=2, T=64)
    a = synth.lowrank_cache(c, T=64)
    lay = kvc.Layout(kvc.desc_from_config(c, capacity=64))
    cache = kvc.Cache(lay, fill=a)
    kn, vn = synth.new_tokens(c, n_new)
    pos = [7, 40]
    kvc.append(lay, cache, to_dev_bf16(kn), to_dev_bf16(vn), pos, n_new)
    torch.cuda.synchronize()
    B, Hkv, d, g = c["B"], c["Hkv"], c["d"], c["g"]
    P = c["page"]
    rows = a["lk_codes"].shape[:3]
    for comp, x_bits, r in (("k", kn, c["rk"]), ("v", vn, c["rv"])):
        codes = fetch(cache, f"l{comp}_codes", np.uint8, rows + (r // 2,))
        sz = fetch(cache, f"l{comp}_sz", np.float16, rows + (O.n_groups(r, g), 2))
        fac = a[f"b{comp}"].astype(np.float64)
        x = O.bf16_bits_to_f64(x_bits)                            # [B, Hkv, n_new, d]
        for b in range(B):
            for i in range(n_new):
                t = pos[b] + i
                if P:
                    pp, sl = a["page_table"][b, t // P], t % P
                    gc, gsz = codes[pp, :, sl], sz[pp, :, sl]
                else:
                    gc, gsz = codes[b, :, t], sz[b, :, t]
                lat = np.einsum("hd,hrd->hr", x[b, :, i], fac)
                ok, qc, qs, qz = check_int4(gc, gsz, lat, g, f"{name} {comp} b{b} i{i}")
                if not c["resid"]:
                    continue
                sg = a[f"signs_{comp}"]
                rc_all = fetch(cache, f"r{comp}_codes", np.uint8, rows + (d // 4,))
                rs_all = fetch(cache, f"r{comp}_scale", np.float16, rows)
                for h in range(Hkv):
                    if not ok[h].all():
                        continue                     # residual depends on an excluded code
                    ref = O.append_lowrank(x[b, h, i], fac[h], g, signs=sg)
                    y = ref["y"]
                    rs = rs_all[pp, h, sl].astype(np.float64)
                    if near_fp16_boundary(np.abs(y).max() / 1.5):
                        continue
                    assert rs == ref["rscale"], f"{name} {comp} residual scale"
                    tt = y / rs
                    eok = np.abs(tt - np.rint(tt)) > EPS
                    gotc = O.unpack_int2(rc_all[pp, h, sl], d)
                    assert not ((gotc != ref["rcodes"]) & eok).any(), f"{name} {comp} residual codes"


def test_lowrank_bulk_append_bit_exact():
    """A prefill-sized append (n_new >= 64) runs the bulk kernel (factor staged
    once per block, one warp per token); its codes must equal the oracle's
    quantizer on every appended token, as the per-token kernel's do."""
    c = synth.config("c2", B=2, T=512)
    a = synth.lowrank_cache(c, T=512)
    lay = kvc.Layout(kvc.desc_from_config(c, capacity=512))
    cache = kvc.Cache(lay, fill=a)
    n_new, pos = 300, [7, 200]
    kn, vn = synth.new_tokens(c, n_new)
    kvc.append(lay, cache, to_dev_bf16(kn), to_dev_bf16(vn), pos, n_new)
    torch.cuda.synchronize()
    g = c["g"]
    rows = a["lk_codes"].shape[:3]
    for comp, x_bits, r in (("k", kn, c["rk"]), ("v", vn, c["rv"])):
        codes = fetch(cache, f"l{comp}_codes", np.uint8, rows + (r // 2,))
        sz = fetch(cache, f"l{comp}_sz", np.float16, rows + (O.n_groups(r, g), 2))
        fac = a[f"b{comp}"].astype(np.float64)
        x = O.bf16_bits_to_f64(x_bits)                            # [B, Hkv, n_new, d]
        for b in range(c["B"]):
            t = np.arange(pos[b], pos[b] + n_new)
            lat = np.einsum("hid,hrd->ihr", x[b], fac)            # [n_new, Hkv, r]
            for i in range(n_new):
                check_int4(codes[b, :, t[i]], sz[b, :, t[i]], lat[i], g, f"bulk {comp} b{b} i{i}")
        # slots outside the appended range keep their previous contents
        before = a[f"l{comp}_codes"]
        np.testing.assert_array_equal(codes[0, :, :pos[0]], before[0, :, :pos[0]])
        np.testing.assert_array_equal(codes[1, :, pos[1] + n_new:], before[1, :, pos[1] + n_new:])


def test_fp16_latent_append():
    c = synth.config("c1")
    a = synth.lowrank_cache(c, T=16)
    lay = kvc.Layout(kvc.desc_from_config(c, capacity=16))
    cache = kvc.Cache(lay, fill=a)
    kn, vn = synth.new_tokens(c, 2)
    kvc.append(lay, cache, to_dev_bf16(kn), to_dev_bf16(vn), [3], 2)
    torch.cuda.synchronize()
    got = fetch(cache, "lk_codes", np.float16, (1, 1, 16, 16))[0, 0, 3:5].astype(np.float64)
    lat = O.bf16_bits_to_f64(kn)[0, 0] @ a["bk"][0].astype(np.float64).T
    # stored as the fp16 rounding of the fp32 projection: within one fp16 ulp
    np.testing.assert_allclose(got, lat, rtol=2 ** -10, atol=1e-7)


def test_varrate_append_records_and_offsets():
    c = synth.config("c4", T=32)
    a = synth.varrate_cache(c, T=20, capacity=32)
    lay = kvc.Layout(kvc.desc_from_config(c, capacity=32))
    cache = kvc.Cache(lay, fill=a)
    n_new = 6
    rng = np.random.default_rng(9)
    ranks = rng.choice([4, 8, 16, 32, 64], size=(2, 1, n_new)).astype(np.uint8)
    kn, vn = synth.new_tokens(c, n_new)
    kvc.append(lay, cache, to_dev_bf16(kn), to_dev_bf16(vn), [20], n_new, new_ranks=ranks)
    torch.cuda.synchronize()
    off = fetch(cache, "offset_k", np.int32, (1, 33))
    rk = fetch(cache, "rank_k", np.uint8, (1, 32))
    np.testing.assert_array_equal(rk[0, 20:26], ranks[0, 0])
    sizes = np.diff(off[0, :27].astype(np.int64))
    exp = [8 * (int(r) // 2 + 4 * ((int(r) + 31) // 32)) for r in rk[0, :26]]
    np.testing.assert_array_equal(sizes, exp)
    stream = cache.bufs["lk_codes"].cpu().numpy().reshape(1, -1)
    x = O.bf16_bits_to_f64(kn)[0]                  # [Hkv, n_new, d]
    fac = a["bk"].astype(np.float64)
    for i in range(n_new):
        t = 20 + i
        r = int(ranks[0, 0, i])
        ng = O.n_groups(r, 32)
        per = r // 2 + 4 * ng
        for h in range(8):
            st = int(off[0, t]) + h * per
            gc = stream[0, st:st + r // 2]
            gsz = stream[0, st + r // 2:st + per].copy().view(np.float16).reshape(ng, 2)
            lat = x[h, i] @ fac[h, :r].T
            check_int4(gc[None], gsz[None], lat[None], 32, f"varrate t{t} h{h}")


def test_block_shared_append():
    c = synth.config("c3", B=2, T=8)
    a = synth.block_shared_cache(c, T=8)
    lay = kvc.Layout(kvc.desc_from_config(c, capacity=8))
    cache = kvc.Cache(lay, fill=a)
    rng = np.random.default_rng(3)
    lat_bits = synth.to_bf16_bits(rng.standard_normal((2, 3, 512)))
    kvc.append(lay, cache, to_dev_bf16(lat_bits), None, [1, 5], 3)
    torch.cuda.synchronize()
    codes = fetch(cache, "lk_codes", np.uint8, (2, 8, 256))
    sc = fetch(cache, "lk_sz", np.float16, (2, 8, 8))
    x = O.bf16_bits_to_f64(lat_bits)
    for b, p0 in ((0, 1), (1, 5)):
        for i in range(3):
            ref_c, ref_s = O.quantize_int4_sym(x[b, i], 64)
            gs = sc[b, p0 + i].astype(np.float64)
            gok = ~near_fp16_boundary(np.abs(x[b, i]).reshape(8, 64).max(-1) / 7)
            assert (gs[gok] == ref_s[gok]).all()
            t = x[b, i] / np.repeat(np.where(ref_s > 0, ref_s, 1), 64)
            eok = (np.abs(t - np.floor(t) - 0.5) > EPS) & np.repeat(gok, 64)
            got = O.unpack_int4(codes[b, p0 + i], 512)
            assert not ((got != ref_c) & eok).any()


def test_dense_append_copies():
    cfg = dict(kind="dense", B=2, Hq=8, Hkv=2, d=128, T=16)
    a = synth.dense_cache(2, 8, 2, 128, 16, seed=1)
    lay = kvc.Layout(kvc.desc_from_config(cfg))
    cache = kvc.Cache(lay, fill=a)
    kn, vn = synth.new_tokens(dict(B=2, Hkv=2, d=128, seed=0), 2)
    kvc.append(lay, cache, to_dev_bf16(kn), to_dev_bf16(vn), [0, 14], 2)
    torch.cuda.synchronize()
    kd = fetch(cache, "k_dense", np.uint16, (2, 2, 16, 128))
    np.testing.assert_array_equal(kd[0, :, 0:2], kn[0])
    np.testing.assert_array_equal(kd[1, :, 14:16], kn[1])


def test_append_then_decode_matches_oracle_on_the_written_codes():
    """A decode step right after an append (the C5-style step): the oracle reads
    the codes the append wrote, so this checks decode, not the quantizer."""
    c = synth.config("c5", B=2, T=96)
    a = synth.lowrank_cache(c, T=96)
    lay = kvc.Layout(kvc.desc_from_config(c, capacity=96))
    cache = kvc.Cache(lay, fill=a)
    kn, vn = synth.new_tokens(c, 1)
    kvc.append(lay, cache, to_dev_bf16(kn), to_dev_bf16(vn), [95, 95], 1)
    cache.n_tokens = 96
    q = to_dev_bf16(a["q"])
    out = torch.empty(q.shape, device="cuda", dtype=torch.float32)
    ws = torch.empty(lay.workspace_bytes(96), dtype=torch.uint8, device="cuda")
    kvc.decode(lay, cache, q, out, ws)
    torch.cuda.synchronize()
    stored = dict(a)
    for k in ("lk_codes", "lk_sz", "lv_codes", "lv_sz", "rk_codes", "rk_scale", "rv_codes", "rv_scale"):
        stored[k] = cache.bufs[k].cpu().numpy().view(a[k].dtype).reshape(a[k].shape)
    from tests.gpu_util import assert_close
    assert_close(out.cpu().numpy(), O.decode_from_storage(c, stored, 96), what="append+decode")
