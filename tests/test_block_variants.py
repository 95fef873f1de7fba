"""Block-shared latents at the BellowsKV page's other operating points
("BellowsKV Architecture ...", "Reading the Retention Table": n = 2 with INT8,
n = 4 with INT4, INT3, a 3-bit key / 2-bit value variant) and a layer of a
block decoded on its own.

The oracle's general symmetric quantizer and bit-stream packing are pinned to
the already-pinned INT4 and 2-bit forms and to their own defining properties;
the GPU decode and append are compared with the oracle on identical codes."""

import numpy as np
import pytest

from oracle import kvc_oracle as O
from rank_bit_kv_b200 import synth

VARIANTS = [  # (n layers, key / shared bits, value bits)
    (2, 8, 0),   # n = 2 INT8
    (4, 4, 0),   # n = 4 INT4 (the block-shared workload)
    (4, 3, 0),   # INT3
    (4, 3, 2),   # 3-bit key latent, 2-bit value latent
]


# ----------------------------------------------------------------- oracle pins (CPU)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_bit_stream_packing_round_trips_and_matches_the_fixed_forms(bits):
    rng = np.random.default_rng(bits)
    c = rng.integers(0, 2 ** bits, (5, 64))
    packed = O.pack_bits(c, bits)
    assert packed.shape == (5, 64 * bits // 8)
    np.testing.assert_array_equal(O.unpack_bits(packed, 64, bits), c)
    if bits == 4:
        np.testing.assert_array_equal(packed, O.pack_int4(c))
    if bits == 2:
        np.testing.assert_array_equal(packed, O.pack_int2(c))
    if bits == 8:
        np.testing.assert_array_equal(packed, c.astype(np.uint8))


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_symmetric_quantizer_properties(bits):
    rng = np.random.default_rng(10 + bits)
    x = rng.standard_normal((50, 128))
    codes, s = O.quantize_sym(x, 64, bits)
    qmax = 2 ** (bits - 1) - 1
    assert codes.min() >= 1 and codes.max() <= 2 ** bits - 1        # offset binary, no -2^(b-1)
    xh = O.dequant_sym(codes, s, 64, bits)
    grp = np.arange(128) // 64
    assert (np.abs(x - xh) <= s[:, grp] / 2 + np.abs(x) * 2 ** -10 + 1e-12).all()
    # the group's largest magnitude maps to +-qmax
    top = np.abs(x.reshape(50, 2, 64)).argmax(-1)
    c2 = codes.reshape(50, 2, 64)
    picked = np.take_along_axis(c2, top[..., None], -1)[..., 0] - 2 ** (bits - 1)
    assert (np.abs(picked) == qmax).all()
    if bits == 4:
        c4, s4 = O.quantize_int4_sym(x, 64)
        np.testing.assert_array_equal(codes, c4)
        np.testing.assert_array_equal(s, s4)


def test_separate_value_latent_and_single_layer_reduce_to_the_shared_form():
    rng = np.random.default_rng(3)
    L, B, Hq, Hkv, d, D, T = 2, 1, 8, 2, 16, 32, 40
    q = rng.standard_normal((L, B, Hq, d))
    lat = rng.standard_normal((B, T, D))
    wk = rng.standard_normal((L, D, Hkv * d)) / np.sqrt(D)
    wv = rng.standard_normal((L, D, Hkv * d)) / np.sqrt(D)
    both = O.decode_block_shared(q, lat, wk, wv, Hkv, 0.25)
    np.testing.assert_allclose(O.decode_block_shared(q, lat, wk, wv, Hkv, 0.25, latent_v=lat), both,
                               rtol=1e-13)
    for l in range(L):
        one = O.decode_block_shared(q[l:l + 1], lat, wk[l:l + 1], wv[l:l + 1], Hkv, 0.25)
        np.testing.assert_allclose(one[0], both[l], rtol=1e-13)


def test_layout_sizes_of_the_variants():
    from rank_bit_kv_b200 import build, kvc

    build.build()
    for nl, bits, vbits in VARIANTS:
        c = synth.config("c3", L=nl, B=2, T=64, bits=bits, vbits=vbits)
        lay = kvc.Layout(kvc.desc_from_config(c))
        sz = lay.buffer_sizes()
        assert sz["lk_codes"] == 2 * 64 * 512 * bits // 8
        assert sz["lk_sz"] == 2 * 64 * 8 * 2
        assert sz["lv_codes"] == (2 * 64 * 512 * vbits // 8 if vbits else 0)
        per = 512 * bits // 8 + 16 + (512 * vbits // 8 + 16 if vbits else 0)
        assert lay.step_bytes(64) == 2 * 64 * per


# ----------------------------------------------------------------- GPU against the oracle


@pytest.mark.gpu
@pytest.mark.parametrize("nl,bits,vbits", VARIANTS)
@pytest.mark.parametrize("T", [1, 300, 1025])
def test_block_variant_decode(nl, bits, vbits, T):
    from tests.gpu_util import assert_close, run_decode

    c = synth.config("c3", L=nl, B=2, T=T, bits=bits, vbits=vbits, seed=30 + bits + vbits)
    a = synth.block_shared_cache(c)
    ref = O.decode_from_storage(c, a, T)
    assert_close(run_decode(c, a, T), ref, what=f"n={nl} {bits}/{vbits} T={T}")
    assert_close(run_decode(c, a, T, seq_lens=[T, T]), ref, what=f"generic n={nl} {bits}/{vbits}")


@pytest.mark.gpu
@pytest.mark.parametrize("bits,vbits", [(4, 0), (3, 2)])
def test_block_single_layer_decode(bits, vbits):
    """Each layer of the block decoded on its own reads the same shared latent."""
    import torch

    from rank_bit_kv_b200 import kvc
    from tests.gpu_util import assert_close

    c = synth.config("c3", B=2, T=700, bits=bits, vbits=vbits, seed=41)
    a = synth.block_shared_cache(c)
    lay = kvc.Layout(kvc.desc_from_config(c))
    cache = kvc.Cache(lay, fill=a)
    cache.n_tokens = 700
    ws = torch.empty(lay.workspace_bytes(700), dtype=torch.uint8, device="cuda")
    for layer in range(1, c["L"] + 1):
        cache.layer = layer
        q = torch.from_numpy(a["q"][layer - 1].view(np.int16)).cuda().view(torch.bfloat16)
        out = torch.empty(q.shape, device="cuda")
        kvc.decode(lay, cache, q, out, ws)
        torch.cuda.synchronize()
        ref = O.decode_from_storage(dict(c, layer=layer), dict(a, q=a["q"][layer - 1]), 700)
        assert_close(out.cpu().numpy(), ref, what=f"layer {layer}")


@pytest.mark.gpu
@pytest.mark.parametrize("bits,vbits", [(8, 0), (3, 0), (3, 2), (4, 8)])
def test_block_variant_append_bit_exact(bits, vbits):
    """Codes written by the append kernel equal the oracle's quantizer, except
    where x / s lies within 1e-5 of a rounding midpoint or the group's scale
    lies within 1e-5 relative of an fp16 rounding boundary."""
    import torch

    from rank_bit_kv_b200 import kvc

    c = synth.config("c3", B=2, T=8, bits=bits, vbits=vbits)
    a = synth.block_shared_cache(c)
    lay = kvc.Layout(kvc.desc_from_config(c))
    cache = kvc.Cache(lay, fill=a)
    rng = np.random.default_rng(bits * 10 + vbits)
    xk = synth.to_bf16_bits(rng.standard_normal((2, 3, 512)))
    xv = synth.to_bf16_bits(rng.standard_normal((2, 3, 512)))
    dev = lambda z: torch.from_numpy(z.view(np.int16)).cuda().view(torch.bfloat16)
    kvc.append(lay, cache, dev(xk), dev(xv) if vbits else None, [1, 4], 3)
    torch.cuda.synchronize()
    compared = []
    for comp, xb, nb in (("k", xk, bits), ("v", xv, vbits)):
        if not nb:
            continue
        codes = cache.bufs[f"l{comp}_codes"].cpu().numpy().reshape(2, 8, 512 * nb // 8)
        sc = cache.bufs[f"l{comp}_sz"].cpu().numpy().view(np.float16).reshape(2, 8, 8)
        x = O.bf16_bits_to_f64(xb)
        qmax = 2 ** (nb - 1) - 1
        for b, p0 in ((0, 1), (1, 4)):
            for i in range(3):
                ref_c, ref_s = O.quantize_sym(x[b, i], 64, nb)
                gmax = np.abs(x[b, i]).reshape(8, 64).max(-1) / qmax
                gok = np.asarray(O.fp16_rn(gmax * (1 + 1e-5)) == O.fp16_rn(gmax * (1 - 1e-5)))
                gs = sc[b, p0 + i].astype(np.float64)
                assert (gs[gok] == ref_s[gok]).all(), f"{comp} scales"
                t = x[b, i] / np.repeat(np.where(ref_s > 0, ref_s, 1), 64)
                eok = (np.abs(t - np.floor(t) - 0.5) > 1e-5) & np.repeat(gok, 64)
                got = O.unpack_bits(codes[b, p0 + i], 512, nb)
                assert not ((got != ref_c) & eok).any(), f"{comp} codes {nb} bits"
                compared.append(eok.mean())
    assert np.mean(compared) > 0.75
