"""Token-importance producers: VarRate's salience-driven per-token ranks
("VarRate: ...", "Summary" / "Method") and BellowsKV-Evict's single keep
decision per block applied to the shared latent ("BellowsKV Architecture ...",
"Three Measurements, Three Operators").

The oracle (oracle/salience.py) is pinned by what the definitions fix: every
window row's softmax contributes exactly 1, uniform scores spread it evenly, a
planted needle takes it, permuting tokens permutes the salience, rung counts
are exact and the ranks monotone in salience, the keep set is the brute-force
top-k.  The library's integer decisions are then compared exactly with the
oracle's rule applied to the library's own fp32 salience, and its salience with
the oracle's within a float tolerance."""

import numpy as np
import pytest

from oracle import kvc_oracle as O
from oracle import salience as S
from rank_bit_kv_b200 import synth

LADDER = [64, 32, 16, 8, 4]
FRACS = [0.05, 0.10, 0.20, 0.25, 0.40]         # the variable-rate workload's mix


def draw(rng, B, Hq, Hkv, W, T, d=128):
    q = rng.standard_normal((B, Hq, W, d))
    k = rng.standard_normal((B, Hkv, T, d))
    return q, k


# ----------------------------------------------------------------- oracle pins (CPU)


def test_salience_totals_and_uniform_case():
    rng = np.random.default_rng(0)
    q, k = draw(rng, 2, 8, 2, 5, 300, 16)
    sal = S.window_salience(q, k, 0.25)
    np.testing.assert_allclose(sal.sum(1), 8 * 5, rtol=1e-12)          # each softmax sums to 1
    sal0 = S.window_salience(np.zeros_like(q), k, 0.25)
    np.testing.assert_allclose(sal0, 8 * 5 / 300, rtol=1e-12)          # uniform scores


def test_salience_needle_and_permutation():
    rng = np.random.default_rng(1)
    q, k = draw(rng, 1, 4, 1, 3, 200, 16)
    u = rng.standard_normal(16)
    q = u + 0.1 * q                                       # every window query near u
    k[0, 0, 77] = 10 * u                                  # the needle: score ~ 10 |u|^2
    sal = S.window_salience(q, k, 1.0)
    assert sal[0, 77] > 0.9 * 12 and sal[0].argmax() == 77
    perm = rng.permutation(200)
    np.testing.assert_allclose(S.window_salience(q, k[:, :, perm], 1.0), sal[:, perm], rtol=1e-12)


def test_ranks_by_salience_counts_order_and_ties():
    rng = np.random.default_rng(2)
    T = 1000
    sal = rng.random((3, T))
    sal[1, 100:200] = 0.5                                  # a run of ties
    counts = S.rung_counts(T, FRACS)
    assert counts == [50, 100, 200, 250, 400]
    r = S.ranks_by_salience(sal, LADDER, counts)
    for b in range(3):
        assert [(r[b] == x).sum() for x in LADDER] == counts
        order = S.descending_order(sal[b])
        ranks_in_order = r[b, order]
        assert (np.diff(ranks_in_order) <= 0).all()        # never a higher rank further down
    tied = np.arange(100, 200)
    rt = r[1, tied]
    assert (np.diff(rt) <= 0).all()                        # ties: lower position first
    assert (r > 0).all()                                   # no token at rank zero


def test_rung_counts_of_the_variable_rate_mix_average_the_budget():
    counts = S.rung_counts(131072, FRACS)
    mean = np.dot(counts, LADDER) / 131072
    assert abs(mean - 13.2) < 1e-3 and abs(mean / 64 - 0.206) < 1e-3


def test_keep_decision_brute_force():
    rng = np.random.default_rng(3)
    imp = rng.random((2, 50))
    kept = S.keep_decision(imp, 12)
    for b in range(2):
        top = sorted(range(50), key=lambda t: (-imp[b, t], t))[:12]
        assert list(kept[b]) == sorted(top)


# ----------------------------------------------------------------- library against the oracle (GPU)


def dev_bf16(a):
    import torch

    bits = synth.to_bf16_bits(a)
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16), \
        O.bf16_bits_to_f64(bits)


@pytest.mark.gpu
@pytest.mark.parametrize("B,Hq,Hkv,W,T", [(2, 32, 8, 32, 3000), (1, 32, 8, 16, 131), (2, 8, 8, 4, 1)])
def test_window_salience_matches_oracle(B, Hq, Hkv, W, T):
    import torch

    from rank_bit_kv_b200 import kvc

    rng = np.random.default_rng(T)
    q, k = draw(rng, B, Hq, Hkv, W, T)
    qd, q64 = dev_bf16(q)
    kd, k64 = dev_bf16(k)
    sal = kvc.window_salience(qd, kd)
    torch.cuda.synchronize()
    ref = S.window_salience(q64, k64, 1 / np.sqrt(128))
    got = sal.cpu().numpy()
    assert np.abs(got - ref).max() <= 1e-3 * ref.max() + 1e-6
    np.testing.assert_allclose(got.sum(1), Hq * W, rtol=1e-3)


@pytest.mark.gpu
@pytest.mark.parametrize("T", [7, 1000, 131072])
def test_ranks_exact_on_the_library_salience(T):
    """Integer decisions: the library's ranks equal the oracle's rule applied to
    the very same fp32 salience (exact counts, ties by position)."""
    import torch

    from rank_bit_kv_b200 import kvc

    rng = np.random.default_rng(T)
    sal = rng.random((2, T)).astype(np.float32)
    sal[0, : T // 3] = sal[0, 0]                          # many exact ties
    counts = S.rung_counts(T, FRACS)
    ranks = kvc.ranks_by_salience(torch.from_numpy(sal).cuda(), LADDER, counts[:-1])
    torch.cuda.synchronize()
    got = ranks.cpu().numpy()
    ref = S.ranks_by_salience(sal.astype(np.float64), LADDER, counts)
    np.testing.assert_array_equal(got[0], ref)
    np.testing.assert_array_equal(got[1], ref)


@pytest.mark.gpu
def test_varrate_salience_to_ranks_to_append_to_decode():
    """The variable-rate path end to end on the GPU: prefill keys and a query
    window -> salience -> ranks by the workload's mix -> one kvc_append of all
    prefill tokens with those ranks -> decode, checked against the oracle on the
    stored records."""
    import torch

    from rank_bit_kv_b200 import kvc
    from tests.gpu_util import assert_close

    c = synth.config("c4", T=2048)
    T = c["T"]
    kb, vb = synth.prefill_kv(c, T)
    rng = np.random.default_rng(11)
    qw = synth.to_bf16_bits(rng.standard_normal((1, 32, 4, 128)))
    qd = torch.from_numpy(qw.view(np.int16)).cuda().view(torch.bfloat16)
    kd = torch.from_numpy(kb.view(np.int16)).cuda().view(torch.bfloat16)
    vd = torch.from_numpy(vb.view(np.int16)).cuda().view(torch.bfloat16)
    sal = kvc.window_salience(qd, kd)
    counts = S.rung_counts(T, FRACS)
    ranks = kvc.ranks_by_salience(sal, LADDER, counts[:-1])
    torch.cuda.synchronize()
    ref_sal = S.window_salience(O.bf16_bits_to_f64(qw), O.bf16_bits_to_f64(kb), 1 / np.sqrt(128))
    assert np.abs(sal.cpu().numpy() - ref_sal).max() <= 1e-3 * ref_sal.max()
    np.testing.assert_array_equal(ranks.cpu().numpy()[0],
                                  S.ranks_by_salience(sal.cpu().numpy().astype(np.float64),
                                                      LADDER, counts))
    # store every prefill token at its rank, then decode over the stored records
    a = synth.varrate_cache(c, T=1, capacity=T)
    lay = kvc.Layout(kvc.desc_from_config(c, capacity=T))
    cache = kvc.Cache(lay, fill=a)
    kvc.append(lay, cache, kd, vd, [0], T, new_ranks=ranks)
    cache.n_tokens = T
    q = torch.from_numpy(a["q"].view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty(q.shape, device="cuda")
    ws = torch.empty(lay.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    kvc.decode(lay, cache, q, out, ws)
    torch.cuda.synchronize()
    stored = dict(a)
    stored["kstream"] = cache.bufs["lk_codes"].cpu().numpy().reshape(1, -1)
    stored["vstream"] = cache.bufs["lv_codes"].cpu().numpy().reshape(1, -1)
    for comp in ("k", "v"):
        stored[f"offset_{comp}"] = cache.bufs[f"offset_{comp}"].cpu().numpy().view(np.int32).reshape(1, -1)
        stored[f"rank_{comp}"] = cache.bufs[f"rank_{comp}"].cpu().numpy().reshape(1, -1)
    assert (stored["rank_k"][0, :T] > 0).all()
    assert_close(out.cpu().numpy(), O.decode_from_storage(c, stored, T), what="salience ranks decode")


@pytest.mark.gpu
def test_block_keep_and_compact():
    """BellowsKV-Evict: the layers' saliences summed into one importance, the
    keep set exact on the library's own importance, the compacted block latent
    holding exactly the kept rows, and a decode over it equal to the oracle's."""
    import torch

    from rank_bit_kv_b200 import kvc
    from tests.gpu_util import assert_close

    c = synth.config("c3", B=2, T=600)
    a = synth.block_shared_cache(c)
    rng = np.random.default_rng(4)
    sal_layers = rng.random((4, 2, 600)).astype(np.float32)
    imp, kept = kvc.block_keep(torch.from_numpy(sal_layers).cuda(), 250)
    torch.cuda.synchronize()
    imp = imp.cpu().numpy()
    kept = kept.cpu().numpy()
    np.testing.assert_allclose(imp, sal_layers.astype(np.float64).sum(0), rtol=1e-6)
    np.testing.assert_array_equal(kept, S.keep_decision(imp.astype(np.float64), 250))
    src_lay = kvc.Layout(kvc.desc_from_config(c))
    src = kvc.Cache(src_lay, fill=a)
    src.n_tokens = 600
    cd = dict(c, T=256)
    dst_lay = kvc.Layout(kvc.desc_from_config(cd))
    dst = kvc.Cache(dst_lay, fill={"wk": a["wk"], "wv": a["wv"]})
    kvc.block_compact(src_lay, src, dst_lay, dst, torch.from_numpy(kept).cuda())
    torch.cuda.synchronize()
    codes = dst.bufs["lk_codes"].cpu().numpy().reshape(2, 256, 256)[:, :250]
    scales = dst.bufs["lk_sz"].cpu().numpy().view(np.float16).reshape(2, 256, 8)[:, :250]
    for b in range(2):
        np.testing.assert_array_equal(codes[b], a["lk_codes"][b, kept[b]])
        np.testing.assert_array_equal(scales[b], a["lk_sz"][b, kept[b]])
    q = torch.from_numpy(a["q"].view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty(q.shape, device="cuda")
    ws = torch.empty(dst_lay.workspace_bytes(250), dtype=torch.uint8, device="cuda")
    kvc.decode(dst_lay, dst, q, out, ws)
    torch.cuda.synchronize()
    comp = dict(a)
    comp["lk_codes"] = np.stack([a["lk_codes"][b, kept[b]] for b in range(2)])
    comp["lk_sz"] = np.stack([a["lk_sz"][b, kept[b]] for b in range(2)])
    assert_close(out.cpu().numpy(), O.decode_from_storage(dict(c, T=250), comp, 250),
                 what="decode over the compacted block latent")


def test_importance_host_errors():
    import ctypes as C

    from rank_bit_kv_b200 import build, kvc

    build.build()
    lib = kvc.lib()
    f = C.c_void_p(0x10000)
    ws = lib.kvc_salience_workspace_bytes(1, 32, 8, 64, 100)
    st = lib.kvc_window_salience(f, f, 1, 32, 8, 64, 100, 100, 128, 0.0, f, f, ws, None)
    assert kvc.STATUS[st] == "KVC_EUNSUPPORTED"                  # 4 x 64 window rows > 128
    rr = (C.c_int32 * 2)(64, 12)
    rc = (C.c_int32 * 1)(5)
    st = lib.kvc_ranks_by_salience(f, 1, 100, 2, rr, rc, f, None)
    assert kvc.STATUS[st] == "KVC_EINVAL"                        # rank 12
    st = lib.kvc_block_keep(f, 4, 1, 100, 101, f, f, None)
    assert kvc.STATUS[st] == "KVC_EINVAL"                        # keep > tokens
