"""Bulk prefill compression: per-head factors by randomized SVD ("A JoLT for
the KV cache ...", "Abstract (arXiv)": FlashJoLT's randomized token-mode SVD;
"JoLT: Near-Lossless KV Cache Compression", "Key findings": per-head factors
of keys before RoPE), then every prefill token projected and quantized by
kvc_append.

The oracle (oracle/flashjolt_fit.py, the textbook randomized SVD steps on the
token-major matrix) is pinned to numpy.linalg.svd: exact recovery of the
subspace and singular values of exactly low-rank matrices, and near-optimal
truncation error (Eckart-Young) with power iterations.  The library's fit
(a Gram matrix on tensor cores, fp64 algebra after it) is compared with the
oracle on the same bf16 inputs and test matrices."""

import numpy as np
import pytest

from oracle import flashjolt_fit as F
from oracle import kvc_oracle as O
from rank_bit_kv_b200 import synth


def low_rank(rng, n, d, r, sv):
    U, _ = np.linalg.qr(rng.standard_normal((n, r)))
    V, _ = np.linalg.qr(rng.standard_normal((d, r)))
    return (U * sv) @ V.T


def projector(F_):
    return F_.T @ F_


# ----------------------------------------------------------------- oracle pins (CPU)


@pytest.mark.parametrize("seed", range(3))
def test_oracle_recovers_an_exactly_low_rank_matrix(seed):
    rng = np.random.default_rng(seed)
    X = low_rank(rng, 2000, 128, 24, np.linspace(5, 1, 24))
    om = rng.standard_normal((128, 40))
    Fo, s2 = F.randomized_factor(X, om, 24, 0)
    _, s, Vt = np.linalg.svd(X, full_matrices=False)
    assert np.abs(projector(Fo) - projector(Vt[:24])).max() < 1e-10
    np.testing.assert_allclose(s2, s[:24] ** 2, rtol=1e-10)
    np.testing.assert_allclose(Fo @ Fo.T, np.eye(24), atol=1e-12)
    # sign convention: each row's entry of largest magnitude is positive
    assert (Fo[np.arange(24), np.abs(Fo).argmax(1)] > 0).all()


def test_oracle_truncation_error_is_near_optimal_with_power_iterations():
    rng = np.random.default_rng(7)
    X = low_rank(rng, 3000, 128, 128, np.exp(-0.05 * np.arange(128)))
    om = rng.standard_normal((128, 48))
    s = np.linalg.svd(X, compute_uv=False)
    best = (s[32:] ** 2).sum()                       # Eckart-Young
    errs = []
    for q in (0, 2):
        Fo, _ = F.randomized_factor(X, om, 32, q)
        errs.append(np.linalg.norm(X - X @ Fo.T @ Fo) ** 2 / best)
    assert errs[1] <= errs[0] + 1e-12
    assert errs[1] < 1 + 1e-3


# ----------------------------------------------------------------- library against the oracle (GPU)


def well_separated_kv(rng, B, Hkv, T, d, r):
    """bf16 bits [B, Hkv, T, d]: per head, singular values 1 - i/64 for the first
    r components and a tail 20x smaller (a clear gap at r, distinct values)."""
    sv = np.concatenate([1 - np.arange(r) / 64, 0.05 * (1 - np.arange(d - r) / (2 * d))])
    x = np.empty((B, Hkv, T, d), np.float32)
    for h in range(Hkv):
        basis, _ = np.linalg.qr(rng.standard_normal((d, d)))
        x[:, h] = (rng.standard_normal((B, T, d)) * sv) @ basis.T
    return synth.to_bf16_bits(x)


def to_dev_bf16(a):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.gpu
@pytest.mark.parametrize("rank,k,q", [(32, 48, 1), (48, 64, 2), (16, 32, 0)])
def test_fit_matches_oracle_on_well_separated_spectra(rank, k, q):
    import torch

    from rank_bit_kv_b200 import kvc

    rng = np.random.default_rng(rank + k)
    B, Hkv, T, d = 2, 4, 1000, 128
    xb = well_separated_kv(rng, B, Hkv, T, d, rank)
    om = synth.gaussian_test_matrix(Hkv, d, k, seed=5)
    fac, s2 = kvc.fit_factors(to_dev_bf16(xb), torch.from_numpy(om).cuda(), rank, q)
    torch.cuda.synchronize()
    fac = fac.float().cpu().numpy()
    s2 = s2.cpu().numpy()
    Fo, So = F.fit_heads(O.bf16_bits_to_f64(xb), om.astype(np.float64), rank, q)
    assert np.abs(fac - Fo).max() < 2e-3                 # fp16 rows, fp32 Gram
    np.testing.assert_allclose(s2[:, :rank], So, rtol=2e-3)


@pytest.mark.gpu
def test_fit_at_full_prefill_size_is_as_good_as_the_oracle():
    """The C2 prefill (8 rows x 32768 tokens x 8 KV heads of pre-RoPE keys with a
    decaying spectrum): the library's factor leaves the same truncation error as
    the oracle's (within 0.1 %), head by head."""
    import torch

    from rank_bit_kv_b200 import kvc

    c = synth.config("c2")
    kb, _ = synth.prefill_kv(c, c["T"])
    om = synth.gaussian_test_matrix(c["Hkv"], 128, 48, seed=9)
    fac, _ = kvc.fit_factors(to_dev_bf16(kb), torch.from_numpy(om).cuda(), 32, 2)
    torch.cuda.synchronize()
    fac = fac.float().cpu().numpy().astype(np.float64)
    x = O.bf16_bits_to_f64(kb)
    for h in range(c["Hkv"]):
        X = x[:, h].reshape(-1, 128)
        Fo, _ = F.randomized_factor(X, om[h].astype(np.float64), 32, 2)
        e_gpu = np.linalg.norm(X - (X @ fac[h].T) @ fac[h]) ** 2
        e_ora = np.linalg.norm(X - (X @ Fo.T) @ Fo) ** 2
        assert e_gpu <= e_ora * (1 + 1e-3), (h, e_gpu / e_ora)


@pytest.mark.gpu
def test_prefill_fit_then_bulk_append_codes_and_decode():
    """Fit the factors of a prefill, append every prefill token in one call
    (n_new = the prefill length), and check the stored codes against the
    oracle's quantizer and a decode over them against the oracle."""
    import torch

    from rank_bit_kv_b200 import kvc
    from tests.gpu_util import assert_close
    from tests.test_gpu_append import check_int4

    c = synth.config("c2", B=2, T=1024, rope=1)
    kb, vb = synth.prefill_kv(c, c["T"])
    omk = synth.gaussian_test_matrix(c["Hkv"], 128, 48, seed=1)
    omv = synth.gaussian_test_matrix(c["Hkv"], 128, 64, seed=2)
    bk, _ = kvc.fit_factors(to_dev_bf16(kb), torch.from_numpy(omk).cuda(), c["rk"], 1)
    bv, _ = kvc.fit_factors(to_dev_bf16(vb), torch.from_numpy(omv).cuda(), c["rv"], 1)
    lay = kvc.Layout(kvc.desc_from_config(c))
    cache = kvc.Cache(lay)
    cache.bufs["bk"].copy_(bk.view(torch.uint8).reshape(-1))
    cache.bufs["bv"].copy_(bv.view(torch.uint8).reshape(-1))
    kvc.append(lay, cache, to_dev_bf16(kb), to_dev_bf16(vb), [0, 0], c["T"])
    torch.cuda.synchronize()
    fk = bk.float().cpu().numpy().astype(np.float64)
    fv = bv.float().cpu().numpy().astype(np.float64)
    rows = (c["B"], c["Hkv"], c["T"])
    x = {"k": O.bf16_bits_to_f64(kb), "v": O.bf16_bits_to_f64(vb)}
    for comp, r, fac in (("k", c["rk"], fk), ("v", c["rv"], fv)):
        codes = cache.bufs[f"l{comp}_codes"].cpu().numpy().reshape(rows + (r // 2,))
        sz = cache.bufs[f"l{comp}_sz"].cpu().numpy().view(np.float16).reshape(
            rows + (O.n_groups(r, 32), 2))
        for t in (0, 511, 1023):
            lat = np.einsum("bhd,hrd->bhr", x[comp][:, :, t], fac)
            check_int4(codes[:, :, t], sz[:, :, t], lat, 32, f"{comp} t={t}")
    # decode over the appended cache: the oracle reads the stored codes
    stored = {k: cache.bufs[k].cpu().numpy() for k in ("lk_codes", "lk_sz", "lv_codes", "lv_sz")}
    arrays = dict(q=synth.lowrank_cache(c, T=8)["q"],
                  bk=bk.cpu().numpy(), bv=bv.cpu().numpy(),
                  lk_codes=stored["lk_codes"].reshape(rows + (16,)),
                  lk_sz=stored["lk_sz"].view(np.float16).reshape(rows + (1, 2)),
                  lv_codes=stored["lv_codes"].reshape(rows + (24,)),
                  lv_sz=stored["lv_sz"].view(np.float16).reshape(rows + (2, 2)))
    q = to_dev_bf16(arrays["q"])
    cache.n_tokens = c["T"]
    out = torch.empty(q.shape, device="cuda")
    ws = torch.empty(lay.workspace_bytes(c["T"]), dtype=torch.uint8, device="cuda")
    kvc.decode(lay, cache, q, out, ws)
    torch.cuda.synchronize()
    assert_close(out.cpu().numpy(), O.decode_from_storage(c, arrays, c["T"]), what="fit+append+decode")


def test_fit_host_errors():
    import ctypes as C

    from rank_bit_kv_b200 import build, kvc

    build.build()
    lib = kvc.lib()
    f = C.c_void_p(0x10000)
    ws = lib.kvc_fit_workspace_bytes(8)
    assert ws > 0
    st = lib.kvc_fit_factors(f, 1, 8, 64, 64, 64, f, 48, 32, 1, f, None, f, ws, None)
    assert kvc.STATUS[st] == "KVC_EUNSUPPORTED"                     # head_dim 64
    st = lib.kvc_fit_factors(f, 1, 8, 64, 64, 128, f, 47, 32, 1, f, None, f, ws, None)
    assert kvc.STATUS[st] == "KVC_EINVAL"                           # odd sketch width
    st = lib.kvc_fit_factors(f, 1, 8, 64, 64, 128, f, 48, 49, 1, f, None, f, ws, None)
    assert kvc.STATUS[st] == "KVC_EINVAL"                           # rank > k
    st = lib.kvc_fit_factors(f, 1, 8, 64, 64, 128, f, 48, 32, 1, f, None, f, ws - 1, None)
    assert kvc.STATUS[st] == "KVC_EWORKSPACE"
    st = lib.kvc_fit_factors(C.c_void_p(0x10004), 1, 8, 64, 64, 128, f, 48, 32, 1, f, None, f, ws,
                             None)
    assert kvc.STATUS[st] == "KVC_EALIGN"
