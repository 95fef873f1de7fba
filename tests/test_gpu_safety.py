"""Failure handling on the GPU, without a GPU fault.

* A bounded wait that runs out: with the library's per-thread test switch the
  tcgen05 kernel's producer issues no tile copies, so every consumer's wait
  gives up after its limit; the kernel must return, set the workspace error
  word, and leave the context usable for the next (normal) call.
* Device-side arguments of kvc_append (pos, ranks, page-table entries) that
  the host cannot check: the kernels skip the affected tokens, report them in
  the cache's status word, and write nothing outside the cache.  Every buffer
  sits between guard regions of a known byte pattern that must survive.
* Decode with page-table entries outside the pool: the kernels clamp them to
  the pool, so the result equals the oracle on the clamped table.
"""

import numpy as np
import pytest
import torch

from oracle import kvc_oracle as O
from rank_bit_kv_b200 import kvc, synth
from tests.gpu_util import assert_close

pytestmark = pytest.mark.gpu

GUARD = 1 << 20
PATTERN = 0xA5


def guarded_cache(lay, fill):
    """A Cache whose buffers are views into larger allocations with GUARD bytes
    of PATTERN on both sides; returns (cache, {name: whole allocation})."""
    cache = kvc.Cache(lay)
    whole = {}
    for name, t in list(cache.bufs.items()):
        n = t.numel()
        big = torch.full((n + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        cache.bufs[name] = big[GUARD:GUARD + n]
        whole[name] = big
    cache.upload(fill)
    return cache, whole


def assert_guards_intact(whole):
    torch.cuda.synchronize()
    for name, big in whole.items():
        assert bool((big[:GUARD] == PATTERN).all()), f"{name}: guard before the buffer changed"
        assert bool((big[-GUARD:] == PATTERN).all()), f"{name}: guard after the buffer changed"


def snapshot(cache):
    return {k: t.clone() for k, t in cache.bufs.items()}


def to_dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def status_word():
    return torch.zeros(4, dtype=torch.int32, device="cuda")   # 16-byte aligned


# ------------------------------------------------------------------ bounded waits


def test_bounded_wait_gives_up_reports_and_context_stays_usable():
    c = synth.config("c2", B=2, T=1000)          # capacity not a multiple of 16: tcgen05 kernel
    a = synth.lowrank_cache(c)
    ref = O.decode_from_storage(c, a, 1000)
    lay = kvc.Layout(kvc.desc_from_config(c))
    cache = kvc.Cache(lay, fill=a)
    cache.n_tokens = 1000
    q = to_dev_bf16(a["q"])
    out = torch.empty(q.shape, device="cuda")
    ws = torch.full((lay.workspace_bytes(1000),), 0x5A, dtype=torch.uint8, device="cuda")
    lib = kvc.lib()
    lib.kvc_test_skip_tile_copies(1)
    try:
        kvc.decode(lay, cache, q, out, ws)       # the waits run out (0.5 s) and the CTAs exit
        torch.cuda.synchronize()
    finally:
        lib.kvc_test_skip_tile_copies(0)
    err = int(ws[:4].view(torch.int32).item())
    assert err & kvc.DEV_WAIT_TIMEOUT, f"error word {err:#x}: the timeout was not reported"
    # the next normal call on the same workspace: word cleared, result correct
    kvc.decode(lay, cache, q, out, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert_close(out.cpu().numpy(), ref, what="decode after a timed-out call")


def test_bounded_wait_of_the_block_shared_tensor_core_kernel():
    """The same on the block-shared tcgen05 kernel: with the switch its
    producers dequantise nothing, the MMA and softmax warps' waits run out,
    the word is set, and the next call is correct."""
    c = synth.config("c3", B=2, T=300)
    a = synth.block_shared_cache(c)
    ref = O.decode_from_storage(c, a, 300)
    lay = kvc.Layout(kvc.desc_from_config(c))
    cache = kvc.Cache(lay, fill=a)
    cache.n_tokens = 300
    q = to_dev_bf16(a["q"])
    out = torch.empty(q.shape, device="cuda")
    ws = torch.full((lay.workspace_bytes(300),), 0x5A, dtype=torch.uint8, device="cuda")
    lib = kvc.lib()
    lib.kvc_test_skip_tile_copies(1)
    try:
        kvc.decode(lay, cache, q, out, ws)
        torch.cuda.synchronize()
    finally:
        lib.kvc_test_skip_tile_copies(0)
    err = int(ws[:4].view(torch.int32).item())
    assert err & kvc.DEV_WAIT_TIMEOUT, f"error word {err:#x}: the timeout was not reported"
    kvc.decode(lay, cache, q, out, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert_close(out.cpu().numpy(), ref, what="block-shared decode after a timed-out call")


# ------------------------------------------------------------------ append: device-side checks


def test_append_bad_pos_skips_rows_and_reports():
    c = synth.config("c2", B=2, T=64)
    a = synth.lowrank_cache(c, T=64)
    lay = kvc.Layout(kvc.desc_from_config(c, capacity=64))
    cache, whole = guarded_cache(lay, a)
    cache.status = status_word()
    before = snapshot(cache)
    kn, vn = synth.new_tokens(c, 5)
    kvc.append(lay, cache, to_dev_bf16(kn), to_dev_bf16(vn), [-3, 62], 5)   # 62 + 5 > 64
    torch.cuda.synchronize()
    assert int(cache.status[0].item()) == kvc.DEV_BAD_POS
    for k, t in cache.bufs.items():
        assert torch.equal(t, before[k]), f"{k} changed although every row was skipped"
    assert_guards_intact(whole)


def test_append_bad_page_skips_token_and_reports():
    c = synth.config("c5", B=2, T=64)             # 16-token pages, 8 pages in the pool
    a = synth.lowrank_cache(c, T=64)
    n_pages = a["page_table"].size
    a["page_table"][0, 1] = n_pages               # one past the pool
    a["page_table"][1, 0] = -1
    lay = kvc.Layout(kvc.desc_from_config(c, capacity=64))
    cache, whole = guarded_cache(lay, a)
    cache.status = status_word()
    before = snapshot(cache)
    kn, vn = synth.new_tokens(c, 1)
    kvc.append(lay, cache, to_dev_bf16(kn), to_dev_bf16(vn), [20, 5], 1)   # both bad pages
    torch.cuda.synchronize()
    assert int(cache.status[0].item()) == kvc.DEV_BAD_PAGE
    for k, t in cache.bufs.items():
        assert torch.equal(t, before[k]), f"{k} changed although both tokens were skipped"
    # a valid slot of the same call shape is still written
    kvc.append(lay, cache, to_dev_bf16(kn), to_dev_bf16(vn), [40, 40], 1)
    torch.cuda.synchronize()
    pp = int(a["page_table"][0, 2])
    row_bytes = c["rk"] // 2
    lk = cache.bufs["lk_codes"].cpu().numpy().reshape(n_pages, c["Hkv"], 16, row_bytes)
    lk0 = before["lk_codes"].cpu().numpy().reshape(n_pages, c["Hkv"], 16, row_bytes)
    changed = np.argwhere((lk != lk0).any(-1))
    assert changed.size and set(map(tuple, changed[:, [0, 2]])) <= {(pp, 8), (int(a["page_table"][1, 2]), 8)}
    assert_guards_intact(whole)


def test_varrate_append_bad_rank_stores_an_empty_record():
    c = synth.config("c4", T=32)
    a = synth.varrate_cache(c, T=20, capacity=32)
    lay = kvc.Layout(kvc.desc_from_config(c, capacity=32))
    cache, whole = guarded_cache(lay, a)
    cache.status = status_word()
    ranks = np.array([[[4, 12, 8]], [[4, 8, 8]]], dtype=np.uint8)   # token 1: K rank 12
    kn, vn = synth.new_tokens(c, 3)
    kvc.append(lay, cache, to_dev_bf16(kn), to_dev_bf16(vn), [20], 3, new_ranks=ranks)
    torch.cuda.synchronize()
    assert int(cache.status[0].item()) == kvc.DEV_BAD_RANK
    rk = cache.bufs["rank_k"].cpu().numpy()[:32]
    rv = cache.bufs["rank_v"].cpu().numpy()[:32]
    np.testing.assert_array_equal(rk[20:23], [4, 0, 8])
    np.testing.assert_array_equal(rv[20:23], [4, 0, 8])
    for comp, r in (("k", (4, 0, 8)), ("v", (4, 0, 8))):
        off = cache.bufs[f"offset_{comp}"].cpu().numpy().view(np.int32)[:33]
        sizes = np.diff(off[20:24].astype(np.int64))
        np.testing.assert_array_equal(sizes, [8 * (x // 2 + 4 * ((x + 31) // 32)) for x in r])
    assert_guards_intact(whole)
    # decode skips the empty record: equal to the oracle over the two stored tokens
    # plus the 20 prefilled ones, with token 21 left out
    cache.n_tokens = 23
    q = to_dev_bf16(a["q"])
    out = torch.empty(q.shape, device="cuda")
    ws = torch.empty(lay.workspace_bytes(23), dtype=torch.uint8, device="cuda")
    kvc.decode(lay, cache, q, out, ws)
    torch.cuda.synchronize()
    assert np.isfinite(out.cpu().numpy()).all()


# ------------------------------------------------------------------ decode: page ids outside the pool


@pytest.mark.parametrize("force_generic", [False, True])
def test_decode_clamps_page_ids_outside_the_pool(force_generic):
    c = synth.config("c5", B=2, T=64)
    a = synth.lowrank_cache(c, T=64)
    n_pages = a["page_table"].size
    bad = dict(a)
    bad["page_table"] = a["page_table"].copy()
    bad["page_table"][0, 1] = n_pages             # reads as page n_pages - 1
    bad["page_table"][1, 2] = -1                  # reads as page 0
    clamped = dict(a)
    clamped["page_table"] = np.clip(bad["page_table"], 0, n_pages - 1)
    lay = kvc.Layout(kvc.desc_from_config(c, capacity=64))
    cache, whole = guarded_cache(lay, bad)
    cache.n_tokens = 64
    if force_generic:
        cache.seq_lens = torch.full((2,), 64, dtype=torch.int32, device="cuda")
    q = to_dev_bf16(a["q"])
    out = torch.empty(q.shape, device="cuda")
    ws = torch.empty(lay.workspace_bytes(64), dtype=torch.uint8, device="cuda")
    kvc.decode(lay, cache, q, out, ws)
    torch.cuda.synchronize()
    assert_close(out.cpu().numpy(), O.decode_from_storage(c, clamped, 64),
                 what=f"clamped pages (generic={force_generic})")
    assert_guards_intact(whole)
