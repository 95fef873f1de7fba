"""C ABI checks that need no GPU: the library loads, exports every symbol the
header declares, validates layouts, and computes the closed-form sizes."""

import ctypes as C
import os
import re

import numpy as np
import pytest

from rank_bit_kv_b200 import build, kvc, synth
from oracle import kvc_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return kvc.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "kvc.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(kvc_\w+)\s*\(", src, re.M)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "kvc_decode_attn" in names and "kvc_append" in names and "kvc_create_layout" in names
    for n in names:
        assert hasattr(lib, n), n
    assert lib.kvc_version().startswith(b"kvc")


def test_struct_sizes_match_header(lib):
    # kvc_layout_desc: 18 int32 + float (+ pad) + double = 88 bytes; kvc_cache: 20 pointers +
    # 2 int32 + the status pointer
    assert C.sizeof(kvc.LayoutDesc) == 88
    assert C.sizeof(kvc.CacheDesc) == 20 * 8 + 8 + 8


@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c4", "c5"])
def test_layouts_of_every_workload(lib, name):
    c = synth.config(name)
    lay = kvc.Layout(kvc.desc_from_config(c))
    sizes = lay.buffer_sizes()
    if c["kind"] == "lowrank":
        per = O.lowrank_bytes_per_token_head(c["rk"], c["rv"], c["bits"], c["g"], c["resid"], c["d"])
        assert lay.step_bytes(c["T"]) == per * c["B"] * c["Hkv"] * c["T"]
        stored = sum(v for k, v in sizes.items() if k[:2] in ("lk", "lv", "rk", "rv"))
        assert stored == per * c["B"] * c["Hkv"] * c["T"]
        assert sizes["bk"] == c["Hkv"] * c["rk"] * c["d"] * 2
    if name == "c2":
        assert lay.step_bytes(c["T"]) == 109051904
    if name == "c3":
        assert lay.step_bytes(c["T"]) == 71303168
    if name == "c5":
        assert lay.step_bytes(c["T"]) == 1073741824
        assert sizes["page_table"] == 262144
    if name == "c4":
        assert abs(lay.step_bytes(c["T"]) - 23.96e6) / 23.96e6 < 2e-3
    assert lay.workspace_bytes(c["T"]) >= lay.workspace_bytes(c["T"] // 2) > 0
    assert lay.decode_launches(c["T"]) in (2, 3)


def test_buffer_sizes_cover_synthetic_arrays(lib):
    for name in ("c1", "c2", "c5"):
        c = synth.config(name)
        lay = kvc.Layout(kvc.desc_from_config(c, capacity=64))
        a = synth.lowrank_cache(c, T=64)
        sizes = lay.buffer_sizes()
        for k, v in a.items():
            if k in sizes:
                assert a[k].nbytes == sizes[k], (name, k)


@pytest.mark.parametrize("bad,status", [
    (dict(head_dim=96), kvc.STATUS and 2),
    (dict(n_q_heads=6, n_kv_heads=4), 1),
    (dict(rank_k=3), 1),
    (dict(resid_bits=3), 2),
    (dict(resid_bits=2, head_dim=64), 2),
    (dict(page_size=8), 2),
    (dict(batch=0), 1),
    (dict(batch=1000), 1),
    (dict(max_tokens=0), 1),
    (dict(rope=1, rope_theta=0.0), 1),
])
def test_invalid_layouts_rejected(lib, bad, status):
    base = dict(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, max_tokens=64, rank_k=32,
                rank_v=48, latent_bits=4, group_size=32)
    base.update(bad)
    with pytest.raises(kvc.KvcError) as ei:
        kvc.Layout(kvc.make_desc("lowrank", **base))
    assert ei.value.status == status
    assert lib.kvc_last_error()


@pytest.mark.parametrize("D", [640, 768, 1024])
def test_block_shared_latent_wider_than_512_rejected(lib, D):
    """The decode kernels keep at most 64 accumulators per thread for the 32
    queries of a CTA, i.e. latent widths up to 512; wider ones are refused at
    layout creation rather than decoded wrongly."""
    with pytest.raises(kvc.KvcError) as ei:
        kvc.Layout(kvc.make_desc("block_shared", batch=1, n_q_heads=32, n_kv_heads=8,
                                 head_dim=128, max_tokens=16, n_layers=4, latent_dim=D,
                                 group_size=64))
    assert kvc.STATUS[ei.value.status] == "KVC_EINVAL" and b"latent_dim" in lib.kvc_last_error()


def test_kind_flag_conflicts(lib):
    with pytest.raises(kvc.KvcError):
        kvc.Layout(kvc.make_desc("varrate", batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128,
                                 max_tokens=16, rank_k=32, rank_v=64, latent_bits=4, group_size=32))
    with pytest.raises(kvc.KvcError):
        kvc.Layout(kvc.make_desc("dense", batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128,
                                 max_tokens=16, rope=1, rope_theta=1e4))
    with pytest.raises(kvc.KvcError):
        kvc.Layout(kvc.make_desc("block_shared", batch=1, n_q_heads=8, n_kv_heads=2,
                                 head_dim=128, max_tokens=16, n_layers=1, latent_dim=512,
                                 group_size=64))   # 8 queries: not a multiple of 32


def _layout_c2(**over):
    c = synth.config("c2", B=2, T=64)
    return kvc.Layout(kvc.desc_from_config(c, capacity=64)), c


def test_decode_host_errors_launch_nothing(lib):
    """Errors that the host detects return before any CUDA call (no GPU needed)."""
    lay, c = _layout_c2()
    cs = kvc.CacheDesc()
    fake = 0x10000  # 16-byte aligned, never dereferenced: every check fails first
    for n in ("lk_codes", "lk_sz", "lv_codes", "lv_sz", "bk", "bv"):
        setattr(cs, n, fake)
    cs.n_tokens = 65
    q = out = C.c_void_p(fake)
    st = lib.kvc_decode_attn(lay.h, C.byref(cs), q, out, C.c_void_p(fake), 1 << 30, None)
    assert kvc.STATUS[st] == "KVC_ECAPACITY"
    cs.n_tokens = 64
    st = lib.kvc_decode_attn(lay.h, C.byref(cs), q, out, C.c_void_p(fake), 16, None)
    assert kvc.STATUS[st] == "KVC_EWORKSPACE"
    cs.lk_sz = None
    st = lib.kvc_decode_attn(lay.h, C.byref(cs), q, out, C.c_void_p(fake), 1 << 30, None)
    assert kvc.STATUS[st] == "KVC_EINVAL" and b"lk_sz" in lib.kvc_last_error()
    cs.lk_sz = fake + 4
    st = lib.kvc_decode_attn(lay.h, C.byref(cs), q, out, C.c_void_p(fake), 1 << 30, None)
    assert kvc.STATUS[st] == "KVC_EALIGN"
    cs.lk_sz = fake
    st = lib.kvc_decode_attn(lay.h, C.byref(cs), C.c_void_p(fake + 2), out, C.c_void_p(fake),
                             1 << 30, None)
    assert kvc.STATUS[st] == "KVC_EALIGN"


def test_append_host_errors(lib):
    """kvc_append takes pos (and the VARRATE ranks) as device arrays: the host
    checks pointers, alignment and sizes and returns before any CUDA call;
    the values themselves are the kernels' to check (tested on the GPU)."""
    lay, c = _layout_c2()
    cs = kvc.CacheDesc()
    fake = 0x10000                   # 16-byte aligned, never dereferenced
    for n in ("lk_codes", "lk_sz", "lv_codes", "lv_sz", "bk", "bv"):
        setattr(cs, n, fake)
    f = C.c_void_p(fake)
    st = lib.kvc_append(lay.h, C.byref(cs), f, f, None, 1, None, None)
    assert kvc.STATUS[st] == "KVC_EINVAL"                   # NULL pos
    st = lib.kvc_append(lay.h, C.byref(cs), f, f, C.c_void_p(fake + 4), 1, None, None)
    assert kvc.STATUS[st] == "KVC_EALIGN"                   # pos not 16-byte aligned
    st = lib.kvc_append(lay.h, C.byref(cs), f, f, f, 65, None, None)
    assert kvc.STATUS[st] == "KVC_ECAPACITY"                # n_new > max_tokens (64)
    st = lib.kvc_append(lay.h, C.byref(cs), f, f, f, 0, None, None)
    assert kvc.STATUS[st] == "KVC_EINVAL"                   # n_new < 1
    st = lib.kvc_append(lay.h, C.byref(cs), f, None, f, 1, None, None)
    assert kvc.STATUS[st] == "KVC_EINVAL"                   # v_new NULL
    cs.status = fake + 2
    st = lib.kvc_append(lay.h, C.byref(cs), f, f, f, 1, None, None)
    assert kvc.STATUS[st] == "KVC_EALIGN" and b"status" in lib.kvc_last_error()
    cs.status = None
    cs.lk_sz = None
    st = lib.kvc_append(lay.h, C.byref(cs), f, f, f, 1, None, None)
    assert kvc.STATUS[st] == "KVC_EINVAL" and b"lk_sz" in lib.kvc_last_error()
    # VARRATE: the ranks are required and must be aligned
    c4 = synth.config("c4", T=16)
    lay4 = kvc.Layout(kvc.desc_from_config(c4))
    cs4 = kvc.CacheDesc()
    for n in ("lk_codes", "lv_codes", "offset_k", "offset_v", "rank_k", "rank_v", "bk", "bv"):
        setattr(cs4, n, fake)
    st = lib.kvc_append(lay4.h, C.byref(cs4), f, f, f, 1, None, None)
    assert kvc.STATUS[st] == "KVC_EINVAL" and b"new_ranks" in lib.kvc_last_error()
    st = lib.kvc_append(lay4.h, C.byref(cs4), f, f, f, 1, C.c_void_p(fake + 1), None)
    assert kvc.STATUS[st] == "KVC_EALIGN"


def test_static_entry_points_validate_before_enqueueing(lib):
    """The workspace-free decode refuses bad calls without touching the GPU:
    its scratch lookup and every enqueue come after the host checks."""
    lay, c = _layout_c2()
    cs = kvc.CacheDesc()
    st = lib.kvc_decode_attn_static(None, C.byref(cs), None, None, None)
    assert kvc.STATUS[st] == "KVC_EINVAL"
    st = lib.kvc_static_error_word(None, None)
    assert kvc.STATUS[st] == "KVC_EINVAL"


def test_header_cites_a_passage_beside_each_operation():
    """Each entry point that computes part of the method names the page and
    section that define it in its own comment."""
    src = open(os.path.join(ROOT, "include", "kvc.h")).read()
    for fn in ("kvc_create_layout", "kvc_append", "kvc_decode_attn", "kvc_buffer_sizes",
               "kvc_step_bytes"):
        i = re.search(rf"^[\w ]+\*?\s*\b{fn}\(", src, re.M).start()   # the declaration
        j = src.rindex("/*", 0, i)
        comment = src[j:i]
        assert re.search(r'"[^"]+"', comment), fn          # a quoted page or section title


def test_library_has_no_oracle_dependency():
    """The product side never imports, links or reads the oracle."""
    pat = re.compile(r"(^\s*(from|import)\s+oracle)|kvc_oracle|oracle/", re.M)
    for root, _, files in os.walk(os.path.join(ROOT, "rank_bit_kv_b200")):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(root, f)).read()
                assert not pat.search(src), f
