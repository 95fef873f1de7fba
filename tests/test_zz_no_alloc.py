"""Decode without a caller-provided workspace (kvc_decode_attn_static).

Some callers cannot allocate device memory: code embedded in a host framework
that owns every device allocation and exposes no allocator, or a serving loop
that must not call cudaMalloc because it can synchronize the device.  For them
the library has one entry point that allocates nothing and runs the same decode
with a fixed scratch area compiled into the library.  These tests compare its
output with kvc_decode_attn given a caller workspace, on two calls in a row (the
area keeps the previous call's contents), within the decode tolerance of the
parity tests, and check that a layout needing more scratch than the area holds
is refused before anything runs.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""

import numpy as np
import pytest
import torch

from rank_bit_kv_b200 import kvc, synth
from tests.gpu_util import MAX_ABS, REL_L2, assert_close

pytestmark = pytest.mark.gpu


def _setup(cfg):
    a = synth.lowrank_cache(cfg)
    lay = kvc.Layout(kvc.desc_from_config(cfg))
    cache = kvc.Cache(lay, fill=a)
    cache.n_tokens = cfg["T"]
    q = torch.from_numpy(a["q"].view(np.int16)).cuda().view(torch.bfloat16)
    return lay, cache, q


@pytest.mark.parametrize("name,over", [
    ("c2", {}),                     # Llama-8B layer, 32K context: warp-level pre-RoPE kernel
    ("c2", {"B": 2, "T": 1000}),    # capacity not a multiple of 16: tcgen05 pre-RoPE kernel,
                                    # the one whose bounded waits use the error word
    ("c5", {"B": 2, "T": 1000}),    # paged, rotated residual: warp-level latent-space kernel
])
def test_static_scratch_decode_matches_workspace_decode(name, over):
    cfg = synth.config(name, **over)
    lay, cache, q = _setup(cfg)
    assert lay.workspace_bytes(cfg["T"]) <= kvc.STATIC_SCRATCH_BYTES
    ref = torch.empty(q.shape, device="cuda")
    ws = torch.empty(lay.workspace_bytes(cfg["T"]), dtype=torch.uint8, device="cuda")
    kvc.decode(lay, cache, q, ref, ws)
    torch.cuda.synchronize()
    ref = ref.cpu().numpy()
    word = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = torch.full(q.shape, float("nan"), device="cuda")
        kvc.decode_static(lay, cache, q, out)
        kvc.static_error_word(word)
        torch.cuda.synchronize()
        assert_close(out.cpu().numpy(), ref, MAX_ABS, REL_L2, what=f"{name} static call {call}")
        assert int(word[0].item()) == 0, "the built-in scratch area reports an aborted wait"


def test_static_scratch_refuses_layouts_beyond_its_size():
    cfg = synth.config("c3")                     # 4 layers x 32 heads x 512 latent: large scratch
    lay = kvc.Layout(kvc.desc_from_config(cfg))
    assert lay.workspace_bytes(cfg["T"]) > kvc.STATIC_SCRATCH_BYTES
    cache = kvc.Cache(lay)
    cache.n_tokens = cfg["T"]
    q = torch.zeros(cfg["L"], cfg["B"], cfg["Hq"], cfg["d"], dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(q.shape, device="cuda")
    with pytest.raises(kvc.KvcError) as ei:
        kvc.decode_static(lay, cache, q, out)
    assert kvc.STATUS[ei.value.status] == "KVC_EWORKSPACE"
    assert "scratch" in str(ei.value)
