"""Helpers for the GPU parity tests: run the library on synthetic storage arrays
and compare with the oracle under the acceptance tolerance."""

import numpy as np

# Decode acceptance: max-abs error <= 1e-2 and relative L2 error <= 2e-3
# against the fp64 oracle on identical integer codes.
MAX_ABS = 1e-2
REL_L2 = 2e-3


def assert_close(got, ref, max_abs=MAX_ABS, rel_l2=REL_L2, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref).max() if got.size else 0.0
    den = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / den if den > 0 else np.linalg.norm(got - ref)
    assert err <= max_abs and rel <= rel_l2, f"{what}: max-abs {err:.3e}, rel-L2 {rel:.3e}"
    return err, rel


def run_decode(cfg, arrays, n_tokens, capacity=None, out_bf16=0, seq_lens=None, q=None):
    """Upload the storage arrays, run kvc_decode_attn once, return the output (numpy f32)."""
    import torch

    from rank_bit_kv_b200 import kvc

    lay = kvc.Layout(kvc.desc_from_config(cfg, capacity=capacity, out_bf16=out_bf16))
    cache = kvc.Cache(lay, fill=arrays)
    cache.n_tokens = n_tokens
    if seq_lens is not None:
        cache.seq_lens = torch.tensor(np.asarray(seq_lens, np.int32), device="cuda")
    qa = arrays["q"] if q is None else q
    qt = torch.from_numpy(np.ascontiguousarray(qa).view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty(qt.shape, device="cuda",
                      dtype=torch.bfloat16 if out_bf16 else torch.float32)
    ws = torch.empty(max(lay.workspace_bytes(n_tokens), 16), dtype=torch.uint8, device="cuda")
    ws[:16].zero_()
    kvc.decode(lay, cache, qt, out, ws)
    torch.cuda.synchronize()
    # word 0 of the workspace: a bounded wait of a tensor-core kernel gave up
    assert int(ws[:4].view(torch.int32).item()) == 0, "decode error word set"
    return out.float().cpu().numpy()


def desc_of(cfg):
    return dict(cfg)
