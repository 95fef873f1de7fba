"""GPU decode parity: the CUDA path through the C ABI against the fp64 oracle on
identical seeded integer codes.  Small cases compare every output; the
full-size workloads (the launch configuration the benchmark times) compare
sampled rows that the oracle recomputes on their own."""

import numpy as np
import pytest

from oracle import kvc_oracle as O
from rank_bit_kv_b200 import synth
from tests.gpu_util import assert_close, run_decode

pytestmark = pytest.mark.gpu


def oracle(cfg, arrays, n):
    return O.decode_from_storage(cfg, arrays, n)


def sub_batch(arrays, rows, keys):
    out = dict(arrays)
    for k in keys:
        if k in out:
            out[k] = arrays[k][rows]
    return out


# ------------------------------------------------------------------ tiny / small


@pytest.mark.parametrize("T", [1, 100, 512])
def test_c1_tiny_single_head(T):
    c = synth.config("c1")
    a = synth.lowrank_cache(c)                  # 512 slots, attend to the first T
    got = run_decode(c, a, T, capacity=512)
    assert_close(got, oracle(c, a, T), what=f"c1 T={T}")


@pytest.mark.parametrize("rope", [0, 1])
@pytest.mark.parametrize("T", [1000, 4161])
def test_c2_shape_small_context(rope, T):
    c = synth.config("c2", B=2, T=T, rope=rope)
    a = synth.lowrank_cache(c)
    got = run_decode(c, a, T)
    assert_close(got, oracle(c, a, T), what=f"c2 rope={rope} T={T}")


def test_c2_quantized_gaussian_latents():
    """Codes produced from N(0,1) latents by the reference quantizer."""
    c = synth.config("c2", B=1, T=777)
    a = synth.lowrank_cache(c)
    lk, lv = synth.gaussian_latents(c, 777)
    for name, lat in (("lk", lk), ("lv", lv)):
        codes, s, z = O.quantize_int4_asym(lat, 32)
        a[f"{name}_codes"] = O.pack_int4(codes)
        a[f"{name}_sz"] = np.stack([s, z], -1).astype(np.float16)
    assert_close(run_decode(c, a, 777), oracle(c, a, 777), what="c2 gaussian")


@pytest.mark.parametrize("mode", ["q_x8", "needle"])
def test_c2_peaked_softmax(mode):
    """The configured scores are nearly uniform; these keep the shapes but
    make the softmax peaked (q scaled by 8, or one planted needle token)."""
    c = synth.config("c2", B=2, T=2048, rope=0)
    a = synth.lowrank_cache(c)
    if mode == "q_x8":
        a["q"] = synth.to_bf16_bits(synth.bf16_bits_to_f32(a["q"]) * 8)
    else:
        q = O.bf16_bits_to_f64(a["q"])
        bk = a["bk"].astype(np.float64)
        for b in range(c["B"]):
            for h in range(c["Hkv"]):
                qt = bk[h] @ q[b, h * 4]                       # first head of the group
                lat = 3 * np.sqrt(32) * qt / np.linalg.norm(qt)
                codes, s_, z_ = O.quantize_int4_asym(lat[None], 32)
                a["lk_codes"][b, h, 1234] = O.pack_int4(codes)[0]
                a["lk_sz"][b, h, 1234] = np.stack([s_, z_], -1).astype(np.float16)[0]
    ref = oracle(c, a, 2048)
    assert_close(run_decode(c, a, 2048), ref, what=mode)


@pytest.mark.parametrize("rope", [0, 1])
def test_c5_shape_small_paged_residual(rope):
    c = synth.config("c5", B=2, T=400, rope=rope, theta=500000.0)
    a = synth.lowrank_cache(c)
    assert_close(run_decode(c, a, 400), oracle(c, a, 400), what=f"c5 rope={rope}")
    assert_close(run_decode(c, a, 333), oracle(c, a, 333), what="c5 ragged")


def test_paging_shuffled_equals_identity_table():
    c = synth.config("c5", B=2, T=256)
    a = synth.lowrank_cache(c)
    ident = dict(a)
    perm = a["page_table"].reshape(-1)
    comps = ("lk_codes", "lk_sz", "lv_codes", "lv_sz", "rk_codes", "rk_scale", "rv_codes",
             "rv_scale")
    for k in comps:
        ident[k] = a[k][perm]            # logical page j now stored at physical j
    ident["page_table"] = np.arange(perm.size, dtype=np.int32).reshape(a["page_table"].shape)
    g1 = run_decode(c, a, 256)
    g2 = run_decode(c, ident, 256)
    np.testing.assert_allclose(g1, g2, rtol=0, atol=1e-6)


@pytest.fixture(params=["tensor_core", "lane_per_head"])
def varrate_kernel(request):
    """Run a variable-rate test on the lane-per-(KV head, query head) kernel
    (default) and on the tensor-core kernel."""
    from rank_bit_kv_b200 import kvc

    kvc.lib().kvc_select_varrate_kernel(1 if request.param == "tensor_core" else 0)
    yield request.param
    kvc.lib().kvc_select_varrate_kernel(0)


@pytest.mark.parametrize("T", [1, 300, 2000])
def test_c4_shape_small_varrate(T, varrate_kernel):
    c = synth.config("c4", T=T)
    a = synth.varrate_cache(c)
    assert_close(run_decode(c, a, T), oracle(c, a, T), what=f"c4 T={T}")


@pytest.mark.parametrize("D,B,n", [(128, 2, 300), (256, 3, 1000), (384, 4, 640)])
def test_block_shared_latent_widths(D, B, n):
    """Latent widths other than 512: the query projection's MMA tiles and the
    staged combine's split of the W_v rows change with D."""
    c = synth.config("c3", B=B, T=n, D=D)
    a = synth.block_shared_cache(c)
    assert_close(run_decode(c, a, n), oracle(c, a, n), what=f"block-shared D={D} B={B} n={n}")


def test_c3_shape_small_block_shared():
    c = synth.config("c3", B=2, T=300)
    a = synth.block_shared_cache(c)
    assert_close(run_decode(c, a, 300), oracle(c, a, 300), what="c3 small")


def test_dense_bf16_small():
    cfg = dict(kind="dense", B=2, Hq=32, Hkv=8, d=128, T=700)
    a = synth.dense_cache(2, 32, 8, 128, 700, seed=5)
    assert_close(run_decode(cfg, a, 700), oracle(cfg, a, 700), what="dense")


@pytest.mark.parametrize("G,T", [(4, 1), (4, 16), (4, 17), (1, 300), (8, 1000)])
def test_dense_tensor_core_shapes(G, T):
    """Dense bf16 decode on the warp-level MMA path: GQA groups 1..8, tiles of
    16 tokens with ragged tails, a single token."""
    Hkv = 4
    cfg = dict(kind="dense", B=2, Hq=G * Hkv, Hkv=Hkv, d=128, T=T)
    a = synth.dense_cache(2, G * Hkv, Hkv, 128, T, seed=11 + G)
    assert_close(run_decode(cfg, a, T), oracle(cfg, a, T), what=f"dense G={G} T={T}")


def test_dense_peaked():
    """q x 8: a near one-hot softmax, so the probabilities' own rounding shows."""
    cfg = dict(kind="dense", B=1, Hq=32, Hkv=8, d=128, T=2000)
    a = synth.dense_cache(1, 32, 8, 128, 2000, seed=21)
    q = synth.to_bf16_bits(synth.bf16_bits_to_f32(a["q"]) * 8.0)
    a["q"] = q
    assert_close(run_decode(cfg, a, 2000), oracle(cfg, a, 2000), what="dense peaked")


def test_dense_layered():
    cfg = dict(kind="dense", B=1, Hq=8, Hkv=2, d=128, T=129, L=2)
    a = synth.dense_cache(1, 8, 2, 128, 129, seed=6, n_layers=2)
    assert_close(run_decode(cfg, a, 129), oracle(cfg, a, 129), what="dense layered")


# ------------------------------------------------------------------ edge cases


def test_empty_context_gives_zero():
    c = synth.config("c2", B=2, T=64)
    a = synth.lowrank_cache(c)
    got = run_decode(c, a, 0, capacity=64)
    assert (got == 0).all()


def test_per_row_lengths():
    c = synth.config("c2", B=3, T=900)
    a = synth.lowrank_cache(c)
    lens = [900, 0, 257]
    got = run_decode(c, a, 900, seq_lens=lens)
    for b, n in enumerate(lens):
        sub = sub_batch(a, [b], ("q", "lk_codes", "lk_sz", "lv_codes", "lv_sz"))
        cb = dict(c, B=1)
        if n == 0:
            assert (got[b] == 0).all()
        else:
            assert_close(got[b:b + 1], oracle(cb, sub, n), what=f"row {b} len {n}")


def test_bf16_output():
    """bf16 output is held to the same tolerance as fp32 output: the combine
    rounds once, from fp32, after the division by the softmax sum."""
    c = synth.config("c2", B=1, T=500)
    a = synth.lowrank_cache(c)
    got = run_decode(c, a, 500, out_bf16=1)
    ref = oracle(c, a, 500)
    assert_close(got, ref, what="bf16 out")


def test_bf16_output_full_size_c2():
    """bf16 output on the benchmark workload (all 8 rows) within the stated
    tolerance."""
    from tests import full_size as F

    ex, futs = F.submit_rows("c2", "uniform", list(range(8)))
    c, a = F.build_arrays("c2", "uniform")
    got = run_decode(c, a, c["T"], out_bf16=1)
    rows = F.collect(ex, futs)
    ref = np.stack([rows[b] for b in range(c["B"])])
    assert_close(got, ref, what="c2 full bf16 out")


# ------------------------------------------------------------------ full-size workloads


@pytest.mark.parametrize("variant", ["uniform", "gaussian"])
@pytest.mark.parametrize("name", ["c2", "c5"])
def test_full_size_every_row(name, variant):
    """The full workloads in the launch configuration the benchmark times,
    every batch row compared with the oracle.  The warp-level kernels cut
    equal byte ranges across (row, KV head) units, so a unit boundary can fall
    inside any warp's range: every row is checked, not a sample.  `gaussian`
    uses codes quantized from N(0,1) latents, as the configurations state."""
    from tests import full_size as F

    c0 = synth.config(name)
    ex, futs = F.submit_rows(name, variant, list(range(c0["B"])))   # oracle overlaps the GPU
    c, a = F.build_arrays(name, variant)
    got = run_decode(c, a, c["T"])
    rows = F.collect(ex, futs)
    for b in range(c["B"]):
        assert_close(got[b:b + 1], rows[b][None], what=f"{name} {variant} full b={b}")
    ref = np.stack([rows[b] for b in range(c["B"])])
    assert_close(got, ref, what=f"{name} {variant} full, all rows")


def test_c4_full_size(varrate_kernel):
    c = synth.config("c4")
    a = synth.varrate_cache(c)
    assert_close(run_decode(c, a, c["T"]), oracle(c, a, c["T"]), what="c4 full")


def test_c3_full_size_every_row():
    """Every batch row at full size (KV heads 0 and 7 of each: the oracle's
    per-head reconstruction is the cost)."""
    c = synth.config("c3")
    a = synth.block_shared_cache(c)
    got = run_decode(c, a, c["T"])
    T, d = c["T"], c["d"]
    for b in range(c["B"]):
        codes = O.unpack_int4(a["lk_codes"][[b], :T], c["D"])
        lat = O.dequant_int4_sym(codes, a["lk_sz"][[b], :T].astype(np.float64), c["g"])
        for kvh in (0, 7):
            sl = slice(kvh * d, (kvh + 1) * d)
            q = O.bf16_bits_to_f64(a["q"][:, [b], kvh * 4:(kvh + 1) * 4])     # [L, 1, 4, d]
            ref = O.decode_block_shared(q, lat, a["wk"][:, :, sl].astype(np.float64),
                                        a["wv"][:, :, sl].astype(np.float64), 1, 1 / np.sqrt(d))
            assert_close(got[:, b:b + 1, kvh * 4:(kvh + 1) * 4], ref,
                         what=f"c3 full b={b} kvh={kvh}")


# ------------------------------------------------------------------ tensor-core path


@pytest.mark.parametrize("B,T", [(1, 1), (2, 127), (2, 128), (1, 129), (2, 3000), (3, 8191)])
def test_rope_tensor_core_path_against_oracle_and_generic(B, T):
    """Pre-RoPE INT4 keys run on the tcgen05 kernel; per-row lengths force the
    generic CUDA-core kernel.  Both must match the oracle, and the tensor-core
    kernel must report no aborted wait in the workspace error word."""
    import torch

    from rank_bit_kv_b200 import kvc

    c = synth.config("c2", B=B, T=T)
    a = synth.lowrank_cache(c)
    ref = oracle(c, a, T)
    lay = kvc.Layout(kvc.desc_from_config(c))
    cache = kvc.Cache(lay, fill=a)
    cache.n_tokens = T
    q = torch.from_numpy(a["q"].view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty(q.shape, device="cuda")
    ws = torch.zeros(lay.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    kvc.decode(lay, cache, q, out, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0, "a bounded wait gave up"
    fast = out.cpu().numpy()
    assert_close(fast, ref, what=f"tcgen05 B={B} T={T}")
    cache.seq_lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
    kvc.decode(lay, cache, q, out, ws)
    torch.cuda.synchronize()
    assert_close(out.cpu().numpy(), ref, what=f"generic B={B} T={T}")


# ------------------------------------------------------------------ latent-space tensor-core path


@pytest.mark.parametrize("rv,resid,page,Hq,B,n,cap", [
    (64, 2, 16, 32, 2, 400, 400),     # C5 shape, paged, whole pages
    (64, 2, 16, 32, 2, 333, 400),     # ragged last page
    (64, 2, 0, 8, 1, 1, 32),          # one token, contiguous, one query head per KV head
    (48, 0, 0, 32, 2, 1000, 1008),    # C2 ranks without RoPE, contiguous
    (48, 2, 16, 16, 3, 4111, 4112),   # two query heads per KV head
    (32, 0, 16, 64, 2, 2049, 2064),   # eight query heads per KV head
    (32, 2, 0, 32, 1, 17, 32),        # one full tile and one token
])
def test_latent_tensor_core_path(rv, resid, page, Hq, B, n, cap):
    """INT4 low-rank layouts without RoPE run on the warp-level mma.sync kernel
    (latent-space scores; codes used as MMA operands without dequantization).
    Per-row lengths force the generic CUDA-core kernel; both must match the oracle."""
    c = synth.config("c5", B=B, Hq=Hq, T=cap, rv=rv, resid=resid, page=page, seed=11 + rv)
    a = synth.lowrank_cache(c)
    ref = oracle(c, a, n)
    assert_close(run_decode(c, a, n, capacity=cap), ref, what=f"latent mma rv={rv} n={n}")
    got = run_decode(c, a, n, capacity=cap, seq_lens=[n] * B)
    assert_close(got, ref, what=f"generic rv={rv} n={n}")


def test_latent_tensor_core_peaked():
    """q scaled by 8: scores spread over tens of log2 units, so the lazily raised
    softmax maximum is raised many times inside a warp's range."""
    c = synth.config("c5", B=2, T=4096)
    a = synth.lowrank_cache(c)
    a["q"] = synth.to_bf16_bits(synth.bf16_bits_to_f32(a["q"]) * 8)
    assert_close(run_decode(c, a, 4096), oracle(c, a, 4096), what="latent peaked")


# ------------------------------------------------------------------ pre-RoPE keys on warp-level MMAs


@pytest.fixture(params=["tcgen05_wg", "mma_sync"])
def rope_kernel(request):
    """Runs a test on both pre-RoPE kernels: the warp-level mma.sync kernel (the
    default) and the tcgen05 warpgroup kernel."""
    from rank_bit_kv_b200 import kvc

    kvc.lib().kvc_select_rope_kernel(1 if request.param == "mma_sync" else 2)
    yield request.param
    kvc.lib().kvc_select_rope_kernel(0)


@pytest.mark.parametrize("rv,page,Hq,B,n,cap", [
    (48, 0, 32, 2, 4096, 4096),       # C2 ranks, whole 128-token tiles
    (48, 0, 32, 2, 4001, 4016),       # ragged last tile, capacity not a multiple of 128
    (48, 0, 32, 1, 1, 16),            # one token
    (32, 16, 16, 3, 1234, 1248),      # paged, two query heads per KV head
    (64, 0, 64, 2, 777, 784),         # eight query heads per KV head
    (48, 16, 32, 3, 2049, 2064),      # paged, C2 ranks, a unit boundary inside most ranges
])
def test_rope_mma_path(rope_kernel, rv, page, Hq, B, n, cap):
    """Pre-RoPE INT4 keys with a capacity that is a multiple of 16 run on the
    tensor-core kernels (tcgen05 reconstruction in TMEM, or reconstruction on
    mma.sync); per-row lengths force the generic kernel.  All match the oracle."""
    c = synth.config("c2", B=B, Hq=Hq, T=cap, rv=rv, page=page, seed=21 + rv)
    a = synth.lowrank_cache(c)
    ref = oracle(c, a, n)
    assert_close(run_decode(c, a, n, capacity=cap), ref, what=f"{rope_kernel} rv={rv} n={n}")
    got = run_decode(c, a, n, capacity=cap, seq_lens=[n] * B)
    assert_close(got, ref, what=f"generic rv={rv} n={n}")


def test_rope_mma_peaked(rope_kernel):
    c = synth.config("c2", B=2, T=2048)
    a = synth.lowrank_cache(c)
    a["q"] = synth.to_bf16_bits(synth.bf16_bits_to_f32(a["q"]) * 8)
    assert_close(run_decode(c, a, 2048), oracle(c, a, 2048), what=f"{rope_kernel} peaked")


def test_rope_kernels_agree_at_full_size():
    """The two pre-RoPE tensor-core kernels on the benchmark workload (every
    row): both within the tolerance of each other's oracle-checked result."""
    from rank_bit_kv_b200 import kvc

    c = synth.config("c2")
    a = synth.lowrank_cache(c)
    got_mma = run_decode(c, a, c["T"])
    kvc.lib().kvc_select_rope_kernel(2)
    try:
        got_wg = run_decode(c, a, c["T"])
    finally:
        kvc.lib().kvc_select_rope_kernel(0)
    assert_close(got_wg, got_mma, what="tcgen05 vs mma.sync, full size")


# ------------------------------------------------------------------ variable rate, one lane per head pair


@pytest.mark.parametrize("B,n", [(1, 1), (1, 17), (1, 31), (1, 32), (1, 33), (2, 2049),
                                 (3, 5000)])
def test_varrate_paths(B, n, varrate_kernel):
    """Variable-rate records run on the tensor-core kernel or on the
    lane-per-(KV head, query head) kernel; per-row lengths force the generic
    kernel.  All must match the oracle."""
    c = synth.config("c4", B=B, T=n)
    a = synth.varrate_cache(c)
    ref = oracle(c, a, n)
    assert_close(run_decode(c, a, n), ref, what=f"varrate warp B={B} n={n}")
    assert_close(run_decode(c, a, n, seq_lens=[n] * B), ref, what=f"generic B={B} n={n}")


@pytest.mark.parametrize("rank", [4, 8, 16, 32, 64])
def test_varrate_single_rank(rank, varrate_kernel):
    """Every token at one rank: the ragged layout degenerates to a uniform one
    (rank 64: two scale groups per record; rank 4: 6-byte head records)."""
    c = synth.config("c4", B=1, T=700)
    r = np.full((1, 700), rank)
    a = synth.varrate_cache(c, ranks={"k": r, "v": r})
    assert_close(run_decode(c, a, 700), oracle(c, a, 700), what=f"varrate rank {rank}")


def test_varrate_k_and_v_ranks_differ(varrate_kernel):
    """K ranks high where V ranks are low and the reverse, so that the score
    and value sides mask different entries of the same tokens."""
    c = synth.config("c4", B=1, T=999)
    rk = np.where(np.arange(999) % 2 == 0, 64, 4)[None, :]
    rv = np.where(np.arange(999) % 2 == 0, 4, 64)[None, :]
    a = synth.varrate_cache(c, ranks={"k": rk, "v": rv})
    assert_close(run_decode(c, a, 999), oracle(c, a, 999), what="varrate k/v ranks differ")


def test_varrate_bf16_output(varrate_kernel):
    """bf16 output of the variable-rate layout within the stated tolerance."""
    c = synth.config("c4", B=2, T=3000)
    a = synth.varrate_cache(c)
    assert_close(run_decode(c, a, 3000, out_bf16=1), oracle(c, a, 3000), what="varrate bf16 out")


def test_varrate_repeated_calls_reuse_the_workspace():
    """Calls on a workspace full of stale bytes, and repeated calls on one
    workspace, must all give the oracle's output (nothing in the workspace may
    carry state from one call to the next)."""
    import torch

    from rank_bit_kv_b200 import kvc

    kvc.lib().kvc_select_varrate_kernel(0)
    c = synth.config("c4", B=3, T=5000)
    a = synth.varrate_cache(c)
    ref = oracle(c, a, 5000)
    lay = kvc.Layout(kvc.desc_from_config(c))
    cache = kvc.Cache(lay, fill=a)
    cache.n_tokens = 5000
    qt = torch.from_numpy(np.ascontiguousarray(a["q"]).view(np.int16)).cuda().view(torch.bfloat16)
    ws = torch.full((lay.workspace_bytes(5000),), 0xA5, dtype=torch.uint8, device="cuda")
    for i in range(4):
        out = torch.empty(qt.shape, device="cuda")
        kvc.decode(lay, cache, qt, out, ws)
        torch.cuda.synchronize()
        assert_close(out.cpu().numpy(), ref, what=f"varrate call {i} on a reused workspace")


# ------------------------------------------------------------------ block-shared latent on warp-level MMAs


@pytest.mark.parametrize("B,n", [(1, 1), (2, 63), (2, 64), (1, 65), (2, 300), (1, 2049),
                                 (3, 8191)])
def test_block_tc_path(B, n):
    """The block-shared latent for 4 layers runs on the tcgen05 kernel (128
    absorbed queries per CTA, 64-token tiles, one CTA per half of the latent
    columns); per-row lengths force the generic kernel.  Both must match the
    oracle."""
    c = synth.config("c3", B=B, T=n)
    a = synth.block_shared_cache(c)
    ref = oracle(c, a, n)
    assert_close(run_decode(c, a, n), ref, what=f"block tc B={B} n={n}")
    assert_close(run_decode(c, a, n, seq_lens=[n] * B), ref, what=f"generic B={B} n={n}")
