"""Joint rank / residual-bit allocation under one byte budget ("JoLT:
Near-Lossless KV Cache Compression", "How JoLT works"; "A JoLT for the KV
cache ...", "Abstract (arXiv)").

The oracle (oracle/jolt_alloc.py) is pinned to what the mathematics fixes:
exhaustive search over every allocation of tiny instances (Everett: the
Lagrangian allocation is optimal among all allocations that use no more
bytes), the minimality of the multiplier, Eckart-Young for the no-residual
distortion of an explicit matrix, and the byte closed forms of the stored
format.  The library's native allocator (host code, no GPU) is then compared
with the oracle on the same tables: identical choices and multipliers.
"""

import itertools

import numpy as np
import pytest

from oracle import jolt_alloc as A
from oracle import kvc_oracle as O

ETA = {0: 1.0, 2: 0.12, 4: 0.01}


def random_tables(rng, C, O_):
    B = rng.uniform(1, 100, (C, O_)).round(3)
    D = rng.uniform(0, 50, (C, O_)).round(3)
    return B, D


def spectra_of(rng, C, n, decay):
    s = np.exp(-decay * np.arange(n))[None] * rng.uniform(0.5, 2.0, (C, 1))
    return s * (1 + 0.05 * rng.random((C, n)))


# ----------------------------------------------------------------- oracle pins


@pytest.mark.parametrize("seed", range(6))
def test_lagrangian_allocation_is_optimal_among_allocations_with_no_more_bytes(seed):
    """Everett's theorem, checked by brute force over every allocation."""
    rng = np.random.default_rng(seed)
    B, D = random_tables(rng, 4, 5)
    budget = B.min(1).sum() + rng.uniform(0.2, 0.8) * (B.max(1).sum() - B.min(1).sum())
    ch, lam = A.allocate(B, D, budget)
    used = B[np.arange(4), ch].sum()
    dist = D[np.arange(4), ch].sum()
    assert used <= budget
    best = min(D[np.arange(4), list(c)].sum() for c in itertools.product(range(5), repeat=4)
               if B[np.arange(4), list(c)].sum() <= used + 1e-9)
    assert dist <= best + 1e-9


@pytest.mark.parametrize("seed", range(4))
def test_multiplier_is_the_smallest_feasible_break_point(seed):
    rng = np.random.default_rng(100 + seed)
    B, D = random_tables(rng, 5, 6)
    budget = B.min(1).sum() + 0.4 * (B.max(1).sum() - B.min(1).sum())
    ch, lam = A.allocate(B, D, budget)
    pts = A.break_points(B, D)
    i = pts.index(lam)
    if i > 0:                             # one break point lower no longer fits
        ch2 = A.choice_at(B, D, pts[i - 1])
        assert B[np.arange(5), ch2].sum() > budget
    # the minimiser of D + lam B really is the chosen option in every cell
    for c in range(5):
        v = D[c] + lam * B[c]
        assert v[ch[c]] == v.min()


def test_infeasible_budget():
    B = np.array([[10.0, 20.0], [5.0, 6.0]])
    D = np.array([[1.0, 0.0], [1.0, 0.0]])
    assert A.allocate(B, D, 14.0) is None
    ch, lam = A.allocate(B, D, 15.0)
    assert list(ch) == [0, 0]
    ch, lam = A.allocate(B, D, 1e9)
    assert list(ch) == [1, 1] and lam == 0.0


def test_no_residual_distortion_is_the_eckart_young_truncation_error():
    """With eta_latent = 0 and no residual the distortion of rank r is the
    squared Frobenius error of the best rank-r approximation, computed here by
    explicit truncation of an SVD."""
    rng = np.random.default_rng(3)
    X = rng.standard_normal((300, 16)) @ np.diag(np.exp(-0.3 * np.arange(16))) @ \
        np.linalg.qr(rng.standard_normal((16, 16)))[0]
    U, s, Vt = np.linalg.svd(X, full_matrices=False)
    opts = A.option_grid([2, 4, 8], [0])
    B, D = A.option_tables((s ** 2)[None], [300], [1], opts, 16, 0.0, {0: 1.0})
    for j, (r, b) in enumerate(opts):
        Xr = (U[:, :r] * s[:r]) @ Vt[:r]
        assert np.isclose(D[0, j], np.linalg.norm(X - Xr) ** 2, rtol=1e-10)


def test_byte_tables_match_the_stored_format():
    """Rows cost what the low-rank layouts store: the C2 row (rank 32, INT4 g32)
    is 20 bytes per component; a 2-bit residual of d = 128 adds 32 + 2."""
    opts = [(32, 0), (48, 0), (64, 2)]
    B, _ = A.option_tables(np.ones((1, 128)), [1000], [8], opts, 128, 0.0, ETA)
    assert B[0, 0] == 1000 * 20 + 8 * 32 * 128 * 2
    assert B[0, 1] == 1000 * (24 + 8) + 8 * 48 * 128 * 2
    assert B[0, 2] == 1000 * (32 + 8 + 34) + 8 * 64 * 128 * 2 + 8 * 128
    # the same per-row figures as the layout's closed form
    assert O.lowrank_bytes_per_token_head(32, 48, 4, 32) == 20 + 32


# ----------------------------------------------------------------- native allocator against the oracle


@pytest.fixture(scope="module")
def kvc():
    from rank_bit_kv_b200 import build, kvc as K

    build.build()
    return K


@pytest.mark.parametrize("seed", range(5))
def test_native_tables_and_allocation_match_the_oracle(kvc, seed):
    rng = np.random.default_rng(200 + seed)
    C = 8                                  # 4 layer groups x {K, V}
    spectra = spectra_of(rng, C, 128, rng.uniform(0.02, 0.08))
    rows = rng.integers(10_000, 200_000, C)
    heads = np.full(C, 8)
    opts = A.option_grid([8, 16, 32, 48, 64], [0, 2, 4])
    Bo, Do = A.option_tables(spectra, rows, heads, opts, 128, 0.006, ETA)
    Bn, Dn = kvc.rank_bit_tables(spectra, rows, heads, opts, 128, 0.006, ETA)
    np.testing.assert_array_equal(Bn, Bo)              # integer byte counts
    np.testing.assert_allclose(Dn, Do, rtol=1e-12)     # summation order only
    for frac in (0.1, 0.3, 0.6, 0.9):
        budget = Bo.min(1).sum() + frac * (Bo.max(1).sum() - Bo.min(1).sum())
        ch_o, lam_o = A.allocate(Bo, Do, budget)
        ch_n, lam_n = kvc.allocate_rank_bits(Bo, Do, budget)
        np.testing.assert_array_equal(ch_n, ch_o)
        assert lam_n == lam_o


def test_native_allocator_reports_an_infeasible_budget(kvc):
    B = np.array([[10.0, 20.0], [5.0, 6.0]])
    D = np.array([[1.0, 0.0], [1.0, 0.0]])
    with pytest.raises(kvc.KvcError) as ei:
        kvc.allocate_rank_bits(B, D, 14.0)
    assert kvc.STATUS[ei.value.status] == "KVC_ECAPACITY"
    with pytest.raises(kvc.KvcError):
        kvc.rank_bit_tables(np.ones((1, 8)), [10], [1], [(9, 0)], 128, 0.0, ETA)   # rank > spectrum
