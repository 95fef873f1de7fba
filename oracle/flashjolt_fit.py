"""Plain fp64 reference of the per-head factor fit by randomized SVD.

TEST INFRASTRUCTURE ONLY.  Only the test-suite imports this module; the library
never calls it and it imports nothing from the library.

What it computes.  "A JoLT for the KV cache ...", "Abstract (arXiv)":
FlashJoLT replaces the exact token-mode SVD of the compressor with a randomized
approximation; "JoLT: Near-Lossless KV Cache Compression", "How JoLT works" and
"Key findings": the decomposition truncates only the token and feature axes,
keeps heads separate (per-head factors), and works on keys before RoPE.  The
stored representation is a per-token latent times a per-head factor B
(r x d): k_t ~ l_t B with l_t = k_t B^T ("BELT Connects KV-Cache Compression to
Faster Long-Context Decoding", section 3).

Readings (the pages name the method, not its steps): the randomized SVD of the
token-major matrix X (N tokens x d) of one KV head by the randomized range
finder with a Gaussian test matrix Omega (d x k, k = r + oversampling, passed
in as an input), q power iterations with re-orthonormalisation, and the exact
SVD of the small projection (the standard randomized SVD of Halko, Martinsson
and Tropp, 2011); the factor rows are the top r right singular vectors; every
row is multiplied by +-1 so that its entry of largest magnitude is positive
(singular vectors are defined up to sign).
"""

from __future__ import annotations

import numpy as np


def sign_normalise(F):
    """Rows times +-1 so that each row's entry of largest magnitude is positive."""
    F = np.asarray(F, np.float64)
    idx = np.abs(F).argmax(axis=1)
    sg = np.sign(F[np.arange(F.shape[0]), idx])
    sg[sg == 0] = 1.0
    return F * sg[:, None]


def randomized_factor(X, omega, rank, power_iters):
    """(factor [rank, d], sigma^2 estimates [rank]) of X [N, d] (fp64).

      Y = X Omega;  Q = orth(Y)
      repeat power_iters times:  Z = orth(X^T Q);  Q = orth(X Z)
      B_s = Q^T X  (k x d);  B_s = U S V^T;  factor = first rank rows of V^T
    """
    X = np.asarray(X, np.float64)
    Q, _ = np.linalg.qr(X @ np.asarray(omega, np.float64))
    for _ in range(power_iters):
        Z, _ = np.linalg.qr(X.T @ Q)
        Q, _ = np.linalg.qr(X @ Z)
    _, s, Vt = np.linalg.svd(Q.T @ X, full_matrices=False)
    return sign_normalise(Vt[:rank]), s[:rank] ** 2


def fit_heads(x, omega, rank, power_iters):
    """Factors of every KV head from prefill keys or values x [B, Hkv, T, d]
    (all batch rows' tokens of a head form its token-major matrix) and a test
    matrix per head omega [Hkv, d, k]."""
    x = np.asarray(x, np.float64)
    B, Hkv, T, d = x.shape
    F = np.zeros((Hkv, rank, d))
    S = np.zeros((Hkv, rank))
    for h in range(Hkv):
        F[h], S[h] = randomized_factor(x[:, h].reshape(B * T, d), omega[h], rank, power_iters)
    return F, S
