"""Plain fp64 reference of the joint rank / residual-bit allocation.

TEST INFRASTRUCTURE ONLY.  Only the test-suite imports this module; the library
never calls it and it imports nothing from the library.

What it computes (pages: "JoLT: Near-Lossless KV Cache Compression", section
"How JoLT works": the layers are grouped, the keys and the values of each group
are separate cells, and one Lagrangian multiplier picks every cell's ranks and
residual bit-width under a shared byte budget before anything is compressed;
"A JoLT for the KV cache ...", "Abstract (arXiv)": a single Lagrangian dual
allocates per-group ranks and residual bit-widths under a global byte
constraint).

Readings where the pages give no formula (stated, not taken from them):
  * a cell's options are pairs (rank r, residual bits b) from caller-given
    grids; each has a byte cost and a distortion;
  * bytes(r, b) = rows * (latent codes + group scales/zeros + residual codes and
    scale when b > 0) + factor bytes (heads * r * d fp16) + signs (d per head
    when b > 0): the stored format of the low-rank layouts;
  * distortion(r, b) = eta_latent * (energy kept in the first r components)
    + eta_resid[b] * (energy of the truncated tail), from the cell's spectrum
    (squared singular values, descending); eta_resid[0] = 1 (no residual: the
    whole tail is lost), so with eta_latent = 0 and b = 0 it is the
    Eckart-Young truncation error;
  * for a multiplier lam every cell takes the option minimising
    distortion + lam * bytes (ties: fewer bytes, then the earlier option);
    the allocation is the one at the smallest lam whose total bytes fit the
    budget.  Total bytes only change at the pairwise break points
    lam = (D_a - D_b) / (B_b - B_a) of a cell's options, so the search runs
    over those points (exactly, no iteration tolerance).
"""

from __future__ import annotations

import math

import numpy as np


def option_grid(ranks, bits):
    """Options as (rank, bits) pairs, rank-major."""
    return [(int(r), int(b)) for r in ranks for b in bits]


def row_bytes(r, b, head_dim, latent_bits=4, group=32):
    """Stored bytes of one token row of one component at rank r, residual bits b."""
    lat = math.ceil(r * latent_bits / 8) + (4 * math.ceil(r / group) if latent_bits < 16 else 0)
    res = (head_dim * b // 8 + 2) if b > 0 else 0
    return lat + res


def option_tables(spectra, rows, heads, options, head_dim, eta_latent, eta_resid,
                  latent_bits=4, group=32):
    """Byte and distortion tables [cells, options] from per-cell spectra.

    spectra: [C, n] squared singular values of each cell's (rows x d) matrix,
    descending; rows, heads: [C]; eta_resid: dict bits -> factor."""
    spectra = np.asarray(spectra, np.float64)
    C = spectra.shape[0]
    B = np.zeros((C, len(options)))
    D = np.zeros((C, len(options)))
    for c in range(C):
        total = spectra[c].sum()
        for j, (r, b) in enumerate(options):
            head = spectra[c, :r].sum()
            tail = total - head
            B[c, j] = (rows[c] * row_bytes(r, b, head_dim, latent_bits, group)
                       + heads[c] * r * head_dim * 2 + (heads[c] * head_dim if b > 0 else 0))
            D[c, j] = eta_latent * head + eta_resid[b] * tail
    return B, D


def choice_at(B, D, lam):
    """Per cell, the option minimising D + lam * B (ties: fewer bytes, then the
    earlier option)."""
    C, O = B.shape
    out = np.zeros(C, np.int64)
    for c in range(C):
        best = 0
        for j in range(1, O):
            vj = D[c, j] + lam * B[c, j]
            vb = D[c, best] + lam * B[c, best]
            if vj < vb or (vj == vb and B[c, j] < B[c, best]):
                best = j
        out[c] = best
    return out


def break_points(B, D):
    """lam = 0 and every pairwise point where a cell's preference can change."""
    pts = {0.0}
    C, O = B.shape
    for c in range(C):
        for a in range(O):
            for b in range(O):
                if B[c, a] < B[c, b] and D[c, a] > D[c, b]:
                    pts.add((D[c, a] - D[c, b]) / (B[c, b] - B[c, a]))
    return sorted(pts)


def allocate(B, D, budget):
    """(choice [C], lam) at the smallest break point whose bytes fit the budget,
    or None when even the cheapest options exceed it."""
    B = np.asarray(B, np.float64)
    D = np.asarray(D, np.float64)
    pts = break_points(B, D)

    def total(lam):
        ch = choice_at(B, D, lam)
        return B[np.arange(len(ch)), ch].sum(), ch

    lo, hi = 0, len(pts) - 1
    if total(pts[hi])[0] > budget:
        return None
    while lo < hi:                        # bytes are non-increasing in lam
        mid = (lo + hi) // 2
        if total(pts[mid])[0] <= budget:
            hi = mid
        else:
            lo = mid + 1
    return total(pts[lo])[1], pts[lo]
