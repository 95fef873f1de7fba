"""Plain fp64 reference of the token-importance producers.

TEST INFRASTRUCTURE ONLY.  Only the test-suite imports this module; the library
never calls it and it imports nothing from the library.

What it computes.
* VarRate ("VarRate: Training-Free Variable-Rate KV Cache Compression for
  Long-Context LLMs", sections "Summary", "Principles", "Method"): every token
  gets a low-rank budget chosen by its query salience, and no token is ever
  dropped (its rank is never zero).
* BellowsKV-Evict ("BellowsKV Architecture ...", section "Three Measurements,
  Three Operators"): the layers of a block agree on which tokens matter, so one
  importance decision per block, computed from all n layers' scores, is applied
  once to the shared latent.

Readings (the pages name the quantities, not their formulas):
  * the salience of token t is the attention probability it receives from an
    observation window of queries (the last W prefill queries), summed over
    the window and over the query heads that share the token's rank (all query
    heads of a batch row, since one rank serves every KV head of a token):
    sal_t = sum_{h, w} softmax_t(scale * q_{h,w} . k_{kv(h), t});
  * ranks by salience quantiles: tokens in descending salience (ties: lower
    position first) take the ranks of a caller-given ladder with caller-given
    counts -- the C4 workload's {64, 32, 16, 8, 4} at {5, 10, 20, 25, 40} % of the
    tokens averages 13.2 of 64, about the 20 % budget the page quotes -- the last
    rung taking every remaining token, so every token keeps a nonzero rank;
  * the block's importance is the same attention mass summed over the n layers
    (each layer's keys read from the shared latent through its own W_k^l), and
    the decision keeps the `keep` most important tokens (ties: lower position
    first) in their original order.
"""

from __future__ import annotations

import numpy as np


def window_salience(q, k, scale):
    """sal [B, T] from window queries q [B, Hq, W, d] and keys k [B, Hkv, T, d]
    (both as the attention sees them), query head h reading KV head h // G."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    B, Hq, W, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    sal = np.zeros((B, k.shape[2]))
    for b in range(B):
        for h in range(Hq):
            s = scale * (q[b, h] @ k[b, h // G].T)          # [W, T]
            s -= s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            sal[b] += p.sum(axis=0)
    return sal


def descending_order(sal):
    """Positions sorted by salience, largest first, ties by lower position."""
    sal = np.asarray(sal)
    return np.lexsort((np.arange(sal.shape[-1]), -sal))


def ranks_by_salience(sal, ladder, counts):
    """Rank per token [B, T]: the first counts[0] tokens of the descending order
    get ladder[0], the next counts[1] ladder[1], ...; the last rung takes every
    remaining token."""
    sal = np.asarray(sal, np.float64)
    B, T = sal.shape
    out = np.zeros((B, T), np.int64)
    for b in range(B):
        order = descending_order(sal[b])
        start = 0
        for i, r in enumerate(ladder):
            n = T - start if i == len(ladder) - 1 else min(counts[i], T - start)
            out[b, order[start:start + n]] = r
            start += n
    return out


def rung_counts(T, fractions):
    """Tokens per rung for a token count T: floor of the cumulative fractions,
    the last rung taking the rest."""
    cum = np.floor(np.cumsum(fractions[:-1]) * T + 1e-9).astype(np.int64)
    counts = np.diff(np.concatenate([[0], cum]))
    return list(counts) + [T - int(cum[-1]) if len(cum) else T]


def block_importance(q_layers, keys_layers, scale):
    """Importance [B, T] of a block: the window salience summed over its layers
    (q_layers [L, B, Hq, W, d], keys_layers [L, B, Hkv, T, d])."""
    return sum(window_salience(q_layers[l], keys_layers[l], scale) for l in range(len(q_layers)))


def keep_decision(importance, keep):
    """Kept positions [B, keep], ascending (the original order), of the `keep`
    most important tokens of every row."""
    imp = np.asarray(importance, np.float64)
    return np.stack([np.sort(descending_order(imp[b])[:keep]) for b in range(imp.shape[0])])
