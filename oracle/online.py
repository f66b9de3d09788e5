"""Float64 online-softmax attention, step by step, for checking the oracle.

TEST INFRASTRUCTURE (same rule as ``oracle.attention``: only the tests,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline use it).

This follows the recurrence the pages give, in their order and notation:

* aiqz.cc "Flash Attention V2/V3 optimization", section "V2 algorithm
  optimisation", steps 1-5: m_new = max(m_old, m_block); the old output is
  multiplied by e^(m_old - m_new); the exponential sum l is rescaled the same
  way and the new block's exponentials are added; the new block contributes
  e^(S_block - m_new) V_block; after the last block the accumulator is
  divided once by l;
* airsota.com card (p=1562), section 3, the online update of m and l, where
  the new block adds the *sum* of its exponentials. The article's printed
  l-update shows a single term e^(m_block - m_new); that is only right for a
  one-element block, so the sum is used (the same article's Python demo sums
  the block's P over its columns too);
* the same demo initialises m = -inf, l = 0, acc = 0 per query row and
  applies the scale to S before the max.

Its purpose is to show that blockwise equals full softmax for any split of
the keys into contiguous blocks (the pages call the two strictly equivalent
up to floating-point rounding).
"""
from __future__ import annotations

import numpy as np


def online_attention(q, k, v, scale: float, blocks, causal: bool = False):
    """O and LSE of one head, visiting the keys in the given contiguous blocks.

    ``blocks`` is a list of (start, end) key ranges that tile [0, n_k).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n_q = q.shape[0]
    m = np.full(n_q, -np.inf)
    l = np.zeros(n_q)
    acc = np.zeros((n_q, v.shape[1]))
    rows = np.arange(n_q)
    for start, end in blocks:
        s_blk = scale * (q @ k[start:end].T)
        if causal:
            cols = np.arange(start, end)
            s_blk = np.where(cols[None, :] > rows[:, None], -np.inf, s_blk)
        m_blk = s_blk.max(axis=1) if end > start else np.full(n_q, -np.inf)
        m_new = np.maximum(m, m_blk)
        # A row that has seen no visible key yet keeps m = -inf; its factors
        # are defined as 0 so that (-inf) - (-inf) never appears.
        seen = np.isfinite(m_new)
        m_ref = np.where(seen, m_new, 0.0)
        alpha = np.where(seen, np.exp(np.where(seen, m, 0.0) - m_ref), 0.0)
        alpha = np.where(np.isfinite(m), alpha, 0.0)
        p_blk = np.where(seen[:, None], np.exp(s_blk - m_ref[:, None]), 0.0)
        acc = acc * alpha[:, None] + p_blk @ v[start:end]
        l = l * alpha + p_blk.sum(axis=1)
        m = m_new
    has = l > 0
    o = np.where(has[:, None], acc / np.where(has, l, 1.0)[:, None], 0.0)
    lse = np.where(has, m + np.log(np.where(has, l, 1.0)), -np.inf)
    return o, lse


def uniform_blocks(n: int, size: int):
    return [(s, min(s + size, n)) for s in range(0, n, size)]


def compositions(n: int):
    """Every split of [0, n) into contiguous non-empty blocks (2^(n-1) of them)."""
    if n == 0:
        yield []
        return
    for mask in range(1 << (n - 1)):
        cuts = [0] + [i + 1 for i in range(n - 1) if mask >> i & 1] + [n]
        yield [(cuts[i], cuts[i + 1]) for i in range(len(cuts) - 1)]
