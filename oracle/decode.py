"""Plain float64 CPU decode attention: the oracle for the split-KV decode path.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import or call this module.
The product path never routes through it and shares no code with it.

What it computes. At inference there is no backward pass, and the key/value
cache of every sequence is long while only its newest q_len tokens are
queried. The agentalpha.top "flash attention" answer says how the method
serves this case:
- section 2 (recomputation) notes that inference versions such as
  FlashDecoding keep the tiling and drop the recomputation;
- its follow-up 2 has the kernel split the sequence (the cache) into blocks,
  compute each block's attention independently, and merge the blocks with
  the online-softmax update. The cache may be paged (vLLM's page attention),
  in which case each block is read from wherever its page lives.

The result is the plain attention of those q_len queries over the cache
prefix. This module writes that definition out and does no splitting: each
query row sees all of its keys at once. The split merge is written
separately (``merge_partials``) so that the tests can pin it against the
unsplit result.

Readings where the pages are silent (each listed in the design notes):

* query i (0-based) of the q_len newest tokens of sequence b sits at position
  len_b - q_len + i of that sequence. Causal masking keeps key j iff j is at
  most that position (the forward's causal rule, with the rows offset);
  non-causal decoding sees all len_b keys;
* grouped-query attention maps query head h to key/value head h // (H / H_kv);
* contiguous cache: position j of sequence b is row b * stride + j of the
  cache arrays ``[rows, H_kv, D]``; paged cache: it is row
  block_table[b][j // page] * page + j % page;
* LSE = m + ln(l) in natural-log units of the scaled logits, laid out
  ``[B * q_len, H]`` like the output rows;
* merging split partials: a split s contributes its own normalised output O_s
  and LSE_s; LSE = ln sum_s exp(LSE_s) and O = sum_s exp(LSE_s - LSE) O_s. A
  split that sees no key has LSE_s = -inf and weight 0.
"""
from __future__ import annotations

import numpy as np

from .attention import _f64, scores, softmax_rows


def cache_rows(b: int, length: int, *, stride: int | None = None, page_size: int | None = None,
               block_table=None) -> np.ndarray:
    """Physical cache rows holding positions 0..length-1 of sequence ``b``."""
    j = np.arange(length, dtype=np.int64)
    if block_table is None:
        return b * int(stride) + j
    table = np.asarray(block_table, dtype=np.int64)
    return table[b, j // page_size] * page_size + j % page_size


def decode_forward(q, k_cache, v_cache, cache_seqlens, *, q_len: int, scale: float,
                   causal: bool, stride: int | None = None, page_size: int | None = None,
                   block_table=None):
    """O ``[B*q_len, H, D]`` and LSE ``[B*q_len, H]`` of the newest q_len tokens.

    ``q`` is ``[B*q_len, H, D]`` (token-major, the q_len tokens of sequence b
    at rows b*q_len ..); the caches are ``[rows, H_kv, D]``.
    """
    q = _f64(q)
    lens = [int(x) for x in np.asarray(cache_seqlens).reshape(-1)]
    B = len(lens)
    H, D = q.shape[1], q.shape[2]
    H_kv = k_cache.shape[1]
    g = H // H_kv
    o = np.zeros((B * q_len, H, D))
    lse = np.zeros((B * q_len, H))
    for b, n in enumerate(lens):
        rows = cache_rows(b, n, stride=stride, page_size=page_size, block_table=block_table)
        kb = _f64(k_cache[rows]) if n else np.zeros((0, H_kv, D))
        vb = _f64(v_cache[rows]) if n else np.zeros((0, H_kv, D))
        pos = n - q_len + np.arange(q_len)        # positions of the query rows
        for h in range(H):
            s = scores(q[b * q_len:(b + 1) * q_len, h], kb[:, h // g], scale, causal, pos)
            p, l = softmax_rows(s)
            o[b * q_len:(b + 1) * q_len, h] = p @ vb[:, h // g]
            lse[b * q_len:(b + 1) * q_len, h] = l
    return o, lse


def partial_forward(q, k, v, scale: float, key_lo: int, key_hi: int, pos=None,
                    causal: bool = False):
    """One split's normalised output and LSE: keys [key_lo, key_hi) only.

    ``q`` is [n, D], ``k``/``v`` are [len, D] of one (sequence, head); ``pos``
    are the query positions for the causal rule.
    """
    q = _f64(q)
    k = _f64(k)[key_lo:key_hi]
    v = _f64(v)[key_lo:key_hi]
    s = scores(q, k, scale, False)
    if causal:
        cols = key_lo + np.arange(k.shape[0])
        s = np.where(cols[None, :] > np.asarray(pos)[:, None], -np.inf, s)
    p, lse = softmax_rows(s)
    return p @ v, lse


def merge_partials(o_parts, lse_parts):
    """Merge split partials: ``o_parts`` [S, n, D], ``lse_parts`` [S, n]."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    has = np.isfinite(m)
    m_safe = np.where(has, m, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - m_safe[None, :]), 0.0)
    tot = w.sum(axis=0)
    lse = np.where(has, m_safe + np.log(np.where(has, tot, 1.0)), -np.inf)
    o = np.where(has[:, None], (w[:, :, None] * o_parts).sum(axis=0) /
                 np.where(has, tot, 1.0)[:, None], 0.0)
    return o, lse
