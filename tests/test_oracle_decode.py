"""Pins for the decode oracle (oracle/decode.py), CPU only.

Each pin checks the oracle against something other than itself:
- the already pinned forward oracle (the decode rows are the last rows of a
  causal forward pass over the whole sequence);
- brute force in pure Python loops;
- closed forms (one key; constant V);
- invariances: paged equals contiguous, and split-and-merge equals unsplit;
- mutations that must fail: a causal rule without the row offset, and a
  merge without the max shift.
"""
import math

import numpy as np
import pytest
import torch

from exact_io_aware_tmem_b200.workloads import decode_case
from oracle import attention as att
from oracle import decode as dec


def _dense_kv(c, b):
    n = int(c.cache_seqlens[b])
    rows = dec.cache_rows(b, n, stride=None if c.paged else c.page_size,
                          page_size=c.page_size if c.paged else None,
                          block_table=None if not c.paged else c.block_table.numpy())
    return c.k_cache[rows], c.v_cache[rows]


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("q_len,causal", [(1, True), (3, True), (3, False), (5, True)])
def test_decode_rows_are_the_last_rows_of_the_forward(paged, q_len, causal):
    # Sequence b's decode rows equal the last q_len rows of the plain forward
    # over the whole sequence, with its own last q_len tokens as queries.
    lengths = [7, 12, 5]
    H, H_kv, D = 4, 2, 8
    c = decode_case(3, dtype="f32", lengths=lengths, q_len=q_len, H=H, H_kv=H_kv, D=D,
                    page_size=4 if paged else None)
    o, lse = dec.decode_forward(c.q, c.k_cache, c.v_cache, c.cache_seqlens, q_len=q_len,
                                scale=0.3, causal=causal, stride=c.page_size,
                                page_size=c.page_size, block_table=c.block_table)
    for b, n in enumerate(lengths):
        k, v = _dense_kv(c, b)
        qf = torch.randn(n, H, D, dtype=torch.float64)
        qf[n - q_len:] = c.q[b * q_len:(b + 1) * q_len].double()
        cu = np.array([0, n])
        of, lsef = att.attention_forward(qf.numpy(), k.double().numpy(), v.double().numpy(), cu,
                                         causal, 0.3)
        np.testing.assert_allclose(o[b * q_len:(b + 1) * q_len], of[n - q_len:], atol=1e-12)
        np.testing.assert_allclose(lse[b * q_len:(b + 1) * q_len], lsef[:, n - q_len:].T,
                                   atol=1e-12)


def test_brute_force_small_case():
    lengths = [4, 6]
    q_len, H, H_kv, D, scale = 2, 2, 1, 3, 0.7
    c = decode_case(5, dtype="f32", lengths=lengths, q_len=q_len, H=H, H_kv=H_kv, D=D)
    o, lse = dec.decode_forward(c.q, c.k_cache, c.v_cache, c.cache_seqlens, q_len=q_len,
                                scale=scale, causal=True, stride=c.page_size)
    for b, n in enumerate(lengths):
        for i in range(q_len):
            pos = n - q_len + i
            for h in range(H):
                qv = [float(x) for x in c.q[b * q_len + i, h]]
                logits = []
                for j in range(pos + 1):
                    kv = [float(x) for x in c.k_cache[b * c.page_size + j, 0]]
                    logits.append(scale * sum(a * bb for a, bb in zip(qv, kv)))
                mx = max(logits)
                w = [math.exp(x - mx) for x in logits]
                tot = sum(w)
                for d in range(D):
                    ref = sum(w[j] * float(c.v_cache[b * c.page_size + j, 0, d])
                              for j in range(pos + 1)) / tot
                    assert abs(o[b * q_len + i, h, d] - ref) < 1e-12
                assert abs(lse[b * q_len + i, h] - (mx + math.log(tot))) < 1e-12


def test_single_key_and_constant_v_closed_forms():
    c = decode_case(6, dtype="f32", lengths=[1, 9], q_len=1, H=2, H_kv=2, D=4)
    v = c.v_cache.clone()
    v[9:18] = torch.tensor([1.0, -2.0, 0.5, 3.0])   # sequence 1: constant V
    o, lse = dec.decode_forward(c.q, c.k_cache, v, c.cache_seqlens, q_len=1, scale=0.5,
                                causal=True, stride=c.page_size)
    # one key: O = V_0, LSE = scale q . k_0
    np.testing.assert_allclose(o[0], c.v_cache[0].double().numpy(), atol=1e-12)
    np.testing.assert_allclose(lse[0], 0.5 * (c.q[0].double() * c.k_cache[0].double()).sum(-1),
                               atol=1e-12)
    # constant V: O = V whatever the weights
    np.testing.assert_allclose(o[1], np.tile([1.0, -2.0, 0.5, 3.0], (2, 1)), atol=1e-12)


def test_paged_equals_contiguous_for_any_block_order():
    lengths = [9, 1, 16, 0]
    args = dict(dtype="f32", lengths=lengths, q_len=1, H=2, H_kv=1, D=4)
    cont = decode_case(8, **args)
    paged = decode_case(8, page_size=3, **args)
    # Same draws except the layout: put the contiguous cache's values into the pages.
    for b, n in enumerate(lengths):
        rows = dec.cache_rows(b, n, page_size=3, block_table=paged.block_table.numpy())
        paged.k_cache[rows] = cont.k_cache[b * cont.page_size:b * cont.page_size + n]
        paged.v_cache[rows] = cont.v_cache[b * cont.page_size:b * cont.page_size + n]
    oc, lc = dec.decode_forward(cont.q, cont.k_cache, cont.v_cache, cont.cache_seqlens,
                                q_len=1, scale=0.5, causal=True, stride=cont.page_size)
    op, lp = dec.decode_forward(cont.q, paged.k_cache, paged.v_cache, paged.cache_seqlens,
                                q_len=1, scale=0.5, causal=True, page_size=3,
                                block_table=paged.block_table)
    np.testing.assert_allclose(op, oc, atol=1e-12)
    np.testing.assert_allclose(lp, lc, atol=1e-12)
    # the empty sequence has no key: O = 0, LSE = -inf
    assert np.all(oc[3] == 0) and np.all(np.isneginf(lc[3]))


@pytest.mark.parametrize("cuts", [[0, 10], [0, 3, 10], [0, 1, 2, 9, 10], [0, 0, 5, 5, 10]])
def test_split_and_merge_equals_unsplit(cuts):
    rng = np.random.default_rng(0)
    q = rng.standard_normal((3, 8)) * 2
    k = rng.standard_normal((10, 8))
    v = rng.standard_normal((10, 8))
    pos = np.array([7, 8, 9])
    full_o, full_lse = dec.partial_forward(q, k, v, 0.4, 0, 10, pos, causal=True)
    parts = [dec.partial_forward(q, k, v, 0.4, a, b, pos, causal=True)
             for a, b in zip(cuts[:-1], cuts[1:])]
    o, lse = dec.merge_partials([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(o, full_o, atol=1e-12)
    np.testing.assert_allclose(lse, full_lse, atol=1e-12)
    # the unsplit partial is the plain softmax definition
    s = 0.4 * q @ k.T
    s[np.arange(10)[None, :] > pos[:, None]] = -np.inf
    p = np.exp(s - s.max(1, keepdims=True))
    np.testing.assert_allclose(full_o, (p / p.sum(1, keepdims=True)) @ v, atol=1e-12)


def test_merge_of_all_empty_splits_is_empty():
    o, lse = dec.merge_partials(np.zeros((2, 3, 4)), np.full((2, 3), -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_mutation_causal_rule_without_row_offset_is_caught():
    # A decode oracle that placed the q_len queries at positions 0..q_len-1
    # (no offset) must fail the forward cross-check above.
    lengths, q_len = [9], 3
    c = decode_case(9, dtype="f32", lengths=lengths, q_len=q_len, H=2, H_kv=2, D=4)
    k, v = _dense_kv(c, 0)
    qf = torch.randn(9, 2, 4, dtype=torch.float64)
    qf[6:] = c.q.double()
    of, _ = att.attention_forward(qf.numpy(), k.double().numpy(), v.double().numpy(),
                                  np.array([0, 9]), True, 0.5)
    bad = np.zeros((3, 2, 4))
    for h in range(2):
        s = att.scores(c.q[:, h].double().numpy(), k[:, h].double().numpy(), 0.5, True,
                       np.arange(q_len))
        p, _ = att.softmax_rows(s)
        bad[:, h] = p @ v[:, h].double().numpy()
    assert np.abs(bad - of[6:]).max() > 1e-3


def test_mutation_merge_without_max_shift_overflows():
    # Merging with raw exp(LSE_s) (no shift) overflows for large logits; the
    # oracle's shifted merge does not.
    lse_parts = np.array([[800.0], [799.0]])
    o_parts = np.array([[[1.0]], [[3.0]]])
    o, lse = dec.merge_partials(o_parts, lse_parts)
    w = np.exp([0.0, -1.0])
    assert abs(o[0, 0] - (w[0] * 1 + w[1] * 3) / w.sum()) < 1e-12
    with np.errstate(over="ignore", invalid="ignore"):
        raw = np.exp(lse_parts)
        naive = (raw[:, :, None] * o_parts).sum(0) / raw.sum(0)[:, None]
    assert not np.isfinite(naive).all()
