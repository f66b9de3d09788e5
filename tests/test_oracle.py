"""Pins for the float64 oracle: things the pages and the mathematics fix.

Each test checks the oracle against something other than itself: closed
forms, invariants the pages state, brute force on tiny inputs, an
independent step-by-step online recurrence, special cases that reduce to the
dense routine, and central finite differences for the backward pass. The
mutation tests at the end plant plausible mistakes in a copy of the oracle's
source and check that at least one pin fails for each.
"""
import itertools
import json
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oa
from oracle.online import compositions, online_attention, uniform_blocks

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand(rng, *shape, std=1.0):
    return rng.standard_normal(shape) * std


# ---------------------------------------------------------------- softmax ---

def test_rows_sum_to_one_and_nonnegative(rng):
    for causal in (False, True):
        q, k = _rand(rng, 40, 8, std=3), _rand(rng, 40, 8, std=3)
        p, lse = oa.softmax_rows(oa.scores(q, k, 0.3, causal))
        assert np.all(p >= 0)
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12, rtol=0)


def test_shift_invariance(rng):
    # softmax(S + c 1^T) = softmax(S): the property the airsota card (section 4,
    # item 1) and the safe-softmax step rest on. LSE moves by exactly c.
    s = _rand(rng, 30, 50, std=5)
    c = rng.uniform(-1e3, 1e3, size=30)
    p0, l0 = oa.softmax_rows(s)
    p1, l1 = oa.softmax_rows(s + c[:, None])
    np.testing.assert_allclose(p1, p0, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l1 - c, l0, atol=1e-9, rtol=0)


def test_no_overflow_for_huge_logits(rng):
    s = _rand(rng, 4, 16) * 1e4  # exp would overflow without the max shift
    p, lse = oa.softmax_rows(s)
    assert np.all(np.isfinite(p)) and np.all(np.isfinite(lse))
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)


# -------------------------------------------------------- online == full ---

@pytest.mark.parametrize("causal", [False, True])
def test_online_equals_full_every_composition(rng, causal):
    for n in range(1, 9):
        q, k, v = _rand(rng, n, 5, std=2), _rand(rng, n, 5, std=2), _rand(rng, n, 3)
        o_ref, lse_ref = oa.head_forward(q, k, v, 0.7, causal)
        for blocks in compositions(n):
            o, lse = online_attention(q, k, v, 0.7, blocks, causal)
            np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
            np.testing.assert_allclose(lse, lse_ref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_online_equals_full_uniform_and_random_blocks(rng, causal):
    n = 37
    q, k, v = _rand(rng, n, 16, std=2), _rand(rng, n, 16, std=2), _rand(rng, n, 16)
    o_ref, lse_ref = oa.head_forward(q, k, v, 0.25, causal)
    splits = [uniform_blocks(n, b) for b in range(1, n + 1)]
    for _ in range(20):
        cuts = sorted(rng.choice(np.arange(1, n), size=rng.integers(1, 10), replace=False))
        edges = [0] + [int(c) for c in cuts] + [n]
        splits.append(list(zip(edges[:-1], edges[1:])))
    for blocks in splits:
        o, lse = online_attention(q, k, v, 0.25, blocks, causal)
        np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse, lse_ref, atol=1e-12, rtol=0)


def test_demo_blockwise_check():
    """The article's own demo check: seed 0, (2,4,256,32), block 64, < 1e-5."""
    with open(os.path.join(HERE, "golden", "demo_blockwise.json")) as f:
        fx = json.load(f)
    torch.manual_seed(0)
    shape = (fx["batch"], fx["heads"], fx["seq_len"], fx["d"])
    q, k, v = (torch.randn(shape).double().numpy() for _ in range(3))
    scale = fx["d"] ** -0.5
    worst = 0.0
    for b, h in itertools.product(range(shape[0]), range(shape[1])):
        o_full, _ = oa.head_forward(q[b, h], k[b, h], v[b, h], scale, False)
        o_blk, _ = online_attention(q[b, h], k[b, h], v[b, h], scale,
                                    uniform_blocks(shape[2], fx["block_size"]))
        worst = max(worst, float(np.abs(o_full - o_blk).max()))
    assert worst < fx["max_abs_err_bound"]
    assert worst < 1e-12  # float64: rounding only


# ----------------------------------------------------------- closed forms ---

@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_gives_constant_output(rng, causal):
    n, d = 33, 7
    q, k = _rand(rng, n, 8, std=3), _rand(rng, n, 8, std=3)
    vrow = _rand(rng, d)
    o, _ = oa.head_forward(q, k, np.tile(vrow, (n, 1)), 0.5, causal)
    np.testing.assert_allclose(o, np.tile(vrow, (n, 1)), atol=1e-12, rtol=0)


def test_causal_mask(rng):
    n = 20
    q, k, v = _rand(rng, n, 6, std=2), _rand(rng, n, 6, std=2), _rand(rng, n, 4)
    p, _ = oa.softmax_rows(oa.scores(q, k, 0.4, True))
    assert np.all(np.triu(p, 1) == 0.0)
    assert np.all(p[np.tril_indices(n)] > 0.0)
    o, lse = oa.head_forward(q, k, v, 0.4, True)
    np.testing.assert_array_equal(o[0], v[0])          # row 0 sees key 0 only
    assert lse[0] == pytest.approx(0.4 * float(q[0] @ k[0]), abs=1e-12)


def test_single_key_closed_form(rng):
    q, k, v = _rand(rng, 1, 9), _rand(rng, 1, 9), _rand(rng, 1, 5)
    for causal in (False, True):
        o, lse = oa.head_forward(q, k, v, 0.6, causal)
        np.testing.assert_allclose(o, v, atol=1e-15)
        assert lse[0] == pytest.approx(0.6 * float(q[0] @ k[0]), abs=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_uniform_scores(rng, causal):
    n = 17
    q = np.zeros((n, 8))
    k, v = _rand(rng, n, 8), _rand(rng, n, 6)
    o, lse = oa.head_forward(q, k, v, 0.5, causal)
    for i in range(n):
        vis = i + 1 if causal else n
        np.testing.assert_allclose(o[i], v[:vis].mean(axis=0), atol=1e-12)
        assert lse[i] == pytest.approx(math.log(vis), abs=1e-12)


def test_lse_against_fsum(rng):
    n = 12
    q, k = _rand(rng, n, 4, std=3), _rand(rng, n, 4, std=3)
    for causal in (False, True):
        _, lse = oa.head_forward(q, k, _rand(rng, n, 2), 0.9, causal)
        for i in range(n):
            zs = [0.9 * math.fsum(q[i, d] * k[j, d] for d in range(4))
                  for j in range(n) if not (causal and j > i)]
            mx = max(zs)
            ref = mx + math.log(math.fsum(math.exp(z - mx) for z in zs))
            assert lse[i] == pytest.approx(ref, abs=1e-12)


def _brute_force(q, k, v, scale, causal):
    """Pure-Python loops over the definition, for tiny inputs."""
    n, d = q.shape
    dv = v.shape[1]
    o = [[0.0] * dv for _ in range(n)]
    lse = [0.0] * n
    for i in range(n):
        z = []
        for j in range(k.shape[0]):
            if causal and j > i:
                continue
            z.append((j, scale * math.fsum(q[i, t] * k[j, t] for t in range(d))))
        mx = max(s for _, s in z)
        w = [(j, math.exp(s - mx)) for j, s in z]
        tot = math.fsum(e for _, e in w)
        for c in range(dv):
            o[i][c] = math.fsum(e * v[j, c] for j, e in w) / tot
        lse[i] = mx + math.log(tot)
    return np.array(o), np.array(lse)


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_tiny(rng, causal):
    for n, d, dv in [(1, 3, 2), (4, 5, 3), (9, 4, 6)]:
        q, k, v = _rand(rng, n, d, std=2), _rand(rng, n, d, std=2), _rand(rng, n, dv)
        o, lse = oa.head_forward(q, k, v, 0.45, causal)
        o_bf, lse_bf = _brute_force(q, k, v, 0.45, causal)
        np.testing.assert_allclose(o, o_bf, atol=1e-12)
        np.testing.assert_allclose(lse, lse_bf, atol=1e-12)


# --------------------------------------------------- layouts and grouping ---

def _packed(rng, lengths, H, H_kv, D):
    T = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return (_rand(rng, T, H, D, std=1.5), _rand(rng, T, H_kv, D, std=1.5),
            _rand(rng, T, H_kv, D), _rand(rng, T, H, D), cu)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_dense_per_sequence(rng, causal):
    lengths = [5, 1, 0, 9, 3]
    q, k, v, do, cu = _packed(rng, lengths, 3, 3, 4)
    o, lse = oa.attention_forward(q, k, v, cu, causal, 0.5)
    dq, dk, dv = oa.attention_backward(q, k, v, do, cu, causal, 0.5)
    for s0, s1 in zip(cu[:-1], cu[1:]):
        if s1 == s0:
            continue
        one = np.array([0, s1 - s0])
        o1, lse1 = oa.attention_forward(q[s0:s1], k[s0:s1], v[s0:s1], one, causal, 0.5)
        g1 = oa.attention_backward(q[s0:s1], k[s0:s1], v[s0:s1], do[s0:s1], one, causal, 0.5)
        np.testing.assert_array_equal(o[s0:s1], o1)
        np.testing.assert_array_equal(lse[:, s0:s1], lse1)
        for a, b in zip((dq, dk, dv), g1):
            np.testing.assert_array_equal(a[s0:s1], b)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_equals_repeated_kv(rng, causal):
    H, H_kv, D = 6, 2, 4
    q, k, v, do, cu = _packed(rng, [7, 4], H, H_kv, D)
    g = H // H_kv
    o, lse = oa.attention_forward(q, k, v, cu, causal, 0.5)
    dq, dk, dv = oa.attention_backward(q, k, v, do, cu, causal, 0.5)
    k_rep, v_rep = np.repeat(k, g, axis=1), np.repeat(v, g, axis=1)
    o_r, lse_r = oa.attention_forward(q, k_rep, v_rep, cu, causal, 0.5)
    dq_r, dk_r, dv_r = oa.attention_backward(q, k_rep, v_rep, do, cu, causal, 0.5)
    np.testing.assert_allclose(o, o_r, atol=1e-14)
    np.testing.assert_allclose(lse, lse_r, atol=1e-14)
    np.testing.assert_allclose(dq, dq_r, atol=1e-14)
    np.testing.assert_allclose(dk, dk_r.reshape(-1, H_kv, g, D).sum(axis=2), atol=1e-13)
    np.testing.assert_allclose(dv, dv_r.reshape(-1, H_kv, g, D).sum(axis=2), atol=1e-13)


def test_lse_dense_layout():
    B, H, N = 2, 3, 4
    lse_ht = np.arange(H * B * N, dtype=np.float64).reshape(H, B * N)
    out = oa.lse_dense_layout(lse_ht, B, N)
    for b, h, i in itertools.product(range(B), range(H), range(N)):
        assert out[b, h, i] == lse_ht[h, b * N + i]


# --------------------------------------------------------------- backward ---

def _loss(q, k, v, do, cu, causal, scale):
    o, _ = oa.attention_forward(q, k, v, cu, causal, scale)
    return float(np.sum(o * do))


def _fd_check(backward, rng, H_kv, lengths, causal, D=4, H=2, scale=0.7, h=1e-6):
    q, k, v, do, cu = _packed(rng, lengths, H, H_kv, D)
    grads = backward(q, k, v, do, cu, causal, scale)
    worst = 0.0
    for idx, (x, g) in enumerate(zip((q, k, v), grads)):
        num = np.zeros_like(x)
        for pos in np.ndindex(x.shape):
            xp = [a.copy() for a in (q, k, v)]
            xm = [a.copy() for a in (q, k, v)]
            xp[idx][pos] += h
            xm[idx][pos] -= h
            num[pos] = (_loss(*xp, do, cu, causal, scale) - _loss(*xm, do, cu, causal, scale)) / (2 * h)
        denom = max(np.abs(num).max(), 1e-3)
        worst = max(worst, float(np.abs(g - num).max() / denom))
    return worst


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H_kv", [1, 2])
@pytest.mark.parametrize("lengths", [[1], [3], [5], [3, 5, 1]])
def test_backward_finite_differences(rng, causal, H_kv, lengths):
    assert _fd_check(oa.attention_backward, rng, H_kv, lengths, causal) < 1e-6


def test_backward_single_key_closed_form(rng):
    # One key: P = 1 whatever the logits, so dV = dO and dQ = dK = 0.
    q, k, v, do, cu = _packed(rng, [1], 2, 2, 5)
    dq, dk, dv = oa.attention_backward(q, k, v, do, cu, False, 0.3)
    np.testing.assert_allclose(dv, do, atol=1e-15)
    assert np.abs(dq).max() < 1e-15 and np.abs(dk).max() < 1e-15


def test_sampled_rows_match_full(rng):
    n = 70
    q, k, v, do = (_rand(rng, n, 8, std=s) for s in (2, 2, 1, 1))
    rows = np.array([0, 5, 33, 69])
    for causal in (False, True):
        o, lse = oa.head_forward(q, k, v, 0.3, causal)
        o_r, lse_r = oa.head_forward(q, k, v, 0.3, causal, rows=rows)
        np.testing.assert_allclose(o_r, o[rows], atol=1e-14)
        np.testing.assert_allclose(lse_r, lse[rows], atol=1e-14)
        dq, dk, dv = oa.head_backward(q, k, v, do, 0.3, causal)
        dq_r, _, _ = oa.head_backward(q, k, v, do, 0.3, causal, q_rows=rows, want_kv=False)
        np.testing.assert_allclose(dq_r, dq[rows], atol=1e-13)


# ------------------------------------------------------------- mutations ---

MUTATIONS = [
    # (description, original text, mutated text)
    ("scale dropped from S", "s = scale * (q @ k.T)", "s = (q @ k.T)"),
    ("diagonal masked", "cols[None, :] > np.asarray(rows)[:, None]",
     "cols[None, :] >= np.asarray(rows)[:, None]"),
    ("LSE sign", "m_safe + np.log(", "m_safe - np.log("),
    ("D term dropped", "ds = p * (dp - delta[:, None])", "ds = p * dp"),
    ("dK operand transposed", "dk += scale * (ds.T @ q[r])", "dk += scale * (ds @ q[r])"),
    ("dQ scale dropped", "dq = scale * (ds @ k)", "dq = (ds @ k)"),
    ("dV from dP", "dv += p.T @ do[r]", "dv += p @ do[r]"),
    ("GQA mapping", "hk = h // g\n            o[", "hk = h % H_kv\n            o["),
]


def _mutant(orig, new):
    src = open(oa.__file__).read()
    assert orig in src, orig
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(orig, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


def _pins_pass(mod, rng):
    """A compact re-run of the pins above against a mutated module."""
    try:
        for causal in (False, True):
            for n, d, dv in [(4, 5, 3), (9, 4, 6)]:
                q, k, v = _rand(rng, n, d, std=2), _rand(rng, n, d, std=2), _rand(rng, n, dv)
                o, lse = mod.head_forward(q, k, v, 0.45, causal)
                o_bf, lse_bf = _brute_force(q, k, v, 0.45, causal)
                if not (np.allclose(o, o_bf, atol=1e-10) and np.allclose(lse, lse_bf, atol=1e-10)):
                    return False
        H, H_kv, D = 4, 2, 4
        q, k, v, do, cu = _packed(rng, [5, 3], H, H_kv, D)
        o, _ = mod.attention_forward(q, k, v, cu, True, 0.5)
        o_r, _ = mod.attention_forward(q, np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1),
                                       cu, True, 0.5)
        if not np.allclose(o, o_r, atol=1e-12):
            return False
        for causal in (False, True):
            worst = _fd_check(mod.attention_backward, rng, 2, [4, 3], causal)
            if not worst < 1e-6:
                return False
    except Exception:
        return False
    return True


def test_pins_pass_on_the_oracle(rng):
    assert _pins_pass(oa, rng)


@pytest.mark.parametrize("desc,orig,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(rng, desc, orig, new):
    assert not _pins_pass(_mutant(orig, new), rng), desc


def test_package_exports():
    assert oracle.attention_forward is oa.attention_forward
