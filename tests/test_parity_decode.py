"""GPU parity of the split-KV decode path (fa_decode) against the float64 oracle.

Tolerances are the forward's bf16 ones: |O - O_ref| <= 1.5e-2 + 2^-9 |O_ref|
and max-abs 1e-3 on LSE, with -inf LSE (no visible key) required exactly where
the oracle has it. Unused cache rows hold NaN (the input generator's fill), so
any read of them that reaches O shows up as a non-finite output.
"""
import numpy as np
import pytest
import torch

import exact_io_aware_tmem_b200 as fa
from exact_io_aware_tmem_b200.workloads import (DECODE_WORKLOADS, decode_case,
                                                make_decode_inputs)
from oracle import decode as od
from tests._util import f64, o_excess_bf16

pytestmark = pytest.mark.gpu

O_TOL = 1.5e-2
LSE_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    from exact_io_aware_tmem_b200 import build
    build.build()


def _run(c, *, causal, n_split=0, scale=None):
    dev = "cuda"
    max_len = int(c.cache_seqlens.max()) if c.cache_seqlens.numel() else 0
    o, lse = fa.decode(c.q.to(dev), c.k_cache.to(dev), c.v_cache.to(dev),
                       c.cache_seqlens.to(dev), q_len=c.q_len, max_seqlen_k=max_len,
                       block_table=None if c.block_table is None else c.block_table.to(dev),
                       page_size=c.page_size, causal=causal, scale=scale, n_split=n_split)
    st, where = fa.check_device_error()
    assert st == 0, f"device error {st} at {where:#x}"
    return f64(o), f64(lse)


def _ref(c, *, causal, scale):
    return od.decode_forward(c.q, c.k_cache, c.v_cache, c.cache_seqlens, q_len=c.q_len,
                             scale=scale, causal=causal, stride=c.page_size,
                             page_size=c.page_size, block_table=c.block_table)


def _check(o, lse, o_ref, lse_ref):
    assert np.isfinite(o).all(), "non-finite output"
    excess = o_excess_bf16(o, o_ref, O_TOL)
    assert excess <= 0, f"O outside the bf16 bound by {excess}"
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), "LSE -inf rows differ"
    if (~empty).any():
        err = np.abs(lse[~empty] - lse_ref[~empty]).max()
        assert err <= LSE_TOL, f"LSE max-abs {err}"
    assert np.all(o[empty] == 0)


@pytest.mark.parametrize("n_split", [1, 3, 0])
@pytest.mark.parametrize("D", [64, 128])
def test_contiguous_ragged_lengths(n_split, D):
    lengths = [1, 127, 128, 129, 1000, 300, 0, 640]
    c = decode_case(21 + D, dtype="bf16", lengths=lengths, q_len=1, H=8, H_kv=2, D=D)
    scale = D ** -0.5
    o, lse = _run(c, causal=True, n_split=n_split)
    _check(o, lse, *_ref(c, causal=True, scale=scale))


@pytest.mark.parametrize("page", [16, 64, 128, 256])
def test_paged_cache_any_block_order(page):
    lengths = [5, 300, 0, 777, 128, 129]
    c = decode_case(31 + page, dtype="bf16", lengths=lengths, q_len=4, H=16, H_kv=2, D=64,
                    page_size=page)
    o, lse = _run(c, causal=True, n_split=2)
    _check(o, lse, *_ref(c, causal=True, scale=0.125))


@pytest.mark.parametrize("causal", [True, False])
def test_full_tile_of_rows_q16_g8(causal):
    # 16 tokens x 8 heads sharing a kv head = one whole 128-row tile.
    lengths = [16, 200, 513]
    c = decode_case(41, dtype="bf16", lengths=lengths, q_len=16, H=16, H_kv=2, D=128)
    o, lse = _run(c, causal=causal, n_split=0)
    _check(o, lse, *_ref(c, causal=causal, scale=128 ** -0.5))


def test_tokens_without_visible_keys():
    # Cache shorter than q_len: the first tokens sit at negative positions and
    # see nothing under the causal rule (O = 0, LSE = -inf).
    lengths = [2, 0, 9]
    c = decode_case(51, dtype="bf16", lengths=lengths, q_len=5, H=4, H_kv=4, D=64)
    o, lse = _run(c, causal=True, n_split=1)
    _check(o, lse, *_ref(c, causal=True, scale=0.125))


def test_many_splits_and_scale():
    lengths = [4096, 1, 2500]
    c = decode_case(61, dtype="bf16", lengths=lengths, q_len=2, H=8, H_kv=1, D=128)
    o, lse = _run(c, causal=True, n_split=32, scale=0.2)
    _check(o, lse, *_ref(c, causal=True, scale=0.2))


# Balanced decode (D = 128, q_len * g <= 64, automatic splits): one persistent
# CTA per SM over equal ranges of (sequence, kv head, key tile) units.
BALANCED_LENGTHS = [1, 127, 128, 129, 0, 1000, 255, 256, 3000, 40, 2049, 7]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("q_len,H,H_kv", [(1, 8, 2), (3, 15, 3), (5, 16, 4), (8, 32, 8),
                                          (16, 16, 4), (9, 21, 3)])
def test_balanced_rows_and_lengths(q_len, H, H_kv, causal):
    # R = q_len * g = 4, 15, 20, 32, 64, 63: the 16-, 32- and 64-column
    # forms, odd g, and rows that do not fill their column block.
    c = decode_case(71 + q_len * H, dtype="bf16", lengths=BALANCED_LENGTHS, q_len=q_len, H=H,
                    H_kv=H_kv, D=128)
    o, lse = _run(c, causal=causal, n_split=0)
    _check(o, lse, *_ref(c, causal=causal, scale=128 ** -0.5))


@pytest.mark.parametrize("page", [16, 64, 128, 256])
def test_balanced_paged(page):
    c = decode_case(81 + page, dtype="bf16", lengths=BALANCED_LENGTHS, q_len=2, H=8, H_kv=2,
                    D=128, page_size=page)
    o, lse = _run(c, causal=True, n_split=0)
    _check(o, lse, *_ref(c, causal=True, scale=128 ** -0.5))


def test_balanced_more_ctas_than_tiles():
    # 6 tiles over one CTA per SM: most ranges are empty, some of them
    # strictly inside a segment whose pieces lie on both sides.
    c = decode_case(91, dtype="bf16", lengths=[300, 5, 0, 390], q_len=1, H=4, H_kv=1, D=128)
    o, lse = _run(c, causal=True, n_split=0)
    _check(o, lse, *_ref(c, causal=True, scale=128 ** -0.5))


def test_balanced_many_sequences():
    # 96 sequences: each CTA's range crosses several segments (Q buffers
    # reused, pieces written whole and as partials).
    rng = np.random.default_rng(17)
    lengths = [int(x) for x in rng.integers(0, 1500, size=96)]
    c = decode_case(101, dtype="bf16", lengths=lengths, q_len=1, H=16, H_kv=4, D=128)
    o, lse = _run(c, causal=True, n_split=0)
    _check(o, lse, *_ref(c, causal=True, scale=128 ** -0.5))


def test_balanced_reference_moves_mid_piece():
    # Keys whose norm grows along the cache: later tiles exceed the running
    # reference by far more than 2^8, so it moves inside pieces and O^T is
    # rescaled in TMEM.
    lengths = [5000, 2600, 900]
    c = decode_case(111, dtype="bf16", lengths=lengths, q_len=2, H=8, H_kv=2, D=128)
    ramp = torch.ones(c.k_cache.shape[0])
    for b, n in enumerate(lengths):
        ramp[b * c.page_size:b * c.page_size + n] = 1 + torch.arange(n) / 1024.0
    c.k_cache = (c.k_cache.float() * ramp[:, None, None]).to(c.k_cache.dtype)
    o, lse = _run(c, causal=True, n_split=0, scale=0.5)
    _check(o, lse, *_ref(c, causal=True, scale=0.5))


@pytest.mark.slow
@pytest.mark.parametrize("name", sorted(DECODE_WORKLOADS))
def test_decode_workload_sampled(name):
    # Full-size workload in the bench's launch configuration (automatic
    # splits); the oracle checks a sample of sequences.
    w = DECODE_WORKLOADS[name]
    c = make_decode_inputs(w)
    o, lse = _run(c, causal=w.causal)
    for b in (0, w.B // 2, w.B - 1):
        sub = decode_case(0, dtype="bf16", lengths=[1], q_len=w.q_len, H=w.H, H_kv=w.H_kv,
                          D=w.D)   # shape holder; replaced below
        n = int(c.cache_seqlens[b])
        rows = od.cache_rows(b, n, stride=c.page_size if not c.paged else None,
                             page_size=c.page_size if c.paged else None,
                             block_table=None if not c.paged else c.block_table.numpy())
        sub.q = c.q[b * w.q_len:(b + 1) * w.q_len]
        sub.k_cache = c.k_cache[rows]
        sub.v_cache = c.v_cache[rows]
        sub.cache_seqlens = torch.tensor([n], dtype=torch.int32)
        sub.block_table = None
        sub.page_size = n
        o_ref, lse_ref = _ref(sub, causal=w.causal, scale=w.scale)
        _check(o[b * w.q_len:(b + 1) * w.q_len], lse[b * w.q_len:(b + 1) * w.q_len],
               o_ref, lse_ref)
