"""GPU forward parity against the float64 oracle (through the C ABI).

Tolerances (from the method's target and the arithmetic):
  float32 path: max-abs <= 1e-5 on O and LSE;
  bf16 path:    |O - O_ref| <= 1.5e-2 + 2^-9 |O_ref| (the bound on the
                computed value plus at most half a bf16 ulp from casting the
                output to bf16), max-abs <= 1e-3 on LSE.
Small cases span several 128-row tiles with ragged tails; the full-size
workloads are checked on sampled rows the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import exact_io_aware_tmem_b200 as fa
from exact_io_aware_tmem_b200.workloads import WORKLOADS, make_inputs, random_case
from oracle import attention as oa
from tests._util import (f64, max_abs, o_excess_bf16, oracle_lse_layout, sample_forward,
                         to_api)

pytestmark = pytest.mark.gpu

O_TOL_BF16 = 1.5e-2
LSE_TOL_BF16 = 1e-3
TOL_F32 = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    from exact_io_aware_tmem_b200 import build
    build.build()


def run_fwd(inp, causal, scale, B, N):
    a = to_api(inp, B, N)
    o, lse = fa.fwd(a["q"], a["k"], a["v"], causal=causal, scale=scale,
                    cu_seqlens=a.get("cu_seqlens"), max_seqlen=a.get("max_seqlen"))
    st, where = fa.check_device_error()
    assert st == 0, f"device error {st} at {where:#x}"
    return o, lse


def check_full(inp, causal, scale, B, N, o_tol, lse_tol):
    o, lse = run_fwd(inp, causal, scale, B, N)
    o_ref, lse_ref = oa.attention_forward(inp.q, inp.k, inp.v, inp.cu_seqlens.numpy(), causal,
                                          scale)
    T = inp.q.shape[0]
    o = f64(o).reshape(T, inp.q.shape[1], -1)
    err_l = max_abs(f64(lse), oracle_lse_layout(lse_ref, inp, B, N))
    assert np.isfinite(o).all()
    if inp.q.dtype == torch.bfloat16:
        excess = o_excess_bf16(o, o_ref, o_tol)
        assert excess <= 0, f"O outside the bf16 bound by {excess} (max-abs {max_abs(o, o_ref)})"
    else:
        err_o = max_abs(o, o_ref)
        assert err_o <= o_tol, f"O max-abs {err_o}"
    assert err_l <= lse_tol, f"LSE max-abs {err_l}"
    return err_l


# ------------------------------------------------------------ float32 path ---

def test_f32_workload_forward():
    w = WORKLOADS["f32_b1_h2_n128_d64"]
    check_full(make_inputs(w), w.causal, w.scale, w.B, w.N, TOL_F32, TOL_F32)


@pytest.mark.parametrize("D", [1, 32, 64, 100, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_f32_dense_shapes(D, causal):
    inp = random_case(10 + D, dtype="f32", lengths=[77, 77], H=3, H_kv=1, D=D, varlen=False)
    check_full(inp, causal, D ** -0.5, 2, 77, TOL_F32, TOL_F32)


@pytest.mark.parametrize("causal", [False, True])
def test_f32_varlen_ragged(causal):
    lengths = [1, 0, 37, 130, 64]
    inp = random_case(5, dtype="f32", lengths=lengths, H=4, H_kv=2, D=64, varlen=True)
    check_full(inp, causal, 0.125, len(lengths), 0, TOL_F32, TOL_F32)


# --------------------------------------------------------------- bf16 path ---

DENSE_CASES = [
    # (B, N, H, H_kv, D)
    (1, 128, 2, 2, 128),
    (2, 300, 4, 2, 128),
    (1, 1, 2, 1, 128),
    (1, 129, 3, 3, 64),
    (2, 255, 4, 4, 64),
    (1, 513, 8, 1, 128),
    (3, 64, 2, 2, 64),
]


@pytest.mark.parametrize("B,N,H,H_kv,D", DENSE_CASES)
@pytest.mark.parametrize("causal", [False, True])
def test_bf16_dense(B, N, H, H_kv, D, causal):
    inp = random_case(B * 1000 + N + D, dtype="bf16", lengths=[N] * B, H=H, H_kv=H_kv, D=D,
                      varlen=False)
    check_full(inp, causal, D ** -0.5, B, N, O_TOL_BF16, LSE_TOL_BF16)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bf16_varlen_ragged(D, causal):
    lengths = [5, 0, 128, 1, 300, 129, 257]
    inp = random_case(77, dtype="bf16", lengths=lengths, H=4, H_kv=2, D=D, varlen=True)
    check_full(inp, causal, D ** -0.5, len(lengths), 0, O_TOL_BF16, LSE_TOL_BF16)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bf16_many_pairs_ragged(D, causal):
    # More query-tile pairs than SMs, so a persistent CTA works on several
    # pairs in turn, many of them with an empty second tile.
    lengths = [int(x) for x in np.random.default_rng(12).integers(1, 700, size=48)]
    lengths[3] = 0
    inp = random_case(13, dtype="bf16", lengths=lengths, H=8, H_kv=4, D=D, varlen=True)
    check_full(inp, causal, D ** -0.5, len(lengths), 0, O_TOL_BF16, LSE_TOL_BF16)


@pytest.mark.parametrize("D", [64, 128])
def test_bf16_large_logits_rescale(D):
    # Logit std ~ 8: the running max moves often and the O rescale path runs
    # (at D = 64 in each softmax group's own accumulator).
    inp = random_case(3, dtype="bf16", lengths=[640], H=2, H_kv=2, D=D, varlen=False, std=2.8)
    for causal in (False, True):
        check_full(inp, causal, D ** -0.5, 1, 640, O_TOL_BF16, LSE_TOL_BF16)


def test_bf16_custom_scale():
    inp = random_case(4, dtype="bf16", lengths=[200], H=2, H_kv=1, D=64, varlen=False)
    check_full(inp, True, 0.37, 1, 200, O_TOL_BF16, LSE_TOL_BF16)


def test_bf16_deterministic():
    inp = random_case(9, dtype="bf16", lengths=[384, 384], H=4, H_kv=4, D=128, varlen=False)
    o1, l1 = run_fwd(inp, True, None, 2, 384)
    o2, l2 = run_fwd(inp, True, None, 2, 384)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ---------------------------------------------- full-size workloads, sampled ---

def _picks(inp, H, n_heads=3, n_rows=24, seed=0):
    rng = np.random.default_rng(seed)
    cu = inp.cu_seqlens.tolist()
    B = len(cu) - 1
    picks = []
    for _ in range(n_heads):
        b = int(rng.integers(B))
        L = cu[b + 1] - cu[b]
        rows = sorted(set([0, L - 1] + rng.integers(0, L, n_rows).tolist()))
        picks.append((b, int(rng.integers(H)), rows))
    return picks


@pytest.mark.parametrize("name", [n for n in WORKLOADS if WORKLOADS[n].dtype == "bf16"])
def test_bf16_workload_sampled(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    B = len(inp.cu_seqlens) - 1
    o, lse = run_fwd(inp, w.causal, w.scale, B, w.N)
    T = inp.q.shape[0]
    o = o.reshape(T, w.H, w.D)
    for b, h, rows, o_ref, lse_ref in sample_forward(inp, w.causal, w.scale, _picks(inp, w.H)):
        s0 = int(inp.cu_seqlens[b])
        idx = torch.as_tensor(s0 + rows, device=o.device)
        got = f64(o[idx, h])
        if inp.varlen:
            got_lse = f64(lse[h, idx])
        else:
            got_lse = f64(lse[b, h, torch.as_tensor(rows, device=o.device)])
        assert o_excess_bf16(got, o_ref, O_TOL_BF16) <= 0
        assert max_abs(got_lse, lse_ref) <= LSE_TOL_BF16
    assert torch.isfinite(o).all()
