"""GPU backward parity against the float64 oracle (through the C ABI).

Tolerances: float32 path max-abs <= 1e-5 on dQ, dK, dV; bf16 path
relative Frobenius error <= 3e-2 on dQ, dK, dV.
"""
import numpy as np
import pytest
import torch

import exact_io_aware_tmem_b200 as fa
from exact_io_aware_tmem_b200.workloads import WORKLOADS, make_inputs, random_case
from oracle import attention as oa
from tests._util import f64, max_abs, rel_fro, to_api

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
REL_BF16 = 3e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    from exact_io_aware_tmem_b200 import build
    build.build()


def run_fwd_bwd(inp, causal, scale, B, N):
    a = to_api(inp, B, N)
    kw = dict(causal=causal, scale=scale, cu_seqlens=a.get("cu_seqlens"),
              max_seqlen=a.get("max_seqlen"))
    o, lse = fa.fwd(a["q"], a["k"], a["v"], **kw)
    dq, dk, dv = fa.bwd(a["do"], a["q"], a["k"], a["v"], o, lse, **kw)
    st, where = fa.check_device_error()
    assert st == 0, f"device error {st} at {where:#x}"
    T = inp.q.shape[0]
    return (f64(dq).reshape(T, inp.q.shape[1], -1), f64(dk).reshape(T, inp.k.shape[1], -1),
            f64(dv).reshape(T, inp.k.shape[1], -1))


def check_f32(inp, causal, scale, B, N):
    got = run_fwd_bwd(inp, causal, scale, B, N)
    ref = oa.attention_backward(inp.q, inp.k, inp.v, inp.do, inp.cu_seqlens.numpy(), causal, scale)
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        err = max_abs(g, r)
        assert err <= TOL_F32, f"{name} max-abs {err}"


def test_f32_workload_backward():
    w = WORKLOADS["f32_b1_h2_n128_d64"]
    check_f32(make_inputs(w), w.causal, w.scale, w.B, w.N)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,H_kv,D", [(2, 2, 64), (4, 1, 32), (6, 3, 128), (2, 1, 17)])
def test_f32_dense(causal, H, H_kv, D):
    inp = random_case(H * 100 + D, dtype="f32", lengths=[70, 70], H=H, H_kv=H_kv, D=D,
                      varlen=False)
    check_f32(inp, causal, D ** -0.5, 2, 70)


@pytest.mark.parametrize("causal", [False, True])
def test_f32_varlen_ragged(causal):
    lengths = [1, 0, 45, 130, 3]
    inp = random_case(8, dtype="f32", lengths=lengths, H=4, H_kv=2, D=64, varlen=True)
    check_f32(inp, causal, 0.125, len(lengths), 0)
