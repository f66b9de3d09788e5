"""The debug build (libfa_b200_debug.so): the same kernels with index checks
that record into the device error word instead of trapping, and per-role
event stamps of one CTA (include/fa.h, "Debug build").

The GPU tests run small causal and packed cases through it, check them against
the float64 oracle with the parity tolerances, check that no index check
fired, and that the stamps of a traced CTA form a timeline.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_io_aware_tmem_b200 as fa
from exact_io_aware_tmem_b200 import _abi
from exact_io_aware_tmem_b200 import attention as fa_att
from exact_io_aware_tmem_b200 import trace
from exact_io_aware_tmem_b200.workloads import random_case
from oracle import attention as oa
from tests._util import f64, o_excess_bf16, rel_fro, to_api


@pytest.fixture(scope="module")
def debug_lib():
    from exact_io_aware_tmem_b200 import build
    build.build()
    build.build(debug=True)
    return _abi.debug_lib()


def test_debug_build_loads_and_reports_itself(debug_lib):
    assert debug_lib.fa_debug_build() == 1
    assert _abi.lib().fa_debug_build() == 0
    # The ordinary build records no stamps.
    assert _abi.lib().fa_debug_set_trace(ctypes.c_void_p(256), _abi.DEBUG_TRACE_BYTES, 0) == \
        _abi.FA_ERR_UNSUPPORTED
    # Argument checks of the debug build's trace switch (no device access).
    assert debug_lib.fa_debug_set_trace(ctypes.c_void_p(256), 8, 0) == _abi.FA_ERR_INVALID_ARG
    assert debug_lib.fa_debug_set_trace(ctypes.c_void_p(256), _abi.DEBUG_TRACE_BYTES, -1) == \
        _abi.FA_ERR_INVALID_ARG
    assert debug_lib.fa_debug_set_trace(None, 0, 0) == _abi.FA_OK


CASES = [
    # (lengths, H, H_kv, D, varlen, causal)
    ([384, 384], 4, 2, 128, False, True),
    ([5, 0, 128, 1, 300, 129, 64], 4, 2, 128, True, False),
    ([300, 129, 257], 4, 4, 64, True, True),
]


@pytest.mark.gpu
@pytest.mark.parametrize("lengths,H,H_kv,D,varlen,causal", CASES)
def test_debug_build_parity_and_clean_checks(debug_lib, lengths, H, H_kv, D, varlen, causal):
    inp = random_case(31, dtype="bf16", lengths=lengths, H=H, H_kv=H_kv, D=D, varlen=varlen)
    B = len(lengths)
    N = 0 if varlen else lengths[0]
    a = to_api(inp, B, N)
    kw = dict(causal=causal, cu_seqlens=a.get("cu_seqlens"), max_seqlen=a.get("max_seqlen"))
    with fa_att.debug_build():
        o, lse = fa.fwd(a["q"], a["k"], a["v"], **kw)
        grads = fa.bwd(a["do"], a["q"], a["k"], a["v"], o, lse, **kw)
        st, where = fa.check_device_error()
    assert st == 0, f"debug build reported {st} at {where:#x}"
    scale = D ** -0.5
    ro, _ = oa.attention_forward(inp.q, inp.k, inp.v, inp.cu_seqlens.numpy(), causal, scale)
    T = inp.q.shape[0]
    assert o_excess_bf16(f64(o).reshape(T, H, D), ro) <= 0
    ref = oa.attention_backward(inp.q, inp.k, inp.v, inp.do, inp.cu_seqlens.numpy(), causal, scale)
    for g, r in zip(grads, ref):
        assert rel_fro(f64(g).reshape(r.shape), r) <= 3e-2


@pytest.mark.gpu
@pytest.mark.parametrize("kernel", ["fwd", "bwd"])
def test_debug_build_stamps_form_a_timeline(debug_lib, kernel):
    """One traced CTA of the causal B2 H16 N8192 workload: every step of the
    traced roles is stamped, in order."""
    stamps, n = trace.run(kernel, "bf16_causal_b2_h16_n8192_d128", cta=0)
    kinds = trace.BWD_KINDS if kernel == "bwd" else trace.FWD_KINDS
    first = "S_SFULL" if kernel == "bwd" else "W1_SFULL"
    # CTA 0 is the longest causal one: 64 key tiles (forward, second query
    # tile of the last pair) or 64 query tiles (backward, key tile 0).
    assert n == 64
    s = stamps[kinds[first]][:n].astype(np.int64)
    assert (np.diff(s) > 0).all()
    table = trace.BWD_SPANS if kernel == "bwd" else trace.FWD_SPANS
    for label, med, mean, p90, cnt in trace.spans(stamps, kinds, table, n):
        assert med is not None and cnt > 0 and med <= p90, label


@pytest.mark.gpu
def test_debug_build_decode_stamps(debug_lib):
    """One traced CTA of the balanced decode (16 sequences, 64-row pages):
    its group of H_kv CTAs takes an equal share of the (sequence, key tile)
    units, and the CTA publishes each of its tiles in order."""
    from exact_io_aware_tmem_b200.workloads import DECODE_WORKLOADS
    name = "bf16_decode_paged64_b16_h32_kv8_d128_q1"
    w = DECODE_WORKLOADS[name]
    units = sum(-(-n // 128) for n in w.lengths())
    groups = 148 // w.H_kv
    stamps, n = trace.run("dec", name, cta=5)
    assert n in (units // groups, units // groups + 1)
    s = stamps[trace.DEC_KINDS["W_ARR"]][:n].astype(np.int64)
    assert (np.diff(s) > 0).all()
    # every CTA's SM and span
    sm, st, en = (stamps[k][:groups * w.H_kv].astype(np.int64)
                  for k in (trace.CTA_SM, trace.CTA_START, trace.CTA_END))
    assert (sm >= 1).all() and (sm <= 148).all() and (en > st).all() and (st > 0).all()
    for label, med, mean, p90, cnt in trace.spans(stamps, trace.DEC_KINDS, trace.DEC_SPANS, n):
        assert med is not None and cnt > 0, label
    assert trace.cta_report(stamps)


@pytest.mark.gpu
def test_debug_build_d64_stamps(debug_lib):
    """The D = 64 forward on B4 H16 N2048: the traced CTA stamps its 16 key
    tiles in order, and all 1024 CTAs record their SM and span, at most two
    resident per SM at a time."""
    name = "bf16_fwd_b4_h16_n2048_d64"
    stamps, n = trace.run("d64", name, cta=3)
    assert n == 16
    s = stamps[trace.D64_KINDS["W_ARR"]][:n].astype(np.int64)
    assert (np.diff(s) > 0).all()
    sm, st, en = (stamps[k].astype(np.int64) for k in (trace.CTA_SM, trace.CTA_START,
                                                         trace.CTA_END))
    assert (sm >= 1).all() and (sm <= 148).all() and (en > st).all() and (st > 0).all()
    for s_id in np.unique(sm):
        ev = sorted([(int(a), 1) for a in st[sm == s_id]] + [(int(b), -1) for b in en[sm == s_id]],
                    key=lambda e: (e[0], e[1]))
        live = np.cumsum([d for _, d in ev])
        assert live.max() <= 2, s_id
    for label, med, mean, p90, cnt in trace.spans(stamps, trace.D64_KINDS, trace.D64_SPANS, n):
        assert med is not None and cnt > 0, label
    assert trace.cta_report(stamps)


def test_cta_report_host_arithmetic():
    """cta_report on hand-made spans: two SMs over a 100 us wall, SM 0 with
    two CTAs back to back (covered all the time, one resident on average),
    SM 1 with one CTA for the first half."""
    stamps = np.zeros((32, 1024), dtype=np.int64)
    rows = [(0, 0, 50_000), (0, 50_000, 100_000), (1, 0, 50_000)]
    for i, (s, a, b) in enumerate(rows):
        stamps[trace.CTA_SM][i] = s + 1
        stamps[trace.CTA_START][i] = 1_000 + a
        stamps[trace.CTA_END][i] = 1_000 + b
    lines = trace.cta_report(stamps)
    assert "CTAs: 3, all done 100.0 us" in lines[0]
    assert "median 50.0" in lines[0]
    assert "SMs: 2; mean CTAs resident 0.75 (min 0.50)" in lines[1]
    assert "time with a CTA resident 75.0 % (min 50.0 %)" in lines[1]
