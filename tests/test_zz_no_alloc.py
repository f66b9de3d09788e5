"""fa_bwd_noalloc: the backward pass for callers that cannot allocate.

Some callers are handed only their inputs and outputs and may not call
cudaMalloc (a plugin inside a framework that owns all device memory, or a
latency-critical path). fa_bwd_noalloc serves them from a scratch array built
into the library instead of a caller workspace. These tests call it through
the C ABI and check it against fa_bwd, the entry point with a caller
workspace, on two calls in a row (the scratch keeps the previous call's
contents, so the second call must not depend on them).
"""
import ctypes

import numpy as np
import pytest
import torch

from exact_io_aware_tmem_b200 import _abi
from exact_io_aware_tmem_b200.workloads import random_case

REL_BF16 = 3e-2   # the bf16 backward tolerance of the parity tests
TOL_F32 = 1e-5    # the fp32 tolerance of the parity tests
SCRATCH_BYTES = 32 * 1024 * 1024


@pytest.fixture(scope="module")
def lib():
    from exact_io_aware_tmem_b200 import build
    build.build()
    return _abi.lib()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _problem(seed, dtype, lengths, H, H_kv, D, varlen, causal):
    inp = random_case(seed, dtype=dtype, lengths=lengths, H=H, H_kv=H_kv, D=D, varlen=varlen)
    dev = {n: getattr(inp, n).cuda().contiguous() for n in ("q", "k", "v", "do")}
    T = inp.q.shape[0]
    B = len(lengths)
    N = 0 if varlen else lengths[0]
    cu = inp.cu_seqlens.cuda() if varlen else None
    lse = torch.empty((H, T) if varlen else (B, H, N), device="cuda", dtype=torch.float32)
    o = torch.empty_like(dev["q"])
    fa_dtype = _abi.FA_BF16 if dtype == "bf16" else _abi.FA_F32
    args = dict(B=B, H=H, H_kv=H_kv, N=N, D=D, dtype=fa_dtype, causal=int(causal),
                cu=cu, max_seqlen=inp.max_seqlen if varlen else 0, T=T)
    return dev, o, lse, args


def _fwd(lib, dev, o, lse, a):
    st = lib.fa_fwd(_p(dev["q"]), _p(dev["k"]), _p(dev["v"]), _p(o), _p(lse), a["B"], a["H"],
                    a["H_kv"], a["N"], a["D"], a["dtype"], a["causal"], -1.0,
                    None if a["cu"] is None else _p(a["cu"]), a["max_seqlen"], a["T"], None)
    assert st == _abi.FA_OK


def _grads(dev):
    return (torch.full_like(dev["q"], float("nan")), torch.full_like(dev["k"], float("nan")),
            torch.full_like(dev["v"], float("nan")))


def _bwd_with_workspace(lib, dev, o, lse, a, mask):
    """fa_bwd_phases(mask) with a caller-allocated workspace."""
    dq, dk, dv = _grads(dev)
    need = lib.fa_bwd_phases_workspace_size(mask, a["T"], a["H"], a["D"], a["dtype"])
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    st = lib.fa_bwd_phases(mask, _p(dev["q"]), _p(dev["k"]), _p(dev["v"]), _p(o), _p(lse),
                           _p(dev["do"]), _p(dq), _p(dk), _p(dv), a["B"], a["H"], a["H_kv"],
                           a["N"], a["D"], a["dtype"], a["causal"], -1.0,
                           None if a["cu"] is None else _p(a["cu"]), a["max_seqlen"], a["T"],
                           _p(ws), need, None)
    assert st == _abi.FA_OK
    return dq, dk, dv


def _bwd_noalloc(lib, dev, o, lse, a):
    dq, dk, dv = _grads(dev)
    st = lib.fa_bwd_noalloc(_p(dev["q"]), _p(dev["k"]), _p(dev["v"]), _p(o), _p(lse),
                            _p(dev["do"]), _p(dq), _p(dk), _p(dv), a["B"], a["H"], a["H_kv"],
                            a["N"], a["D"], a["dtype"], a["causal"], -1.0,
                            None if a["cu"] is None else _p(a["cu"]), a["max_seqlen"], a["T"],
                            None)
    assert st == _abi.FA_OK
    return dq, dk, dv


def _close(got, ref, dtype):
    """Within the parity tolerance of the backward tests."""
    for g, r in zip(got, ref):
        g = g.double().cpu().numpy()
        r = r.double().cpu().numpy()
        assert np.isfinite(g).all()
        if dtype == "bf16":
            assert np.linalg.norm(g - r) / np.linalg.norm(r) <= REL_BF16
        else:
            assert np.abs(g - r).max() <= TOL_F32


def _same_bits(got, ref):
    """fa_bwd_noalloc runs the split backward's kernels, which add nothing
    atomically, so its results must be identical to the split backward run
    with a caller workspace; a difference would mean the built-in scratch fed
    a kernel something the caller's workspace did not."""
    for g, r in zip(got, ref):
        assert torch.equal(g, r)


CASES = [
    # (seed, dtype, lengths, H, H_kv, D, varlen, causal)
    (1, "bf16", [700, 700], 4, 2, 128, False, True),
    (2, "bf16", [5, 0, 300, 129], 4, 4, 64, True, False),
    (3, "f32", [130, 130], 2, 1, 64, False, True),
]
# Run through fa_bwd_noalloc between a case's two calls, so the shared scratch
# holds another problem's values when the second call starts.
OTHER = (9, "bf16", [1000], 8, 8, 128, False, False)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice_in_a_row(lib):
    other = _problem(*OTHER)
    _fwd(lib, *other)
    for case in CASES:
        dtype = case[1]
        dev, o, lse, a = _problem(*case)
        _fwd(lib, dev, o, lse, a)
        ref = _bwd_with_workspace(lib, dev, o, lse, a, _abi.BWD_FUSED)       # fa_bwd's path
        ref_split = _bwd_with_workspace(lib, dev, o, lse, a, _abi.BWD_SPLIT)
        first = _bwd_noalloc(lib, dev, o, lse, a)
        _bwd_noalloc(lib, *other)
        second = _bwd_noalloc(lib, dev, o, lse, a)
        torch.cuda.synchronize()
        where = ctypes.c_uint(0)
        assert lib.fa_check_device_error(None, ctypes.byref(where)) == _abi.FA_OK
        _close(first, ref, dtype)
        _close(second, ref, dtype)
        _same_bits(first, ref_split)
        _same_bits(second, ref_split)


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    # T * H * 4 bytes > 32 MiB: refused before anything is enqueued (no pointer
    # is touched, so none is needed).
    T, H, D = 9_000_000, 1, 128
    need = lib.fa_bwd_phases_workspace_size(_abi.BWD_SPLIT, T, H, D, _abi.FA_BF16)
    assert need > SCRATCH_BYTES
    st = lib.fa_bwd_noalloc(None, None, None, None, None, None, None, None, None, 1, H, H, T, D,
                            _abi.FA_BF16, 0, -1.0, None, 0, 0, None)
    assert st == _abi.FA_ERR_UNSUPPORTED


@pytest.mark.parametrize("B,H,H_kv,N,D,dtype", [
    (1, 6, 4, 9_000_000, 128, _abi.FA_BF16),    # H % H_kv != 0, and beyond the scratch
    (1, 4, 4, 9_000_000, 96, _abi.FA_BF16),     # unsupported head dim, and beyond the scratch
    (1, 4, 4, 1024, 128, 7),                    # unknown dtype
    (-1, 4, 4, 1024, 128, _abi.FA_BF16),        # negative batch
])
def test_noalloc_reports_argument_errors_as_fa_bwd_does(lib, B, H, H_kv, N, D, dtype):
    # Argument errors are found before any pointer is read or anything is
    # enqueued, so null pointers are enough to compare the two statuses.
    ref = lib.fa_bwd(None, None, None, None, None, None, None, None, None, B, H, H_kv, N, D,
                     dtype, 0, -1.0, None, 0, 0, None, 0, None)
    got = lib.fa_bwd_noalloc(None, None, None, None, None, None, None, None, None, B, H, H_kv,
                             N, D, dtype, 0, -1.0, None, 0, 0, None)
    assert ref != _abi.FA_OK
    assert got == ref
