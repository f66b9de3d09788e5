"""Host-side checks of the C ABI: symbols, error codes, argument validation.

None of these calls launches a kernel; they run without a GPU.
"""
import ctypes
import os
import re

import pytest

from exact_io_aware_tmem_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    return sorted(set(re.findall(r"^\s*(?:fa_status|size_t|const char\*|void|int)\s+(fa_\w+)\(",
                                 text, re.M)))


@pytest.fixture(scope="module")
def lib():
    from exact_io_aware_tmem_b200 import build
    build.build()
    return _abi.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 8
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(_abi.SIGNATURES), "binding and header disagree"


def test_version_and_error_strings(lib):
    assert lib.fa_version() == 100
    for code in range(5):
        s = lib.fa_get_error_string(code).decode()
        assert s.startswith("FA_")
    assert b"unknown" in lib.fa_get_error_string(99)


def test_workspace_size(lib):
    T, H, D = 1000, 16, 128
    r = lambda x: (x + 255) // 256 * 256
    assert lib.fa_bwd_workspace_size(T, H, D, _abi.FA_BF16) == r(T * H * 4) + 256
    assert lib.fa_bwd_workspace_size(T, H, D, _abi.FA_F32) == r(T * H * 4) + 256
    assert lib.fa_bwd_workspace_size(-1, H, D, _abi.FA_BF16) == 0


def _fwd(lib, **kw):
    a = dict(q=16, k=16, v=16, o=16, lse=16, B=1, H=2, H_kv=2, N=8, D=64, dtype=_abi.FA_BF16,
             causal=0, scale=0.0, cu=None, max_seqlen=0, total=0, stream=None)
    a.update(kw)
    return lib.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["H_kv"],
                      a["N"], a["D"], a["dtype"], a["causal"], a["scale"], a["cu"],
                      a["max_seqlen"], a["total"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(H=3, H_kv=2), _abi.FA_ERR_INVALID_ARG),        # H % H_kv != 0
    (dict(H=0), _abi.FA_ERR_INVALID_ARG),
    (dict(D=0), _abi.FA_ERR_INVALID_ARG),
    (dict(B=-1), _abi.FA_ERR_INVALID_ARG),
    (dict(N=-5), _abi.FA_ERR_INVALID_ARG),
    (dict(causal=2), _abi.FA_ERR_INVALID_ARG),
    (dict(dtype=7), _abi.FA_ERR_INVALID_ARG),
    (dict(D=96), _abi.FA_ERR_UNSUPPORTED),               # bf16 kernels: D in {64, 128}
    (dict(D=256, dtype=_abi.FA_F32), _abi.FA_ERR_UNSUPPORTED),
    (dict(q=None), _abi.FA_ERR_INVALID_ARG),
    (dict(lse=None), _abi.FA_ERR_INVALID_ARG),
    (dict(k=24), _abi.FA_ERR_INVALID_ARG),               # not 16-byte aligned
    (dict(cu=16, max_seqlen=-1, total=4), _abi.FA_ERR_INVALID_ARG),
    (dict(cu=16, max_seqlen=4, total=-1), _abi.FA_ERR_INVALID_ARG),
    (dict(B=70000), _abi.FA_ERR_UNSUPPORTED),
])
def test_fwd_rejects_bad_arguments_before_launch(lib, kw, code):
    assert _fwd(lib, **kw) == code


@pytest.mark.parametrize("kw", [dict(B=0), dict(N=0), dict(cu=16, B=2, max_seqlen=0, total=0)])
def test_empty_problems_are_no_ops(lib, kw):
    # Nothing to compute: returns before touching the device, even with null
    # pointers.
    assert _fwd(lib, q=None, k=None, v=None, o=None, lse=None, **kw) == _abi.FA_OK


def test_bwd_rejects_small_workspace(lib):
    need = lib.fa_bwd_workspace_size(8, 2, 64, _abi.FA_BF16)  # T = B * N = 8
    args = [256] * 9 + [1, 2, 2, 8, 64, _abi.FA_BF16, 0, 0.0, None, 0, 0, 256, need - 1, None]
    assert lib.fa_bwd(*args) == _abi.FA_ERR_INVALID_ARG
    args[-3] = 100  # workspace must be 256-byte aligned
    args[-2] = need
    assert lib.fa_bwd(*args) == _abi.FA_ERR_INVALID_ARG


def test_no_gpu_reports_cuda_error_not_crash(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _fwd(lib) == _abi.FA_ERR_CUDA
    where = ctypes.c_uint(0)
    assert lib.fa_check_device_error(None, ctypes.byref(where)) == _abi.FA_ERR_CUDA


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no non-CUDA fallback"):
        _abi.lib()
