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
    # fa_bwd (fused): D_i rows plus the fp32 dQ accumulator for bf16.
    assert lib.fa_bwd_workspace_size(T, H, D, _abi.FA_BF16) == r(T * H * 4) + r(T * H * D * 4) + 256
    assert lib.fa_bwd_workspace_size(T, H, D, _abi.FA_F32) == r(T * H * 4) + 256
    assert lib.fa_bwd_workspace_size(-1, H, D, _abi.FA_BF16) == 0
    ws = lib.fa_bwd_phases_workspace_size
    assert ws(_abi.BWD_SPLIT, T, H, D, _abi.FA_BF16) == r(T * H * 4) + 256
    assert ws(_abi.BWD_FUSED, T, H, D, _abi.FA_BF16) == lib.fa_bwd_workspace_size(T, H, D, 0)
    assert ws(_abi.BWD_DQ_CONVERT, T, H, D, _abi.FA_BF16) == r(T * H * 4) + r(T * H * D * 4) + 256
    assert ws(0, T, H, D, _abi.FA_BF16) == 0
    assert ws(0x20, T, H, D, _abi.FA_BF16) == 0


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


def test_bwd_phases_rejects_bad_masks(lib):
    need = lib.fa_bwd_workspace_size(8, 2, 64, _abi.FA_BF16)

    def call(mask, dtype=_abi.FA_BF16):
        return lib.fa_bwd_phases(mask, *([256] * 9), 1, 2, 2, 8, 64, dtype, 0, 0.0, None, 0, 0,
                                 256, need, None)
    assert call(0) == _abi.FA_ERR_INVALID_ARG
    assert call(0x20) == _abi.FA_ERR_INVALID_ARG
    # The fp32 backward is one pass: its phases cannot be enqueued one by one.
    assert call(_abi.BWD_FUSED_KERNEL, _abi.FA_F32) == _abi.FA_ERR_UNSUPPORTED
    assert call(_abi.BWD_DKDV, _abi.FA_F32) == _abi.FA_ERR_UNSUPPORTED
    # The split path needs only the D_i rows; a fused mask needs the accumulator.
    small = lib.fa_bwd_phases_workspace_size(_abi.BWD_SPLIT, 8, 2, 64, _abi.FA_BF16)
    assert small < need
    args = [*([256] * 9), 1, 2, 2, 8, 64, _abi.FA_BF16, 0, 0.0, None, 0, 0, 256, small, None]
    assert lib.fa_bwd_phases(_abi.BWD_FUSED, *args) == _abi.FA_ERR_INVALID_ARG


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


# ------------------------------------------------------------------ decode ---

def _decode(lib, **kw):
    a = dict(q=None, k=None, v=None, o=None, lse=None, lens=None, table=None, B=2, q_len=1, H=8,
             H_kv=2, D=128, page=1024, max_blocks=0, rows=2048, max_len=1000, causal=1,
             scale=-1.0, n_split=0, ws=None, ws_bytes=0)
    a.update(kw)
    return lib.fa_decode(a["q"], a["k"], a["v"], a["o"], a["lse"], a["lens"], a["table"], a["B"],
                         a["q_len"], a["H"], a["H_kv"], a["D"], a["page"], a["max_blocks"],
                         a["rows"], a["max_len"], a["causal"], a["scale"], a["n_split"], a["ws"],
                         a["ws_bytes"], None)


def test_decode_rejects_bad_shapes_before_any_launch(lib):
    assert _decode(lib, D=96) == _abi.FA_ERR_UNSUPPORTED
    assert _decode(lib, q_len=17, H=64, H_kv=8) == _abi.FA_ERR_UNSUPPORTED   # 136 rows > 128
    assert _decode(lib, H=6, H_kv=4) == _abi.FA_ERR_INVALID_ARG
    assert _decode(lib, q_len=0) == _abi.FA_ERR_INVALID_ARG
    assert _decode(lib, page=999) == _abi.FA_ERR_INVALID_ARG       # stride < max_seqlen_k
    assert _decode(lib, rows=1500) == _abi.FA_ERR_INVALID_ARG      # contiguous cache too short
    assert _decode(lib, rows=0) == _abi.FA_ERR_INVALID_ARG
    assert _decode(lib, rows=1 << 31) == _abi.FA_ERR_UNSUPPORTED
    fake = ctypes.c_void_p(16)
    assert _decode(lib, table=fake, page=48, max_blocks=64) == _abi.FA_ERR_UNSUPPORTED
    assert _decode(lib, table=fake, page=64, max_blocks=15) == _abi.FA_ERR_INVALID_ARG
    assert _decode(lib, table=fake, page=64, max_blocks=16, rows=2000) == _abi.FA_ERR_INVALID_ARG
    # null tensors with otherwise valid sizes
    assert _decode(lib) == _abi.FA_ERR_INVALID_ARG
    assert _decode(lib, B=0) == _abi.FA_OK


def test_decode_split_count_and_workspace_size(lib):
    # automatic: about 4 * 148 CTAs over B * H_kv units, clamped to the tiles
    assert lib.fa_decode_num_splits(16, 8, 32768, 0) == 5     # ceil(592 / 128) = 5 of 256 tiles
    assert lib.fa_decode_num_splits(1, 1, 1000, 0) == 8       # clamped to 8 tiles
    assert lib.fa_decode_num_splits(2, 2, 1000, 3) == 3       # chunk 3 -> 3 splits
    assert lib.fa_decode_num_splits(2, 2, 1000, 7) == 4       # chunk 2 -> 4 splits
    assert lib.fa_decode_num_splits(2, 2, 0, 0) == 1
    assert lib.fa_decode_workspace_size(2, 1, 8, 2, 128, 1000, 1) == 0
    ns = lib.fa_decode_num_splits(2, 2, 1000, 3)
    rows = ns * 2 * 1 * 8

    def r256(x):
        return (x + 255) // 256 * 256
    assert lib.fa_decode_workspace_size(2, 1, 8, 2, 128, 1000, 3) == r256(rows * 128 * 4) + \
        r256(rows * 4)


def test_balanced_decode_workspace_size(lib):
    # Automatic splits at D = 128 with q_len * g <= 64 take the balanced
    # kernel: partial rows for (B * H_kv + CTAs) slots, plus two int arrays
    # of B * H_kv. The CTAs are whole groups of H_kv; without a device the
    # library assumes 148 SMs (B200).
    def r256(x):
        return (x + 255) // 256 * 256
    for B, q_len, H, H_kv in [(16, 1, 32, 8), (16, 8, 32, 8), (3, 16, 16, 4), (2, 1, 5, 5)]:
        segs = B * H_kv
        rows = (segs + 148 // H_kv * H_kv) * q_len * (H // H_kv)
        want = r256(rows * 128 * 4) + r256(rows * 4) + 2 * r256(segs * 4)
        assert lib.fa_decode_workspace_size(B, q_len, H, H_kv, 128, 32768, 0) == want
    # more than 64 rows (16 tokens x 8 heads), or an explicit split count:
    # the split kernel's partials
    rows = lib.fa_decode_num_splits(2, 2, 1000, 0) * 2 * 16 * 16
    assert lib.fa_decode_workspace_size(2, 16, 16, 2, 128, 1000, 0) == \
        r256(rows * 128 * 4) + r256(rows * 4)
    assert lib.fa_decode_workspace_size(2, 1, 8, 2, 128, 1000, 1) == 0


# --------------------------------------------------------------------- FP8 ---

def test_fp8_entry_points_reject_bad_shapes(lib):
    assert lib.fa_fp8_quantize(None, None, None, 1, 10, 2, 12, None) == _abi.FA_ERR_UNSUPPORTED
    assert lib.fa_fp8_quantize(None, None, None, 1, 10, 2, 512, None) == _abi.FA_ERR_UNSUPPORTED
    assert lib.fa_fp8_quantize(None, None, None, 1, 10, 2, 128, None) == _abi.FA_ERR_INVALID_ARG
    assert lib.fa_fp8_quantize(None, None, None, 0, 10, 2, 128, None) == _abi.FA_OK
    f = lib.fa_fwd_fp8
    assert f(None, None, None, None, None, None, None, 1, 4, 2, 64, 64, 1, -1.0, None) == \
        _abi.FA_ERR_UNSUPPORTED   # D = 64: one 128-byte E4M3 row per token is required
    assert f(None, None, None, None, None, None, None, 1, 4, 3, 64, 128, 1, -1.0, None) == \
        _abi.FA_ERR_INVALID_ARG   # H % H_kv != 0
    assert f(None, None, None, None, None, None, None, 1, 4, 2, 64, 128, 1, -1.0, None) == \
        _abi.FA_ERR_INVALID_ARG   # null tensors
