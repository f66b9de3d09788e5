"""Python entry points over the C ABI (argument marshalling only).

Every step of the forward and backward passes runs in the CUDA kernels of
libfa_b200.so; this module checks torch tensors, allocates the outputs with
torch (device memory and streams are all PyTorch provides), and passes raw
pointers and the current stream to ``fa_fwd`` / ``fa_bwd``.

Layouts (token-major, as in include/fa.h):
  dense : q [B, N, H, D], k / v [B, N, H_kv, D]; lse [B, H, N]
  packed: q [T, H, D],    k / v [T, H_kv, D] with cu_seqlens int32 [B+1]
          on the device; lse [H, T]
"""
from __future__ import annotations

import contextlib
import math
from typing import Optional

import torch

from . import _abi

# The library the entry points call: libfa_b200.so, or, inside debug_build(),
# the same kernels built with index checks and event stamps.
_lib = _abi.lib


@contextlib.contextmanager
def debug_build():
    """Route the entry points through libfa_b200_debug.so (include/fa.h,
    "Debug build") for the duration of the block."""
    global _lib
    prev = _lib
    _lib = _abi.debug_lib
    try:
        yield _abi.debug_lib()
    finally:
        _lib = prev

_DTYPES = {torch.bfloat16: _abi.FA_BF16, torch.float32: _abi.FA_F32}


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _shape(q: torch.Tensor, k: torch.Tensor, cu_seqlens, max_seqlen):
    if q.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {q.dtype}; use bfloat16 or float32")
    for t in (q, k):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    if cu_seqlens is None:
        if q.dim() != 4 or k.dim() != 4:
            raise ValueError("dense inputs are [B, N, H, D]")
        B, N, H, D = q.shape
        H_kv = k.shape[2]
        return B, N, H, H_kv, D, 0, B * N
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("packed inputs are [T, H, D]")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda:
        raise ValueError("cu_seqlens must be an int32 CUDA tensor")
    T, H, D = q.shape
    if max_seqlen is None:
        raise ValueError("packed inputs need max_seqlen")
    return cu_seqlens.numel() - 1, 0, H, k.shape[1], D, int(max_seqlen), T


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool = False,
        scale: Optional[float] = None, cu_seqlens: Optional[torch.Tensor] = None,
        max_seqlen: Optional[int] = None, out: Optional[torch.Tensor] = None,
        lse: Optional[torch.Tensor] = None):
    """Attention forward. Returns (O, LSE)."""
    B, N, H, H_kv, D, max_sl, T = _shape(q, k, cu_seqlens, max_seqlen)
    if v.shape != k.shape or v.dtype != q.dtype or k.dtype != q.dtype:
        raise ValueError("k and v must match in shape and dtype with q's dtype")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N) if cu_seqlens is None else (H, T), device=q.device,
                          dtype=torch.float32)
    s = -1.0 if scale is None else float(scale)
    st = _lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, H_kv, N, D,
                           _DTYPES[q.dtype], int(bool(causal)), s, _ptr(cu_seqlens), max_sl, T,
                           _stream(q.device))
    _abi.check(st, "fa_fwd")
    return out, lse


BWD_FUSED = _abi.BWD_FUSED
BWD_SPLIT = _abi.BWD_SPLIT


def workspace_size(T: int, H: int, D: int, dtype: torch.dtype, phases: int = BWD_FUSED) -> int:
    """Bytes of backward workspace for ``phases`` (fa_bwd_phases_workspace_size)."""
    return int(_lib().fa_bwd_phases_workspace_size(int(phases), T, H, D, _DTYPES[dtype]))


def bwd(dout: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
        o: torch.Tensor, lse: torch.Tensor, *, causal: bool = False,
        scale: Optional[float] = None, cu_seqlens: Optional[torch.Tensor] = None,
        max_seqlen: Optional[int] = None, workspace: Optional[torch.Tensor] = None,
        dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
        dv: Optional[torch.Tensor] = None, phases: int = BWD_FUSED):
    """Attention backward for the loss sum(O * dO). Returns (dQ, dK, dV).

    ``phases`` selects the kernels to enqueue (the FA_BWD_PHASE_* bits of
    include/fa.h): the default ``BWD_FUSED`` runs the preprocess, the fused
    kernel and the dQ conversion; ``BWD_SPLIT`` runs the preprocess, the
    dK / dV kernel and the dQ kernel (bitwise reproducible dQ, smaller
    workspace); single bits enqueue one kernel, to time it.
    """
    B, N, H, H_kv, D, max_sl, T = _shape(q, k, cu_seqlens, max_seqlen)
    for t in (dout, o, v, lse):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = workspace_size(T, H, D, q.dtype, phases)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    s = -1.0 if scale is None else float(scale)
    st = _lib().fa_bwd_phases(int(phases), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                  _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), B, H, H_kv, N, D,
                                  _DTYPES[q.dtype], int(bool(causal)), s, _ptr(cu_seqlens),
                                  max_sl, T, _ptr(workspace),
                                  workspace.numel() * workspace.element_size(),
                                  _stream(q.device))
    _abi.check(st, "fa_bwd")
    return dq, dk, dv


def decode_num_splits(B: int, H_kv: int, max_seqlen_k: int, n_split: int = 0) -> int:
    return int(_lib().fa_decode_num_splits(B, H_kv, max_seqlen_k, n_split))


def decode_balanced(D: int, q_len: int, H: int, H_kv: int, n_split: int = 0) -> bool:
    """Whether fa_decode takes its balanced kernel for this shape: automatic
    splits, D = 128 and at most 64 query rows (q_len x H / H_kv) per kv head
    (include/fa.h, fa_decode)."""
    return n_split == 0 and D == 128 and H % H_kv == 0 and q_len * (H // H_kv) <= 64


def decode_workspace_size(B: int, q_len: int, H: int, H_kv: int, D: int, max_seqlen_k: int,
                          n_split: int = 0) -> int:
    return int(_lib().fa_decode_workspace_size(B, q_len, H, H_kv, D, max_seqlen_k, n_split))


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
           cache_seqlens: torch.Tensor, *, q_len: int, max_seqlen_k: int,
           block_table: Optional[torch.Tensor] = None, page_size: Optional[int] = None,
           causal: bool = True, scale: Optional[float] = None, n_split: int = 0,
           out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None):
    """Split-KV decode (fa_decode): O [B*q_len, H, D] bf16 and LSE [B*q_len, H].

    ``q`` is [B*q_len, H, D]; the caches are [rows, H_kv, D]. Contiguous
    cache: ``page_size`` is the rows per sequence (default: rows // B).
    Paged cache: ``block_table`` [B, max_blocks] int32 and ``page_size``.
    """
    B = cache_seqlens.numel()
    H, D = q.shape[1], q.shape[2]
    H_kv = k_cache.shape[1]
    rows = k_cache.shape[0]
    if block_table is None and page_size is None:
        page_size = rows // max(B, 1)
    max_blocks = block_table.shape[1] if block_table is not None else 0
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((q.shape[0], H), device=q.device, dtype=torch.float32)
    need = decode_workspace_size(B, q_len, H, H_kv, D, max_seqlen_k, n_split)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    st = _lib().fa_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse), _ptr(cache_seqlens),
        _ptr(block_table), B, int(q_len), H, H_kv, D, int(page_size), int(max_blocks), rows,
        int(max_seqlen_k), int(causal), -1.0 if scale is None else float(scale), int(n_split),
        _ptr(workspace) if need else None, need, _stream(q.device))
    _abi.check(st, "fa_decode")
    return out, lse


def fp8_quantize(x: torch.Tensor, B: int, N: int, *, out: Optional[torch.Tensor] = None,
                 scale: Optional[torch.Tensor] = None):
    """Pass 1 of the FP8 forward: E4M3 codes (uint8, x's shape) and per-block
    steps fp32 [B, Hx, ceil(N / 128)] of a bf16 [B*N, Hx, D] (or [B, N, Hx, D]) tensor."""
    Hx, D = x.shape[-2], x.shape[-1]
    x8 = torch.empty(x.shape, dtype=torch.uint8, device=x.device) if out is None else out
    sc = torch.empty((B, Hx, (N + 127) // 128), dtype=torch.float32, device=x.device) \
        if scale is None else scale
    st = _lib().fa_fp8_quantize(_ptr(x), _ptr(x8), _ptr(sc), B, N, Hx, D, _stream(x.device))
    _abi.check(st, "fa_fp8_quantize")
    return x8, sc


def fwd_fp8(q8: torch.Tensor, k8: torch.Tensor, v: torch.Tensor, q_scale: torch.Tensor,
            k_scale: torch.Tensor, *, B: int, N: int, causal: bool = False,
            scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
            lse: Optional[torch.Tensor] = None):
    """Pass 2 of the FP8 forward (fa_fwd_fp8). Returns (O bf16, LSE [B, H, N])."""
    H, D = q8.shape[-2], q8.shape[-1]
    H_kv = k8.shape[-2]
    if out is None:
        out = torch.empty(q8.shape, dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    st = _lib().fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v), _ptr(q_scale), _ptr(k_scale),
                               _ptr(out), _ptr(lse), B, H, H_kv, N, D, int(bool(causal)),
                               -1.0 if scale is None else float(scale), _stream(q8.device))
    _abi.check(st, "fa_fwd_fp8")
    return out, lse


def check_device_error(device: Optional[torch.device] = None) -> tuple:
    """Synchronise the current stream; return (status, where) and clear the flag."""
    import ctypes
    dev = torch.device("cuda") if device is None else device
    where = ctypes.c_uint(0)
    st = _lib().fa_check_device_error(_stream(dev), ctypes.byref(where))
    return st, where.value


def selftest_wait_timeout(cycles: int, device: Optional[torch.device] = None) -> None:
    dev = torch.device("cuda") if device is None else device
    _abi.check(_lib().fa_selftest_wait_timeout(int(cycles), _stream(dev)),
               "fa_selftest_wait_timeout")


def selftest_exp2(x: torch.Tensor) -> torch.Tensor:
    """2^x by the kernels' FMA-pipe exponential (fa_selftest_exp2), for a
    contiguous fp32 CUDA tensor."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("selftest_exp2 takes a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    _abi.check(_lib().fa_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream(x.device)),
               "fa_selftest_exp2")
    return y


def set_wait_budget(cycles: int) -> None:
    _lib().fa_set_wait_budget(int(cycles))


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
