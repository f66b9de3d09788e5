"""Helpers shared by the tests: device transfer, oracle runs, error metrics."""
from __future__ import annotations

import numpy as np
import torch

from oracle import attention as oa


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def max_abs(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.size == 0:
        return 0.0
    return float(np.abs(a - b).max())


def o_excess_bf16(got, ref, tol: float = 1.5e-2) -> float:
    """Largest amount by which |got - ref| exceeds the bf16 output bound.

    The bound is tol on the computed value plus the bf16 cast of the output,
    which moves it by at most half an ulp, 2^-9 |ref|. Returns <= 0 when every
    element is inside the bound.
    """
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if got.size == 0:
        return -tol
    return float((np.abs(got - ref) - (tol + np.abs(ref) * 2.0 ** -9)).max())


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def to_api(inp, B: int, N: int, device="cuda"):
    """Inputs (token-major CPU tensors) -> device tensors in the API layout."""
    def dev(t):
        t = t.to(device)
        if not inp.varlen:
            t = t.view(B, N, t.shape[1], t.shape[2])
        return t.contiguous()
    out = dict(q=dev(inp.q), k=dev(inp.k), v=dev(inp.v), do=dev(inp.do))
    if inp.varlen:
        out["cu_seqlens"] = inp.cu_seqlens.to(device)
        out["max_seqlen"] = inp.max_seqlen
    return out


def oracle_lse_layout(lse_ht: np.ndarray, inp, B: int, N: int) -> np.ndarray:
    return lse_ht if inp.varlen else oa.lse_dense_layout(lse_ht, B, N)


def sample_forward(inp, causal: bool, scale: float, picks):
    """Oracle O / LSE rows for a list of (seq, head, rows) picks."""
    cu = inp.cu_seqlens.tolist()
    H, H_kv = inp.q.shape[1], inp.k.shape[1]
    g = H // H_kv
    res = []
    for b, h, rows in picks:
        s0, s1 = cu[b], cu[b + 1]
        o, lse = oa.head_forward(inp.q[s0:s1, h], inp.k[s0:s1, h // g], inp.v[s0:s1, h // g],
                                 scale, causal, rows=np.asarray(rows))
        res.append((b, h, np.asarray(rows), o, lse))
    return res
