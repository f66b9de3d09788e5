"""Plain float64 CPU attention: the oracle for the CUDA path.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import or call this module.
The product path (the C-ABI library and its Python binding) never routes
through it and shares no code with it.

What it computes is the plain definition of exact scaled dot-product
attention; the method under test reaches the same result, up to rounding,
by tiling and the online-softmax recurrence:

* aiqz.cc "Flash Attention V2/V3 optimization" article, section "IO bottleneck
  analysis": Attn(Q, K, V) = softmax(Q K^T / sqrt(d)) V;
* same article, section "Python demo": the scale multiplies S before the row
  max is taken;
* airsota.com interview card (p=1562), section 3 (mathematical principles):
  safe softmax subtracts the row max before exponentiating; section 4 item 1:
  the result is unchanged by that shift, which is why the method is exact;
* agentalpha.top "flash attention" answer, section 2 (recomputation) and the
  airsota card section 4 item 2: the backward pass rebuilds S and P from the
  saved statistics. The pages only ask for the gradient relations (Flash
  Attention self-test, book.bogosort.top, section D); the ones below are the
  textbook derivation for the loss L = sum(O * dO):
      dV = P^T dO,   dP = dO V^T,   D_i = sum_j P_ij dP_ij = dO_i . O_i,
      dS = P * (dP - D),   dQ = scale * dS K,   dK = scale * dS^T Q.

Readings where the pages are silent (each is listed with its reason in the
design notes of the repository):

* the log-sum-exp saved for the backward pass is LSE_i = m_i + ln(l_i) in
  natural-log units of the *scaled* logits;
* causal masking keeps key j for query i iff j <= i, with i and j counted
  from the start of their own sequence;
* packed variable-length batches share one ``cu_seqlens`` prefix-sum array
  between queries and keys; attention never crosses a sequence boundary;
* grouped-query attention maps query head h to key/value head
  h // (H / H_kv) (contiguous groups);
* a row with no visible key (cannot happen with the masks above unless a
  caller passes an empty sequence) has O = 0, LSE = -inf and zero gradients.

There is no blocking over keys here: every query row sees all of its keys at
once. Rows are processed in chunks only to bound memory.
"""
from __future__ import annotations

import numpy as np

ROW_CHUNK = 1024


def _f64(x) -> np.ndarray:
    """Upcast a numpy array or a CPU torch tensor (any float dtype) to float64."""
    if hasattr(x, "detach"):  # torch tensor, possibly bf16
        x = x.detach().to("cpu")
        import torch  # local: the oracle itself needs numpy only
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def scores(q: np.ndarray, k: np.ndarray, scale: float, causal: bool,
           rows: np.ndarray | None = None) -> np.ndarray:
    """S = scale * Q K^T for one (sequence, head); -inf where causally hidden.

    ``q`` is [n, D], ``k`` is [n_k, D]; ``rows`` are the query positions of the
    rows of ``q`` (default 0..n-1), used by the causal mask.
    """
    s = scale * (q @ k.T)
    if causal:
        if rows is None:
            rows = np.arange(q.shape[0])
        cols = np.arange(k.shape[0])
        s = np.where(cols[None, :] > np.asarray(rows)[:, None], -np.inf, s)
    return s


def softmax_rows(s: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Safe row softmax and the row log-sum-exp.

    P_ij = exp(S_ij - m_i) / sum_j exp(S_ij - m_i) with m_i = max_j S_ij, and
    LSE_i = m_i + ln sum_j exp(S_ij - m_i). Rows whose entries are all -inf
    give P = 0 and LSE = -inf.
    """
    m = s.max(axis=1) if s.shape[1] else np.full(s.shape[0], -np.inf)
    has_key = np.isfinite(m)
    m_safe = np.where(has_key, m, 0.0)
    e = np.exp(s - m_safe[:, None]) if s.shape[1] else np.zeros_like(s)
    l = e.sum(axis=1)
    p = np.where(has_key[:, None], e / np.where(has_key, l, 1.0)[:, None], 0.0)
    lse = np.where(has_key, m_safe + np.log(np.where(has_key, l, 1.0)), -np.inf)
    return p, lse


def head_forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                 causal: bool, rows: np.ndarray | None = None):
    """O and LSE of one (sequence, head). ``rows`` selects query rows."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    if rows is None:
        rows = np.arange(q.shape[0])
    rows = np.asarray(rows, dtype=np.int64)
    o = np.zeros((rows.size, v.shape[1]))
    lse = np.zeros(rows.size)
    for c0 in range(0, rows.size, ROW_CHUNK):
        r = rows[c0:c0 + ROW_CHUNK]
        p, lse[c0:c0 + r.size] = softmax_rows(scores(q[r], k, scale, causal, r))
        o[c0:c0 + r.size] = p @ v
    return o, lse


def head_backward(q, k, v, do, scale: float, causal: bool,
                  q_rows: np.ndarray | None = None, want_kv: bool = True):
    """dQ (for ``q_rows``), dK and dV of one (sequence, head).

    dK/dV need every query row; when ``want_kv`` is False only dQ rows are
    formed, which costs O(len(q_rows) * n * D).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(do)
    n = q.shape[0]
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    rows_all = np.arange(n) if want_kv else np.asarray(q_rows, dtype=np.int64)
    want_q = np.arange(n) if q_rows is None else np.asarray(q_rows, dtype=np.int64)
    dq_full = {}
    for c0 in range(0, rows_all.size, ROW_CHUNK):
        r = rows_all[c0:c0 + ROW_CHUNK]
        p, _ = softmax_rows(scores(q[r], k, scale, causal, r))
        o = p @ v
        dp = do[r] @ v.T
        delta = (do[r] * o).sum(axis=1)           # D_i = dO_i . O_i
        ds = p * (dp - delta[:, None])
        if want_kv:
            dv += p.T @ do[r]
            dk += scale * (ds.T @ q[r])
        dq = scale * (ds @ k)
        for i, row in enumerate(r):
            dq_full[int(row)] = dq[i]
    dq_out = np.stack([dq_full[int(i)] for i in want_q]) if want_q.size else \
        np.zeros((0, q.shape[1]))
    return dq_out, (dk if want_kv else None), (dv if want_kv else None)


def _sequences(cu_seqlens):
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    return [(cu[i], cu[i + 1]) for i in range(len(cu) - 1)]


def attention_forward(q, k, v, cu_seqlens, causal: bool, scale: float):
    """Token-major forward over a packed batch.

    q: [T, H, D]; k, v: [T, H_kv, D]; cu_seqlens: B+1 prefix sums.
    Returns O [T, H, D] and LSE [H, T] (float64).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    T, H, D = q.shape
    H_kv = k.shape[1]
    g = H // H_kv
    o = np.zeros((T, H, v.shape[2]))
    lse = np.full((H, T), -np.inf)
    for s0, s1 in _sequences(cu_seqlens):
        if s1 == s0:
            continue
        for h in range(H):
            hk = h // g
            o[s0:s1, h], lse[h, s0:s1] = head_forward(q[s0:s1, h], k[s0:s1, hk],
                                                      v[s0:s1, hk], scale, causal)
    return o, lse


def attention_backward(q, k, v, do, cu_seqlens, causal: bool, scale: float):
    """Token-major backward for the loss sum(O * dO) over a packed batch.

    Returns dQ [T, H, D], dK [T, H_kv, D], dV [T, H_kv, D] (float64). For
    grouped-query attention dK and dV of a key/value head are the sums over
    the query heads that share it.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(do)
    T, H, D = q.shape
    H_kv = k.shape[1]
    g = H // H_kv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for s0, s1 in _sequences(cu_seqlens):
        if s1 == s0:
            continue
        for h in range(H):
            hk = h // g
            dq_h, dk_h, dv_h = head_backward(q[s0:s1, h], k[s0:s1, hk], v[s0:s1, hk],
                                             do[s0:s1, h], scale, causal)
            dq[s0:s1, h] = dq_h
            dk[s0:s1, hk] += dk_h
            dv[s0:s1, hk] += dv_h
    return dq, dk, dv


def lse_dense_layout(lse_ht: np.ndarray, B: int, N: int) -> np.ndarray:
    """[H, B*N] -> [B, H, N], the layout the library uses for dense batches."""
    H = lse_ht.shape[0]
    return lse_ht.reshape(H, B, N).transpose(1, 0, 2)
