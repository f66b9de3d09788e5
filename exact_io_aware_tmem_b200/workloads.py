"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and lays them out. It holds none of the
attention arithmetic, so both the CUDA path and the float64 oracle can take
their inputs from it without sharing any of the method.

Recipe (the pages fix no inputs; every workload is synthetic Gaussian):

* one ``torch.Generator('cpu').manual_seed(seed)`` per workload;
* Q, K, V, dO drawn in that order as float32 N(0, 1) in the SDPA layout
  ``[B, H, N, D]`` (K and V with ``H_kv`` heads), then transposed to the
  token-major boundary layout ``[B*N, H, D]``;
* bf16 workloads cast the float32 draws to bf16 (round to nearest even);
* the causal B=2, N=8192 workload multiplies Q and K by 2.0 after the cast
  (exact in bf16) so that logits are large and the running max moves often;
* the packed variable-length workload first draws its 16 lengths with
  ``torch.randint(128, 4097, (16,))`` from the same generator, then Q, K, V, dO
  directly in ``[total, H, D]``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" or "bf16"
    B: int                # batch (number of sequences when varlen)
    H: int                # query heads
    H_kv: int             # key/value heads
    N: int                # sequence length (max_seqlen when varlen)
    D: int                # head dim
    causal: bool
    seed: int
    backward: bool        # whether the workload runs the backward pass
    qk_mult: float = 1.0  # multiplier applied to Q and K after the cast
    varlen: Optional[int] = None  # number of packed sequences (lengths drawn)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


# The five workloads, smallest first. The first is the float32 case the oracle
# finishes well under a second; the rest are the bf16 tensor-core cases.
WORKLOADS = {
    "f32_b1_h2_n128_d64": Workload("f32_b1_h2_n128_d64", "f32", 1, 2, 2, 128, 64,
                                   False, 0, True),
    "bf16_fwd_b4_h16_n2048_d64": Workload("bf16_fwd_b4_h16_n2048_d64", "bf16", 4, 16, 16,
                                          2048, 64, False, 1, False),
    "bf16_causal_b2_h16_n8192_d128": Workload("bf16_causal_b2_h16_n8192_d128", "bf16", 2, 16,
                                              16, 8192, 128, True, 2, True, qk_mult=2.0),
    "bf16_gqa_causal_b1_h32_kv8_n16384_d128": Workload(
        "bf16_gqa_causal_b1_h32_kv8_n16384_d128", "bf16", 1, 32, 8, 16384, 128, True, 3, True),
    "bf16_varlen_h16_d128_16seqs": Workload("bf16_varlen_h16_d128_16seqs", "bf16", 16, 16, 16,
                                            4096, 128, False, 4, True, varlen=16),
}
WORKLOAD_ORDER = list(WORKLOADS)


@dataclasses.dataclass
class Inputs:
    """Token-major CPU tensors plus the sequence layout."""
    q: torch.Tensor           # [T, H, D]
    k: torch.Tensor           # [T, H_kv, D]
    v: torch.Tensor           # [T, H_kv, D]
    do: torch.Tensor          # [T, H, D]
    cu_seqlens: torch.Tensor  # int32 [B+1]
    max_seqlen: int
    varlen: bool              # True when the boundary receives cu_seqlens


def _to_dtype(x: torch.Tensor, dtype: str) -> torch.Tensor:
    return x.to(torch.bfloat16) if dtype == "bf16" else x.to(torch.float32)


def make_inputs(w: Workload, *, N: Optional[int] = None, B: Optional[int] = None,
                lengths: Optional[list] = None) -> Inputs:
    """Draw the seeded inputs of workload ``w``.

    ``N``/``B`` override the dense shape (for small parity cases with the same
    recipe); ``lengths`` overrides the drawn varlen lengths.
    """
    g = torch.Generator("cpu").manual_seed(w.seed)
    if w.varlen is not None or lengths is not None:
        if lengths is None:
            lengths = torch.randint(128, 4097, (w.varlen,), generator=g).tolist()
        total = int(sum(lengths))
        shape_q = (total, w.H, w.D)
        shape_kv = (total, w.H_kv, w.D)
        q = torch.randn(shape_q, generator=g)
        k = torch.randn(shape_kv, generator=g)
        v = torch.randn(shape_kv, generator=g)
        do = torch.randn(shape_q, generator=g)
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
        max_seqlen = max(lengths) if lengths else 0
        varlen = True
    else:
        B_ = w.B if B is None else B
        N_ = w.N if N is None else N
        q = torch.randn((B_, w.H, N_, w.D), generator=g)
        k = torch.randn((B_, w.H_kv, N_, w.D), generator=g)
        v = torch.randn((B_, w.H_kv, N_, w.D), generator=g)
        do = torch.randn((B_, w.H, N_, w.D), generator=g)
        # [B, H, N, D] -> [B*N, H, D]
        q, k, v, do = (x.transpose(1, 2).reshape(B_ * N_, x.shape[1], w.D).contiguous()
                       for x in (q, k, v, do))
        cu = torch.arange(0, (B_ + 1) * N_, N_, dtype=torch.int32)
        max_seqlen = N_
        varlen = False
    q, k, v, do = (_to_dtype(x, w.dtype) for x in (q, k, v, do))
    if w.qk_mult != 1.0:
        q = q * w.qk_mult
        k = k * w.qk_mult
    return Inputs(q, k, v, do, cu, max_seqlen, varlen)


def random_case(seed: int, *, dtype: str, lengths: list, H: int, H_kv: int, D: int,
                varlen: bool, std: float = 1.0) -> Inputs:
    """Small seeded case with arbitrary (possibly ragged) lengths.

    With ``varlen=False`` all lengths must be equal and the case is dense.
    """
    g = torch.Generator("cpu").manual_seed(seed)
    total = int(sum(lengths))
    q = torch.randn((total, H, D), generator=g) * std
    k = torch.randn((total, H_kv, D), generator=g) * std
    v = torch.randn((total, H_kv, D), generator=g)
    do = torch.randn((total, H, D), generator=g)
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
    if lengths:
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    if not varlen:
        assert len(set(lengths)) <= 1, "dense cases need equal lengths"
    q, k, v, do = (_to_dtype(x, dtype) for x in (q, k, v, do))
    return Inputs(q, k, v, do, cu, max(lengths) if lengths else 0, varlen)


def flops(w_or_lengths, H: int, D: int, causal: bool) -> tuple:
    """Forward and backward FLOP counts of the method's two matmuls.

    Forward 4*H*sum(L^2)*D; backward 2.5x that; causal halves both.
    """
    lengths = w_or_lengths
    s = sum(int(L) * int(L) for L in lengths)
    fwd = 4.0 * H * s * D
    if causal:
        fwd *= 0.5
    return fwd, 2.5 * fwd


# ------------------------------------------------------------------ decode ---
#
# Decode inputs: the q_len newest tokens of B sequences against each
# sequence's key/value cache. The recipe draws, from one
# ``torch.Generator('cpu').manual_seed(seed)``: Q ``[B*q_len, H, D]``, then the
# K cache and the V cache ``[rows, H_kv, D]`` as float32 N(0, 1) (cast to the
# workload dtype), then, for a paged cache, one permutation of all block ids
# (``torch.randperm``) handed out to the sequences in order. Cache rows that no
# sequence position uses are set to ``fill`` (NaN by default) so that a kernel
# which read them would show it.


@dataclasses.dataclass
class DecodeInputs:
    q: torch.Tensor                    # [B*q_len, H, D]
    k_cache: torch.Tensor              # [rows, H_kv, D]
    v_cache: torch.Tensor              # [rows, H_kv, D]
    cache_seqlens: torch.Tensor        # int32 [B]
    block_table: Optional[torch.Tensor]  # int32 [B, max_blocks] (paged) or None
    page_size: int                     # paged: rows per page; contiguous: per-sequence stride
    q_len: int

    @property
    def paged(self) -> bool:
        return self.block_table is not None


def decode_case(seed: int, *, dtype: str, lengths: list, q_len: int, H: int, H_kv: int, D: int,
                page_size: Optional[int] = None, stride: Optional[int] = None,
                extra_blocks: int = 3, fill: float = float("nan")) -> DecodeInputs:
    """Seeded decode case; paged when ``page_size`` is given, else contiguous.

    Contiguous: sequence b owns rows [b*stride, b*stride + stride) with
    ``stride`` (default: the longest length) >= every length. Paged: sequence
    b owns ceil(len_b / page_size) pages of a shared pool that also holds
    ``extra_blocks`` unused pages; unused block-table entries are -1.
    """
    g = torch.Generator("cpu").manual_seed(seed)
    B = len(lengths)
    q = torch.randn((B * q_len, H, D), generator=g)
    if page_size is None:
        stride = max(lengths) if stride is None else stride
        assert stride >= max(lengths)
        rows = B * stride
        used = torch.zeros(rows, dtype=torch.bool)
        for b, n in enumerate(lengths):
            used[b * stride:b * stride + n] = True
        table = None
        ps = stride
    else:
        pages = [-(-n // page_size) for n in lengths]
        n_blocks = sum(pages) + extra_blocks
        rows = n_blocks * page_size
        used = torch.zeros(rows, dtype=torch.bool)
        table = torch.full((B, max(max(pages), 1)), -1, dtype=torch.int32)
        ps = page_size
    k = torch.randn((rows, H_kv, D), generator=g)
    v = torch.randn((rows, H_kv, D), generator=g)
    if table is not None:
        perm = torch.randperm(n_blocks, generator=g)
        nxt = 0
        for b, n in enumerate(lengths):
            for i in range(pages[b]):
                blk = int(perm[nxt])
                nxt += 1
                table[b, i] = blk
                m = min(page_size, n - i * page_size)
                used[blk * page_size:blk * page_size + m] = True
    q, k, v = (_to_dtype(x, dtype) for x in (q, k, v))
    k[~used] = fill
    v[~used] = fill
    return DecodeInputs(q, k, v, torch.tensor(lengths, dtype=torch.int32), table, ps, q_len)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    q_len: int
    H: int
    H_kv: int
    D: int
    len_lo: int            # cache lengths drawn uniformly from [len_lo, len_hi]
    len_hi: int
    page_size: Optional[int]
    seed: int
    causal: bool = True
    dtype: str = "bf16"

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def lengths(self) -> list:
        g = torch.Generator("cpu").manual_seed(self.seed + 1000)
        return torch.randint(self.len_lo, self.len_hi + 1, (self.B,), generator=g).tolist()


# Decode workloads (no configuration on the pages or in the task fixes these;
# they are sized so the caches are far larger than L2): GQA 32/8 heads, D=128,
# 16 sequences with cache lengths in [4096, 32768]; one new token per sequence,
# or 8 (a speculative-decoding verify step), over a contiguous or a paged cache.
DECODE_WORKLOADS = {
    "bf16_decode_b16_h32_kv8_d128_q1": DecodeWorkload(
        "bf16_decode_b16_h32_kv8_d128_q1", 16, 1, 32, 8, 128, 4096, 32768, None, 11),
    "bf16_decode_paged64_b16_h32_kv8_d128_q1": DecodeWorkload(
        "bf16_decode_paged64_b16_h32_kv8_d128_q1", 16, 1, 32, 8, 128, 4096, 32768, 64, 12),
    "bf16_decode_b16_h32_kv8_d128_q8": DecodeWorkload(
        "bf16_decode_b16_h32_kv8_d128_q8", 16, 8, 32, 8, 128, 4096, 32768, None, 13),
}


def make_decode_inputs(w: DecodeWorkload) -> DecodeInputs:
    return decode_case(w.seed, dtype=w.dtype, lengths=w.lengths(), q_len=w.q_len, H=w.H,
                       H_kv=w.H_kv, D=w.D, page_size=w.page_size)


def decode_bytes(lengths, H_kv: int, D: int, elem: int = 2) -> float:
    """K and V cache bytes a decode step must read: 2 * sum(len) * H_kv * D * elem."""
    return 2.0 * sum(int(n) for n in lengths) * H_kv * D * elem


def decode_flops(lengths, q_len: int, H: int, D: int) -> float:
    """4 * q_len * H * D * sum(len): the two products over every cached key."""
    return 4.0 * q_len * H * D * sum(int(n) for n in lengths)
