"""Float64 CPU oracle of the FP8 (E4M3) forward: block scales, E4M3 rounding,
attention on the dequantised Q and K.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import or call this module.
The product path never routes through it and shares no code with it.

What it computes (aiqz.cc "Flash Attention V2/V3 optimization" article,
section "FP8 low precision"):

* E4M3 (largest finite value 448) is the forward's format;
* pass 1 scans each block for max |x| and sets its step Delta = max|x| / 448;
  each element becomes round(x / Delta), an E4M3 value;
* pass 2 multiplies the quantised Q and K on the tensor cores with an fp32
  accumulator.

The oracle is the plain definition of that result: attention (oracle.attention)
on Q_hat * Delta_Q and K_hat * Delta_K, the dequantised inputs, in float64.
V is not quantised (the article quantises only Q and K for the matmul).

Readings where the article is silent (each listed in the design notes):

* a block is the 128 consecutive tokens of one head of one sequence that one
  CTA's tile holds (the last block of a sequence may be shorter);
* max|x| is taken over the bf16 inputs; Delta = max|x| / 448 and x / Delta are
  single-precision IEEE divisions, the precision the GPU takes these
  decisions in, so both sides pick the same E4M3 code; a block of zeros gets
  Delta = 1 (all its codes are 0);
* "round" is round-to-nearest-even onto the E4M3 grid (subnormals included,
  step 2^-9 below 2^-6), saturating at +-448.
"""
from __future__ import annotations

import numpy as np

from .attention import attention_forward

E4M3_MAX = 448.0
BLOCK = 128


def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3 value (ties to even), saturating at +-448; float64 out.

    E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; normal
    values 2^(e-7) * (1 + m/8) for e = 1..15 (e = 15, m = 7 is NaN), so the
    largest is 448; subnormals m/8 * 2^-6, step 2^-9.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6, 8)                     # below 2^-6: the subnormal step
    step = np.exp2(e - 3)
    r = np.rint(a / step) * step              # np.rint rounds half to even
    r = np.minimum(r, E4M3_MAX)
    return np.where(np.isnan(x), np.nan, np.copysign(r, x))


def quantize_blocks(x, B: int, N: int):
    """Pass 1 for a token-major tensor [B*N, Hx, D] (bf16 or float32).

    Returns (x_hat, delta): the E4M3 values round(x / Delta) (float64, same
    shape) and the float32 steps Delta [B, Hx, ceil(N / 128)].
    """
    if hasattr(x, "detach"):
        import torch  # local: the oracle itself needs numpy only
        x = x.detach().to("cpu", torch.float32).numpy()
    x = np.asarray(x, dtype=np.float32)
    Hx = x.shape[1]
    nt = -(-N // BLOCK)
    delta = np.ones((B, Hx, nt), dtype=np.float32)
    x_hat = np.zeros(x.shape, dtype=np.float64)
    for b in range(B):
        for t in range(nt):
            r0, r1 = b * N + t * BLOCK, b * N + min((t + 1) * BLOCK, N)
            blk = x[r0:r1]                                   # [rows, Hx, D]
            amax = np.abs(blk).max(axis=(0, 2)).astype(np.float32)
            d = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
            delta[b, :, t] = d
            q = (blk / d[None, :, None]).astype(np.float32)  # single-precision division
            x_hat[r0:r1] = e4m3_round(q)
    return x_hat, delta


def dequantize(x_hat, delta, B: int, N: int) -> np.ndarray:
    """x_hat * Delta of its block, float64."""
    out = np.array(x_hat, dtype=np.float64)
    for b in range(B):
        for t in range(delta.shape[2]):
            r0, r1 = b * N + t * BLOCK, b * N + min((t + 1) * BLOCK, N)
            out[r0:r1] *= delta[b, :, t].astype(np.float64)[None, :, None]
    return out


def fp8_forward(q, k, v, B: int, N: int, causal: bool, scale: float):
    """O [B*N, H, D] and LSE [H, B*N] of attention on the dequantised Q, K."""
    qh, dq = quantize_blocks(q, B, N)
    kh, dk = quantize_blocks(k, B, N)
    cu = np.arange(0, (B + 1) * N, N)
    return attention_forward(dequantize(qh, dq, B, N), dequantize(kh, dk, B, N), v, cu,
                             causal, scale)
