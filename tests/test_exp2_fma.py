"""The FMA-pipe exponential that the D = 64 forward and the fused backward use
for a share of their softmax exponentials (``ex2_fma`` in csrc/ex2_fma.cuh).

Pins, against the mathematics rather than against the kernels:
- its polynomial for 2^f on [-1/2, 1/2] is the minimax one: the relative
  error equioscillates (five alternating extrema of equal size) at 7.49e-5;
- the whole function, range reduction and exponent insertion included, run
  on the GPU through fa_selftest_exp2, stays within 7.5e-5 of 2^x (float64)
  on [-125, 127] and goes to about 2^-126 below.
"""
import os
import re

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
COMMON = os.path.join(HERE, "..", "exact_io_aware_tmem_b200", "csrc", "ex2_fma.cuh")
BOUND = 7.5e-5


def coefficients():
    src = open(COMMON).read()
    c = {}
    for k in range(4):
        m = re.search(rf"constexpr float EX2_C{k} = ([0-9.eE+-]+)f;", src)
        assert m, f"EX2_C{k} not found"
        c[k] = float(m.group(1))
    return c


def test_polynomial_is_the_minimax_fit():
    c = coefficients()
    f = np.linspace(-0.5, 0.5, 400_001)
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    rel = p / np.exp2(f) - 1.0
    assert np.abs(rel).max() <= BOUND
    # Equioscillation: the end points and the interior extrema alternate in
    # sign with (nearly) the same size, which fixes the minimax polynomial.
    turn = np.where(np.diff(np.sign(np.diff(rel))) != 0)[0] + 1
    ext = np.concatenate([[0], turn, [len(f) - 1]])
    vals = rel[ext]
    assert len(vals) == 5, vals
    assert np.all(np.sign(vals[1:]) == -np.sign(vals[:-1])), vals
    assert np.abs(vals).min() >= 0.99 * np.abs(vals).max(), vals


def test_entry_point_rejects_bad_arguments():
    from exact_io_aware_tmem_b200 import _abi, build
    build.build()
    lib = _abi.lib()
    assert lib.fa_selftest_exp2(None, None, -1, None) == _abi.FA_ERR_INVALID_ARG
    assert lib.fa_selftest_exp2(None, None, 4, None) == _abi.FA_ERR_INVALID_ARG
    assert lib.fa_selftest_exp2(None, None, 0, None) == _abi.FA_OK


@pytest.mark.gpu
def test_exp2_on_the_gpu_against_float64():
    import exact_io_aware_tmem_b200 as fa
    g = torch.Generator().manual_seed(11)
    x = torch.cat([torch.linspace(-125.0, 127.0, 1_000_001, dtype=torch.float64),
                   torch.arange(-125, 128, dtype=torch.float64),          # integers
                   torch.arange(-125, 127, dtype=torch.float64) + 0.5,    # rounding ties
                   -30.0 * torch.rand(200_000, generator=g, dtype=torch.float64),
                   torch.tensor([0.0, -0.0, 1e-7, -1e-7, 8.0, -8.0], dtype=torch.float64)])
    x32 = x.float()
    y = fa.selftest_exp2(x32.cuda()).cpu().double()
    ref = torch.exp2(x32.double())
    rel = (y / ref - 1.0).abs()
    assert rel.max().item() <= BOUND, (rel.max().item(), x32[rel.argmax()].item())
    low = torch.tensor([-126.0, -130.0, -1000.0, float("-inf")], dtype=torch.float32)
    yl = fa.selftest_exp2(low.cuda()).cpu().double()
    assert torch.all(yl >= 0) and torch.all(yl <= 2.0 ** -125), yl
