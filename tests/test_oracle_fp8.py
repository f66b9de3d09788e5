"""Pins for the FP8 (E4M3) forward oracle (oracle/fp8.py), CPU only.

- E4M3 rounding against torch's float8_e4m3fn conversion (an independent
  implementation of the same format), on the whole grid, on random values and
  on every midpoint between neighbouring grid values (ties to even);
- pass 1: each block's largest |x| lands exactly on +-448, every dequantised
  element is within half an E4M3 step of the input, zero blocks get Delta = 1,
  and scaling a block by a power of two scales Delta only;
- pass 2: inputs already on the scaled grid quantise losslessly, so the FP8
  forward equals the plain forward on them; a planted per-tensor (instead of
  per-block) scale is caught.
"""
import numpy as np
import pytest
import torch

from exact_io_aware_tmem_b200.workloads import random_case
from oracle import attention as oa
from oracle import fp8


def _torch_e4m3(x):
    return torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def _grid():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    v = codes.to(torch.float64).numpy()
    return np.unique(v[np.isfinite(v)])


def test_grid_values_round_to_themselves_and_span_448():
    g = _grid()
    assert g.max() == 448.0 and g.min() == -448.0
    assert len(g) == 253   # 254 finite codes, +0 and -0 collapse
    np.testing.assert_array_equal(fp8.e4m3_round(g), g)


def test_rounding_matches_torch_on_random_values_and_ties():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.uniform(-0.05, 0.05, 20000),
                        rng.standard_normal(20000) * 8]).astype(np.float32)
    np.testing.assert_array_equal(fp8.e4m3_round(x), _torch_e4m3(x))
    g = _grid()
    pos = g[g >= 0]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)     # exact in float32
    np.testing.assert_array_equal(fp8.e4m3_round(mids), _torch_e4m3(mids))
    np.testing.assert_array_equal(fp8.e4m3_round(-mids), _torch_e4m3(-mids))


def test_saturation_at_448():
    assert fp8.e4m3_round(np.float32(448.00003)) == 448.0
    assert fp8.e4m3_round(np.float32(-1000.0)) == -448.0


def test_pass1_block_max_hits_448_and_error_is_half_a_step():
    inp = random_case(3, dtype="bf16", lengths=[300, 300], H=3, H_kv=3, D=64, varlen=False)
    x = inp.q.float().numpy()
    xh, d = fp8.quantize_blocks(inp.q, 2, 300)
    assert d.shape == (2, 3, 3)
    for b in range(2):
        for t in range(3):
            r0, r1 = b * 300 + t * 128, b * 300 + min(t * 128 + 128, 300)
            for h in range(3):
                assert np.abs(xh[r0:r1, h]).max() == 448.0
                q = (x[r0:r1, h] / d[b, h, t]).astype(np.float64)
                # half an E4M3 step: 2^(e-4) for |q| in [2^e, 2^(e+1)), 2^-10 in the subnormals
                e = np.floor(np.log2(np.maximum(np.abs(q), 2.0 ** -6)))
                assert np.all(np.abs(xh[r0:r1, h] - q) <= np.exp2(e - 4) + 1e-12)


def test_zero_block_and_power_of_two_scaling():
    x = torch.zeros(256, 1, 8)
    x[128:] = torch.randn(128, 1, 8)
    xh, d = fp8.quantize_blocks(x, 1, 256)
    assert d[0, 0, 0] == 1.0 and np.all(xh[:128] == 0)
    xh2, d2 = fp8.quantize_blocks(x * 8.0, 1, 256)
    np.testing.assert_array_equal(xh2, xh)
    assert d2[0, 0, 1] == np.float32(8.0) * d[0, 0, 1]


def test_grid_inputs_quantise_losslessly_so_fp8_forward_is_the_plain_forward():
    rng = np.random.default_rng(1)
    g = _grid()
    B, N, H, D = 1, 200, 2, 16
    # values on the E4M3 grid times a per-block power of two, block max exactly 448
    q = rng.choice(g, size=(B * N, H, D)) * 0.25
    k = rng.choice(g, size=(B * N, H, D)) * 0.5
    for arr in (q, k):
        for t in range(2):
            arr[t * 128, :, 0] = 448.0 * (0.25 if arr is q else 0.5)
    v = rng.standard_normal((B * N, H, D))
    o8, l8 = fp8.fp8_forward(q.astype(np.float32), k.astype(np.float32), v, B, N, True, 0.05)
    o, l = oa.attention_forward(q, k, v, np.array([0, N]), True, 0.05)
    np.testing.assert_allclose(o8, o, atol=1e-12)
    np.testing.assert_allclose(l8, l, atol=1e-12)


def test_mutation_per_tensor_scale_is_caught():
    # One block much larger than the other: a per-tensor step would not put
    # the small block's max on 448.
    x = torch.randn(256, 1, 8)
    x[128:] *= 100.0
    xh, d = fp8.quantize_blocks(x, 1, 256)
    per_tensor = float(np.abs(x.numpy()).max() / 448.0)
    bad = fp8.e4m3_round((x.numpy() / np.float32(per_tensor)).astype(np.float32))
    assert np.abs(xh[:128]).max() == 448.0
    assert np.abs(bad[:128]).max() < 448.0
