"""GPU parity of the FP8 (E4M3) forward against the float64 oracle (oracle/fp8.py).

Pass 1 (fa_fp8_quantize) takes integer decisions - which E4M3 code each
element gets - in single precision on both sides, so its codes and steps must
match the oracle's exactly. Pass 2 (fa_fwd_fp8) is checked against attention on
the dequantised inputs with the forward's bf16 bounds: |O - O_ref| <= 1.5e-2 +
2^-9 |O_ref| and max-abs 1e-3 on LSE.
"""
import numpy as np
import pytest
import torch

import exact_io_aware_tmem_b200 as fa
from exact_io_aware_tmem_b200.workloads import WORKLOADS, make_inputs, random_case
from oracle import attention as oa
from oracle import fp8 as of
from tests._util import f64, max_abs, o_excess_bf16

pytestmark = pytest.mark.gpu

O_TOL = 1.5e-2
LSE_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    from exact_io_aware_tmem_b200 import build
    build.build()


def _codes_as_values(x8: torch.Tensor) -> np.ndarray:
    return x8.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


# The last two cases are a few thousand blocks (several waves of CTAs).
@pytest.mark.parametrize("B,N,Hx,D", [(2, 300, 3, 128), (1, 128, 2, 64), (3, 1, 1, 128),
                                      (1, 1000, 4, 8), (1, 4096, 64, 128), (2, 2000, 64, 64)])
def test_quantize_codes_and_steps_are_exact(B, N, Hx, D):
    inp = random_case(7 + N, dtype="bf16", lengths=[N] * B, H=Hx, H_kv=Hx, D=D, varlen=False,
                      std=3.0)
    x = inp.q
    x[: min(N, 128)] = 0.0          # an all-zero first block (Delta = 1)
    x8, sc = fa.fp8_quantize(x.cuda(), B, N)
    torch.cuda.synchronize()
    xh, d = of.quantize_blocks(x, B, N)
    np.testing.assert_array_equal(sc.cpu().numpy(), d)
    np.testing.assert_array_equal(_codes_as_values(x8), xh)


def _hard_blocks(seed: int, n_blocks: int, D: int) -> torch.Tensor:
    """n_blocks blocks of 128 tokens x D (one head), each with its own max |x|
    and elements drawn uniformly over bf16 bit patterns below it (every
    exponent down to the subnormals), so x / Delta lands everywhere on the
    E4M3 grid, at its rounding midpoints and in its subnormal range. Block 0
    holds the midpoints of the grid and their bf16 neighbours with Delta = 1
    (max |x| = 448); block 1 has a max |x| whose Delta is an fp32 subnormal,
    block 2 a max |x| that is itself a bf16 subnormal."""
    g = torch.Generator().manual_seed(seed)
    per = 128 * D
    amax_bits = torch.randint(0x3000, 0x4700, (n_blocks,), generator=g, dtype=torch.int32)
    amax_bits[1] = 0x0100                                      # 2^-125: Delta an fp32 subnormal
    amax_bits[2] = 0x0045                                      # a bf16 subnormal max |x|
    amax = (amax_bits << 16).view(torch.float32)
    bits = torch.randint(0, 1 << 30, (n_blocks, per), generator=g, dtype=torch.int32)
    bits = bits % (amax_bits[:, None] + 1)                     # bf16 patterns in [0, max |x|]
    x = (bits << 16).view(torch.float32)
    # grid midpoints of E4M3 (normal and subnormal) and their bf16 neighbours
    grid = torch.arange(0, 127, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    grid = grid.to(torch.float32)
    mid = (grid[:-1] + grid[1:]) / 2
    nb = torch.cat([mid, torch.nextafter(mid.bfloat16().float(), torch.tensor(0.0)),
                    torch.nextafter(mid.bfloat16().float(), torch.tensor(1e9))]).bfloat16().float()
    x[0, : nb.numel()] = nb
    amax[0] = 448.0
    x[:, -1] = amax                                            # the block's max
    sign = torch.randint(0, 2, x.shape, generator=g).float() * 2 - 1
    return (x * sign).bfloat16()


def test_quantize_codes_exact_on_every_exponent_and_midpoint():
    D, n_blocks = 128, 24
    x = _hard_blocks(5, n_blocks, D).view(n_blocks * 128, 1, D)
    x8, sc = fa.fp8_quantize(x.cuda(), 1, n_blocks * 128)
    torch.cuda.synchronize()
    xh, d = of.quantize_blocks(x, 1, n_blocks * 128)
    np.testing.assert_array_equal(sc.cpu().numpy(), d)
    np.testing.assert_array_equal(_codes_as_values(x8), xh)


def _fp8_case(inp, B, N, causal, scale):
    q8, qs = fa.fp8_quantize(inp.q.cuda(), B, N)
    k8, ks = fa.fp8_quantize(inp.k.cuda(), B, N)
    o, lse = fa.fwd_fp8(q8, k8, inp.v.cuda(), qs, ks, B=B, N=N, causal=causal, scale=scale)
    st, where = fa.check_device_error()
    assert st == 0, f"device error {st} at {where:#x}"
    return f64(o), f64(lse)


def _check(o, lse, o_ref, lse_ref):
    assert np.isfinite(o).all()
    excess = o_excess_bf16(o, o_ref, O_TOL)
    assert excess <= 0, f"O outside the bf16 bound by {excess} (max-abs {max_abs(o, o_ref)})"
    err = max_abs(lse, lse_ref)
    assert err <= LSE_TOL, f"LSE max-abs {err}"


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,H,H_kv", [(2, 300, 4, 2), (1, 129, 2, 1), (1, 1024, 8, 8)])
def test_fp8_forward_small(B, N, H, H_kv, causal):
    inp = random_case(11 + N, dtype="bf16", lengths=[N] * B, H=H, H_kv=H_kv, D=128, varlen=False,
                      std=2.0)
    scale = 128 ** -0.5
    o, lse = _fp8_case(inp, B, N, causal, scale)
    o_ref, lse_ref = of.fp8_forward(inp.q, inp.k, inp.v, B, N, causal, scale)
    _check(o.reshape(B * N, H, 128), lse, o_ref, oa.lse_dense_layout(lse_ref, B, N))


@pytest.mark.slow
def test_fp8_forward_full_workload_sampled():
    # The causal B2 H16 N8192 D128 inputs (Q, K x 2.0) through both passes; the
    # oracle dequantises Q and K in full and forms sampled rows.
    w = WORKLOADS["bf16_causal_b2_h16_n8192_d128"]
    inp = make_inputs(w)
    B, N, H = w.B, w.N, w.H
    o, lse = _fp8_case(inp, B, N, True, w.scale)
    o = o.reshape(B * N, H, w.D)
    qh, dq = of.quantize_blocks(inp.q, B, N)
    kh, dk = of.quantize_blocks(inp.k, B, N)
    qd, kd = of.dequantize(qh, dq, B, N), of.dequantize(kh, dk, B, N)
    v = inp.v.double().numpy()
    rows = np.array([0, 1, 127, 128, 4095, 5000, 8190, 8191])
    for b in range(B):
        for h in (0, 7, 15):
            sl = slice(b * N, (b + 1) * N)
            o_ref, lse_ref = oa.head_forward(qd[sl, h], kd[sl, h], v[sl, h], w.scale, True, rows)
            _check(o[b * N + rows, h], lse[b, h, rows], o_ref, lse_ref)
