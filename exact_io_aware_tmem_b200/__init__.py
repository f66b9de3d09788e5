"""Exact IO-aware attention for B200 (sm_100a): tcgen05 / TMEM / TMA kernels.

``fwd``, ``bwd`` and ``decode`` call the C ABI of libfa_b200.so (see include/fa.h).
"""
from .attention import (BWD_FUSED, BWD_SPLIT, bwd, check_device_error, decode, decode_balanced,
                        decode_num_splits, decode_workspace_size, default_scale, fp8_quantize, fwd, fwd_fp8,
                        selftest_exp2, selftest_wait_timeout, set_wait_budget, workspace_size)

__all__ = ["fwd", "bwd", "workspace_size", "BWD_FUSED", "BWD_SPLIT", "decode", "decode_balanced",
           "decode_num_splits", "decode_workspace_size",
           "fp8_quantize", "fwd_fp8",
           "check_device_error", "selftest_exp2", "selftest_wait_timeout", "set_wait_budget",
           "default_scale"]
