"""Float64 CPU oracle for exact attention (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` may import this package. The product path never does.
"""
from .attention import (attention_backward, attention_forward, head_backward,
                        head_forward, lse_dense_layout, scores, softmax_rows)
from .online import compositions, online_attention, uniform_blocks

__all__ = ["attention_forward", "attention_backward", "head_forward", "head_backward",
           "scores", "softmax_rows", "lse_dense_layout", "online_attention",
           "uniform_blocks", "compositions"]
