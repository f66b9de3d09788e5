"""Bounded in-kernel waits: a wait that nothing satisfies gives up and reports.

The self-test kernel waits on an mbarrier no thread arrives on, with a budget
of a few million cycles; the error comes back through fa_check_device_error
and the context stays usable for the next launch.
"""
import pytest
import torch

import exact_io_aware_tmem_b200 as fa
from exact_io_aware_tmem_b200 import _abi

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from exact_io_aware_tmem_b200 import build
    build.build()


def test_wait_gives_up_and_reports():
    fa.check_device_error()  # clear any earlier state
    fa.selftest_wait_timeout(5_000_000)  # a few milliseconds
    st, where = fa.check_device_error()
    assert st == _abi.FA_ERR_DEVICE_TIMEOUT
    assert where == 0x5E1F7E57
    # cleared after being reported
    assert fa.check_device_error()[0] == _abi.FA_OK


def test_context_usable_after_timeout():
    fa.selftest_wait_timeout(1_000_000)
    assert fa.check_device_error()[0] == _abi.FA_ERR_DEVICE_TIMEOUT
    q = torch.randn(1, 130, 2, 64, device="cuda", dtype=torch.bfloat16)
    o, lse = fa.fwd(q, q, q, causal=True)
    assert fa.check_device_error()[0] == _abi.FA_OK
    assert torch.isfinite(o.float()).all()


def test_inconsistent_cu_seqlens_reported_not_read():
    # cu_seqlens claims 200 tokens but the tensors (and total_tokens) hold 100:
    # the kernel reports the sequence instead of reading past the buffers.
    q = torch.randn(100, 2, 64, device="cuda", dtype=torch.bfloat16)
    cu = torch.tensor([0, 50, 200], dtype=torch.int32, device="cuda")
    fa.fwd(q, q, q, cu_seqlens=cu, max_seqlen=150)
    assert fa.check_device_error()[0] == _abi.FA_ERR_INVALID_ARG
