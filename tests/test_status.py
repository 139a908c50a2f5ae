"""Failure detection without a GPU fault: a kernel whose wait can never be
satisfied gives up after its bounded limit, reports SAMBA_ERR_TIMEOUT through
the status word, and leaves the context usable for the next launch."""

import pytest
import torch

from hybrid_ssm_sliding_b200 import _lib as L
from hybrid_ssm_sliding_b200 import build as B
from hybrid_ssm_sliding_b200 import ops

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def test_status_is_clear_after_normal_work():
    q = torch.randn((1, 100, 8, 64), device="cuda").to(torch.bfloat16)
    k = torch.randn((1, 100, 1, 64), device="cuda").to(torch.bfloat16)
    ops.swa_fwd(q, k, k, 32)
    assert ops.get_status() == L.SAMBA_OK


def test_bounded_wait_times_out_and_reports():
    lib = L.load()
    s = torch.cuda.current_stream().cuda_stream
    assert ops.get_status() == L.SAMBA_OK
    assert lib.samba_selftest_wait_timeout(s) == L.SAMBA_OK
    assert ops.get_status() == L.SAMBA_ERR_TIMEOUT      # read and cleared
    assert ops.get_status() == L.SAMBA_OK
    # the context is still healthy: a real kernel runs and is correct
    q = torch.zeros((1, 40, 2, 16), device="cuda", dtype=torch.bfloat16)
    v = torch.randn((1, 40, 2, 16), device="cuda").to(torch.bfloat16)
    o = ops.swa_fwd(q, v, v, 1)
    torch.cuda.synchronize()
    assert torch.equal(o, v)
    assert ops.get_status() == L.SAMBA_OK
