"""samba_swa_step_noalloc: the decode step for callers that cannot allocate
device memory (a host framework that owns all device allocations, or code
where cudaMalloc is refused), which therefore cannot hand samba_swa_step a
workspace.  Its scratch is a fixed 4 MiB array inside the library.

The test calls both entry points through the C ABI on the same state and
checks that two consecutive steps agree within the attention tolerance of the
other tests, and that oversized problems are refused.  It lives in its own
file, collected last, and passes alone or after the rest of the suite."""

import ctypes

import numpy as np
import pytest
import torch

from hybrid_ssm_sliding_b200 import _lib as L
from hybrid_ssm_sliding_b200 import build as B
from hybrid_ssm_sliding_b200 import ops
from tests._helpers import SWA_MAX_ABS, SWA_MEAN_ABS, host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def _state(Bsz, L1, Hkv, d, W, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    k = torch.randn((Bsz, L1, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((Bsz, L1, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    return ops.swa_ring_fill(k, v, W)


def test_noalloc_step_matches_workspace_step_on_two_calls():
    lib = L.load()
    Bsz, Hq, Hkv, d, W = 16, 32, 4, 64, 2048
    kr, vr, pos = _state(Bsz, 1500, Hkv, d, W, seed=11)
    kr2, vr2, pos2 = kr.clone(), vr.clone(), pos.clone()
    s = torch.cuda.current_stream().cuda_stream
    g = torch.Generator(device="cuda")
    g.manual_seed(12)
    for _ in range(2):  # two calls in a row: the shared scratch keeps the previous call's contents
        q_t = torch.randn((Bsz, Hq, d), generator=g, device="cuda").to(torch.bfloat16)
        k_t = torch.randn((Bsz, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
        v_t = torch.randn((Bsz, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
        o_ref = ops.swa_step(q_t, k_t, v_t, kr, vr, pos, W)
        o_na = torch.empty_like(q_t)
        rc = lib.samba_swa_step_noalloc(q_t.data_ptr(), k_t.data_ptr(), v_t.data_ptr(), kr2.data_ptr(),
                                        vr2.data_ptr(), pos2.data_ptr(), o_na.data_ptr(), Bsz, Hq, Hkv, d, W,
                                        ctypes.c_float(0.0), s)
        assert rc == L.SAMBA_OK, lib.samba_last_error().decode()
        torch.cuda.synchronize()
        err = np.abs(host64(o_na) - host64(o_ref))
        assert err.max() <= SWA_MAX_ABS and err.mean() <= SWA_MEAN_ABS
        assert torch.equal(pos2, pos)
    assert torch.equal(kr2, kr) and torch.equal(vr2, vr)
    assert ops.get_status() == L.SAMBA_OK


def test_noalloc_step_refuses_sizes_beyond_its_scratch():
    lib = L.load()
    Bsz, Hq, Hkv, d, W = 64, 64, 4, 128, 4096  # the split partials need far more than 4 MiB
    assert lib.samba_swa_step_workspace_size(Bsz, Hq, d, W) > (4 << 20)
    buf = torch.empty((16,), dtype=torch.uint8, device="cuda")
    pos = torch.zeros((Bsz,), dtype=torch.int64, device="cuda")
    p = buf.data_ptr()
    rc = lib.samba_swa_step_noalloc(p, p, p, p, p, pos.data_ptr(), p, Bsz, Hq, Hkv, d, W, ctypes.c_float(0.0),
                                    torch.cuda.current_stream().cuda_stream)
    assert rc == L.SAMBA_ERR_WORKSPACE
    assert "4194304" in lib.samba_last_error().decode()
