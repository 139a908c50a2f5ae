"""GPU parity of the tcgen05 sliding-window attention against the float64
oracle, through the C ABI.

Tolerance: bf16 output within 2e-2 max abs and 1e-2 mean abs of the
float64 result on the same bf16 inputs; lse within 2e-3 abs."""

import math

import numpy as np
import pytest
import torch

import oracle.samba_oracle as orc
from hybrid_ssm_sliding_b200 import build as B
from hybrid_ssm_sliding_b200 import ops
from hybrid_ssm_sliding_b200.workloads import WORKLOADS, Workload, make_prefill_inputs
from tests._helpers import SWA_MAX_ABS, SWA_MEAN_ABS, host64, record_margin

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def _qkv(Bsz, Ln, Hq, Hkv, d, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    q = torch.randn((Bsz, Ln, Hq, d), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((Bsz, Ln, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((Bsz, Ln, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    return q, k, v


def _gpu(q, k, v, W, scale=None):
    Bsz, Ln, Hq, _ = q.shape
    lse = torch.full((Bsz, Hq, Ln), float("nan"), device="cuda")
    o = torch.full_like(q, float("nan"))  # poison: every element must be written
    ops.swa_fwd(q, k, v, W, scale=scale, o=o, lse=lse)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    return o, lse


def _compare(o, lse, ref_o, ref_lse, name=None):
    got = host64(o)
    assert np.all(np.isfinite(got)), "unwritten or non-finite output"
    err = np.abs(got - ref_o)
    if name:
        el_ = np.abs(host64(lse) - ref_lse)
        record_margin(name, "o", max_abs=err.max(), mean_abs=err.mean(), tol_max_abs=SWA_MAX_ABS,
                      tol_mean_abs=SWA_MEAN_ABS, lse_max_abs=el_.max(), rows=int(got.shape[1]))
    assert err.max() <= SWA_MAX_ABS, f"max abs {err.max():.3e}"
    assert err.mean() <= SWA_MEAN_ABS, f"mean abs {err.mean():.3e}"
    el = np.abs(host64(lse) - ref_lse)
    assert el.max() <= 2e-3, f"lse max abs {el.max():.3e}"
    return err.max(), err.mean()


def test_tiny_workload():
    wl = WORKLOADS["tiny"]
    inp = make_prefill_inputs(wl, device="cuda")
    o, lse = _gpu(inp["q"], inp["k"], inp["v"], wl.window)
    ref_o, ref_lse = orc.swa(host64(inp["q"]), host64(inp["k"]), host64(inp["v"]), wl.window)
    _compare(o, lse, ref_o, ref_lse, name="swa tiny")


@pytest.mark.parametrize("Bsz,Ln,Hq,Hkv,d,W", [
    (1, 300, 8, 1, 64, 100),
    (2, 257, 32, 4, 64, 64),
    (1, 1000, 4, 4, 32, 1),
    (1, 513, 16, 1, 16, 1000),      # W >= L: full causal attention
    (3, 130, 2, 1, 64, 17),
    (1, 200, 16, 1, 64, 50),        # 16 query heads per kv head
    (1, 700, 8, 2, 64, 333),
    (2, 64, 2, 2, 16, 16),
    (1, 1, 8, 1, 64, 4),            # a single token
    (1, 1500, 32, 4, 64, 2048),
])
def test_small_cases(Bsz, Ln, Hq, Hkv, d, W):
    q, k, v = _qkv(Bsz, Ln, Hq, Hkv, d, seed=Ln * 7 + W)
    o, lse = _gpu(q, k, v, W)
    ref_o, ref_lse = orc.swa(host64(q), host64(k), host64(v), W)
    _compare(o, lse, ref_o, ref_lse)


def test_explicit_scale():
    q, k, v = _qkv(1, 260, 8, 1, 64, seed=3)
    o, lse = _gpu(q, k, v, 90, scale=0.05)
    ref_o, ref_lse = orc.swa(host64(q), host64(k), host64(v), 90, scale=0.05)
    _compare(o, lse, ref_o, ref_lse)


def test_window_one_returns_v_exactly():
    q, k, v = _qkv(1, 300, 8, 2, 64, seed=9)
    o, _ = _gpu(q, k, v, 1)
    assert torch.equal(o, v.repeat_interleave(4, dim=2))


def test_constant_query_gives_window_mean():
    _, k, v = _qkv(1, 400, 8, 1, 64, seed=10)
    q = torch.zeros((1, 400, 8, 64), device="cuda", dtype=torch.bfloat16)
    W = 150
    o, _ = _gpu(q, k, v, W)
    vv = host64(v)[0, :, 0, :]
    csum = np.concatenate([np.zeros((1, 64)), np.cumsum(vv, 0)])
    i = np.arange(400)
    j0 = np.maximum(0, i - W + 1)
    mean = (csum[i + 1] - csum[j0]) / (i + 1 - j0)[:, None]
    err = np.abs(host64(o)[0] - mean[:, None, :])
    assert err.max() <= SWA_MAX_ABS


def _sample_blocks(Ln, W, n, seed, block=64):
    """Starts of n query blocks: the ramp at row 0, the block around row W
    (where the window first fills), the last block, and random others."""
    g = np.random.default_rng(seed)
    fixed = [0, max(0, W - block // 2), max(0, Ln - block)]
    extra = g.choice(max(1, Ln - block), max(0, n - len(fixed)), replace=False)
    return sorted(set(int(s) for s in list(fixed) + list(extra)))


def _check_blocks(q, k, v, W, o, lse, starts, name):
    rows, ref_o, ref_lse = orc.swa_blocks(host64(q), host64(k), host64(v), W, starts)
    rows_t = torch.from_numpy(rows).cuda()
    _compare(o[:, rows_t], lse[:, :, rows_t], ref_o, ref_lse, name=name)


def test_pair_4k_sampled_rows():
    wl = WORKLOADS["pair_4k"]
    inp = make_prefill_inputs(wl, device="cuda", with_scan=False)
    o, lse = _gpu(inp["q"], inp["k"], inp["v"], wl.window)
    _check_blocks(inp["q"], inp["k"], inp["v"], wl.window, o, lse, _sample_blocks(wl.seqlen, wl.window, 16, 1),
                  "swa pair_4k (16 blocks of 64 rows)")


@pytest.mark.slow
@pytest.mark.parametrize("name", ["prefill_128k", "batched_32k"])
def test_full_size_sampled_rows(name):
    """Full-size workloads in the launch configuration bench.py times; the
    oracle checks 4096 query rows in all (64-row blocks, every head)."""
    wl = WORKLOADS[name]
    inp = make_prefill_inputs(wl, device="cuda", with_scan=False)
    o, lse = _gpu(inp["q"], inp["k"], inp["v"], wl.window)
    per_row = 64 // wl.batch
    for b in range(wl.batch):
        sl = slice(b, b + 1)
        starts = _sample_blocks(wl.seqlen, wl.window, per_row, wl.seed * 100 + b)
        _check_blocks(inp["q"][sl], inp["k"][sl], inp["v"][sl], wl.window, o[sl], lse[sl], starts,
                      f"swa {name} batch row {b} ({len(starts)} blocks of 64 rows)")
