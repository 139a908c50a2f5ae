"""Sequence-parallel prefill on one GPU: a prompt split into segments, each
segment's phases run in turn (the exchanges become references), against the
float64 oracle over the whole prompt and against the library's single pass.

The segments join through the library's conv-state, delta-sum and scan-carry
kernels; the result must match one pass within the tolerances of the prefill
tests."""

import numpy as np
import pytest
import torch

import oracle.samba_oracle as orc
from hybrid_ssm_sliding_b200 import build as B
from hybrid_ssm_sliding_b200 import ops, seqpar
from hybrid_ssm_sliding_b200.workloads import Workload, make_prefill_inputs
from tests._helpers import SCAN_TOL, SWA_MAX_ABS, SWA_MEAN_ABS, host64, record_margin, scan_errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def _split(inp, keys, parts):
    Ln = inp["x"].shape[1]
    bounds = np.linspace(0, Ln, parts + 1).astype(int)
    out = []
    for r in range(parts):
        sl = slice(bounds[r], bounds[r + 1])
        out.append({k: (v[:, sl].contiguous() if k in keys else v) for k, v in inp.items()})
    return out, bounds


@pytest.mark.parametrize("Bsz,Ln,D,N,W,parts,dt", [
    (1, 4096, 64, 16, 256, 4, torch.bfloat16),
    (2, 1800, 48, 8, 100, 3, torch.float32),
    (1, 777, 32, 16, 300, 2, torch.bfloat16),
])
def test_segments_in_turn_match_one_pass(Bsz, Ln, D, N, W, parts, dt):
    wl = Workload("sp", Bsz, Ln, D, N, 4, 32, 4, 64, W, 90 + parts, act_dtype=dt)
    inp = make_prefill_inputs(wl, device="cuda")
    seq_keys = ("x", "z", "delta", "B", "C", "q", "k", "v")
    segs, bounds = _split(inp, seq_keys, parts)
    scans = [dict(x=s["x"], delta=s["delta"], A=s["A"], B=s["B"], C=s["C"], D=s["D"], z=s["z"], conv_w=s["conv_w"],
                  conv_b=s["conv_b"], y_dtype=torch.float32) for s in segs]
    swas = [dict(q=s["q"], k=s["k"], v=s["v"], window=W) for s in segs]
    res = seqpar.prefill_in_turn(scans, swas)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    y = torch.cat([r[0] for r in res], dim=1)
    o = torch.cat([r[1] for r in res], dim=1)
    h_final, cs_final = res[-1][2], res[-1][3]

    # against the oracle over the whole prompt
    ref = orc.selective_scan(host64(inp["x"]), host64(inp["delta"]), host64(inp["A"]), host64(inp["B"]),
                             host64(inp["C"]), host64(inp["D"]), host64(inp["z"]), conv_w=host64(inp["conv_w"]),
                             conv_b=host64(inp["conv_b"]), magnitudes=True)
    ey = scan_errors(host64(y), ref["y"], ref["y_mag"])
    eh = scan_errors(host64(h_final), ref["h"], ref["h_mag"])
    record_margin(f"seqpar {parts} segments, L={Ln}", "y", tol=SCAN_TOL, **ey)
    record_margin(f"seqpar {parts} segments, L={Ln}", "h_final", tol=SCAN_TOL, **eh)
    assert ey["rel_to_mag"] <= SCAN_TOL, f"y rel err {ey['rel_to_mag']:.3e}"
    assert eh["rel_to_mag"] <= SCAN_TOL, f"h rel err {eh['rel_to_mag']:.3e}"
    np.testing.assert_array_equal(host64(cs_final), ref["conv_state"])
    ref_o, _ = orc.swa(host64(inp["q"]), host64(inp["k"]), host64(inp["v"]), W)
    err = np.abs(host64(o) - ref_o)
    record_margin(f"seqpar {parts} segments, L={Ln}", "o", max_abs=err.max(), mean_abs=err.mean(),
                  tol_max_abs=SWA_MAX_ABS, tol_mean_abs=SWA_MEAN_ABS)
    assert err.max() <= SWA_MAX_ABS and err.mean() <= SWA_MEAN_ABS

    # the attention of the segments agrees with the single pass up to fp32
    # rounding: the halo gives every query the same keys, only grouped into
    # key tiles differently
    o_one = ops.swa_fwd(inp["q"], inp["k"], inp["v"], W)
    torch.cuda.synchronize()
    assert float((o.float() - o_one.float()).abs().max()) <= 2 * 2.0 ** -8


def test_carry_kernel_matches_its_definition():
    """h_out = exp(A * dsum) * h_in + h_local, elementwise (and h_in = None
    for a zero start state)."""
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    Bsz, D, N = 3, 40, 16
    A = -torch.rand((D, N), generator=g, device="cuda") * 4
    dsum = torch.rand((Bsz, D), generator=g, device="cuda") * 3
    h_in = torch.randn((Bsz, D, N), generator=g, device="cuda")
    h_loc = torch.randn((Bsz, D, N), generator=g, device="cuda")
    out = ops.scan_carry(h_in, dsum, A, h_loc)
    out0 = ops.scan_carry(None, dsum, A, h_loc)
    torch.cuda.synchronize()
    ref = np.exp(host64(A)[None] * host64(dsum)[:, :, None]) * host64(h_in) + host64(h_loc)
    np.testing.assert_allclose(host64(out), ref, rtol=2e-6, atol=2e-6)
    np.testing.assert_array_equal(host64(out0), host64(h_loc))


def test_delta_sum_is_the_sum_of_the_step_sizes():
    wl = Workload("ds", 2, 333, 48, 16, 4, 1, 1, 16, 16, 4, act_dtype=torch.bfloat16)
    inp = make_prefill_inputs(wl, device="cuda", with_attention=False)
    dsum = torch.full((2, 48), float("nan"), device="cuda")
    ops.selective_scan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                           conv_w=inp["conv_w"], conv_b=inp["conv_b"], delta_sum=dsum)
    torch.cuda.synchronize()
    ref = orc.softplus(host64(inp["delta"])).sum(axis=1)
    np.testing.assert_allclose(host64(dsum), ref, rtol=1e-5)


def test_conv_state_kernel_hands_on_the_last_inputs():
    wl = Workload("cs", 2, 50, 24, 16, 4, 1, 1, 16, 16, 6, act_dtype=torch.bfloat16)
    inp = make_prefill_inputs(wl, device="cuda", with_attention=False)
    cs_in = torch.randn((2, 24, 3), device="cuda")
    for Ln in (1, 2, 50):
        x = inp["x"][:, :Ln].contiguous()
        got = ops.conv_state(x, 4, conv_state_in=cs_in)
        torch.cuda.synchronize()
        xpad = np.concatenate([host64(cs_in).transpose(0, 2, 1), host64(x)], axis=1)   # [B, 3 + L, D]
        np.testing.assert_array_equal(host64(got), xpad[:, -3:].transpose(0, 2, 1))
