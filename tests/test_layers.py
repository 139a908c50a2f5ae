"""GPU parity of the Mamba and SWA layers (projections around the mixers,
through samba_gemm, samba_conv1d_fwd, samba_selective_scan_fwd and
samba_swa_fwd) against the float64 layer oracles, which store the same
activations in bf16 as the GPU dataflow does.

Tolerance: every output element within one bf16 unit in the last place of
the oracle's (2^-7 |ref|: the two sides round values that differ in their
last bits, so the final roundings may fall one unit apart) plus a share of
the output's rms for what reaches the output from the mixer: 1e-2 for the
Mamba layer (the scan's own errors are of order 1e-6, but an activation
rounded to bf16 may fall the other way), 5e-2 for the SWA layer, whose
attention rounds P to bf16 before P·V (errors of order 1e-2 in o, the
tolerance of the attention tests, mixed by the output projection)."""

import numpy as np
import pytest
import torch

import oracle.samba_oracle as orc
from hybrid_ssm_sliding_b200 import build as B
from hybrid_ssm_sliding_b200 import layers, ops
from tests._helpers import SCAN_TOL, host64, record_margin, scan_errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def _bound_check(got, ref, name, share):
    got = host64(got)
    assert np.all(np.isfinite(got)), "unwritten or non-finite output"
    rms = float(np.sqrt(np.mean(ref * ref)))
    worst = float(np.max(np.abs(got - ref) / (2.0 ** -7 * np.abs(ref) + share * rms)))
    record_margin(name, "out", worst_over_bound=worst, max_abs=float(np.max(np.abs(got - ref))), rms=rms)
    assert worst <= 1.0, f"{name}: error {worst:.2f} x the bound"


@pytest.mark.parametrize("Bsz,Ln,dm,D,N,R", [(1, 300, 256, 512, 16, 32), (2, 130, 128, 256, 8, 16)])
def test_mamba_layer_matches_oracle(Bsz, Ln, dm, D, N, R):
    w = layers.random_mamba_weights(dm, D, N, 4, R, seed=Ln)
    g = torch.Generator(device="cuda")
    g.manual_seed(Ln + 1)
    hidden = torch.randn((Bsz, Ln, dm), generator=g, device="cuda").to(torch.bfloat16)
    taps = {}
    out, h_final, cs = layers.mamba_layer_prefill(hidden, w, taps=taps)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    ref = orc.mamba_layer(host64(hidden), host64(w.in_proj), host64(w.conv_w), host64(w.conv_b), host64(w.x_proj),
                          host64(w.dt_proj), host64(w.dt_bias), host64(w.A), host64(w.D), host64(w.out_proj))
    _bound_check(out, ref["out"], f"mamba layer B{Bsz} L{Ln} d_model {dm} D {D}", 1e-2)
    # the conv state holds x, the bf16 of a GEMM output: its fp32 accumulation
    # and the oracle's float64 sum may round one bf16 unit apart
    cs_err = np.abs(host64(cs) - ref["conv_state"])
    assert np.all(cs_err <= 2.0 ** -7 * np.abs(ref["conv_state"])), f"conv state off by {cs_err.max():.3e}"
    # The final state: an activation that rounds to the other bf16 neighbour
    # than the oracle's moves h by a few units in the third digit where h is
    # small, so h is checked against the oracle's scan over the activations
    # the layer actually used (its taps), at the scan's own tolerance.
    sc = orc.selective_scan(host64(taps["u"]), host64(taps["delta"]), host64(w.A), host64(taps["B"]),
                            host64(taps["C"]), host64(w.D), host64(taps["z"]), magnitudes=True)
    eh = scan_errors(host64(h_final), sc["h"], sc["h_mag"])
    record_margin(f"mamba layer B{Bsz} L{Ln} d_model {dm} D {D}", "h", tol=SCAN_TOL, **eh)
    assert eh["rel_to_mag"] <= SCAN_TOL, f"h rel err {eh['rel_to_mag']:.3e}"
    y_err = np.abs(host64(taps["y"]) - sc["y"]) / (SCAN_TOL * sc["y_mag"] + 2.0 ** -8 * np.abs(sc["y"]))
    assert y_err.max() <= 1.0, f"y off by {y_err.max():.2f} x its bound"


@pytest.mark.parametrize("Bsz,Ln,dm,Hq,Hkv,d,W", [(1, 300, 256, 8, 2, 64, 128), (2, 200, 128, 4, 4, 32, 1000)])
def test_swa_layer_matches_oracle(Bsz, Ln, dm, Hq, Hkv, d, W):
    w = layers.random_swa_weights(dm, Hq, Hkv, d, W, seed=Ln + W)
    g = torch.Generator(device="cuda")
    g.manual_seed(Ln + 2)
    hidden = torch.randn((Bsz, Ln, dm), generator=g, device="cuda").to(torch.bfloat16)
    out, k, v = layers.swa_layer_prefill(hidden, w)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    ref = orc.swa_layer(host64(hidden), host64(w.qkv_proj), host64(w.o_proj), Hq, Hkv, d, W)
    _bound_check(out, ref["out"], f"swa layer B{Bsz} L{Ln} d_model {dm} {Hq}/{Hkv}x{d} W{W}", 5e-2)
