"""GPU parity of the fused selective scan (conv -> softplus -> scan -> D skip
-> gate) against the float64 oracle, through the C ABI.

Tolerance: max relative error <= 1e-4 on y (fp32 output) and on the final
state h, each error taken relative to the size of the sum that produced the
value (the oracle's y_mag / h_mag), and exact equality of the conv state (a
copy of inputs)."""

import numpy as np
import pytest
import torch

import oracle.samba_oracle as orc
from hybrid_ssm_sliding_b200 import build as B
from hybrid_ssm_sliding_b200 import ops
from hybrid_ssm_sliding_b200.workloads import WORKLOADS, Workload, make_prefill_inputs
from tests._helpers import SCAN_TOL, host64, nan_tensor, record_margin, scan_errors, scan_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def _run_gpu(inp, y_dtype=torch.float32, z=True, conv=True, softplus=True, silu=True, Dskip=True,
             h0=None, cs_in=None):
    Bsz, Ln, D = inp["x"].shape
    N = inp["A"].shape[1]
    K = inp["conv_w"].shape[1]
    # every output starts as NaN, so an element the kernel never writes fails
    h_final = nan_tensor((Bsz, D, N), torch.float32)
    cs_out = nan_tensor((Bsz, D, K - 1), torch.float32) if conv else None
    y = nan_tensor((Bsz, Ln, D), y_dtype)
    ops.selective_scan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                               D=inp["D"] if Dskip else None, z=inp["z"] if z else None,
                               conv_w=inp["conv_w"] if conv else None, conv_b=inp["conv_b"] if conv else None,
                               conv_state_in=cs_in, h0=h0, y=y, h_final=h_final,
                               conv_state_out=cs_out, delta_softplus=softplus, conv_silu=silu)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    return y, h_final, cs_out


def _run_oracle(inp, chans=None, z=True, conv=True, softplus=True, silu=True, Dskip=True, h0=None, cs_in=None):
    sel = slice(None) if chans is None else chans
    x = host64(inp["x"][:, :, sel])
    out = orc.selective_scan(
        x, host64(inp["delta"][:, :, sel]), host64(inp["A"][sel]), host64(inp["B"]), host64(inp["C"]),
        Dskip=host64(inp["D"][sel]) if Dskip else None, z=host64(inp["z"][:, :, sel]) if z else None,
        h0=None if h0 is None else host64(h0[:, sel]),
        conv_w=host64(inp["conv_w"][sel]) if conv else None, conv_b=host64(inp["conv_b"][sel]) if conv else None,
        conv_state=None if cs_in is None else host64(cs_in[:, sel]),
        delta_softplus=softplus, conv_silu=silu, magnitudes=True)
    return out


def _check(y, hf, cs, ref, chans=None, name=None):
    sel = slice(None) if chans is None else chans
    gy, gh = host64(y[:, :, sel]), host64(hf[:, sel])
    assert np.all(np.isfinite(gy)) and np.all(np.isfinite(gh)), "unwritten or non-finite output"
    e_y = scan_errors(gy, ref["y"], ref["y_mag"])
    e_h = scan_errors(gh, ref["h"], ref["h_mag"])
    ey, eh = e_y["rel_to_mag"], e_h["rel_to_mag"]
    if name:
        record_margin(name, "y", tol=SCAN_TOL, **e_y)
        record_margin(name, "h_final", tol=SCAN_TOL, **e_h)
    assert ey <= SCAN_TOL, f"y rel err {ey:.3e} (floor metric {e_y['rel_floor']:.3e})"
    assert eh <= SCAN_TOL, f"h rel err {eh:.3e} (floor metric {e_h['rel_floor']:.3e})"
    if cs is not None and ref["conv_state"] is not None:
        np.testing.assert_array_equal(host64(cs[:, sel]), ref["conv_state"])
    return ey, eh


def _inputs(wl):
    return make_prefill_inputs(wl, device="cuda", with_attention=False)


def test_tiny_workload_fp32():
    wl = WORKLOADS["tiny"]
    inp = _inputs(wl)
    y, hf, cs = _run_gpu(inp)
    _check(y, hf, cs, _run_oracle(inp), name="scan tiny")


@pytest.mark.parametrize("Bsz,Ln,D,N,dt", [
    (2, 200, 48, 16, torch.bfloat16),   # ragged time tile and channel block
    (1, 64, 32, 16, torch.float32),
    (3, 131, 40, 8, torch.bfloat16),
    (2, 150, 48, 8, torch.float32),     # N = 8 with fp32 x: two TMA stages, 4 epilogue warps
    (2, 77, 24, 4, torch.float32),
    (1, 1, 16, 16, torch.bfloat16),     # L = 1
    (2, 2, 16, 16, torch.float32),      # L < K - 1
    (1, 3, 8, 4, torch.bfloat16),
])
def test_ragged_shapes(Bsz, Ln, D, N, dt):
    wl = Workload("t", Bsz, Ln, D, N, 4, 1, 1, 16, 16, 11 + Ln, act_dtype=dt)
    inp = _inputs(wl)
    y, hf, cs = _run_gpu(inp)
    _check(y, hf, cs, _run_oracle(inp))


@pytest.mark.parametrize("opts", [
    dict(z=False), dict(conv=False), dict(softplus=False), dict(silu=False), dict(Dskip=False),
    dict(z=False, conv=False, Dskip=False),
])
def test_flag_variants(opts):
    wl = Workload("t", 2, 150, 32, 16, 4, 1, 1, 16, 16, 5, act_dtype=torch.bfloat16)
    inp = _inputs(wl)
    if opts.get("softplus") is False:
        inp["delta"] = torch.nn.functional.softplus(inp["delta"])  # positive step sizes, used as Δ directly
    y, hf, cs = _run_gpu(inp, **opts)
    _check(y, hf, cs, _run_oracle(inp, **opts))


@pytest.mark.parametrize("K", [2, 3, 4])
def test_conv_widths(K):
    wl = Workload("t", 2, 70, 16, 16, K, 1, 1, 16, 16, 40 + K, act_dtype=torch.float32)
    inp = _inputs(wl)
    y, hf, cs = _run_gpu(inp)
    _check(y, hf, cs, _run_oracle(inp))


def test_initial_state_and_split_carry():
    """Running [0, L1) then [L1, L) with the carried (h, conv state) equals
    one pass, on the GPU and against the oracle."""
    wl = Workload("t", 2, 300, 32, 16, 4, 1, 1, 16, 16, 21, act_dtype=torch.float32)
    inp = _inputs(wl)
    y_full, h_full, cs_full = _run_gpu(inp)
    L1 = 113
    first = {k: (v[:, :L1].contiguous() if k in ("x", "z", "delta", "B", "C") else v) for k, v in inp.items()}
    rest = {k: (v[:, L1:].contiguous() if k in ("x", "z", "delta", "B", "C") else v) for k, v in inp.items()}
    y1, h1, cs1 = _run_gpu(first)
    y2, h2, cs2 = _run_gpu(rest, h0=h1, cs_in=cs1)
    ref = _run_oracle(inp)
    _check(torch.cat([y1, y2], 1), h2, cs2, ref)
    ref2 = _run_oracle(rest, h0=h1, cs_in=cs1)
    _check(y2, h2, cs2, ref2)


def test_h_final_may_alias_h0():
    wl = Workload("t", 1, 100, 16, 16, 4, 1, 1, 16, 16, 8, act_dtype=torch.float32)
    inp = _inputs(wl)
    h = torch.randn((1, 16, 16), device="cuda")
    ref = _run_oracle(inp, h0=h)
    ops.selective_scan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                           conv_w=inp["conv_w"], conv_b=inp["conv_b"], h0=h, h_final=h, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert scan_rel_err(host64(h), ref["h"], ref["h_mag"]) <= SCAN_TOL


def test_pair_4k_full():
    wl = WORKLOADS["pair_4k"]
    inp = _inputs(wl)
    y, hf, cs = _run_gpu(inp)
    _check(y, hf, cs, _run_oracle(inp), name="scan pair_4k (all channels)")
    # The bf16-output instantiation (the one bench.py times) differs only in
    # the final rounding of y.
    yb, hb, _ = _run_gpu(inp, y_dtype=torch.bfloat16)
    assert torch.equal(hb, hf)
    assert torch.equal(yb, y.to(torch.bfloat16))


def _sample_channels(D, n, seed):
    g = np.random.default_rng(seed)
    ch = np.unique(np.concatenate([[0, 1, D - 1], g.choice(D, n - 3, replace=False)]))
    return torch.from_numpy(ch).cuda()


@pytest.mark.slow
@pytest.mark.parametrize("name", ["prefill_128k", "batched_32k"])
def test_full_size_sampled_channels(name):
    """Full-size workloads in the launch configuration bench.py times (bf16
    y) plus the fp32-y instantiation; the oracle checks a channel subset."""
    wl = WORKLOADS[name]
    inp = _inputs(wl)
    y, hf, cs = _run_gpu(inp)
    chans = _sample_channels(wl.dim, 64, wl.seed)
    sub = {k: (v[..., chans] if k in ("x", "z", "delta") else v) for k, v in inp.items()}
    sub["A"], sub["D"] = inp["A"][chans], inp["D"][chans]
    sub["conv_w"], sub["conv_b"] = inp["conv_w"][chans], inp["conv_b"][chans]
    ref = _run_oracle(sub)
    _check(y[..., chans], hf[:, chans], cs[:, chans], ref, name=f"scan {name} ({len(chans)} channels)")
    yb, hb, _ = _run_gpu(inp, y_dtype=torch.bfloat16)
    assert torch.equal(hb, hf)
    assert torch.equal(yb, y.to(torch.bfloat16))


@pytest.mark.parametrize("Bsz,Ln,D,N,dt", [(2, 75, 40, 16, torch.float32), (1, 64, 32, 8, torch.bfloat16),
                                           (1, 5, 16, 4, torch.float32)])
def test_forward_checkpoints_are_the_chunk_start_states(Bsz, Ln, D, N, dt):
    """h_ckpt[:, c] is the state before token 16 c: h0 for c = 0, else the
    oracle's final state after the first 16 c tokens (same inputs, conv state
    and h0)."""
    wl = Workload("ck", Bsz, Ln, D, N, 4, 1, 1, 16, 16, 400 + Ln, act_dtype=dt)
    inp = make_prefill_inputs(wl, device="cuda", with_attention=False)
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    h0 = torch.randn((Bsz, D, N), generator=g, device="cuda")
    cs = torch.randn((Bsz, D, 3), generator=g, device="cuda")
    ck = torch.full(ops.scan_ckpt_shape(Bsz, Ln, D, N), float("nan"), device="cuda")
    kw = dict(D=inp["D"], z=inp["z"], conv_w=inp["conv_w"], conv_b=inp["conv_b"], conv_state_in=cs, h0=h0)
    ops.selective_scan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], h_ckpt=ck, **kw)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    got = host64(ck)                                     # [B, nck, N, D]
    np.testing.assert_array_equal(got[:, 0], host64(h0).transpose(0, 2, 1))
    for c in range(1, got.shape[1]):
        t = 16 * c
        ref = orc.selective_scan(host64(inp["x"][:, :t]), host64(inp["delta"][:, :t]), host64(inp["A"]),
                                 host64(inp["B"][:, :t]), host64(inp["C"][:, :t]), host64(inp["D"]),
                                 host64(inp["z"][:, :t]), h0=host64(h0), conv_w=host64(inp["conv_w"]),
                                 conv_b=host64(inp["conv_b"]), conv_state=host64(cs), magnitudes=True)
        e = scan_errors(got[:, c].transpose(0, 2, 1), ref["h"], ref["h_mag"])
        assert e["rel_to_mag"] <= SCAN_TOL, (c, e["rel_to_mag"])
