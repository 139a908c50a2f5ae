"""Parity of samba_selective_scan_bwd against the float64 oracle's
selective_scan_bwd, through the C ABI.

Bound, per gradient tensor G: max |G_gpu - G_ref| <= 1e-4 · max |G_ref| (a
normwise bound: the gradients are long sums of products, some over all
channels or all tokens, evaluated in fp32 with approximate exps and added
with atomics), plus 2^-8 · |G_ref| per element for gradients stored in bf16.
"""

import numpy as np
import pytest
import torch

import oracle.samba_oracle as orc
from hybrid_ssm_sliding_b200 import build as B
from hybrid_ssm_sliding_b200 import ops
from hybrid_ssm_sliding_b200.workloads import WORKLOADS, Workload, make_output_grads, make_prefill_inputs
from tests._helpers import host64, record_margin

pytestmark = pytest.mark.gpu

BWD_TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


_KEYS = {"dx": "dx", "ddelta": "ddelta", "dA": "dA", "dB": "dB", "dC": "dC", "dD": "dD", "dz": "dz",
         "dconv_w": "dconv_w", "dconv_b": "dconv_b", "dh0": "dh0", "dconv_state": "dconv_state"}


def _check(name, got, ref, bf16_keys=()):
    worst = 0.0
    for key in _KEYS:
        r = ref.get(key)
        g = got.get(key)
        if r is None:
            assert g is None, key
            continue
        g = host64(g)
        assert np.all(np.isfinite(g)), f"{key}: non-finite"
        scale = float(np.max(np.abs(r))) or 1.0
        bound = BWD_TOL * scale + (2.0 ** -8 * np.abs(r) if key in bf16_keys else 0.0)
        ratio = float(np.max(np.abs(g - r) / bound))
        record_margin(name, key, worst_over_bound=ratio, max_abs=float(np.max(np.abs(g - r))), scale=scale)
        worst = max(worst, ratio)
        assert ratio <= 1.0, f"{name} {key}: error {ratio:.2f} x the bound"
    return worst


def _fwd_ckpt(inp, **kw):
    """The forward on the same inputs, writing its 16-token chunk checkpoints."""
    Bsz, Ln, D = inp["x"].shape
    ck = torch.full(ops.scan_ckpt_shape(Bsz, Ln, D, inp["A"].shape[1]), float("nan"), device="cuda")
    ops.selective_scan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], h_ckpt=ck, **kw)
    return ck


def _run(inp, dy, with_conv=True, with_z=True, with_D=True, softplus=True, h0=None, cs=None, conv_silu=True,
         fwd_ckpt=False):
    kw = dict(D=inp["D"] if with_D else None, z=inp["z"] if with_z else None,
              conv_w=inp["conv_w"] if with_conv else None, conv_b=inp["conv_b"] if with_conv else None,
              conv_state_in=cs, h0=h0, delta_softplus=softplus, conv_silu=conv_silu)
    ck = _fwd_ckpt(inp, **kw) if fwd_ckpt else None
    got = ops.selective_scan_bwd(dy, inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], want_dh0=True,
                                 want_dconv_state=with_conv, ckpt=ck, **kw)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    ref = orc.selective_scan_bwd(host64(dy), host64(inp["x"]), host64(inp["delta"]), host64(inp["A"]),
                                 host64(inp["B"]), host64(inp["C"]), host64(kw["D"]), host64(kw["z"]), host64(h0),
                                 host64(kw["conv_w"]), host64(kw["conv_b"]), host64(cs), softplus, conv_silu)
    if not with_conv:
        ref["dconv_state"] = None
    return got, ref


@pytest.mark.parametrize("Bsz,Ln,D,N,K,dt", [
    (2, 37, 40, 16, 4, torch.float32),     # ragged L and a partial channel block
    (1, 16, 32, 16, 4, torch.float32),     # exactly one chunk
    (1, 1, 8, 16, 4, torch.float32),       # one token
    (2, 2, 16, 8, 3, torch.float32),       # L < K - 1
    (3, 50, 24, 4, 2, torch.float32),
    (1, 300, 64, 16, 4, torch.bfloat16),
    (2, 129, 96, 8, 4, torch.bfloat16),
])
@pytest.mark.parametrize("fwd_ckpt", [False, True])
def test_scan_bwd_matches_oracle(Bsz, Ln, D, N, K, dt, fwd_ckpt):
    wl = Workload("sb", Bsz, Ln, D, N, K, 1, 1, 16, 16, 200 + Ln, act_dtype=dt)
    inp = make_prefill_inputs(wl, device="cuda", with_attention=False)
    dy = make_output_grads(wl, device="cuda", with_attention=False)["dy"]
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    h0 = torch.randn((Bsz, D, N), generator=g, device="cuda")
    cs = torch.randn((Bsz, D, K - 1), generator=g, device="cuda")
    got, ref = _run(inp, dy, h0=h0, cs=cs, fwd_ckpt=fwd_ckpt)
    bf = ("dx", "dz") if dt == torch.bfloat16 else ()
    _check(f"scan bwd B{Bsz} L{Ln} D{D} N{N} K{K} {str(dt)[6:]}{' fwd ckpt' if fwd_ckpt else ''}", got, ref, bf)


@pytest.mark.parametrize("conv,z,Dk,sp,silu", [
    (False, False, False, False, True),
    (False, True, True, True, True),
    (True, False, True, True, False),
    (True, True, False, False, True),
])
def test_scan_bwd_optional_parts(conv, z, Dk, sp, silu):
    wl = Workload("sbo", 2, 45, 32, 16, 4, 1, 1, 16, 16, 300, act_dtype=torch.float32)
    inp = make_prefill_inputs(wl, device="cuda", with_attention=False)
    if not sp:
        # without softplus the step sizes are taken as given: pass positive ones
        inp["delta"] = torch.nn.functional.softplus(inp["delta"]).contiguous()
    dy = make_output_grads(wl, device="cuda", with_attention=False)["dy"]
    got, ref = _run(inp, dy, with_conv=conv, with_z=z, with_D=Dk, softplus=sp, conv_silu=silu, fwd_ckpt=conv)
    _check(f"scan bwd options conv={conv} z={z} D={Dk} softplus={sp} silu={silu}", got, ref)


def test_scan_bwd_all_channels_of_a_layer():
    """d_inner 4096 (128 channel blocks adding into every dB, dC element)."""
    wl = Workload("sbw", 1, 256, 4096, 16, 4, 1, 1, 16, 16, 301)
    inp = make_prefill_inputs(wl, device="cuda", with_attention=False)
    dy = make_output_grads(wl, device="cuda", with_attention=False)["dy"]
    got, ref = _run(inp, dy)
    _check("scan bwd B1 L256 D4096 bf16", got, ref, ("dx", "dz"))


def test_scan_bwd_long_sequence():
    """4096 tokens, two sequences, 256 channels (256 chunks walked backwards)."""
    wl = Workload("sbl", 2, 4096, 256, 16, 4, 1, 1, 16, 16, 302)
    inp = make_prefill_inputs(wl, device="cuda", with_attention=False)
    dy = make_output_grads(wl, device="cuda", with_attention=False)["dy"]
    got, ref = _run(inp, dy, fwd_ckpt=True)
    _check("scan bwd B2 L4096 D256 bf16 fwd ckpt", got, ref, ("dx", "dz"))


def test_scan_bwd_training_workload_sampled_channels():
    """The training workload in the launch configuration bench.py times
    (8 x 4096 tokens, d_inner 4096): every per-channel gradient of 32 sampled
    channels against the oracle run on those channels alone (they depend on
    no other channel); dB and dC, which sum over all channels, are covered by
    the tests above."""
    wl = WORKLOADS["train_4k"]
    inp = make_prefill_inputs(wl, device="cuda", with_attention=False)
    dy = make_output_grads(wl, device="cuda", with_attention=False)["dy"]
    kw = dict(D=inp["D"], z=inp["z"], conv_w=inp["conv_w"], conv_b=inp["conv_b"])
    ck = _fwd_ckpt(inp, y_dtype=torch.bfloat16, **kw)   # as the training step runs it
    got = ops.selective_scan_bwd(dy, inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], want_dh0=True, ckpt=ck,
                                 **kw)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    rng = np.random.default_rng(5)
    chans = np.unique(np.concatenate([[0, 31, 32, 4095], rng.choice(4096, 28, replace=False)]))
    ci = torch.as_tensor(chans, device="cuda")
    sub = lambda t: host64(t.index_select(-1, ci))
    ref = orc.selective_scan_bwd(sub(dy), sub(inp["x"]), sub(inp["delta"]), host64(inp["A"][ci]), host64(inp["B"]),
                                 host64(inp["C"]), host64(inp["D"][ci]), sub(inp["z"]), None,
                                 host64(inp["conv_w"][ci]), host64(inp["conv_b"][ci]))
    got_sub = {"dx": got["dx"].index_select(-1, ci), "ddelta": got["ddelta"].index_select(-1, ci),
               "dz": got["dz"].index_select(-1, ci), "dA": got["dA"][ci], "dD": got["dD"][ci],
               "dconv_w": got["dconv_w"][ci], "dconv_b": got["dconv_b"][ci], "dh0": got["dh0"][:, ci]}
    for key in ("dB", "dC", "dconv_state"):
        ref[key] = None
    _check("scan bwd train_4k 32 channels", got_sub, ref, ("dx", "dz"))
