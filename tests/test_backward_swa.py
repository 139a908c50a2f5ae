"""Parity of samba_swa_bwd against the float64 oracle's swa_bwd, through the C
ABI (the forward's o and lse come from samba_swa_fwd on the same inputs).

Bound, element by element for each bf16 gradient G:
    |G_gpu - G_ref| <= 2^-8 |G_ref| + 2^-7 · G_mag
with G_mag the oracle's magnitude of the sum that produces G (the same sum
over absolute values of its terms).  The first term is the final bf16
rounding.  The kernels round P (for dv), dS (for dq, dk) and, through the
forward's stored o, D = dO · o to bf16: relative errors of at most 2^-8 on the
terms that G_mag sizes, so 2^-8 · G_mag to first order; 2^-7 leaves room for
the fp32 sums and the second-order terms.
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

MAG_FACTOR = 2.0 ** -7


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def _ratio(g, r, mag):
    return float(np.max(np.abs(g - r) / (2.0 ** -8 * np.abs(r) + MAG_FACTOR * mag + 1e-30)))


def _bound_check(name, got, ref):
    worst = 0.0
    dq, dk, dv, mags = ref
    for key, g, r in zip(("dq", "dk", "dv"), got, (dq, dk, dv)):
        g = host64(g) if torch.is_tensor(g) else g
        assert np.all(np.isfinite(g)), f"{name} {key}: non-finite"
        ratio = _ratio(g, r, mags[key])
        rms = float(np.sqrt(np.mean(r * r)))
        record_margin(name, key, worst_over_bound=ratio, max_abs=float(np.max(np.abs(g - r))),
                      mean_abs=float(np.mean(np.abs(g - r))), rms=rms)
        worst = max(worst, ratio)
        assert ratio <= 1.0, f"{name} {key}: error {ratio:.2f} x the bound"
    return worst


def _inputs(Bsz, Ln, Hq, Hkv, d, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    mk = lambda H: torch.randn((Bsz, Ln, H, d), generator=g, device="cuda").to(torch.bfloat16)
    return mk(Hq), mk(Hkv), mk(Hkv), mk(Hq)


def _fwd_bwd(q, k, v, do, W, scale=None):
    Bsz, Ln, Hq, d = q.shape
    lse = torch.empty((Bsz, Hq, Ln), dtype=torch.float32, device="cuda")
    o = ops.swa_fwd(q, k, v, W, scale=scale, lse=lse)
    dq = torch.full_like(q, float("nan"))
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(v, float("nan"))
    ops.swa_bwd(do, q, k, v, o, lse, W, scale=scale, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    return dq, dk, dv


@pytest.mark.parametrize("Bsz,Ln,Hq,Hkv,d,W", [
    (1, 64, 2, 2, 16, 16),
    (1, 300, 8, 1, 64, 100),
    (2, 257, 32, 4, 64, 64),
    (1, 1500, 32, 4, 64, 2048),
    (1, 200, 4, 4, 32, 1000),
    (2, 130, 16, 1, 64, 1),
    (1, 513, 16, 8, 32, 129),
    (1, 1, 8, 4, 64, 16),
    (3, 70, 32, 2, 16, 40),
])
def test_swa_bwd_matches_oracle(Bsz, Ln, Hq, Hkv, d, W):
    q, k, v, do = _inputs(Bsz, Ln, Hq, Hkv, d, Ln + W + d)
    got = _fwd_bwd(q, k, v, do, W)
    ref = orc.swa_bwd(host64(do), host64(q), host64(k), host64(v), W, magnitudes=True)
    _bound_check(f"swa bwd B{Bsz} L{Ln} {Hq}/{Hkv}x{d} W{W}", got, ref)


def test_swa_bwd_explicit_scale():
    q, k, v, do = _inputs(1, 200, 8, 2, 64, 11)
    got = _fwd_bwd(q, k, v, do, 50, scale=0.07)
    ref = orc.swa_bwd(host64(do), host64(q), host64(k), host64(v), 50, scale=0.07, magnitudes=True)
    _bound_check("swa bwd scale 0.07", got, ref)


def test_swa_bwd_window_one_gives_do_and_zero():
    """W = 1: o_i = v_i, so dv is the summed dO of the query heads that read
    each kv head and dq = dk = 0 (P = 1, dS = dO·v - dO·o = 0); in fp32 the
    two dot products leave residues that the magnitudes bound."""
    q, k, v, do = _inputs(1, 100, 8, 2, 64, 12)
    dq, dk, dv = _fwd_bwd(q, k, v, do, 1)
    _, _, _, mags = orc.swa_bwd(host64(do), host64(q), host64(k), host64(v), 1, magnitudes=True)
    ref_dv = host64(do).reshape(1, 100, 2, 4, 64).sum(axis=3)
    assert _ratio(host64(dv), ref_dv, mags["dv"]) <= 1.0
    assert _ratio(host64(dq), np.zeros(dq.shape), mags["dq"]) <= 1.0
    assert _ratio(host64(dk), np.zeros(dk.shape), mags["dk"]) <= 1.0


def test_swa_bwd_training_workload_sampled_blocks():
    """The training workload (8 x 4096 tokens, 32/4 heads x 64, W = 2048) in the
    launch configuration bench.py times.  dq of sampled 64-row query blocks and
    dk, dv of the first and last 64-key blocks against the oracle run on a
    slice of the sequence that holds every window those rows touch."""
    wl = WORKLOADS["train_4k"]
    inp = make_prefill_inputs(wl, device="cuda", with_scan=False)
    do = make_output_grads(wl, device="cuda", with_scan=False)["do"]
    q, k, v = inp["q"], inp["k"], inp["v"]
    dq, dk, dv = _fwd_bwd(q, k, v, do, wl.window)
    W, Ln = wl.window, wl.seqlen
    for b, i0 in ((0, 0), (3, 2048), (7, Ln - 64)):
        j0 = max(0, i0 - W + 1)
        sl = slice(j0, i0 + 64)
        rq, _, _, mags = orc.swa_bwd(host64(do[b:b + 1, sl]), host64(q[b:b + 1, sl]), host64(k[b:b + 1, sl]),
                                     host64(v[b:b + 1, sl]), W, magnitudes=True)
        ratio = _ratio(host64(dq[b:b + 1, i0:i0 + 64]), rq[:, i0 - j0:], mags["dq"][:, i0 - j0:])
        record_margin(f"swa bwd train_4k dq rows {i0}..{i0 + 63} of b{b}", "dq", worst_over_bound=ratio)
        assert ratio <= 1.0, (b, i0, ratio)
    for b, j0 in ((1, 0), (6, Ln - 64)):
        s0, s1 = max(0, j0 - W + 1), min(Ln, j0 + 63 + W)
        sl = slice(s0, s1)
        _, rk, rv, mags = orc.swa_bwd(host64(do[b:b + 1, sl]), host64(q[b:b + 1, sl]), host64(k[b:b + 1, sl]),
                                      host64(v[b:b + 1, sl]), W, magnitudes=True)
        for key, gt, rr in (("dk", dk, rk), ("dv", dv, rv)):
            a = j0 - s0
            ratio = _ratio(host64(gt[b:b + 1, j0:j0 + 64]), rr[:, a:a + 64], mags[key][:, a:a + 64])
            record_margin(f"swa bwd train_4k {key} keys {j0}..{j0 + 63} of b{b}", key, worst_over_bound=ratio)
            assert ratio <= 1.0, (key, b, j0, ratio)


@pytest.mark.parametrize("use_aux", [False, True])
def test_mixer_bwd_equals_separate_calls(use_aux):
    """samba_mixer_bwd (both backward passes, the attention's on a second
    stream when given one) against samba_selective_scan_bwd and samba_swa_bwd
    called one after the other: the attention's gradients bit for bit, the
    scan's up to the order of its atomic sums (the per-token sums over the
    state groups too, so a bf16 gradient may round one unit apart)."""
    wl = Workload("mb", 2, 300, 64, 16, 4, 8, 2, 64, 128, 61)
    inp = make_prefill_inputs(wl, device="cuda")
    gr = make_output_grads(wl, device="cuda")
    kw = dict(D=inp["D"], z=inp["z"], conv_w=inp["conv_w"], conv_b=inp["conv_b"])
    lse = torch.empty((2, 8, 300), device="cuda")
    o = ops.swa_fwd(inp["q"], inp["k"], inp["v"], 128, lse=lse)
    scan = dict(dy=gr["dy"], x=inp["x"], delta=inp["delta"], A=inp["A"], B=inp["B"], C=inp["C"], **kw)
    swa = dict(do=gr["do"], q=inp["q"], k=inp["k"], v=inp["v"], o=o, lse=lse, window=128)
    ref_scan = ops.selective_scan_bwd(**scan)
    ref_swa = ops.swa_bwd(**swa)
    aux = torch.cuda.Stream() if use_aux else None
    got_scan, got_swa = ops.mixer_bwd(scan, swa, aux_stream=aux)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    bad = []
    for name, a, b in zip(("dq", "dk", "dv"), got_swa, ref_swa):
        if not torch.equal(a, b):
            bad.append(f"{name}: max diff {float((a.float() - b.float()).abs().max()):.3e}")
    for key, ref in ref_scan.items():
        if ref is None:
            assert got_scan[key] is None
            continue
        g, r = host64(got_scan[key]), host64(ref)
        bf = 2.0 ** -7 * np.abs(r) if ref.dtype == torch.bfloat16 else 0.0  # one bf16 unit
        bound = bf + 1e-5 * (np.max(np.abs(r)) or 1.0)
        if not np.all(np.abs(g - r) <= bound):
            bad.append(f"{key}: worst {float(np.max(np.abs(g - r) / bound)):.2f} x the bound")
    assert not bad, "; ".join(bad)
