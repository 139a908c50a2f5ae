"""GPU parity of the decode path (conv1d, scan_step, ring fill, swa_step) and
the mixer prefill, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle.samba_oracle as orc
from hybrid_ssm_sliding_b200 import build as B
from hybrid_ssm_sliding_b200 import ops
from hybrid_ssm_sliding_b200.workloads import WORKLOADS, Workload, make_decode_step_inputs, make_prefill_inputs
from tests._helpers import SCAN_TOL, SWA_MAX_ABS, SWA_MEAN_ABS, host64, scan_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


# -------------------------------------------------------------------- conv1d
@pytest.mark.parametrize("dt,K,silu,state", [
    (torch.float32, 4, True, False), (torch.bfloat16, 4, True, True), (torch.float32, 3, False, True),
    (torch.bfloat16, 2, True, False),
])
def test_conv1d(dt, K, silu, state):
    wl = Workload("c", 2, 37, 24, 16, K, 1, 1, 16, 16, 30 + K, act_dtype=dt)
    inp = make_prefill_inputs(wl, device="cuda", with_attention=False)
    cs_in = torch.randn((2, 24, K - 1), device="cuda") if state else None
    cs_out = torch.empty((2, 24, K - 1), device="cuda")
    u = ops.conv1d_fwd(inp["x"], inp["conv_w"], inp["conv_b"], conv_state_in=cs_in, silu=silu,
                       u_dtype=torch.float32, conv_state_out=cs_out)
    torch.cuda.synchronize()
    ref, ref_state = orc.causal_conv1d(host64(inp["x"]), host64(inp["conv_w"]), host64(inp["conv_b"]),
                                       host64(cs_in), apply_silu=silu)
    assert scan_rel_err(host64(u), ref) <= 1e-5
    np.testing.assert_array_equal(host64(cs_out), ref_state)


def test_conv1d_short_sequence_keeps_old_state():
    wl = Workload("c", 1, 2, 8, 16, 4, 1, 1, 16, 16, 3, act_dtype=torch.float32)
    inp = make_prefill_inputs(wl, device="cuda", with_attention=False)
    cs_in = torch.randn((1, 8, 3), device="cuda")
    cs_out = torch.empty((1, 8, 3), device="cuda")
    ops.conv1d_fwd(inp["x"], inp["conv_w"], None, conv_state_in=cs_in, conv_state_out=cs_out)
    torch.cuda.synchronize()
    _, ref_state = orc.causal_conv1d(host64(inp["x"]), host64(inp["conv_w"]), None, host64(cs_in))
    np.testing.assert_array_equal(host64(cs_out), ref_state)


# ----------------------------------------------------------------- scan step
@pytest.mark.parametrize("dt,N", [(torch.float32, 16), (torch.bfloat16, 16), (torch.bfloat16, 8), (torch.float32, 4)])
def test_prefill_then_scan_steps_match_oracle(dt, N):
    wl = Workload("d", 3, 40, 32, N, 4, 1, 1, 16, 16, 50 + N, act_dtype=dt)
    inp = make_prefill_inputs(wl, device="cuda", with_attention=False)
    L1 = 25
    pre = {k: (v[:, :L1].contiguous() if k in ("x", "z", "delta", "B", "C") else v) for k, v in inp.items()}
    h = torch.empty((3, 32, N), device="cuda")
    cs = torch.empty((3, 32, 3), device="cuda")
    ops.selective_scan_fwd(pre["x"], pre["delta"], pre["A"], pre["B"], pre["C"], D=pre["D"], z=pre["z"],
                           conv_w=pre["conv_w"], conv_b=pre["conv_b"], h_final=h, conv_state_out=cs,
                           y_dtype=torch.float32)
    full = orc.selective_scan(host64(inp["x"]), host64(inp["delta"]), host64(inp["A"]), host64(inp["B"]),
                              host64(inp["C"]), host64(inp["D"]), host64(inp["z"]), conv_w=host64(inp["conv_w"]),
                              conv_b=host64(inp["conv_b"]), magnitudes=True)
    for t in range(L1, 40):
        y_t = ops.scan_step(h, cs, inp["x"][:, t].contiguous(), inp["delta"][:, t].contiguous(), inp["A"],
                            inp["B"][:, t].contiguous(), inp["C"][:, t].contiguous(), D=inp["D"],
                            z_t=inp["z"][:, t].contiguous(), conv_w=inp["conv_w"], conv_b=inp["conv_b"],
                            y_dtype=torch.float32)
        torch.cuda.synchronize()
        assert scan_rel_err(host64(y_t), full["y"][:, t], full["y_mag"][:, t]) <= SCAN_TOL
    assert scan_rel_err(host64(h), full["h"], full["h_mag"]) <= SCAN_TOL
    np.testing.assert_array_equal(host64(cs), full["conv_state"])


# ------------------------------------------------------------------ SWA step
@pytest.mark.parametrize("L1,W,Hq,Hkv,d,Bsz,poison", [
    (10, 16, 8, 2, 64, 2, False), (40, 16, 4, 4, 32, 2, False), (300, 256, 32, 4, 64, 2, False),
    (1, 700, 8, 1, 64, 2, False), (600, 300, 16, 1, 16, 2, False), (200, 150, 8, 2, 128, 2, False),
    # slots past the newest position start as NaN: they hold no position and
    # must not reach the output
    (5, 300, 8, 2, 64, 3, True), (100, 2048, 32, 4, 64, 16, True), (3, 64, 4, 1, 128, 2, True),
    # a full 2048-slot ring at the decode batch width: several splits of
    # several sub-chunks per CTA
    (2100, 2048, 32, 4, 64, 16, False),
    # one sequence over a long ring: many splits
    (9000, 8192, 8, 1, 64, 1, False),
])
def test_ring_fill_then_swa_steps_match_oracle(L1, W, Hq, Hkv, d, Bsz, poison):
    steps = 24
    g = torch.Generator(device="cuda")
    g.manual_seed(L1 + W)
    Ln = L1 + steps
    q = torch.randn((Bsz, Ln, Hq, d), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((Bsz, Ln, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((Bsz, Ln, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    kr = vr = None
    if poison:
        kr = torch.full((Bsz, W, Hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        vr = torch.full((Bsz, W, Hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    kr, vr, pos = ops.swa_ring_fill(k[:, :L1].contiguous(), v[:, :L1].contiguous(), W, k_ring=kr, v_ring=vr)
    rk, rv, rpos = orc.ring_fill(host64(k[:, :L1]), host64(v[:, :L1]), W)
    full, _ = orc.swa(host64(q), host64(k), host64(v), W)
    ws = torch.zeros((ops.swa_step_workspace_size(Bsz, Hq, d, W),), dtype=torch.uint8, device="cuda")
    for t in range(L1, Ln):
        o_t = ops.swa_step(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(), kr, vr, pos, W,
                           workspace=ws)
        torch.cuda.synchronize()
        err = np.abs(host64(o_t) - full[:, t])
        assert err.max() <= SWA_MAX_ABS and err.mean() <= SWA_MEAN_ABS
    assert torch.equal(pos.cpu(), torch.full((Bsz,), Ln, dtype=torch.int64))
    # ring contents equal the oracle's ring after the same steps
    for t in range(L1, Ln):
        _, rk, rv, rpos = orc.swa_step(host64(q[:, t]), host64(k[:, t]), host64(v[:, t]), rk, rv, rpos, W)
    keep = min(Ln, W)
    slots = [p % W for p in range(Ln - keep, Ln)]
    np.testing.assert_array_equal(host64(kr)[:, slots], rk[:, slots])
    np.testing.assert_array_equal(host64(vr)[:, slots], rv[:, slots])
    if poison and Ln < W:    # the slots never written keep their NaN
        assert torch.isnan(kr[:, Ln:].float()).all() and torch.isnan(vr[:, Ln:].float()).all()


@pytest.mark.parametrize("Bsz,Hq,Hkv,d,W,L1", [(1, 8, 2, 64, 256, 300), (2, 4, 1, 32, 64, 20), (1, 16, 4, 64, 2048, 2100)])
@pytest.mark.parametrize("graph", [False, True])
def test_back_to_back_swa_steps_on_one_ring(Bsz, Hq, Hkv, d, W, L1, graph):
    """Steps on the same ring launched one right after the other (all inputs
    prepared beforehand, nothing else on the stream in between), eagerly and
    captured in a CUDA graph: each step starts reading the ring before the
    previous one has finished, and must still see the key that step wrote."""
    steps = 40
    g = torch.Generator(device="cuda")
    g.manual_seed(Bsz * 100 + W)
    Ln = L1 + steps
    q = torch.randn((Bsz, Ln, Hq, d), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((Bsz, Ln, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((Bsz, Ln, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    kr, vr, pos = ops.swa_ring_fill(k[:, :L1].contiguous(), v[:, :L1].contiguous(), W)
    ins = [(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous()) for t in range(L1, Ln)]
    outs = [torch.empty((Bsz, Hq, d), dtype=torch.bfloat16, device="cuda") for _ in ins]
    ws = torch.empty((ops.swa_step_workspace_size(Bsz, Hq, d, W),), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()

    def run():
        for (qt, kt, vt), ot in zip(ins, outs):
            ops.swa_step(qt, kt, vt, kr, vr, pos, W, o_t=ot, workspace=ws)

    if graph:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        gr = torch.cuda.CUDAGraph()
        kr0, vr0, pos0 = kr.clone(), vr.clone(), pos.clone()
        with torch.cuda.stream(side):
            with torch.cuda.graph(gr, stream=side):
                run()
        torch.cuda.current_stream().wait_stream(side)
        kr.copy_(kr0), vr.copy_(vr0), pos.copy_(pos0)   # the capture ran nothing; restore to be safe
        gr.replay()
    else:
        run()
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    assert torch.equal(pos.cpu(), torch.full((Bsz,), Ln, dtype=torch.int64))
    full, _ = orc.swa(host64(q), host64(k), host64(v), W)
    for i, t in enumerate(range(L1, Ln)):
        err = np.abs(host64(outs[i]) - full[:, t])
        assert err.max() <= SWA_MAX_ABS and err.mean() <= SWA_MEAN_ABS, (t, err.max())


def test_swa_step_at_a_large_batch():
    """16384 sequences of one step (a grid of 65536 split CTAs): sampled
    sequences against the oracle, every pos advanced."""
    Bsz, Hq, Hkv, d, W, L1 = 16384, 8, 4, 16, 200, 150
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    k = torch.randn((Bsz, L1 + 1, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((Bsz, L1 + 1, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn((Bsz, Hq, d), generator=g, device="cuda").to(torch.bfloat16)
    kr, vr, pos = ops.swa_ring_fill(k[:, :L1].contiguous(), v[:, :L1].contiguous(), W)
    o_t = ops.swa_step(q, k[:, L1].contiguous(), v[:, L1].contiguous(), kr, vr, pos, W)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    assert torch.equal(pos.cpu(), torch.full((Bsz,), L1 + 1, dtype=torch.int64))
    for b in (0, 1, 777, 8191, 16383):
        full, _ = orc.swa(host64(q[b:b + 1, None].expand(1, L1 + 1, Hq, d).contiguous()), host64(k[b:b + 1]),
                          host64(v[b:b + 1]), W)
        err = np.abs(host64(o_t[b]) - full[0, L1])
        assert err.max() <= SWA_MAX_ABS, (b, err.max())


def test_decode_checkpoint_restore_is_bit_identical():
    """Saving the decode state (h, conv state, K/V ring, pos) and resuming
    from it reproduces the uninterrupted run bit for bit."""
    wl = Workload("ck", 2, 64, 32, 16, 4, 8, 2, 64, 32, 77, decode_steps=12)
    inp = make_prefill_inputs(wl, device="cuda")
    h = torch.empty((2, 32, 16), device="cuda")
    cs = torch.empty((2, 32, 3), device="cuda")
    ops.selective_scan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                           conv_w=inp["conv_w"], conv_b=inp["conv_b"], h_final=h, conv_state_out=cs)
    kr, vr, pos = ops.swa_ring_fill(inp["k"], inp["v"], wl.window)

    def run(state, steps):
        hh, cc, kk, vv, pp = [t.clone() for t in state]
        outs = []
        for s in steps:
            si = make_decode_step_inputs(wl, s, device="cuda")
            y = ops.scan_step(hh, cc, si["x"], si["delta"], inp["A"], si["B"], si["C"], D=inp["D"], z_t=si["z"],
                              conv_w=inp["conv_w"], conv_b=inp["conv_b"])
            o = ops.swa_step(si["q"], si["k"], si["v"], kk, vv, pp, wl.window)
            outs.append((y.clone(), o.clone()))
        return outs, (hh, cc, kk, vv, pp)

    state0 = (h, cs, kr, vr, pos)
    ref, _ = run(state0, range(12))
    first, mid = run(state0, range(5))
    saved = [t.cpu() for t in mid]                      # checkpoint to host
    restored = tuple(t.cuda() for t in saved)           # restore
    second, _ = run(restored, range(5, 12))
    for (ya, oa), (yb, ob) in zip(ref, first + second):
        assert torch.equal(ya, yb) and torch.equal(oa, ob)


# ------------------------------------------------------------- mixer prefill
@pytest.mark.parametrize("use_aux", [False, True])
def test_mixer_prefill_equals_separate_calls(use_aux):
    wl = Workload("m", 2, 777, 64, 16, 4, 32, 4, 64, 256, 31)
    inp = make_prefill_inputs(wl, device="cuda")
    scan_kw = dict(x=inp["x"], delta=inp["delta"], A=inp["A"], B=inp["B"], C=inp["C"], D=inp["D"], z=inp["z"],
                   conv_w=inp["conv_w"], conv_b=inp["conv_b"])
    swa_kw = dict(q=inp["q"], k=inp["k"], v=inp["v"], window=wl.window)
    y_ref = ops.selective_scan_fwd(**scan_kw)
    o_ref = ops.swa_fwd(**swa_kw)
    aux = torch.cuda.Stream() if use_aux else None
    y, o = ops.mixer_prefill(scan_kw, swa_kw, aux_stream=aux)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref) and torch.equal(o, o_ref)
    assert ops.get_status() == 0
