"""GPU parity of the streaming-decode workload at its own shape, through the C
ABI: 16 sequences, a 4096-token prefill (selective scan with its final state
and conv state, then the ring hand-off of the last 2048 keys/values), then
65 536 single-token steps of samba_scan_step and samba_swa_step, run in CUDA
graphs of 32 steps as bench.py runs them.

Page "SAMBA混合注意力状态空间模型", section 推理效率: generate() runs
forward(prompt) and then mamba_step / swa_step once per new token.

The float64 oracle follows the same decode on 64 of the 4096 channels (all 16
sequences): it runs the prefill and then every one of the 65 536 steps of the
recurrence, carrying (h, conv state) and the magnitudes the tolerance is
measured against.  Step t's inputs come from the generator keyed by (seed, t),
so the oracle sees exactly the values the GPU saw.  Compared:

  * y_t (fp32 output) of the 64 channels at steps 0, 1, 2047, 2048 and every
    4096th step, and the state h and conv state of those channels at the
    steps that end a 32-step graph (2047 and every 4096th step);
  * o_t of every head of every sequence at the same steps: the query attends
    the W = 2048 newest keys, which the oracle takes from the prefill and the
    stored per-step keys (attention does not depend on the order of the keys,
    so they are handed to the oracle's ring in position order);
  * pos after the last step.

Tolerances are those of the prefill tests: y and h within 1e-4 relative to
the size of the sums that produce them, the conv state exactly, o within
2e-2 max abs and 1e-2 mean abs."""

import numpy as np
import pytest
import torch

import oracle.samba_oracle as orc
from hybrid_ssm_sliding_b200 import build as B
from hybrid_ssm_sliding_b200 import ops
from hybrid_ssm_sliding_b200.workloads import WORKLOADS, make_decode_step_inputs, make_prefill_inputs
from tests._helpers import SCAN_TOL, SWA_MAX_ABS, SWA_MEAN_ABS, host64, record_margin, scan_errors

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

GRAPH_STEPS = 32


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def _channels(D, n, seed):
    g = np.random.default_rng(seed)
    ch = np.unique(np.concatenate([[0, 1, D - 1], g.choice(D, n - 3, replace=False)]))
    return ch


def test_decode_64k_matches_oracle():
    wl = WORKLOADS["decode_64k"]
    dev = torch.device("cuda")
    Bsz, L0, D, N, K, W = wl.batch, wl.seqlen, wl.dim, wl.dstate, wl.dconv, wl.window
    Hq, Hkv, d = wl.heads_q, wl.heads_kv, wl.head_dim
    steps = wl.decode_steps
    assert steps % GRAPH_STEPS == 0
    chans = _channels(D, 64, wl.seed)
    ch_t = torch.from_numpy(chans).to(dev)

    # ---------------------------------------------------------------- prefill
    pre = make_prefill_inputs(wl, device=dev)
    h = torch.full((Bsz, D, N), float("nan"), device=dev)
    cs = torch.full((Bsz, D, K - 1), float("nan"), device=dev)
    ops.selective_scan_fwd(pre["x"], pre["delta"], pre["A"], pre["B"], pre["C"], D=pre["D"], z=pre["z"],
                           conv_w=pre["conv_w"], conv_b=pre["conv_b"], h_final=h, conv_state_out=cs,
                           y_dtype=torch.bfloat16)
    k_ring, v_ring, pos = ops.swa_ring_fill(pre["k"], pre["v"], W)
    A, Dsk, cw, cb = pre["A"], pre["D"], pre["conv_w"], pre["conv_b"]
    sub = lambda t: host64(t[..., ch_t])                      # noqa: E731  channel subset, last dim
    ref = orc.selective_scan(sub(pre["x"]), sub(pre["delta"]), host64(A[ch_t]), host64(pre["B"]),
                             host64(pre["C"]), host64(Dsk[ch_t]), sub(pre["z"]), conv_w=host64(cw[ch_t]),
                             conv_b=host64(cb[ch_t]), magnitudes=True)
    torch.cuda.synchronize()
    e = scan_errors(host64(h[:, ch_t]), ref["h"], ref["h_mag"])
    assert e["rel_to_mag"] <= SCAN_TOL, f"prefill h rel err {e['rel_to_mag']:.3e}"
    np.testing.assert_array_equal(host64(cs[:, ch_t]), ref["conv_state"])
    k_pre, v_pre = pre["k"].clone(), pre["v"].clone()          # [B, L0, Hkv, d], for the early windows
    del pre

    # ------------------------------------------- decode on the GPU, in graphs
    G = GRAPH_STEPS
    shapes = make_decode_step_inputs(wl, 0, device=dev)
    slots = {k: torch.empty((G,) + tuple(v.shape), dtype=v.dtype, device=dev) for k, v in shapes.items()}
    y_slots = torch.full((G, Bsz, D), float("nan"), device=dev)
    o_slots = torch.full((G, Bsz, Hq, d), float("nan"), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros((ops.swa_step_workspace_size(Bsz, Hq, d, W),), dtype=torch.uint8, device=dev)

    def body(j):
        ops.scan_step(h, cs, slots["x"][j], slots["delta"][j], A, slots["B"][j], slots["C"][j], D=Dsk,
                      z_t=slots["z"][j], conv_w=cw, conv_b=cb, y_t=y_slots[j])
        ops.swa_step(slots["q"][j], slots["k"][j], slots["v"][j], k_ring, v_ring, pos, W, o_t=o_slots[j],
                     workspace=ws)

    # one step on a scratch copy of the state first, so that the kernels are
    # loaded and set up before the capture
    scratch = [t.clone() for t in (h, cs, k_ring, v_ring, pos)]
    ops.scan_step(scratch[0], scratch[1], shapes["x"], shapes["delta"], A, shapes["B"], shapes["C"], D=Dsk,
                  z_t=shapes["z"], conv_w=cw, conv_b=cb, y_t=y_slots[0])
    ops.swa_step(shapes["q"], shapes["k"], shapes["v"], scratch[2], scratch[3], scratch[4], W, o_t=o_slots[0],
                 workspace=ws)
    torch.cuda.synchronize()
    del scratch
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for j in range(G):
            body(j)

    y_checks = {0, 1, 2047, 2048} | {m * 4096 - 1 for m in range(1, steps // 4096 + 1)}
    state_checks = {s for s in y_checks if s % G == G - 1}
    x_all = torch.empty((steps, Bsz, len(chans)), dtype=shapes["x"].dtype, device=dev)
    z_all = torch.empty_like(x_all)
    d_all = torch.empty((steps, Bsz, len(chans)), dtype=torch.float32, device=dev)
    b_all = torch.empty((steps, Bsz, N), dtype=torch.float32, device=dev)
    c_all = torch.empty_like(b_all)
    k_all = torch.empty((steps, Bsz, Hkv, d), dtype=torch.bfloat16, device=dev)
    v_all = torch.empty_like(k_all)
    got_y, got_o, got_q, got_h, got_cs = {}, {}, {}, {}, {}
    for c0 in range(0, steps, G):
        for j in range(G):
            for key, t in make_decode_step_inputs(wl, c0 + j, device=dev).items():
                slots[key][j].copy_(t)
        graph.replay()
        sl = slice(c0, c0 + G)
        x_all[sl] = slots["x"][:, :, ch_t]
        z_all[sl] = slots["z"][:, :, ch_t]
        d_all[sl] = slots["delta"][:, :, ch_t]
        b_all[sl] = slots["B"]
        c_all[sl] = slots["C"]
        k_all[sl] = slots["k"]
        v_all[sl] = slots["v"]
        for s in range(c0, c0 + G):
            if s in y_checks:
                got_y[s] = y_slots[s - c0][:, ch_t].clone()
                got_o[s] = o_slots[s - c0].clone()
                got_q[s] = slots["q"][s - c0].clone()
            if s in state_checks:
                got_h[s] = h[:, ch_t].clone()
                got_cs[s] = cs[:, ch_t].clone()
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    del graph
    assert torch.equal(pos.cpu(), torch.full((Bsz,), L0 + steps, dtype=torch.int64))

    # ------------------------------------- the oracle over the same 65 536 steps
    xs, zs, ds = host64(x_all), host64(z_all), host64(d_all)
    bs, cs_in = host64(b_all), host64(c_all)
    A64, D64, cw64, cb64 = host64(A[ch_t]), host64(Dsk[ch_t]), host64(cw[ch_t]), host64(cb[ch_t])
    hh, hm, cst = ref["h"], ref["h_mag"], ref["conv_state"]
    worst = {"y": 0.0, "h": 0.0, "o_max": 0.0, "o_mean": 0.0}
    prev = 0
    for s in sorted(y_checks):
        seg = slice(prev, s + 1)
        tm = lambda a: np.ascontiguousarray(np.swapaxes(a[seg], 0, 1))   # noqa: E731  [steps, B, .] -> [B, steps, .]
        out = orc.selective_scan(tm(xs), tm(ds), A64, tm(bs), tm(cs_in), D64, tm(zs), h0=hh, conv_w=cw64,
                                 conv_b=cb64, conv_state=cst, magnitudes=True, h0_mag=hm)
        hh, hm, cst = out["h"], out["h_mag"], out["conv_state"]
        prev = s + 1
        ey = scan_errors(host64(got_y[s]), out["y"][:, -1], out["y_mag"][:, -1])
        assert ey["rel_to_mag"] <= SCAN_TOL, f"step {s}: y rel err {ey['rel_to_mag']:.3e}"
        worst["y"] = max(worst["y"], ey["rel_to_mag"])
        if s in state_checks:
            eh = scan_errors(host64(got_h[s]), hh, hm)
            assert eh["rel_to_mag"] <= SCAN_TOL, f"step {s}: h rel err {eh['rel_to_mag']:.3e}"
            worst["h"] = max(worst["h"], eh["rel_to_mag"])
            np.testing.assert_array_equal(host64(got_cs[s]), cst)
        # attention: keys of positions p - W + 1 .. p, p = L0 + s
        p = L0 + s
        first = p - W + 1
        ks, vs = [], []
        if first < L0:
            ks.append(host64(k_pre[:, first:L0]))
            vs.append(host64(v_pre[:, first:L0]))
        a0 = max(0, first - L0)
        ks.append(np.swapaxes(host64(k_all[a0:s]), 0, 1))
        vs.append(np.swapaxes(host64(v_all[a0:s]), 0, 1))
        kw, vw = np.concatenate(ks, 1), np.concatenate(vs, 1)                # positions first .. p - 1
        assert kw.shape[1] == W - 1
        rk, rv, rpos = orc.ring_fill(kw, vw, W)
        o_ref, _, _, _ = orc.swa_step(host64(got_q[s]), host64(k_all[s]), host64(v_all[s]), rk, rv, rpos, W)
        err = np.abs(host64(got_o[s]) - o_ref)
        assert err.max() <= SWA_MAX_ABS and err.mean() <= SWA_MEAN_ABS, \
            f"step {s}: o max abs {err.max():.3e}, mean abs {err.mean():.3e}"
        worst["o_max"] = max(worst["o_max"], err.max())
        worst["o_mean"] = max(worst["o_mean"], err.mean())
    record_margin("decode_64k (64 channels x 16 sequences, 65536 steps)", "y_t", rel_to_mag=worst["y"],
                  tol=SCAN_TOL, checks=len(y_checks))
    record_margin("decode_64k (64 channels x 16 sequences, 65536 steps)", "h", rel_to_mag=worst["h"],
                  tol=SCAN_TOL, checks=len(state_checks))
    record_margin("decode_64k (all heads, 16 sequences)", "o_t", max_abs=worst["o_max"], mean_abs=worst["o_mean"],
                  tol_max_abs=SWA_MAX_ABS, tol_mean_abs=SWA_MEAN_ABS, checks=len(y_checks))
