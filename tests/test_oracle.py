"""Pins for the float64 oracle: each check ties it to something other than
itself -- hand-worked values, closed forms, library routines on special
cases, invariants and brute force on tiny inputs.  CPU only.

A second group plants plausible mistakes in the oracle (monkeypatched, on
the CPU) and shows that some pin catches each one.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle.samba_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed=0):
    return np.random.default_rng(seed)


def _tiny_scan_inputs(seed=0, Bsz=1, L=64, D=16, N=4, K=4):
    r = _rng(seed)
    step = np.exp(r.uniform(math.log(1e-3), math.log(1e-1), size=(Bsz, L, D)))
    return dict(
        x=r.standard_normal((Bsz, L, D)),
        z=r.standard_normal((Bsz, L, D)),
        delta=np.log(np.expm1(step)),
        A=-np.tile(np.arange(1, N + 1, dtype=np.float64), (D, 1)),
        Bm=r.standard_normal((Bsz, L, N)),
        Cm=r.standard_normal((Bsz, L, N)),
        Dskip=r.standard_normal(D),
        conv_w=r.uniform(-0.5, 0.5, size=(D, K)),
        conv_b=r.uniform(-0.5, 0.5, size=D),
    )


# ----------------------------------------------------------- hand-worked values
def test_scan_handworked_golden():
    g = _load("scan_handworked.json")
    i = g["inputs"]
    out = orc.selective_scan(i["x"], i["delta"], i["A"], i["B"], i["C"], Dskip=i["D"],
                             delta_softplus=False)
    np.testing.assert_allclose(out["y"], g["expected"]["y"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(out["h"], g["expected"]["h"], rtol=0, atol=1e-13)


def test_conv_handworked_golden():
    g = _load("conv_handworked.json")
    i = g["inputs"]
    u, st = orc.causal_conv1d(i["x"], i["w"], i["bias"], None, apply_silu=False)
    np.testing.assert_allclose(u, g["expected"]["u_zero_state"], atol=1e-13)
    np.testing.assert_allclose(st, g["expected"]["state_out"], atol=1e-13)
    x3 = np.asarray(i["x"])[:, :3]
    u2, _ = orc.causal_conv1d(x3, i["w"], i["bias"], i["state"], apply_silu=False)
    np.testing.assert_allclose(u2, g["expected"]["u_with_state_first3"], atol=1e-13)


def test_swa_handworked_golden():
    g = _load("swa_handworked.json")
    i = g["inputs"]
    for fn in (orc.swa, lambda q, k, v, w: orc.swa_rows(q, k, v, w, np.arange(3))):
        o, lse = fn(i["q"], i["k"], i["v"], i["window"])
        np.testing.assert_allclose(o, g["expected"]["o"], atol=1e-13)
        np.testing.assert_allclose(lse, g["expected"]["lse"], atol=1e-13)


# ------------------------------------------------------------------ activations
def test_softplus_closed_forms():
    w = np.linspace(-40, 40, 2001)
    sp = orc.softplus(w)
    assert abs(orc.softplus(np.array([0.0]))[0] - math.log(2.0)) < 1e-15
    np.testing.assert_allclose(sp - orc.softplus(-w), w, atol=1e-12)        # sp(w) - sp(-w) = w
    # derivative is the logistic function (central differences)
    eps = 1e-5
    deriv = (orc.softplus(w + eps) - orc.softplus(w - eps)) / (2 * eps)
    np.testing.assert_allclose(deriv, scipy.special.expit(w), atol=1e-8)
    # inverse used by the input recipe: softplus(log(expm1(s))) = s
    s = np.exp(np.linspace(math.log(1e-3), math.log(1e-1), 101))
    np.testing.assert_allclose(orc.softplus(np.log(np.expm1(s))), s, rtol=1e-13)


def test_silu_closed_forms():
    x = np.linspace(-30, 30, 1201)
    y = orc.silu(x)
    assert orc.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(y - orc.silu(-x), x, atol=1e-12)              # odd part is x/2
    np.testing.assert_allclose(y, x * scipy.special.expit(x), rtol=1e-14, atol=1e-300)


# ------------------------------------------------------------------------- conv
def test_conv_matches_torch_conv1d():
    i = _tiny_scan_inputs(1, Bsz=2, L=37, D=8)
    x = torch.from_numpy(i["x"])                                              # [B, L, D]
    w = torch.from_numpy(i["conv_w"])                                         # [D, K]
    b = torch.from_numpy(i["conv_b"])
    ref = torch.nn.functional.conv1d(x.transpose(1, 2), w[:, None, :], b, padding=3,
                                     groups=x.shape[2])[..., :x.shape[1]].transpose(1, 2)
    u, _ = orc.causal_conv1d(i["x"], i["conv_w"], i["conv_b"], apply_silu=False)
    np.testing.assert_allclose(u, ref.numpy(), atol=1e-13)
    u_silu, _ = orc.causal_conv1d(i["x"], i["conv_w"], i["conv_b"], apply_silu=True)
    np.testing.assert_allclose(u_silu, torch.nn.functional.silu(ref).numpy(), atol=1e-13)


def test_conv_state_carry_equals_one_pass():
    i = _tiny_scan_inputs(2, Bsz=2, L=40, D=8)
    full, st_full = orc.causal_conv1d(i["x"], i["conv_w"], i["conv_b"])
    for cut in (1, 2, 3, 17, 39):
        a, st = orc.causal_conv1d(i["x"][:, :cut], i["conv_w"], i["conv_b"])
        b, st2 = orc.causal_conv1d(i["x"][:, cut:], i["conv_w"], i["conv_b"], st)
        np.testing.assert_allclose(np.concatenate([a, b], 1), full, atol=1e-13)
        np.testing.assert_allclose(st2, st_full, atol=0)


# ------------------------------------------------------------------------- scan
def _brute_force_scan(i, h0=None):
    """Unrolled sum, written from the definition with explicit loops:
    y_t = (C_t . sum_{s<=t} (prod_{r=s+1}^{t} exp(Δ_r A)) Δ_s B_s u_s
           + C_t . (prod_{r<=t} exp(Δ_r A)) h0 + D u_t) * silu(z_t)."""
    x, z = i["x"], i["z"]
    Bsz, L, D = x.shape
    K = i["conv_w"].shape[1]
    N = i["A"].shape[1]
    u = np.zeros_like(x)
    for b in range(Bsz):
        for t in range(L):
            for c in range(D):
                acc = i["conv_b"][c]
                for k in range(K):
                    tt = t - (K - 1) + k
                    if tt >= 0:
                        acc += i["conv_w"][c, k] * x[b, tt, c]
                u[b, t, c] = acc / (1.0 + math.exp(-acc))
    dt = np.vectorize(lambda w: math.log1p(math.exp(w)))(i["delta"])
    y = np.zeros_like(x)
    for b in range(Bsz):
        for c in range(D):
            for t in range(L):
                tot = 0.0
                for n in range(N):
                    hn = 0.0
                    if h0 is not None:
                        hn = math.exp(i["A"][c, n] * dt[b, :t + 1, c].sum()) * h0[b, c, n]
                    for s in range(t + 1):
                        decay = math.exp(i["A"][c, n] * dt[b, s + 1:t + 1, c].sum())
                        hn += decay * dt[b, s, c] * i["Bm"][b, s, n] * u[b, s, c]
                    tot += i["Cm"][b, t, n] * hn
                g = z[b, t, c] / (1.0 + math.exp(-z[b, t, c]))
                y[b, t, c] = (tot + i["Dskip"][c] * u[b, t, c]) * g
    return y


def test_scan_matches_unrolled_sum():
    i = _tiny_scan_inputs(0, L=24, D=6, N=4)
    out = orc.selective_scan(**i)
    np.testing.assert_allclose(out["y"], _brute_force_scan(i), rtol=1e-12, atol=1e-12)
    h0 = _rng(5).standard_normal((1, 6, 4))
    out = orc.selective_scan(**i, h0=h0)
    np.testing.assert_allclose(out["y"], _brute_force_scan(i, h0), rtol=1e-12, atol=1e-12)


def test_scan_A_zero_is_prefix_sum():
    i = _tiny_scan_inputs(3, Bsz=2, L=50, D=5, N=3)
    dt = np.exp(_rng(4).uniform(-5, 0, size=i["x"].shape))
    out = orc.selective_scan(i["x"], dt, np.zeros((5, 3)), i["Bm"], i["Cm"], delta_softplus=False)
    inc = (dt * i["x"])[..., None] * i["Bm"][:, :, None, :]                  # [B, L, D, N]
    h = np.cumsum(inc, axis=1)
    np.testing.assert_allclose(out["h"], h[:, -1], rtol=1e-12)
    np.testing.assert_allclose(out["y"], np.einsum("bldn,bln->bld", h, i["Cm"]), rtol=1e-12, atol=1e-12)


def test_scan_delta_zero_keeps_state():
    i = _tiny_scan_inputs(5, Bsz=2, L=20, D=4, N=4)
    h0 = _rng(6).standard_normal((2, 4, 4))
    out = orc.selective_scan(i["x"], np.zeros_like(i["x"]), i["A"], i["Bm"], i["Cm"], i["Dskip"],
                             h0=h0, delta_softplus=False)
    np.testing.assert_array_equal(out["h"], h0)
    exp_y = np.einsum("bdn,bln->bld", h0, i["Cm"]) + i["Dskip"] * i["x"]
    np.testing.assert_allclose(out["y"], exp_y, rtol=1e-13, atol=1e-13)


def test_scan_linear_in_input_and_state():
    i = _tiny_scan_inputs(7, Bsz=1, L=30, D=4, N=4)
    r = _rng(8)
    u1, u2 = r.standard_normal(i["x"].shape), r.standard_normal(i["x"].shape)
    h1, h2 = r.standard_normal((1, 4, 4)), r.standard_normal((1, 4, 4))
    a, b = 0.7, -1.9

    def run(u, h):
        o = orc.selective_scan(u, i["delta"], i["A"], i["Bm"], i["Cm"], i["Dskip"], h0=h)
        return o["y"], o["h"]

    y, h = run(a * u1 + b * u2, a * h1 + b * h2)
    ya, ha = run(u1, h1)
    yb, hb = run(u2, h2)
    np.testing.assert_allclose(y, a * ya + b * yb, atol=1e-11)
    np.testing.assert_allclose(h, a * ha + b * hb, atol=1e-11)


def test_scan_split_with_carry_equals_one_pass():
    i = _tiny_scan_inputs(9, Bsz=2, L=64, D=8, N=4)
    full = orc.selective_scan(**i)
    for cut in (1, 3, 31, 63):
        first = {k: (v[:, :cut] if k in ("x", "z", "delta", "Bm", "Cm") else v) for k, v in i.items()}
        rest = {k: (v[:, cut:] if k in ("x", "z", "delta", "Bm", "Cm") else v) for k, v in i.items()}
        a = orc.selective_scan(**first)
        b = orc.selective_scan(**rest, h0=a["h"], conv_state=a["conv_state"])
        np.testing.assert_allclose(np.concatenate([a["y"], b["y"]], 1), full["y"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(b["h"], full["h"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(b["conv_state"], full["conv_state"], atol=0)


def test_scan_magnitudes_carry_across_a_split():
    """A run split in two, the second segment started from the first one's
    state, conv state and h_mag, gives the magnitudes of one pass."""
    i = _tiny_scan_inputs(24, Bsz=2, L=50, D=8, N=4)
    full = orc.selective_scan(**i, magnitudes=True)
    for cut in (1, 17, 49):
        first = {k: (v[:, :cut] if k in ("x", "z", "delta", "Bm", "Cm") else v) for k, v in i.items()}
        rest = {k: (v[:, cut:] if k in ("x", "z", "delta", "Bm", "Cm") else v) for k, v in i.items()}
        a = orc.selective_scan(**first, magnitudes=True)
        b = orc.selective_scan(**rest, h0=a["h"], conv_state=a["conv_state"], magnitudes=True, h0_mag=a["h_mag"])
        np.testing.assert_allclose(np.concatenate([a["y_mag"], b["y_mag"]], 1), full["y_mag"], rtol=1e-12)
        np.testing.assert_allclose(b["h_mag"], full["h_mag"], rtol=1e-12)
        # without the carried magnitude the second segment restarts from |h|, which is smaller
        c = orc.selective_scan(**rest, h0=a["h"], conv_state=a["conv_state"], magnitudes=True)
        assert np.all(c["h_mag"] <= b["h_mag"] * (1 + 1e-12))


def _scan_steps_match_prefill(L1=25, L=40):
    """Prefill of L1 tokens, then L - L1 single-token steps, against one
    prefill of L tokens: True when every step output and the final state
    agree to 1e-12."""
    i = _tiny_scan_inputs(10, Bsz=2, L=L, D=8, N=4)
    full = orc.selective_scan(**i)
    pre = orc.selective_scan(**{k: (v[:, :L1] if k in ("x", "z", "delta", "Bm", "Cm") else v)
                                for k, v in i.items()})
    h, cs = pre["h"], pre["conv_state"]
    ok = True
    for t in range(L1, L):
        y_t, h, cs = orc.scan_step(h, cs, i["x"][:, t], i["delta"][:, t], i["A"], i["Bm"][:, t],
                                   i["Cm"][:, t], i["Dskip"], i["z"][:, t], i["conv_w"], i["conv_b"])
        ok = ok and np.allclose(y_t, full["y"][:, t], rtol=1e-12, atol=1e-12)
    return ok and np.allclose(h, full["h"], rtol=1e-12, atol=1e-12)


def test_scan_step_sequence_equals_prefill():
    assert _scan_steps_match_prefill()


# -------------------------------------------------------------------------- SWA
def _attn_inputs(seed, Bsz, L, Hq, Hkv, d):
    r = _rng(seed)
    return (r.standard_normal((Bsz, L, Hq, d)), r.standard_normal((Bsz, L, Hkv, d)),
            r.standard_normal((Bsz, L, Hkv, d)))


def _sdpa_causal(q, k, v):
    group = q.shape[2] // k.shape[2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(np.repeat(k, group, axis=2)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(np.repeat(v, group, axis=2)).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("W", [40, 41, 1000])
def test_swa_wide_window_is_full_causal_sdpa(W):
    q, k, v = _attn_inputs(11, 2, 40, 8, 2, 16)
    ref = _sdpa_causal(q, k, v)
    o, _ = orc.swa(q, k, v, W, block=16)
    np.testing.assert_allclose(o, ref, atol=1e-12)
    o2, _ = orc.swa_rows(q, k, v, W, np.arange(40))
    np.testing.assert_allclose(o2, ref, atol=1e-12)


def test_swa_window_one_returns_v():
    q, k, v = _attn_inputs(12, 2, 33, 4, 2, 16)
    o, lse = orc.swa(q, k, v, 1, block=8)
    np.testing.assert_allclose(o, np.repeat(v, 2, axis=2), atol=1e-14)
    s = np.einsum("blhd,blhd->bhl", q, np.repeat(k, 2, axis=2)) / 4.0
    np.testing.assert_allclose(lse, s, atol=1e-12)


@pytest.mark.parametrize("W", [1, 5, 16, 70])
def test_swa_equal_scores_give_window_mean(W):
    _, k, v = _attn_inputs(13, 1, 50, 4, 4, 8)
    q = np.zeros((1, 50, 4, 8))
    o, lse = orc.swa(q, k, v, W, block=16)
    for i in range(50):
        j0 = max(0, i - W + 1)
        np.testing.assert_allclose(o[0, i], v[0, j0:i + 1].mean(axis=0), atol=1e-13)
        np.testing.assert_allclose(lse[0, :, i], math.log(i + 1 - j0), atol=1e-13)


def test_swa_gqa_equals_mha_with_repeated_kv():
    q, k, v = _attn_inputs(14, 2, 45, 8, 2, 16)
    o, lse = orc.swa(q, k, v, 9, block=16)
    o2, lse2 = orc.swa(q, np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2), 9, block=16)
    np.testing.assert_allclose(o, o2, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, atol=1e-14)


@pytest.mark.parametrize("W", [1, 3, 16, 64])
def test_swa_matches_full_masked_softmax(W):
    q, k, v = _attn_inputs(15, 1, 64, 2, 2, 16)
    L, d = 64, 16
    o, lse = orc.swa(q, k, v, W, block=16)
    for h in range(2):
        s = q[0, :, h, :] @ k[0, :, h, :].T / math.sqrt(d)
        i, j = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
        s = np.where((j <= i) & (j > i - W), s, -np.inf)
        p = scipy.special.softmax(s, axis=1)
        np.testing.assert_allclose(o[0, :, h, :], p @ v[0, :, h, :], atol=1e-12)
        np.testing.assert_allclose(lse[0, h], scipy.special.logsumexp(s, axis=1), atol=1e-12)


def test_swa_rows_equals_blocked():
    q, k, v = _attn_inputs(16, 2, 70, 8, 2, 16)
    o, lse = orc.swa(q, k, v, 20, block=32)
    rows = np.array([0, 1, 19, 20, 21, 45, 69])
    o2, lse2 = orc.swa_rows(q, k, v, 20, rows)
    np.testing.assert_allclose(o2, o[:, rows], atol=1e-13)
    np.testing.assert_allclose(lse2, lse[:, :, rows], atol=1e-13)


@pytest.mark.parametrize("W", [1, 20, 200])
def test_swa_blocks_match_full_masked_softmax_and_sdpa(W):
    """The sampled-block form against a full L x L masked softmax (scipy) on
    every requested row, and against torch's causal SDPA when W >= L."""
    q, k, v = _attn_inputs(18, 2, 150, 8, 2, 16)
    L, group = 150, 4
    starts = [0, 37, 64, 140]           # the ramp, a ragged block, the tail clipped at L
    rows, o, lse = orc.swa_blocks(q, k, v, W, starts, block=32)
    np.testing.assert_array_equal(rows, np.concatenate([np.arange(s, min(L, s + 32)) for s in starts]))
    i, j = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
    visible = (j <= i) & (j > i - W)
    for b in range(2):
        for h in range(8):
            sc = q[b, :, h, :] @ k[b, :, h // group, :].T / 4.0
            sc = np.where(visible, sc, -np.inf)
            p = scipy.special.softmax(sc, axis=1)
            np.testing.assert_allclose(o[b, :, h, :], (p @ v[b, :, h // group, :])[rows], atol=1e-12)
            np.testing.assert_allclose(lse[b, h], scipy.special.logsumexp(sc, axis=1)[rows], atol=1e-12)
    if W >= L:
        np.testing.assert_allclose(o, _sdpa_causal(q, k, v)[:, rows], atol=1e-12)


def test_planted_swa_blocks_window_off_by_one_is_caught(monkeypatch):
    q, k, v = _attn_inputs(19, 1, 80, 4, 2, 16)
    _, good, _ = orc.swa_blocks(q, k, v, 16, [10, 50], block=16)
    monkeypatch.setattr(orc, "_visible", lambda i, j, W: (i - j >= 0) & (i - j <= W))
    _, bad, _ = orc.swa_blocks(q, k, v, 16, [10, 50], block=16)
    assert not np.allclose(good, bad, atol=1e-6)
    full = np.stack([scipy.special.softmax(np.where((np.arange(80)[None] <= r) & (np.arange(80)[None] > r - 16),
                                                    q[0, r, 0] @ k[0, :, 0].T / 4.0, -np.inf), axis=1)[0]
                     @ v[0, :, 0] for r in range(16, 26)])
    assert not np.allclose(bad[0, 6:16, 0], full, atol=1e-6)


def _swa_steps_match_prefill(L1, W):
    """Ring fill after L1 tokens, then 20 decode steps, against the banded
    prefill of L1 + 20 tokens: True when every step output agrees to 1e-12
    and pos ends at L1 + 20."""
    L = L1 + 20
    q, k, v = _attn_inputs(17, 2, L, 8, 2, 16)
    full, _ = orc.swa(q, k, v, W, block=16)
    kr, vr, pos = orc.ring_fill(k[:, :L1], v[:, :L1], W)
    ok = bool(np.all(pos == L1))
    for t in range(L1, L):
        o_t, kr, vr, pos = orc.swa_step(q[:, t], k[:, t], v[:, t], kr, vr, pos, W)
        ok = ok and np.allclose(o_t, full[:, t], atol=1e-12)
    return ok and bool(np.all(pos == L))


@pytest.mark.parametrize("L1,W", [(10, 16), (40, 16), (16, 16), (1, 4)])
def test_swa_decode_steps_equal_prefill(L1, W):
    assert _swa_steps_match_prefill(L1, W)


# ----------------------------------------------- planted mistakes are caught
def test_planted_symmetric_mask_is_caught(monkeypatch):
    """The page's literal symmetric band |i - j| <= W is non-causal."""
    monkeypatch.setattr(orc, "_visible", lambda i, j, W: np.abs(i - j) < W)
    q, k, v = _attn_inputs(18, 1, 30, 2, 2, 8)
    o, _ = orc.swa_rows(q, k, v, 1000, np.arange(30))
    assert not np.allclose(o, _sdpa_causal(q, k, v), atol=1e-6)


def test_planted_window_off_by_one_is_caught(monkeypatch):
    monkeypatch.setattr(orc, "_visible", lambda i, j, W: (i - j >= 0) & (i - j <= W))
    q, k, v = _attn_inputs(19, 1, 30, 2, 2, 8)
    o, _ = orc.swa_rows(q, k, v, 1, np.arange(30))
    assert not np.allclose(o, v, atol=1e-6)


def test_planted_scan_mistakes_are_caught(monkeypatch):
    i = _tiny_scan_inputs(20, L=12, D=3, N=2)
    ref = _brute_force_scan(i)
    good = orc.selective_scan(**i)["y"]
    assert np.allclose(good, ref, atol=1e-12)
    # (a) softplus dropped
    monkeypatch.setattr(orc, "softplus", lambda w: np.asarray(w, dtype=np.float64))
    assert not np.allclose(orc.selective_scan(**i)["y"], ref, atol=1e-6)
    monkeypatch.undo()
    # (b) SiLU after the conv dropped
    bad = orc.selective_scan(**i, conv_silu=False)["y"]
    assert not np.allclose(bad, ref, atol=1e-6)
    # (c) D skip dropped
    j = dict(i)
    j["Dskip"] = None
    assert not np.allclose(orc.selective_scan(**j)["y"], ref, atol=1e-6)
    # (d) conv taps reversed (weight[c, 0] on x_t)
    j = dict(i)
    j["conv_w"] = i["conv_w"][:, ::-1].copy()
    assert not np.allclose(orc.selective_scan(**j)["y"], ref, atol=1e-6)


# --------------------------------------------------- error-scale magnitudes
def test_scan_magnitudes_bound_the_outputs():
    i = _tiny_scan_inputs(21, Bsz=2, L=40, D=8, N=4)
    h0 = _rng(22).standard_normal((2, 8, 4))
    out = orc.selective_scan(**i, h0=h0, magnitudes=True)
    assert np.all(out["y_mag"] >= np.abs(out["y"]) * (1 - 1e-12))
    assert np.all(out["h_mag"] >= np.abs(out["h"]) * (1 - 1e-12))
    # the magnitudes do not change the outputs themselves
    plain = orc.selective_scan(**i, h0=h0)
    np.testing.assert_array_equal(plain["y"], out["y"])


def test_scan_magnitudes_equal_outputs_when_no_term_is_negative():
    """With every term of the sums non-negative (u, B, C, D > 0, no gate,
    no conv) nothing cancels and the magnitudes equal the outputs."""
    r = _rng(23)
    Bsz, L, D, N = 1, 30, 5, 4
    x = r.uniform(0.1, 2.0, (Bsz, L, D))
    dt = r.uniform(0.01, 0.3, (Bsz, L, D))
    A = -r.uniform(0.5, 3.0, (D, N))
    Bm = r.uniform(0.1, 1.0, (Bsz, L, N))
    Cm = r.uniform(0.1, 1.0, (Bsz, L, N))
    Ds = r.uniform(0.1, 1.0, D)
    out = orc.selective_scan(x, dt, A, Bm, Cm, Ds, delta_softplus=False, magnitudes=True)
    np.testing.assert_allclose(out["y_mag"], out["y"], rtol=1e-13)
    np.testing.assert_allclose(out["h_mag"], out["h"], rtol=1e-13)


# ------------------------------------------- planted mistakes in the decode steps
def test_planted_decode_window_one_too_wide_is_caught(monkeypatch):
    """W + 1 positions per query: the ring then hands the newest key twice."""
    monkeypatch.setattr(orc, "_window_positions", lambda p, W: range(max(0, p - W), p + 1))
    assert not _swa_steps_match_prefill(40, 16)


def test_planted_decode_window_one_too_narrow_is_caught(monkeypatch):
    monkeypatch.setattr(orc, "_window_positions", lambda p, W: range(max(0, p - W + 2), p + 1))
    assert not _swa_steps_match_prefill(40, 16)


def test_planted_scan_step_state_dropped_is_caught(monkeypatch):
    """A step that restarts the SSM state (h0 = None) or the conv state."""
    real = orc.selective_scan

    def no_h(x, delta, A, Bm, Cm, Dskip=None, z=None, h0=None, *rest, **kw):
        return real(x, delta, A, Bm, Cm, Dskip, z, None if x.shape[1] == 1 else h0, *rest, **kw)

    monkeypatch.setattr(orc, "selective_scan", no_h)
    assert not _scan_steps_match_prefill()
    monkeypatch.undo()

    def no_conv_state(x, delta, A, Bm, Cm, Dskip=None, z=None, h0=None, conv_w=None, conv_b=None,
                      conv_state=None, *rest, **kw):
        return real(x, delta, A, Bm, Cm, Dskip, z, h0, conv_w, conv_b,
                    None if x.shape[1] == 1 else conv_state, *rest, **kw)

    monkeypatch.setattr(orc, "selective_scan", no_conv_state)
    assert not _scan_steps_match_prefill()
    monkeypatch.undo()
    assert _scan_steps_match_prefill()


# ------------------------------------------------------------------ layers
def test_round_bf16_matches_torch_conversion():
    r = _rng(30)
    vals = np.concatenate([r.standard_normal(4000) * 10.0 ** r.integers(-8, 8, 4000),
                           1.0 + np.arange(64) * 2.0 ** -8])          # exact ties included
    ref = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(orc.round_bf16(vals), ref)


def _layer_weights(seed, dm=24, D=16, N=4, K=4, R=3):
    r = _rng(seed)
    return dict(in_proj=r.standard_normal((2 * D, dm)) / 5, conv_w=r.uniform(-0.5, 0.5, (D, K)),
                conv_b=r.uniform(-0.5, 0.5, D), x_proj=r.standard_normal((R + 2 * N, D)) / 4,
                dt_proj=r.standard_normal((D, R)) / 2, dt_bias=r.uniform(-6.9, -2.3, D),
                A=-np.tile(np.arange(1, N + 1, dtype=np.float64), (D, 1)), Dskip=r.standard_normal(D),
                out_proj=r.standard_normal((dm, D)) / 4)


def _mamba_layer_by_torch(h, w):
    """The same layer from torch.nn.functional (linear, conv1d) in float64 and
    the oracle's scan: pins the weight layouts and the column ranges."""
    F = torch.nn.functional
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))  # noqa: E731
    D, N, R = w["A"].shape[0], w["A"].shape[1], w["dt_proj"].shape[1]
    ht = t(h)
    x = F.linear(ht, t(w["in_proj"][:D]))
    z = F.linear(ht, t(w["in_proj"][D:]))
    K = w["conv_w"].shape[1]
    u = F.conv1d(x.transpose(1, 2), t(w["conv_w"])[:, None, :], t(w["conv_b"]), padding=K - 1, groups=D)
    u = F.silu(u[..., :x.shape[1]]).transpose(1, 2)
    dt_low = F.linear(u, t(w["x_proj"][:R]))
    Bm = F.linear(u, t(w["x_proj"][R:R + N]))
    Cm = F.linear(u, t(w["x_proj"][R + N:]))
    delta = F.linear(dt_low, t(w["dt_proj"]), t(w["dt_bias"]))
    sc = orc.selective_scan(u.numpy(), delta.numpy(), w["A"], Bm.numpy(), Cm.numpy(), w["Dskip"], z.numpy())
    return F.linear(t(sc["y"]), t(w["out_proj"])).numpy()


def test_mamba_layer_matches_torch_functional_composition():
    w = _layer_weights(31)
    h = _rng(32).standard_normal((2, 30, 24))
    got = orc.mamba_layer(h, bf16_activations=False, **w)["out"]
    np.testing.assert_allclose(got, _mamba_layer_by_torch(h, w), rtol=1e-11, atol=1e-11)


def test_planted_swapped_b_and_c_ranges_are_caught(monkeypatch):
    w = _layer_weights(33)
    h = _rng(34).standard_normal((1, 20, 24))
    real = orc.selective_scan

    def swapped(x, delta, A, Bm, Cm, *a, **k):
        return real(x, delta, A, Cm, Bm, *a, **k)

    monkeypatch.setattr(orc, "selective_scan", swapped)
    got = orc.mamba_layer(h, bf16_activations=False, **w)["out"]
    monkeypatch.undo()
    assert not np.allclose(got, _mamba_layer_by_torch(h, w), atol=1e-6)


def test_swa_layer_matches_torch_functional_composition():
    r = _rng(35)
    dm, Hq, Hkv, d, L = 32, 4, 2, 8, 40
    qkv = r.standard_normal(((Hq + 2 * Hkv) * d, dm)) / 5
    o_proj = r.standard_normal((dm, Hq * d)) / 5
    h = r.standard_normal((2, L, dm))
    got = orc.swa_layer(h, qkv, o_proj, Hq, Hkv, d, L, bf16_activations=False)["out"]   # W = L: causal
    F = torch.nn.functional
    ht, W = torch.from_numpy(h), torch.from_numpy(qkv)
    q = F.linear(ht, W[:Hq * d]).reshape(2, L, Hq, d).transpose(1, 2)
    k = F.linear(ht, W[Hq * d:(Hq + Hkv) * d]).reshape(2, L, Hkv, d).repeat_interleave(Hq // Hkv, 2).transpose(1, 2)
    v = F.linear(ht, W[(Hq + Hkv) * d:]).reshape(2, L, Hkv, d).repeat_interleave(Hq // Hkv, 2).transpose(1, 2)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(2, L, Hq * d)
    ref = F.linear(o, torch.from_numpy(o_proj)).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("bf16", [False, True])
def test_mamba_layer_step_continues_the_layer_prefill(bf16):
    """Decoding one token is the prefill of one more position: the layer
    prefill over L tokens, then s steps from its final states, reproduce the
    prefill over L + s tokens (a prefill pinned above against torch's
    functional layers)."""
    w = _layer_weights(41)
    h = _rng(42).standard_normal((2, 13, 24))
    L0 = 9
    pre = orc.mamba_layer(h[:, :L0], bf16_activations=bf16, **w)
    full = orc.mamba_layer(h, bf16_activations=bf16, **w)
    hs, cs = pre["h"], pre["conv_state"]
    for t in range(L0, h.shape[1]):
        out, hs, cs = orc.mamba_layer_step(h[:, t], h=hs, conv_state=cs, bf16_activations=bf16, **w)
        np.testing.assert_allclose(out, full["out"][:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hs, full["h"], rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(cs, full["conv_state"])


def test_planted_step_without_conv_state_is_caught():
    w = _layer_weights(43)
    h = _rng(44).standard_normal((1, 6, 24))
    pre = orc.mamba_layer(h[:, :5], bf16_activations=False, **w)
    full = orc.mamba_layer(h, bf16_activations=False, **w)
    out, _, _ = orc.mamba_layer_step(h[:, 5], h=pre["h"], conv_state=np.zeros_like(pre["conv_state"]),
                                     bf16_activations=False, **w)
    assert not np.allclose(out, full["out"][:, 5], atol=1e-6)


@pytest.mark.parametrize("W", [1, 5, 40])
def test_swa_layer_step_continues_the_layer_prefill(W):
    r = _rng(45 + W)
    dm, Hq, Hkv, d, L = 32, 4, 2, 8, 17
    qkv = r.standard_normal(((Hq + 2 * Hkv) * d, dm)) / 5
    o_proj = r.standard_normal((dm, Hq * d)) / 5
    h = r.standard_normal((2, L, dm))
    L0 = 11
    pre = orc.swa_layer(h[:, :L0], qkv, o_proj, Hq, Hkv, d, W)
    full = orc.swa_layer(h, qkv, o_proj, Hq, Hkv, d, W)
    kr, vr, pos = orc.ring_fill(pre["k"], pre["v"], W)
    for t in range(L0, L):
        out, kr, vr, pos = orc.swa_layer_step(h[:, t], qkv, o_proj, Hq, Hkv, d, kr, vr, pos, W)
        np.testing.assert_allclose(out, full["out"][:, t], rtol=1e-12, atol=1e-12)
    assert np.all(pos == L)


# ----------------------------------------------------------------- backward
def _scan_bwd_inputs(seed, Bsz=2, L=7, D=3, N=2, K=4):
    r = _rng(seed)
    return {
        "x": r.standard_normal((Bsz, L, D)), "delta": r.standard_normal((Bsz, L, D)) * 0.7 - 1.0,
        "A": -r.uniform(0.2, 2.0, (D, N)), "Bm": r.standard_normal((Bsz, L, N)), "Cm": r.standard_normal((Bsz, L, N)),
        "Dskip": r.standard_normal(D), "z": r.standard_normal((Bsz, L, D)), "h0": r.standard_normal((Bsz, D, N)),
        "conv_w": r.standard_normal((D, K)) * 0.5, "conv_b": r.standard_normal(D) * 0.3,
        "conv_state": r.standard_normal((Bsz, D, K - 1)),
    }


_SCAN_GRAD_OF = {"x": "dx", "delta": "ddelta", "A": "dA", "Bm": "dB", "Cm": "dC", "Dskip": "dD", "z": "dz",
                 "h0": "dh0", "conv_w": "dconv_w", "conv_b": "dconv_b", "conv_state": "dconv_state"}


@pytest.mark.parametrize("name", list(_SCAN_GRAD_OF))
def test_scan_bwd_matches_central_differences(name):
    """Directional derivative of <dy, y> along a random direction, by central
    differences in float64, equals <gradient, direction> (brute force, no
    shared derivation)."""
    inp = _scan_bwd_inputs(40)
    r = _rng(41)
    dy = r.standard_normal(inp["x"].shape)
    g = orc.selective_scan_bwd(dy, **inp)[_SCAN_GRAD_OF[name]]
    direction = r.standard_normal(np.shape(inp[name]))
    eps = 1e-6

    def f(sign):
        args = dict(inp)
        args[name] = inp[name] + sign * eps * direction
        return float(np.sum(dy * orc.selective_scan(**args)["y"]))

    fd = (f(1) - f(-1)) / (2 * eps)
    an = float(np.sum(g * direction))
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (name, fd, an)


def test_scan_bwd_matches_torch_autograd():
    """All gradients against torch autograd of the same recurrence written
    with plain torch operations in float64."""
    inp = _scan_bwd_inputs(42, Bsz=2, L=12, D=5, N=3)
    dy = _rng(43).standard_normal(inp["x"].shape)
    got = orc.selective_scan_bwd(dy, **inp)
    t = {k: torch.tensor(v, requires_grad=True) for k, v in inp.items()}
    F = torch.nn.functional
    Bsz, L, D = inp["x"].shape
    K = inp["conv_w"].shape[1]
    xpad = torch.cat([t["conv_state"].transpose(1, 2), t["x"]], dim=1)
    pre = F.conv1d(xpad.transpose(1, 2), t["conv_w"][:, None, :], t["conv_b"], groups=D).transpose(1, 2)
    u = F.silu(pre)
    dt = F.softplus(t["delta"])
    h = t["h0"]
    ys = []
    for s in range(L):
        h = torch.exp(dt[:, s, :, None] * t["A"]) * h + (dt[:, s] * u[:, s])[:, :, None] * t["Bm"][:, s, None, :]
        ys.append((h * t["Cm"][:, s, None, :]).sum(-1))
    y = (torch.stack(ys, 1) + t["Dskip"] * u) * F.silu(t["z"])
    y.backward(torch.from_numpy(dy))
    for name, key in _SCAN_GRAD_OF.items():
        np.testing.assert_allclose(got[key], t[name].grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=name)


def test_scan_bwd_without_conv_gate_or_skip():
    """Optional parts absent: the gradient of y = C·h alone, against autograd."""
    inp = _scan_bwd_inputs(44, Bsz=1, L=9, D=4, N=3)
    dy = _rng(45).standard_normal(inp["x"].shape)
    got = orc.selective_scan_bwd(dy, inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], delta_softplus=False)
    assert got["dz"] is None and got["dD"] is None and got["dconv_w"] is None
    t = {k: torch.tensor(inp[k], requires_grad=True) for k in ("x", "delta", "A", "Bm", "Cm")}
    h = torch.zeros((1, 4, 3), dtype=torch.float64)
    ys = []
    for s in range(9):
        h = torch.exp(t["delta"][:, s, :, None] * t["A"]) * h + (t["delta"][:, s] * t["x"][:, s])[:, :, None] * t["Bm"][:, s, None, :]
        ys.append((h * t["Cm"][:, s, None, :]).sum(-1))
    torch.stack(ys, 1).backward(torch.from_numpy(dy))
    for name, key in (("x", "dx"), ("delta", "ddelta"), ("A", "dA"), ("Bm", "dB"), ("Cm", "dC")):
        np.testing.assert_allclose(got[key], t[name].grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=name)


def test_scan_bwd_zero_step_closed_form():
    """Δ = 0 (no softplus): the state never changes and y_t = C_t·h0, so
    dC_t = Σ_c dy_t,c h0_c, dh0 = Σ_t dy_t ⊗ C_t, dA = 0, dB = 0 and dx = 0."""
    r = _rng(46)
    Bsz, L, D, N = 2, 6, 3, 4
    h0 = r.standard_normal((Bsz, D, N))
    Bm, Cm, dy = r.standard_normal((Bsz, L, N)), r.standard_normal((Bsz, L, N)), r.standard_normal((Bsz, L, D))
    got = orc.selective_scan_bwd(dy, r.standard_normal((Bsz, L, D)), np.zeros((Bsz, L, D)), -np.ones((D, N)), Bm, Cm,
                                 h0=h0, delta_softplus=False)
    np.testing.assert_allclose(got["dC"], np.einsum("bld,bdn->bln", dy, h0), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dh0"], np.einsum("bld,bln->bdn", dy, Cm), rtol=1e-12, atol=1e-12)
    for key in ("dA", "dB", "dx"):
        assert np.all(got[key] == 0), key


def _swa_bwd_inputs(seed, Bsz=1, L=11, Hq=4, Hkv=2, d=3):
    r = _rng(seed)
    return (r.standard_normal((Bsz, L, Hq, d)), r.standard_normal((Bsz, L, Hkv, d)),
            r.standard_normal((Bsz, L, Hkv, d)), r.standard_normal((Bsz, L, Hq, d)))


@pytest.mark.parametrize("W", [1, 3, 5, 100])
@pytest.mark.parametrize("which", [0, 1, 2])
def test_swa_bwd_matches_central_differences(W, which):
    q, k, v, do = _swa_bwd_inputs(50 + W)
    grads = orc.swa_bwd(do, q, k, v, W, block=4)
    args = [q, k, v]
    direction = _rng(60 + which).standard_normal(args[which].shape)
    eps = 1e-6

    def f(sign):
        a = list(args)
        a[which] = args[which] + sign * eps * direction
        return float(np.sum(do * orc.swa(a[0], a[1], a[2], W)[0]))

    fd = (f(1) - f(-1)) / (2 * eps)
    an = float(np.sum(grads[which] * direction))
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (W, which, fd, an)


@pytest.mark.parametrize("W", [1, 4, 17, 64])
def test_swa_bwd_matches_torch_autograd_of_masked_softmax(W):
    q, k, v, do = _swa_bwd_inputs(70 + W, Bsz=2, L=40, Hq=6, Hkv=2, d=8)
    dq, dk, dv = orc.swa_bwd(do, q, k, v, W, block=16)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    g = 3
    i = torch.arange(40)[:, None]
    j = torch.arange(40)[None, :]
    mask = (i - j >= 0) & (i - j < W)
    s = torch.einsum("bihd,bjhd->bhij", tq, tk.repeat_interleave(g, 2)) / math.sqrt(8)
    p = torch.softmax(s.masked_fill(~mask, float("-inf")), dim=-1)
    o = torch.einsum("bhij,bjhd->bihd", p, tv.repeat_interleave(g, 2))
    o.backward(torch.from_numpy(do))
    for got, ref in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, ref.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_swa_bwd_window_one_closed_form():
    """W = 1: o_i = v_i, so dv = the dO of the query heads that read each kv
    head summed, and dq = dk = 0."""
    q, k, v, do = _swa_bwd_inputs(80, Bsz=2, L=9, Hq=6, Hkv=3, d=4)
    dq, dk, dv = orc.swa_bwd(do, q, k, v, 1)
    np.testing.assert_allclose(dv, do.reshape(2, 9, 3, 2, 4).sum(axis=3), rtol=1e-12, atol=1e-12)
    assert np.all(dq == 0) and np.all(dk == 0)


def test_planted_swa_bwd_without_row_correction_is_caught():
    """A backward that drops the Σ P dP term of dS fails the same
    central-difference check that the oracle passes."""
    q, k, v, do = _swa_bwd_inputs(81)
    W = 5
    direction = _rng(82).standard_normal(q.shape)
    eps = 1e-6
    fd = (np.sum(do * orc.swa(q + eps * direction, k, v, W)[0]) -
          np.sum(do * orc.swa(q - eps * direction, k, v, W)[0])) / (2 * eps)
    good = orc.swa_bwd(do, q, k, v, W)[0]
    bad = _swa_bwd_dq_without_correction(do, q, k, v, W)
    assert abs(fd - np.sum(good * direction)) <= 1e-7 * max(1.0, abs(fd))
    assert abs(fd - np.sum(bad * direction)) > 1e-3 * max(1.0, abs(fd))


def _swa_bwd_dq_without_correction(do, q, k, v, W):
    """dq of a backward with dS = P ⊙ dP (the Σ P dP term dropped): the
    planted mistake for the test above, written out here so the oracle itself
    is not modified."""
    Bsz, L, Hq, d = q.shape
    group = Hq // k.shape[2]
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q)
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    mask = (i - j >= 0) & (i - j < W)
    for h in range(Hq):
        s = np.where(mask, np.einsum("bid,bjd->bij", q[:, :, h], k[:, :, h // group]) * scale, -np.inf)
        p = np.exp(s - s.max(axis=2, keepdims=True))
        p /= p.sum(axis=2, keepdims=True)
        dp = np.einsum("bid,bjd->bij", do[:, :, h], v[:, :, h // group])
        dq[:, :, h] = scale * np.einsum("bij,bjd->bid", p * dp, k[:, :, h // group])
    return dq


def test_swa_bwd_magnitudes_bound_the_gradients():
    """The magnitudes are sums of absolute values of the terms of each
    gradient, so they bound it (triangle inequality), and the gradients they
    come with are unchanged."""
    q, k, v, do = _swa_bwd_inputs(90, Bsz=2, L=30, Hq=4, Hkv=2, d=5)
    plain = orc.swa_bwd(do, q, k, v, 7, block=8)
    dq, dk, dv, mag = orc.swa_bwd(do, q, k, v, 7, block=8, magnitudes=True)
    for g, p_, key in ((dq, plain[0], "dq"), (dk, plain[1], "dk"), (dv, plain[2], "dv")):
        np.testing.assert_array_equal(g, p_)
        assert np.all(mag[key] >= np.abs(g) * (1 - 1e-12)), key


def test_swa_bwd_magnitudes_by_brute_force():
    """Each magnitude against explicit loops over (query, key) pairs on a tiny
    case, with P, dS and the size of o written out from their definitions."""
    q, k, v, do = _swa_bwd_inputs(91, Bsz=1, L=6, Hq=2, Hkv=1, d=3)
    W, sc = 3, 1.0 / math.sqrt(3)
    _, _, _, mag = orc.swa_bwd(do, q, k, v, W, magnitudes=True)
    mq, mk, mv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for h in range(2):
        for i in range(6):
            js = [j for j in range(6) if 0 <= i - j < W]
            s = np.array([q[0, i, h] @ k[0, j, 0] * sc for j in js])
            p = np.exp(s - s.max())
            p /= p.sum()
            omag = sum(pj * np.abs(v[0, j, 0]) for pj, j in zip(p, js))
            dmag = float(np.abs(do[0, i, h]) @ omag)
            dp = np.array([do[0, i, h] @ v[0, j, 0] for j in js])
            ds = p * (dp - p @ dp)
            for a, j in enumerate(js):
                mv[0, j, 0] += p[a] * np.abs(do[0, i, h])
                w = abs(ds[a]) + p[a] * dmag
                mq[0, i, h] += sc * w * np.abs(k[0, j, 0])
                mk[0, j, 0] += sc * w * np.abs(q[0, i, h])
    for key, ref in (("dq", mq), ("dk", mk), ("dv", mv)):
        np.testing.assert_allclose(mag[key], ref, rtol=1e-12, atol=1e-14, err_msg=key)
