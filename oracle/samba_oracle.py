"""Float64 CPU oracle for Samba's two token mixers (test infrastructure only).

This module is the slow, plain reference that the CUDA library is checked
against.  It is test infrastructure: only the test suite, the smoke check in
``__graft_entry__`` and the ``cpu_baseline`` / reference leg of ``bench.py``
may import it.  It shares no code, constants or helpers with the CUDA path,
and the CUDA path never imports it.

Sources (pages on Samba, "Samba: Simple Hybrid State Space Models for
Efficient Unlimited Context Language Modeling", Ren et al.):

* "SAMBA混合注意力状态空间模型" (metaphor-xennon.pages.dev), section
  "数学框架 / Mamba层": the selective recurrence h_t = Ā_t h_{t-1} + B̄_t x_t,
  y_t = C_t h_t, with B_t, C_t and Δ_t = τ_Δ(Linear_Δ(x_t)) depending on the
  input (the selective-parameter equation that follows it).
* same page, section "滑动窗口注意力": softmax(Q Kᵀ / √d_k + M) V with a
  window mask M.
* same page, section "推理效率": the prefill ``forward`` followed by
  ``mamba_step`` / ``swa_step`` decoding.
* hackernoon page, §2.1.2 "Sliding Window Attention (SWA) Layer": a window
  that slides over the sequence (w = 2048 in the paper).

Readings taken where the pages are silent or garbled (each one is listed in
the design notes as well):

* Discretisation: Ā = exp(Δ·A) with a diagonal real A (one value per
  channel and state), B̄·x = Δ·B·x.  The pages write Ā_t and B̄_t without a
  formula; this is the zero-order-hold decay with an Euler input term of the
  Mamba layer the paper builds on.
* τ_Δ = softplus, applied to the raw per-channel input ``delta`` when
  ``delta_softplus`` is set; no bias is added.
* In front of the scan: a depthwise causal conv1d of width K (K = 4) with a
  bias, followed by SiLU when ``conv_silu`` is set.  The scan input u is the
  conv output.
* Output: y = (C_t · h_t + D ⊙ u_t) ⊙ silu(z_t); the D skip and the z gate are
  optional.
* One group for B and C: B_t, C_t have N entries shared by all channels.
* Window mask: key j is visible to query i exactly when 0 <= i - j < W
  (causal, W keys including the query itself).  The page writes the mask
  inverted and symmetric (|i - j| > W ↦ 0, else -inf); that cannot be meant
  literally, since it would attend only to far-away keys.
* Grouped-query attention: query head h reads key/value head
  h // (H_q / H_kv).
* Softmax scale 1/√d_k, as on the page.

Every function works in float64.  Parity unpinned: none (each function has a
pin in ``tests/test_oracle.py``).
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "softplus",
    "silu",
    "causal_conv1d",
    "selective_scan",
    "swa",
    "swa_rows",
    "swa_blocks",
    "selective_scan_bwd",
    "swa_bwd",
    "round_bf16",
    "mamba_layer",
    "swa_layer",
    "scan_step",
    "swa_step",
    "ring_fill",
    "mamba_layer_step",
    "swa_layer_step",
]


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------- activations
def softplus(w):
    """τ_Δ = softplus(w) = log(1 + e^w), written to stay exact for large |w|.

    Page "SAMBA混合注意力状态空间模型", §数学框架 / Mamba层, the selective-
    parameter equation Δ_t = τ_Δ(Linear_Δ(x_t)).
    """
    w = _f64(w)
    out = np.empty_like(w)
    pos = w > 0
    out[pos] = w[pos] + np.log1p(np.exp(-w[pos]))
    out[~pos] = np.log1p(np.exp(w[~pos]))
    return out


def silu(x):
    """SiLU / swish: x · σ(x) = x / (1 + e^{-x}).

    The page's training configuration names "swish" (SiLU) as the activation.
    """
    x = _f64(x)
    return x / (1.0 + np.exp(-x))


# ----------------------------------------------------------------------- conv
def causal_conv1d(x, weight, bias=None, state=None, apply_silu=True):
    """Depthwise causal conv1d over time, channel-last.

    u[b, t, c] = bias[c] + sum_{k=0}^{K-1} weight[c, k] * xpad[b, t + k, c]

    where xpad is x with K-1 earlier inputs in front of it: ``state`` (shape
    [B, D, K-1], oldest first) when given, else zeros.  weight[c, K-1] thus
    multiplies x_t itself.  Returns (u, new_state) with new_state the last
    K-1 inputs of xpad, i.e. the state a following call continues from.

    x: [B, L, D]; weight: [D, K]; bias: [D] or None.
    """
    x = _f64(x)
    weight = _f64(weight)
    Bsz, L, D = x.shape
    K = weight.shape[1]
    if state is None:
        state = np.zeros((Bsz, D, K - 1))
    state = _f64(state)
    xpad = np.concatenate([np.transpose(state, (0, 2, 1)), x], axis=1)  # [B, L+K-1, D]
    u = np.zeros((Bsz, L, D))
    for k in range(K):
        u += weight[None, None, :, k] * xpad[:, k:k + L, :]
    if bias is not None:
        u += _f64(bias)[None, None, :]
    if apply_silu:
        u = silu(u)
    new_state = np.transpose(xpad[:, L:L + K - 1, :], (0, 2, 1)).copy()
    return u, new_state


# ----------------------------------------------------------------------- scan
def selective_scan(x, delta, A, Bm, Cm, Dskip=None, z=None, h0=None,
                   conv_w=None, conv_b=None, conv_state=None,
                   delta_softplus=True, conv_silu=True, magnitudes=False, h0_mag=None):
    """Selective SSM prefill, sequential in time.

    Page "SAMBA混合注意力状态空间模型", §数学框架 / Mamba层:
        h_t = Ā_t h_{t-1} + B̄_t x_t,   y_t = C_t h_t
    with, per channel c and state n (readings in the module docstring):
        Δ[t, c]      = softplus(delta[t, c])          (if delta_softplus)
        Ā[t, c, n]   = exp(Δ[t, c] * A[c, n])
        B̄x[t, c, n]  = Δ[t, c] * B[t, n] * u[t, c]
        y[t, c]      = (sum_n C[t, n] h[t, c, n] + D[c] u[t, c]) * silu(z[t, c])
    where u = SiLU(conv1d(x)) if conv_w is given, else u = x.

    Shapes: x, delta, z: [B, L, D]; A: [D, N]; Bm, Cm: [B, L, N]; Dskip: [D];
    h0: [B, D, N]; conv_w: [D, K]; conv_b: [D]; conv_state: [B, D, K-1].
    Returns dict(y [B, L, D], h [B, D, N], conv_state [B, D, K-1] or None).

    With ``magnitudes`` the dict also holds y_mag and h_mag: the same
    recurrence run on the absolute values of its terms,
        hm_t = Ā_t hm_{t-1} + |B̄x_t|,   y_mag = (sum_n |C| hm + |D u|) |silu(z)|
    (Ā > 0), i.e. the size of the sums that produce y and h.  Rounding error
    of a finite-precision evaluation scales with these, not with |y|, which
    can be far smaller through cancellation; the tests measure relative
    error against them.  The magnitudes start from ``h0_mag`` (the h_mag of
    an earlier segment, [B, D, N]) when it is given, else from |h0|, so that
    a run split into segments carries its magnitudes like its state.
    """
    x = _f64(x)
    delta = _f64(delta)
    A = _f64(A)
    Bm = _f64(Bm)
    Cm = _f64(Cm)
    Bsz, L, D = x.shape
    N = A.shape[1]

    if conv_w is not None:
        u, conv_state_out = causal_conv1d(x, conv_w, conv_b, conv_state, apply_silu=conv_silu)
    else:
        u, conv_state_out = x, None
    dt = softplus(delta) if delta_softplus else delta

    h = np.zeros((Bsz, D, N)) if h0 is None else _f64(h0).copy()
    y = np.empty((Bsz, L, D))
    if magnitudes:
        hm = np.abs(h) if h0_mag is None else _f64(h0_mag).copy()
        ym = np.empty((Bsz, L, D))
    for t in range(L):
        dA = np.exp(dt[:, t, :, None] * A[None, :, :])                       # [B, D, N]
        dBx = (dt[:, t, :] * u[:, t, :])[:, :, None] * Bm[:, t, None, :]      # [B, D, N]
        h = dA * h + dBx
        y[:, t, :] = np.einsum("bdn,bn->bd", h, Cm[:, t, :])
        if magnitudes:
            hm = dA * hm + np.abs(dBx)
            ym[:, t, :] = np.einsum("bdn,bn->bd", hm, np.abs(Cm[:, t, :]))
    if Dskip is not None:
        y = y + _f64(Dskip)[None, None, :] * u
        if magnitudes:
            ym = ym + np.abs(_f64(Dskip)[None, None, :] * u)
    if z is not None:
        y = y * silu(z)
        if magnitudes:
            ym = ym * np.abs(silu(z))
    out = {"y": y, "h": h, "conv_state": conv_state_out}
    if magnitudes:
        out["y_mag"] = ym
        out["h_mag"] = hm
    return out


def scan_step(h, conv_state, x_t, delta_t, A, B_t, C_t, Dskip=None, z_t=None,
              conv_w=None, conv_b=None, delta_softplus=True, conv_silu=True):
    """One decoding step of the selective scan (``mamba_step`` on the page's
    §推理效率 pseudo-code): the recurrence of ``selective_scan`` with L = 1,
    carrying the SSM state h [B, D, N] and the conv state [B, D, K-1].

    x_t, delta_t, z_t: [B, D]; B_t, C_t: [B, N].  Returns (y_t, h, conv_state).
    """
    out = selective_scan(_f64(x_t)[:, None, :], _f64(delta_t)[:, None, :], A,
                         _f64(B_t)[:, None, :], _f64(C_t)[:, None, :], Dskip,
                         None if z_t is None else _f64(z_t)[:, None, :], h,
                         conv_w, conv_b, conv_state, delta_softplus, conv_silu)
    return out["y"][:, 0, :], out["h"], out["conv_state"]


# ------------------------------------------------------------------------ SWA
def _visible(i, j, window):
    """Band mask of the sliding window: key j is visible to query i."""
    return (i - j >= 0) & (i - j < window)


def swa_rows(q, k, v, window, rows, scale=None):
    """Sliding-window attention for the query rows ``rows`` only.

    Page "SAMBA混合注意力状态空间模型", §滑动窗口注意力:
        o_i = sum_j softmax_j(q_i · k_j / √d_k + M_ij) v_j
    with M_ij = 0 for visible keys (0 <= i - j < W) and -inf otherwise, and
    query head h reading kv head h // (H_q / H_kv).

    q: [B, L, Hq, d]; k, v: [B, L, Hkv, d].  Returns (o [B, R, Hq, d],
    lse [B, Hq, R]) for the R requested rows (natural-log logsumexp of the
    scaled scores).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    Bsz, L, Hq, d = q.shape
    Hkv = k.shape[2]
    group = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rows = np.asarray(rows, dtype=np.int64)
    R = rows.shape[0]
    o = np.zeros((Bsz, R, Hq, d))
    lse = np.zeros((Bsz, Hq, R))
    every_key = np.arange(L)
    for r, i in enumerate(rows):
        js = every_key[_visible(int(i), every_key, window)]
        for h in range(Hq):
            kv = h // group
            s = np.einsum("bd,bjd->bj", q[:, i, h, :], k[:, js, kv, :]) * scale   # [B, J]
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            den = p.sum(axis=1, keepdims=True)
            o[:, r, h, :] = np.einsum("bj,bjd->bd", p / den, v[:, js, kv, :])
            lse[:, h, r] = (m + np.log(den))[:, 0]
    return o, lse


def swa(q, k, v, window, scale=None, block=64):
    """Sliding-window attention over all rows, processed per query block with
    the banded slice of keys each block needs (same definition as swa_rows).

    Returns (o [B, L, Hq, d], lse [B, Hq, L]).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    Bsz, L, Hq, d = q.shape
    Hkv = k.shape[2]
    group = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = np.zeros((Bsz, L, Hq, d))
    lse = np.zeros((Bsz, Hq, L))
    for i0 in range(0, L, block):
        i1 = min(L, i0 + block)
        j0 = max(0, i0 - window + 1)
        ii = np.arange(i0, i1)[:, None]
        jj = np.arange(j0, i1)[None, :]
        mask = _visible(ii, jj, window)                                     # [I, J]
        for h in range(Hq):
            kv = h // group
            s = np.einsum("bid,bjd->bij", q[:, i0:i1, h, :], k[:, j0:i1, kv, :]) * scale
            s = np.where(mask[None], s, -np.inf)
            m = s.max(axis=2, keepdims=True)
            p = np.exp(s - m)
            den = p.sum(axis=2, keepdims=True)
            o[:, i0:i1, h, :] = np.einsum("bij,bjd->bid", p / den, v[:, j0:i1, kv, :])
            lse[:, h, i0:i1] = (m + np.log(den))[:, :, 0]
    return o, lse


def swa_blocks(q, k, v, window, starts, block=64, scale=None):
    """Sliding-window attention for the query rows [s, s + block) of each
    start s in ``starts`` (clipped at L), by the same definition as ``swa``:
    the block's scores against the banded slice of keys it can see, the mask
    0 <= i - j < W, and a max-subtracted softmax in float64.  The products
    go through ``np.matmul``.

    Returns (rows [R], o [B, R, Hq, d], lse [B, Hq, R]) with the rows of the
    blocks in the order given.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    Bsz, L, Hq, d = q.shape
    Hkv = k.shape[2]
    group = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    spans = [(int(s), min(L, int(s) + block)) for s in starts]
    R = sum(i1 - i0 for i0, i1 in spans)
    rows = np.empty(R, dtype=np.int64)
    o = np.zeros((Bsz, R, Hq, d))
    lse = np.zeros((Bsz, Hq, R))
    r0 = 0
    for i0, i1 in spans:
        n = i1 - i0
        j0 = max(0, i0 - window + 1)
        mask = _visible(np.arange(i0, i1)[:, None], np.arange(j0, i1)[None, :], window)   # [I, J]
        for h in range(Hq):
            kv = h // group
            qh = q[:, i0:i1, h, :]                                   # [B, I, d]
            kh = k[:, j0:i1, kv, :]                                  # [B, J, d]
            s = np.matmul(qh, np.swapaxes(kh, 1, 2)) * scale         # [B, I, J]
            s = np.where(mask[None], s, -np.inf)
            m = s.max(axis=2, keepdims=True)
            p = np.exp(s - m)
            den = p.sum(axis=2, keepdims=True)
            o[:, r0:r0 + n, h, :] = np.matmul(p / den, v[:, j0:i1, kv, :])
            lse[:, h, r0:r0 + n] = (m + np.log(den))[:, :, 0]
        rows[r0:r0 + n] = np.arange(i0, i1)
        r0 += n
    return rows, o, lse


# ------------------------------------------------------------- backward
def _sigmoid(x):
    x = _f64(x)
    return 1.0 / (1.0 + np.exp(-x))


def _silu_grad(x):
    """d silu(x) / dx = σ(x) (1 + x (1 - σ(x)))."""
    sg = _sigmoid(x)
    return sg * (1.0 + x * (1.0 - sg))


def selective_scan_bwd(dy, x, delta, A, Bm, Cm, Dskip=None, z=None, h0=None,
                       conv_w=None, conv_b=None, conv_state=None,
                       delta_softplus=True, conv_silu=True):
    """Reverse-mode gradients of ``selective_scan``'s output y.

    The forward is the recurrence of page "SAMBA混合注意力状态空间模型",
    §数学框架 / Mamba层, with the readings of ``selective_scan``.  Given
    dy = ∂L/∂y [B, L, D], the chain rule taken step by step through that
    definition (the forward states recomputed and kept, then one sequential
    walk from t = L-1 down to 0):

        g_y   = dy ⊙ silu(z)                       (gradient of C·h + D u)
        dz    = dy ⊙ (C·h + D u) ⊙ silu'(z)
        G_t   = ∂L/∂h_t = C_t g_y,t + Ā_{t+1} ⊙ G_{t+1}
        dC_t  = Σ_c g_y,t,c h_t,c              dB_t = Σ_c G_t,c Δ_t,c u_t,c
        dΔ_t  = Σ_n G_t (A Ā_t h_{t-1} + B_t u_t)
        dA    = Σ_t Δ_t Ā_t G_t h_{t-1}        du_t = D g_y,t + Δ_t Σ_n G_t B_t
        dD    = Σ_t g_y,t u_t                  dh0  = Ā_0 ⊙ G_0
    then through softplus (dδ = dΔ σ(δ)), the SiLU after the conv and the
    depthwise causal conv (a correlation, so its input gradient is the
    transposed correlation and its weight gradient a correlation of the
    output gradient with the padded input).

    Arguments as ``selective_scan``.  Returns dict(dx, ddelta, dA, dB, dC,
    dD, dz, dh0, dconv_w, dconv_b, dconv_state); entries whose input was
    None are None.
    """
    x = _f64(x)
    delta = _f64(delta)
    A = _f64(A)
    Bm = _f64(Bm)
    Cm = _f64(Cm)
    dy = _f64(dy)
    Bsz, L, D = x.shape
    N = A.shape[1]

    # forward recompute, keeping every state
    if conv_w is not None:
        conv_w = _f64(conv_w)
        K = conv_w.shape[1]
        st = np.zeros((Bsz, D, K - 1)) if conv_state is None else _f64(conv_state)
        xpad = np.concatenate([np.transpose(st, (0, 2, 1)), x], axis=1)      # [B, L+K-1, D]
        pre = np.zeros((Bsz, L, D))
        for k in range(K):
            pre += conv_w[None, None, :, k] * xpad[:, k:k + L, :]
        if conv_b is not None:
            pre += _f64(conv_b)[None, None, :]
        u = silu(pre) if conv_silu else pre
    else:
        u = x
    dt = softplus(delta) if delta_softplus else delta
    hs = np.empty((L + 1, Bsz, D, N))
    hs[0] = np.zeros((Bsz, D, N)) if h0 is None else _f64(h0)
    for t in range(L):
        hs[t + 1] = np.exp(dt[:, t, :, None] * A[None]) * hs[t] + (dt[:, t, :] * u[:, t, :])[:, :, None] * Bm[:, t, None, :]
    ypre = np.einsum("lbdn,bln->bld", hs[1:], Cm)
    if Dskip is not None:
        ypre = ypre + _f64(Dskip)[None, None, :] * u

    # output gate
    if z is not None:
        z = _f64(z)
        gy = dy * silu(z)
        dz = dy * ypre * _silu_grad(z)
    else:
        gy = dy
        dz = None
    dD = None if Dskip is None else np.einsum("bld,bld->d", gy, u)
    du = np.zeros((Bsz, L, D)) if Dskip is None else gy * _f64(Dskip)[None, None, :]

    # reverse walk
    G = np.zeros((Bsz, D, N))
    dB = np.zeros((Bsz, L, N))
    dC = np.zeros((Bsz, L, N))
    ddt = np.zeros((Bsz, L, D))
    dA = np.zeros((D, N))
    for t in range(L - 1, -1, -1):
        G = G + gy[:, t, :, None] * Cm[:, t, None, :]
        dC[:, t, :] = np.einsum("bd,bdn->bn", gy[:, t, :], hs[t + 1])
        decay = np.exp(dt[:, t, :, None] * A[None])                            # Ā_t [B, D, N]
        hprev = hs[t]
        dB[:, t, :] = np.einsum("bdn,bd->bn", G, dt[:, t, :] * u[:, t, :])
        ddt[:, t, :] = np.einsum("bdn,bdn->bd", G, A[None] * decay * hprev) + \
            u[:, t, :] * np.einsum("bdn,bn->bd", G, Bm[:, t, :])
        dA += np.einsum("bdn,bd->dn", G * decay * hprev, dt[:, t, :])
        du[:, t, :] += dt[:, t, :] * np.einsum("bdn,bn->bd", G, Bm[:, t, :])
        G = G * decay
    dh0 = G
    ddelta = ddt * _sigmoid(delta) if delta_softplus else ddt

    # conv and its SiLU
    if conv_w is not None:
        dpre = du * _silu_grad(pre) if conv_silu else du
        dxpad = np.zeros((Bsz, L + K - 1, D))
        dconv_w = np.zeros((D, K))
        for k in range(K):
            dxpad[:, k:k + L, :] += conv_w[None, None, :, k] * dpre
            dconv_w[:, k] = np.einsum("bld,bld->d", dpre, xpad[:, k:k + L, :])
        dconv_b = dpre.sum(axis=(0, 1)) if conv_b is not None else None
        dx = dxpad[:, K - 1:, :]
        dconv_state = np.transpose(dxpad[:, :K - 1, :], (0, 2, 1)).copy()
    else:
        dx, dconv_w, dconv_b, dconv_state = du, None, None, None
    return {"dx": dx, "ddelta": ddelta, "dA": dA, "dB": dB, "dC": dC, "dD": dD, "dz": dz, "dh0": dh0,
            "dconv_w": dconv_w, "dconv_b": dconv_b, "dconv_state": dconv_state}


def swa_bwd(do, q, k, v, window, scale=None, block=64, magnitudes=False):
    """Reverse-mode gradients of ``swa`` (the banded attention of page
    "SAMBA混合注意力状态空间模型", §滑动窗口注意力, read as the causal band
    0 <= i - j < W with grouped kv heads).

    Per query row i and head h, with P the row's softmax over its visible
    keys and dO = ∂L/∂o:  dV_j += P_ij dO_i,  dP_ij = dO_i · v_j,
    dS_ij = P_ij (dP_ij - Σ_j' P_ij' dP_ij'),  dq_i = scale Σ_j dS_ij k_j,
    dk_j += scale dS_ij q_i; the gradients of a kv head sum over the query
    heads that read it.  Processed per query block over the banded keys.

    Returns (dq [B, L, Hq, d], dk, dv [B, L, Hkv, d]).  With ``magnitudes``
    also a dict of the sizes of the sums that produce them, the same sums over
    the absolute values of their terms (what rounding error of a finite-
    precision evaluation scales with):
        dv_mag = Σ_i P |dO_i|,  dq_mag = scale Σ_j (|dS| + P Dm_i) |k_j|,
        dk_mag = scale Σ_i (|dS| + P Dm_i) |q_i|,  Dm_i = Σ_d |dO_id| Σ_j P_ij |v_jd|,
    where the P Dm term sizes D_i = dO_i · o_i, which an implementation takes
    from its stored o (itself a sum of size Σ_j P |v_j|) rather than as
    Σ_j P dP.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(do)
    Bsz, L, Hq, d = q.shape
    Hkv = k.shape[2]
    group = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    if magnitudes:
        mq, mk, mv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for i0 in range(0, L, block):
        i1 = min(L, i0 + block)
        j0 = max(0, i0 - window + 1)
        mask = _visible(np.arange(i0, i1)[:, None], np.arange(j0, i1)[None, :], window)
        for h in range(Hq):
            kv = h // group
            s = np.einsum("bid,bjd->bij", q[:, i0:i1, h, :], k[:, j0:i1, kv, :]) * scale
            s = np.where(mask[None], s, -np.inf)
            e = np.exp(s - s.max(axis=2, keepdims=True))
            p = e / e.sum(axis=2, keepdims=True)
            dv[:, j0:i1, kv, :] += np.einsum("bij,bid->bjd", p, do[:, i0:i1, h, :])
            dp = np.einsum("bid,bjd->bij", do[:, i0:i1, h, :], v[:, j0:i1, kv, :])
            ds = p * (dp - (p * dp).sum(axis=2, keepdims=True))
            dq[:, i0:i1, h, :] += scale * np.einsum("bij,bjd->bid", ds, k[:, j0:i1, kv, :])
            dk[:, j0:i1, kv, :] += scale * np.einsum("bij,bid->bjd", ds, q[:, i0:i1, h, :])
            if magnitudes:
                omag = np.einsum("bij,bjd->bid", p, np.abs(v[:, j0:i1, kv, :]))
                dmag = np.einsum("bid,bid->bi", np.abs(do[:, i0:i1, h, :]), omag)[:, :, None]
                w = np.abs(ds) + p * dmag
                mv[:, j0:i1, kv, :] += np.einsum("bij,bid->bjd", p, np.abs(do[:, i0:i1, h, :]))
                mq[:, i0:i1, h, :] += scale * np.einsum("bij,bjd->bid", w, np.abs(k[:, j0:i1, kv, :]))
                mk[:, j0:i1, kv, :] += scale * np.einsum("bij,bid->bjd", w, np.abs(q[:, i0:i1, h, :]))
    if magnitudes:
        return dq, dk, dv, {"dq": mq, "dk": mk, "dv": mv}
    return dq, dk, dv


# --------------------------------------------------------------- layers
def round_bf16(a):
    """Rounds to bfloat16 (round to nearest, ties to even) and back to
    float64: the value a bf16 activation holds.  The rounding goes through
    float32 (as a kernel's fp32 result is stored as bf16)."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    bits = f.view(np.uint32).astype(np.uint64)
    rounded = ((bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return rounded.view(np.float32).astype(np.float64)


def mamba_layer(hidden, in_proj, conv_w, conv_b, x_proj, dt_proj, dt_bias, A, Dskip, out_proj,
                bf16_activations=True):
    """A Mamba layer around the selective scan (page "SAMBA混合注意力状态空间
    模型", section 数学框架 / Mamba层: B_t = Linear_B(x_t), C_t = Linear_C(x_t),
    Δ_t = τ_Δ(Linear_Δ(x_t))), with the readings of the layer the paper builds
    on: [x, z] = hidden · in_projᵀ; u = SiLU(conv1d(x)); [δ_low, B, C] =
    u · x_projᵀ; delta = δ_low · dt_projᵀ + dt_bias, Δ = softplus(delta);
    y = scan(u, Δ, A, B, C, D, z); out = y · out_projᵀ.

    hidden [B, L, d_model]; in_proj [2D, d_model]; conv_w [D, K]; conv_b [D];
    x_proj [R + 2N, D]; dt_proj [D, R]; dt_bias [D]; A [D, N]; Dskip [D];
    out_proj [d_model, D].  With ``bf16_activations`` the tensors a bf16
    dataflow stores in bf16 (x, z, u, δ_low, y, out) are rounded to bf16.
    Returns dict(out, h, conv_state).
    """
    rnd = round_bf16 if bf16_activations else (lambda t: t)
    hidden = _f64(hidden)
    D, N, R = _f64(A).shape[0], _f64(A).shape[1], _f64(dt_proj).shape[1]
    xz = np.matmul(hidden, _f64(in_proj).T)
    x, z = rnd(xz[..., :D]), rnd(xz[..., D:])
    u, conv_state = causal_conv1d(x, conv_w, conv_b, None, apply_silu=True)
    u = rnd(u)
    dbc = np.matmul(u, _f64(x_proj).T)
    dt_low = rnd(dbc[..., :R])
    Bm, Cm = dbc[..., R:R + N], dbc[..., R + N:R + 2 * N]
    delta = np.matmul(dt_low, _f64(dt_proj).T) + _f64(dt_bias)
    sc = selective_scan(u, delta, A, Bm, Cm, Dskip, z)
    y = rnd(sc["y"])
    out = rnd(np.matmul(y, _f64(out_proj).T))
    return {"out": out, "h": sc["h"], "conv_state": conv_state}


def swa_layer(hidden, qkv_proj, o_proj, heads_q, heads_kv, head_dim, window, bf16_activations=True):
    """A sliding-window attention layer around the banded attention: [q, k, v]
    = hidden · qkv_projᵀ (column ranges H_q·d, H_kv·d, H_kv·d, each row of a
    range laid out as heads × head_dim); o = SWA(q, k, v); out = o · o_projᵀ.
    With ``bf16_activations`` q, k, v, o and out are rounded to bf16.
    Returns dict(out, k, v)."""
    rnd = round_bf16 if bf16_activations else (lambda t: t)
    hidden = _f64(hidden)
    Bsz, L, _ = hidden.shape
    nq, nk = heads_q * head_dim, heads_kv * head_dim
    qkv = np.matmul(hidden, _f64(qkv_proj).T)
    q = rnd(qkv[..., :nq]).reshape(Bsz, L, heads_q, head_dim)
    k = rnd(qkv[..., nq:nq + nk]).reshape(Bsz, L, heads_kv, head_dim)
    v = rnd(qkv[..., nq + nk:nq + 2 * nk]).reshape(Bsz, L, heads_kv, head_dim)
    o, _ = swa(q, k, v, window)
    o = rnd(o)
    out = rnd(np.matmul(o.reshape(Bsz, L, nq), _f64(o_proj).T))
    return {"out": out, "k": k, "v": v}


def _window_positions(p, window):
    """Absolute positions a query at position p attends under the causal band
    0 <= p - j < W: max(0, p - W + 1) .. p."""
    return range(max(0, p - window + 1), p + 1)


def ring_fill(k, v, window):
    """Decode state after a prefill of L tokens (the page's ``forward(prompt)``
    filling the cache): the last min(L, W) keys and values, key of absolute
    position p stored in slot p mod W, and the next position pos = L.

    k, v: [B, L, Hkv, d].  Returns (k_ring, v_ring [B, W, Hkv, d], pos [B]).
    """
    k = _f64(k)
    v = _f64(v)
    Bsz, L, Hkv, d = k.shape
    k_ring = np.zeros((Bsz, window, Hkv, d))
    v_ring = np.zeros((Bsz, window, Hkv, d))
    for p in _window_positions(L - 1, window):  # the keys position L - 1 sees
        k_ring[:, p % window] = k[:, p]
        v_ring[:, p % window] = v[:, p]
    return k_ring, v_ring, np.full((Bsz,), L, dtype=np.int64)


def swa_step(q_t, k_t, v_t, k_ring, v_ring, pos, window, scale=None):
    """One decoding step of sliding-window attention (``swa_step`` on the
    page's §推理效率 pseudo-code).

    The new key/value (absolute position p = pos[b]) goes into slot p mod W;
    the query then attends the keys of positions max(0, p - W + 1) .. p, which
    are exactly the filled slots.  Softmax does not depend on the order of
    the keys, so the slot order is irrelevant.

    q_t: [B, Hq, d]; k_t, v_t: [B, Hkv, d]; rings [B, W, Hkv, d]; pos [B].
    Returns (o_t [B, Hq, d], k_ring, v_ring, pos + 1) (rings updated copies).
    """
    q_t = _f64(q_t)
    k_ring = _f64(k_ring).copy()
    v_ring = _f64(v_ring).copy()
    pos = np.asarray(pos, dtype=np.int64).copy()
    Bsz, Hq, d = q_t.shape
    Hkv = k_ring.shape[2]
    group = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = np.zeros((Bsz, Hq, d))
    for b in range(Bsz):
        p = int(pos[b])
        k_ring[b, p % window] = _f64(k_t)[b]
        v_ring[b, p % window] = _f64(v_t)[b]
        slots = np.array([a % window for a in _window_positions(p, window)])
        for h in range(Hq):
            kv = h // group
            s = k_ring[b, slots, kv, :] @ q_t[b, h] * scale
            e = np.exp(s - s.max())
            o[b, h] = (e / e.sum()) @ v_ring[b, slots, kv, :]
        pos[b] = p + 1
    return o, k_ring, v_ring, pos


# ------------------------------------------------------------ layer decode
def mamba_layer_step(hidden_t, in_proj, conv_w, conv_b, x_proj, dt_proj, dt_bias, A, Dskip, out_proj, h, conv_state,
                     bf16_activations=True):
    """One decoding step of the Mamba layer (the layer of ``mamba_layer``
    with ``mamba_step`` of the page's §推理效率 pseudo-code as its mixer):
    the same projections, roundings and conv as the prefill on one position,
    the conv continuing from ``conv_state`` and the scan from ``h``.

    hidden_t [B, d_model]; h [B, D, N]; conv_state [B, D, K-1].  Returns
    (out_t [B, d_model], h, conv_state) (new arrays).
    """
    rnd = round_bf16 if bf16_activations else (lambda t: t)
    hidden_t = _f64(hidden_t)
    D, N, R = _f64(A).shape[0], _f64(A).shape[1], _f64(dt_proj).shape[1]
    xz = hidden_t @ _f64(in_proj).T
    x, z = rnd(xz[:, :D]), rnd(xz[:, D:])
    u, conv_state = causal_conv1d(x[:, None, :], conv_w, conv_b, conv_state, apply_silu=True)
    u = rnd(u[:, 0, :])
    dbc = u @ _f64(x_proj).T
    dt_low = rnd(dbc[:, :R])
    B_t, C_t = dbc[:, R:R + N], dbc[:, R + N:R + 2 * N]
    delta_t = dt_low @ _f64(dt_proj).T + _f64(dt_bias)
    y, h, _ = scan_step(h, None, u, delta_t, A, B_t, C_t, Dskip, z)
    out = rnd(rnd(y) @ _f64(out_proj).T)
    return out, h, conv_state


def swa_layer_step(hidden_t, qkv_proj, o_proj, heads_q, heads_kv, head_dim, k_ring, v_ring, pos, window,
                   bf16_activations=True):
    """One decoding step of the SWA layer: the projections of ``swa_layer``
    on one position around ``swa_step`` on the ring.

    hidden_t [B, d_model]; rings [B, W, Hkv, d]; pos [B].  Returns (out_t
    [B, d_model], k_ring, v_ring, pos) (new arrays)."""
    rnd = round_bf16 if bf16_activations else (lambda t: t)
    hidden_t = _f64(hidden_t)
    Bsz = hidden_t.shape[0]
    nq, nk = heads_q * head_dim, heads_kv * head_dim
    qkv = hidden_t @ _f64(qkv_proj).T
    q = rnd(qkv[:, :nq]).reshape(Bsz, heads_q, head_dim)
    k = rnd(qkv[:, nq:nq + nk]).reshape(Bsz, heads_kv, head_dim)
    v = rnd(qkv[:, nq + nk:nq + 2 * nk]).reshape(Bsz, heads_kv, head_dim)
    o, k_ring, v_ring, pos = swa_step(q, k, v, k_ring, v_ring, pos, window)
    out = rnd(rnd(o).reshape(Bsz, nq) @ _f64(o_proj).T)
    return out, k_ring, v_ring, pos
