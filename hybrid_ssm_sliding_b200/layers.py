"""A Mamba layer and a sliding-window-attention layer around the two mixers:
the projections (samba_gemm) feeding the mixers' inputs in the layouts they
read, and the output projections.

Page "SAMBA混合注意力状态空间模型", section 数学框架 / Mamba层: the selective
parameters are linear maps of the layer's input, B_t = Linear_B(x_t),
C_t = Linear_C(x_t), Δ_t = τ_Δ(Linear_Δ(x_t)); the forward of its inference
section stacks a Mamba layer and an SWA layer.  Readings (where the pages are
silent) follow the Mamba layer the paper builds on:

* Mamba layer, d_inner = D channels: the input projection gives x and z
  ([B, L, D] each, one GEMM whose epilogue splits the columns); u =
  SiLU(conv1d(x)); the selective-parameter projection of u gives a rank-R
  step input, B and C (one GEMM, three column ranges: bf16, fp32, fp32);
  delta = dt_proj(rank-R input) + dt_bias (fp32), and Δ = softplus(delta)
  inside the scan; y = scan(u, Δ, A, B, C, D, z); out = out_proj(y).
* SWA layer: one GEMM gives q, k, v (column ranges of H_q·d, H_kv·d, H_kv·d),
  o = SWA(q, k, v), out = o_proj(o).

Activations between kernels are bf16 (x, z, u, the rank-R input, y, q, k, v,
o, the outputs); B, C, delta and the states are fp32.  No norm, residual or
MLP: these are the two token-mixing layers only.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import ops


@dataclass
class MambaLayerWeights:
    in_proj: torch.Tensor    # [2D, d_model] bf16: rows [0, D) give x, [D, 2D) give z
    conv_w: torch.Tensor     # [D, K] fp32
    conv_b: torch.Tensor     # [D] fp32
    x_proj: torch.Tensor     # [R + 2N, D] bf16: rank-R step input, B, C
    dt_proj: torch.Tensor    # [D, R] bf16
    dt_bias: torch.Tensor    # [D] fp32
    A: torch.Tensor          # [D, N] fp32
    D: torch.Tensor          # [D] fp32
    out_proj: torch.Tensor   # [d_model, D] bf16

    @property
    def dims(self):
        D, K = self.conv_w.shape
        N = self.A.shape[1]
        R = self.dt_proj.shape[1]
        return D, N, K, R


@dataclass
class SwaLayerWeights:
    qkv_proj: torch.Tensor   # [(Hq + 2 Hkv) d, d_model] bf16
    o_proj: torch.Tensor     # [d_model, Hq d] bf16
    heads_q: int
    heads_kv: int
    head_dim: int
    window: int


def mamba_layer_prefill(hidden, w: MambaLayerWeights, stream=None, taps=None):
    """hidden [B, L, d_model] bf16 -> (out [B, L, d_model] bf16, h_final
    [B, D, N] fp32, conv_state [B, D, K-1] fp32).  A dict passed as ``taps``
    receives the intermediate activations (x, z, u, delta, B, C, y)."""
    Bsz, Ln, dm = hidden.shape
    D, N, K, R = w.dims
    M = Bsz * Ln
    dev = hidden.device
    h2 = hidden.reshape(M, dm)
    x = torch.empty((Bsz, Ln, D), dtype=torch.bfloat16, device=dev)
    z = torch.empty_like(x)
    ops.gemm(h2, w.in_proj, outs=[(x.view(M, D), 0, D, None), (z.view(M, D), D, 2 * D, None)], stream=stream)
    cs = torch.empty((Bsz, D, K - 1), dtype=torch.float32, device=dev)
    u = ops.conv1d_fwd(x, w.conv_w, w.conv_b, silu=True, conv_state_out=cs, stream=stream)
    dt_low = torch.empty((M, R), dtype=torch.bfloat16, device=dev)
    Bm = torch.empty((Bsz, Ln, N), dtype=torch.float32, device=dev)
    Cm = torch.empty_like(Bm)
    ops.gemm(u.view(M, D), w.x_proj, outs=[(dt_low, 0, R, None), (Bm.view(M, N), R, R + N, None),
                                            (Cm.view(M, N), R + N, R + 2 * N, None)], stream=stream)
    delta = torch.empty((Bsz, Ln, D), dtype=torch.float32, device=dev)
    ops.gemm(dt_low, w.dt_proj, outs=[(delta.view(M, D), 0, D, w.dt_bias)], stream=stream)
    h_final = torch.empty((Bsz, D, N), dtype=torch.float32, device=dev)
    y = ops.selective_scan_fwd(u, delta, w.A, Bm, Cm, D=w.D, z=z, fuse_conv=False, h_final=h_final,
                               y_dtype=torch.bfloat16, stream=stream)
    out = ops.gemm(y.view(M, D), w.out_proj, stream=stream).view(Bsz, Ln, dm)
    if taps is not None:
        taps.update(x=x, z=z, u=u, delta=delta, B=Bm, C=Cm, y=y)
    return out, h_final, cs


def swa_layer_prefill(hidden, w: SwaLayerWeights, stream=None):
    """hidden [B, L, d_model] bf16 -> out [B, L, d_model] bf16 (and the k, v
    the decode ring is filled from)."""
    Bsz, Ln, dm = hidden.shape
    Hq, Hkv, d = w.heads_q, w.heads_kv, w.head_dim
    M = Bsz * Ln
    dev = hidden.device
    q = torch.empty((Bsz, Ln, Hq, d), dtype=torch.bfloat16, device=dev)
    k = torch.empty((Bsz, Ln, Hkv, d), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    nq, nk = Hq * d, Hkv * d
    ops.gemm(hidden.reshape(M, dm), w.qkv_proj, outs=[(q.view(M, nq), 0, nq, None), (k.view(M, nk), nq, nq + nk, None),
                                                     (v.view(M, nk), nq + nk, nq + 2 * nk, None)], stream=stream)
    o = ops.swa_fwd(q, k, v, w.window, stream=stream)
    out = ops.gemm(o.view(M, nq), w.o_proj, stream=stream).view(Bsz, Ln, dm)
    return out, k, v


def random_mamba_weights(d_model, D, N, K, R, seed, device="cuda"):
    """Seeded random weights of the Mamba layer's shapes (no trained weights
    exist here): projections ~ N(0, 1/fan_in) in bf16, conv U(-1/sqrt(K),
    1/sqrt(K)), dt_bias the inverse softplus of a log-uniform [1e-3, 1e-1]
    step, A = -(n + 1), D ~ N(0, 1)."""
    import math

    g = torch.Generator(device=device)
    g.manual_seed(seed)

    def lin(o, i):
        return (torch.randn((o, i), generator=g, device=device) / math.sqrt(i)).to(torch.bfloat16)

    bound = 1.0 / math.sqrt(K)
    step = torch.exp(math.log(1e-3) + (math.log(1e-1) - math.log(1e-3)) *
                     torch.rand((D,), generator=g, device=device, dtype=torch.float64))
    return MambaLayerWeights(
        in_proj=lin(2 * D, d_model),
        conv_w=(torch.rand((D, K), generator=g, device=device) * 2 - 1) * bound,
        conv_b=(torch.rand((D,), generator=g, device=device) * 2 - 1) * bound,
        x_proj=lin(R + 2 * N, D),
        dt_proj=lin(D, R),
        dt_bias=torch.log(torch.expm1(step)).float(),
        A=(-torch.arange(1, N + 1, device=device, dtype=torch.float32)).repeat(D, 1).contiguous(),
        D=torch.randn((D,), generator=g, device=device),
        out_proj=lin(d_model, D),
    )


def random_swa_weights(d_model, Hq, Hkv, d, window, seed, device="cuda"):
    """Seeded random weights of the SWA layer's shapes, N(0, 1/fan_in) bf16."""
    import math

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    n = (Hq + 2 * Hkv) * d
    return SwaLayerWeights(
        qkv_proj=(torch.randn((n, d_model), generator=g, device=device) / math.sqrt(d_model)).to(torch.bfloat16),
        o_proj=(torch.randn((d_model, Hq * d), generator=g, device=device) / math.sqrt(Hq * d)).to(torch.bfloat16),
        heads_q=Hq, heads_kv=Hkv, head_dim=d, window=window)


# ----------------------------------------------------------------- decode
@dataclass
class MambaDecodeState:
    """Decode state of a Mamba layer: the SSM state and the conv state (the
    conv of one position updates its state in place), and the zero-filled
    workspace of the split-K projections (None: tiled projections)."""
    h: torch.Tensor                      # [B, D, N] fp32
    conv: torch.Tensor                   # [B, D, K-1] fp32
    gemm_ws: torch.Tensor = field(default=None)


@dataclass
class SwaDecodeState:
    """Decode state of an SWA layer: the K/V ring and the next position, the
    SWA step's workspace and the projections' (as for the Mamba layer)."""
    k_ring: torch.Tensor                 # [B, W, Hkv, d] bf16
    v_ring: torch.Tensor
    pos: torch.Tensor                    # [B] int64
    workspace: torch.Tensor = field(default=None)
    gemm_ws: torch.Tensor = field(default=None)


def _gemm_workspace(M, widths, device):
    """One zero-filled workspace for projections of M rows to each of the
    given widths, run one after another (None when M is above the split-K
    limit)."""
    n = max(ops.gemm_workspace_size(M, w) for w in widths)
    return torch.zeros((n,), dtype=torch.uint8, device=device) if n > 0 else None


def mamba_decode_state(h_final, conv_state, w: MambaLayerWeights = None, split_k=True):
    """The decode state after a prefill (mamba_layer_prefill's h_final and
    conv state).  Given the layer's weights (and ``split_k``), it also
    carries the workspace of the split-K projections."""
    Bsz = h_final.shape[0]
    ws = None
    if w is not None and split_k:
        D, N, K, R = w.dims
        ws = _gemm_workspace(Bsz, (2 * D, R + 2 * N, D, w.out_proj.shape[0]), h_final.device)
    return MambaDecodeState(h=h_final.clone(), conv=conv_state.clone(), gemm_ws=ws)


def swa_decode_state(k, v, w: SwaLayerWeights, split_k=True):
    """The decode state after a prefill (swa_layer_prefill's k, v): the ring
    of the last W positions, the SWA step's workspace and (with ``split_k``)
    the split-K projections' workspace."""
    k_ring, v_ring, pos = ops.swa_ring_fill(k, v, w.window)
    Bsz = k.shape[0]
    ws = torch.zeros((max(ops.swa_step_workspace_size(Bsz, w.heads_q, w.head_dim, w.window), 16),),
                     dtype=torch.uint8, device=k.device)
    gws = None
    if split_k:
        nqkv = (w.heads_q + 2 * w.heads_kv) * w.head_dim
        gws = _gemm_workspace(Bsz, (nqkv, w.o_proj.shape[0]), k.device)
    return SwaDecodeState(k_ring, v_ring, pos, ws, gws)


def mamba_layer_step(hidden_t, w: MambaLayerWeights, st: MambaDecodeState, stream=None, taps=None):
    """One token per sequence through the Mamba layer: hidden_t [B, d_model]
    bf16 -> out_t [B, d_model] bf16, the state advanced in place.  The same
    steps as mamba_layer_prefill at L = 1: in_proj -> (x, z); the conv over
    the carried inputs -> u; x_proj -> (rank-R input, B, C); dt_proj + bias ->
    delta; one scan step (samba_scan_step, conv not fused: u is its input);
    out_proj.  A dict passed as ``taps`` receives the step's activations
    (x, z, u, delta, B, C, y; [B, ...] each)."""
    Bsz, dm = hidden_t.shape
    D, N, K, R = w.dims
    dev = hidden_t.device
    x = torch.empty((Bsz, D), dtype=torch.bfloat16, device=dev)
    z = torch.empty_like(x)
    ops.gemm(hidden_t, w.in_proj, outs=[(x, 0, D, None), (z, D, 2 * D, None)], workspace=st.gemm_ws, stream=stream)
    u = ops.conv1d_fwd(x.view(Bsz, 1, D), w.conv_w, w.conv_b, conv_state_in=st.conv, silu=True,
                       conv_state_out=st.conv, stream=stream).view(Bsz, D)
    dt_low = torch.empty((Bsz, R), dtype=torch.bfloat16, device=dev)
    Bt = torch.empty((Bsz, N), dtype=torch.float32, device=dev)
    Ct = torch.empty_like(Bt)
    ops.gemm(u, w.x_proj, outs=[(dt_low, 0, R, None), (Bt, R, R + N, None), (Ct, R + N, R + 2 * N, None)],
             workspace=st.gemm_ws, stream=stream)
    delta = torch.empty((Bsz, D), dtype=torch.float32, device=dev)
    ops.gemm(dt_low, w.dt_proj, outs=[(delta, 0, D, w.dt_bias)], workspace=st.gemm_ws, stream=stream)
    y = ops.scan_step(st.h, None, u, delta, w.A, Bt, Ct, D=w.D, z_t=z, y_dtype=torch.bfloat16, stream=stream)
    if taps is not None:
        taps.update(x=x, z=z, u=u, delta=delta, B=Bt, C=Ct, y=y)
    return ops.gemm(y, w.out_proj, workspace=st.gemm_ws, stream=stream)


def swa_layer_step(hidden_t, w: SwaLayerWeights, st: SwaDecodeState, stream=None):
    """One token per sequence through the SWA layer: qkv projection, one SWA
    step on the ring (samba_swa_step, pos advanced), output projection."""
    Bsz, dm = hidden_t.shape
    Hq, Hkv, d = w.heads_q, w.heads_kv, w.head_dim
    dev = hidden_t.device
    q = torch.empty((Bsz, Hq, d), dtype=torch.bfloat16, device=dev)
    k = torch.empty((Bsz, Hkv, d), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    nq, nk = Hq * d, Hkv * d
    ops.gemm(hidden_t, w.qkv_proj, outs=[(q.view(Bsz, nq), 0, nq, None), (k.view(Bsz, nk), nq, nq + nk, None),
                                        (v.view(Bsz, nk), nq + nk, nq + 2 * nk, None)],
             workspace=st.gemm_ws, stream=stream)
    o = ops.swa_step(q, k, v, st.k_ring, st.v_ring, st.pos, w.window, workspace=st.workspace, stream=stream)
    return ops.gemm(o.view(Bsz, nq), w.o_proj, workspace=st.gemm_ws, stream=stream)
