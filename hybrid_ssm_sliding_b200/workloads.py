"""Seeded synthetic workloads for the Samba mixer prefill and decode paths.

This module only draws random numbers in the shapes, dtypes and distributions
of the workloads; it holds none of the mixers' arithmetic.  The tests feed
the very same tensors (copied to the host) to the float64 oracle and to the
CUDA library, and ``bench.py`` times the library on them.

Recipe (per workload; draws in this order from one seeded torch.Generator on
the target device, each drawn in float32 and rounded to-nearest-even to bf16
where the workload says bf16):

  x, z   ~ N(0, 1)                      [B, L, D]
  delta  = inverse softplus of a log-uniform step size:
           Δ = exp(U(ln 1e-3, ln 1e-1)), delta = log(expm1(Δ)) (float64 math,
           stored float32), so that softplus(delta) is log-uniform in
           [1e-3, 1e-1]                 [B, L, D]
  B, C   ~ N(0, 1) float32              [B, L, N]
  D      ~ N(0, 1) float32              [D]
  conv_w, conv_b ~ U(-1/sqrt(K), 1/sqrt(K)) float32   [D, K], [D]
  q      ~ N(0, 1)                      [B, L, Hq, d]
  k, v   ~ N(0, 1)                      [B, L, Hkv, d]
  A      = -(n + 1) for state n, float32 (no draw)    [D, N]
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = ["Workload", "WORKLOADS", "make_prefill_inputs", "make_decode_step_inputs"]


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    dim: int            # d_inner channels of the Mamba mixer
    dstate: int         # N
    dconv: int          # K
    heads_q: int
    heads_kv: int
    head_dim: int
    window: int
    seed: int
    act_dtype: torch.dtype = torch.bfloat16     # x, z, y (timing) dtype
    attn_dtype: torch.dtype = torch.bfloat16    # q, k, v, o
    decode_steps: int = 0
    d_model: int = 0      # layer workloads: model width around the mixers (0: mixers only)
    dt_rank: int = 0      # layer workloads: rank of the step-size projection
    train: bool = False   # forward + backward of both mixers
    notes: str = field(default="", compare=False)

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


WORKLOADS = {
    "tiny": Workload("tiny", 1, 64, 16, 4, 4, 2, 2, 16, 16, 0, act_dtype=torch.float32,
                     notes="fp32 scan I/O; q/k/v drawn fp32 and rounded to bf16"),
    "pair_4k": Workload("pair_4k", 1, 4096, 4096, 16, 4, 32, 4, 64, 2048, 1),
    "prefill_128k": Workload("prefill_128k", 1, 131072, 4096, 16, 4, 32, 4, 64, 2048, 2),
    "batched_32k": Workload("batched_32k", 8, 32768, 4096, 16, 4, 32, 4, 64, 2048, 3),
    "decode_64k": Workload("decode_64k", 16, 4096, 4096, 16, 4, 32, 4, 64, 2048, 4,
                           decode_steps=65536),
    # one 32K-token prompt at the same widths: every input still exceeds L2,
    # but the whole problem holds ~1.5 GB, small enough for profiler captures
    "prefill_32k": Workload("prefill_32k", 1, 32768, 4096, 16, 4, 32, 4, 64, 2048, 5),
    # a Mamba layer and an SWA layer with their projections (d_model 2048,
    # d_inner 4096, step-size rank 128) on the 4K and 128K prompts
    "layers_4k": Workload("layers_4k", 1, 4096, 4096, 16, 4, 32, 4, 64, 2048, 6, d_model=2048, dt_rank=128),
    "layers_128k": Workload("layers_128k", 1, 131072, 4096, 16, 4, 32, 4, 64, 2048, 7, d_model=2048,
                            dt_rank=128),
    # the serving loop of a layer stack: 16 sequences after 4096-token
    # prompts decode one token each per step through Mamba + SWA layer pairs
    # with their projections (d_model 2048, step-size rank 128)
    "serve_64k": Workload("serve_64k", 16, 4096, 4096, 16, 4, 32, 4, 64, 2048, 10, decode_steps=65536,
                          d_model=2048, dt_rank=128),
    # forward + backward of both mixers at the pages' 4K training context,
    # 8 sequences per step
    "train_4k": Workload("train_4k", 8, 4096, 4096, 16, 4, 32, 4, 64, 2048, 8, train=True),
    # two sequences of the same shape: a small case for profiler captures
    "train_4k_b2": Workload("train_4k_b2", 2, 4096, 4096, 16, 4, 32, 4, 64, 2048, 9, train=True),
}


def _normal(shape, gen, device, dtype):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return t if dtype == torch.float32 else t.to(dtype)


def _delta_raw(shape, gen, device):
    lo, hi = math.log(1e-3), math.log(1e-1)
    u = torch.rand(shape, generator=gen, device=device, dtype=torch.float32)
    step = torch.exp(lo + (hi - lo) * u.double())
    return torch.log(torch.expm1(step)).float()


def make_prefill_inputs(wl: Workload, device="cpu", with_attention=True, with_scan=True):
    """Draw one prefill batch of ``wl`` on ``device`` (seeded by ``wl.seed``).

    Returns a dict of contiguous tensors: x, z, delta, A, B, C, D, conv_w,
    conv_b (scan) and q, k, v (attention).  Layouts are channel-last:
    x/z/delta [B, L, D], B/C [B, L, N], q [B, L, Hq, d], k/v [B, L, Hkv, d].
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed)
    Bsz, L, D, N, K = wl.batch, wl.seqlen, wl.dim, wl.dstate, wl.dconv
    out = {}
    # The scan tensors are drawn first even when only attention is wanted, so
    # that q/k/v do not depend on the with_scan flag.
    out["x"] = _normal((Bsz, L, D), gen, device, wl.act_dtype)
    out["z"] = _normal((Bsz, L, D), gen, device, wl.act_dtype)
    out["delta"] = _delta_raw((Bsz, L, D), gen, device)
    out["B"] = _normal((Bsz, L, N), gen, device, torch.float32)
    out["C"] = _normal((Bsz, L, N), gen, device, torch.float32)
    out["D"] = _normal((D,), gen, device, torch.float32)
    bound = 1.0 / math.sqrt(K)
    out["conv_w"] = (torch.rand((D, K), generator=gen, device=device) * 2 - 1) * bound
    out["conv_b"] = (torch.rand((D,), generator=gen, device=device) * 2 - 1) * bound
    out["A"] = (-torch.arange(1, N + 1, device=device, dtype=torch.float32)).repeat(D, 1).contiguous()
    if with_attention:
        out["q"] = _normal((Bsz, L, wl.heads_q, wl.head_dim), gen, device, wl.attn_dtype)
        out["k"] = _normal((Bsz, L, wl.heads_kv, wl.head_dim), gen, device, wl.attn_dtype)
        out["v"] = _normal((Bsz, L, wl.heads_kv, wl.head_dim), gen, device, wl.attn_dtype)
    if not with_scan:
        for key in ("x", "z", "delta", "B", "C"):
            del out[key]
    return out


def make_decode_step_inputs(wl: Workload, step: int, device="cpu"):
    """Per-step decode inputs for step ``step``, from a generator keyed by
    (seed, step) so any step can be regenerated on its own.

    x_t, z_t [B, D] (act dtype), delta_t [B, D] f32, B_t, C_t [B, N] f32,
    q_t [B, Hq, d], k_t, v_t [B, Hkv, d] (attn dtype).
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed * 1_000_003 + 7919 * (step + 1))
    Bsz, D, N = wl.batch, wl.dim, wl.dstate
    return {
        "x": _normal((Bsz, D), gen, device, wl.act_dtype),
        "z": _normal((Bsz, D), gen, device, wl.act_dtype),
        "delta": _delta_raw((Bsz, D), gen, device),
        "B": _normal((Bsz, N), gen, device, torch.float32),
        "C": _normal((Bsz, N), gen, device, torch.float32),
        "q": _normal((Bsz, wl.heads_q, wl.head_dim), gen, device, wl.attn_dtype),
        "k": _normal((Bsz, wl.heads_kv, wl.head_dim), gen, device, wl.attn_dtype),
        "v": _normal((Bsz, wl.heads_kv, wl.head_dim), gen, device, wl.attn_dtype),
    }


def make_output_grads(wl: Workload, device="cpu", y_dtype=None, with_attention=True, with_scan=True):
    """Seeded gradients of a loss with respect to the mixers' outputs, for the
    backward: dy [B, L, D] (y_dtype, default the activation dtype) and dO
    [B, L, Hq, d] bf16, N(0, 1), from a generator of their own (seed + 1000)
    so that the forward inputs do not depend on them."""
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed + 1000)
    out = {}
    dy = _normal((wl.batch, wl.seqlen, wl.dim), gen, device, y_dtype or wl.act_dtype)
    do = _normal((wl.batch, wl.seqlen, wl.heads_q, wl.head_dim), gen, device, wl.attn_dtype)
    if with_scan:
        out["dy"] = dy
    if with_attention:
        out["do"] = do
    return out
