"""Sequence-parallel mixer prefill: a long prompt split into consecutive
segments, one per rank (one GPU per process), with the exact result of one
pass over the whole prompt.

Each rank holds one segment of every input.  Three exchanges join them:

* the conv state: the last K-1 inputs x of segment r-1 (``ops.conv_state``)
  are the conv state segment r starts from;
* the scan state: every segment is first scanned from a zero state, which
  gives its final state h_local and the sum of its step sizes dsum
  (``samba_scan_args.delta_sum``).  The recurrence is linear in its state, so
  the state segment r starts from is the fold of (dsum, h_local) of the
  segments before it, h <- exp(A * dsum) * h + h_local (``ops.scan_carry``,
  one kernel per earlier segment), after which a second pass from that state
  gives the outputs (page "SAMBA混合注意力状态空间模型", section 数学框架 /
  Mamba层: the recurrence is the same in every segment; the split is only an
  order of evaluation);
* the attention halo: the keys and values of the last W-1 positions of
  segment r-1, which the first W-1 queries of segment r still see.  Segment r
  runs the banded attention over [halo; segment] and keeps the rows of its own
  positions.

The phases of one rank are methods of ``SegmentPrefill``; ``prefill_distributed``
runs them with torch.distributed (NCCL between GPUs: point-to-point for the
halos, an all-gather for the scan summaries), and ``prefill_in_turn`` runs all
ranks' phases in one process, one after the other, on one device.  Both call
the same phases.  Every step of the arithmetic runs in the library's kernels;
this module only moves tensors between ranks.

Requirements: every segment has at least max(W - 1, K - 1) tokens, and all
segments have the same batch, widths and dtypes.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass
class Tails:
    """What a segment hands to the next one."""
    conv: torch.Tensor            # [B, D, K-1] fp32: its last K-1 inputs
    k: torch.Tensor | None        # [B, W-1, Hkv, d] bf16: keys of its last W-1 positions
    v: torch.Tensor | None


class SegmentPrefill:
    """The phases of one segment.

    ``scan`` holds the keyword arguments of ``ops.selective_scan_fwd`` for the
    segment (x, delta, A, B, C and optionally D, z, conv_w, conv_b) and
    ``swa`` those of ``ops.swa_fwd`` (q, k, v, window) or None.  ``ops`` is the
    module that runs the kernels (the library's ``ops`` unless a caller
    supplies another with the same functions).
    """

    def __init__(self, scan: dict, swa: dict | None, rank: int, ops=None):
        if ops is None:
            from . import ops as _ops
            ops = _ops
        self.ops = ops
        # the outputs and carried states are this module's to supply
        self.scan = {k: v for k, v in scan.items()
                     if k not in ("y", "h0", "h_final", "conv_state_in", "conv_state_out", "delta_sum")}
        self.swa = None if swa is None else dict(swa)
        self.rank = rank
        x = self.scan["x"]
        self.batch, self.seqlen, self.dim = x.shape
        self.dstate = self.scan["A"].shape[1]
        self.dconv = self.scan["conv_w"].shape[1] if self.scan.get("conv_w") is not None else 4
        if self.seqlen < self.dconv - 1:
            raise ValueError("a segment needs at least K - 1 tokens")
        if self.swa is not None and self.seqlen < self.swa["window"] - 1:
            raise ValueError("a segment needs at least W - 1 tokens")

    # ---------------------------------------------------------------- phase 1
    def tails(self) -> Tails:
        """The conv state and the attention halo this segment hands on."""
        conv = self.ops.conv_state(self.scan["x"], self.dconv)
        k = v = None
        if self.swa is not None:
            w1 = self.swa["window"] - 1
            k = self.swa["k"][:, self.seqlen - w1:].contiguous()
            v = self.swa["v"][:, self.seqlen - w1:].contiguous()
        return Tails(conv, k, v)

    # ---------------------------------------------------------------- phase 2
    def local(self, conv_in: torch.Tensor | None):
        """Scans the segment from a zero state: returns (dsum [B, D],
        h_local [B, D, N]).  The outputs written here are rewritten by
        ``final``."""
        x = self.scan["x"]
        dsum = torch.empty((self.batch, self.dim), dtype=torch.float32, device=x.device)
        h_local = torch.empty((self.batch, self.dim, self.dstate), dtype=torch.float32, device=x.device)
        self._y = self.ops.selective_scan_fwd(**self.scan, conv_state_in=conv_in, h0=None, h_final=h_local,
                                              delta_sum=dsum)
        return dsum, h_local

    # ---------------------------------------------------------------- phase 3
    def start_state(self, summaries, h0=None):
        """The state this segment starts from: the fold of the summaries
        (dsum, h_local) of every earlier segment, from h0 (zeros if None)."""
        h = h0
        A = self.scan["A"]
        for dsum, h_local in summaries[: self.rank]:
            h = self.ops.scan_carry(h, dsum, A, h_local)
        return h

    def final(self, conv_in, summaries, halo: Tails | None, h0=None):
        """The second pass: returns (y, o, h_final, conv_state_out) of the
        segment (o is None without attention)."""
        h_in = self.start_state(summaries, h0)
        x = self.scan["x"]
        h_final = torch.empty((self.batch, self.dim, self.dstate), dtype=torch.float32, device=x.device)
        conv_out = torch.empty((self.batch, self.dim, self.dconv - 1), dtype=torch.float32, device=x.device)
        y = self.ops.selective_scan_fwd(**self.scan, conv_state_in=conv_in, h0=h_in, h_final=h_final,
                                        conv_state_out=conv_out, y=getattr(self, "_y", None))
        o = None
        if self.swa is not None:
            q, k, v, W = self.swa["q"], self.swa["k"], self.swa["v"], self.swa["window"]
            if halo is None or halo.k is None:
                o = self.ops.swa_fwd(q, k, v, W, scale=self.swa.get("scale"))
            else:
                # [halo; segment]: the halo's query rows are filler whose outputs are dropped
                filler = torch.zeros((q.shape[0], W - 1) + tuple(q.shape[2:]), dtype=q.dtype, device=q.device)
                q_ext = torch.cat([filler, q], dim=1)
                k_ext = torch.cat([halo.k, k], dim=1)
                v_ext = torch.cat([halo.v, v], dim=1)
                o = self.ops.swa_fwd(q_ext, k_ext, v_ext, W, scale=self.swa.get("scale"))[:, W - 1:]
        return y, o, h_final, conv_out


def prefill_in_turn(scans: list[dict], swas: list[dict | None], h0=None, ops=None):
    """Runs every segment's phases in one process, segment after segment (the
    exchanges become plain references).  Returns a list of (y, o, h_final,
    conv_state_out), one per segment."""
    segs = [SegmentPrefill(sc, sw, r, ops) for r, (sc, sw) in enumerate(zip(scans, swas))]
    tails = [s.tails() for s in segs]
    conv_in = [None] + [t.conv for t in tails[:-1]]
    summaries = [s.local(conv_in[r]) for r, s in enumerate(segs)]
    halos = [None] + tails[:-1]
    return [s.final(conv_in[r], summaries, halos[r], h0) for r, s in enumerate(segs)]


def prefill_distributed(scan: dict, swa: dict | None, group=None, ops=None):
    """One segment per rank of ``group`` (rank r holds segment r).  Returns
    (y, o, h_final, conv_state_out) of this rank's segment; the last rank's
    h_final and conv_state_out are those of the whole prompt."""
    import torch.distributed as dist

    rank, world = dist.get_rank(group), dist.get_world_size(group)
    seg = SegmentPrefill(scan, swa, rank, ops)
    mine = seg.tails()

    def shift(t_send, like):
        """Sends t_send to rank + 1 and returns what rank - 1 sent (None on rank 0)."""
        ops_ = []
        recv = None
        if rank + 1 < world:
            ops_.append(dist.P2POp(dist.isend, t_send.contiguous(), dist.get_global_rank(group, rank + 1)
                                   if group is not None else rank + 1, group))
        if rank > 0:
            recv = torch.empty_like(like)
            ops_.append(dist.P2POp(dist.irecv, recv, dist.get_global_rank(group, rank - 1)
                                   if group is not None else rank - 1, group))
        if ops_:
            for req in dist.batch_isend_irecv(ops_):
                req.wait()
        return recv

    conv_in = shift(mine.conv, mine.conv)
    halo = None
    if swa is not None:
        hk = shift(mine.k, mine.k)
        hv = shift(mine.v, mine.v)
        halo = None if rank == 0 else Tails(None, hk, hv)
    dsum, h_local = seg.local(conv_in)
    all_dsum = [torch.empty_like(dsum) for _ in range(world)]
    all_h = [torch.empty_like(h_local) for _ in range(world)]
    dist.all_gather(all_dsum, dsum, group=group)
    dist.all_gather(all_h, h_local, group=group)
    return seg.final(conv_in, list(zip(all_dsum, all_h)), halo)
