"""The exchanges of the sequence-parallel prefill with two gloo ranks on CPU.

Each rank holds one segment of a prompt; ``seqpar.prefill_distributed`` joins
them with point-to-point halos and an all-gather of the scan summaries.  The
kernels are replaced here by CPU stand-ins written from the float64 oracle
(this test file's own, with the contracts of the library's functions), so
that the test exercises exactly the exchange and fold logic; the concatenated
result must equal the oracle over the whole prompt."""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle.samba_oracle as orc
from hybrid_ssm_sliding_b200 import seqpar
from hybrid_ssm_sliding_b200.workloads import Workload, make_prefill_inputs


class OracleOps:
    """CPU stand-ins with the contracts of the library's ops (float64 inside)."""

    @staticmethod
    def _np(t):
        return None if t is None else t.detach().double().numpy()

    def conv_state(self, x, dconv, conv_state_in=None, conv_state_out=None):
        xs = self._np(x)
        pad = np.zeros((xs.shape[0], dconv - 1, xs.shape[2])) if conv_state_in is None else \
            self._np(conv_state_in).transpose(0, 2, 1)
        tail = np.concatenate([pad, xs], axis=1)[:, -(dconv - 1):]
        return torch.from_numpy(tail.transpose(0, 2, 1).copy()).float()

    def selective_scan_fwd(self, x, delta, A, B, C, D=None, z=None, conv_w=None, conv_b=None, conv_state_in=None,
                           h0=None, y=None, y_dtype=None, h_final=None, conv_state_out=None, delta_sum=None, **_):
        out = orc.selective_scan(self._np(x), self._np(delta), self._np(A), self._np(B), self._np(C), self._np(D),
                                 self._np(z), h0=self._np(h0), conv_w=self._np(conv_w), conv_b=self._np(conv_b),
                                 conv_state=self._np(conv_state_in))
        yt = torch.from_numpy(out["y"]).float()
        if y is None:
            y = yt
        else:
            y.copy_(yt)
        if h_final is not None:
            h_final.copy_(torch.from_numpy(out["h"]))
        if conv_state_out is not None:
            conv_state_out.copy_(torch.from_numpy(out["conv_state"]))
        if delta_sum is not None:
            delta_sum.copy_(torch.from_numpy(orc.softplus(self._np(delta)).sum(axis=1)))
        return y

    def scan_carry(self, h_in, dsum, A, h_local, h_out=None):
        h = self._np(h_local) + (0.0 if h_in is None else
                                 np.exp(self._np(A)[None] * self._np(dsum)[:, :, None]) * self._np(h_in))
        return torch.from_numpy(h).float()

    def swa_fwd(self, q, k, v, window, scale=None, o=None, lse=None):
        out, _ = orc.swa(self._np(q), self._np(k), self._np(v), window, scale=scale)
        return torch.from_numpy(out).float()


WL = Workload("spg", 1, 240, 16, 4, 4, 4, 2, 16, 40, 17, act_dtype=torch.float32)


def _segment(inp, rank, world):
    Ln = inp["x"].shape[1]
    b = np.linspace(0, Ln, world + 1).astype(int)
    sl = slice(b[rank], b[rank + 1])
    seg = {k: (v[:, sl].contiguous() if k in ("x", "z", "delta", "B", "C", "q", "k", "v") else v)
           for k, v in inp.items()}
    scan = dict(x=seg["x"], delta=seg["delta"], A=seg["A"], B=seg["B"], C=seg["C"], D=seg["D"], z=seg["z"],
                conv_w=seg["conv_w"], conv_b=seg["conv_b"])
    swa = dict(q=seg["q"].float(), k=seg["k"].float(), v=seg["v"].float(), window=WL.window)
    return scan, swa


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = make_prefill_inputs(WL, device="cpu")
        scan, swa = _segment(inp, rank, world)
        y, o, h, cs = seqpar.prefill_distributed(scan, swa, ops=OracleOps())
        out[rank] = (y.numpy(), o.numpy(), h.numpy(), cs.numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_distributed_segments_equal_one_pass(world):
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = [out[r] for r in range(world)]
    inp = make_prefill_inputs(WL, device="cpu")
    np_ = OracleOps._np  # a staticmethod: np_(t)
    ref = orc.selective_scan(np_(inp["x"]), np_(inp["delta"]), np_(inp["A"]), np_(inp["B"]),
                             np_(inp["C"]), np_(inp["D"]), np_(inp["z"]),
                             conv_w=np_(inp["conv_w"]), conv_b=np_(inp["conv_b"]))
    y = np.concatenate([r[0] for r in res], axis=1)
    np.testing.assert_allclose(y, ref["y"], rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(res[-1][2], ref["h"], rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(res[-1][3], ref["conv_state"], rtol=0, atol=1e-6)
    ref_o, _ = orc.swa(np_(inp["q"]), np_(inp["k"]), np_(inp["v"]), WL.window)
    o = np.concatenate([r[1] for r in res], axis=1)
    np.testing.assert_allclose(o, ref_o, rtol=1e-5, atol=1e-5)
