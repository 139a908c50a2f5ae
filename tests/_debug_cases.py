"""Runs a set of small library calls and saves their outputs (a helper of
tests/test_debug_build.py, run in a child process so that the library the
binding loads can be chosen with SAMBA_LIBRARY).

    python tests/_debug_cases.py OUT.npz

Every call is followed by a status check; the script exits non-zero if any
status word is set.  With SAMBA_LIBRARY=debug it first runs the debug
build's check self-test and requires it to report SAMBA_ERR_CHECK."""

import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from hybrid_ssm_sliding_b200 import _lib as L  # noqa: E402
from hybrid_ssm_sliding_b200 import layers, ops  # noqa: E402
from hybrid_ssm_sliding_b200.workloads import Workload, make_output_grads, make_prefill_inputs  # noqa: E402


def main(out_path):
    lib = L.load()
    out = {}

    def status(what):
        st = ops.get_status()
        if st != 0:
            raise SystemExit(f"{what}: status {st}")

    if os.environ.get("SAMBA_LIBRARY") == "debug":
        L.check(lib.samba_selftest_check(None))
        if ops.get_status() != L.SAMBA_ERR_CHECK:
            raise SystemExit("the check self-test did not report SAMBA_ERR_CHECK")
        status("after the self-test")  # read once, the word is clear again

    wl = Workload("dbg", 2, 100, 64, 16, 4, 8, 2, 64, 48, 77)
    inp = make_prefill_inputs(wl, device="cuda")
    gr = make_output_grads(wl, device="cuda")
    kw = dict(D=inp["D"], z=inp["z"], conv_w=inp["conv_w"], conv_b=inp["conv_b"])
    h = torch.empty((2, 64, 16), device="cuda")
    ck = torch.empty(ops.scan_ckpt_shape(2, 100, 64, 16), device="cuda")
    out["y"] = ops.selective_scan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], h_final=h, h_ckpt=ck,
                                      **kw)
    out["h"] = h
    status("scan forward")
    g = ops.selective_scan_bwd(gr["dy"], inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], ckpt=ck, **kw)
    out.update({"scan_" + k: v for k, v in g.items() if v is not None})
    status("scan backward")
    lse = torch.empty((2, 8, 100), device="cuda")
    o = ops.swa_fwd(inp["q"], inp["k"], inp["v"], 48, lse=lse)
    out["o"], out["lse"] = o, lse
    status("swa forward")
    dq, dk, dv = ops.swa_bwd(gr["do"], inp["q"], inp["k"], inp["v"], o, lse, 48)
    out.update(dq=dq, dk=dk, dv=dv)
    status("swa backward")
    # the layers' prefill and decode steps (tiled and split-K projections,
    # the one-position conv, the scan and SWA steps)
    mw = layers.random_mamba_weights(128, 64, 16, 4, 16, seed=5)
    sw = layers.random_swa_weights(128, 8, 2, 64, 48, seed=6)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    hid = torch.randn((3, 40, 128), generator=gen, device="cuda").to(torch.bfloat16)
    mo, hf, cs = layers.mamba_layer_prefill(hid, mw)
    so, k, v = layers.swa_layer_prefill(mo, sw)
    ms, ss = layers.mamba_decode_state(hf, cs, mw), layers.swa_decode_state(k, v, sw)
    steps = []
    for t in range(5):
        steps.append(layers.swa_layer_step(layers.mamba_layer_step(hid[:, t].contiguous(), mw, ms), sw, ss))
    out["layers_prefill"] = so
    out["layers_steps"] = torch.stack(steps)
    status("layers")
    np.savez(out_path, **{k: v.detach().float().cpu().numpy() for k, v in out.items()})


if __name__ == "__main__":
    main(sys.argv[1])
