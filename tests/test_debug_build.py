"""The debug build (libsamba_debug.so: every global output store's index
checked on the device, a failed check skipped and reported as
SAMBA_ERR_CHECK) on the GPU: its check self-test reports, and a set of
small calls (both mixers forward and backward, the layers' prefill and
decode steps) runs with no check firing and gives the release build's
results.  Each library runs in a child process (the binding loads one per
process)."""

import os
import subprocess
import sys

import numpy as np
import pytest

from hybrid_ssm_sliding_b200 import build as B

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(tmp_path, which):
    out = str(tmp_path / f"{which}.npz")
    env = dict(os.environ)
    env.pop("SAMBA_LIBRARY", None)
    if which == "debug":
        env["SAMBA_LIBRARY"] = "debug"
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "_debug_cases.py"), out], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, f"{which} build: {r.stdout[-2000:]}{r.stderr[-4000:]}"
    return np.load(out)


def test_debug_build_runs_clean_and_matches_release(tmp_path):
    B.build()
    B.build(debug=True)
    rel = _run(tmp_path, "release")
    dbg = _run(tmp_path, "debug")
    assert set(rel.files) == set(dbg.files)
    for k in rel.files:
        a, b = rel[k], dbg[k]
        assert np.all(np.isfinite(b)), k
        # the same arithmetic; sums added with atomics (dA, dB, dC, dD, conv
        # gradients) and the split-K projections may add in another order, so
        # a bf16 result may round one unit apart (2^-8 of the largest value),
        # and through the layers' chain of steps a little more
        scale = float(np.max(np.abs(a))) or 1.0
        tol = (2.0 ** -6 if k.startswith("layers") else 2.0 ** -7) * scale
        assert float(np.max(np.abs(a - b))) <= tol, k
