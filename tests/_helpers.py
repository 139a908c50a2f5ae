"""Shared test helpers: error metrics and host copies of device tensors."""

import json
import os

import numpy as np
import torch


def host64(t):
    """Exact float64 host copy of a tensor (bf16/fp32 upcast exactly)."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()


def scan_rel_err(got, ref, mag=None):
    """Max relative error of a scan output.

    With ``mag`` (the oracle's y_mag / h_mag: the same sums taken over the
    absolute values of their terms) each error is divided by the size of the
    sum that produced the value: max_i |g_i - r_i| / mag_i.  mag_i >= |r_i|,
    and the two agree when nothing cancels; rounding error scales with mag_i,
    so near-zero results of large cancelling sums are judged fairly.
    Without ``mag``: max_i |g_i - r_i| / max(|r_i|, 1e-2 rms(r))."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    if mag is not None:
        den = np.maximum(np.asarray(mag, dtype=np.float64), 1e-300)
    else:
        rms = float(np.sqrt(np.mean(ref * ref)))
        den = np.maximum(np.abs(ref), 1e-2 * rms + 1e-300)
    return float(np.max(np.abs(got - ref) / den))


def plain_rel_err(got, ref):
    """max |g - r| / |r| over the entries with |r| >= rms(r) (reported, not gated)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    sel = np.abs(ref) >= rms
    return float(np.max(np.abs(got - ref)[sel] / np.abs(ref)[sel])) if np.any(sel) else 0.0


SCAN_TOL = 1e-4          # max relative error of fp32 scan outputs and final states
SWA_MAX_ABS = 2e-2       # bf16 attention output against the float64 oracle
SWA_MEAN_ABS = 1e-2


def scan_errors(got, ref, mag):
    """The gated error (relative to the oracle's magnitudes) and the two
    reported ones: relative to max(|r|, 1e-2 rms(r)), and plain relative
    error over the entries with |r| >= rms(r)."""
    return {"rel_to_mag": scan_rel_err(got, ref, mag), "rel_floor": scan_rel_err(got, ref),
            "rel_plain": plain_rel_err(got, ref)}


def record_margin(test, quantity, **values):
    """Appends one measured error to the JSON-lines file named by the
    SAMBA_MARGINS_FILE environment variable (nothing when it is unset)."""
    path = os.environ.get("SAMBA_MARGINS_FILE")
    if not path:
        return
    rec = {"test": test, "quantity": quantity}
    rec.update({k: (float(v) if isinstance(v, (float, np.floating)) else v) for k, v in values.items()})
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def nan_tensor(shape, dtype, device="cuda"):
    """A tensor filled with NaN: outputs start poisoned, so that an element
    the kernel never writes fails the comparison."""
    return torch.full(shape, float("nan"), dtype=dtype, device=device)
