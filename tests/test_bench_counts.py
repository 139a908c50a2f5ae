"""The algorithmic work bench.py divides by: band pairs, exps, MUFU operations
and bytes, counted here by brute force on small shapes (CPU only)."""
import dataclasses

import numpy as np
import pytest

import bench
from hybrid_ssm_sliding_b200.workloads import WORKLOADS


def _band_pairs(L, W):
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    return int(((i - j >= 0) & (i - j < W)).sum())


@pytest.mark.parametrize("L,W", [(64, 16), (10, 16), (16, 16), (33, 1), (200, 64)])
def test_exact_band_flops_counts_the_causal_window(L, W):
    wl = dataclasses.replace(WORKLOADS["tiny"], seqlen=L, window=W, batch=3, heads_q=5, head_dim=16)
    pairs = _band_pairs(L, W)
    assert bench.swa_exact_band_flops(wl) == 4.0 * pairs * 16 * 3 * 5
    assert bench.swa_exps(wl) == pairs * 3 * 5


def test_band_flops_upper_bound():
    wl = WORKLOADS["prefill_128k"]
    # 4·L·W·d per (batch, head) counts W keys for every query, including the
    # first W-1 queries that see fewer; the exact band is W²/2-ish smaller.
    exact = bench.swa_exact_band_flops(wl)
    nominal = bench.swa_flops(wl)
    W, L = wl.window, wl.seqlen
    assert nominal - exact == 4.0 * (W * (W - 1) // 2) * wl.head_dim * wl.batch * wl.heads_q
    assert exact < nominal


def test_scan_counts():
    wl = dataclasses.replace(WORKLOADS["tiny"], batch=2, seqlen=7, dim=5, dstate=4)
    tc = 2 * 7 * 5
    assert bench.scan_mufu_ops(wl) == tc * (4 + 6)
    # 10 bytes per (token, channel), 2·N·4 per token for B and C, and the
    # per-channel state and parameters
    small = 2 * 5 * (4 + 3) * 4 + 5 * (4 + 4 + 2) * 4
    assert bench.scan_bytes(wl) == tc * 10 + 2 * 7 * 2 * 4 * 4 + small


def test_mufu_roof_arithmetic():
    r = bench.mufu_roof(ops_count=2.0e12, ms=1000.0, sms=148, sm_mhz=1965.0)
    assert r["achieved"] == pytest.approx(2.0)
    assert r["peak"] == pytest.approx(16 * 148 * 1.965e9 / 1e12)
    assert r["frac"] == pytest.approx(2.0 / r["peak"])
    assert r["bound"] == "alu"


def test_backward_counts():
    """The attention backward's five band products and the scan backward's
    bytes, written out term by term."""
    wl = dataclasses.replace(WORKLOADS["tiny"], batch=2, seqlen=7, dim=5, dstate=4, heads_q=3, window=4,
                             head_dim=16, dconv=4)
    assert bench.swa_bwd_flops(wl) == 5 * 2.0 * 2 * 3 * 7 * 4 * 16
    assert bench.swa_bwd_flops(wl) == 2.5 * bench.swa_flops(wl)
    tc = 2 * 7 * 5
    per_tc = 2 + 2 + 2 + 4 + 2 + 2 + 4          # x, z, dy, delta in; dx, dz, ddelta out
    per_token = 4 * 4 * 4                       # B, C in; dB, dC out (fp32, N = 4)
    small = 5 * (4 + 4 + 2) * 4 * 2             # A, conv w/b, D and their gradients
    assert bench.scan_bwd_bytes(wl) == tc * per_tc + 2 * 7 * per_token + small


def test_serve_step_bytes_term_by_term():
    """The serving loop's bytes per decode step, listed tensor by tensor for
    one layer pair (times the pairs)."""
    wl = dataclasses.replace(WORKLOADS["serve_64k"], batch=3, dim=40, dstate=8, d_model=24, dt_rank=4, heads_q=4,
                             heads_kv=2, head_dim=16, window=32, seqlen=100)
    B, D, N, K, R, dm = 3, 40, 8, 4, 4, 24
    nq, nk = 4 * 16, 2 * 16
    bf, f4 = 2, 4
    want = {
        "in_proj": 2 * D * dm * bf + B * dm * bf + B * 2 * D * bf,
        "x_proj": (R + 2 * N) * D * bf + B * D * bf + B * R * bf + B * 2 * N * f4,
        "dt_proj": D * R * bf + B * R * bf + B * D * f4 + D * f4,
        "out_proj": dm * D * bf + B * D * bf + B * dm * bf,
        "qkv_proj": (nq + 2 * nk) * dm * bf + B * dm * bf + B * (nq + 2 * nk) * bf,
        "o_proj": dm * nq * bf + B * nq * bf + B * dm * bf,
        # x in, u out; conv state in and out; weights and bias
        "conv": B * D * bf * 2 + 2 * B * D * (K - 1) * f4 + D * (K + 1) * f4,
        # h in and out; u, z in, y out (bf16); delta in (fp32); B, C; A; skip D
        "scan_step": 2 * B * D * N * f4 + B * D * (bf + bf + bf) + B * D * f4 + 2 * B * N * f4 + D * N * f4 + D * f4,
        # the W ring slots of K and V read, k_t, v_t written, q_t in, o_t out
        "swa_step": 2 * 32 * B * nk * bf + 2 * B * nk * bf + 2 * B * nq * bf,
    }
    got = bench.serve_step_bytes(wl)
    assert set(got) == set(want)
    for k in want:
        assert got[k] == bench.SERVE_PAIRS * want[k], k


def test_recorded_traffic_only_for_the_captured_source(monkeypatch):
    """bench.py reports a kernel's DRAM bytes only while its source still
    hashes to the one the capture was taken from, and only for a recorded
    (kernel, workload) pair."""
    import json
    import os

    from hybrid_ssm_sliding_b200 import build as B

    with open(os.path.join(os.path.dirname(bench.__file__), "profiles", "traffic.json")) as f:
        rec = json.load(f)
    ent = rec["scan"]["prefill_128k"]
    assert ent["bytes_per_launch"] == ent["read"] + ent["write"]
    monkeypatch.setattr(B, "kernel_hash", lambda src: ent["kernel_hash"])
    assert bench.recorded_traffic("scan", "prefill_128k", "scan_fwd") == ent["bytes_per_launch"]
    assert bench.recorded_traffic("scan", "no_such_workload", "scan_fwd") is None
    assert bench.recorded_traffic("no_such_kernel", "prefill_128k", "scan_fwd") is None
    monkeypatch.setattr(B, "kernel_hash", lambda src: "0" * 12)    # the source changed since
    assert bench.recorded_traffic("scan", "prefill_128k", "scan_fwd") is None
