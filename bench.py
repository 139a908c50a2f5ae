#!/usr/bin/env python
"""Throughput of the Samba mixer prefill on B200.

One step = one samba_mixer_prefill call: the fused selective scan (conv,
softplus, scan, D skip, gate; bf16 y, fp32 final state and conv state) and
the banded sliding-window attention (bf16, 32 q / 4 kv heads, d = 64,
W = 2048) over one batch of the 128K-token workload (B = 1, L = 131072,
d_inner = 4096, N = 16).  Inputs are synthetic (seeded) and resident in HBM;
each input is larger than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl samba|reference]

With N > 1 (torchrun) every rank runs its own batch (weak scaling, no
collective on the data path); the time is the max over ranks.  --impl
reference times the float64 CPU oracle on bounded samples of the same
workload.  Prints one JSON line on rank 0.

    python bench.py --workload decode_64k [--steps K] [--warmup W]

times decoding instead: after a 4096-token prefill of 16 sequences, one step
is samba_scan_step + samba_swa_step of one layer for all 16 sequences (one
token each; the SWA step reads the full 2048-slot K/V ring).  Four layer
states (scan state, conv state, K/V rings: 154 MB, more than L2) rotate from
step to step, as in a multi-layer model, so every step reads its state from
HBM; 32 steps per CUDA graph, inputs of 32 distinct steps resident in HBM.
"""

from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Samba mixer prefill tokens/s @128K; scan HBM GB/s; SWA tensor-pipe %"
UNIT = "tokens/s"
DECODE_METRIC = "Samba mixer decode tokens/s (16 sequences, one token each per step; SWA ring W = 2048)"
DECODE_GRAPH_STEPS = 32
DECODE_LAYERS = 4
SERVE_PAIRS = 4
SERVE_METRIC = ("Samba layer-stack decode tokens/s (16 sequences after 4096-token prompts, one token each per step "
                "through 4 Mamba + SWA layer pairs with their projections; SWA ring W = 2048)")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="samba", choices=["samba", "reference"])
    ap.add_argument("--workload", default="prefill_128k")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--kernel-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graphs", type=int, default=0,
                    help="decode workloads: timed replays of the 32-step graph (default: the workload's decode "
                         "steps / 32)")
    return ap.parse_args()


# ------------------------------------------------------------- ranks (N > 1)
# Replicas only: every rank runs its own batch of the workload (its own seed),
# no data crosses ranks, and the reported time is the max over ranks.
def rank_workload(wl, rank):
    """The workload of rank `rank`: same shapes, its own seeded inputs."""
    from dataclasses import replace

    return replace(wl, seed=wl.seed + 1000 * rank)


def max_over_ranks(x, device):
    """Max of the float x over all ranks (x itself without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms):
    """Units per second of the whole job: every rank's units over the slowest rank's time."""
    return world * units_per_rank / (ms / 1e3)


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mp = json.load(f)
        return {"hbm_gbs": mp["hbm_gbs"], "bf16_tflops": mp["bf16_tflops"],
                "bf16_tflops_sustained": mp.get("bf16_tflops_sustained", mp["bf16_tflops"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def recorded_traffic(kind, workload, src):
    """DRAM bytes per launch of one kernel on one workload, as an ncu capture
    recorded them (read + write), or None when there is no capture or the
    kernel's sources have changed since it was taken."""
    from hybrid_ssm_sliding_b200 import build as B

    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            ent = json.load(f).get(kind, {}).get(workload)
        if ent and ent.get("kernel_hash") == B.kernel_hash(src):
            return ent["bytes_per_launch"]
    except Exception:
        pass
    return None


def workload_config(wl):
    return {"workload": wl.name, "batch": wl.batch, "seq_len": wl.seqlen, "d_inner": wl.dim, "d_state": wl.dstate,
            "d_conv": wl.dconv, "heads_q": wl.heads_q, "heads_kv": wl.heads_kv, "head_dim": wl.head_dim,
            "window": wl.window, "l2": "no flush: every input tensor is larger than the 126 MB L2"}


# ----------------------------------------------------------------- algorithmic work
def scan_bytes(wl):
    """HBM bytes the scan must move once: x, z (bf16), delta (fp32) in, y
    (bf16) out per (token, channel); B and C per token; the final state and
    conv state out and the small per-channel parameters."""
    tc = wl.batch * wl.seqlen * wl.dim
    per_token = 2 * wl.dstate * 4
    small = wl.batch * wl.dim * (wl.dstate + 3) * 4 + wl.dim * (wl.dstate + wl.dconv + 2) * 4
    return tc * (2 + 2 + 4 + 2) + wl.batch * wl.seqlen * per_token + small


def decode_bytes(wl):
    """Algorithmic HBM bytes of one decode step for the whole batch: the scan
    step reads and writes h [B, D, N] f32 and the conv state [B, D, K-1] f32,
    reads x_t, z_t (bf16), delta_t (f32), A, conv weights and writes y_t
    (bf16); the SWA step reads the valid K and V ring slots (all W of them
    after a prefill longer than W), q_t, writes k_t, v_t into the ring and
    o_t."""
    Bsz, D, N, K = wl.batch, wl.dim, wl.dstate, wl.dconv
    scan = (2 * Bsz * D * N * 4 + 2 * Bsz * D * (K - 1) * 4 + Bsz * D * (2 + 2 + 4) + Bsz * D * 2
            + D * N * 4 + D * (K + 2) * 4 + 2 * Bsz * N * 4)
    slots = min(wl.window, wl.seqlen + 1)
    kv = Bsz * wl.heads_kv * wl.head_dim * 2
    swa = 2 * slots * kv + 2 * kv + 2 * Bsz * wl.heads_q * wl.head_dim * 2
    return scan, swa


def swa_flops(wl):
    """Band FLOPs 4·L·W·d per (batch, query head)."""
    return 4.0 * wl.seqlen * wl.window * wl.head_dim * wl.batch * wl.heads_q


def swa_exact_band_flops(wl):
    L, W = wl.seqlen, wl.window
    pairs = sum(min(i + 1, W) for i in range(0, min(L, W))) + max(0, L - W) * W
    return 4.0 * pairs * wl.head_dim * wl.batch * wl.heads_q


# Special-function (MUFU) work.  The SM's MUFU pipe evaluates 16 ex2 / rcp /
# lg2 per clock (measured on B200 with a dependent-free ex2 loop), so the peak
# is 16 x SMs x the SM clock sampled during the run.
MUFU_PER_CLK_SM = 16


def scan_mufu_ops(wl):
    """Special-function operations per (token, channel) of the fused scan:
    one exp per state for exp(Δ A), exp and reciprocal for the conv SiLU,
    exp and reciprocal for softplus(delta), exp and reciprocal for the silu(z)
    gate."""
    return wl.batch * wl.seqlen * wl.dim * (wl.dstate + 6)


def swa_exps(wl):
    """One exp per (query, key) pair of the band per query head."""
    return swa_exact_band_flops(wl) / (4.0 * wl.head_dim)


def mufu_roof(ops_count, ms, sms, sm_mhz):
    """Special-function operations per second against the MUFU peak."""
    achieved = ops_count / (ms / 1e3) / 1e12
    peak = MUFU_PER_CLK_SM * sms * sm_mhz * 1e6 / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Tops/s", "frac": achieved / peak,
            "ops": ops_count, "sms": sms, "sm_mhz": sm_mhz}


# ----------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------- oracle leg
# The float64 oracle, as it stands, timed on the host cores: independent units
# of the workload (blocks of channels for the scan; one KV head with its query
# heads over blocks of query rows for SWA) run in a pool of one process per
# core (spawn start method, NumPy single-threaded in each), and the throughput
# of the whole pool is extrapolated to whole-workload tokens/s.

def host_cores():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


def _oracle_scan_unit(args):
    """Oracle selective_scan on n_chan channels x n_tok tokens (one sequence)."""
    n_chan, n_tok, N, K, seed = args
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle.samba_oracle as orc

    rng = np.random.default_rng(seed)
    x = rng.standard_normal((1, n_tok, n_chan))
    z = rng.standard_normal((1, n_tok, n_chan))
    delta = np.log(np.expm1(np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), (1, n_tok, n_chan)))))
    A = -np.tile(np.arange(1, N + 1, dtype=np.float64), (n_chan, 1))
    Bm = rng.standard_normal((1, n_tok, N))
    Cm = rng.standard_normal((1, n_tok, N))
    with threadpool_limits(1):
        orc.selective_scan(x, delta, A, Bm, Cm, rng.standard_normal(n_chan), z,
                           conv_w=rng.uniform(-0.5, 0.5, (n_chan, K)), conv_b=rng.uniform(-0.5, 0.5, n_chan))
    return n_chan * n_tok


def _oracle_swa_unit(args):
    """Oracle swa_blocks: n_blocks blocks of 64 query rows of the `group`
    query heads of one KV head, each block at a full window."""
    group, d, W, n_blocks, seed = args
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle.samba_oracle as orc

    rng = np.random.default_rng(seed)
    span = W + 64 * n_blocks
    q = rng.standard_normal((1, span, group, d))
    k = rng.standard_normal((1, span, 1, d))
    v = rng.standard_normal((1, span, 1, d))
    with threadpool_limits(1):
        rows, _, _ = orc.swa_blocks(q, k, v, W, [W + 64 * i for i in range(n_blocks)])
    return len(rows)


def _oracle_decode_unit(args):
    """`reps` decode steps of one sequence with the oracle: scan_step on
    n_chan channels (kind "scan") or swa_step of every head at a full ring
    (kind "swa")."""
    kind, n_chan, N, K, Hq, Hkv, d, W, reps, seed = args
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle.samba_oracle as orc

    rng = np.random.default_rng(seed)
    with threadpool_limits(1):
        if kind == "scan":
            h = rng.standard_normal((1, n_chan, N)) * 0.1
            cs = rng.standard_normal((1, n_chan, K - 1))
            A = -np.tile(np.arange(1, N + 1, dtype=np.float64), (n_chan, 1))
            for _ in range(reps):
                _, h, cs = orc.scan_step(h, cs, rng.standard_normal((1, n_chan)), rng.uniform(-6.9, -2.3, (1, n_chan)),
                                         A, rng.standard_normal((1, N)), rng.standard_normal((1, N)),
                                         rng.standard_normal(n_chan), rng.standard_normal((1, n_chan)),
                                         conv_w=rng.uniform(-0.5, 0.5, (n_chan, K)),
                                         conv_b=rng.uniform(-0.5, 0.5, n_chan))
        else:
            kr = rng.standard_normal((1, W, Hkv, d))
            vr = rng.standard_normal((1, W, Hkv, d))
            pos = np.full((1,), W + 7, dtype=np.int64)
            for _ in range(reps):
                _, kr, vr, pos = orc.swa_step(rng.standard_normal((1, Hq, d)), rng.standard_normal((1, Hkv, d)),
                                              rng.standard_normal((1, Hkv, d)), kr, vr, pos, W)
    return reps


def oracle_pool():
    """A pool of one oracle process per host core.  The spawn start method
    gives every worker a fresh interpreter (no state inherited from a parent
    that may already hold a CUDA context)."""
    import multiprocessing as mp

    return mp.get_context("spawn").Pool(host_cores())


def _timed_map(pool, fn, units):
    t0 = time.perf_counter()
    done = sum(pool.map(fn, units, chunksize=1))
    return done, time.perf_counter() - t0


def oracle_throughput(wl, pool, scale=1.0, seed=0):
    """Prefill tokens/s of the oracle on the host cores, from one timed
    sample per mixer: the scan on 8 units of 32 channels x 16384 tokens per
    core, SWA on 8 units per core of 4 blocks of 64 rows (a KV head with its
    query heads, full window).  Returns (tokens/s, cores, sample text)."""
    P = host_cores()
    group = wl.heads_q // wl.heads_kv
    n_tok = max(256, int(16384 * scale))
    _timed_map(pool, _oracle_scan_unit, [(8, 64, wl.dstate, wl.dconv, seed)] * P)         # workers import
    sc_units = [(32, n_tok, wl.dstate, wl.dconv, seed * 1000 + i) for i in range(8 * P)]
    sw_units = [(group, wl.head_dim, wl.window, max(1, int(4 * scale)), seed * 1000 + i) for i in range(8 * P)]
    sc_done, t_sc = _timed_map(pool, _oracle_scan_unit, sc_units)
    sw_done, t_sw = _timed_map(pool, _oracle_swa_unit, sw_units)
    per_token = t_sc / sc_done * wl.dim + t_sw / sw_done * wl.heads_kv
    sample = (f"{P} processes on {cpu_model()}: scan {len(sc_units)} units of 32 channels x {n_tok} tokens "
              f"({t_sc:.1f} s), SWA {len(sw_units)} units of {sw_units[0][3]} x 64 query rows x {group} heads "
              f"at W = {wl.window} ({t_sw:.1f} s); float64 NumPy; extrapolated to whole-workload tokens/s "
              f"(scan x {wl.dim} channels, SWA x {wl.heads_kv} KV heads per token)")
    return 1.0 / per_token, P, sample


def oracle_decode_throughput(wl, pool, scale=1.0, seed=0):
    """Decode tokens/s of the oracle on the host cores: 4 units per core of
    `reps` steps of one sequence, for the scan step (512 channels, scaled to
    all of them) and for the SWA step (every head at a full ring)."""
    P = host_cores()
    reps = max(1, int(16 * scale))
    n_chan = 512
    dims = (wl.dstate, wl.dconv, wl.heads_q, wl.heads_kv, wl.head_dim)
    _timed_map(pool, _oracle_decode_unit, [("scan", 8) + dims + (64, 1, 0)] * P)   # workers import
    sc_steps, t_sc = _timed_map(pool, _oracle_decode_unit,
                                [("scan", n_chan) + dims + (wl.window, reps, seed * 1000 + i) for i in range(4 * P)])
    sw_steps, t_sw = _timed_map(pool, _oracle_decode_unit,
                                [("swa", n_chan) + dims + (wl.window, reps, seed * 1000 + i) for i in range(4 * P)])
    per_token = t_sc / sc_steps * (wl.dim / n_chan) + t_sw / sw_steps
    sample = (f"{P} processes on {cpu_model()}: {4 * P} units of {reps} scan steps of one sequence on {n_chan} of "
              f"{wl.dim} channels ({t_sc:.1f} s, scaled by channels) and {4 * P} units of {reps} SWA steps of "
              f"{wl.heads_q} heads over a full {wl.window}-slot ring ({t_sw:.1f} s); float64 NumPy; extrapolated "
              f"to tokens/s")
    return 1.0 / per_token, P, sample


def _oracle_serve_unit(args):
    """`reps` decode steps of one sequence through one Mamba + SWA layer pair
    with the oracle's layer steps, at the workload's widths (random float64
    weights of the layer shapes, a full ring).  Returns (reps, seconds the
    steps took)."""
    dm, D, N, K, R, Hq, Hkv, d, W, reps, seed = args
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle.samba_oracle as orc

    rng = np.random.default_rng(seed)
    mw = dict(in_proj=rng.standard_normal((2 * D, dm)) / dm ** 0.5, conv_w=rng.uniform(-0.5, 0.5, (D, K)),
              conv_b=rng.uniform(-0.5, 0.5, D), x_proj=rng.standard_normal((R + 2 * N, D)) / D ** 0.5,
              dt_proj=rng.standard_normal((D, R)) / R ** 0.5, dt_bias=rng.uniform(-6.9, -2.3, D),
              A=-np.tile(np.arange(1, N + 1, dtype=np.float64), (D, 1)), Dskip=rng.standard_normal(D),
              out_proj=rng.standard_normal((dm, D)) / D ** 0.5)
    qkv = rng.standard_normal(((Hq + 2 * Hkv) * d, dm)) / dm ** 0.5
    o_proj = rng.standard_normal((dm, Hq * d)) / (Hq * d) ** 0.5
    h = rng.standard_normal((1, D, N)) * 0.1
    cs = rng.standard_normal((1, D, K - 1))
    kr = rng.standard_normal((1, W, Hkv, d))
    vr = rng.standard_normal((1, W, Hkv, d))
    pos = np.full((1,), W + 7, dtype=np.int64)
    xs = rng.standard_normal((reps, 1, dm))
    with threadpool_limits(1):
        t0 = time.perf_counter()
        for r in range(reps):
            x, h, cs = orc.mamba_layer_step(xs[r], h=h, conv_state=cs, **mw)
            _, kr, vr, pos = orc.swa_layer_step(x, qkv, o_proj, Hq, Hkv, d, kr, vr, pos, W)
        return reps, time.perf_counter() - t0


def _oracle_layers_unit(args):
    """The oracle's Mamba layer (kind "mamba") or the projections of its SWA
    layer (kind "swa_proj": swa_layer with a one-key window, so that its
    attention costs next to nothing) on n_tok tokens of one sequence at the
    workload's widths, random float64 weights of the layer shapes.  Returns
    the tokens done."""
    kind, n_tok, dm, D, N, K, R, Hq, Hkv, d, seed = args
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle.samba_oracle as orc

    rng = np.random.default_rng(seed)
    hidden = rng.standard_normal((1, n_tok, dm))
    with threadpool_limits(1):
        if kind == "mamba":
            orc.mamba_layer(hidden, rng.standard_normal((2 * D, dm)) / dm ** 0.5, rng.uniform(-0.5, 0.5, (D, K)),
                            rng.uniform(-0.5, 0.5, D), rng.standard_normal((R + 2 * N, D)) / D ** 0.5,
                            rng.standard_normal((D, R)) / R ** 0.5, rng.uniform(-6.9, -2.3, D),
                            -np.tile(np.arange(1, N + 1, dtype=np.float64), (D, 1)), rng.standard_normal(D),
                            rng.standard_normal((dm, D)) / D ** 0.5)
        else:
            orc.swa_layer(hidden, rng.standard_normal(((Hq + 2 * Hkv) * d, dm)) / dm ** 0.5,
                          rng.standard_normal((dm, Hq * d)) / (Hq * d) ** 0.5, Hq, Hkv, d, 1)
    return n_tok


def oracle_layers_throughput(wl, pool, scale=1.0, seed=0):
    """Tokens/s of the oracle's Mamba layer plus SWA layer on the host cores,
    from three timed samples: the Mamba layer on one unit of n tokens per
    core; the SWA layer's projections (the layer with a one-key window) on
    one unit per core; its attention at the full window as in the prefill
    baseline (blocks of 64 rows of one KV head's query heads)."""
    P = host_cores()
    n_tok = max(32, int(1024 * scale))
    dims = (wl.d_model, wl.dim, wl.dstate, wl.dconv, wl.dt_rank, wl.heads_q, wl.heads_kv, wl.head_dim)
    _timed_map(pool, _oracle_layers_unit, [("swa_proj", 8, 64, 64, 4, 4, 8, 2, 1, 16, 0)] * P)   # workers import
    m_done, t_m = _timed_map(pool, _oracle_layers_unit, [("mamba", n_tok) + dims + (seed * 1000 + i,)
                                                         for i in range(P)])
    p_done, t_p = _timed_map(pool, _oracle_layers_unit, [("swa_proj", n_tok) + dims + (seed * 1000 + i,)
                                                         for i in range(P)])
    group = wl.heads_q // wl.heads_kv
    sw_units = [(group, wl.head_dim, wl.window, 2, seed * 1000 + i) for i in range(2 * P)]
    a_done, t_a = _timed_map(pool, _oracle_swa_unit, sw_units)
    per_token = t_m / m_done + t_p / p_done + t_a / a_done * wl.heads_kv
    sample = (f"{P} processes on {cpu_model()}: the Mamba layer on {P} units of {n_tok} tokens ({t_m:.1f} s), the "
              f"SWA layer's projections on {P} units of {n_tok} tokens ({t_p:.1f} s), its attention on "
              f"{len(sw_units)} units of 2 x 64 query rows x {group} heads at W = {wl.window} ({t_a:.1f} s); "
              f"d_model {wl.d_model}, d_inner {wl.dim}; float64 NumPy; extrapolated to tokens/s (attention x "
              f"{wl.heads_kv} KV heads per token)")
    return 1.0 / per_token, P, sample


def _oracle_train_unit(args):
    """One training step's worth of the oracle on a sample: kind "scan" runs
    selective_scan and selective_scan_bwd on n_chan channels x n_tok tokens
    and returns channel-tokens done; kind "swa" runs swa and swa_bwd on one
    KV head and its `group` query heads over n_tok tokens and returns
    full-window row equivalents done (the band's (query, key) pairs over W)."""
    kind, n_chan, n_tok, N, K, group, d, W, seed = args
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle.samba_oracle as orc

    rng = np.random.default_rng(seed)
    with threadpool_limits(1):
        if kind == "scan":
            x = rng.standard_normal((1, n_tok, n_chan))
            z = rng.standard_normal((1, n_tok, n_chan))
            delta = rng.uniform(-6.9, -2.3, (1, n_tok, n_chan))
            A = -np.tile(np.arange(1, N + 1, dtype=np.float64), (n_chan, 1))
            Bm, Cm = rng.standard_normal((1, n_tok, N)), rng.standard_normal((1, n_tok, N))
            Dsk = rng.standard_normal(n_chan)
            cw, cb = rng.uniform(-0.5, 0.5, (n_chan, K)), rng.uniform(-0.5, 0.5, n_chan)
            orc.selective_scan(x, delta, A, Bm, Cm, Dsk, z, conv_w=cw, conv_b=cb)
            orc.selective_scan_bwd(rng.standard_normal((1, n_tok, n_chan)), x, delta, A, Bm, Cm, Dsk, z,
                                   conv_w=cw, conv_b=cb)
            return float(n_chan * n_tok)
        q = rng.standard_normal((1, n_tok, group, d))
        k = rng.standard_normal((1, n_tok, 1, d))
        v = rng.standard_normal((1, n_tok, 1, d))
        orc.swa(q, k, v, W)
        orc.swa_bwd(rng.standard_normal((1, n_tok, group, d)), q, k, v, W)
        pairs = sum(min(i + 1, W) for i in range(n_tok))
        return pairs / W


def oracle_train_throughput(wl, pool, scale=1.0, seed=0):
    """Training-step tokens/s of the oracle on the host cores: the scan's
    forward and backward on one unit of 32 channels x n tokens per core, the
    attention's forward and backward on one unit per core of one KV head over
    W + 256 tokens, extrapolated by channels and by the band's pairs."""
    P = host_cores()
    n_tok = max(256, int(16384 * scale))
    group = wl.heads_q // wl.heads_kv
    _timed_map(pool, _oracle_train_unit, [("scan", 8, 64, wl.dstate, wl.dconv, 1, 16, 16, 0)] * P)   # workers import
    sc_units = [("scan", 32, n_tok, wl.dstate, wl.dconv, group, wl.head_dim, wl.window, seed * 1000 + i)
                for i in range(P)]
    sw_tok = wl.window + max(64, int(256 * scale))
    sw_units = [("swa", 0, sw_tok, wl.dstate, wl.dconv, group, wl.head_dim, wl.window, seed * 1000 + i)
                for i in range(P)]
    sc_done, t_sc = _timed_map(pool, _oracle_train_unit, sc_units)
    sw_done, t_sw = _timed_map(pool, _oracle_train_unit, sw_units)
    per_token = t_sc / sc_done * wl.dim + t_sw / sw_done * wl.heads_kv
    sample = (f"{P} processes on {cpu_model()}: the scan's forward and backward on {P} units of 32 channels x "
              f"{n_tok} tokens ({t_sc:.1f} s), the attention's forward and backward on {P} units of one KV head "
              f"with {group} query heads over {sw_tok} tokens at W = {wl.window} ({t_sw:.1f} s); float64 NumPy; "
              f"extrapolated to tokens/s (scan x {wl.dim} channels, attention by the band's pairs x "
              f"{wl.heads_kv} KV heads per token)")
    return 1.0 / per_token, P, sample


def oracle_serve_throughput(wl, pool, scale=1.0, seed=0, pairs=None):
    """Decode tokens/s of the oracle's layer steps on the host cores: one unit
    per core of `reps` steps of one sequence through one layer pair (the steps
    timed inside the unit), scaled to the stack's pairs."""
    P = host_cores()
    pairs = pairs or SERVE_PAIRS
    reps = max(2, int(128 * scale))
    dims = (wl.d_model, wl.dim, wl.dstate, wl.dconv, wl.dt_rank, wl.heads_q, wl.heads_kv, wl.head_dim, wl.window)
    pool.map(_oracle_serve_unit, [(64, 64, 4, 4, 8, 2, 1, 16, 16, 1, 0)] * P, chunksize=1)   # workers import
    res = pool.map(_oracle_serve_unit, [dims + (reps, seed * 1000 + i) for i in range(P)], chunksize=1)
    done, t = sum(r[0] for r in res), sum(r[1] for r in res)
    # the P units run at the same time, one per core: the pool decodes P
    # token-pairs in the time one unit takes for one
    per_token = t / done / P * pairs
    sample = (f"{P} processes on {cpu_model()}, at the same time: each {reps} decode steps of one sequence through "
              f"one Mamba + SWA layer pair at d_model {wl.d_model}, d_inner {wl.dim}, {wl.heads_q}/{wl.heads_kv} "
              f"heads, a full {wl.window}-slot ring ({t / P:.1f} s of steps per process, weight setup untimed); "
              f"float64 NumPy; scaled to {pairs} pairs and extrapolated to tokens/s")
    return 1.0 / per_token, P, sample


def run_reference(args):
    """The reference arm: the float64 oracle, as it stands, on the host cores.
    Each step is one bounded parallel sample of the workload (a few seconds of
    wall time); `value` is the median over the steps of the throughput
    extrapolated to the whole workload, and `ms_per_step` the measured wall
    time of one sampled step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from hybrid_ssm_sliding_b200.workloads import WORKLOADS

    wl = WORKLOADS[args.workload]
    decode = wl.decode_steps > 0
    serve = decode and wl.d_model > 0
    measure = oracle_serve_throughput if serve else (oracle_decode_throughput if decode else oracle_throughput)
    with oracle_pool() as pool:
        for i in range(max(0, args.warmup)):
            measure(wl, pool, scale=0.05, seed=1000 + i)
        vals, walls, sample, cores = [], [], "", host_cores()
        for i in range(max(1, args.steps)):
            t0 = time.perf_counter()
            v, cores, sample = measure(wl, pool, scale=0.25, seed=i)
            walls.append(time.perf_counter() - t0)
            vals.append(v)
    value = statistics.median(vals)
    tokens_per_step = wl.batch if decode else wl.batch * wl.seqlen
    line = {
        "impl": "reference", "metric": SERVE_METRIC if serve else (DECODE_METRIC if decode else METRIC),
        "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": len(vals), "warmup": args.warmup,
        "ms_per_step": statistics.mean(walls) * 1e3,
        "extrapolated_ms_per_workload_step": tokens_per_step / value * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample + f"; each step one such sample, median of {len(vals)} steps; value and "
                                            f"extrapolated_ms_per_workload_step are extrapolated from the samples"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------ layers GPU leg
LAYERS_METRIC = "Samba Mamba + SWA layer prefill tokens/s (projections, conv, scan, attention)"


def layer_gemm_flops(wl):
    """Dense FLOPs of the layers' projections for one step (2 per multiply-add)."""
    M, dm, D, N, R = wl.batch * wl.seqlen, wl.d_model, wl.dim, wl.dstate, wl.dt_rank
    nq, nk = wl.heads_q * wl.head_dim, wl.heads_kv * wl.head_dim
    per_token = 2 * D * dm + (R + 2 * N) * D + D * R + dm * D + (nq + 2 * nk) * dm + dm * nq
    return 2.0 * M * per_token


def run_layers(args, wl, dev, rank, world):
    """Times one Mamba layer and one SWA layer with their projections on the
    same hidden state (random weights of the layer shapes)."""
    import torch
    import torch.distributed as dist

    from hybrid_ssm_sliding_b200 import layers, ops

    wl_rank = rank_workload(wl, rank)
    mw = layers.random_mamba_weights(wl.d_model, wl.dim, wl.dstate, wl.dconv, wl.dt_rank, wl_rank.seed, dev)
    sw = layers.random_swa_weights(wl.d_model, wl.heads_q, wl.heads_kv, wl.head_dim, wl.window, wl_rank.seed + 1,
                                   dev)
    g = torch.Generator(device=dev)
    g.manual_seed(wl_rank.seed + 2)
    hidden = torch.randn((wl.batch, wl.seqlen, wl.d_model), generator=g, device=dev).to(torch.bfloat16)
    stream = torch.cuda.current_stream()

    def step():
        layers.mamba_layer_prefill(hidden, mw)
        layers.swa_layer_prefill(hidden, sw)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(e0.elapsed_time(e1), dev)
    clk = clocks.stop()
    ms_step = ms_total / args.steps
    # the largest projection alone, for the tensor roofline
    M = wl.batch * wl.seqlen
    h2 = hidden.view(M, wl.d_model)
    xz = torch.empty((M, 2 * wl.dim), dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        ops.gemm(h2, mw.in_proj, outs=[(xz, 0, 2 * wl.dim, None)])
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    n = max(5, args.kernel_steps // 4)
    for _ in range(n):
        ops.gemm(h2, mw.in_proj, outs=[(xz, 0, 2 * wl.dim, None)])
    b.record(stream)
    torch.cuda.synchronize()
    ms_in = a.elapsed_time(b) / n
    peaks = load_peaks()
    fl_in = 2.0 * M * 2 * wl.dim * wl.d_model
    tfs = fl_in / (ms_in / 1e3) / 1e12
    roof = {"bound": "tensor", "achieved": tfs, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": tfs / peaks["bf16_tflops"], "traffic": recorded_traffic("in_proj", wl.name, "gemm"),
            "kernel": "gemm_kernel (input projection)",
            "ms": ms_in, "flops": fl_in, "peak_source": peaks["source"] + " burst"}
    # ---- end to end: every step copies the hidden state in from pinned host
    # memory and reads both layers' outputs back, pipelined over two device
    # buffers and three streams (copy in, compute, copy out) as in the mixer
    # prefill line
    e2e = None
    if not args.no_e2e:
        host_h = hidden.cpu().pin_memory()
        host_out = [torch.empty(host_h.shape, dtype=host_h.dtype).pin_memory() for _ in range(2)]
        sets = [{"h": hidden if j == 0 else torch.empty_like(hidden), "in_done": torch.cuda.Event(),
                 "comp_done": torch.cuda.Event()} for j in range(2)]
        s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_step(i):
            st = sets[i % 2]
            if i >= 2:
                s_in.wait_event(st["comp_done"])     # step i-2 has read this buffer
            with torch.cuda.stream(s_in):
                st["h"].copy_(host_h, non_blocking=True)
                st["in_done"].record(s_in)
            s_comp.wait_event(st["in_done"])
            with torch.cuda.stream(s_comp):
                m_out = layers.mamba_layer_prefill(st["h"], mw)[0]
                w_out = layers.swa_layer_prefill(st["h"], sw)[0]
                st["comp_done"].record(s_comp)
            s_out.wait_event(st["comp_done"])
            with torch.cuda.stream(s_out):
                for t_, h_ in ((m_out, host_out[0]), (w_out, host_out[1])):
                    t_.record_stream(s_out)           # not reused before this copy has run
                    h_.copy_(t_, non_blocking=True)

        e2e_step(0)
        e2e_step(1)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(4, args.e2e_steps)
        a.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        b.record(s_out)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(a.elapsed_time(b) / n_e2e, dev)
        nb = host_h.numel() * host_h.element_size()
        e2e = {"value": whole_job_rate(wl.batch * wl.seqlen, world, ms_e2e), "unit": UNIT,
               "h2d_bytes_per_step": nb, "d2h_bytes_per_step": 2 * nb, "ms_per_step": ms_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with oracle_pool() as pool:
            v, cores, sample = oracle_layers_throughput(wl, pool)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
    cfg = workload_config(wl)
    cfg.update({"d_model": wl.d_model, "dt_rank": wl.dt_rank,
                "layer_gemm_flops_per_step": layer_gemm_flops(wl)})
    return {
        "metric": LAYERS_METRIC, "value": whole_job_rate(wl.batch * wl.seqlen, world, ms_step), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (random weights of the layer shapes)", "config": cfg, "roofline": roof,
        "cpu_baseline": cpu, "e2e": e2e, "clocks": clk, "gpu_launches": 11 * args.steps,
        "status": ops.get_status(),
    }


# ------------------------------------------------------------ serving GPU leg
def serve_gemm_shapes(wl):
    """(name, N, K, output bytes per element; 0 for mixed outputs) of every
    projection of one layer pair, in the order a decode step runs them."""
    D, N, R, dm = wl.dim, wl.dstate, wl.dt_rank, wl.d_model
    nq, nk = wl.heads_q * wl.head_dim, wl.heads_kv * wl.head_dim
    return [("in_proj", 2 * D, dm, 2), ("x_proj", R + 2 * N, D, 0), ("dt_proj", D, R, 4), ("out_proj", dm, D, 2),
            ("qkv_proj", nq + 2 * nk, dm, 2), ("o_proj", dm, nq, 2)]


def serve_step_bytes(wl):
    """Algorithmic HBM bytes of one decode step of the stack for the whole
    batch, per kernel class summed over the pairs: each projection reads its
    weights once and its [B, K] bf16 input and writes its [B, N] output (x_proj
    writes the rank-R part in bf16 and B, C in fp32; dt_proj writes fp32 and
    reads its bias); the conv step reads x and writes u (bf16), reads and
    writes the conv state and reads its weights and bias; the scan step is the
    mixer's decode step without the conv (u in instead of x, no conv state or
    conv weights, the dt bias not read); the SWA step as the mixer's."""
    Bsz, D, N, K, R = wl.batch, wl.dim, wl.dstate, wl.dconv, wl.dt_rank
    out = {}
    for name, n, k, ob in serve_gemm_shapes(wl):
        if name == "x_proj":
            wr = Bsz * (R * 2 + 2 * N * 4)
        elif name == "dt_proj":
            wr = Bsz * n * 4 + n * 4
        else:
            wr = Bsz * n * ob
        out[name] = SERVE_PAIRS * (n * k * 2 + Bsz * k * 2 + wr)
    out["conv"] = SERVE_PAIRS * (2 * Bsz * D * (K - 1) * 4 + Bsz * D * 2 * 2 + D * (K + 1) * 4)
    sb, wb = decode_bytes(wl)
    # the layer's scan step takes u (bf16) instead of x and fuses no conv
    out["scan_step"] = SERVE_PAIRS * (sb - 2 * Bsz * D * (K - 1) * 4 - D * (K + 2) * 4 + D * 4)
    # (decode_bytes counts D (K + 2) fp32 for the conv weights, the conv bias
    # and the skip D; the layer's scan step reads only the skip)
    out["swa_step"] = SERVE_PAIRS * wb
    return out


def run_serve(args, wl, dev, rank, world):
    """The prefill-to-decode serving loop of a layer stack: SERVE_PAIRS Mamba
    + SWA layer pairs (random weights of the layer shapes), a 4096-token
    prompt per sequence through every layer's prefill, then decode steps of
    one token per sequence through the whole stack (each layer's output the
    next layer's input; the tokens' input rows are seeded, as the embeddings
    of a given continuation would be), 32 steps per CUDA graph."""
    import torch
    import torch.distributed as dist

    from hybrid_ssm_sliding_b200 import layers, ops

    wl_rank = rank_workload(wl, rank)
    Bsz, dm, W = wl.batch, wl.d_model, wl.window
    stack = []
    for i in range(SERVE_PAIRS):
        stack.append(("mamba", layers.random_mamba_weights(dm, wl.dim, wl.dstate, wl.dconv, wl.dt_rank,
                                                           wl_rank.seed + 10 * i, dev)))
        stack.append(("swa", layers.random_swa_weights(dm, wl.heads_q, wl.heads_kv, wl.head_dim, W,
                                                       wl_rank.seed + 10 * i + 1, dev)))
    g = torch.Generator(device=dev)
    g.manual_seed(wl_rank.seed + 2)
    prompt = torch.randn((Bsz, wl.seqlen, dm), generator=g, device=dev).to(torch.bfloat16)
    G = DECODE_GRAPH_STEPS
    tokens = torch.randn((G, Bsz, dm), generator=g, device=dev).to(torch.bfloat16)
    stream = torch.cuda.current_stream()

    def prefill():
        states, h = [], prompt
        for kind, w in stack:
            if kind == "mamba":
                h, hf, cs = layers.mamba_layer_prefill(h, w)
                states.append(layers.mamba_decode_state(hf, cs, w))
            else:
                h, k, v = layers.swa_layer_prefill(h, w)
                states.append(layers.swa_decode_state(k, v, w))
        return states, h

    prefill()
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    states, _ = prefill()
    p1.record(stream)
    torch.cuda.synchronize()
    ms_prefill = p0.elapsed_time(p1)
    del prompt

    def decode_step(x, st=states):
        for (kind, w), s_ in zip(stack, st):
            x = (layers.mamba_layer_step if kind == "mamba" else layers.swa_layer_step)(x, w, s_)
        return x

    # warm-up outside capture (first-call setup)
    for j in range(2):
        decode_step(tokens[j])
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        outs = [decode_step(tokens[j]) for j in range(G)]
    reps = args.graphs if args.graphs > 0 else max(4, min(64, wl.decode_steps // G // 32))
    for _ in range(max(1, args.warmup)):
        graph.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(e0.elapsed_time(e1), dev)
    clk = clocks.stop()
    n_steps = reps * G
    ms_step = ms_total / n_steps
    value = whole_job_rate(Bsz, world, ms_step)
    status = ops.get_status()

    # each kernel class alone: the same calls as one decode step makes, over
    # every pair, G steps per graph
    mam = [w for kind, w in stack if kind == "mamba"]
    swl = [w for kind, w in stack if kind == "swa"]
    mst = [s_ for (kind, _), s_ in zip(stack, states) if kind == "mamba"]
    sst = [s_ for (kind, _), s_ in zip(stack, states) if kind == "swa"]
    D, N, R = wl.dim, wl.dstate, wl.dt_rank
    nq, nk = wl.heads_q * wl.head_dim, wl.heads_kv * wl.head_dim

    def bf(*shape):
        return torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)

    x_in, u_in, dtl_in, y_in, o_in = bf(Bsz, dm), bf(Bsz, D), bf(Bsz, R), bf(Bsz, D), bf(Bsz, nq)
    xz_out = torch.empty((Bsz, 2 * D), dtype=torch.bfloat16, device=dev)
    dl_out = torch.empty((Bsz, R), dtype=torch.bfloat16, device=dev)
    bc_out = torch.empty((Bsz, 2 * N), dtype=torch.float32, device=dev)
    delta_out = torch.empty((Bsz, D), dtype=torch.float32, device=dev)
    dm_out = torch.empty((Bsz, dm), dtype=torch.bfloat16, device=dev)
    qkv_out = torch.empty((Bsz, nq + 2 * nk), dtype=torch.bfloat16, device=dev)
    u_out = torch.empty((Bsz, D), dtype=torch.bfloat16, device=dev)
    y_out = torch.empty((Bsz, D), dtype=torch.bfloat16, device=dev)
    o_out = torch.empty((Bsz, wl.heads_q, wl.head_dim), dtype=torch.bfloat16, device=dev)
    delta_in = torch.full((Bsz, D), -3.0, device=dev)
    b_in = torch.randn((Bsz, N), generator=g, device=dev)
    c_in = torch.randn((Bsz, N), generator=g, device=dev)
    q_in, kv_in = bf(Bsz, wl.heads_q, wl.head_dim), bf(Bsz, wl.heads_kv, wl.head_dim)
    kernels = {
        "in_proj": lambda i: ops.gemm(x_in, mam[i].in_proj, outs=[(xz_out, 0, 2 * D, None)],
                                      workspace=mst[i].gemm_ws),
        "x_proj": lambda i: ops.gemm(u_in, mam[i].x_proj, outs=[(dl_out, 0, R, None),
                                                                 (bc_out, R, R + 2 * N, None)],
                                     workspace=mst[i].gemm_ws),
        "dt_proj": lambda i: ops.gemm(dtl_in, mam[i].dt_proj, outs=[(delta_out, 0, D, mam[i].dt_bias)],
                                      workspace=mst[i].gemm_ws),
        "out_proj": lambda i: ops.gemm(y_in, mam[i].out_proj, outs=[(dm_out, 0, dm, None)],
                                       workspace=mst[i].gemm_ws),
        "qkv_proj": lambda i: ops.gemm(x_in, swl[i].qkv_proj, outs=[(qkv_out, 0, nq + 2 * nk, None)],
                                       workspace=sst[i].gemm_ws),
        "o_proj": lambda i: ops.gemm(o_in, swl[i].o_proj, outs=[(dm_out, 0, dm, None)], workspace=sst[i].gemm_ws),
        "conv": lambda i: ops.conv1d_fwd(u_in.view(Bsz, 1, D), mam[i].conv_w, mam[i].conv_b,
                                         conv_state_in=mst[i].conv, conv_state_out=mst[i].conv,
                                         u=u_out.view(Bsz, 1, D)),
        "scan_step": lambda i: ops.scan_step(mst[i].h, None, u_in, delta_in, mam[i].A, b_in, c_in, D=mam[i].D,
                                             z_t=y_in, y_t=y_out),
        "swa_step": lambda i: ops.swa_step(q_in, kv_in, kv_in, sst[i].k_ring, sst[i].v_ring, sst[i].pos, W,
                                           o_t=o_out, workspace=sst[i].workspace),
    }
    nbytes = serve_step_bytes(wl)
    peaks = load_peaks()
    kern = {}
    for name, fn in kernels.items():
        for i in range(SERVE_PAIRS):
            fn(i)
        torch.cuda.synchronize()
        kg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(kg):
            for _ in range(G):
                for i in range(SERVE_PAIRS):
                    fn(i)
        kg.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = max(4, reps // 2)
        a.record(stream)
        for _ in range(n):
            kg.replay()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / (n * G)            # per decode step, all pairs
        gbs = nbytes[name] / (ms / 1e3) / 1e9
        # DRAM bytes per step where a capture of this class's kernel in this
        # workload is recorded: per launch, times the launches of a step
        per_launch = recorded_traffic(name, wl.name, "misc") if name in ("swa_step", "scan_step") else None
        kern[name] = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                      "frac": gbs / peaks["hbm_gbs"],
                      "traffic": per_launch * SERVE_PAIRS if per_launch is not None else None, "ms_per_step": ms,
                      "algorithmic_bytes_per_step": nbytes[name], "peak_source": peaks["source"]}
        del kg
    dom = max(kern, key=lambda k: kern[k]["ms_per_step"])
    roofline = {k: kern[dom][k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
    roofline["kernel"] = dom
    total_bytes = sum(nbytes.values())
    step_gbs = total_bytes / (ms_step / 1e3) / 1e9
    whole = {"achieved": step_gbs, "frac": step_gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_step": total_bytes}

    # end to end through the layer API: every step copies its token rows from
    # pinned host memory and reads the stack's output back, 32 steps per graph,
    # pipelined over two input buffers and three streams (copy in, compute,
    # copy out): the rows of step j+1 arrive and the output of step j-1 leaves
    # while step j computes.  Each step's output tensor stays referenced until
    # the graph is released, so no later step's allocation reuses it before
    # its copy out has run.
    e2e = None
    if not args.no_e2e:
        host_in = [tokens[j].cpu().pin_memory() for j in range(G)]
        host_out = [torch.empty((Bsz, dm), dtype=torch.bfloat16).pin_memory() for _ in range(G)]
        dev_in = [torch.empty((Bsz, dm), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_steps():
            cur = torch.cuda.current_stream()
            for st_ in (s_in, s_comp, s_out):
                st_.wait_stream(cur)
            kept = []
            for j in range(G):
                b_ = j % 2
                if j >= 2:
                    s_in.wait_event(ev_comp[b_])        # step j-2 has read this input buffer
                with torch.cuda.stream(s_in):
                    dev_in[b_].copy_(host_in[j], non_blocking=True)
                    ev_in[b_].record(s_in)
                s_comp.wait_event(ev_in[b_])
                with torch.cuda.stream(s_comp):
                    out = decode_step(dev_in[b_])
                    ev_comp[b_].record(s_comp)
                kept.append(out)
                s_out.wait_event(ev_comp[b_])
                with torch.cuda.stream(s_out):
                    host_out[j].copy_(out, non_blocking=True)
            for st_ in (s_in, s_comp, s_out):
                cur.wait_stream(st_)
            return kept

        e2e_steps()
        torch.cuda.synchronize()
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e):
            kept_outs = e2e_steps()
        g_e2e.replay()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        n_rep = max(4, reps // 4)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_rep):
            g_e2e.replay()
        b.record(stream)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(a.elapsed_time(b) / (n_rep * G), dev)
        e2e = {"value": whole_job_rate(Bsz, world, ms_e2e), "unit": UNIT, "h2d_bytes_per_step": Bsz * dm * 2,
               "d2h_bytes_per_step": Bsz * dm * 2, "ms_per_step": ms_e2e}
        del g_e2e, kept_outs
    del graph, outs

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with oracle_pool() as pool:
            v, cores, sample = oracle_serve_throughput(wl, pool)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
    cfg = workload_config(wl)
    state_bytes = SERVE_PAIRS * (Bsz * D * N * 4 + 2 * Bsz * D * (wl.dconv - 1) * 4
                                 + 2 * Bsz * W * wl.heads_kv * wl.head_dim * 2)
    weight_bytes = SERVE_PAIRS * sum(n * k * 2 for _, n, k, _ in serve_gemm_shapes(wl))
    cfg.update({"d_model": dm, "dt_rank": R, "layer_pairs": SERVE_PAIRS, "prompt_tokens": wl.seqlen,
                "graph_steps": G, "prefill_ms": ms_prefill,
                "prefill_tokens_per_s": whole_job_rate(Bsz * wl.seqlen, 1, ms_prefill),
                "l2": f"inputs larger than L2: every step reads the stack's weights ({weight_bytes / 1e6:.0f} MB) "
                      f"and states ({state_bytes / 1e6:.0f} MB)"})
    per_pair_launches = 6 + 4       # Mamba: 4 GEMMs, the conv step, the scan step; SWA: 2 GEMMs, the 2-kernel SWA step
    return {
        "metric": SERVE_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": n_steps,
        "warmup": max(1, args.warmup) * G, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (random weights of the layer shapes)",
        "config": cfg, "roofline": roofline, "step_roofline": whole, "kernels": kern, "cpu_baseline": cpu,
        "e2e": e2e, "clocks": clk, "gpu_launches": n_steps * SERVE_PAIRS * per_pair_launches, "status": status,
    }


TRAIN_METRIC = "Samba mixer training step tokens/s (forward + backward of the selective scan and SWA)"


def swa_bwd_flops(wl):
    """Band FLOPs of the attention backward: the five products of the chain
    rule (S recomputed, dP, dV, dK, dQ), each 2·L·W·d per (batch, query head)
    on the band, i.e. 10·L·W·d (the forward's 4·L·W·d is two of them)."""
    return 10.0 * wl.batch * wl.heads_q * wl.seqlen * wl.window * wl.head_dim


def scan_bwd_bytes(wl):
    """HBM bytes the scan backward must move once: x, z, dy (bf16) and delta
    (fp32) in, dx, dz (bf16) and ddelta (fp32) out per (token, channel); B, C
    in and dB, dC out per token; the per-channel parameters and gradients."""
    tc = wl.batch * wl.seqlen * wl.dim
    per_token = 4 * wl.dstate * 4
    small = wl.dim * (wl.dstate + wl.dconv + 2) * 4 * 2
    return tc * (2 + 2 + 2 + 4 + 2 + 2 + 4) + wl.batch * wl.seqlen * per_token + small


def run_train(args, wl, dev, rank, world):
    """Times one training step of the two mixers: the fused scan and SWA
    forwards (with the attention's log-sum-exp) and both backwards from
    seeded output gradients."""
    import torch
    import torch.distributed as dist

    from hybrid_ssm_sliding_b200 import ops
    from hybrid_ssm_sliding_b200.workloads import make_output_grads, make_prefill_inputs

    wl_rank = rank_workload(wl, rank)
    inp = make_prefill_inputs(wl_rank, device=dev)
    grads = make_output_grads(wl_rank, device=dev)
    Bsz, Ln, D, N, K = wl.batch, wl.seqlen, wl.dim, wl.dstate, wl.dconv
    y = torch.empty((Bsz, Ln, D), dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(inp["q"])
    lse = torch.empty((Bsz, wl.heads_q, Ln), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(inp["q"]), torch.empty_like(inp["k"]), torch.empty_like(inp["v"])
    ws_scan = torch.empty((ops.scan_bwd_workspace_size(Bsz, Ln, D, N),), dtype=torch.uint8, device=dev)
    ws_swa = torch.empty((ops.swa_bwd_workspace_size(Bsz, Ln, wl.heads_q),), dtype=torch.uint8, device=dev)
    scan_in = dict(D=inp["D"], z=inp["z"], conv_w=inp["conv_w"], conv_b=inp["conv_b"])
    # the forward stores the state at every 16-token chunk start; the
    # backward starts its chunks from them instead of recomputing them
    ckpt = torch.empty(ops.scan_ckpt_shape(Bsz, Ln, D, N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def fwd():
        ops.selective_scan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], y=y, h_ckpt=ckpt, **scan_in)
        ops.swa_fwd(inp["q"], inp["k"], inp["v"], wl.window, o=o, lse=lse)

    def bwd_scan():
        return ops.selective_scan_bwd(grads["dy"], inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                      workspace=ws_scan, ckpt=ckpt, **scan_in)

    def bwd_swa():
        ops.swa_bwd(grads["do"], inp["q"], inp["k"], inp["v"], o, lse, wl.window, dq=dq, dk=dk, dv=dv,
                    workspace=ws_swa)

    aux = torch.cuda.Stream()

    def train_step(ins, gr):
        """Forward and backward of both mixers on the activations `ins` and
        output gradients `gr` (the parameters A, D and the conv stay put);
        returns the scan's and the attention's gradients."""
        sin = dict(scan_in, z=ins["z"])
        ops.selective_scan_fwd(ins["x"], ins["delta"], inp["A"], ins["B"], ins["C"], y=y, h_ckpt=ckpt, **sin)
        ops.swa_fwd(ins["q"], ins["k"], ins["v"], wl.window, o=o, lse=lse)
        # the two backward passes are independent: the attention's runs on a
        # second stream and takes the SMs the scan's last wave leaves free
        return ops.mixer_bwd(dict(dy=gr["dy"], x=ins["x"], delta=ins["delta"], A=inp["A"], B=ins["B"], C=ins["C"],
                                  workspace=ws_scan, ckpt=ckpt, **sin),
                             dict(do=gr["do"], q=ins["q"], k=ins["k"], v=ins["v"], o=o, lse=lse, window=wl.window,
                                  dq=dq, dk=dk, dv=dv, workspace=ws_swa),
                             aux_stream=aux)

    def step():
        train_step(inp, grads)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(e0.elapsed_time(e1), dev)
    clk = clocks.stop()
    ms_step = ms_total / args.steps

    def timed(fn, n):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    n = max(5, args.kernel_steps // 5)
    ms_fwd, ms_bscan, ms_bswa = timed(fwd, n), timed(bwd_scan, n), timed(bwd_swa, n)
    peaks = load_peaks()
    fl = swa_bwd_flops(wl)
    swa_tfs = fl / (ms_bswa / 1e3) / 1e12
    sb = scan_bwd_bytes(wl)
    scan_gbs = sb / (ms_bscan / 1e3) / 1e9
    kernels = {
        "swa_bwd": {"bound": "tensor", "achieved": swa_tfs, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": swa_tfs / peaks["bf16_tflops"], "traffic": None, "ms": ms_bswa, "band_flops": fl,
                    "peak_source": peaks["source"] + " burst"},
        "scan_bwd": {"bound": "hbm", "achieved": scan_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": scan_gbs / peaks["hbm_gbs"],
                     "traffic": recorded_traffic("scan_bwd", wl.name, "scan_bwd"), "ms": ms_bscan,
                     "algorithmic_bytes": sb, "peak_source": peaks["source"]},
    }
    dom = "scan_bwd" if ms_bscan >= ms_bswa else "swa_bwd"
    roof = {k: kernels[dom][k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
    roof["kernel"] = "scan_bwd_kernel" if dom == "scan_bwd" else "swa_bwd_kv_kernel + swa_bwd_q_kernel"
    # ---- end to end: every step copies its activations (x, z, delta, B, C,
    # q, k, v) and output gradients (dy, dO) in from pinned host memory and
    # reads the parameters' gradients (dA, dD, dconv_w, dconv_b) back; the
    # activations' gradients stay on the device for the layer below.
    # Pipelined over two device buffer sets and three streams (copy in,
    # compute, copy out) as in the mixer prefill line.
    e2e = None
    if not args.no_e2e:
        act_keys, grad_keys = ("x", "z", "delta", "B", "C", "q", "k", "v"), ("dy", "do")
        param_grads = ("dA", "dD", "dconv_w", "dconv_b")
        host_act = {k: inp[k].cpu().pin_memory() for k in act_keys}
        host_gr = {k: grads[k].cpu().pin_memory() for k in grad_keys}
        sets = []
        for j in range(2):
            sets.append({"ins": {k: inp[k] if j == 0 else torch.empty_like(inp[k]) for k in act_keys},
                         "gr": {k: grads[k] if j == 0 else torch.empty_like(grads[k]) for k in grad_keys},
                         "in_done": torch.cuda.Event(), "comp_done": torch.cuda.Event()})
        e2e_sg = train_step(inp, grads)[0]
        host_pg = {k: torch.empty(e2e_sg[k].shape, dtype=e2e_sg[k].dtype).pin_memory() for k in param_grads}
        s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_step(i):
            st = sets[i % 2]
            if i >= 2:
                s_in.wait_event(st["comp_done"])     # step i-2 has read these buffers
            with torch.cuda.stream(s_in):
                for k in act_keys:
                    st["ins"][k].copy_(host_act[k], non_blocking=True)
                for k in grad_keys:
                    st["gr"][k].copy_(host_gr[k], non_blocking=True)
                st["in_done"].record(s_in)
            s_comp.wait_event(st["in_done"])
            with torch.cuda.stream(s_comp):
                sg = train_step(st["ins"], st["gr"])[0]
                st["comp_done"].record(s_comp)
            s_out.wait_event(st["comp_done"])
            with torch.cuda.stream(s_out):
                for k in param_grads:
                    sg[k].record_stream(s_out)         # not reused before this copy has run
                    host_pg[k].copy_(sg[k], non_blocking=True)

        e2e_step(0)
        e2e_step(1)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(4, args.e2e_steps)
        a.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        b.record(s_out)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(a.elapsed_time(b) / n_e2e, dev)
        h2d = sum(t.numel() * t.element_size() for t in list(host_act.values()) + list(host_gr.values()))
        d2h = sum(t.numel() * t.element_size() for t in host_pg.values())
        e2e = {"value": whole_job_rate(wl.batch * wl.seqlen, world, ms_e2e), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with oracle_pool() as pool:
            v, cores, sample = oracle_train_throughput(wl, pool)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
    cfg = workload_config(wl)
    cfg["step"] = ("scan and SWA forward (with log-sum-exp and the scan's 16-token state checkpoints), then scan "
                   "and SWA backward from seeded dy, dO (samba_mixer_bwd, the SWA backward on a second stream)")
    return {
        "metric": TRAIN_METRIC, "value": whole_job_rate(wl.batch * wl.seqlen, world, ms_step), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": cfg, "roofline": roof, "kernels": kernels,
        "phases_ms": {"forward": ms_fwd, "scan_backward": ms_bscan, "swa_backward": ms_bswa},
        "cpu_baseline": cpu, "e2e": e2e, "clocks": clk, "gpu_launches": 7 * args.steps,
        "status": ops.get_status(),
    }


# ------------------------------------------------------------ decode GPU leg
def run_decode(args, wl, lib, dev, rank, world):
    """Times decode steps (scan step + SWA step over the whole batch) in
    CUDA graphs of DECODE_GRAPH_STEPS steps; returns the JSON line."""
    import torch
    import torch.distributed as dist

    from hybrid_ssm_sliding_b200 import _lib as L
    from hybrid_ssm_sliding_b200 import build as B
    from hybrid_ssm_sliding_b200 import ops
    from hybrid_ssm_sliding_b200.workloads import make_decode_step_inputs, make_prefill_inputs

    wl_rank = rank_workload(wl, rank)
    Bsz, D, N, K = wl.batch, wl.dim, wl.dstate, wl.dconv
    # state after a prefill of wl.seqlen tokens, through the library itself
    pre = make_prefill_inputs(wl_rank, device=dev)
    h = torch.empty((Bsz, D, N), dtype=torch.float32, device=dev)
    cs = torch.empty((Bsz, D, K - 1), dtype=torch.float32, device=dev)
    ops.selective_scan_fwd(pre["x"], pre["delta"], pre["A"], pre["B"], pre["C"], D=pre["D"], z=pre["z"],
                           conv_w=pre["conv_w"], conv_b=pre["conv_b"], h_final=h, conv_state_out=cs,
                           y_dtype=torch.bfloat16)
    k_ring, v_ring, pos = ops.swa_ring_fill(pre["k"], pre["v"], wl.window)
    A, Dsk, cw, cb = pre["A"], pre["D"], pre["conv_w"], pre["conv_b"]
    del pre
    NLY = DECODE_LAYERS
    layers = [dict(h=h.clone(), cs=cs.clone(), k_ring=k_ring.clone(), v_ring=v_ring.clone(), pos=pos.clone())
              for _ in range(NLY)]
    del h, cs, k_ring, v_ring, pos
    G = DECODE_GRAPH_STEPS
    steps_in = [make_decode_step_inputs(wl_rank, s, device=dev) for s in range(G)]
    y_t = torch.empty((Bsz, D), dtype=torch.bfloat16, device=dev)
    o_t = torch.empty((Bsz, wl.heads_q, wl.head_dim), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros((max(ops.swa_step_workspace_size(Bsz, wl.heads_q, wl.head_dim, wl.window), 16),),
                     dtype=torch.uint8, device=dev)

    def scan_one(si, ly, y_out=None):
        ops.scan_step(ly["h"], ly["cs"], si["x"], si["delta"], A, si["B"], si["C"], D=Dsk, z_t=si["z"], conv_w=cw,
                      conv_b=cb, y_t=y_t if y_out is None else y_out)

    def swa_one(si, ly, o_out=None):
        ops.swa_step(si["q"], si["k"], si["v"], ly["k_ring"], ly["v_ring"], ly["pos"], wl.window,
                     o_t=o_t if o_out is None else o_out, workspace=ws)

    def capture(body):
        for s_ in range(2):  # warm-up outside capture (first-call setup, attributes)
            body(steps_in[s_], layers[s_ % NLY])
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for s_, si in enumerate(steps_in):
                body(si, layers[s_ % NLY])
        return g

    # One decode step of the mixer pair: the two mixers' steps are independent
    # (each reads its own inputs and state), so the SWA step is forked onto a
    # second stream and both are joined before the next step starts, as the
    # mixer prefill's two-stream form does.  The SWA step is issued first: its
    # CTAs take their four slots per SM, and the scan step's CTAs run in the
    # threads and registers left beside them (issued the other way round, the
    # scan step's CTAs fill the SMs and the SWA step waits for them).  The same
    # steps on one stream are timed too.
    aux = torch.cuda.Stream()

    def step_pair(si, ly, y_out=None, o_out=None):
        cur = torch.cuda.current_stream()
        aux.wait_stream(cur)
        with torch.cuda.stream(aux):
            swa_one(si, ly, o_out)
        scan_one(si, ly, y_out)
        cur.wait_stream(aux)

    g_step = capture(step_pair)
    g_one_stream = capture(lambda si, ly: (scan_one(si, ly), swa_one(si, ly)))
    g_scan = capture(scan_one)
    g_swa = capture(swa_one)
    stream = torch.cuda.current_stream()
    reps = args.graphs if args.graphs > 0 else max(1, wl.decode_steps // G)
    for _ in range(max(1, args.warmup)):
        g_step.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g_step.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(e0.elapsed_time(e1), dev)
    clk = clocks.stop()
    n_steps = reps * G
    ms_step = ms_total / n_steps
    value = whole_job_rate(Bsz, world, ms_step)

    def time_graph(g, n=max(4, reps // 2)):
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / (n * G)

    ms_scan = time_graph(g_scan)
    ms_swa = time_graph(g_swa)
    ms_one_stream = time_graph(g_one_stream)
    status = ops.get_status()
    peaks = load_peaks()
    sb, wb = decode_bytes(wl)
    kern = {}
    for name, ms, nb in (("scan_step", ms_scan, sb), ("swa_step", ms_swa, wb)):
        gbs = nb / (ms / 1e3) / 1e9
        kern[name] = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                      "frac": gbs / peaks["hbm_gbs"], "traffic": recorded_traffic(name, wl.name, "misc"),
                      "ms": ms, "algorithmic_bytes": nb, "peak_source": peaks["source"]}
    dom = "swa_step" if ms_swa >= ms_scan else "scan_step"
    roofline = {k: kern[dom][k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
    roofline["kernel"] = dom

    # end to end: every step copies its inputs from pinned host memory (all of
    # a step's inputs packed in one buffer, one copy) and reads y_t and o_t
    # back (one copy), around the library calls; 32 steps in a CUDA graph.
    # The steps are pipelined over two device buffer sets and three streams
    # (copy in, compute, copy out), as a serving loop would run them: the
    # inputs of step s+1 arrive and the outputs of step s-1 leave while step
    # s computes.
    e2e = None
    if not args.no_e2e:
        keys = list(steps_in[0].keys())

        def nbytes(t):
            return t.numel() * t.element_size()

        offs, off = {}, 0
        for k in keys:
            offs[k] = off
            off += (nbytes(steps_in[0][k]) + 255) // 256 * 256
        pack_bytes = off
        host_packs = []
        for si in steps_in:
            hp = torch.zeros(pack_bytes, dtype=torch.uint8).pin_memory()
            for k in keys:
                hp[offs[k]:offs[k] + nbytes(si[k])].copy_(si[k].cpu().reshape(-1).view(torch.uint8))
            host_packs.append(hp)
        y_bytes = (nbytes(y_t) + 255) // 256 * 256
        sets = []
        for j in range(2):
            dev_pack = torch.empty(pack_bytes, dtype=torch.uint8, device=dev)
            out_pack = torch.empty(y_bytes + nbytes(o_t), dtype=torch.uint8, device=dev)
            sets.append({
                "pack": dev_pack,
                "in": {k: dev_pack[offs[k]:offs[k] + nbytes(steps_in[0][k])].view(steps_in[0][k].dtype)
                       .view(steps_in[0][k].shape) for k in keys},
                "out": out_pack,
                "y": out_pack[:nbytes(y_t)].view(y_t.dtype).view(y_t.shape),
                "o": out_pack[y_bytes:].view(o_t.dtype).view(o_t.shape),
                "in_done": torch.cuda.Event(), "comp_done": torch.cuda.Event(), "out_done": torch.cuda.Event()})
        host_out = torch.empty(sets[0]["out"].numel(), dtype=torch.uint8).pin_memory()
        h2d, d2h = pack_bytes, sets[0]["out"].numel()
        s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_steps():
            cur = torch.cuda.current_stream()
            for st in (s_in, s_comp, s_out):
                st.wait_stream(cur)
            for s_ in range(G):
                st, ly = sets[s_ % 2], layers[s_ % NLY]
                if s_ >= 2:
                    s_in.wait_event(st["comp_done"])     # step s-2 has read this input pack
                with torch.cuda.stream(s_in):
                    st["pack"].copy_(host_packs[s_], non_blocking=True)
                    st["in_done"].record(s_in)
                s_comp.wait_event(st["in_done"])
                if s_ >= 2:
                    s_comp.wait_event(st["out_done"])    # the outputs of step s-2 have been read back
                with torch.cuda.stream(s_comp):
                    step_pair(st["in"], ly, st["y"], st["o"])
                    st["comp_done"].record(s_comp)
                s_out.wait_event(st["comp_done"])
                with torch.cuda.stream(s_out):
                    host_out.copy_(st["out"], non_blocking=True)
                    st["out_done"].record(s_out)
            for st in (s_in, s_comp, s_out):
                cur.wait_stream(st)

        e2e_steps()
        torch.cuda.synchronize()
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e):
            e2e_steps()
        g_e2e.replay()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        n_rep = max(4, reps // 16)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_rep):
            g_e2e.replay()
        b.record(stream)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(a.elapsed_time(b) / (n_rep * G), dev)
        e2e = {"value": whole_job_rate(Bsz, world, ms_e2e), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with oracle_pool() as pool:
            v, cores, sample = oracle_decode_throughput(wl, pool)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
    cfg = workload_config(wl)
    sb_state = Bsz * D * N * 4 + Bsz * D * (K - 1) * 4
    ring_bytes = Bsz * wl.window * wl.heads_kv * wl.head_dim * 2
    cfg.update({"prefill_tokens": wl.seqlen, "graph_steps": G, "layers": NLY,
                "step": "scan step, and the SWA step forked onto a second stream, joined before the next step",
                "l2": f"inputs larger than L2: {NLY} layer states (scan state, conv state, K/V rings; "
                      f"{NLY * (sb_state + 2 * ring_bytes) / 1e6:.0f} MB) rotate from step to step"})
    return {
        "metric": DECODE_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": n_steps,
        "warmup": max(1, args.warmup) * G, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg, "roofline": roofline,
        "kernels": kern, "one_stream_ms_per_step": ms_one_stream, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
        "gpu_launches": n_steps * 3, "status": status,
    }


# -------------------------------------------------------------------- GPU leg
def main():
    args = parse()
    if args.impl == "reference":
        sys.exit(run_reference(args))

    import torch
    import torch.distributed as dist

    from hybrid_ssm_sliding_b200 import _lib as L
    from hybrid_ssm_sliding_b200 import build as B
    from hybrid_ssm_sliding_b200 import ops
    from hybrid_ssm_sliding_b200.workloads import WORKLOADS, make_prefill_inputs

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)
    if local == 0:
        B.build()
    if world > 1:
        dist.barrier()
    lib = L.load()

    wl = WORKLOADS[args.workload]
    if wl.train:
        line = run_train(args, wl, dev, rank, world)
        if rank == 0:
            print(json.dumps(line))
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    if wl.d_model > 0:
        line = (run_serve if wl.decode_steps > 0 else run_layers)(args, wl, dev, rank, world)
        if rank == 0:
            print(json.dumps(line))
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    if wl.decode_steps > 0:
        line = run_decode(args, wl, lib, dev, rank, world)
        if rank == 0:
            print(json.dumps(line))
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    wl_rank = rank_workload(wl, rank)   # each rank its own batch
    inp = make_prefill_inputs(wl_rank, device=dev)
    Bsz, Ln, D, N, K = wl.batch, wl.seqlen, wl.dim, wl.dstate, wl.dconv
    y = torch.empty((Bsz, Ln, D), dtype=torch.bfloat16, device=dev)
    h_final = torch.empty((Bsz, D, N), dtype=torch.float32, device=dev)
    cs_out = torch.empty((Bsz, D, K - 1), dtype=torch.float32, device=dev)
    o = torch.empty_like(inp["q"])
    scan_kw = dict(x=inp["x"], delta=inp["delta"], A=inp["A"], B=inp["B"], C=inp["C"], D=inp["D"], z=inp["z"],
                   conv_w=inp["conv_w"], conv_b=inp["conv_b"], y=y, h_final=h_final, conv_state_out=cs_out)
    swa_kw = dict(q=inp["q"], k=inp["k"], v=inp["v"], window=wl.window, o=o)
    sa, _ = ops._scan_struct(**scan_kw)
    wa, _ = ops._swa_struct(**swa_kw)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    def step():
        rc = lib.samba_mixer_prefill(ctypes.byref(sa), ctypes.byref(wa), sh, None)
        if rc != 0:
            L.check(rc)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- timed region: K mixer-prefill steps
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(e0.elapsed_time(e1), dev)
    clk = clocks.stop()
    ms_step = ms_total / args.steps
    value = whole_job_rate(Bsz * Ln, world, ms_step)
    status = ops.get_status()

    # ---- per-kernel times (each kernel alone, back to back, same stream)
    def time_kernel(fn, n):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    ms_scan = time_kernel(lambda: L.check(lib.samba_selective_scan_fwd(ctypes.byref(sa), sh)), args.kernel_steps)
    ms_swa = time_kernel(lambda: L.check(lib.samba_swa_fwd(ctypes.byref(wa), sh)), args.kernel_steps)
    # the same call with the attention forked onto a second stream (reported
    # beside the headline, which runs both mixers on one stream)
    aux = torch.cuda.Stream()
    ms_two_stream = time_kernel(
        lambda: L.check(lib.samba_mixer_prefill(ctypes.byref(sa), ctypes.byref(wa), sh, aux.cuda_stream)),
        args.kernel_steps)
    peaks = load_peaks()
    sb = scan_bytes(wl)
    sf = swa_flops(wl)
    scan_gbs = sb / (ms_scan / 1e3) / 1e9
    swa_tfs = sf / (ms_swa / 1e3) / 1e12
    scan_roof = {"bound": "hbm", "achieved": scan_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                 "frac": scan_gbs / peaks["hbm_gbs"], "traffic": None, "ms": ms_scan,
                 "algorithmic_bytes": sb, "peak_source": peaks["source"]}
    swa_roof = {"bound": "tensor", "achieved": swa_tfs, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": swa_tfs / peaks["bf16_tflops"], "traffic": None, "ms": ms_swa, "band_flops": sf,
                "exact_band_flops": swa_exact_band_flops(wl), "peak_source": peaks["source"] + " burst"}
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = (clk or {}).get("sm_mhz") or (clk or {}).get("sm_max_mhz") or 1965.0
    scan_roof["mufu"] = mufu_roof(scan_mufu_ops(wl), ms_scan, sms, mhz)
    swa_roof["mufu"] = mufu_roof(swa_exps(wl), ms_swa, sms, mhz)
    scan_roof["traffic"] = recorded_traffic("scan", wl.name, "scan_fwd")
    swa_roof["traffic"] = recorded_traffic("swa", wl.name, "swa_fwd")
    dominant = swa_roof if ms_swa >= ms_scan else scan_roof
    roofline = {k: dominant[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
    roofline["kernel"] = "swa_fwd_kernel" if dominant is swa_roof else "scan_fwd_kernel"

    # ---- end to end through the public API with host buffers.  Every step
    # copies its inputs from pinned host memory and reads y and o back; the
    # steps are pipelined over two device buffer sets and three streams
    # (copy in, compute, copy out), as a serving loop would run them.
    e2e = None
    if not args.no_e2e:
        host = {k: v.to("cpu").pin_memory() for k, v in inp.items()}
        y_h = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = y_h.numel() * y_h.element_size() + o_h.numel() * o_h.element_size()
        sets = []
        for j in range(2):
            dev_in = inp if j == 0 else {k: torch.empty_like(v) for k, v in inp.items()}
            y_j = y if j == 0 else torch.empty_like(y)
            o_j = o if j == 0 else torch.empty_like(o)
            skw = dict(scan_kw, y=y_j)
            wkw = dict(swa_kw, o=o_j)
            for kk in ("x", "delta", "A", "B", "C", "D", "z", "conv_w", "conv_b"):
                skw[kk] = dev_in[kk]
            for kk in ("q", "k", "v"):
                wkw[kk] = dev_in[kk]
            sets.append({"in": dev_in, "y": y_j, "o": o_j, "skw": skw, "wkw": wkw,
                         "in_done": torch.cuda.Event(), "comp_done": torch.cuda.Event(),
                         "out_done": torch.cuda.Event()})
        s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_step(i):
            st = sets[i % 2]
            if i >= 2:
                s_in.wait_event(st["comp_done"])     # compute of step i-2 has read these inputs
            with torch.cuda.stream(s_in):
                for kk in host:
                    st["in"][kk].copy_(host[kk], non_blocking=True)
                st["in_done"].record(s_in)
            s_comp.wait_event(st["in_done"])
            if i >= 2:
                s_comp.wait_event(st["out_done"])    # y, o of step i-2 have been read back
            with torch.cuda.stream(s_comp):
                ops.mixer_prefill(st["skw"], st["wkw"])
                st["comp_done"].record(s_comp)
            s_out.wait_event(st["comp_done"])
            with torch.cuda.stream(s_out):
                y_h.copy_(st["y"], non_blocking=True)
                o_h.copy_(st["o"], non_blocking=True)
                st["out_done"].record(s_out)

        e2e_step(0)
        e2e_step(1)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        for i in range(args.e2e_steps):
            e2e_step(i)
        b.record(s_out)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(a.elapsed_time(b) / args.e2e_steps, dev)
        e2e = {"value": whole_job_rate(Bsz * Ln, world, ms_e2e), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with oracle_pool() as pool:
            v, cores, sample = oracle_throughput(wl, pool)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(wl),
            "roofline": roofline, "kernels": {"scan": scan_roof, "swa": swa_roof},
            "two_stream_ms_per_step": ms_two_stream,
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clk, "gpu_launches": 2 * args.steps,
            "status": status,
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
