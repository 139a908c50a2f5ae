"""The oracle baselines of the layer and training bench lines (CPU only):
what each timed unit counts as work, and that both run on the host-core
pool and return a rate, at small widths."""
import dataclasses
import math

import numpy as np

import bench
from hybrid_ssm_sliding_b200.workloads import WORKLOADS


def _band_pairs(L, W):
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    return int(((i - j >= 0) & (i - j < W)).sum())


def test_train_unit_counts_channel_tokens_and_band_pairs():
    # scan: channels x tokens of the sample
    assert bench._oracle_train_unit(("scan", 3, 20, 4, 4, 2, 8, 16, 0)) == 60.0
    # attention: the band's (query, key) pairs over W, i.e. full-window rows;
    # fewer than the rows while the first W rows see partial windows
    for L, W in ((80, 16), (16, 16), (40, 1)):
        got = bench._oracle_train_unit(("swa", 0, L, 4, 4, 2, 8, W, 1))
        assert math.isclose(got, _band_pairs(L, W) / W)
        assert got <= L


def test_layers_unit_counts_tokens():
    dims = (16, 8, 4, 4, 4, 2, 1, 8)   # d_model, D, N, K, R, Hq, Hkv, d
    assert bench._oracle_layers_unit(("mamba", 5) + dims + (0,)) == 5
    assert bench._oracle_layers_unit(("swa_proj", 7) + dims + (1,)) == 7


def _small(name):
    return dataclasses.replace(WORKLOADS[name], dim=64, d_model=32, dt_rank=8, heads_q=4, heads_kv=2, head_dim=16,
                               window=32)


def test_train_and_layers_baselines_run_on_the_pool():
    with bench.oracle_pool() as pool:
        for fn, name in ((bench.oracle_train_throughput, "train_4k"), (bench.oracle_layers_throughput, "layers_128k")):
            rate, cores, sample = fn(_small(name), pool, scale=0.01)
            assert math.isfinite(rate) and rate > 0
            assert cores == bench.host_cores()
            assert "float64" in sample and str(cores) in sample
