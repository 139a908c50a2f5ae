"""GPU parity of the projection GEMM (samba_gemm: C = A · Bᵀ on the tensor
cores, bf16 in, fp32 accumulation, column-split epilogue) against np.matmul
in float64 on the same bf16 inputs, through the C ABI.

Tolerance: each output within one bf16 rounding of the exact value (fp32
outputs: 1e-5 of the magnitude sum_k |a||b| that bounds the accumulation's
rounding), on shapes that span several tiles with ragged M, N and K."""

import numpy as np
import pytest
import torch

from hybrid_ssm_sliding_b200 import build as B
from hybrid_ssm_sliding_b200 import ops
from tests._helpers import host64, record_margin

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def _operands(M, N, K, seed, lda=None):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    a_full = torch.randn((M, lda or K), generator=g, device="cuda").to(torch.bfloat16)
    a = a_full[:, :K]
    w = (torch.randn((N, K), generator=g, device="cuda") / K ** 0.5).to(torch.bfloat16)
    return a, w


def _check(got, ref, mag, dtype, name):
    got = host64(got)
    assert np.all(np.isfinite(got)), "unwritten or non-finite output"
    err = np.abs(got - ref)
    if dtype == torch.bfloat16:
        bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * mag + 1e-30
    else:
        bound = 1e-5 * mag + 1e-30
    worst = float(np.max(err / bound))
    record_margin(name, "C", max_abs=err.max(), worst_over_bound=worst)
    assert worst <= 1.0, f"{name}: error {worst:.2f} x the bound"


@pytest.mark.parametrize("M,N,K,dt", [
    (128, 256, 64, torch.bfloat16),     # one tile
    (300, 200, 100, torch.float32),     # ragged M, N, K (N < 256: 128-wide tiles); rows padded to 104
    (1000, 2560, 2048, torch.bfloat16), # attention Q/K/V projection of d_model 2048
    (513, 160, 4096, torch.float32),    # selective-parameter projection (dt rank 128 + 2 x 16)
    (64, 8192, 2048, torch.bfloat16),   # Mamba input projection, a short prompt
    (777, 4096, 128, torch.float32),    # Δ up-projection
])
def test_gemm_matches_float64(M, N, K, dt):
    # rows of A and B start on 16-byte boundaries: K itself need not be a multiple of 8
    a, w = _operands(M, N, K, M + N + K, lda=(K + 7) // 8 * 8)
    if K % 8:
        w = torch.nn.functional.pad(w, (0, 8 - K % 8))[:, :K]
    c = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    ops.gemm(a, w, outs=[(c, 0, N, None)])
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    A64, W64 = host64(a), host64(w)
    _check(c, A64 @ W64.T, np.abs(A64) @ np.abs(W64).T, dt, f"gemm {M}x{N}x{K}")


def test_column_split_bias_and_strided_rows():
    """One pass writing three column ranges to three outputs (bf16, fp32 with
    a bias, fp32 into a wider matrix), from an A with padded rows."""
    M, N, K = 390, 160, 4096
    a, w = _operands(M, N, K, 7, lda=K + 64)
    dt_low = torch.full((M, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    bias = torch.randn((16,), device="cuda")
    Bm = torch.full((M, 16), float("nan"), device="cuda")
    wide = torch.full((M, 40), float("nan"), device="cuda")
    Cm = wide[:, 8:24]
    ops.gemm(a, w, outs=[(dt_low, 0, 128, None), (Bm, 128, 144, bias), (Cm, 144, 160, None)])
    torch.cuda.synchronize()
    A64, W64 = host64(a), host64(w)
    ref, mag = A64 @ W64.T, np.abs(A64) @ np.abs(W64).T
    _check(dt_low, ref[:, :128], mag[:, :128], torch.bfloat16, "gemm split dt_low")
    _check(Bm, ref[:, 128:144] + host64(bias)[None], mag[:, 128:144], torch.float32, "gemm split B + bias")
    _check(Cm, ref[:, 144:], mag[:, 144:], torch.float32, "gemm split C")
    w64 = host64(wide)
    assert np.all(np.isnan(w64[:, :8])) and np.all(np.isnan(w64[:, 24:]))  # nothing outside its range


def test_in_projection_split_into_x_and_z():
    M, K, D = 257, 2048, 4096
    a, w = _operands(M, 2 * D, K, 9)
    x = torch.full((M, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    z = torch.full((M, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    ops.gemm(a, w, outs=[(x, 0, D, None), (z, D, 2 * D, None)])
    torch.cuda.synchronize()
    A64, W64 = host64(a), host64(w)
    ref, mag = A64 @ W64.T, np.abs(A64) @ np.abs(W64).T
    _check(x, ref[:, :D], mag[:, :D], torch.bfloat16, "gemm in-proj x")
    _check(z, ref[:, D:], mag[:, D:], torch.bfloat16, "gemm in-proj z")


# ----------------------------------------------------------- split-K (M <= 32)
@pytest.mark.parametrize("M,N,K,dt", [
    (16, 8192, 2048, torch.bfloat16),   # Mamba input projection, 16 sequences decoding
    (16, 160, 4096, torch.float32),     # selective-parameter projection: 2 blocks of the weight, 64 k-steps each
    (16, 4096, 128, torch.float32),     # Δ up-projection: two k-steps per block
    (16, 2048, 4096, torch.bfloat16),   # Mamba output projection
    (1, 2560, 2048, torch.bfloat16),    # one sequence
    (3, 300, 200, torch.float32),       # ragged N and K (K not a multiple of 64)
    (17, 1000, 64, torch.bfloat16),     # 17 rows: the 32-row form; one k-step per block (direct store)
    (32, 777, 4104, torch.float32),     # 32 rows, ragged everything
])
def test_split_k_gemm_matches_float64_and_leaves_the_workspace_zero(M, N, K, dt):
    a, w = _operands(M, N, K, 3 * M + N + K, lda=(K + 7) // 8 * 8)
    nbytes = ops.gemm_workspace_size(M, N)
    assert nbytes > 0
    ws = torch.zeros((nbytes,), dtype=torch.uint8, device="cuda")
    A64, W64 = host64(a), host64(w)
    ref, mag = A64 @ W64.T, np.abs(A64) @ np.abs(W64).T
    for rep in range(3):      # the same workspace, call after call
        c = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
        ops.gemm(a, w, outs=[(c, 0, N, None)], workspace=ws)
        torch.cuda.synchronize()
        assert ops.get_status() == 0
        _check(c, ref, mag, dt, f"split-K gemm {M}x{N}x{K} call {rep}")
        assert int(torch.count_nonzero(ws)) == 0, "workspace not returned to zero"


def test_split_k_column_split_with_bias():
    """The decode form of the selective-parameter projection: three column
    ranges (bf16; fp32 with a bias; fp32 into a wider matrix) from 16 rows."""
    M, N, K = 16, 160, 4096
    a, w = _operands(M, N, K, 21, lda=K + 64)
    ws = torch.zeros((ops.gemm_workspace_size(M, N),), dtype=torch.uint8, device="cuda")
    dt_low = torch.full((M, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    bias = torch.randn((16,), device="cuda")
    Bm = torch.full((M, 16), float("nan"), device="cuda")
    wide = torch.full((M, 40), float("nan"), device="cuda")
    Cm = wide[:, 8:24]
    ops.gemm(a, w, outs=[(dt_low, 0, 128, None), (Bm, 128, 144, bias), (Cm, 144, 160, None)], workspace=ws)
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    A64, W64 = host64(a), host64(w)
    ref, mag = A64 @ W64.T, np.abs(A64) @ np.abs(W64).T
    _check(dt_low, ref[:, :128], mag[:, :128], torch.bfloat16, "split-K split dt_low")
    _check(Bm, ref[:, 128:144] + host64(bias), mag[:, 128:144], torch.float32, "split-K split B")
    _check(Cm, ref[:, 144:], mag[:, 144:], torch.float32, "split-K split C")
    assert torch.isnan(wide[:, :8]).all() and torch.isnan(wide[:, 24:]).all()
    assert int(torch.count_nonzero(ws)) == 0


def test_split_k_agrees_with_the_tiled_form():
    """The same 16-row product with and without a workspace: the two forms
    add the k-steps in different orders, so they agree to fp32 rounding."""
    M, N, K = 16, 4096, 2048
    a, w = _operands(M, N, K, 22)
    ws = torch.zeros((ops.gemm_workspace_size(M, N),), dtype=torch.uint8, device="cuda")
    c1 = ops.gemm(a, w, out_dtype=torch.float32, workspace=ws)
    c2 = ops.gemm(a, w, out_dtype=torch.float32)
    torch.cuda.synchronize()
    mag = host64(a).__abs__() @ host64(w).__abs__().T
    assert np.max(np.abs(host64(c1) - host64(c2)) / (1e-5 * mag)) <= 1.0
