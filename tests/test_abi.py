"""CPU checks of the C ABI: the library builds and loads, exports every
function the header declares, and rejects bad arguments on the host (no
kernel is launched and no GPU is needed)."""

import ctypes
import os
import re

import pytest

from hybrid_ssm_sliding_b200 import _lib as L
from hybrid_ssm_sliding_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "samba.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\**(samba_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("samba_conv1d_fwd", "samba_selective_scan_fwd", "samba_swa_fwd", "samba_mixer_prefill",
              "samba_scan_step", "samba_swa_step", "samba_swa_ring_fill", "samba_get_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_debug_build_exports_every_declared_symbol():
    """libsamba_debug.so: the same sources with the device-side checks; it
    must export the same entry points (loaded here by path, beside the
    release library the other tests use)."""
    dbg = ctypes.CDLL(B.build(debug=True))
    for name in declared_functions():
        assert hasattr(dbg, name), name


def test_release_build_has_no_check_selftest(lib):
    """Without SAMBA_DEBUG the check self-test refuses on the host (it
    launches nothing, so no GPU is needed)."""
    assert lib.samba_selftest_check(None) == L.SAMBA_ERR_UNSUPPORTED


def test_version(lib):
    assert lib.samba_version() >= 100


def _scan_args(**over):
    a = L.ScanArgs()
    fake = 0x10000  # 16-byte aligned dummy address; never dereferenced on rejected calls
    for f in ("x", "delta", "A", "Bm", "Cm", "y", "conv_w"):
        setattr(a, f, fake)
    a.batch, a.seqlen, a.dim, a.dstate, a.dconv = 1, 64, 16, 16, 4
    a.x_dtype = a.y_dtype = a.z_dtype = L.SAMBA_BF16
    a.flags = L.SCAN_FUSE_CONV | L.SCAN_DELTA_SOFTPLUS | L.SCAN_CONV_SILU
    for k, v in over.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("over,code", [
    (dict(x=None), L.SAMBA_ERR_INVALID_ARG),
    (dict(y=None), L.SAMBA_ERR_INVALID_ARG),
    (dict(batch=0), L.SAMBA_ERR_INVALID_ARG),
    (dict(seqlen=0), L.SAMBA_ERR_INVALID_ARG),
    (dict(dim=12), L.SAMBA_ERR_INVALID_ARG),
    (dict(dstate=32), L.SAMBA_ERR_UNSUPPORTED),
    (dict(dconv=5), L.SAMBA_ERR_UNSUPPORTED),
    (dict(x_dtype=7), L.SAMBA_ERR_UNSUPPORTED),
    (dict(conv_w=None), L.SAMBA_ERR_INVALID_ARG),
    (dict(flags=64), L.SAMBA_ERR_INVALID_ARG),
    (dict(x=0x10008), L.SAMBA_ERR_INVALID_ARG),
    (dict(h_ckpt=0x10004), L.SAMBA_ERR_INVALID_ARG),   # checkpoints are a base pointer too
])
def test_scan_rejects_bad_arguments_on_host(lib, over, code):
    a = _scan_args(**over)
    assert lib.samba_selective_scan_fwd(ctypes.byref(a), None) == code
    assert lib.samba_last_error().decode()


def test_scan_rejects_null_struct(lib):
    assert lib.samba_selective_scan_fwd(None, None) == L.SAMBA_ERR_INVALID_ARG


def _swa_args(**over):
    a = L.SwaArgs()
    for f in ("q", "k", "v", "o"):
        setattr(a, f, 0x20000)
    a.batch, a.seqlen, a.window, a.heads_q, a.heads_kv, a.head_dim = 1, 128, 64, 32, 4, 64
    for k, v in over.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("over,code", [
    (dict(q=None), L.SAMBA_ERR_INVALID_ARG),
    (dict(window=0), L.SAMBA_ERR_INVALID_ARG),
    (dict(heads_kv=5), L.SAMBA_ERR_INVALID_ARG),
    (dict(heads_q=96, heads_kv=3), L.SAMBA_ERR_UNSUPPORTED),
    (dict(head_dim=80), L.SAMBA_ERR_UNSUPPORTED),
    (dict(o=0x20004), L.SAMBA_ERR_INVALID_ARG),
])
def test_swa_rejects_bad_arguments_on_host(lib, over, code):
    a = _swa_args(**over)
    assert lib.samba_swa_fwd(ctypes.byref(a), None) == code
    assert lib.samba_mixer_prefill(ctypes.byref(_scan_args()), ctypes.byref(a), None, None) == code


def test_conv_rejects_bad_arguments_on_host(lib):
    f = 0x30000
    assert lib.samba_conv1d_fwd(None, 1, f, None, None, f, 1, None, 1, 8, 8, 4, 1, None) == L.SAMBA_ERR_INVALID_ARG
    assert lib.samba_conv1d_fwd(f, 1, f, None, None, f, 1, None, 1, 8, 8, 7, 1, None) == L.SAMBA_ERR_UNSUPPORTED
    assert lib.samba_conv1d_fwd(f, 1, f, None, f, f, 1, f, 1, 8, 8, 4, 1, None) == L.SAMBA_ERR_INVALID_ARG


def test_decode_rejects_bad_arguments_on_host(lib):
    f = 0x40000
    assert lib.samba_scan_step(None, None, f, 1, None, 1, f, f, f, f, None, None, None, f, 1, 1, 8, 16, 4, 0,
                               None) == L.SAMBA_ERR_INVALID_ARG
    assert lib.samba_scan_step(f, None, f, 1, None, 1, f, f, f, f, None, None, None, f, 1, 1, 8, 16, 4,
                               L.SCAN_FUSE_CONV, None) == L.SAMBA_ERR_INVALID_ARG
    assert lib.samba_scan_step(f, None, f, 1, None, 1, f, f, f, f, None, None, None, f, 1, 70000, 8, 16, 4, 0,
                               None) == L.SAMBA_ERR_UNSUPPORTED  # batch above 65535
    assert lib.samba_swa_ring_fill(f, f, 8, f, f, None, 1, 4, 64, 16, None) == L.SAMBA_ERR_INVALID_ARG
    assert lib.samba_swa_ring_fill(f, f, 8, f, f, f, 1, 4, 80, 16, None) == L.SAMBA_ERR_UNSUPPORTED
    need = lib.samba_swa_step_workspace_size(16, 32, 64, 2048)
    assert need == 16 * 32 * (2048 // 128) * 66 * 4  # (max, sum, 64 outputs) per head and 128-position split
    assert lib.samba_swa_step(f, f, f, f, f, f, f, 16, 32, 4, 64, 2048, 0.0, f, need - 1, None) == \
        L.SAMBA_ERR_WORKSPACE
    assert lib.samba_swa_step(f, f, f, f, f, f, f, 16, 32, 4, 64, 2048, 0.0, None, 0, None) == \
        L.SAMBA_ERR_WORKSPACE


def test_scan_step_argument_checks_on_host(lib):
    f = 0x50000

    def call(h=f, x_dtype=1, y_dtype=1, batch=1, dstate=16, dconv=4, flags=0):
        return lib.samba_scan_step(h, None, f, x_dtype, None, 1, f, f, f, f, None, None, None, f, y_dtype,
                                   batch, 8, dstate, dconv, flags, None)

    assert call(batch=0) == L.SAMBA_ERR_INVALID_ARG
    assert call(dstate=32) == L.SAMBA_ERR_UNSUPPORTED
    assert call(dconv=1) == L.SAMBA_ERR_UNSUPPORTED
    assert call(dconv=5) == L.SAMBA_ERR_UNSUPPORTED
    assert call(x_dtype=7) == L.SAMBA_ERR_UNSUPPORTED
    assert call(y_dtype=7) == L.SAMBA_ERR_UNSUPPORTED
    assert call(flags=8) == L.SAMBA_ERR_INVALID_ARG
    assert call(h=f + 4) == L.SAMBA_ERR_INVALID_ARG  # the state is read as 16-byte vectors


def test_swa_step_argument_checks_on_host(lib):
    f = 0x60000

    def call(q=f, batch=16, hq=32, hkv=4, d=64, W=2048, ws=f, nbytes=None):
        need = lib.samba_swa_step_workspace_size(max(batch, 1), max(hq, 1), max(d, 1), max(W, 1))
        return lib.samba_swa_step(q, f, f, f, f, f, f, batch, hq, hkv, d, W, 0.0, ws,
                                  need if nbytes is None else nbytes, None)

    assert call(W=0) == L.SAMBA_ERR_INVALID_ARG
    assert call(batch=0) == L.SAMBA_ERR_INVALID_ARG
    assert call(d=80) == L.SAMBA_ERR_UNSUPPORTED
    assert call(hq=33) == L.SAMBA_ERR_INVALID_ARG           # heads_q not a multiple of heads_kv
    assert call(hq=68) == L.SAMBA_ERR_UNSUPPORTED           # 17 query heads per KV head
    assert call(q=f + 8) == L.SAMBA_ERR_INVALID_ARG         # misaligned
    assert call(ws=f + 4) == L.SAMBA_ERR_INVALID_ARG        # misaligned workspace
    assert call(batch=70000) == L.SAMBA_ERR_UNSUPPORTED     # grid limit, refused before any launch
    assert call(W=(1 << 30) + 1) == L.SAMBA_ERR_UNSUPPORTED  # ring slots are 32-bit indices
    assert call(hq=70000, hkv=70000) == L.SAMBA_ERR_UNSUPPORTED  # KV heads on a 65535-block grid dimension


def test_swa_step_workspace_size_saturates_instead_of_wrapping(lib):
    size_max = ctypes.c_size_t(-1).value
    # 65535 sequences x 2^20 query heads x 2^24 splits x 66 floats does not fit in 64 bits
    assert lib.samba_swa_step_workspace_size(65535, 1 << 20, 64, 1 << 30) == size_max
    assert lib.samba_swa_step_workspace_size(0, 32, 64, 2048) == 0
    f = 0x68000
    # no workspace can satisfy a saturated size, so the step refuses before any launch
    assert lib.samba_swa_step(f, f, f, f, f, f, f, 65535, 1 << 20, 1 << 16, 64, 1 << 30, 0.0, f, size_max - 15,
                              None) in (L.SAMBA_ERR_UNSUPPORTED, L.SAMBA_ERR_WORKSPACE)


def test_swa_step_noalloc_checks_on_host(lib):
    f = 0x70000

    def call(q=f, batch=16, hq=32, hkv=4, d=64, W=2048):
        return lib.samba_swa_step_noalloc(q, f, f, f, f, f, f, batch, hq, hkv, d, W, 0.0, None)

    assert call(hq=68) == L.SAMBA_ERR_UNSUPPORTED
    assert call(q=f + 8) == L.SAMBA_ERR_INVALID_ARG
    # 64 sequences x 32 heads x 16 splits x 66 floats = 8.6 MB: more than the built-in 4 MiB
    assert lib.samba_swa_step_workspace_size(64, 32, 64, 2048) > 4 << 20
    assert call(batch=64) == L.SAMBA_ERR_WORKSPACE
    # argument limits are reported as for samba_swa_step, before the scratch size
    assert call(batch=70000) == L.SAMBA_ERR_UNSUPPORTED
    assert call(W=(1 << 30) + 1) == L.SAMBA_ERR_UNSUPPORTED


def test_gemm_rejects_bad_arguments_on_host(lib):
    f = 0x80000

    def call(M=128, N=256, K=64, lda=64, ldb=64, nout=1, ptr=f, col0=0, col1=256, ld=256, dtype=1, A=f, ws=None):
        a = L.GemmArgs()
        a.A, a.B, a.lda, a.ldb, a.M, a.N, a.K = A, f, lda, ldb, M, N, K
        o = a.out[0]
        o.ptr, o.bias, o.ld, o.col0, o.col1, o.dtype = ptr, None, ld, col0, col1, dtype
        a.nout = nout
        a.workspace, a.workspace_bytes = ws, 1 << 20
        return lib.samba_gemm(ctypes.byref(a), None)

    assert call(A=None) == L.SAMBA_ERR_INVALID_ARG
    assert call(K=0) == L.SAMBA_ERR_INVALID_ARG
    assert call(lda=60) == L.SAMBA_ERR_INVALID_ARG          # below K
    assert call(lda=68, K=64) == L.SAMBA_ERR_INVALID_ARG    # not a multiple of 8
    assert call(A=f + 8) == L.SAMBA_ERR_INVALID_ARG         # misaligned
    assert call(nout=0) == L.SAMBA_ERR_UNSUPPORTED
    assert call(nout=4) == L.SAMBA_ERR_UNSUPPORTED
    assert call(ptr=None) == L.SAMBA_ERR_INVALID_ARG
    assert call(col1=300) == L.SAMBA_ERR_INVALID_ARG        # past N
    assert call(col0=10, col1=10) == L.SAMBA_ERR_INVALID_ARG
    assert call(ld=100) == L.SAMBA_ERR_INVALID_ARG          # row stride below the range
    assert call(dtype=7) == L.SAMBA_ERR_UNSUPPORTED
    assert call(M=65535 * 128 + 1) == L.SAMBA_ERR_UNSUPPORTED
    assert call(M=16, ws=f + 4) == L.SAMBA_ERR_INVALID_ARG    # misaligned workspace


def test_gemm_workspace_size(lib):
    """fp32 partial sums for 128-row blocks of the weight x 16 or 32 rows, and
    four counters per block, rounded up to 256 bytes; none above 32 rows."""
    def want(M, N):
        nblk = -(-N // 128)
        mp = 16 if M <= 16 else 32
        return -(-(nblk * 128 * mp * 4 + nblk * 16) // 256) * 256

    for M, N in ((1, 1), (16, 8192), (17, 160), (32, 4096), (3, 129)):
        assert lib.samba_gemm_workspace_size(M, N) == want(M, N)
    assert lib.samba_gemm_workspace_size(33, 4096) == 0
    assert lib.samba_gemm_workspace_size(0, 4096) == 0


def test_scan_bwd_rejects_bad_arguments_on_host(lib):
    f = 0x80000
    need = lib.samba_scan_bwd_workspace_size(2, 100, 64, 16)
    # ceil(100 / 16) chunk checkpoints, then per-32-channel-block partials of dB and dC
    assert need == 2 * 7 * 16 * 64 * 4 + (64 // 32) * 2 * 2 * 100 * 16 * 4
    assert lib.samba_scan_bwd_workspace_size(0, 100, 64, 16) == 0
    assert lib.samba_scan_bwd_workspace_size(2**40, 2**40, 2**20, 16) == 2**64 - 1   # saturates

    def call(**over):
        a = L.ScanBwdArgs()
        for k in ("x", "delta", "A", "Bm", "Cm", "dy", "dx", "ddelta", "dA", "dB", "dC", "workspace"):
            setattr(a, k, f)
        a.batch, a.seqlen, a.dim, a.dstate, a.dconv = 2, 100, 64, 16, 4
        a.workspace_bytes = need
        a.x_dtype = a.y_dtype = 1
        for k, v in over.items():
            setattr(a, k, v)
        return lib.samba_selective_scan_bwd(ctypes.byref(a), None)

    assert lib.samba_selective_scan_bwd(None, None) == L.SAMBA_ERR_INVALID_ARG
    assert call(dy=None) == L.SAMBA_ERR_INVALID_ARG
    assert call(dB=None) == L.SAMBA_ERR_INVALID_ARG
    assert call(z=f, z_dtype=1) == L.SAMBA_ERR_INVALID_ARG              # z without dz
    assert call(Dskip=f) == L.SAMBA_ERR_INVALID_ARG                     # Dskip without dD
    assert call(flags=L.SCAN_FUSE_CONV, conv_w=f) == L.SAMBA_ERR_INVALID_ARG   # no dconv_w
    assert call(dx=f + 4) == L.SAMBA_ERR_INVALID_ARG                     # misaligned
    assert call(dstate=12) == L.SAMBA_ERR_UNSUPPORTED
    assert call(workspace=None) == L.SAMBA_ERR_WORKSPACE
    assert call(workspace_bytes=need - 1) == L.SAMBA_ERR_WORKSPACE
    assert call(ckpt=f + 4) == L.SAMBA_ERR_INVALID_ARG                   # the forward's checkpoints, misaligned


def test_mixer_bwd_checks_both_arguments_before_any_launch(lib):
    """samba_mixer_bwd validates the scan's and the attention's arguments
    before it creates its events or launches anything (with or without an
    aux stream), and returns the first failing check's code."""
    f = 0x80000
    s = L.ScanBwdArgs()
    for k in ("x", "delta", "A", "Bm", "Cm", "dy", "dx", "ddelta", "dA", "dB", "dC", "workspace"):
        setattr(s, k, f)
    s.batch, s.seqlen, s.dim, s.dstate, s.dconv = 2, 100, 64, 16, 4
    s.workspace_bytes = lib.samba_scan_bwd_workspace_size(2, 100, 64, 16)
    s.x_dtype = s.y_dtype = 1
    w = L.SwaBwdArgs()
    for key in ("q", "k", "v", "o", "lse", "dO", "dq", "dk", "dv", "workspace"):
        setattr(w, key, f)
    w.workspace_bytes = lib.samba_swa_bwd_workspace_size(2, 100, 8)
    w.batch, w.seqlen, w.window, w.heads_q, w.heads_kv, w.head_dim = 2, 100, 16, 8, 2, 64
    for aux in (None, 0x1234):  # the aux handle is never used when a check fails
        assert lib.samba_mixer_bwd(None, ctypes.byref(w), None, aux) == L.SAMBA_ERR_INVALID_ARG
        assert lib.samba_mixer_bwd(ctypes.byref(s), None, None, aux) == L.SAMBA_ERR_INVALID_ARG
        s.dstate = 12
        assert lib.samba_mixer_bwd(ctypes.byref(s), ctypes.byref(w), None, aux) == L.SAMBA_ERR_UNSUPPORTED
        s.dstate = 16
        w.head_dim = 48
        assert lib.samba_mixer_bwd(ctypes.byref(s), ctypes.byref(w), None, aux) == L.SAMBA_ERR_UNSUPPORTED
        w.head_dim = 64
        w.workspace_bytes -= 4
        assert lib.samba_mixer_bwd(ctypes.byref(s), ctypes.byref(w), None, aux) == L.SAMBA_ERR_WORKSPACE
        w.workspace_bytes += 4


def test_swa_bwd_rejects_bad_arguments_on_host(lib):
    f = 0x80000
    need = lib.samba_swa_bwd_workspace_size(2, 100, 8)
    assert need == 2 * 128 * 8 * 2 * 4          # per row: base-2 lse and D, rows padded to 128
    assert lib.samba_swa_bwd_workspace_size(2**40, 2**40, 2**20) == 2**64 - 1

    def call(**over):
        a = L.SwaBwdArgs()
        for key in ("q", "k", "v", "o", "lse", "dO", "dq", "dk", "dv", "workspace"):
            setattr(a, key, f)
        a.workspace_bytes = need
        a.batch, a.seqlen, a.window, a.heads_q, a.heads_kv, a.head_dim = 2, 100, 16, 8, 2, 64
        for key, val in over.items():
            setattr(a, key, val)
        return lib.samba_swa_bwd(ctypes.byref(a), None)

    assert lib.samba_swa_bwd(None, None) == L.SAMBA_ERR_INVALID_ARG
    assert call(lse=None) == L.SAMBA_ERR_INVALID_ARG
    assert call(dO=None) == L.SAMBA_ERR_INVALID_ARG
    assert call(dk=f + 8) == L.SAMBA_ERR_INVALID_ARG
    assert call(head_dim=48) == L.SAMBA_ERR_UNSUPPORTED
    assert call(heads_kv=3) == L.SAMBA_ERR_INVALID_ARG
    assert call(workspace=None) == L.SAMBA_ERR_WORKSPACE
    assert call(workspace_bytes=need - 4) == L.SAMBA_ERR_WORKSPACE
