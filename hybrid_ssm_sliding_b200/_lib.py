"""ctypes binding of libsamba.so (the C ABI in include/samba.h).

Argument marshalling only: every step of the mixers runs in the CUDA kernels
of the library.  PyTorch provides device memory and streams.  There is no
fallback: if the library is missing or a call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# SAMBA_LIBRARY=debug loads the debug build (libsamba_debug.so: the same
# kernels with device-side index checks); it is never a fallback
LIB_PATH = os.path.join(_HERE, "libsamba_debug.so" if os.environ.get("SAMBA_LIBRARY") == "debug" else "libsamba.so")

SAMBA_F32, SAMBA_BF16 = 0, 1
SAMBA_OK = 0
SAMBA_ERR_INVALID_ARG, SAMBA_ERR_UNSUPPORTED, SAMBA_ERR_WORKSPACE = -1, -2, -3
SAMBA_ERR_CUDA, SAMBA_ERR_TIMEOUT, SAMBA_ERR_CHECK = -4, -5, -6
SCAN_FUSE_CONV, SCAN_DELTA_SOFTPLUS, SCAN_CONV_SILU = 1, 2, 4

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32


class ScanArgs(ctypes.Structure):
    _fields_ = [
        ("x", _vp), ("z", _vp), ("delta", _vp), ("A", _vp), ("Bm", _vp), ("Cm", _vp),
        ("Dskip", _vp), ("conv_w", _vp), ("conv_b", _vp), ("conv_state_in", _vp),
        ("conv_state_out", _vp), ("h0", _vp), ("h_final", _vp), ("y", _vp),
        ("batch", _i64), ("seqlen", _i64), ("dim", _i64),
        ("dstate", _i32), ("dconv", _i32), ("x_dtype", _i32), ("z_dtype", _i32), ("y_dtype", _i32),
        ("flags", ctypes.c_uint32), ("delta_sum", _vp), ("h_ckpt", _vp),
    ]


class ScanBwdArgs(ctypes.Structure):
    _fields_ = [
        ("x", _vp), ("z", _vp), ("delta", _vp), ("A", _vp), ("Bm", _vp), ("Cm", _vp), ("Dskip", _vp),
        ("conv_w", _vp), ("conv_b", _vp), ("conv_state_in", _vp), ("h0", _vp), ("dy", _vp),
        ("dx", _vp), ("ddelta", _vp), ("dz", _vp), ("dA", _vp), ("dB", _vp), ("dC", _vp), ("dD", _vp),
        ("dconv_w", _vp), ("dconv_b", _vp), ("dh0", _vp), ("dconv_state", _vp),
        ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
        ("batch", _i64), ("seqlen", _i64), ("dim", _i64),
        ("dstate", _i32), ("dconv", _i32), ("x_dtype", _i32), ("z_dtype", _i32), ("y_dtype", _i32),
        ("flags", ctypes.c_uint32), ("ckpt", _vp),
    ]


class SwaArgs(ctypes.Structure):
    _fields_ = [
        ("q", _vp), ("k", _vp), ("v", _vp), ("o", _vp), ("lse", _vp),
        ("batch", _i64), ("seqlen", _i64), ("window", _i64),
        ("heads_q", _i32), ("heads_kv", _i32), ("head_dim", _i32), ("scale", ctypes.c_float),
    ]


class SwaBwdArgs(ctypes.Structure):
    _fields_ = [
        ("q", _vp), ("k", _vp), ("v", _vp), ("o", _vp), ("lse", _vp), ("dO", _vp), ("dq", _vp), ("dk", _vp),
        ("dv", _vp), ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
        ("batch", _i64), ("seqlen", _i64), ("window", _i64),
        ("heads_q", _i32), ("heads_kv", _i32), ("head_dim", _i32), ("scale", ctypes.c_float),
    ]


class GemmOut(ctypes.Structure):
    _fields_ = [("ptr", _vp), ("bias", _vp), ("ld", _i64), ("col0", _i64), ("col1", _i64), ("dtype", _i32)]


class GemmArgs(ctypes.Structure):
    _fields_ = [("A", _vp), ("B", _vp), ("lda", _i64), ("ldb", _i64), ("M", _i64), ("N", _i64), ("K", _i64),
                ("out", GemmOut * 3), ("nout", _i32), ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class SambaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"samba error {code}: {msg}")
        self.code = code


_lib = None


def load() -> ctypes.CDLL:
    """Loads libsamba.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m hybrid_ssm_sliding_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    lib.samba_version.restype = ctypes.c_int
    lib.samba_last_error.restype = ctypes.c_char_p
    lib.samba_get_status.argtypes = [_vp]
    lib.samba_selftest_wait_timeout.argtypes = [_vp]
    lib.samba_selftest_check.argtypes = [_vp]
    lib.samba_conv1d_fwd.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _vp, ctypes.c_int, _vp,
                                     _i64, _i64, _i64, ctypes.c_int, ctypes.c_int, _vp]
    lib.samba_selective_scan_fwd.argtypes = [ctypes.POINTER(ScanArgs), _vp]
    lib.samba_swa_fwd.argtypes = [ctypes.POINTER(SwaArgs), _vp]
    lib.samba_mixer_prefill.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(SwaArgs), _vp, _vp]
    lib.samba_scan_step.argtypes = [_vp, _vp, _vp, ctypes.c_int, _vp, ctypes.c_int, _vp, _vp, _vp, _vp,
                                    _vp, _vp, _vp, _vp, ctypes.c_int, _i64, _i64, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_uint32, _vp]
    lib.samba_swa_ring_fill.argtypes = [_vp, _vp, _i64, _vp, _vp, _vp, _i64, ctypes.c_int, ctypes.c_int,
                                        _i64, _vp]
    lib.samba_swa_step_workspace_size.argtypes = [_i64, ctypes.c_int, ctypes.c_int, _i64]
    lib.samba_swa_step_workspace_size.restype = ctypes.c_size_t
    lib.samba_swa_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, _i64, ctypes.c_float, _vp, ctypes.c_size_t, _vp]
    lib.samba_swa_step_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, _i64, ctypes.c_float, _vp]
    lib.samba_gemm.argtypes = [ctypes.POINTER(GemmArgs), _vp]
    lib.samba_gemm_workspace_size.argtypes = [_i64, _i64]
    lib.samba_gemm_workspace_size.restype = ctypes.c_size_t
    lib.samba_scan_carry.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, ctypes.c_int, _vp]
    lib.samba_scan_bwd_workspace_size.argtypes = [_i64, _i64, _i64, _i32]
    lib.samba_scan_bwd_workspace_size.restype = ctypes.c_size_t
    lib.samba_selective_scan_bwd.argtypes = [ctypes.POINTER(ScanBwdArgs), _vp]
    lib.samba_swa_bwd_workspace_size.argtypes = [_i64, _i64, _i32]
    lib.samba_swa_bwd_workspace_size.restype = ctypes.c_size_t
    lib.samba_swa_bwd.argtypes = [ctypes.POINTER(SwaBwdArgs), _vp]
    lib.samba_mixer_bwd.argtypes = [ctypes.POINTER(ScanBwdArgs), ctypes.POINTER(SwaBwdArgs), _vp, _vp]
    lib.samba_conv_state.argtypes = [_vp, ctypes.c_int, _vp, _vp, _i64, _i64, _i64, ctypes.c_int, _vp]
    for name in ("samba_conv1d_fwd", "samba_selective_scan_fwd", "samba_swa_fwd", "samba_mixer_prefill",
                 "samba_scan_step", "samba_swa_ring_fill", "samba_swa_step", "samba_get_status",
                 "samba_scan_carry", "samba_conv_state", "samba_gemm", "samba_selective_scan_bwd", "samba_swa_bwd",
                 "samba_selftest_wait_timeout", "samba_swa_step_noalloc", "samba_selftest_check", "samba_mixer_bwd"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def check(rc: int) -> None:
    if rc != SAMBA_OK:
        raise SambaError(rc, load().samba_last_error().decode())


def ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SAMBA_F32
    if t.dtype == torch.bfloat16:
        return SAMBA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def stream_handle(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream
