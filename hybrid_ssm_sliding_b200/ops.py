"""Python entry points over the C ABI (same names as the C functions).

Each function checks that tensors are CUDA, contiguous and of the right
dtype, allocates outputs that were not given (torch.empty, on the same
device), and calls into libsamba.so on the current (or given) stream.
"""

from __future__ import annotations

import ctypes
import math

import torch

from . import _lib as L


def _need(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _opt(t, name, dtype=None, shape=None):
    return None if t is None else _need(t, name, dtype, shape)


def version() -> int:
    return L.load().samba_version()


def get_status(stream=None) -> int:
    """Synchronises the stream and returns/clears the device status word
    (SAMBA_OK or SAMBA_ERR_TIMEOUT)."""
    return L.load().samba_get_status(L.stream_handle(stream))


def conv1d_fwd(x, w, bias=None, conv_state_in=None, silu=True, u=None, u_dtype=None,
               conv_state_out=None, stream=None):
    """Causal depthwise conv1d: x [B, L, D] -> u [B, L, D] (see samba_conv1d_fwd)."""
    _need(x, "x")
    Bsz, Ln, D = x.shape
    K = w.shape[1]
    _need(w, "w", torch.float32, (D, K))
    _opt(bias, "bias", torch.float32, (D,))
    _opt(conv_state_in, "conv_state_in", torch.float32, (Bsz, D, K - 1))
    if u is None:
        u = torch.empty_like(x, dtype=u_dtype or x.dtype)
    _need(u, "u", None, x.shape)
    _opt(conv_state_out, "conv_state_out", torch.float32, (Bsz, D, K - 1))
    lib = L.load()
    L.check(lib.samba_conv1d_fwd(L.ptr(x), L.dtype_code(x), L.ptr(w), L.ptr(bias), L.ptr(conv_state_in),
                                 L.ptr(u), L.dtype_code(u), L.ptr(conv_state_out), Bsz, Ln, D, K,
                                 1 if silu else 0, L.stream_handle(stream)))
    return u


def scan_ckpt_shape(batch, seqlen, dim, dstate):
    """Shape of the forward's chunk checkpoints (samba_scan_args.h_ckpt)."""
    return (batch, (seqlen + 15) // 16, dstate, dim)


def _scan_struct(x, delta, A, B, C, D=None, z=None, conv_w=None, conv_b=None, conv_state_in=None,
                 h0=None, y=None, y_dtype=None, h_final=None, conv_state_out=None,
                 delta_softplus=True, conv_silu=True, fuse_conv=None, delta_sum=None, h_ckpt=None):
    _need(x, "x")
    Bsz, Ln, Dm = x.shape
    N = A.shape[1]
    _need(delta, "delta", torch.float32, x.shape)
    _need(A, "A", torch.float32, (Dm, N))
    _need(B, "B", torch.float32, (Bsz, Ln, N))
    _need(C, "C", torch.float32, (Bsz, Ln, N))
    _opt(D, "D", torch.float32, (Dm,))
    _opt(z, "z", x.dtype, x.shape)
    if fuse_conv is None:
        fuse_conv = conv_w is not None
    K = conv_w.shape[1] if conv_w is not None else 4
    _opt(conv_w, "conv_w", torch.float32, (Dm, K))
    _opt(conv_b, "conv_b", torch.float32, (Dm,))
    _opt(conv_state_in, "conv_state_in", torch.float32, (Bsz, Dm, K - 1))
    _opt(conv_state_out, "conv_state_out", torch.float32, (Bsz, Dm, K - 1))
    _opt(h0, "h0", torch.float32, (Bsz, Dm, N))
    _opt(h_final, "h_final", torch.float32, (Bsz, Dm, N))
    _opt(delta_sum, "delta_sum", torch.float32, (Bsz, Dm))
    _opt(h_ckpt, "h_ckpt", torch.float32, scan_ckpt_shape(Bsz, Ln, Dm, N))
    if y is None:
        y = torch.empty_like(x, dtype=y_dtype or x.dtype)
    _need(y, "y", None, x.shape)
    flags = ((L.SCAN_FUSE_CONV if fuse_conv else 0) | (L.SCAN_DELTA_SOFTPLUS if delta_softplus else 0)
             | (L.SCAN_CONV_SILU if conv_silu else 0))
    a = L.ScanArgs(L.ptr(x), L.ptr(z), L.ptr(delta), L.ptr(A), L.ptr(B), L.ptr(C), L.ptr(D), L.ptr(conv_w),
                   L.ptr(conv_b), L.ptr(conv_state_in), L.ptr(conv_state_out), L.ptr(h0), L.ptr(h_final),
                   L.ptr(y), Bsz, Ln, Dm, N, K, L.dtype_code(x), L.dtype_code(z) if z is not None else 0,
                   L.dtype_code(y), flags, L.ptr(delta_sum), L.ptr(h_ckpt))
    return a, y


def selective_scan_fwd(x, delta, A, B, C, D=None, z=None, conv_w=None, conv_b=None, conv_state_in=None,
                       h0=None, y=None, y_dtype=None, h_final=None, conv_state_out=None,
                       delta_softplus=True, conv_silu=True, fuse_conv=None, delta_sum=None, h_ckpt=None,
                       stream=None):
    """Fused selective-scan prefill (see samba_selective_scan_fwd).  Returns y.
    ``h_ckpt`` ([B, ceil(L/16), N, D] fp32) receives the state at every
    16-token chunk start, for selective_scan_bwd(ckpt=...)."""
    a, y = _scan_struct(x, delta, A, B, C, D, z, conv_w, conv_b, conv_state_in, h0, y, y_dtype, h_final,
                        conv_state_out, delta_softplus, conv_silu, fuse_conv, delta_sum, h_ckpt)
    L.check(L.load().samba_selective_scan_fwd(ctypes.byref(a), L.stream_handle(stream)))
    return y


def scan_bwd_workspace_size(batch, seqlen, dim, dstate):
    return int(L.load().samba_scan_bwd_workspace_size(batch, seqlen, dim, dstate))


def selective_scan_bwd(dy, x, delta, A, B, C, D=None, z=None, conv_w=None, conv_b=None, conv_state_in=None,
                       h0=None, delta_softplus=True, conv_silu=True, fuse_conv=None, want_dh0=False,
                       want_dconv_state=False, workspace=None, ckpt=None, stream=None):
    """Gradients of selective_scan_fwd's y given dy (see
    samba_selective_scan_bwd).  Returns a dict with dx, ddelta, dA, dB, dC
    and, where the forward input exists, dz, dD, dconv_w, dconv_b, plus dh0 /
    dconv_state when asked for.  ``ckpt``: the forward's h_ckpt for these
    inputs (the backward then skips its own checkpoint pass)."""
    a, out, _ws = _scan_bwd_struct(dy, x, delta, A, B, C, D, z, conv_w, conv_b, conv_state_in, h0, delta_softplus,
                                   conv_silu, fuse_conv, want_dh0, want_dconv_state, workspace, ckpt)
    L.check(L.load().samba_selective_scan_bwd(ctypes.byref(a), L.stream_handle(stream)))
    return out


def _scan_bwd_struct(dy, x, delta, A, B, C, D=None, z=None, conv_w=None, conv_b=None, conv_state_in=None,
                     h0=None, delta_softplus=True, conv_silu=True, fuse_conv=None, want_dh0=False,
                     want_dconv_state=False, workspace=None, ckpt=None):
    """The samba_scan_bwd_args of selective_scan_bwd, its output dict and the
    workspace (kept alive by the caller until the call is enqueued)."""
    _need(x, "x")
    Bsz, Ln, Dm = x.shape
    N = A.shape[1]
    _need(dy, "dy", None, x.shape)
    _need(delta, "delta", torch.float32, x.shape)
    _need(A, "A", torch.float32, (Dm, N))
    _need(B, "B", torch.float32, (Bsz, Ln, N))
    _need(C, "C", torch.float32, (Bsz, Ln, N))
    _opt(D, "D", torch.float32, (Dm,))
    _opt(z, "z", x.dtype, x.shape)
    if fuse_conv is None:
        fuse_conv = conv_w is not None
    K = conv_w.shape[1] if conv_w is not None else 4
    _opt(conv_w, "conv_w", torch.float32, (Dm, K))
    _opt(conv_b, "conv_b", torch.float32, (Dm,))
    _opt(conv_state_in, "conv_state_in", torch.float32, (Bsz, Dm, K - 1))
    _opt(h0, "h0", torch.float32, (Bsz, Dm, N))
    _opt(ckpt, "ckpt", torch.float32, scan_ckpt_shape(Bsz, Ln, Dm, N))
    dev = x.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dx": torch.empty_like(x), "ddelta": torch.empty((Bsz, Ln, Dm), **f32), "dA": torch.empty((Dm, N), **f32),
           "dB": torch.empty((Bsz, Ln, N), **f32), "dC": torch.empty((Bsz, Ln, N), **f32),
           "dz": torch.empty_like(x) if z is not None else None,
           "dD": torch.empty((Dm,), **f32) if D is not None else None,
           "dconv_w": torch.empty((Dm, K), **f32) if fuse_conv else None,
           "dconv_b": torch.empty((Dm,), **f32) if fuse_conv and conv_b is not None else None,
           "dh0": torch.empty((Bsz, Dm, N), **f32) if want_dh0 else None,
           "dconv_state": torch.empty((Bsz, Dm, K - 1), **f32) if want_dconv_state else None}
    need = scan_bwd_workspace_size(Bsz, Ln, Dm, N)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=dev)
    flags = ((L.SCAN_FUSE_CONV if fuse_conv else 0) | (L.SCAN_DELTA_SOFTPLUS if delta_softplus else 0)
             | (L.SCAN_CONV_SILU if conv_silu else 0))
    a = L.ScanBwdArgs(L.ptr(x), L.ptr(z), L.ptr(delta), L.ptr(A), L.ptr(B), L.ptr(C), L.ptr(D), L.ptr(conv_w),
                      L.ptr(conv_b), L.ptr(conv_state_in), L.ptr(h0), L.ptr(dy),
                      L.ptr(out["dx"]), L.ptr(out["ddelta"]), L.ptr(out["dz"]), L.ptr(out["dA"]), L.ptr(out["dB"]),
                      L.ptr(out["dC"]), L.ptr(out["dD"]), L.ptr(out["dconv_w"]), L.ptr(out["dconv_b"]),
                      L.ptr(out["dh0"]), L.ptr(out["dconv_state"]), L.ptr(workspace),
                      workspace.numel() * workspace.element_size(), Bsz, Ln, Dm, N, K, L.dtype_code(x),
                      L.dtype_code(z) if z is not None else 0, L.dtype_code(dy), flags, L.ptr(ckpt))
    return a, out, workspace


def _swa_struct(q, k, v, window, scale=None, o=None, lse=None):
    _need(q, "q", torch.bfloat16)
    Bsz, Ln, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(k, "k", torch.bfloat16, (Bsz, Ln, Hkv, d))
    _need(v, "v", torch.bfloat16, (Bsz, Ln, Hkv, d))
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", torch.bfloat16, q.shape)
    _opt(lse, "lse", torch.float32, (Bsz, Hq, Ln))
    a = L.SwaArgs(L.ptr(q), L.ptr(k), L.ptr(v), L.ptr(o), L.ptr(lse), Bsz, Ln, int(window), Hq, Hkv, d,
                  float(scale) if scale else 0.0)
    return a, o


def swa_fwd(q, k, v, window, scale=None, o=None, lse=None, stream=None):
    """Banded causal sliding-window attention (see samba_swa_fwd).  Returns o."""
    a, o = _swa_struct(q, k, v, window, scale, o, lse)
    L.check(L.load().samba_swa_fwd(ctypes.byref(a), L.stream_handle(stream)))
    return o


def swa_bwd_workspace_size(batch, seqlen, heads_q):
    return int(L.load().samba_swa_bwd_workspace_size(batch, seqlen, heads_q))


def swa_bwd(do, q, k, v, o, lse, window, scale=None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients of swa_fwd given dO (see samba_swa_bwd): o and lse are the
    forward's outputs for the same q, k, v.  Returns (dq, dk, dv)."""
    a, grads, _ws = _swa_bwd_struct(do, q, k, v, o, lse, window, scale, dq, dk, dv, workspace)
    L.check(L.load().samba_swa_bwd(ctypes.byref(a), L.stream_handle(stream)))
    return grads


def _swa_bwd_struct(do, q, k, v, o, lse, window, scale=None, dq=None, dk=None, dv=None, workspace=None):
    """The samba_swa_bwd_args of swa_bwd, (dq, dk, dv) and the workspace."""
    _need(q, "q", torch.bfloat16)
    Bsz, Ln, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(k, "k", torch.bfloat16, (Bsz, Ln, Hkv, d))
    _need(v, "v", torch.bfloat16, (Bsz, Ln, Hkv, d))
    _need(o, "o", torch.bfloat16, q.shape)
    _need(do, "dO", torch.bfloat16, q.shape)
    _need(lse, "lse", torch.float32, (Bsz, Hq, Ln))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _need(dq, "dq", torch.bfloat16, q.shape)
    _need(dk, "dk", torch.bfloat16, k.shape)
    _need(dv, "dv", torch.bfloat16, v.shape)
    need = swa_bwd_workspace_size(Bsz, Ln, Hq)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=q.device)
    a = L.SwaBwdArgs(L.ptr(q), L.ptr(k), L.ptr(v), L.ptr(o), L.ptr(lse), L.ptr(do), L.ptr(dq), L.ptr(dk), L.ptr(dv),
                     L.ptr(workspace), workspace.numel() * workspace.element_size(), Bsz, Ln, int(window), Hq, Hkv, d,
                     float(scale) if scale else 0.0)
    return a, (dq, dk, dv), workspace


def mixer_bwd(scan: dict, swa: dict, stream=None, aux_stream=None):
    """The backward of both mixers (see samba_mixer_bwd): ``scan`` and
    ``swa`` hold the keyword arguments of selective_scan_bwd and swa_bwd
    (without stream).  With ``aux_stream`` the attention's backward runs
    there, beside the scan's.  Returns (scan gradients dict, (dq, dk, dv))."""
    sa, sgrads, ws1 = _scan_bwd_struct(**scan)
    wa, wgrads, ws2 = _swa_bwd_struct(**swa)
    L.check(L.load().samba_mixer_bwd(ctypes.byref(sa), ctypes.byref(wa), L.stream_handle(stream),
                                     L.stream_handle(aux_stream) if aux_stream is not None else None))
    del ws1, ws2
    return sgrads, wgrads


def mixer_prefill(scan: dict, swa: dict, stream=None, aux_stream=None):
    """One Mamba mixer and one SWA mixer (see samba_mixer_prefill).
    ``scan`` / ``swa`` hold the keyword arguments of selective_scan_fwd /
    swa_fwd.  Returns (y, o)."""
    sa, y = _scan_struct(**scan)
    wa, o = _swa_struct(**swa)
    aux = None if aux_stream is None else aux_stream.cuda_stream
    L.check(L.load().samba_mixer_prefill(ctypes.byref(sa), ctypes.byref(wa), L.stream_handle(stream), aux))
    return y, o


def scan_step(h, conv_state, x_t, delta_t, A, B_t, C_t, D=None, z_t=None, conv_w=None, conv_b=None,
              y_t=None, y_dtype=None, delta_softplus=True, conv_silu=True, stream=None):
    """One decode step of the scan; updates h and conv_state in place (see
    samba_scan_step).  Returns y_t."""
    _need(x_t, "x_t")
    Bsz, Dm = x_t.shape
    N = A.shape[1]
    _need(h, "h", torch.float32, (Bsz, Dm, N))
    _need(delta_t, "delta_t", torch.float32, (Bsz, Dm))
    _need(A, "A", torch.float32, (Dm, N))
    _need(B_t, "B_t", torch.float32, (Bsz, N))
    _need(C_t, "C_t", torch.float32, (Bsz, N))
    _opt(D, "D", torch.float32, (Dm,))
    _opt(z_t, "z_t", x_t.dtype, (Bsz, Dm))
    K = conv_w.shape[1] if conv_w is not None else 4
    _opt(conv_w, "conv_w", torch.float32, (Dm, K))
    _opt(conv_b, "conv_b", torch.float32, (Dm,))
    _opt(conv_state, "conv_state", torch.float32, (Bsz, Dm, K - 1))
    if y_t is None:
        y_t = torch.empty_like(x_t, dtype=y_dtype or x_t.dtype)
    flags = ((L.SCAN_FUSE_CONV if conv_w is not None else 0) | (L.SCAN_DELTA_SOFTPLUS if delta_softplus else 0)
             | (L.SCAN_CONV_SILU if conv_silu else 0))
    L.check(L.load().samba_scan_step(L.ptr(h), L.ptr(conv_state), L.ptr(x_t), L.dtype_code(x_t), L.ptr(z_t),
                                     L.dtype_code(z_t) if z_t is not None else 0, L.ptr(delta_t), L.ptr(B_t),
                                     L.ptr(C_t), L.ptr(A), L.ptr(D), L.ptr(conv_w), L.ptr(conv_b), L.ptr(y_t),
                                     L.dtype_code(y_t), Bsz, Dm, N, K, flags, L.stream_handle(stream)))
    return y_t


def gemm_workspace_size(M, N) -> int:
    """Bytes of workspace the split-K form of samba_gemm uses for M rows and
    N columns (0 when M > 32)."""
    return int(L.load().samba_gemm_workspace_size(M, N))


def gemm(a, w, outs=None, out_dtype=torch.bfloat16, bias=None, workspace=None, stream=None):
    """C = a @ w.T on the tensor cores (see samba_gemm): a [M, K] bf16 (rows
    may be strided), w [N, K] bf16.  ``outs`` is a list of up to three
    (tensor, col0, col1, bias) entries that receive columns [col0, col1) of C
    (tensors 2-D [M, col1 - col0], row stride any, bf16 or fp32); by default
    one new [M, N] tensor of out_dtype (with ``bias``) is returned.
    ``workspace`` (uint8, zero-filled before its first use, left zero-filled
    by every call) selects the split-K form for M <= 32."""
    if a.dim() != 2 or w.dim() != 2:
        raise ValueError("a and w must be 2-D")
    if a.dtype != torch.bfloat16 or w.dtype != torch.bfloat16:
        raise TypeError("a and w must be bfloat16")
    if not (a.is_cuda and w.is_cuda):
        raise ValueError("a and w must be CUDA tensors")
    if a.stride(1) != 1 or w.stride(1) != 1:
        raise ValueError("a and w need contiguous rows")
    M, K = a.shape
    N = w.shape[0]
    if w.shape[1] != K:
        raise ValueError("a and w disagree on K")
    ret = None
    if outs is None:
        ret = torch.empty((M, N), dtype=out_dtype, device=a.device)
        outs = [(ret, 0, N, bias)]
    args = L.GemmArgs()
    args.A, args.B = L.ptr(a), L.ptr(w)
    args.lda, args.ldb = a.stride(0), w.stride(0)
    args.M, args.N, args.K = M, N, K
    if not 1 <= len(outs) <= 3:
        raise ValueError("one to three outputs")
    for i, (t, c0, c1, b) in enumerate(outs):
        if t.dim() != 2 or t.shape[0] != M or t.shape[1] != c1 - c0 or t.stride(1) != 1:
            raise ValueError(f"output {i} must be a [M, {c1 - c0}] matrix with contiguous rows")
        _opt(b, f"bias {i}", torch.float32, (c1 - c0,))
        o = args.out[i]
        o.ptr, o.bias, o.ld, o.col0, o.col1, o.dtype = L.ptr(t), L.ptr(b), t.stride(0), c0, c1, L.dtype_code(t)
    args.nout = len(outs)
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8)
        args.workspace, args.workspace_bytes = L.ptr(workspace), workspace.numel()
    L.check(L.load().samba_gemm(ctypes.byref(args), L.stream_handle(stream)))
    return ret if ret is not None else [o[0] for o in outs]


def scan_carry(h_in, dsum, A, h_local, h_out=None, stream=None):
    """Joins a scan segment to its predecessor (see samba_scan_carry):
    h_out = exp(A * dsum) * h_in + h_local.  h_in may be None (zero state)."""
    _need(h_local, "h_local", torch.float32)
    Bsz, Dm, N = h_local.shape
    _need(dsum, "dsum", torch.float32, (Bsz, Dm))
    _need(A, "A", torch.float32, (Dm, N))
    _opt(h_in, "h_in", torch.float32, (Bsz, Dm, N))
    if h_out is None:
        h_out = torch.empty_like(h_local)
    _need(h_out, "h_out", torch.float32, (Bsz, Dm, N))
    L.check(L.load().samba_scan_carry(L.ptr(h_in), L.ptr(dsum), L.ptr(A), L.ptr(h_local), L.ptr(h_out), Bsz, Dm,
                                      N, L.stream_handle(stream)))
    return h_out


def conv_state(x, dconv, conv_state_in=None, conv_state_out=None, stream=None):
    """The conv state after x (see samba_conv_state): [B, D, K-1] fp32."""
    _need(x, "x")
    Bsz, Ln, Dm = x.shape
    _opt(conv_state_in, "conv_state_in", torch.float32, (Bsz, Dm, dconv - 1))
    if conv_state_out is None:
        conv_state_out = torch.empty((Bsz, Dm, dconv - 1), dtype=torch.float32, device=x.device)
    _need(conv_state_out, "conv_state_out", torch.float32, (Bsz, Dm, dconv - 1))
    L.check(L.load().samba_conv_state(L.ptr(x), L.dtype_code(x), L.ptr(conv_state_in), L.ptr(conv_state_out), Bsz,
                                      Ln, Dm, dconv, L.stream_handle(stream)))
    return conv_state_out


def swa_ring_fill(k, v, window, k_ring=None, v_ring=None, pos=None, stream=None):
    """Prefill -> decode hand-off of the KV window (see samba_swa_ring_fill).
    Returns (k_ring, v_ring, pos)."""
    _need(k, "k", torch.bfloat16)
    Bsz, Ln, Hkv, d = k.shape
    _need(v, "v", torch.bfloat16, k.shape)
    if k_ring is None:
        k_ring = torch.zeros((Bsz, window, Hkv, d), dtype=torch.bfloat16, device=k.device)
    if v_ring is None:
        v_ring = torch.zeros((Bsz, window, Hkv, d), dtype=torch.bfloat16, device=k.device)
    if pos is None:
        pos = torch.zeros((Bsz,), dtype=torch.int64, device=k.device)
    _need(k_ring, "k_ring", torch.bfloat16, (Bsz, window, Hkv, d))
    _need(v_ring, "v_ring", torch.bfloat16, (Bsz, window, Hkv, d))
    _need(pos, "pos", torch.int64, (Bsz,))
    L.check(L.load().samba_swa_ring_fill(L.ptr(k), L.ptr(v), Ln, L.ptr(k_ring), L.ptr(v_ring), L.ptr(pos), Bsz,
                                         Hkv, d, window, L.stream_handle(stream)))
    return k_ring, v_ring, pos


def swa_step_workspace_size(batch, heads_q, head_dim, window) -> int:
    return int(L.load().samba_swa_step_workspace_size(batch, heads_q, head_dim, window))


def swa_step(q_t, k_t, v_t, k_ring, v_ring, pos, window, scale=None, o_t=None, workspace=None, stream=None):
    """One decode step of SWA (see samba_swa_step); advances pos in place.
    Returns o_t."""
    _need(q_t, "q_t", torch.bfloat16)
    Bsz, Hq, d = q_t.shape
    Hkv = k_t.shape[1]
    _need(k_t, "k_t", torch.bfloat16, (Bsz, Hkv, d))
    _need(v_t, "v_t", torch.bfloat16, (Bsz, Hkv, d))
    _need(k_ring, "k_ring", torch.bfloat16, (Bsz, window, Hkv, d))
    _need(v_ring, "v_ring", torch.bfloat16, (Bsz, window, Hkv, d))
    _need(pos, "pos", torch.int64, (Bsz,))
    if o_t is None:
        o_t = torch.empty_like(q_t)
    nbytes = swa_step_workspace_size(Bsz, Hq, d, window)
    if workspace is None:
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=q_t.device)
    _need(workspace, "workspace", torch.uint8)
    L.check(L.load().samba_swa_step(L.ptr(q_t), L.ptr(k_t), L.ptr(v_t), L.ptr(k_ring), L.ptr(v_ring), L.ptr(pos),
                                    L.ptr(o_t), Bsz, Hq, Hkv, d, window, float(scale) if scale else 0.0,
                                    L.ptr(workspace), workspace.numel(), L.stream_handle(stream)))
    return o_t


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
