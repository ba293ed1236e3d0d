"""Thin ctypes binding of libkdn (include/kdn.h).

Argument marshalling only: every function checks that its tensors are CUDA
(host, for kdn_forward_host), contiguous and of the right dtype, allocates
outputs with PyTorch when the caller gives none, and passes raw pointers and
the current CUDA stream to the C ABI.  All arithmetic happens in the library's kernels.  If
``libkdn.so`` cannot be loaded the first call raises; there is no fallback.
Function names match the C entry points.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, 'libkdn.so')

KDN_OK, KDN_ERR_INVALID_ARG, KDN_ERR_UNSUPPORTED, KDN_ERR_WORKSPACE, KDN_ERR_TIMEOUT, \
    KDN_ERR_CUDA = range(6)
KDN_F32, KDN_BF16 = 0, 1
KDN_ISO, KDN_DIAG = 0, 1
KDN_CHUNK_AUTO, KDN_CHUNK_RECURRENT, KDN_CHUNK_64 = 0, 1, 64

_lib = None
_vp, _i64, _i32, _f32, _sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                              ctypes.c_size_t)


class KdnError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f'{where}: {lib().kdn_status_string(status).decode()}')


def lib():
    """Load libkdn.so (once) and declare the prototypes of include/kdn.h."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f'{LIB_PATH} is missing: build it with '
                           '`python -m kalman_filter_linear_b200.build`')
    L = ctypes.CDLL(LIB_PATH)
    L.kdn_status_string.restype = ctypes.c_char_p
    L.kdn_status_string.argtypes = [_i32]
    L.kdn_version.restype = _i32
    L.kdn_mobius_scan_workspace_size.restype = _sz
    L.kdn_mobius_scan_workspace_size.argtypes = [_i64, _i64]
    L.kdn_mobius_scan.restype = _i32
    L.kdn_mobius_scan.argtypes = [_vp] * 5 + [_f32] + [_vp] * 3 + [_i64, _i64, _vp, _sz, _vp]
    L.kdn_mobius_scan_noalloc.restype = _i32
    L.kdn_mobius_scan_noalloc.argtypes = [_vp] * 5 + [_f32] + [_vp] * 3 + [_i64, _i64, _vp]
    L.kdn_forward_workspace_size.restype = _sz
    L.kdn_forward_workspace_size.argtypes = [_i32] * 7
    L.kdn_iso_forward.restype = _i32
    L.kdn_iso_forward.argtypes = [_vp, _vp, _vp, _i32] + [_vp] * 8 + [_i32] * 5 + \
        [_f32, _i32, _vp, _sz, _vp]
    L.kdn_forward_varlen_workspace_size.restype = _sz
    L.kdn_forward_varlen_workspace_size.argtypes = [_i32] * 6
    L.kdn_forward_varlen.restype = _i32
    L.kdn_forward_varlen.argtypes = [_i32, _vp, _vp, _vp, _i32] + [_vp] * 9 + [_i32] * 5 + \
        [_f32, _i32, _vp, _sz, _vp]
    L.kdn_forward_host_workspace_size.restype = _sz
    L.kdn_forward_host_workspace_size.argtypes = [_i32] * 9
    L.kdn_forward_host.restype = _i32
    L.kdn_forward_host.argtypes = [_i32, _vp, _vp, _vp, _i32] + [_vp] * 8 + [_i32] * 5 + \
        [_f32, _i32, _i32, _vp, _sz, _vp]
    L.kdn_diag_forward.restype = _i32
    L.kdn_diag_forward.argtypes = [_vp, _vp, _vp, _i32] + [_vp] * 8 + [_i32] * 5 + \
        [_i32, _vp, _sz, _vp]
    L.kdn_decode_step.restype = _i32
    L.kdn_decode_step.argtypes = [_i32, _vp, _vp, _vp, _i32] + [_vp] * 6 + [_i32] * 4 + \
        [_f32, _vp]
    L.kdn_exact_forward.restype = _i32
    L.kdn_exact_forward.argtypes = [_i32, _vp, _vp, _vp, _i32] + [_vp] * 8 + [_i32] * 5 + [_vp]
    L.kdn_backward_workspace_size.restype = _sz
    L.kdn_backward_workspace_size.argtypes = [_i32] * 6
    L.kdn_backward.restype = _i32
    L.kdn_backward.argtypes = [_i32, _vp, _vp, _vp, _i32] + [_vp] * 16 + [_i32] * 5 + \
        [_f32, _vp, _sz, _vp]
    L.kdn_kla_forward.restype = _i32
    L.kdn_kla_forward.argtypes = [_vp, _vp, _vp, _i32] + [_vp] * 8 + [_i32] * 5 + [_vp]
    L.kdn_kla_workspace_size.restype = _sz
    L.kdn_kla_workspace_size.argtypes = [_i32] * 5
    L.kdn_kla_forward_ws.restype = _i32
    L.kdn_kla_forward_ws.argtypes = [_vp, _vp, _vp, _i32] + [_vp] * 8 + [_i32] * 5 + \
        [_vp, _sz, _vp]
    L.kdn_read_workspace_status.restype = _i32
    L.kdn_read_workspace_status.argtypes = [_vp, _sz, _vp]
    L.kdn_testing_mobius_scan_unpublished_tile.restype = _i32
    L.kdn_testing_kla_skip_v_copy.restype = _i32
    L.kdn_testing_kla_skip_v_copy.argtypes = [_vp] * 9 + [_i32] * 4 + [_vp, _sz, _vp]
    L.kdn_testing_forward_skip_v_copy.restype = _i32
    L.kdn_testing_forward_skip_v_copy.argtypes = [_i32] + [_vp] * 9 + [_i32] * 4 + [_vp, _sz, _vp]
    L.kdn_testing_mobius_scan_unpublished_tile.argtypes = [_vp] * 5 + [_f32, _vp, _i64, _i64,
                                                                       _vp, _sz, _i64, _vp]
    _lib = L
    return L


def _check(status, where):
    if status != KDN_OK:
        raise KdnError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _req(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f'{name} must be a CUDA tensor')
    if not t.is_contiguous():
        raise ValueError(f'{name} must be contiguous')
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f'{name} must be {dtype}, got {t.dtype}')
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f'{name} must have shape {tuple(shape)}, got {tuple(t.shape)}')
    return t


def _opt(t, name, dtype, shape):
    return None if t is None else _req(t, name, dtype, shape)


def _in_dtype(t):
    if t.dtype == torch.bfloat16:
        return KDN_BF16
    if t.dtype == torch.float32:
        return KDN_F32
    raise TypeError(f'q/k/v must be bfloat16 or float32, got {t.dtype}')


def _workspace(nbytes, device, ws):
    if nbytes == 0:
        return ws
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws


def kdn_mobius_scan_workspace_size(N, T):
    return int(lib().kdn_mobius_scan_workspace_size(N, T))


def kdn_mobius_scan(a, w, r, n, lambda0=None, info_scale=1.0, lambda_out=None, prior_out=None,
                    gain_out=None, workspace=None, want_prior=False, want_gain=False):
    """Variance (Mobius) scan over [N, T] lanes.  Returns (lambda, prior, gain,
    workspace); prior / gain are None unless requested or given."""
    N, T = a.shape
    f = torch.float32
    for name, t in (('a', a), ('w', w), ('r', r), ('n', n)):
        _req(t, name, f, (N, T))
    _opt(lambda0, 'lambda0', f, (N,))
    lambda_out = _opt(lambda_out, 'lambda_out', f, (N, T)) if lambda_out is not None else \
        torch.empty_like(a)
    if prior_out is None and want_prior:
        prior_out = torch.empty_like(a)
    if gain_out is None and want_gain:
        gain_out = torch.empty_like(a)
    _opt(prior_out, 'prior_out', f, (N, T))
    _opt(gain_out, 'gain_out', f, (N, T))
    need = kdn_mobius_scan_workspace_size(N, T)
    workspace = _workspace(need, a.device, workspace)
    st = lib().kdn_mobius_scan(_ptr(a), _ptr(w), _ptr(r), _ptr(n), _ptr(lambda0),
                               float(info_scale), _ptr(lambda_out), _ptr(prior_out),
                               _ptr(gain_out), N, T, _ptr(workspace),
                               workspace.numel() if workspace is not None else 0, _stream())
    _check(st, 'kdn_mobius_scan')
    return lambda_out, prior_out, gain_out, workspace


KDN_SCAN_NOALLOC_MAX_TILES = 229376


def kdn_mobius_scan_noalloc(a, w, r, n, lambda0=None, info_scale=1.0, lambda_out=None,
                            prior_out=None, gain_out=None, want_prior=False, want_gain=False):
    """kdn_mobius_scan with the library's internal scratch (no workspace):
    for callers that cannot allocate device memory at the call.  Returns
    (lambda, prior, gain); calls that overlap on the GPU race."""
    N, T = a.shape
    f = torch.float32
    for name, t in (('a', a), ('w', w), ('r', r), ('n', n)):
        _req(t, name, f, (N, T))
    _opt(lambda0, 'lambda0', f, (N,))
    lambda_out = _opt(lambda_out, 'lambda_out', f, (N, T)) if lambda_out is not None else \
        torch.empty_like(a)
    if prior_out is None and want_prior:
        prior_out = torch.empty_like(a)
    if gain_out is None and want_gain:
        gain_out = torch.empty_like(a)
    _opt(prior_out, 'prior_out', f, (N, T))
    _opt(gain_out, 'gain_out', f, (N, T))
    st = lib().kdn_mobius_scan_noalloc(_ptr(a), _ptr(w), _ptr(r), _ptr(n), _ptr(lambda0),
                                       float(info_scale), _ptr(lambda_out), _ptr(prior_out),
                                       _ptr(gain_out), N, T, _stream())
    _check(st, 'kdn_mobius_scan_noalloc')
    return lambda_out, prior_out, gain_out


def kdn_forward_workspace_size(variant, B, T, H, dk, dv, chunk=KDN_CHUNK_AUTO):
    return int(lib().kdn_forward_workspace_size(variant, B, T, H, dk, dv, chunk))


def _forward(variant, q, k, v, a, w, r, S0, p0, info_scale, chunk, o, S_out, p_out, workspace):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _in_dtype(q)
    _req(q, 'q', dt)
    _req(k, 'k', dt, (B, T, H, dk))
    _req(v, 'v', dt, (B, T, H, dv))
    f = torch.float32
    _req(a, 'a', f, (B, T, H))
    _req(r, 'r', f, (B, T, H))
    pshape = (B, H) if variant == KDN_ISO else (B, H, dk)
    _req(w, 'w', f, (B, T, H) if variant == KDN_ISO else (B, T, H, dk))
    _opt(S0, 'S0', f, (B, H, dv, dk))
    _opt(p0, 'p0', f, pshape)
    dev = q.device
    o = _req(o, 'o', f, (B, T, H, dv)) if o is not None else \
        torch.empty((B, T, H, dv), dtype=f, device=dev)
    S_out = _req(S_out, 'S_out', f, (B, H, dv, dk)) if S_out is not None else \
        torch.empty((B, H, dv, dk), dtype=f, device=dev)
    p_out = _req(p_out, 'p_out', f, pshape) if p_out is not None else \
        torch.empty(pshape, dtype=f, device=dev)
    need = kdn_forward_workspace_size(variant, B, T, H, dk, dv, chunk)
    workspace = _workspace(need, dev, workspace)
    wsb = workspace.numel() if workspace is not None else 0
    L = lib()
    if variant == KDN_ISO:
        st = L.kdn_iso_forward(_ptr(q), _ptr(k), _ptr(v), _in_dtype(q), _ptr(a), _ptr(w), _ptr(r),
                               _ptr(S0), _ptr(p0), _ptr(o), _ptr(S_out), _ptr(p_out), B, T, H, dk,
                               dv, float(info_scale), int(chunk), _ptr(workspace), wsb, _stream())
        _check(st, 'kdn_iso_forward')
    else:
        st = L.kdn_diag_forward(_ptr(q), _ptr(k), _ptr(v), _in_dtype(q), _ptr(a), _ptr(w),
                                _ptr(r), _ptr(S0), _ptr(p0), _ptr(o), _ptr(S_out), _ptr(p_out), B,
                                T, H, dk, dv, int(chunk), _ptr(workspace), wsb, _stream())
        _check(st, 'kdn_diag_forward')
    return o, S_out, p_out


def kdn_iso_forward(q, k, v, a, w, r, S0=None, p0=None, info_scale=0.0, chunk=KDN_CHUNK_AUTO,
                    o=None, S_out=None, p_out=None, workspace=None):
    """Isotropic KDN forward.  Returns (o fp32 [B,T,H,dv], S_T, p_T)."""
    return _forward(KDN_ISO, q, k, v, a, w, r, S0, p0, info_scale, chunk, o, S_out, p_out,
                    workspace)


def kdn_diag_forward(q, k, v, a, w, r, S0=None, p0=None, chunk=KDN_CHUNK_AUTO, o=None,
                     S_out=None, p_out=None, workspace=None):
    """Diagonal KDN forward.  Returns (o fp32 [B,T,H,dv], S_T, p_T [B,H,dk])."""
    return _forward(KDN_DIAG, q, k, v, a, w, r, S0, p0, 1.0, chunk, o, S_out, p_out, workspace)


def kdn_forward_varlen_workspace_size(variant, N, H, dk, dv, chunk=KDN_CHUNK_AUTO):
    return int(lib().kdn_forward_varlen_workspace_size(variant, N, H, dk, dv, chunk))


def kdn_forward_varlen(variant, q, k, v, a, w, r, cu_seqlens, S0=None, p0=None, info_scale=0.0,
                       chunk=KDN_CHUNK_AUTO, o=None, S_out=None, p_out=None, workspace=None):
    """The forward over packed sequences: q, k [total, H, dk], v [total, H, dv],
    a, r [total, H], w [total, H] (iso) or [total, H, dk] (diag), cu_seqlens
    [N + 1] int32.  Returns (o [total, H, dv], S_T [N, H, dv, dk], p_T)."""
    total, H, dk = q.shape
    dv = v.shape[-1]
    N = cu_seqlens.numel() - 1
    dt = q.dtype
    _in_dtype(q)
    _req(q, 'q', dt)
    _req(k, 'k', dt, (total, H, dk))
    _req(v, 'v', dt, (total, H, dv))
    f = torch.float32
    _req(a, 'a', f, (total, H))
    _req(r, 'r', f, (total, H))
    pshape = (N, H) if variant == KDN_ISO else (N, H, dk)
    _req(w, 'w', f, (total, H) if variant == KDN_ISO else (total, H, dk))
    _req(cu_seqlens, 'cu_seqlens', torch.int32, (N + 1,))
    _opt(S0, 'S0', f, (N, H, dv, dk))
    _opt(p0, 'p0', f, pshape)
    dev = q.device
    o = _req(o, 'o', f, (total, H, dv)) if o is not None else \
        torch.empty((total, H, dv), dtype=f, device=dev)
    S_out = _req(S_out, 'S_out', f, (N, H, dv, dk)) if S_out is not None else \
        torch.empty((N, H, dv, dk), dtype=f, device=dev)
    p_out = _req(p_out, 'p_out', f, pshape) if p_out is not None else \
        torch.empty(pshape, dtype=f, device=dev)
    need = kdn_forward_varlen_workspace_size(variant, N, H, dk, dv, chunk)
    workspace = _workspace(need, dev, workspace)
    st = lib().kdn_forward_varlen(variant, _ptr(q), _ptr(k), _ptr(v), _in_dtype(q), _ptr(a),
                                  _ptr(w), _ptr(r), _ptr(cu_seqlens), _ptr(S0), _ptr(p0), _ptr(o),
                                  _ptr(S_out), _ptr(p_out), N, total, H, dk, dv,
                                  float(info_scale), int(chunk), _ptr(workspace),
                                  workspace.numel(), _stream())
    _check(st, 'kdn_forward_varlen')
    return o, S_out, p_out


def _req_host(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise TypeError(f'{name} must be a host (CPU) tensor')
    if not t.is_contiguous():
        raise ValueError(f'{name} must be contiguous')
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f'{name} must be {dtype}, got {t.dtype}')
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f'{name} must have shape {tuple(shape)}, got {tuple(t.shape)}')
    return t


def kdn_forward_host_workspace_size(variant, B, T, H, dk, dv, in_dtype=KDN_BF16,
                                    chunk=KDN_CHUNK_AUTO, slice_b=0):
    return int(lib().kdn_forward_host_workspace_size(variant, B, T, H, dk, dv, in_dtype, chunk,
                                                     slice_b))


def kdn_forward_host(variant, q, k, v, a, w, r, S0=None, p0=None, info_scale=0.0,
                     chunk=KDN_CHUNK_AUTO, slice_b=0, o=None, S_out=None, p_out=None,
                     workspace=None, device=None):
    """The forward with host tensors (pinned for overlap); outputs are host
    tensors, valid once the current stream has been synchronised.  Returns
    (o, S_T, p_T)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _in_dtype(q)
    _req_host(q, 'q', dt)
    _req_host(k, 'k', dt, (B, T, H, dk))
    _req_host(v, 'v', dt, (B, T, H, dv))
    f = torch.float32
    _req_host(a, 'a', f, (B, T, H))
    _req_host(r, 'r', f, (B, T, H))
    pshape = (B, H) if variant == KDN_ISO else (B, H, dk)
    _req_host(w, 'w', f, (B, T, H) if variant == KDN_ISO else (B, T, H, dk))
    if S0 is not None:
        _req_host(S0, 'S0', f, (B, H, dv, dk))
    if p0 is not None:
        _req_host(p0, 'p0', f, pshape)
    o = _req_host(o, 'o', f, (B, T, H, dv)) if o is not None else \
        torch.empty((B, T, H, dv), dtype=f).pin_memory()
    S_out = _req_host(S_out, 'S_out', f, (B, H, dv, dk)) if S_out is not None else \
        torch.empty((B, H, dv, dk), dtype=f).pin_memory()
    p_out = _req_host(p_out, 'p_out', f, pshape) if p_out is not None else \
        torch.empty(pshape, dtype=f).pin_memory()
    need = kdn_forward_host_workspace_size(variant, B, T, H, dk, dv, _in_dtype(q), chunk, slice_b)
    dev = device if device is not None else torch.device('cuda', torch.cuda.current_device())
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _req(workspace, 'workspace', torch.uint8)
    st = lib().kdn_forward_host(variant, _ptr(q), _ptr(k), _ptr(v), _in_dtype(q), _ptr(a),
                                _ptr(w), _ptr(r), _ptr(S0), _ptr(p0), _ptr(o), _ptr(S_out),
                                _ptr(p_out), B, T, H, dk, dv, float(info_scale), int(chunk),
                                int(slice_b), _ptr(workspace), workspace.numel(), _stream())
    _check(st, 'kdn_forward_host')
    return o, S_out, p_out


def kdn_decode_step(variant, q, k, v, a, w, r, S, p, o=None, info_scale=0.0):
    """One decode step; S and p are updated in place.  Returns o [B,H,dv]."""
    var = KDN_DIAG if variant in ('diag', KDN_DIAG) else KDN_ISO
    B, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _req(q, 'q', dt)
    _req(k, 'k', dt, (B, H, dk))
    _req(v, 'v', dt, (B, H, dv))
    f = torch.float32
    _req(a, 'a', f, (B, H))
    _req(r, 'r', f, (B, H))
    _req(w, 'w', f, (B, H) if var == KDN_ISO else (B, H, dk))
    _req(S, 'S', f, (B, H, dv, dk))
    _req(p, 'p', f, (B, H) if var == KDN_ISO else (B, H, dk))
    o = _req(o, 'o', f, (B, H, dv)) if o is not None else \
        torch.empty((B, H, dv), dtype=f, device=q.device)
    st = lib().kdn_decode_step(var, _ptr(q), _ptr(k), _ptr(v), _in_dtype(q), _ptr(a), _ptr(w),
                               _ptr(r), _ptr(S), _ptr(p), _ptr(o), B, H, dk, dv,
                               float(info_scale), _stream())
    _check(st, 'kdn_decode_step')
    return o


def kdn_exact_forward(variant, q, k, v, a, w, r, S0=None, P0=None, o=None, S_out=None,
                      P_out=None):
    """The dense (full-covariance) Kalman filter: q, k [B,T,H,dk], v [B,T,H,dv],
    a, r [B,T,H], w [B,T,H] (iso: W = w I) or [B,T,H,dk] (diag: W = diag(w)).
    Returns (o [B,T,H,dv], S_T [B,H,dv,dk], P_T [B,H,dk,dk])."""
    var = KDN_DIAG if variant in ('diag', KDN_DIAG) else KDN_ISO
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _in_dtype(q)
    _req(q, 'q', dt)
    _req(k, 'k', dt, (B, T, H, dk))
    _req(v, 'v', dt, (B, T, H, dv))
    f = torch.float32
    _req(a, 'a', f, (B, T, H))
    _req(r, 'r', f, (B, T, H))
    _req(w, 'w', f, (B, T, H) if var == KDN_ISO else (B, T, H, dk))
    _opt(S0, 'S0', f, (B, H, dv, dk))
    _opt(P0, 'P0', f, (B, H, dk, dk))
    dev = q.device
    o = _req(o, 'o', f, (B, T, H, dv)) if o is not None else \
        torch.empty((B, T, H, dv), dtype=f, device=dev)
    S_out = _req(S_out, 'S_out', f, (B, H, dv, dk)) if S_out is not None else \
        torch.empty((B, H, dv, dk), dtype=f, device=dev)
    P_out = _req(P_out, 'P_out', f, (B, H, dk, dk)) if P_out is not None else \
        torch.empty((B, H, dk, dk), dtype=f, device=dev)
    st = lib().kdn_exact_forward(var, _ptr(q), _ptr(k), _ptr(v), _in_dtype(q), _ptr(a), _ptr(w),
                                 _ptr(r), _ptr(S0), _ptr(P0), _ptr(o), _ptr(S_out), _ptr(P_out),
                                 B, T, H, dk, dv, _stream())
    _check(st, 'kdn_exact_forward')
    return o, S_out, P_out


def kdn_backward_workspace_size(variant, B, T, H, dk, dv):
    return int(lib().kdn_backward_workspace_size(variant, B, T, H, dk, dv))


def kdn_backward(variant, q, k, v, a, w, r, dO, S0=None, p0=None, dS_T=None, dp_T=None,
                 info_scale=0.0, workspace=None):
    """Backward of the layer forward: returns a dict of the gradients
    q, k, v, a, w, r, S0, p0 (fp32, shaped like the inputs) of the loss whose
    gradients with respect to o, S_T and p_T are dO, dS_T, dp_T."""
    var = KDN_DIAG if variant in ('diag', KDN_DIAG) else KDN_ISO
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _in_dtype(q)
    _req(q, 'q', dt)
    _req(k, 'k', dt, (B, T, H, dk))
    _req(v, 'v', dt, (B, T, H, dv))
    f = torch.float32
    _req(a, 'a', f, (B, T, H))
    _req(r, 'r', f, (B, T, H))
    wshape = (B, T, H) if var == KDN_ISO else (B, T, H, dk)
    pshape = (B, H) if var == KDN_ISO else (B, H, dk)
    _req(w, 'w', f, wshape)
    _req(dO, 'dO', f, (B, T, H, dv))
    _opt(S0, 'S0', f, (B, H, dv, dk))
    _opt(p0, 'p0', f, pshape)
    _opt(dS_T, 'dS_T', f, (B, H, dv, dk))
    _opt(dp_T, 'dp_T', f, pshape)
    dev = q.device
    g = dict(q=torch.empty((B, T, H, dk), dtype=f, device=dev),
             k=torch.empty((B, T, H, dk), dtype=f, device=dev),
             v=torch.empty((B, T, H, dv), dtype=f, device=dev),
             a=torch.empty((B, T, H), dtype=f, device=dev),
             w=torch.empty(wshape, dtype=f, device=dev),
             r=torch.empty((B, T, H), dtype=f, device=dev),
             S0=torch.empty((B, H, dv, dk), dtype=f, device=dev),
             p0=torch.empty(pshape, dtype=f, device=dev))
    need = kdn_backward_workspace_size(var, B, T, H, dk, dv)
    workspace = _workspace(need, dev, workspace)
    st = lib().kdn_backward(var, _ptr(q), _ptr(k), _ptr(v), _in_dtype(q), _ptr(a), _ptr(w),
                            _ptr(r), _ptr(S0), _ptr(p0), _ptr(dO), _ptr(dS_T), _ptr(dp_T),
                            _ptr(g['q']), _ptr(g['k']), _ptr(g['v']), _ptr(g['a']), _ptr(g['w']),
                            _ptr(g['r']), _ptr(g['S0']), _ptr(g['p0']), B, T, H, dk, dv,
                            float(info_scale), _ptr(workspace), workspace.numel(), _stream())
    _check(st, 'kdn_backward')
    return g


def kdn_kla_workspace_size(B, T, H, dk, dv):
    return int(lib().kdn_kla_workspace_size(B, T, H, dk, dv))


def kdn_kla_forward(q, k, v, a, w, r, S0=None, lam0=None, o=None, S_out=None, lam_out=None,
                    workspace=None, recurrent=False):
    """The information-form diagonal filter (KLA): q, k [B,T,H,dk], v [B,T,H,dv],
    a, r [B,T,H], w [B,T,H,dk].  Returns (o [B,T,H,dv], S_T [B,H,dv,dk],
    lam_T [B,H,dk]) -- lam is the precision.  By default this is
    kdn_kla_forward_ws (the chunked tensor-core engine at dk = dv = 128 with
    bf16 inputs, the token-recurrent kernel otherwise); recurrent=True calls
    kdn_kla_forward, the token-recurrent kernel for every shape."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _in_dtype(q)
    _req(q, 'q', dt)
    _req(k, 'k', dt, (B, T, H, dk))
    _req(v, 'v', dt, (B, T, H, dv))
    f = torch.float32
    _req(a, 'a', f, (B, T, H))
    _req(r, 'r', f, (B, T, H))
    _req(w, 'w', f, (B, T, H, dk))
    _opt(S0, 'S0', f, (B, H, dv, dk))
    _opt(lam0, 'lam0', f, (B, H, dk))
    dev = q.device
    o = _req(o, 'o', f, (B, T, H, dv)) if o is not None else \
        torch.empty((B, T, H, dv), dtype=f, device=dev)
    S_out = _req(S_out, 'S_out', f, (B, H, dv, dk)) if S_out is not None else \
        torch.empty((B, H, dv, dk), dtype=f, device=dev)
    lam_out = _req(lam_out, 'lam_out', f, (B, H, dk)) if lam_out is not None else \
        torch.empty((B, H, dk), dtype=f, device=dev)
    if recurrent:
        st = lib().kdn_kla_forward(_ptr(q), _ptr(k), _ptr(v), _in_dtype(q), _ptr(a), _ptr(w),
                                   _ptr(r), _ptr(S0), _ptr(lam0), _ptr(o), _ptr(S_out),
                                   _ptr(lam_out), B, T, H, dk, dv, _stream())
        _check(st, 'kdn_kla_forward')
        return o, S_out, lam_out
    need = kdn_kla_workspace_size(B, T, H, dk, dv)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    st = lib().kdn_kla_forward_ws(_ptr(q), _ptr(k), _ptr(v), _in_dtype(q), _ptr(a), _ptr(w),
                                  _ptr(r), _ptr(S0), _ptr(lam0), _ptr(o), _ptr(S_out),
                                  _ptr(lam_out), B, T, H, dk, dv, _ptr(workspace),
                                  workspace.numel(), _stream())
    _check(st, 'kdn_kla_forward_ws')
    return o, S_out, lam_out


def kdn_read_workspace_status(workspace):
    """Synchronise the current stream and return the workspace's status code."""
    return int(lib().kdn_read_workspace_status(_ptr(workspace), workspace.numel(), _stream()))


def kdn_testing_mobius_scan_unpublished_tile(a, w, r, n, silent_tile, info_scale=1.0):
    """Fault-injection hook: the scan with one tile that never publishes."""
    N, T = a.shape
    out = torch.empty_like(a)
    need = kdn_mobius_scan_workspace_size(N, T)
    ws = torch.empty(need, dtype=torch.uint8, device=a.device)
    st = lib().kdn_testing_mobius_scan_unpublished_tile(
        _ptr(a), _ptr(w), _ptr(r), _ptr(n), None, float(info_scale), _ptr(out), N, T, _ptr(ws),
        need, int(silent_tile), _stream())
    _check(st, 'kdn_testing_mobius_scan_unpublished_tile')
    return out, ws


def kdn_testing_forward_skip_v_copy(variant, q, k, v, a, w, r, skip_chunk, workspace):
    """Fault-injection hook: the chunked forward (d = 128, bf16) with one V
    copy left out, so a bounded wait gives up.  Returns (o, S_T, p_T); the
    status is in the workspace."""
    B, T, H, d = q.shape
    for t, n in ((q, 'q'), (k, 'k'), (v, 'v')):
        _req(t, n, torch.bfloat16, (B, T, H, d))
    f = torch.float32
    _req(a, 'a', f, (B, T, H))
    _req(r, 'r', f, (B, T, H))
    _req(w, 'w', f, (B, T, H) if variant == KDN_ISO else (B, T, H, d))
    _req(workspace, 'workspace', torch.uint8)
    o = torch.empty((B, T, H, d), dtype=f, device=q.device)
    S = torch.empty((B, H, d, d), dtype=f, device=q.device)
    p = torch.empty((B, H) if variant == KDN_ISO else (B, H, d), dtype=f, device=q.device)
    st = lib().kdn_testing_forward_skip_v_copy(variant, _ptr(q), _ptr(k), _ptr(v), _ptr(a),
                                               _ptr(w), _ptr(r), _ptr(o), _ptr(S), _ptr(p), B, T,
                                               H, int(skip_chunk), _ptr(workspace),
                                               workspace.numel(), _stream())
    _check(st, 'kdn_testing_forward_skip_v_copy')
    return o, S, p


def kdn_testing_kla_skip_v_copy(q, k, v, a, w, r, skip_chunk, workspace):
    """Fault-injection hook: the KLA engine (d = 128, bf16) with one V copy
    left out, so a bounded wait gives up.  Returns (o, S_T, lam_T); the status
    is in the workspace."""
    B, T, H, d = q.shape
    for t, n in ((q, 'q'), (k, 'k'), (v, 'v')):
        _req(t, n, torch.bfloat16, (B, T, H, d))
    f = torch.float32
    _req(a, 'a', f, (B, T, H))
    _req(r, 'r', f, (B, T, H))
    _req(w, 'w', f, (B, T, H, d))
    _req(workspace, 'workspace', torch.uint8)
    o = torch.empty((B, T, H, d), dtype=f, device=q.device)
    S = torch.empty((B, H, d, d), dtype=f, device=q.device)
    lam = torch.empty((B, H, d), dtype=f, device=q.device)
    st = lib().kdn_testing_kla_skip_v_copy(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(w), _ptr(r),
                                           _ptr(o), _ptr(S), _ptr(lam), B, T, H, int(skip_chunk),
                                           _ptr(workspace), workspace.numel(), _stream())
    _check(st, 'kdn_testing_kla_skip_v_copy')
    return o, S, lam
