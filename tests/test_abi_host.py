"""The C-ABI library loads and exports what include/*.h declares (CPU only).

Only calls that must fail argument validation are made here: those return
before touching the CUDA runtime, so no GPU is needed.
"""
import ctypes
import glob
import os
import re

import pytest

from kalman_filter_linear_b200 import kdn, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope='module')
def L():
    if build.is_stale():
        build.build()
    return kdn.lib()


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, 'include', '*.h')):
        src = open(h).read()
        src = re.sub(r'/\*.*?\*/', '', src, flags=re.S)
        for m in re.finditer(r'\b(kdn_[a-z0-9_]+)\s*\(', src):
            names.add(m.group(1))
    return sorted(names)


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert 'kdn_iso_forward' in names and 'kdn_mobius_scan' in names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    for s in range(6):
        assert L.kdn_status_string(s).startswith(b'KDN_')
    assert L.kdn_status_string(99) == b'unknown kdn_status'
    assert L.kdn_version() >= 200


def test_workspace_sizes_are_host_computable(L):
    assert kdn.kdn_mobius_scan_workspace_size(0, 10) == 0
    s1 = kdn.kdn_mobius_scan_workspace_size(4096, 65536)
    s2 = kdn.kdn_mobius_scan_workspace_size(4096, 65537)
    assert s1 > 0 and s2 > s1 and s1 % 256 == 0
    assert kdn.kdn_forward_workspace_size(kdn.KDN_ISO, 1, 1, 1, 64, 64,
                                          kdn.KDN_CHUNK_RECURRENT) == 0


FAKE = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced
MIS = ctypes.c_void_p(0x10004)   # misaligned


def test_scan_rejects_bad_arguments(L):
    ws = ctypes.c_void_p(0x20000)
    big = ctypes.c_size_t(1 << 40)
    call = lambda *a: L.kdn_mobius_scan(*a)
    assert call(None, FAKE, FAKE, FAKE, None, 1.0, FAKE, None, None, 4, 8, ws, big, None) == \
        kdn.KDN_ERR_INVALID_ARG
    assert call(FAKE, FAKE, FAKE, FAKE, None, 1.0, FAKE, None, None, 0, 8, ws, big, None) == \
        kdn.KDN_ERR_INVALID_ARG
    assert call(FAKE, FAKE, FAKE, FAKE, None, -1.0, FAKE, None, None, 4, 8, ws, big, None) == \
        kdn.KDN_ERR_INVALID_ARG
    assert call(MIS, FAKE, FAKE, FAKE, None, 1.0, FAKE, None, None, 4, 8, ws, big, None) == \
        kdn.KDN_ERR_INVALID_ARG
    assert call(FAKE, FAKE, FAKE, FAKE, None, 1.0, FAKE, None, None, 4, 8, ws, 16, None) == \
        kdn.KDN_ERR_WORKSPACE
    assert call(FAKE, FAKE, FAKE, FAKE, None, 1.0, FAKE, None, None, 4, 8, None, big, None) == \
        kdn.KDN_ERR_WORKSPACE


def _fwd(L, **kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, dt=kdn.KDN_BF16, a=FAKE, w=FAKE, r=FAKE, S0=None,
                p0=None, o=FAKE, S=FAKE, p=FAKE, B=1, T=8, H=1, dk=128, dv=128, kappa=0.0,
                chunk=kdn.KDN_CHUNK_RECURRENT, ws=None, wsb=0, stream=None)
    args.update(kw)
    return L.kdn_iso_forward(*args.values())


def test_forward_rejects_bad_arguments(L):
    assert _fwd(L, q=None) == kdn.KDN_ERR_INVALID_ARG
    assert _fwd(L, o=None) == kdn.KDN_ERR_INVALID_ARG
    assert _fwd(L, dt=7) == kdn.KDN_ERR_INVALID_ARG
    assert _fwd(L, B=0) == kdn.KDN_ERR_INVALID_ARG
    assert _fwd(L, T=-3) == kdn.KDN_ERR_INVALID_ARG
    assert _fwd(L, k=MIS) == kdn.KDN_ERR_INVALID_ARG
    assert _fwd(L, S0=MIS) == kdn.KDN_ERR_INVALID_ARG
    assert _fwd(L, kappa=float('nan')) == kdn.KDN_ERR_INVALID_ARG
    assert _fwd(L, dk=96) == kdn.KDN_ERR_UNSUPPORTED
    assert _fwd(L, dv=200) == kdn.KDN_ERR_UNSUPPORTED
    assert _fwd(L, chunk=5) == kdn.KDN_ERR_INVALID_ARG
    # the chunked engine takes bf16 inputs only
    assert _fwd(L, dt=kdn.KDN_F32, chunk=kdn.KDN_CHUNK_64) == kdn.KDN_ERR_UNSUPPORTED
    assert L.kdn_diag_forward(FAKE, FAKE, FAKE, kdn.KDN_BF16, FAKE, FAKE, FAKE, None, None, FAKE,
                              FAKE, FAKE, 1, 8, 1, 128, 128, 3, None, 0, None) == \
        kdn.KDN_ERR_INVALID_ARG


def test_decode_rejects_bad_arguments(L):
    d = lambda **kw: L.kdn_decode_step(*dict(dict(var=kdn.KDN_DIAG, q=FAKE, k=FAKE, v=FAKE,
                                                  dt=kdn.KDN_BF16, a=FAKE, w=FAKE, r=FAKE, S=FAKE,
                                                  p=FAKE, o=FAKE, B=2, H=2, dk=128, dv=128,
                                                  kappa=0.0, stream=None), **kw).values())
    assert d(var=5) == kdn.KDN_ERR_INVALID_ARG
    assert d(S=None) == kdn.KDN_ERR_INVALID_ARG
    assert d(p=MIS) == kdn.KDN_ERR_INVALID_ARG
    assert d(H=0) == kdn.KDN_ERR_INVALID_ARG
    assert d(dk=48) == kdn.KDN_ERR_UNSUPPORTED
    assert L.kdn_read_workspace_status(None, 0, None) == kdn.KDN_ERR_INVALID_ARG


def test_exact_forward_rejects_bad_arguments(L):
    base = dict(var=kdn.KDN_ISO, q=FAKE, k=FAKE, v=FAKE, dt=kdn.KDN_F32, a=FAKE, w=FAKE, r=FAKE,
                S0=None, P0=None, o=FAKE, S=FAKE, P=FAKE, B=1, T=8, H=1, dk=64, dv=64,
                stream=None)
    x = lambda **kw: L.kdn_exact_forward(*dict(base, **kw).values())
    assert x(q=None) == kdn.KDN_ERR_INVALID_ARG
    assert x(P=None) == kdn.KDN_ERR_INVALID_ARG
    assert x(var=7) == kdn.KDN_ERR_INVALID_ARG
    assert x(dt=9) == kdn.KDN_ERR_INVALID_ARG
    assert x(T=0) == kdn.KDN_ERR_INVALID_ARG
    assert x(B=0) == kdn.KDN_ERR_INVALID_ARG
    assert x(P0=MIS) == kdn.KDN_ERR_INVALID_ARG
    assert x(o=MIS) == kdn.KDN_ERR_INVALID_ARG
    assert x(dk=128) == kdn.KDN_ERR_UNSUPPORTED   # small d_k only
    assert x(dk=16) == kdn.KDN_ERR_UNSUPPORTED
    assert x(dv=12) == kdn.KDN_ERR_UNSUPPORTED    # d_v a multiple of 8
    assert x(dv=136) == kdn.KDN_ERR_UNSUPPORTED


def test_kla_forward_rejects_bad_arguments(L):
    base = dict(q=FAKE, k=FAKE, v=FAKE, dt=kdn.KDN_BF16, a=FAKE, w=FAKE, r=FAKE, S0=None,
                lam0=None, o=FAKE, S=FAKE, lam=FAKE, B=1, T=8, H=1, dk=128, dv=128, stream=None)
    x = lambda **kw: L.kdn_kla_forward(*dict(base, **kw).values())
    assert x(v=None) == kdn.KDN_ERR_INVALID_ARG
    assert x(lam=None) == kdn.KDN_ERR_INVALID_ARG
    assert x(dt=9) == kdn.KDN_ERR_INVALID_ARG
    assert x(T=0) == kdn.KDN_ERR_INVALID_ARG
    assert x(lam0=MIS) == kdn.KDN_ERR_INVALID_ARG
    assert x(dk=96) == kdn.KDN_ERR_UNSUPPORTED
    assert x(dv=4) == kdn.KDN_ERR_UNSUPPORTED
    assert x(dv=130) == kdn.KDN_ERR_UNSUPPORTED


def test_backward_rejects_bad_arguments(L):
    base = dict(var=kdn.KDN_ISO, q=FAKE, k=FAKE, v=FAKE, dt=kdn.KDN_F32, a=FAKE, w=FAKE, r=FAKE,
                S0=None, p0=None, dO=FAKE, dS_T=None, dp_T=None, dq=FAKE, dk=FAKE, dv=FAKE,
                da=FAKE, dw=FAKE, dr=FAKE, dS0=FAKE, dp0=FAKE, B=1, T=8, H=1, dkk=64, dvv=64,
                kappa=0.0, ws=ctypes.c_void_p(0x20000), wsb=1 << 40, stream=None)
    x = lambda **kw: L.kdn_backward(*dict(base, **kw).values())
    assert x(dO=None) == kdn.KDN_ERR_INVALID_ARG
    assert x(dp0=None) == kdn.KDN_ERR_INVALID_ARG
    assert x(var=5) == kdn.KDN_ERR_INVALID_ARG
    assert x(T=0) == kdn.KDN_ERR_INVALID_ARG
    assert x(dS_T=MIS) == kdn.KDN_ERR_INVALID_ARG
    assert x(dkk=96) == kdn.KDN_ERR_UNSUPPORTED
    assert x(dvv=129) == kdn.KDN_ERR_INVALID_ARG or x(dvv=129) == kdn.KDN_ERR_UNSUPPORTED
    assert x(ws=None) == kdn.KDN_ERR_WORKSPACE
    assert x(wsb=16) == kdn.KDN_ERR_WORKSPACE
    # per head: one state checkpoint (T = 10 < 16) and 16 rebuilt states
    assert L.kdn_backward_workspace_size(kdn.KDN_DIAG, 2, 10, 3, 32, 16) >= 2 * 3 * 17 * 16 * 32 * 4
    assert L.kdn_backward_workspace_size(kdn.KDN_ISO, 1, 8, 1, 128, 128) > 0


def test_varlen_rejects_bad_arguments(L):
    ws = ctypes.c_void_p(0x20000)
    base = dict(var=kdn.KDN_ISO, q=FAKE, k=FAKE, v=FAKE, dt=kdn.KDN_BF16, a=FAKE, w=FAKE, r=FAKE,
                cu=FAKE, S0=None, p0=None, o=FAKE, S=FAKE, p=FAKE, N=4, total=100, H=2, dk=128,
                dv=128, kappa=0.0, chunk=0, ws=ws, wsb=1 << 30, stream=None)
    x = lambda **kw: L.kdn_forward_varlen(*dict(base, **kw).values())
    assert x(cu=None) == kdn.KDN_ERR_INVALID_ARG         # offsets are required
    assert x(total=-1) == kdn.KDN_ERR_INVALID_ARG
    assert x(var=3) == kdn.KDN_ERR_INVALID_ARG
    assert x(N=0) == kdn.KDN_ERR_INVALID_ARG
    assert x(o=MIS) == kdn.KDN_ERR_INVALID_ARG
    assert x(ws=None) == kdn.KDN_ERR_WORKSPACE
    assert x(wsb=64) == kdn.KDN_ERR_WORKSPACE              # at least the 256-byte error word
    assert x(chunk=kdn.KDN_CHUNK_64, dv=64, dk=128) == kdn.KDN_ERR_UNSUPPORTED
    assert L.kdn_forward_varlen_workspace_size(kdn.KDN_ISO, 4, 2, 128, 128, 0) >= 256
    assert L.kdn_forward_varlen_workspace_size(kdn.KDN_ISO, 0, 2, 128, 128, 0) == 0


def test_host_forward_rejects_bad_arguments(L):
    ws = ctypes.c_void_p(0x20000)
    base = dict(var=kdn.KDN_ISO, q=FAKE, k=FAKE, v=FAKE, dt=kdn.KDN_BF16, a=FAKE, w=FAKE, r=FAKE,
                S0=None, p0=None, o=FAKE, S=FAKE, p=FAKE, B=2, T=64, H=2, dk=128, dv=128,
                kappa=0.0, chunk=0, slice_b=1, ws=ws, wsb=1 << 40, stream=None)
    x = lambda **kw: L.kdn_forward_host(*dict(base, **kw).values())
    assert x(var=2) == kdn.KDN_ERR_INVALID_ARG
    assert x(p=None) == kdn.KDN_ERR_INVALID_ARG
    assert x(dt=5) == kdn.KDN_ERR_INVALID_ARG
    assert x(T=0) == kdn.KDN_ERR_INVALID_ARG
    assert x(dk=96) == kdn.KDN_ERR_UNSUPPORTED
    assert x(ws=None) == kdn.KDN_ERR_WORKSPACE
    assert x(wsb=1024) == kdn.KDN_ERR_WORKSPACE
    assert x(ws=ctypes.c_void_p(0x20010)) == kdn.KDN_ERR_INVALID_ARG  # not 256-byte aligned
    need = L.kdn_forward_host_workspace_size(kdn.KDN_ISO, 2, 64, 2, 128, 128, kdn.KDN_BF16, 0, 1)
    assert need > 256


def test_read_status_rejects_a_missing_workspace(L):
    assert L.kdn_read_workspace_status(None, 256, None) == kdn.KDN_ERR_INVALID_ARG
    assert L.kdn_read_workspace_status(FAKE, 2, None) == kdn.KDN_ERR_INVALID_ARG
