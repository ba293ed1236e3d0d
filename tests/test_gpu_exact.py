"""The dense (full-covariance) Kalman filter kernel (kdn_exact_forward)
against the fp64 dense oracle, run head by head (needs a B200).

The kernel computes in fp32 from fp32 (or exact bf16) inputs and the
recursion contracts (decay below 1, gains below 1), so its error stays at a
few fp32 roundings per token: o and S within 1e-4 of max-abs over RMS, P
within 1e-4.  The axis-aligned pin checks the kernel against the diagonal KDN
kernel (where the exact covariance stays diagonal, both are the same filter).
"""
import numpy as np
import pytest
import torch

from kalman_filter_linear_b200 import kdn, synth
from oracle import exact_kalman
from gpu_util import rel_maxabs, f64

pytestmark = pytest.mark.gpu

EXACT_TOL = 1e-4


def _W(w, variant, dk):
    """Process-noise covariances [T, dk, dk] of one head: w I or diag(w)."""
    w = np.asarray(w, np.float64)
    if variant == 'iso':
        return w[:, None, None] * np.eye(dk)[None]
    return np.einsum('ti,ij->tij', w, np.eye(dk))


def _spd(g, n, dk):
    A = torch.randn(n, dk, dk, generator=g) / dk ** 0.5
    return (A @ A.transpose(-1, -2) * 0.5 + 0.3 * torch.eye(dk)).contiguous()


def _oracle(variant, x, S0, P0, heads):
    """o, S_T, P_T of the given (b, h) heads from the fp64 dense filter."""
    out = {}
    dk = x['k'].shape[-1]
    for b, h in heads:
        o, S_all, P_all, _ = exact_kalman.exact_forward(
            f64(x['q'][b, :, h]), f64(x['k'][b, :, h]), f64(x['v'][b, :, h]),
            f64(x['a'][b, :, h]), _W(f64(x['w'][b, :, h]), variant, dk), f64(x['r'][b, :, h]),
            f64(S0[b, h]) if S0 is not None else np.zeros((x['v'].shape[-1], dk)),
            f64(P0[b, h]) if P0 is not None else np.eye(dk))
        out[(b, h)] = (o, S_all[-1], P_all[-1])
    return out


@pytest.mark.parametrize("variant", ["iso", "diag"])
@pytest.mark.parametrize("dk,dv,dtype", [(64, 64, 'bf16'), (32, 128, 'f32'), (64, 40, 'f32'),
                                         (32, 24, 'bf16'), (64, 8, 'f32'), (64, 24, 'bf16'),
                                         (32, 48, 'f32'), (64, 128, 'bf16')])
def test_exact_matches_dense_oracle(variant, dk, dv, dtype):
    """Random SPD P0 and a non-zero S0; T = 150 spans nine 16-token stages
    and a ragged one.  The shapes take every state-warp count the kernel has:
    one (d_v rows of d_k / 32 lanes fit in a warp: (32, 24), (64, 8)), two
    ((64, 24), (32, 48)), four ((64, 64), (32, 128), (64, 40)) and eight
    ((64, 128))."""
    B, T, H = 2, 150, 2
    x = synth.layer_inputs(B, T, H, dk, dv, variant, seed=31 + dk + dv, dtype=dtype)
    g = torch.Generator().manual_seed(5)
    S0 = 0.05 * torch.randn(B, H, dv, dk, generator=g)
    P0 = _spd(g, B * H, dk).reshape(B, H, dk, dk)
    xd = {k: v.cuda() for k, v in x.items()}
    o, S, P = kdn.kdn_exact_forward(variant, xd['q'], xd['k'], xd['v'], xd['a'], xd['w'],
                                    xd['r'], S0.cuda(), P0.cuda())
    torch.cuda.synchronize()
    ref = _oracle(variant, x, S0, P0, [(b, h) for b in range(B) for h in range(H)])
    for (b, h), (o_r, S_r, P_r) in ref.items():
        assert rel_maxabs(o[b, :, h], o_r) <= EXACT_TOL, (b, h)
        assert rel_maxabs(S[b, h], S_r) <= EXACT_TOL, (b, h)
        assert rel_maxabs(P[b, h], P_r) <= EXACT_TOL, (b, h)
    # the covariance stays exactly symmetric
    assert torch.equal(P, P.transpose(-1, -2))


def test_exact_default_state_and_in_place():
    """NULL S0 / P0 mean zeros and the identity; S_out and P_out may be the
    same buffers as S0 and P0."""
    B, T, H, d = 1, 40, 3, 32
    x = synth.layer_inputs(B, T, H, d, d, 'diag', seed=8, dtype='f32')
    xd = {k: v.cuda() for k, v in x.items()}
    o1, S1, P1 = kdn.kdn_exact_forward('diag', xd['q'], xd['k'], xd['v'], xd['a'], xd['w'],
                                       xd['r'])
    S = torch.zeros(B, H, d, d, device='cuda')
    P = torch.eye(d, device='cuda').expand(B, H, d, d).contiguous()
    o2, _, _ = kdn.kdn_exact_forward('diag', xd['q'], xd['k'], xd['v'], xd['a'], xd['w'],
                                     xd['r'], S, P, S_out=S, P_out=P)
    assert torch.equal(o1, o2) and torch.equal(S1, S) and torch.equal(P1, P)
    ref = _oracle('diag', x, None, None, [(0, 2)])[(0, 2)]
    assert rel_maxabs(o1[0, :, 2], ref[0]) <= EXACT_TOL


def test_exact_axis_aligned_keys_is_the_diagonal_kdn():
    """With one-hot keys the exact covariance stays diagonal, so the dense
    filter and the diagonal KDN filter are one filter: the two kernels agree
    on o, S and the variances, and P's off-diagonal stays exactly zero."""
    B, T, H, d = 2, 96, 2, 64
    x = synth.layer_inputs(B, T, H, d, d, 'diag', seed=12, dtype='f32')
    g = torch.Generator().manual_seed(13)
    idx = torch.randint(0, d, (B, T, H), generator=g)
    x['k'] = torch.nn.functional.one_hot(idx, d).float()
    p0 = torch.rand(B, H, d, generator=g) + 0.2
    xd = {k: v.cuda() for k, v in x.items()}
    o_e, S_e, P_e = kdn.kdn_exact_forward('diag', xd['q'], xd['k'], xd['v'], xd['a'], xd['w'],
                                          xd['r'], None, torch.diag_embed(p0).cuda())
    o_k, S_k, p_k = kdn.kdn_diag_forward(xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                                         p0=p0.cuda(), chunk=kdn.KDN_CHUNK_RECURRENT)
    assert rel_maxabs(o_e, f64(o_k)) <= EXACT_TOL
    assert rel_maxabs(S_e, f64(S_k)) <= EXACT_TOL
    assert rel_maxabs(torch.diagonal(P_e, dim1=-2, dim2=-1), f64(p_k)) <= EXACT_TOL
    off = P_e - torch.diag_embed(torch.diagonal(P_e, dim1=-2, dim2=-1))
    assert torch.count_nonzero(off).item() == 0


def test_exact_full_size_sampled_heads():
    """The benchmark shape (B8 T4096 H16, d_k = d_v = 64, bf16): sampled heads
    against the oracle over all 4096 tokens."""
    c = synth.WORKLOADS['exact_d64']
    B, T, H, d = c['B'], c['T'], c['H'], c['dk']
    x = synth.layer_inputs(B, T, H, d, d, c['variant'], seed=c['seed'], dtype=c['dtype'])
    xd = {k: v.cuda() for k, v in x.items()}
    o, S, P = kdn.kdn_exact_forward(c['variant'], xd['q'], xd['k'], xd['v'], xd['a'], xd['w'],
                                    xd['r'])
    torch.cuda.synchronize()
    ref = _oracle(c['variant'], x, None, None, [(0, 0), (3, 9), (7, 15)])
    for (b, h), (o_r, S_r, P_r) in ref.items():
        assert rel_maxabs(o[b, :, h], o_r) <= EXACT_TOL, (b, h)
        assert rel_maxabs(S[b, h], S_r) <= EXACT_TOL, (b, h)
        assert rel_maxabs(P[b, h], P_r) <= EXACT_TOL, (b, h)
