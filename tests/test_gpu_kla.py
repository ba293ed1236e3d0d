"""The information-form diagonal filter kernel (kdn_kla_forward) against the
fp64 oracle (needs a B200).

The kernel computes in fp32 from fp32 (or exact bf16) inputs.  The gates lie
in (0, 1) and the recursion contracts, so the error stays at a few fp32
roundings per token: o and S within 1e-4 of max-abs over RMS, the precision
within 1e-5 relative.
"""
import numpy as np
import pytest
import torch

from kalman_filter_linear_b200 import kdn, synth
from oracle import kla_ref
from gpu_util import rel_maxabs, f64

pytestmark = pytest.mark.gpu

KLA_TOL = 1e-4


def _run(x, S0=None, lam0=None):
    """kdn_kla_forward: the token-recurrent kernel (the chunked engine has its
    own tests in test_gpu_kla_engine.py)."""
    xd = {k: v.cuda() for k, v in x.items()}
    return kdn.kdn_kla_forward(xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                               None if S0 is None else S0.cuda(),
                               None if lam0 is None else lam0.cuda(), recurrent=True)


@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, 'bf16'), (64, 64, 'f32'), (32, 40, 'bf16'),
                                         (128, 56, 'f32'), (64, 128, 'bf16'), (128, 8, 'f32'),
                                         (64, 16, 'bf16'), (32, 32, 'f32'), (128, 24, 'bf16')])
def test_kla_matches_oracle(dk, dv, dtype):
    """Non-zero S0 and random precisions; T = 150 spans nine 16-token chunks
    and a ragged one.  The shapes take every state-warp count the kernel has
    (8 rows of S a warp): one (d_v 8), two (16), four (24, 32), eight (40 to
    64) and sixteen (128)."""
    B, T, H = 2, 150, 2
    x = synth.layer_inputs(B, T, H, dk, dv, 'diag', seed=61 + dk + dv, dtype=dtype)
    g = torch.Generator().manual_seed(62)
    S0 = 0.05 * torch.randn(B, H, dv, dk, generator=g)
    lam0 = torch.rand(B, H, dk, generator=g) * 4 + 0.5
    o, S, lam = _run(x, S0, lam0)
    torch.cuda.synchronize()
    o_r, S_r, lam_r = kla_ref.kla_forward(*(f64(x[n]) for n in ('q', 'k', 'v', 'a', 'w', 'r')),
                                          f64(S0), f64(lam0))
    assert rel_maxabs(o, o_r) <= KLA_TOL
    assert rel_maxabs(S, S_r) <= KLA_TOL
    np.testing.assert_allclose(f64(lam), lam_r, rtol=1e-5)


def test_kla_defaults_and_in_place():
    """NULL S0 / lam0 mean zeros and ones; the outputs may be the inputs."""
    B, T, H, d = 1, 70, 3, 64
    x = synth.layer_inputs(B, T, H, d, d, 'diag', seed=64, dtype='bf16')
    o1, S1, l1 = _run(x)
    xd = {k: v.cuda() for k, v in x.items()}
    S = torch.zeros(B, H, d, d, device='cuda')
    lam = torch.ones(B, H, d, device='cuda')
    o2, _, _ = kdn.kdn_kla_forward(xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'], S, lam,
                                   S_out=S, lam_out=lam, recurrent=True)
    assert torch.equal(o1, o2) and torch.equal(S1, S) and torch.equal(l1, lam)


def test_kla_resumes_from_its_final_state():
    """Running T tokens, or T1 then T - T1 from the returned (S, lam), gives
    the same outputs and state (the handoff a decode loop relies on)."""
    B, T, H, d = 2, 96, 2, 128
    x = synth.layer_inputs(B, T, H, d, d, 'diag', seed=65, dtype='bf16')
    o, S, lam = _run(x)
    a = {k: v[:, :37].contiguous() for k, v in x.items()}
    b = {k: v[:, 37:].contiguous() for k, v in x.items()}
    oa, Sa, la = _run(a)
    ob, Sb, lb = _run(b, Sa.cpu(), la.cpu())
    assert rel_maxabs(torch.cat([oa, ob], 1), f64(o)) <= 1e-6
    assert rel_maxabs(Sb, f64(S)) <= 1e-6


def test_kla_full_size_sampled_heads():
    """The Diagonal KDN benchmark inputs (B8 T4096 H16 d128, bf16): sampled
    heads against the oracle over all 4096 tokens."""
    c = synth.WORKLOADS['diag_1p3b']
    B, T, H, d = c['B'], c['T'], c['H'], c['dk']
    x = synth.layer_inputs(B, T, H, d, d, 'diag', seed=c['seed'], dtype=c['dtype'])
    o, S, lam = _run(x)
    torch.cuda.synchronize()
    for b, h in [(0, 0), (5, 11), (7, 15)]:
        sl = {n: f64(x[n][b:b + 1, :, h:h + 1]) for n in ('q', 'k', 'v', 'a', 'w', 'r')}
        o_r, S_r, lam_r = kla_ref.kla_forward(sl['q'], sl['k'], sl['v'], sl['a'], sl['w'], sl['r'])
        assert rel_maxabs(o[b, :, h], o_r[0, :, 0]) <= KLA_TOL, (b, h)
        assert rel_maxabs(S[b, h], S_r[0, 0]) <= KLA_TOL, (b, h)
        np.testing.assert_allclose(f64(lam[b, h]), lam_r[0, 0], rtol=1e-5)
