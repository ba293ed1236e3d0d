"""The backward pass (kdn_backward) against the fp64 adjoint oracle
(oracle/kdn_grad.py), which is pinned by finite differences (needs a B200).

The kernel computes in fp32 from fp32 (or exact bf16) inputs; each gradient
is within 1e-4 of max-abs over its RMS."""
import numpy as np
import pytest
import torch

from kalman_filter_linear_b200 import kdn, synth
from oracle import kdn_grad
from gpu_util import rel_maxabs, f64

pytestmark = pytest.mark.gpu

GRAD_TOL = 1e-4


@pytest.mark.parametrize("variant", ["iso", "diag"])
@pytest.mark.parametrize("dk,dv,dtype", [(32, 24, 'f32'), (64, 64, 'bf16'), (32, 128, 'f32'),
                                         (128, 128, 'bf16'), (128, 40, 'f32')])
def test_backward_matches_oracle(variant, dk, dv, dtype):
    """T = 40: two whole 16-token blocks of rebuilt states and a ragged one."""
    B, T, H = 2, 40, 2
    x = synth.layer_inputs(B, T, H, dk, dv, variant, seed=71 + dk + dv, dtype=dtype)
    g = torch.Generator().manual_seed(72)
    S0 = 0.1 * torch.randn(B, H, dv, dk, generator=g)
    p0 = torch.rand((B, H) if variant == 'iso' else (B, H, dk), generator=g) + 0.2
    dO = torch.randn(B, T, H, dv, generator=g)
    dS_T = torch.randn(B, H, dv, dk, generator=g)
    dp_T = torch.randn(p0.shape, generator=g)
    xd = {k: v.cuda() for k, v in x.items()}
    got = kdn.kdn_backward(variant, xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                           dO.cuda(), S0.cuda(), p0.cuda(), dS_T.cuda(), dp_T.cuda())
    torch.cuda.synchronize()
    ref = kdn_grad.kdn_backward(variant, *(f64(x[n]) for n in ('q', 'k', 'v', 'a', 'w', 'r')),
                                f64(dO), f64(S0), f64(p0), f64(dS_T), f64(dp_T))
    for name in ('q', 'k', 'v', 'a', 'w', 'r', 'S0', 'p0'):
        assert rel_maxabs(got[name], ref[name]) <= GRAD_TOL, name


def test_backward_defaults():
    """NULL S0, p0, dS_T and dp_T mean zeros, ones, and no final-state seed."""
    B, T, H, d = 1, 30, 2, 64
    x = synth.layer_inputs(B, T, H, d, d, 'iso', seed=73, dtype='bf16')
    dO = torch.randn(B, T, H, d, generator=torch.Generator().manual_seed(74))
    xd = {k: v.cuda() for k, v in x.items()}
    got = kdn.kdn_backward('iso', xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'], dO.cuda())
    torch.cuda.synchronize()
    ref = kdn_grad.kdn_backward('iso', *(f64(x[n]) for n in ('q', 'k', 'v', 'a', 'w', 'r')),
                                f64(dO))
    for name in ref:
        assert rel_maxabs(got[name], ref[name]) <= GRAD_TOL, name


def test_backward_full_size_sampled_heads():
    """The benchmark shape (B8 T4096 H16, d_k = d_v = 64, bf16, isotropic):
    sampled heads against the oracle over all 4096 tokens."""
    c = synth.WORKLOADS['exact_d64']
    B, T, H, d = c['B'], c['T'], c['H'], c['dk']
    x = synth.layer_inputs(B, T, H, d, d, 'iso', seed=c['seed'], dtype=c['dtype'])
    dO = torch.randn(B, T, H, d, generator=torch.Generator().manual_seed(c['seed'] + 100))
    xd = {k: v.cuda() for k, v in x.items()}
    got = kdn.kdn_backward('iso', xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                           dO.cuda())
    torch.cuda.synchronize()
    for b, h in [(0, 0), (7, 15)]:
        sl = {n: f64(x[n][b:b + 1, :, h:h + 1]) for n in ('q', 'k', 'v', 'a', 'w', 'r')}
        ref = kdn_grad.kdn_backward('iso', sl['q'], sl['k'], sl['v'], sl['a'], sl['w'], sl['r'],
                                    f64(dO[b:b + 1, :, h:h + 1]))
        for name in ('q', 'k', 'v', 'a', 'w', 'r'):
            assert rel_maxabs(got[name][b, :, h], ref[name][0, :, 0]) <= GRAD_TOL, (name, b, h)
        assert rel_maxabs(got['S0'][b, h], ref['S0'][0, 0]) <= GRAD_TOL


@pytest.mark.parametrize("variant", ["iso", "diag"])
@pytest.mark.parametrize("T", [1, 16, 17])
def test_backward_block_edges_d128(variant, T):
    """Sequence lengths at the edges of the 16-token checkpoint blocks."""
    B, H, d = 1, 2, 128
    x = synth.layer_inputs(B, T, H, d, d, variant, seed=90 + T, dtype='bf16')
    g = torch.Generator().manual_seed(91)
    S0 = 0.1 * torch.randn(B, H, d, d, generator=g)
    p0 = torch.rand((B, H) if variant == 'iso' else (B, H, d), generator=g) + 0.2
    dO = torch.randn(B, T, H, d, generator=g)
    dS_T = torch.randn(B, H, d, d, generator=g)
    dp_T = torch.randn(p0.shape, generator=g)
    xd = {k: v.cuda() for k, v in x.items()}
    got = kdn.kdn_backward(variant, xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                           dO.cuda(), S0.cuda(), p0.cuda(), dS_T.cuda(), dp_T.cuda())
    torch.cuda.synchronize()
    ref = kdn_grad.kdn_backward(variant, *(f64(x[n]) for n in ('q', 'k', 'v', 'a', 'w', 'r')),
                                f64(dO), f64(S0), f64(p0), f64(dS_T), f64(dp_T))
    for name in ('q', 'k', 'v', 'a', 'w', 'r', 'S0', 'p0'):
        assert rel_maxabs(got[name], ref[name]) <= GRAD_TOL, name


@pytest.mark.parametrize("name", ["iso_1p3b", "diag_1p3b"])
def test_backward_full_size_d128_sampled_heads(name):
    """The 1.3B-layer shape (B8 T4096 H16, d_k = d_v = 128, bf16): a sampled
    head against the oracle over all 4096 tokens, every gradient."""
    c = synth.WORKLOADS[name]
    B, T, H, d, variant = c['B'], c['T'], c['H'], c['dk'], c['variant']
    x = synth.layer_inputs(B, T, H, d, d, variant, seed=c['seed'], dtype=c['dtype'])
    dO = torch.randn(B, T, H, d, generator=torch.Generator().manual_seed(c['seed'] + 100))
    xd = {k: v.cuda() for k, v in x.items()}
    got = kdn.kdn_backward(variant, xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                           dO.cuda())
    torch.cuda.synchronize()
    for b, h in [(5, 9)]:
        sl = {n: f64(x[n][b:b + 1, :, h:h + 1]) for n in ('q', 'k', 'v', 'a', 'w', 'r')}
        ref = kdn_grad.kdn_backward(variant, sl['q'], sl['k'], sl['v'], sl['a'], sl['w'],
                                    sl['r'], f64(dO[b:b + 1, :, h:h + 1]))
        for n in ('q', 'k', 'v', 'a', 'w', 'r'):
            assert rel_maxabs(got[n][b, :, h], ref[n][0, :, 0]) <= GRAD_TOL, (n, b, h)
        assert rel_maxabs(got['S0'][b, h], ref['S0'][0, 0]) <= GRAD_TOL
        assert rel_maxabs(got['p0'][b, h], ref['p0'][0, 0]) <= GRAD_TOL
