"""Pins of the backward oracle (oracle/kdn_grad.py): every gradient it
returns must equal a central finite difference of the forward oracle
(kdn_ref, separate code), for every element of every input, on tiny inputs
in the model's valid range."""
import numpy as np
import pytest

from oracle import kdn_grad, kdn_ref

RNG = np.random.default_rng


def _inputs(rng, variant, B=1, T=5, H=2, dk=3, dv=2):
    x = dict(q=rng.standard_normal((B, T, H, dk)), k=rng.standard_normal((B, T, H, dk)),
             v=rng.standard_normal((B, T, H, dv)), a=rng.uniform(0.5, 0.95, (B, T, H)),
             r=rng.uniform(0.3, 2.0, (B, T, H)))
    x['w'] = rng.uniform(0.05, 0.5, (B, T, H) if variant == 'iso' else (B, T, H, dk))
    x['S0'] = 0.5 * rng.standard_normal((B, H, dv, dk))
    x['p0'] = rng.uniform(0.2, 1.5, (B, H) if variant == 'iso' else (B, H, dk))
    return x


def _loss(variant, x, dO, dS_T, dp_T, kappa):
    if variant == 'iso':
        o, S, p = kdn_ref.iso_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'],
                                      x['S0'], x['p0'], info_scale=kappa)
    else:
        o, S, p = kdn_ref.diag_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'],
                                       x['S0'], x['p0'])
    return float(np.sum(dO * o) + np.sum(dS_T * S) + np.sum(dp_T * p))


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_adjoint_equals_finite_differences(variant):
    rng = RNG(17 if variant == 'iso' else 18)
    x = _inputs(rng, variant)
    kappa = 0.4
    o_shape = x['v'].shape
    dO = rng.standard_normal(o_shape)
    dS_T = rng.standard_normal(x['S0'].shape)
    dp_T = rng.standard_normal(x['p0'].shape)
    g = kdn_grad.kdn_backward(variant, x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], dO,
                              x['S0'], x['p0'], dS_T, dp_T,
                              info_scale=kappa if variant == 'iso' else None)
    eps = 1e-6
    for name in ('q', 'k', 'v', 'a', 'w', 'r', 'S0', 'p0'):
        fd = np.zeros_like(x[name])
        for idx in np.ndindex(*x[name].shape):
            xp = {n: t.copy() for n, t in x.items()}
            xm = {n: t.copy() for n, t in x.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            fd[idx] = (_loss(variant, xp, dO, dS_T, dp_T, kappa) -
                       _loss(variant, xm, dO, dS_T, dp_T, kappa)) / (2 * eps)
        np.testing.assert_allclose(g[name], fd, rtol=1e-6, atol=1e-8, err_msg=name)


def test_zero_output_gradient_gives_zero_input_gradients():
    """With dO, dS_T and dp_T all zero every gradient is zero (no stray
    source term)."""
    rng = RNG(19)
    x = _inputs(rng, 'diag')
    g = kdn_grad.kdn_backward('diag', x['q'], x['k'], x['v'], x['a'], x['w'], x['r'],
                              np.zeros(x['v'].shape), x['S0'], x['p0'])
    for name, val in g.items():
        assert np.all(val == 0), name


def test_output_gradient_is_linear_in_the_seed():
    """The backward is linear in (dO, dS_T, dp_T): twice the seed gives
    twice every gradient."""
    rng = RNG(20)
    x = _inputs(rng, 'iso', T=7, dk=4, dv=3)
    dO = rng.standard_normal(x['v'].shape)
    g1 = kdn_grad.kdn_backward('iso', x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], dO,
                               x['S0'], x['p0'])
    g2 = kdn_grad.kdn_backward('iso', x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], 2 * dO,
                               x['S0'], x['p0'])
    for name in g1:
        np.testing.assert_allclose(g2[name], 2 * g1[name], rtol=1e-13, atol=1e-15)
