"""fp64 check of the chunkwise (UT / WY) form of the KDN memory update.

This is not a second oracle: it evaluates, in plain fp64 NumPy written here,
the per-chunk formulas the CUDA chunk engine implements, and checks that they
reproduce the oracle's token loop.  A slip in the algebra (a decay ratio off
by one token, a missing strict-lower mask, the wrong operand of the state
update) fails it.

Per chunk of C tokens that starts from the state S0, with write vectors g_t
(iso: beta_t k_t, diag: p^-_t * k_t / s_t) and in-chunk cumulative decays
gamma_t = prod_{s<=t} a_s:
    A_tj  = (gamma_t / gamma_j) k_t . g_j         j < t   (strictly lower)
    T     = (I + A)^{-1}
    Z     = V - diag(gamma) K S0'
    U     = T Z                                    (pseudo-values u_t)
    O     = diag(gamma) Q S0' + ((Q G') o D) U     D_tj = gamma_t/gamma_j, j <= t
    S_C   = gamma_C S0 + U' diag(gamma_C / gamma) G
The variance recursion crosses chunks through the 2x2 Mobius product of each
chunk; the carried value at a chunk start is that product applied to the
previous carry.
"""
import numpy as np
import pytest

from oracle import kdn_ref


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def chunk_forward(q, k, v, a, g, S0, C):
    """q, k: [T,dk]; v: [T,dv]; a: [T]; g: [T,dk] write vectors; S0: [dv,dk]."""
    T = len(a)
    S = S0.copy()
    o = np.empty((T, v.shape[1]))
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        Q, K, V, G = q[sl], k[sl], v[sl], g[sl]
        lg = np.cumsum(np.log(a[sl]))
        n = len(lg)
        ratio = np.exp(lg[:, None] - lg[None, :])
        strict = np.tril(np.ones((n, n)), -1)
        causal = np.tril(np.ones((n, n)))
        A = ratio * (K @ G.T) * strict
        Tm = np.linalg.inv(np.eye(n) + A)
        gam = np.exp(lg)
        Z = V - gam[:, None] * (K @ S.T)
        U = Tm @ Z
        o[sl] = gam[:, None] * (Q @ S.T) + (ratio * causal * (Q @ G.T)) @ U
        S = gam[-1] * S + (U * np.exp(lg[-1] - lg)[:, None]).T @ G
    return o, S


@pytest.mark.parametrize("variant,T,C", [("iso", 200, 64), ("diag", 200, 64),
                                         ("iso", 64, 64), ("diag", 37, 16), ("iso", 5, 64)])
def test_chunk_form_reproduces_token_loop(variant, T, C):
    rng = np.random.default_rng(21)
    B, H, dk, dv = 1, 2, 16, 12
    q = _unit(rng.standard_normal((B, T, H, dk)))
    k = _unit(rng.standard_normal((B, T, H, dk)))
    v = rng.standard_normal((B, T, H, dv))
    a = 1 / (1 + np.exp(-rng.normal(2, 0.5, (B, T, H))))
    r = np.log1p(np.exp(rng.normal(0, 1, (B, T, H))))
    S0 = 0.3 * rng.standard_normal((B, H, dv, dk))
    if variant == 'iso':
        w = np.log1p(np.exp(rng.normal(-2, 0.5, (B, T, H))))
        o, S, _, aux = kdn_ref.iso_forward(q, k, v, a, w, r, S0=S0, p0=np.full((B, H), 0.6),
                                           return_aux=True)
        g = aux['beta'][..., None] * k
    else:
        w = np.log1p(np.exp(rng.normal(-2, 0.5, (B, T, H, dk))))
        o, S, _, aux = kdn_ref.diag_forward(q, k, v, a, w, r, S0=S0, return_aux=True)
        g = aux['gain']
    for h in range(H):
        oc, Sc = chunk_forward(q[0, :, h], k[0, :, h], v[0, :, h], a[0, :, h], g[0, :, h],
                               S0[0, h], C)
        np.testing.assert_allclose(oc, o[0, :, h], rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(Sc, S[0, h], rtol=1e-9, atol=1e-11)


def test_chunk_carry_of_variance_products():
    """Per-chunk Mobius products, carried across chunk boundaries, give the
    sequential variances at every token."""
    rng = np.random.default_rng(22)
    T, C = 300, 64
    a = 1 / (1 + np.exp(-rng.normal(2, 0.5, T)))
    w = np.log1p(np.exp(rng.normal(-2, 0.5, T)))
    r = np.log1p(np.exp(rng.normal(0, 1, T)))
    c = rng.uniform(0.5, 1.5, T) / 128
    lam0 = 0.8
    _, post = kdn_ref.variance_scan(a, w, r, c, lam0)
    M = kdn_ref.mobius_matrices(a, w, r, c)
    carry = lam0
    out = np.empty(T)
    for c0 in range(0, T, C):
        P = np.eye(2)
        for t in range(c0, min(c0 + C, T)):
            P = M[t] @ P
            out[t] = kdn_ref.mobius_apply(P, carry)
        carry = out[min(c0 + C, T) - 1]
    np.testing.assert_allclose(out, post, rtol=1e-12)
