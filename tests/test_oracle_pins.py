"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test would fail for a plausible slip in the oracle: a dropped a^2 or w,
a transposed gain, the wrong KL direction in the projection, a wrong kappa, a
sign error in the residual, or an off-by-one in the predict/update order.
"""
from fractions import Fraction

import numpy as np
import pytest
from scipy.optimize import minimize

from oracle import kdn_ref, exact_kalman, deltanet

RNG = np.random.default_rng


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_layer(rng, B, T, H, dk, dv, diag=False):
    q = _unit(rng.standard_normal((B, T, H, dk)))
    k = _unit(rng.standard_normal((B, T, H, dk)))
    v = rng.standard_normal((B, T, H, dv))
    a = 1 / (1 + np.exp(-rng.normal(2, 0.5, (B, T, H))))
    wshape = (B, T, H, dk) if diag else (B, T, H)
    w = np.log1p(np.exp(rng.normal(-2, 0.5, wshape)))
    r = np.log1p(np.exp(rng.normal(0, 1, (B, T, H))))
    return q, k, v, a, w, r


# ---------------------------------------------------------------------------
# 1. The dense filter itself, against brute-force Gaussian conditioning
# ---------------------------------------------------------------------------

def _joint_conditioning(k, v_row, a, W, r, m0, P0, t_end):
    """Mean/cov of x_{t_end} given y_1..y_{t_end} by conditioning the joint
    Gaussian of the whole trajectory (no recursion)."""
    T, d = k.shape
    n_z = d * (T + 1) + T
    L0 = np.linalg.cholesky(P0)
    # x_t = mu_t + A_t z, built forward as affine maps of the noise vector z
    mu = m0.copy()
    A = np.zeros((d, n_z))
    A[:, :d] = L0
    ys_mu, ys_A = [], []
    for t in range(t_end + 1):
        Lw = np.linalg.cholesky(W[t])
        mu = a[t] * mu
        A = a[t] * A
        A[:, d * (t + 1):d * (t + 2)] += Lw
        row = np.zeros(n_z)
        row[d * (T + 1) + t] = np.sqrt(r[t])
        ys_mu.append(k[t] @ mu)
        ys_A.append(k[t] @ A + row)
    Ay = np.array(ys_A)
    my = np.array(ys_mu)
    Syy = Ay @ Ay.T
    Sxy = A @ Ay.T
    Sxx = A @ A.T
    gain = np.linalg.solve(Syy, Sxy.T).T
    mean = mu + gain @ (v_row[:t_end + 1] - my)
    cov = Sxx - gain @ Sxy.T
    return mean, cov


def test_exact_kalman_equals_joint_gaussian_conditioning():
    rng = RNG(11)
    T, d, dv = 5, 3, 2
    k = rng.standard_normal((T, d))
    q = rng.standard_normal((T, d))
    v = rng.standard_normal((T, dv))
    a = rng.uniform(0.5, 1.2, T)
    W = np.stack([np.diag(rng.uniform(0.05, 0.5, d)) for _ in range(T)])
    W[2] += 0.05 * np.ones((d, d))       # a non-diagonal process noise too
    r = rng.uniform(0.3, 2.0, T)
    S0 = rng.standard_normal((dv, d))
    X = rng.standard_normal((d, d))
    P0 = X @ X.T + 0.5 * np.eye(d)
    o, S_all, P_all, _ = exact_kalman.exact_forward(q, k, v, a, W, r, S0, P0)
    for t in range(T):
        for j in range(dv):
            mean, cov = _joint_conditioning(k, v[:, j], a, W, r, S0[j], P0, t)
            np.testing.assert_allclose(S_all[t, j], mean, rtol=1e-10, atol=1e-11)
            np.testing.assert_allclose(P_all[t], cov, rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(o[t], S_all[t] @ q[t], rtol=1e-12)


# ---------------------------------------------------------------------------
# 2. KDN coincides with the exact filter where the exact covariance stays in
#    the tracked family
# ---------------------------------------------------------------------------

def test_diag_kdn_equals_exact_for_axis_aligned_keys():
    rng = RNG(1)
    T, dk, dv = 40, 6, 4
    idx = rng.integers(0, dk, T)
    scale = rng.uniform(0.3, 1.5, T)
    k = np.zeros((T, dk))
    k[np.arange(T), idx] = scale
    q = rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    a = rng.uniform(0.6, 1.0, T)
    w = rng.uniform(0.01, 0.3, (T, dk))
    r = rng.uniform(0.2, 2.0, T)
    S0 = rng.standard_normal((dv, dk))
    p0 = rng.uniform(0.2, 1.5, dk)
    W = np.stack([np.diag(w[t]) for t in range(T)])
    o_ex, S_ex, P_ex, _ = exact_kalman.exact_forward(q, k, v, a, W, r, S0, np.diag(p0))
    o, S, p, aux = kdn_ref.diag_forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                        a[None, :, None], w[None, :, None], r[None, :, None],
                                        S0=S0[None, None], p0=p0[None, None], return_aux=True)
    for t in range(T):
        np.testing.assert_allclose(np.diag(P_ex[t]), aux['post'][0, t, 0], rtol=1e-12)
        assert np.abs(P_ex[t] - np.diag(np.diag(P_ex[t]))).max() < 1e-14
    np.testing.assert_allclose(o[0, :, 0], o_ex, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], S_ex[-1], rtol=1e-11, atol=1e-12)


def test_iso_kdn_equals_exact_for_scalar_keys():
    rng = RNG(2)
    T, dv = 50, 3
    k = rng.uniform(-1.5, 1.5, (T, 1))
    q = rng.standard_normal((T, 1))
    v = rng.standard_normal((T, dv))
    a = rng.uniform(0.5, 1.0, T)
    w = rng.uniform(0.01, 0.3, T)
    r = rng.uniform(0.2, 2.0, T)
    S0 = rng.standard_normal((dv, 1))
    p0 = 0.7
    W = w[:, None, None] * np.ones((T, 1, 1))
    o_ex, S_ex, P_ex, _ = exact_kalman.exact_forward(q, k, v, a, W, r, S0, np.array([[p0]]))
    o, S, p, aux = kdn_ref.iso_forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                       a[None, :, None], w[None, :, None], r[None, :, None],
                                       S0=S0[None, None], p0=np.array([[p0]]), return_aux=True)
    np.testing.assert_allclose(aux['post'][0, :, 0], P_ex[:, 0, 0], rtol=1e-12)
    np.testing.assert_allclose(o[0, :, 0], o_ex, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], S_ex[-1], rtol=1e-11)


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_one_step_mean_is_exact_posterior_mean(variant):
    """From a prior in the tracked family one KDN step gives the exact
    posterior mean for an arbitrary (non-aligned) key."""
    rng = RNG(3)
    dk, dv = 7, 5
    k = rng.standard_normal(dk)
    q = rng.standard_normal(dk)
    v = rng.standard_normal(dv)
    a, r = 0.8, 0.6
    S0 = rng.standard_normal((dv, dk))
    if variant == 'iso':
        w, p0 = 0.2, 0.9
        W, P0 = w * np.eye(dk), p0 * np.eye(dk)
        o, S, _ = kdn_ref.iso_forward(q[None, None, None], k[None, None, None], v[None, None, None],
                                      np.full((1, 1, 1), a), np.full((1, 1, 1), w),
                                      np.full((1, 1, 1), r), S0=S0[None, None],
                                      p0=np.full((1, 1), p0))
    else:
        w, p0 = rng.uniform(0.05, 0.4, dk), rng.uniform(0.2, 1.5, dk)
        W, P0 = np.diag(w), np.diag(p0)
        o, S, _ = kdn_ref.diag_forward(q[None, None, None], k[None, None, None], v[None, None, None],
                                       np.full((1, 1, 1), a), w[None, None, None],
                                       np.full((1, 1, 1), r), S0=S0[None, None], p0=p0[None, None])
    o_ex, S_ex, _, _ = exact_kalman.exact_forward(q[None], k[None], v[None], np.array([a]),
                                                  W[None], np.array([r]), S0, P0)
    np.testing.assert_allclose(S[0, 0], S_ex[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o[0, 0, 0], o_ex[0], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# 3. The projection is mean-field VI, KL(q || p), found numerically
# ---------------------------------------------------------------------------

def _kl_q_p(mu_q, cov_q, mu_p, prec_p):
    d = len(mu_q)
    dm = mu_p - mu_q
    _, logdet_prec = np.linalg.slogdet(prec_p)
    _, logdet_q = np.linalg.slogdet(cov_q)
    return 0.5 * (np.trace(prec_p @ cov_q) + dm @ prec_p @ dm - d - logdet_prec - logdet_q)


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_variance_projection_minimises_reverse_kl(variant):
    rng = RNG(4)
    dk = 6
    k = rng.standard_normal(dk)
    a, r = 0.9, 0.4
    if variant == 'iso':
        w, p0 = 0.1, 0.8
        Pprior = (a * a * p0 + w) * np.eye(dk)
        _, p_post = kdn_ref.variance_step(p0, a, w, r, np.dot(k, k) / dk)
    else:
        w, p0 = rng.uniform(0.05, 0.3, dk), rng.uniform(0.3, 1.2, dk)
        Pprior = np.diag(a * a * p0 + w)
        _, p_post = kdn_ref.variance_step(p0, a, w, r, k * k)
    prec = exact_kalman.one_step_posterior_precision(Pprior, k, r)
    mu = np.zeros(dk)
    if variant == 'iso':
        f = lambda x: _kl_q_p(mu, np.exp(x[0]) * np.eye(dk), mu, prec)
        res = minimize(f, x0=[0.0], method='BFGS', options=dict(gtol=1e-12))
        best = np.exp(res.x[0])
    else:
        f = lambda x: _kl_q_p(mu, np.diag(np.exp(x)), mu, prec)
        res = minimize(f, x0=np.zeros(dk), method='BFGS', options=dict(gtol=1e-12))
        best = np.exp(res.x)
    np.testing.assert_allclose(p_post, best, rtol=1e-5)
    # The other KL direction (moment matching) gives a different variance, so
    # this test tells the two readings apart.
    cov = np.linalg.inv(prec)
    mm = np.trace(cov) / dk if variant == 'iso' else np.diag(cov)
    assert np.max(np.abs(np.asarray(mm) - p_post) / p_post) > 1e-3


def test_orthonormal_sweeps_pin_information_scale():
    """a=1, w=0, unit keys sweeping an orthonormal basis at equal r: after each
    full sweep the exact covariance is isotropic again and equals Isotropic
    KDN's variance only with kappa = 1/d_k."""
    rng = RNG(5)
    dk, dv, sweeps = 5, 2, 3
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = np.concatenate([Qm.T] * sweeps)
    T = len(k)
    q = rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    a, w, r = np.ones(T), np.zeros(T), np.full(T, 0.7)
    p0 = 1.3
    _, _, P_ex, _ = exact_kalman.exact_forward(q, k, v, a, np.zeros((T, dk, dk)), r,
                                               np.zeros((dv, dk)), p0 * np.eye(dk))
    _, _, _, aux = kdn_ref.iso_forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                       a[None, :, None], w[None, :, None], r[None, :, None],
                                       p0=np.array([[p0]]), return_aux=True)
    for s in range(1, sweeps + 1):
        t = s * dk - 1
        assert np.abs(P_ex[t] - P_ex[t, 0, 0] * np.eye(dk)).max() < 1e-12
        np.testing.assert_allclose(aux['post'][0, t, 0], P_ex[t, 0, 0], rtol=1e-12)
    _, _, _, aux1 = kdn_ref.iso_forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                        a[None, :, None], w[None, :, None], r[None, :, None],
                                        p0=np.array([[p0]]), info_scale=1.0, return_aux=True)
    assert abs(aux1['post'][0, dk - 1, 0] - P_ex[dk - 1, 0, 0]) > 1e-3


def test_scalar_filter_exact_rationals():
    """d_k = d_v = 1 against the textbook scalar Kalman filter in exact
    rational arithmetic (covariance form, written here independently)."""
    vals = dict(a=[Fraction(9, 10), Fraction(3, 4), Fraction(1, 1), Fraction(1, 2)],
                w=[Fraction(1, 10), Fraction(1, 5), Fraction(0), Fraction(1, 3)],
                r=[Fraction(1, 2), Fraction(2, 1), Fraction(3, 4), Fraction(1, 7)],
                k=[Fraction(1, 1), Fraction(-1, 2), Fraction(3, 2), Fraction(2, 3)],
                v=[Fraction(1, 3), Fraction(-2, 1), Fraction(5, 4), Fraction(1, 2)],
                q=[Fraction(1, 1), Fraction(2, 1), Fraction(-1, 3), Fraction(1, 5)])
    m, P = Fraction(1, 4), Fraction(1, 1)
    outs, Ps = [], []
    for t in range(4):
        a, w, r, h, y, qq = (vals[x][t] for x in 'awrkvq')
        Pp = a * a * P + w
        mp = a * m
        K = Pp * h / (h * h * Pp + r)
        m = mp + K * (y - h * mp)
        P = (1 - K * h) * Pp
        outs.append(m * qq)
        Ps.append(P)
    arr = lambda x: np.array([float(f) for f in vals[x]])[None, :, None, None]
    o, S, p, aux = kdn_ref.iso_forward(arr('q'), arr('k'), arr('v'), arr('a')[..., 0],
                                       arr('w')[..., 0], arr('r')[..., 0],
                                       S0=np.full((1, 1, 1, 1), 0.25), p0=np.ones((1, 1)),
                                       return_aux=True)
    np.testing.assert_allclose(o[0, :, 0, 0], [float(x) for x in outs], rtol=1e-14)
    np.testing.assert_allclose(aux['post'][0, :, 0], [float(x) for x in Ps], rtol=1e-14)


# ---------------------------------------------------------------------------
# 4. Closed forms of the variance recursion
# ---------------------------------------------------------------------------

def test_static_state_closed_form():
    rng = RNG(6)
    B, T, H, dk, dv = 2, 30, 3, 8, 4
    q, k, v, a, w, r = _rand_layer(rng, B, T, H, dk, dv)
    k = k * rng.uniform(0.5, 1.5, (B, T, H, 1))
    a[:] = 1.0
    w[:] = 0.0
    p0 = rng.uniform(0.5, 2.0, (B, H))
    _, _, pT = kdn_ref.iso_forward(q, k, v, a, w, r, p0=p0)
    n = (k * k).sum(-1)
    np.testing.assert_allclose(1 / pT, 1 / p0 + (n / r).sum(1) / dk, rtol=1e-12)
    wd = np.zeros((B, T, H, dk))
    p0d = rng.uniform(0.5, 2.0, (B, H, dk))
    _, _, pTd = kdn_ref.diag_forward(q, k, v, a, wd, r, p0=p0d)
    np.testing.assert_allclose(1 / pTd, 1 / p0d + (k * k / r[..., None]).sum(1), rtol=1e-12)


def test_constant_coefficients_reach_fixed_point():
    a, w, r, c = 0.9, 0.05, 0.7, 0.8
    al, be, ga, de = kdn_ref.mobius_coefficients(a, w, r, c)
    lam_star = ((al - de) + np.sqrt((al - de) ** 2 + 4 * be * ga)) / (2 * ga)
    T = 400
    ones = np.ones((3, T))
    _, post = kdn_ref.variance_scan(a * ones, w * ones, r * ones, c * ones,
                                    np.array([0.01, 1.0, 50.0]))
    np.testing.assert_allclose(post[:, -1], lam_star, rtol=1e-12)
    # the fixed point solves p = 1/(1/(a^2 p + w) + c/r) directly
    pp = a * a * lam_star + w
    np.testing.assert_allclose(1 / (1 / pp + c / r), lam_star, rtol=1e-13)


# ---------------------------------------------------------------------------
# 5. Mobius algebra
# ---------------------------------------------------------------------------

def test_mobius_matrix_reproduces_step_and_is_positive():
    rng = RNG(7)
    a = rng.uniform(0.01, 1.0, 1000)
    w = rng.uniform(0.0, 2.0, 1000)
    r = rng.uniform(0.01, 5.0, 1000)
    c = rng.uniform(0.0, 3.0, 1000)
    p = rng.uniform(1e-3, 10.0, 1000)
    M = kdn_ref.mobius_matrices(a, w, r, c)
    assert (M >= 0).all()
    np.testing.assert_allclose(kdn_ref.mobius_apply(M, p), kdn_ref.variance_step(p, a, w, r, c)[1],
                               rtol=1e-13)


def test_mobius_composition_is_associative():
    rng = RNG(8)
    A, Bm, C = (rng.uniform(0.01, 3.0, (500, 2, 2)) for _ in range(3))
    lam = rng.uniform(0.01, 5.0, 500)
    lhs = (A @ Bm) @ C
    rhs = A @ (Bm @ C)
    np.testing.assert_allclose(kdn_ref.mobius_apply(lhs, lam), kdn_ref.mobius_apply(rhs, lam),
                               rtol=1e-13)
    np.testing.assert_allclose(kdn_ref.mobius_apply(A @ Bm, lam),
                               kdn_ref.mobius_apply(A, kdn_ref.mobius_apply(Bm, lam)), rtol=1e-13)


def test_tree_scan_equals_sequential_recursion():
    rng = RNG(9)
    N, T = 6, 1537
    a = 1 / (1 + np.exp(-rng.normal(2, 0.5, (N, T))))
    w = np.log1p(np.exp(rng.normal(-2, 0.5, (N, T))))
    r = np.log1p(np.exp(rng.normal(0, 1, (N, T))))
    c = rng.uniform(0.5, 1.5, (N, T)) / 64
    lam0 = rng.uniform(0.1, 3.0, N)
    _, post = kdn_ref.variance_scan(a, w, r, c, lam0)
    tree = kdn_ref.variance_scan_tree(a, w, r, c, lam0)
    np.testing.assert_allclose(tree, post, rtol=1e-12)


# ---------------------------------------------------------------------------
# 6. The memory update is the gated delta rule with the Kalman strength
# ---------------------------------------------------------------------------

def test_iso_memory_is_gated_delta_rule_with_kalman_strength():
    rng = RNG(10)
    B, T, H, dk, dv = 1, 60, 2, 8, 5
    q, k, v, a, w, r = _rand_layer(rng, B, T, H, dk, dv)
    k = k * rng.uniform(0.6, 1.4, (B, T, H, 1))
    S0 = rng.standard_normal((B, H, dv, dk))
    o, S, _, aux = kdn_ref.iso_forward(q, k, v, a, w, r, S0=S0, return_aux=True)
    for h in range(H):
        o_d, S_d = deltanet.gated_delta_rule(q[0, :, h], k[0, :, h], v[0, :, h], a[0, :, h],
                                             aux['beta'][0, :, h], S0[0, h])
        np.testing.assert_allclose(o[0, :, h], o_d, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(S[0, h], S_d, rtol=1e-11, atol=1e-12)
    # with a = 1 it is the plain delta rule: S k moves toward v by beta
    p_prior = aux['prior']
    n = (k * k).sum(-1)
    np.testing.assert_allclose(aux['beta'], p_prior / (p_prior * n + r), rtol=1e-13)


# ---------------------------------------------------------------------------
# 7. Invariants
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_variance_invariants_and_residual_shrink(variant):
    rng = RNG(12)
    B, T, H, dk, dv = 2, 80, 2, 8, 4
    diag = variant == 'diag'
    q, k, v, a, w, r = _rand_layer(rng, B, T, H, dk, dv, diag)
    fwd = kdn_ref.diag_forward if diag else kdn_ref.iso_forward
    _, _, _, aux = fwd(q, k, v, a, w, r, return_aux=True)
    assert (aux['post'] > 0).all()
    assert (aux['post'] <= aux['prior'] * (1 + 1e-15)).all()
    assert (aux['prior'] >= w * (1 - 1e-15)).all()
    # residual after the update shrinks by r / (innovation variance)
    S0 = rng.standard_normal((B, H, dv, dk))
    t = 17
    _, S_prev, _ = fwd(q[:, :t], k[:, :t], v[:, :t], a[:, :t], w[:, :t], r[:, :t], S0=S0)
    _, S_t, _, aux = fwd(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1], a[:, :t + 1],
                         w[:, :t + 1], r[:, :t + 1], S0=S0, return_aux=True)
    kt, vt, at, rt = k[:, t], v[:, t], a[:, t], r[:, t]
    pre = vt - at[..., None] * np.einsum('bhvk,bhk->bhv', S_prev, kt)
    post = vt - np.einsum('bhvk,bhk->bhv', S_t, kt)
    if diag:
        s = aux['innov'][:, t]
    else:
        s = aux['prior'][:, t] * (kt * kt).sum(-1) + rt
    np.testing.assert_allclose(post, pre * (rt / s)[..., None], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_rows_are_equivariant_and_split_resumes(variant):
    rng = RNG(13)
    B, T, H, dk, dv = 1, 64, 2, 6, 5
    diag = variant == 'diag'
    q, k, v, a, w, r = _rand_layer(rng, B, T, H, dk, dv, diag)
    fwd = kdn_ref.diag_forward if diag else kdn_ref.iso_forward
    S0 = rng.standard_normal((B, H, dv, dk))
    o, S, p = fwd(q, k, v, a, w, r, S0=S0)
    perm = rng.permutation(dv)
    o2, S2, p2 = fwd(q, k, v[..., perm], a, w, r, S0=S0[:, :, perm])
    np.testing.assert_allclose(o2, o[..., perm], rtol=1e-12)
    np.testing.assert_allclose(S2, S[:, :, perm], rtol=1e-12)
    h = 27
    oa, Sa, pa = fwd(q[:, :h], k[:, :h], v[:, :h], a[:, :h], w[:, :h], r[:, :h], S0=S0)
    ob, Sb, pb = fwd(q[:, h:], k[:, h:], v[:, h:], a[:, h:], w[:, h:], r[:, h:], S0=Sa, p0=pa)
    np.testing.assert_allclose(np.concatenate([oa, ob], 1), o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(Sb, S, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(pb, p, rtol=1e-13)


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_decode_steps_reproduce_forward(variant):
    rng = RNG(14)
    B, T, H, dk, dv = 2, 9, 3, 4, 3
    diag = variant == 'diag'
    q, k, v, a, w, r = _rand_layer(rng, B, T, H, dk, dv, diag)
    fwd = kdn_ref.diag_forward if diag else kdn_ref.iso_forward
    S = rng.standard_normal((B, H, dv, dk))
    p = rng.uniform(0.1, 1.0, (B, H, dk) if diag else (B, H))
    o, S_T, p_T = fwd(q, k, v, a, w, r, S0=S, p0=p)
    for t in range(T):
        ot, S, p = kdn_ref.decode_step(variant, q[:, t], k[:, t], v[:, t], a[:, t], w[:, t],
                                       r[:, t], S, p)
        np.testing.assert_allclose(ot, o[:, t], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S, S_T, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(p, p_T, rtol=1e-13)
