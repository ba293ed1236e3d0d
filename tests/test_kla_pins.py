"""Pins of the information-form diagonal filter oracle (oracle/kla_ref.py)
against facts that do not reuse its formulas: exact Gaussian conditioning of
each scalar chain, the Diagonal KDN where the two filters must coincide, the
Mobius form and its composition, and the precision's closed-form fixed point.
"""
import numpy as np
import pytest

from oracle import kla_ref, kdn_ref

RNG = np.random.default_rng


def _inputs(rng, B, T, H, dk, dv):
    k = rng.standard_normal((B, T, H, dk))
    q = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    a = rng.uniform(0.5, 1.0, (B, T, H))
    w = rng.uniform(0.05, 0.6, (B, T, H, dk))
    r = rng.uniform(0.3, 2.0, (B, T, H))
    return q, k, v, a, w, r


def _scalar_chain_posterior(a, w, r, kk, y, m0, var0, t_end):
    """Posterior mean and variance of x_{t_end} given y_0..y_{t_end} for
    x_t = a_t x_{t-1} + N(0, w_t), y_t = k_t x_t + N(0, r_t), x_{-1} ~ N(m0,
    var0), by conditioning the joint Gaussian of (x, y)."""
    n = t_end + 1
    # x_t = prod(a_0..a_t) x_{-1} + sum_s prod(a_{s+1}..a_t) e_s: linear map
    # from (x_{-1}, e_0..e_{n-1}) to x_0..x_{n-1}
    L = np.zeros((n, n + 1))
    for t in range(n):
        L[t, 0] = np.prod(a[:t + 1])
        for s in range(t + 1):
            L[t, 1 + s] = np.prod(a[s + 1:t + 1])
    cov_z = np.diag(np.concatenate([[var0], w[:n]]))
    mean_z = np.concatenate([[m0], np.zeros(n)])
    mx = L @ mean_z
    Cxx = L @ cov_z @ L.T
    K = np.diag(kk[:n])
    my = K @ mx
    Cyy = K @ Cxx @ K.T + np.diag(r[:n])
    Cxy = Cxx @ K.T
    gain = np.linalg.solve(Cyy, Cxy.T).T
    mean = mx + gain @ (y[:n] - my)
    cov = Cxx - gain @ Cxy.T
    return mean[-1], cov[-1, -1]


def test_each_element_is_the_exact_scalar_filter():
    """Every S[j, i] is the exact posterior mean of its own scalar chain
    (observing v_j through k_i), and 1 / lam its posterior variance."""
    rng = RNG(3)
    B, T, H, dk, dv = 1, 7, 1, 3, 2
    q, k, v, a, w, r = _inputs(rng, B, T, H, dk, dv)
    S0 = rng.standard_normal((B, H, dv, dk))
    lam0 = rng.uniform(0.5, 3.0, (B, H, dk))
    o, S, lam = kla_ref.kla_forward(q, k, v, a, w, r, S0, lam0)
    for t_end in range(T):
        o_t, S_t, lam_t = kla_ref.kla_forward(q[:, :t_end + 1], k[:, :t_end + 1],
                                              v[:, :t_end + 1], a[:, :t_end + 1],
                                              w[:, :t_end + 1], r[:, :t_end + 1], S0, lam0)
        for i in range(dk):
            for j in range(dv):
                mean, var = _scalar_chain_posterior(a[0, :, 0], w[0, :, 0, i], r[0, :, 0],
                                                    k[0, :, 0, i], v[0, :, 0, j],
                                                    S0[0, 0, j, i], 1.0 / lam0[0, 0, i], t_end)
                assert S_t[0, 0, j, i] == pytest.approx(mean, rel=1e-10, abs=1e-12)
                assert 1.0 / lam_t[0, 0, i] == pytest.approx(var, rel=1e-10)
        np.testing.assert_allclose(o_t[0, -1, 0], S_t[0, 0] @ q[0, t_end, 0], rtol=1e-12)
    np.testing.assert_allclose(o[:, -1], o_t[:, -1], rtol=1e-12)


def test_single_key_dimension_is_the_diagonal_kdn():
    """With d_k = 1 there is nothing to decouple: the information-form
    diagonal filter and the Diagonal KDN are the same filter."""
    rng = RNG(5)
    q, k, v, a, w, r = _inputs(rng, 2, 30, 2, 1, 3)
    S0 = rng.standard_normal((2, 2, 3, 1))
    lam0 = rng.uniform(0.5, 2.0, (2, 2, 1))
    o, S, lam = kla_ref.kla_forward(q, k, v, a, w, r, S0, lam0)
    o_d, S_d, p_d = kdn_ref.diag_forward(q, k, v, a, w, r, S0=S0, p0=1.0 / lam0)
    np.testing.assert_allclose(o, o_d, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S, S_d, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(1.0 / lam, p_d, rtol=1e-10)


def test_axis_aligned_keys_are_the_diagonal_kdn():
    """With one-hot keys both filters are exact (the covariance stays
    diagonal), so they agree token by token."""
    rng = RNG(6)
    B, T, H, dk, dv = 1, 50, 2, 5, 3
    q, _, v, a, w, r = _inputs(rng, B, T, H, dk, dv)
    idx = rng.integers(0, dk, (B, T, H))
    k = np.eye(dk)[idx] * rng.uniform(0.4, 1.6, (B, T, H, 1))
    o, S, lam = kla_ref.kla_forward(q, k, v, a, w, r)
    o_d, S_d, p_d = kdn_ref.diag_forward(q, k, v, a, w, r)
    np.testing.assert_allclose(o, o_d, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(S, S_d, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(1.0 / lam, p_d, rtol=1e-10)


def test_general_keys_differ_from_the_diagonal_kdn():
    """With dense keys the two filters are different models (the KDN couples
    the dimensions through the shared innovation): the pin above is not
    vacuous."""
    rng = RNG(7)
    q, k, v, a, w, r = _inputs(rng, 1, 20, 1, 4, 2)
    o, _, _ = kla_ref.kla_forward(q, k, v, a, w, r)
    o_d, _, _ = kdn_ref.diag_forward(q, k, v, a, w, r)
    assert np.max(np.abs(o - o_d)) > 1e-2


def test_mobius_form_and_its_composition():
    """Steps 1-2 are the printed fractional-linear map, and composing two
    steps' 2x2 matrices gives the two-step precision (associativity, which
    the parallel scan relies on)."""
    rng = RNG(8)
    n = 200
    lam = rng.uniform(0.1, 5.0, n)
    a1, a2 = rng.uniform(0.3, 1.0, (2, n))
    w1, w2 = rng.uniform(0.01, 1.0, (2, n))
    r1, r2 = rng.uniform(0.2, 3.0, (2, n))
    k1, k2 = rng.standard_normal((2, n))
    _, one = kla_ref.precision_step(lam, a1, w1, r1, k1)
    np.testing.assert_allclose(kla_ref.mobius_precision(lam, a1, w1, r1, k1), one, rtol=1e-13)
    _, two = kla_ref.precision_step(one, a2, w2, r2, k2)

    def mat(a, w, r, k):
        c = k * k / r
        return np.array([[1 + c * w, c * a * a], [w, a * a]])

    for i in range(n):
        M = mat(a2[i], w2[i], r2[i], k2[i]) @ mat(a1[i], w1[i], r1[i], k1[i])
        assert (M[0, 0] * lam[i] + M[0, 1]) / (M[1, 0] * lam[i] + M[1, 1]) == \
            pytest.approx(two[i], rel=1e-12)


def test_constant_inputs_reach_the_fixed_point():
    """Under constant a, w, r, k the precision converges to the positive root
    of w lam^2 + (a^2 - 1 - c w) lam - c a^2 = 0 (c = k^2 / r)."""
    a, w, r, k = 0.9, 0.2, 0.5, 0.7
    c = k * k / r
    A, Bq, C = w, a * a - 1 - c * w, -c * a * a
    root = (-Bq + np.sqrt(Bq * Bq - 4 * A * C)) / (2 * A)
    lam = np.array([1.0])
    for _ in range(400):
        _, lam = kla_ref.precision_step(lam, a, w, r, np.array([k]))
    assert lam[0] == pytest.approx(root, rel=1e-12)


def test_gates_reproduce_the_mean():
    """S_t = S_{t-1} diag(f_t) + v_t u_t^T with the returned forget and write
    gates (the covariance-form reading of the information-mean update)."""
    rng = RNG(9)
    q, k, v, a, w, r = _inputs(rng, 1, 25, 2, 4, 3)
    S0 = rng.standard_normal((1, 2, 3, 4))
    lam0 = rng.uniform(0.5, 2.0, (1, 2, 4))
    o, S, lam, fg, wg = kla_ref.kla_forward(q, k, v, a, w, r, S0, lam0, return_aux=True)
    Sg = S0.copy()
    for t in range(25):
        Sg = Sg * fg[:, t][:, :, None, :] + v[:, t][..., None] * wg[:, t][:, :, None, :]
    np.testing.assert_allclose(Sg, S, rtol=1e-10, atol=1e-12)
    assert np.all(fg > 0) and np.all(fg < 1)  # a < 1 and lam^- <= lam
