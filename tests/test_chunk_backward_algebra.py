"""fp64 check of the chunkwise form of the KDN backward pass.

This is not another oracle.  It is the algebra a chunked (tensor-core)
backward would implement, written in plain fp64 NumPy, and checked against
the pinned adjoint oracle (oracle/kdn_grad.py).  Per chunk of C tokens from
the state S0, with write vectors g_t and cumulative log-decays lg_t:

forward (as the forward engine):
    R_tj = exp(lg_t - lg_j);  A = (R o K G') o strict;  T = (I + A)^-1
    Z = V - diag(gamma) K S0';  U = T Z;  P = (Q G') o R o causal
    O = diag(gamma) Q S0' + P U;  S_C = gamma_C S0 + U' diag(gamma_C / gamma) G
backward, given dO and dS_C (reverse-mode through the same formulas):
    dU = P' dO + diag(gamma_C / gamma) G dS_C'
    dZ = T' dU;  dA = -(T' dU Z' T') o strict
    dQ = diag(gamma) dO S0 + ((dO U') o R o causal) G
    dK = (dA o R) G - diag(gamma) dZ S0
    dG = (dA o R)' K + ((dO U') o R o causal)' Q + diag(gamma_C / gamma) U dS_C
    dV = dZ;  dS0 = gamma_C dS_C + dO' diag(gamma) Q - dZ' diag(gamma) K
    and d lg from every gamma and ratio, then d log a by a reverse cumulative sum.
The gain g depends on the token's own k, a, w, r and the variance carried in;
its terms and the variance adjoint (a reverse linear recurrence in dp) are per
token and are added after the memory part.
"""
import numpy as np
import pytest

from oracle import kdn_grad, kdn_ref


def chunk_backward_memory(q, k, v, a, g, S0, dO, dS_T, C):
    """Gradients of <dO, o> + <dS_T, S_T> for the memory recurrence with
    given write vectors g (S_t = a S + (v - a S k) g', o = S q), by chunks.
    Shapes per head: q, k, g [T, dk]; v [T, dv]; a [T]; S0, dS_T [dv, dk].
    Returns dq, dk, dv, dg, da, dS0."""
    Tn, dk = k.shape
    starts = list(range(0, Tn, C))
    # forward: the state at every chunk start
    S_starts, S = [], S0.copy()
    for c0 in starts:
        S_starts.append(S)
        sl = slice(c0, min(c0 + C, Tn))
        K, V, G = k[sl], v[sl], g[sl]
        lg = np.cumsum(np.log(a[sl]))
        n = len(lg)
        R = np.exp(lg[:, None] - lg[None, :])
        A = R * (K @ G.T) * np.tril(np.ones((n, n)), -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        gam = np.exp(lg)
        U = Tm @ (V - gam[:, None] * (K @ S.T))
        S = gam[-1] * S + (U * np.exp(lg[-1] - lg)[:, None]).T @ G
    dq, dkk, dvv, dg, dloga = (np.zeros_like(q), np.zeros_like(k), np.zeros_like(v),
                               np.zeros_like(g), np.zeros(Tn))
    dS = dS_T.copy()
    for ci in range(len(starts) - 1, -1, -1):
        c0 = starts[ci]
        sl = slice(c0, min(c0 + C, Tn))
        Q, K, V, G, dOc = q[sl], k[sl], v[sl], g[sl], dO[sl]
        S0c = S_starts[ci]
        lg = np.cumsum(np.log(a[sl]))
        n = len(lg)
        strict = np.tril(np.ones((n, n)), -1)
        causal = np.tril(np.ones((n, n)))
        R = np.exp(lg[:, None] - lg[None, :])
        M = K @ G.T
        A = R * M * strict
        Tm = np.linalg.inv(np.eye(n) + A)
        gam = np.exp(lg)
        cg = np.exp(lg[-1] - lg)  # gamma_C / gamma_j
        KS = K @ S0c.T
        Z = V - gam[:, None] * KS
        U = Tm @ Z
        QG = Q @ G.T
        P = QG * R * causal
        # backward
        dU = P.T @ dOc + (cg[:, None] * G) @ dS.T
        dP = dOc @ U.T
        dB = U @ dS                      # d (diag(cg) G)
        dZ = Tm.T @ dU
        dT = dU @ Z.T
        dA = -(Tm.T @ dT @ Tm.T) * strict
        dM = dA * R
        dQG = dP * R * causal
        dR = dA * M + dP * QG * causal
        dQc = gam[:, None] * (dOc @ S0c) + dQG @ G
        dKc = dM @ G - gam[:, None] * (dZ @ S0c)
        dGc = dM.T @ K + dQG.T @ Q + cg[:, None] * dB
        dVc = dZ
        dgam = np.einsum('tv,tv->t', dOc, Q @ S0c.T) - np.einsum('tv,tv->t', dZ, KS)
        dcg = np.einsum('jk,jk->j', dB, G)
        dgamC = np.sum(dS * S0c)
        dS_new = gam[-1] * dS + dOc.T @ (gam[:, None] * Q) - dZ.T @ (gam[:, None] * K)
        # d lg: ratios, gammas, gamma_C / gamma, gamma_C
        dlg = (dR * R).sum(1) - (dR * R).sum(0) + dgam * gam - dcg * cg
        dlg[-1] += (dcg * cg).sum() + dgamC * gam[-1]
        dloga[sl] = np.cumsum(dlg[::-1])[::-1]  # lg_t = sum_{s <= t} log a_s
        dq[sl], dkk[sl], dvv[sl], dg[sl] = dQc, dKc, dVc, dGc
        dS = dS_new
    return dq, dkk, dvv, dg, dloga / a, dS


def _memory_loss(q, k, v, a, g, S0, dO, dS_T):
    S = S0.copy()
    L = 0.0
    for t in range(len(a)):
        S = a[t] * S + np.outer(v[t] - a[t] * S @ k[t], g[t])
        L += dO[t] @ (S @ q[t])
    return L + np.sum(dS_T * S)


@pytest.mark.parametrize("T,C", [(11, 4), (8, 8), (13, 5)])
def test_chunk_backward_memory_equals_finite_differences(T, C):
    rng = np.random.default_rng(31)
    dk, dv = 3, 2
    q, k, g = (rng.standard_normal((T, dk)) for _ in range(3))
    g *= 0.3
    v = rng.standard_normal((T, dv))
    a = rng.uniform(0.5, 0.95, T)
    S0, dS_T = rng.standard_normal((dv, dk)), rng.standard_normal((dv, dk))
    dO = rng.standard_normal((T, dv))
    got = chunk_backward_memory(q, k, v, a, g, S0, dO, dS_T, C)
    args = dict(q=q, k=k, v=v, a=a, g=g, S0=S0)
    eps = 1e-6
    for name, gi in zip(('q', 'k', 'v', 'g', 'a', 'S0'), got):
        fd = np.zeros_like(args[name])
        for idx in np.ndindex(*args[name].shape):
            xp = {n: x.copy() for n, x in args.items()}
            xm = {n: x.copy() for n, x in args.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            fd[idx] = (_memory_loss(**xp, dO=dO, dS_T=dS_T) -
                       _memory_loss(**xm, dO=dO, dS_T=dS_T)) / (2 * eps)
        np.testing.assert_allclose(gi, fd, rtol=1e-6, atol=1e-8, err_msg=name)


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_chunk_backward_plus_gain_terms_is_the_oracle(variant):
    """The chunked memory backward, followed by the per-token gain and
    variance terms, gives the adjoint oracle's gradients."""
    rng = np.random.default_rng(32)
    B, T, H, dk, dv, C = 1, 23, 1, 4, 3, 8
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk)) * 0.6
    v = rng.standard_normal((B, T, H, dv))
    a = rng.uniform(0.5, 0.95, (B, T, H))
    r = rng.uniform(0.3, 2.0, (B, T, H))
    w = rng.uniform(0.05, 0.5, (B, T, H) if variant == 'iso' else (B, T, H, dk))
    S0 = 0.5 * rng.standard_normal((B, H, dv, dk))
    p0 = rng.uniform(0.2, 1.5, (B, H) if variant == 'iso' else (B, H, dk))
    dO = rng.standard_normal((B, T, H, dv))
    dS_T = rng.standard_normal((B, H, dv, dk))
    ref = kdn_grad.kdn_backward(variant, q, k, v, a, w, r, dO, S0, p0, dS_T)
    # forward quantities per token: the gains and the variance carried in
    fwd = kdn_ref.iso_forward if variant == 'iso' else kdn_ref.diag_forward
    _, _, _, aux = fwd(q, k, v, a, w, r, S0=S0, p0=p0, return_aux=True)
    kk, aa, rr, ww = k[0, :, 0], a[0, :, 0], r[0, :, 0], w[0, :, 0]
    if variant == 'iso':
        g = aux['beta'][0, :, 0, None] * kk
        p_prev = np.concatenate([[p0[0, 0]], aux['post'][0, :-1, 0]])
    else:
        g = aux['gain'][0, :, 0]
        p_prev = np.concatenate([p0[0, 0][None], aux['post'][0, :-1, 0]], 0)
    dq, dk_m, dv_, dg, da_m, dS0 = chunk_backward_memory(q[0, :, 0], kk, v[0, :, 0], aa, g,
                                                          S0[0, 0], dO[0, :, 0], dS_T[0, 0], C)
    # the gain and variance terms, token by token from the last (dp_T = 0)
    dkk, da, dw, dr = dk_m.copy(), da_m.copy(), np.zeros_like(ww), np.zeros(T)
    dp = np.zeros_like(p_prev[0])
    kappa = 1.0 / dk
    for t in range(T - 1, -1, -1):
        kt, at, rt, wt, p = kk[t], aa[t], rr[t], ww[t], p_prev[t]
        if variant == 'iso':
            n = kt @ kt
            pm = at * at * p + wt
            den = pm * n + rt
            beta = pm / den
            pn = 1.0 / (1.0 / pm + kappa * n / rt)
            dkk[t] += beta * dg[t]
            dbeta = dg[t] @ kt
            dpm = dbeta * rt / den ** 2
            dn = -dbeta * pm ** 2 / den ** 2
            dr[t] = -dbeta * pm / den ** 2
            dD = -dp * pn ** 2
            dpm -= dD / pm ** 2
            dn += dD * kappa / rt
            dr[t] -= dD * kappa * n / rt ** 2
            dkk[t] += 2.0 * dn * kt
            da[t] += 2.0 * at * p * dpm
            dw[t] = dpm
            dp = at * at * dpm
        else:
            pm = at * at * p + wt
            s = pm @ (kt * kt) + rt
            gt = pm * kt / s
            pn = 1.0 / (1.0 / pm + kt * kt / rt)
            dpm = dg[t] * kt / s
            dkk[t] += dg[t] * pm / s
            ds = -(dg[t] @ gt) / s
            dpm += ds * kt * kt
            dkk[t] += 2.0 * ds * pm * kt
            dr[t] = ds
            dD = -dp * pn ** 2
            dpm -= dD / pm ** 2
            dkk[t] += 2.0 * dD * kt / rt
            dr[t] -= (dD @ (kt * kt)) / rt ** 2
            da[t] += 2.0 * at * (p @ dpm)
            dw[t] = dpm
            dp = at * at * dpm
    for name, got in (('q', dq), ('k', dkk), ('v', dv_), ('a', da), ('w', dw), ('r', dr),
                      ('S0', dS0), ('p0', dp)):
        want = ref[name][0, :, 0] if name in 'qkvawr' else ref[name][0, 0]
        np.testing.assert_allclose(got, want, rtol=1e-8, atol=1e-10, err_msg=name)
