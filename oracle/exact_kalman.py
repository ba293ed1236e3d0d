"""Dense (full-covariance) Kalman filter of the KDN state-space model, fp64.

Test infrastructure only.  This is the exact, optimal recursive estimator the
pages name for the linear-Gaussian memory model ([KDN-abs]: the Kalman filter
is optimal for it; exact tracking needs the dense, state-dependent Riccati
recursion).  It is used on tiny inputs to validate ``kdn_ref``: the KDN
variants must coincide with it wherever the exact covariance stays inside the
tracked family (isotropic or diagonal), and the variance they carry must be
the mean-field projection of its one-step posterior.

Model per (b, h), every row of S independent with a shared covariance P:
    S_t = a_t S_{t-1} + E_t,  rows of E_t ~ N(0, W_t)
    v_t = S_t k_t + e_t,      e_t ~ N(0, r_t I)
Textbook covariance-form recursion per token:
    P^- = a^2 P + W;  s = k' P^- k + r;  K = P^- k / s
    S   = a S + (v - a S k) K';  P = P^- - (P^- k)(P^- k)' / s
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def exact_forward(q, k, v, a, W, r, S0, P0):
    """Run the dense filter over one (b, h) sequence.

    q, k: [T, d_k]; v: [T, d_v]; a, r: [T]; W: [T, d_k, d_k] process-noise
    covariances; S0: [d_v, d_k]; P0: [d_k, d_k].
    Returns o [T, d_v], S_all [T, d_v, d_k] (filtered means),
    P_all [T, d_k, d_k] (filtered covariances), Pprior_all [T, d_k, d_k].
    """
    q, k, v, a, W, r = (np.asarray(x, F64) for x in (q, k, v, a, W, r))
    S = np.array(S0, F64, copy=True)
    P = np.array(P0, F64, copy=True)
    T, dk = k.shape
    dv = v.shape[1]
    o = np.empty((T, dv))
    S_all = np.empty((T, dv, dk))
    P_all = np.empty((T, dk, dk))
    Pp_all = np.empty((T, dk, dk))
    for t in range(T):
        Pp = a[t] ** 2 * P + W[t]
        Pk = Pp @ k[t]
        s = k[t] @ Pk + r[t]
        gain = Pk / s
        pred = a[t] * S
        S = pred + np.outer(v[t] - pred @ k[t], gain)
        P = Pp - np.outer(Pk, Pk) / s
        P = 0.5 * (P + P.T)
        o[t] = S @ q[t]
        S_all[t], P_all[t], Pp_all[t] = S, P, Pp
    return o, S_all, P_all, Pp_all


def one_step_posterior_precision(Pprior, k, r):
    """Exact one-step posterior precision Lambda = (P^-)^{-1} + k k' / r."""
    Pprior = np.asarray(Pprior, F64)
    k = np.asarray(k, F64)
    return np.linalg.inv(Pprior) + np.outer(k, k) / float(r)
