"""Token-by-token fp64 reference of the information-form diagonal filter
(KLA), test infrastructure only.

[KLA] 方法论 describes a diagonal linear-Gaussian Kalman filter carried in
information form: a precision per state dimension, updated by a Mobius
(fractional-linear) map of the previous precision (§2, 精度递归), then the
information mean, which given the precision path is an affine recursion
(§2, 均值递归); the read-out projects the posterior mean with the query
(§1, 读出).  Its forget and write gates are ratios of precisions (§3).

Reading used here (the pages print no equation beyond the Mobius form):
the same memory model as the Diagonal KDN -- state S (d_v x d_k), decay a_t,
process noise w_t per key dimension (the OU prior's p-bar_t), value precision
1 / r_t -- but every element S[j, i] is filtered on its own, observing v_j
through k_i, so the filter stays exactly diagonal.  Per token and key
dimension i, with precision lam (all rows j share it):

  1. prior precision    lam^-_i = 1 / (a^2 / lam_i + w_i)
  2. posterior precision lam_i  = lam^-_i + k_i^2 / r
     (1 and 2 together: lam_i = ((1 + c w) lam + c a^2) / (w lam + a^2),
      c = k_i^2 / r, the Mobius map)
  3. information mean   H[j, i] = lam_i S[j, i]
                        H_t = (a lam^-_t / lam_{t-1}) H_{t-1} + (k_i / r) v_j
  4. posterior mean     S = H / lam;  read-out o_j = sum_i S[j, i] q_i

so S_t = S_{t-1} diag(f_t) + v_t u_t^T with forget gate f = a lam^- / lam and
write gate u = (k / r) / lam.  The OU discretisation that turns a rate and a
variance into (a_t, p-bar_t) is the caller's parameterisation and is not part
of this path.  All arithmetic is fp64 NumPy; inputs are converted first.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def precision_step(lam, a, w, r, k):
    """Steps 1-2 for one token: returns (lam_prior, lam_post), elementwise.
    lam, w, k: [..., d_k]; a, r broadcast against them."""
    lam_prior = 1.0 / (a * a / lam + w)
    lam_post = lam_prior + k * k / r
    return lam_prior, lam_post


def mobius_precision(lam, a, w, r, k):
    """The same step written as the Mobius map of [KLA] §2:
    lam' = (alpha lam + beta) / (gamma lam + delta)."""
    c = k * k / r
    alpha, beta, gamma, delta = 1.0 + c * w, c * a * a, w, a * a
    return (alpha * lam + beta) / (gamma * lam + delta)


def kla_forward(q, k, v, a, w, r, S0=None, lam0=None, return_aux=False):
    """Information-form diagonal filter over [B, T, H] tokens.

    q, k [B,T,H,dk]; v [B,T,H,dv]; a, r [B,T,H]; w [B,T,H,dk];
    S0 [B,H,dv,dk] (posterior mean, default 0); lam0 [B,H,dk] (precision,
    default 1).  Returns o [B,T,H,dv], S_T, lam_T (and, with return_aux, the
    forget and write gates [B,T,H,dk]).
    """
    q, k, v, a, w, r = (np.asarray(x, F64) for x in (q, k, v, a, w, r))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dv, dk)) if S0 is None else np.array(S0, F64, copy=True)
    lam = np.ones((B, H, dk)) if lam0 is None else np.array(lam0, F64, copy=True)
    Hm = S * lam[:, :, None, :]  # information mean
    o = np.empty((B, T, H, dv))
    fg = np.empty((B, T, H, dk))
    wg = np.empty((B, T, H, dk))
    for t in range(T):
        at, rt = a[:, t][..., None], r[:, t][..., None]
        lam_prior, lam_post = precision_step(lam, at, w[:, t], rt, k[:, t])
        # information mean: predicted H^- = lam^- (a S) = (a lam^- / lam) H,
        # then the observation adds (k / r) v
        Hm = (at * lam_prior / lam)[:, :, None, :] * Hm + \
            v[:, t][..., None] * (k[:, t] / rt)[:, :, None, :]
        fg[:, t] = at * lam_prior / lam_post
        wg[:, t] = (k[:, t] / rt) / lam_post
        lam = lam_post
        S = Hm / lam[:, :, None, :]
        o[:, t] = np.einsum('bhji,bhi->bhj', S, q[:, t])
    if return_aux:
        return o, S, lam, fg, wg
    return o, S, lam
