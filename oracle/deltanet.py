"""Gated delta rule driven by given per-token write strengths, fp64.

Test infrastructure only.  [KDN-abs] and [KDN-sum] 核心洞察 (third point) state
that delta-rule memories are the fixed-gain special case of the KDN filter:
the gain is beta_t k_t with a per-token strength and no covariance is carried.
This module is written independently of ``kdn_ref`` so that the KDN mean
update can be checked against it: fed the strengths beta_t that Isotropic KDN
computes, it must reproduce the KDN memory exactly.

    S_t = a_t S_{t-1} (I - beta_t k_t k_t') + beta_t v_t k_t'     (gated)
    o_t = S_t q_t
With a_t = 1 this is the plain delta rule.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def gated_delta_rule(q, k, v, a, beta, S0=None):
    """q, k: [T, d_k]; v: [T, d_v]; a, beta: [T]; S0: [d_v, d_k] or None.

    Returns o [T, d_v] and S_T [d_v, d_k].
    """
    q, k, v, a, beta = (np.asarray(x, F64) for x in (q, k, v, a, beta))
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, F64, copy=True)
    eye = np.eye(dk)
    o = np.empty((T, dv))
    for t in range(T):
        erase = eye - beta[t] * np.outer(k[t], k[t])
        S = a[t] * S @ erase + beta[t] * np.outer(v[t], k[t])
        o[t] = S @ q[t]
    return o, S
