"""Reverse-mode gradient of the KDN layer forward, fp64 (test infrastructure
only).

The layer is trained end to end ([KDN-sum] 实验: the layers are pretrained in
language models), so its forward has a backward pass: given the gradients of
a loss with respect to the outputs o and the final state (S_T, p_T), it
returns the gradients with respect to every input q, k, v, a, w, r, S0, p0.
It is the plain definition -- the chain rule applied to the token recurrence
that kdn_ref runs -- written as the reverse-time (adjoint) recursion a
backward kernel carries: dS and dp travel from the last token to the first.

Forward of one token (per (b, h); S is d_v x d_k, k, q in R^d_k, v in R^d_v):
  isotropic: n = k.k, p- = a^2 p + w, den = p- n + r, beta = p- / den,
             p' = 1 / (1/p- + kappa n / r), g = beta k
  diagonal:  p-_i = a^2 p_i + w_i, s = sum_i p-_i k_i^2 + r, g = p- k / s,
             p'_i = 1 / (1/p-_i + k_i^2 / r)
  both:      e = v - a S k,  S' = a S + e g^T,  o = S' q

Reverse step, with dS, dp the gradients with respect to S', p':
  dS += do q^T;  dq = S'^T do
  de = dS g;  dg = dS^T e;  da += <dS, S> - <de, S k>;  dv = de
  dk += -a S^T de;  dS_prev = a (dS - de k^T)
  then the gain and variance terms of each variant (below), and finally
  p- = a^2 p + w:  da += 2 a p dp-,  dw += dp-,  dp_prev = a^2 dp-
"""
from __future__ import annotations

import numpy as np

from oracle import kdn_ref

F64 = np.float64


def _states(variant, q, k, v, a, w, r, S0, p0, info_scale):
    """The states before every token: S_prev [T, ...], p_prev [T, ...], and
    the final ones, from the forward oracle run one token at a time."""
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dv, dk)) if S0 is None else np.array(S0, F64, copy=True)
    if variant == 'iso':
        p = np.ones((B, H)) if p0 is None else np.array(p0, F64, copy=True)
    else:
        p = np.ones((B, H, dk)) if p0 is None else np.array(p0, F64, copy=True)
    S_prev, p_prev = [], []
    for t in range(T):
        S_prev.append(S)
        p_prev.append(p)
        sl = lambda x: x[:, t:t + 1]
        if variant == 'iso':
            _, S, p = kdn_ref.iso_forward(sl(q), sl(k), sl(v), sl(a), sl(w), sl(r), S, p,
                                          info_scale=info_scale)
        else:
            _, S, p = kdn_ref.diag_forward(sl(q), sl(k), sl(v), sl(a), sl(w), sl(r), S, p)
    return S_prev, p_prev, S, p


def kdn_backward(variant, q, k, v, a, w, r, dO, S0=None, p0=None, dS_T=None, dp_T=None,
                 info_scale=None):
    """Gradients of L = <dO, o> + <dS_T, S_T> + <dp_T, p_T> with respect to
    (q, k, v, a, w, r, S0, p0), as a dict of fp64 arrays shaped like the
    inputs.  variant 'iso' or 'diag'; shapes as kdn_ref's forwards."""
    q, k, v, a, w, r, dO = (np.asarray(x, F64) for x in (q, k, v, a, w, r, dO))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    kappa = (1.0 / dk) if (info_scale is None or info_scale <= 0) else float(info_scale)
    S_prev, p_prev, S_T, p_T = _states(variant, q, k, v, a, w, r, S0, p0, info_scale)
    g_ = {n: np.zeros_like(x) for n, x in (('q', q), ('k', k), ('v', v), ('a', a), ('w', w),
                                          ('r', r))}
    dS = np.zeros((B, H, dv, dk)) if dS_T is None else np.array(dS_T, F64, copy=True)
    dp = np.zeros_like(p_T) if dp_T is None else np.array(dp_T, F64, copy=True)
    for t in range(T - 1, -1, -1):
        S, p = S_prev[t], p_prev[t]
        kt, qt, vt, do = k[:, t], q[:, t], v[:, t], dO[:, t]
        at, wt, rt = a[:, t], w[:, t], r[:, t]
        # recompute the token's forward quantities
        if variant == 'iso':
            n = np.einsum('bhk,bhk->bh', kt, kt)
            pm = at * at * p + wt
            den = pm * n + rt
            beta = pm / den
            p_new = 1.0 / (1.0 / pm + kappa * n / rt)
            g = beta[..., None] * kt
        else:
            pm = (at * at)[..., None] * p + wt
            s = np.einsum('bhk,bhk->bh', pm, kt * kt) + rt
            g = pm * kt / s[..., None]
            p_new = 1.0 / (1.0 / pm + kt * kt / rt[..., None])
        Sk = np.einsum('bhvk,bhk->bhv', S, kt)
        e = vt - at[..., None] * Sk
        S_new = at[..., None, None] * S + e[..., :, None] * g[..., None, :]
        # o = S' q
        dS = dS + do[..., :, None] * qt[..., None, :]
        g_['q'][:, t] = np.einsum('bhvk,bhv->bhk', S_new, do)
        # S' = a S + e g^T and e = v - a S k
        de = np.einsum('bhvk,bhk->bhv', dS, g)
        dg = np.einsum('bhvk,bhv->bhk', dS, e)
        da = np.einsum('bhvk,bhvk->bh', dS, S) - np.einsum('bhv,bhv->bh', de, Sk)
        g_['v'][:, t] = de
        dk = -at[..., None] * np.einsum('bhvk,bhv->bhk', S, de)
        dS = at[..., None, None] * (dS - de[..., :, None] * kt[..., None, :])
        dr = np.zeros_like(rt)
        if variant == 'iso':
            # g = beta k; beta = pm / den, den = pm n + r
            dk = dk + beta[..., None] * dg
            dbeta = np.einsum('bhk,bhk->bh', dg, kt)
            dpm = dbeta * rt / den ** 2
            dn = -dbeta * pm ** 2 / den ** 2
            dr = dr - dbeta * pm / den ** 2
            # p' = 1 / D, D = 1/pm + kappa n / r
            dD = -dp * p_new ** 2
            dpm = dpm - dD / pm ** 2
            dn = dn + dD * kappa / rt
            dr = dr - dD * kappa * n / rt ** 2
            dk = dk + 2.0 * dn[..., None] * kt
            da = da + 2.0 * at * p * dpm
            g_['w'][:, t] = dpm
        else:
            # g = pm k / s, s = sum pm k^2 + r
            dpm = dg * kt / s[..., None]
            dk = dk + dg * pm / s[..., None]
            ds = -np.einsum('bhk,bhk->bh', dg, g) / s
            dpm = dpm + ds[..., None] * kt * kt
            dk = dk + 2.0 * ds[..., None] * pm * kt
            dr = dr + ds
            # p'_i = 1 / D_i, D_i = 1/pm_i + k_i^2 / r
            dD = -dp * p_new ** 2
            dpm = dpm - dD / pm ** 2
            dk = dk + 2.0 * dD * kt / rt[..., None]
            dr = dr - np.einsum('bhk,bhk->bh', dD, kt * kt) / rt ** 2
            da = da + 2.0 * at * np.einsum('bhk,bhk->bh', p, dpm)
            g_['w'][:, t] = dpm
        g_['k'][:, t] = dk
        g_['a'][:, t] = da
        g_['r'][:, t] = dr
        dp = (at * at)[..., None] * dpm if variant == 'diag' else at * at * dpm
    g_['S0'] = dS
    g_['p0'] = dp
    return g_
