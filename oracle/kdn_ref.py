"""Token-by-token fp64 reference of the KDN layer (test infrastructure only).

Model, per (batch b, head h), from [KDN-abs] and [KDN-sum] 方法 — 输入与状态建模:
the associative memory S_t (d_v x d_k) is the latent state of a linear-Gaussian
state-space model and each token is a noisy observation of it:

    transition   S_t = a_t S_{t-1} + E_t,   every row of E_t ~ N(0, W_t)
    observation  v_t = S_t k_t + e_t,       e_t ~ N(0, r_t I_{d_v})

Every row of S sees the same key and iid noise, so all d_v rows share one
d_k x d_k covariance.  Per token the filter does, in the order the pages give
([KDN-sum] 方法 — 关键模块 steps 1-2, then 输出与差异点):

  1. predict:  mean a_t S_{t-1};  covariance a_t^2 P_{t-1} + W_t
  2. update:   Kalman gain g_t = P^-_t k_t / (k_t' P^-_t k_t + r_t) weights the
               residual write  S_t = a_t S_{t-1} + (v_t - a_t S_{t-1} k_t) g_t'
  3. project:  the exact one-step posterior precision
               Lambda = (P^-_t)^{-1} + k_t k_t' / r_t is projected back onto the
               tracked family by online mean-field VI (KL(q||p)):
                 Diagonal KDN   p_{t,i} = 1 / Lambda_ii
                 Isotropic KDN  p_t     = d_k / tr(Lambda)
               ([KDN-abs]: the diagonal variant is a mean-field VI projection
               after every step; the isotropic variant keeps one variance per
               head)
  4. query:    o_t = S_t q_t (the posterior memory is read).

With W_t = w_t I (iso) or diag(w_t) (diag) the variance recursion is, per lane,

    p^-_t = a_t^2 p_{t-1} + w_t,     p_t = 1 / (1/p^-_t + c_t / r_t)

with c_t = kappa * ||k_t||^2 (iso, kappa = 1/d_k) or c_t = k_{t,i}^2 (diag).
Written as a ratio of affine functions of p_{t-1} it is the Mobius map

    p_t = (r a^2 p_{t-1} + r w) / (c a^2 p_{t-1} + r + c w)

i.e. the 2x2 matrix [[r a^2, r w], [c a^2, r + c w]] acting projectively
([KDN-abs] states that both variance recursions are Mobius maps; [KLA]
方法论 §2 prints the same fractional-linear form for a precision).

All arithmetic is fp64 NumPy.  Inputs may be any float arrays; they are
converted to fp64 first (bf16 inputs therefore enter with their exact values).
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def _f64(x):
    return None if x is None else np.asarray(x, dtype=F64)


# ----------------------------------------------------------------------------
# Variance recurrence (the Mobius map) -- one lane-vectorised step
# ----------------------------------------------------------------------------

def variance_step(p, a, w, r, c):
    """One predict+project step of the per-lane variance.

    Returns (p_prior, p_post) with p_prior = a^2 p + w and
    p_post = 1 / (1/p_prior + c/r).  [KDN-sum] 方法 — 关键模块 steps 1 and 3.
    """
    p_prior = a * a * p + w
    p_post = 1.0 / (1.0 / p_prior + c / r)
    return p_prior, p_post


def mobius_coefficients(a, w, r, c):
    """The 2x2 homogeneous matrix of one variance step, entrywise arrays.

    Returns (alpha, beta, gamma, delta) with
    p_post = (alpha p + beta) / (gamma p + delta):
        alpha = r a^2, beta = r w, gamma = c a^2, delta = r + c w.
    All entries are >= 0 for a real, w >= 0, r > 0, c >= 0.
    """
    a, w, r, c = map(_f64, (a, w, r, c))
    return r * a * a, r * w, c * a * a, r + c * w


def variance_scan(a, w, r, c, lam0):
    """Sequential variance recursion along the last axis.

    a, w, r, c: [..., T];  lam0: [...] (the initial variance p_0).
    Returns (prior [..., T], post [..., T]).
    """
    a, w, r, c = map(_f64, (a, w, r, c))
    p = np.broadcast_to(_f64(lam0), a.shape[:-1]).copy()
    T = a.shape[-1]
    prior = np.empty(a.shape, F64)
    post = np.empty(a.shape, F64)
    for t in range(T):
        pp, p = variance_step(p, a[..., t], w[..., t], r[..., t], c[..., t])
        prior[..., t] = pp
        post[..., t] = p
    return prior, post


def mobius_apply(M, lam):
    """Projective action of 2x2 matrices M [..., 2, 2] on lam [...]."""
    return (M[..., 0, 0] * lam + M[..., 0, 1]) / (M[..., 1, 0] * lam + M[..., 1, 1])


def mobius_matrices(a, w, r, c):
    """Stack the per-step coefficients as matrices [..., T, 2, 2]."""
    al, be, ga, de = mobius_coefficients(a, w, r, c)
    M = np.empty(al.shape + (2, 2), F64)
    M[..., 0, 0] = al
    M[..., 0, 1] = be
    M[..., 1, 0] = ga
    M[..., 1, 1] = de
    return M


def mobius_prefix_tree(M):
    """Inclusive prefix compositions P_t = M_t M_{t-1} ... M_1 (later maps on
    the left) by recursive doubling over the T axis, fp64.

    M: [..., T, 2, 2].  Each combine renormalises by the largest entry, which
    leaves the projective action unchanged.  Composition of Mobius maps is
    associative, so the prefixes can be formed in log2(T) rounds ([KDN-abs];
    [KLA] 方法论 §2 gives O(T) work and O(log T) depth).
    """
    P = np.array(M, dtype=F64, copy=True)
    T = P.shape[-3]
    shift = 1
    while shift < T:
        later = P[..., shift:, :, :]
        earlier = P[..., :-shift, :, :]
        comb = later @ earlier
        scale = np.max(np.abs(comb), axis=(-2, -1), keepdims=True)
        P = P.copy()
        P[..., shift:, :, :] = comb / scale
        shift *= 2
    return P


def variance_scan_tree(a, w, r, c, lam0):
    """Posterior variances via the tree scan: p_t = P_t(lam0)."""
    P = mobius_prefix_tree(mobius_matrices(a, w, r, c))
    lam0 = np.broadcast_to(_f64(lam0), P.shape[:-3])
    return mobius_apply(P, lam0[..., None])


# ----------------------------------------------------------------------------
# Layer forward, token by token
# ----------------------------------------------------------------------------

def _prep(q, k, v, a, w, r):
    q, k, v, a, w, r = map(_f64, (q, k, v, a, w, r))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == (B, T, H, dk) and v.shape == (B, T, H, dv)
    assert a.shape == (B, T, H) and r.shape == (B, T, H)
    return q, k, v, a, w, r, B, T, H, dk, dv


def iso_forward(q, k, v, a, w, r, S0=None, p0=None, info_scale=None,
                return_aux=False):
    """Isotropic KDN forward, token by token.

    q, k: [B,T,H,d_k]; v: [B,T,H,d_v]; a, w, r: [B,T,H];
    S0: [B,H,d_v,d_k] (None -> 0); p0: [B,H] (None -> 1);
    info_scale: kappa (None or <= 0 -> 1/d_k).
    Returns o [B,T,H,d_v], S_T [B,H,d_v,d_k], p_T [B,H]; with return_aux also a
    dict of the per-token write strength beta [B,T,H] and prior/posterior
    variances [B,T,H].

    Per token ([KDN-sum] 方法 — 关键模块 1-2, [KDN-abs]):
      n = ||k||^2, p^- = a^2 p + w, beta = p^- / (p^- n + r)   (g = beta k)
      p = 1 / (1/p^- + kappa n / r)
      S = a S + (v - a S k) (beta k)'
      o = S q
    """
    q, k, v, a, w, r, B, T, H, dk, dv = _prep(q, k, v, a, w, r)
    assert w.shape == (B, T, H)
    kappa = (1.0 / dk) if (info_scale is None or info_scale <= 0) else float(info_scale)
    S = np.zeros((B, H, dv, dk), F64) if S0 is None else _f64(S0).copy()
    p = np.ones((B, H), F64) if p0 is None else _f64(p0).copy()
    o = np.empty((B, T, H, dv), F64)
    beta_all = np.empty((B, T, H), F64)
    prior_all = np.empty((B, T, H), F64)
    post_all = np.empty((B, T, H), F64)
    for t in range(T):
        kt, qt, vt = k[:, t], q[:, t], v[:, t]
        at, wt, rt = a[:, t], w[:, t], r[:, t]
        n = np.einsum('bhk,bhk->bh', kt, kt)
        p_prior, p = variance_step(p, at, wt, rt, kappa * n)
        beta = p_prior / (p_prior * n + rt)
        pred = at[:, :, None, None] * S
        resid = vt - np.einsum('bhvk,bhk->bhv', pred, kt)
        S = pred + (beta[:, :, None, None] * resid[:, :, :, None]) * kt[:, :, None, :]
        o[:, t] = np.einsum('bhvk,bhk->bhv', S, qt)
        beta_all[:, t], prior_all[:, t], post_all[:, t] = beta, p_prior, p
    if return_aux:
        return o, S, p, dict(beta=beta_all, prior=prior_all, post=post_all)
    return o, S, p


def diag_forward(q, k, v, a, w, r, S0=None, p0=None, return_aux=False):
    """Diagonal KDN forward, token by token.

    As iso_forward but w: [B,T,H,d_k] and p0 / p_T: [B,H,d_k].
    Per token and key dimension i (the mean-field VI projection of [KDN-abs]):
      p^-_i = a^2 p_i + w_i
      s = sum_i p^-_i k_i^2 + r          (innovation variance)
      g = p^- * k / s                    (Kalman gain under the diagonal prior)
      p_i = 1 / (1/p^-_i + k_i^2 / r)    (= 1 / Lambda_ii)
      S = a S + (v - a S k) g';  o = S q
    With return_aux the dict holds gain g [B,T,H,d_k], innovation s [B,T,H],
    prior / posterior variances [B,T,H,d_k].
    """
    q, k, v, a, w, r, B, T, H, dk, dv = _prep(q, k, v, a, w, r)
    assert w.shape == (B, T, H, dk)
    S = np.zeros((B, H, dv, dk), F64) if S0 is None else _f64(S0).copy()
    p = np.ones((B, H, dk), F64) if p0 is None else _f64(p0).copy()
    o = np.empty((B, T, H, dv), F64)
    aux = dict(gain=np.empty((B, T, H, dk), F64), innov=np.empty((B, T, H), F64),
               prior=np.empty((B, T, H, dk), F64), post=np.empty((B, T, H, dk), F64))
    for t in range(T):
        kt, qt, vt = k[:, t], q[:, t], v[:, t]
        at, wt, rt = a[:, t], w[:, t], r[:, t]
        p_prior, p = variance_step(p, at[..., None], wt, rt[..., None], kt * kt)
        s = np.einsum('bhk,bhk->bh', p_prior, kt * kt) + rt
        g = p_prior * kt / s[..., None]
        pred = at[:, :, None, None] * S
        resid = vt - np.einsum('bhvk,bhk->bhv', pred, kt)
        S = pred + resid[:, :, :, None] * g[:, :, None, :]
        o[:, t] = np.einsum('bhvk,bhk->bhv', S, qt)
        aux['gain'][:, t], aux['innov'][:, t] = g, s
        aux['prior'][:, t], aux['post'][:, t] = p_prior, p
    if return_aux:
        return o, S, p, aux
    return o, S, p


def decode_step(variant, q, k, v, a, w, r, S, p, info_scale=None):
    """One recurrent decode step: the layer forward for a single token.

    variant: 'iso' or 'diag'.  q, k: [B,H,d_k]; v: [B,H,d_v]; a, r: [B,H];
    w: [B,H] (iso) or [B,H,d_k] (diag); S: [B,H,d_v,d_k]; p: [B,H] or
    [B,H,d_k].  Returns (o [B,H,d_v], S_new, p_new); inputs are not modified.
    Only the fixed-size state (S, p) is carried from token to token, which is
    the constant-memory decoding [KDN-abs] names as the reason for the
    recurrent form.
    """
    fwd = iso_forward if variant == 'iso' else diag_forward
    kw = dict(info_scale=info_scale) if variant == 'iso' else {}
    e = lambda x: _f64(x)[:, None]
    o, S1, p1 = fwd(e(q), e(k), e(v), e(a), e(w), e(r), S0=S, p0=p, **kw)
    return o[:, 0], S1, p1
