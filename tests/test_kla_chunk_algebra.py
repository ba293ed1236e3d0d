"""fp64 check of the chunkwise form of the information-form diagonal filter
(KLA), the algebra a tensor-core KLA engine would implement.

Within a chunk of C tokens from the state S0, with per-dimension cumulative
log forget gates b_t = sum_{s<=t} log f_s (relative to the chunk start):
    S_t = S0 diag(e^{b_t}) + sum_{s<=t} v_s (u_s o e^{b_t - b_s})'
so, with Qt = Q o e^{b} and Ut = U o e^{-b}:
    A   = (Qt Ut') o causal
    O   = Qt S0' + A V
    S_C = S0 diag(e^{b_C}) + V' (U o e^{b_C - b})
Qt and Ut carry e^{+-b}: over a chunk of C tokens |b| grows by up to
C |log f_min| per dimension, so the chunk length bounds the exponent range
(checked below for fp32 at C = 16 with forget gates down to 1e-2).
"""
import numpy as np
import pytest

from oracle import kla_ref


def kla_chunk_forward(q, k, v, a, w, r, C, S0=None, lam0=None):
    """One head: q, k, w [T, dk]; v [T, dv]; a, r [T].  The gates come from
    the oracle's own recursion (returned with return_aux); the memory runs
    by chunks."""
    T, dk = k.shape
    dv = v.shape[1]
    _, _, _, f, u = kla_ref.kla_forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                         a[None, :, None], w[None, :, None], r[None, :, None],
                                         None if S0 is None else S0[None, None],
                                         None if lam0 is None else lam0[None, None],
                                         return_aux=True)
    f, u = f[0, :, 0], u[0, :, 0]
    S = np.zeros((dv, dk)) if S0 is None else S0.copy()
    o = np.empty((T, dv))
    max_exp = 0.0
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        Q, U, V = q[sl], u[sl], v[sl]
        b = np.cumsum(np.log(f[sl]), axis=0)           # [n, dk], <= 0
        n = len(b)
        max_exp = max(max_exp, float(np.max(-b)))
        Qt = Q * np.exp(b)
        Ut = U * np.exp(-b)
        A = (Qt @ Ut.T) * np.tril(np.ones((n, n)))
        o[sl] = Qt @ S.T + A @ V
        S = S * np.exp(b[-1])[None, :] + V.T @ (U * np.exp(b[-1] - b))
    return o, S, max_exp


@pytest.mark.parametrize("T,C", [(50, 16), (64, 16), (37, 8), (20, 64)])
def test_kla_chunk_form_reproduces_the_token_loop(T, C):
    rng = np.random.default_rng(41)
    dk, dv = 6, 4
    q, k = rng.standard_normal((T, dk)), rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    a = rng.uniform(0.5, 0.98, T)
    w = rng.uniform(0.05, 0.5, (T, dk))
    r = rng.uniform(0.3, 2.0, T)
    S0 = rng.standard_normal((dv, dk))
    lam0 = rng.uniform(0.5, 3.0, dk)
    o_c, S_c, _ = kla_chunk_forward(q, k, v, a, w, r, C, S0, lam0)
    o, S, _ = kla_ref.kla_forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                  a[None, :, None], w[None, :, None], r[None, :, None],
                                  S0[None, None], lam0[None, None])
    np.testing.assert_allclose(o_c, o[0, :, 0], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(S_c, S[0, 0], rtol=1e-9, atol=1e-11)


def test_kla_chunk_exponents_fit_fp32_at_chunk_16():
    """Forget gates down to about 1e-2 (small decay, precise observations)
    keep e^{-b} within fp32 range over 16 tokens, and the chunk form still
    reproduces the loop."""
    rng = np.random.default_rng(42)
    T, dk, dv = 48, 5, 3
    q, v = rng.standard_normal((T, dk)), rng.standard_normal((T, dv))
    k = 3.0 * rng.standard_normal((T, dk))        # strong keys: k^2 / r large
    a = rng.uniform(0.2, 0.5, T)                  # fast decay
    w = rng.uniform(0.01, 0.05, (T, dk))
    r = rng.uniform(0.05, 0.2, T)                 # precise observations
    o_c, S_c, max_exp = kla_chunk_forward(q, k, v, a, w, r, 16)
    _, _, _, f, _ = kla_ref.kla_forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                        a[None, :, None], w[None, :, None], r[None, :, None],
                                        return_aux=True)
    assert f.min() < 2e-2                         # the gates do get small
    assert max_exp < np.log(np.finfo(np.float32).max)
    o, S, _ = kla_ref.kla_forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                  a[None, :, None], w[None, :, None], r[None, :, None])
    np.testing.assert_allclose(o_c, o[0, :, 0], rtol=1e-7, atol=1e-9)


def kla_piece_forward(q, k, v, a, w, r, C=64, floor=2.0 ** -100):
    """The form the tensor-core engine computes, in fp64: chunks of C tokens
    cut into pieces so that the running product G of the forget gates from a
    piece's start (inclusive) stays >= floor; per piece, with Q~ = Q . G and
    U~ = U / G (rows = tokens),
        o_t   = S_start Q~_t + sum_{s <= t} (Q~_t . U~_s) v_s
        S_end = (S_start + V^T U~) diag(G_L)
    A token whose own gate is below the floor is a piece of its own, scaled by
    the floor.  Returns o, S_T and the number of pieces."""
    T, dk = k.shape
    dv = v.shape[1]
    _, _, _, f, u = kla_ref.kla_forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                        a[None, :, None], w[None, :, None], r[None, :, None],
                                        return_aux=True)
    f, u = f[0, :, 0], u[0, :, 0]
    S = np.zeros((dv, dk))
    o = np.empty((T, dv))
    pieces = 0

    def run_piece(lo, hi, G):
        nonlocal S, pieces
        Qt, Ut = q[lo:hi] * G, u[lo:hi] / G
        A = np.tril(Qt @ Ut.T)
        o[lo:hi] = Qt @ S.T + A @ v[lo:hi]
        S = (S + v[lo:hi].T @ Ut) * G[-1][None, :]
        pieces += 1

    for c0 in range(0, T, C):
        c1 = min(c0 + C, T)
        start, G = c0, []
        g = np.ones(dk)
        for t in range(c0, c1):
            gt = g * f[t]
            if np.any(gt < floor):
                if t > start:
                    run_piece(start, t, np.array(G))
                start, G = t, []
                gt = np.maximum(f[t], floor)
            g = gt
            G.append(g)
        run_piece(start, c1, np.array(G))
    return o, S, pieces


@pytest.mark.parametrize("case", ["plain", "strong", "floor"])
def test_kla_piece_form_reproduces_the_token_loop(case):
    """The engine's piece form against the oracle's token loop: plain gates
    (one piece per chunk), gates that multiply below 2^-100 within a chunk
    (cuts), and a decay of 1e-40 that puts one gate below the floor on its
    own (a single-token piece scaled by the floor: the result moves by at
    most 2^-100 of the state)."""
    rng = np.random.default_rng(51)
    T, dk, dv = 150, 6, 4
    q, k = rng.standard_normal((T, dk)), rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    a = rng.uniform(0.6, 0.98, T)
    w = rng.uniform(0.05, 0.5, (T, dk))
    r = rng.uniform(0.3, 2.0, T)
    if case == "strong":
        k = 3.0 * k
        a = rng.uniform(1e-3, 2e-2, T)
        r = rng.uniform(0.05, 0.2, T)
    if case == "floor":
        a[70] = 1e-40
    o_p, S_p, pieces = kla_piece_forward(q, k, v, a, w, r)
    o, S, _ = kla_ref.kla_forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                  a[None, :, None], w[None, :, None], r[None, :, None])
    chunks = -(-T // 64)
    if case == "plain":
        assert pieces == chunks
    else:
        assert pieces > chunks
    np.testing.assert_allclose(o_p, o[0, :, 0], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(S_p, S[0, 0], rtol=1e-9, atol=1e-11)
