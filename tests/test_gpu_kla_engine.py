"""The chunked tensor-core engine of the information-form diagonal filter
(kdn_kla_forward_ws at d_k = d_v = 128, bf16 inputs) against the fp64 oracle
and, on every head, against the token-recurrent kernel (needs a B200).

Tolerances, from the engine's arithmetic: every fp32 operand of a product
(Q~, U~, the state, A) is split into bf16 hi + lo, 16 significant bits, and
products accumulate in fp32.  A CPU emulation of that plan (operands rounded
as the tensor cores see them) gives 7.8e-5 (output) and 3.1e-5 (state) of
max-abs error over RMS against fp64 on the Diagonal KDN's inputs; the bounds
below leave a factor of about six.  Dropping any lo term takes the output to
6e-3 or more, which these bounds reject.  The precision recursion runs in
fp32 per key dimension, as in the token-recurrent kernel: 1e-5 relative.
"""
import numpy as np
import pytest
import torch

from kalman_filter_linear_b200 import kdn, synth
from oracle import kla_ref
from gpu_util import rel_maxabs, f64

pytestmark = pytest.mark.gpu

O_TOL = 5e-4
S_TOL = 2e-4
LAM_RTOL = 1e-5
D = 128


def _engine(x, S0=None, lam0=None, **kw):
    xd = {k: v.cuda() for k, v in x.items()}
    return kdn.kdn_kla_forward(xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                               None if S0 is None else S0.cuda(),
                               None if lam0 is None else lam0.cuda(), **kw)


def _oracle(x, S0=None, lam0=None):
    return kla_ref.kla_forward(*(f64(x[n]) for n in ('q', 'k', 'v', 'a', 'w', 'r')),
                               None if S0 is None else f64(S0),
                               None if lam0 is None else f64(lam0))


def _check(got, ref, o_tol=O_TOL, s_tol=S_TOL):
    o, S, lam = got
    o_r, S_r, lam_r = ref
    assert rel_maxabs(o, o_r) <= o_tol
    assert rel_maxabs(S, S_r) <= s_tol
    np.testing.assert_allclose(f64(lam), lam_r, rtol=LAM_RTOL)


@pytest.mark.parametrize("T", [1, 16, 37, 64, 65, 150, 200])
def test_engine_matches_oracle(T):
    """Non-zero S0 and random precisions; T spans one token, a quarter, a
    ragged chunk, whole chunks and ragged tails."""
    B, H = 2, 3
    x = synth.layer_inputs(B, T, H, D, D, 'diag', seed=300 + T, dtype='bf16')
    g = torch.Generator().manual_seed(301)
    S0 = 0.05 * torch.randn(B, H, D, D, generator=g)
    lam0 = torch.rand(B, H, D, generator=g) * 4 + 0.5
    got = _engine(x, S0, lam0)
    torch.cuda.synchronize()
    _check(got, _oracle(x, S0, lam0))


@pytest.mark.parametrize("T", [63, 129, 300])
def test_engine_extreme_gates(T):
    """a of 1e-3 on a third of the tokens and exactly 1 on another third, w
    exactly 0 on every fifth token, r over 1e-3 to 1e3 and key norms off 1:
    the forget gates drive the running product below 2^-100 within a chunk,
    so chunks are cut into shorter pieces."""
    B, H = 1, 2
    x = synth.layer_inputs_extreme(B, T, H, D, D, 'diag', seed=310 + T, dtype='bf16')
    g = torch.Generator().manual_seed(311)
    S0 = 0.05 * torch.randn(B, H, D, D, generator=g)
    got = _engine(x, S0)
    torch.cuda.synchronize()
    _check(got, _oracle(x, S0))


def test_engine_single_token_below_the_range_floor():
    """A decay of 1e-33 makes a forget gate below 2^-100 on its own: that
    token is a piece by itself, scaled by the floor (its own term q.u does
    not depend on the scale)."""
    B, T, H = 1, 96, 2
    x = synth.layer_inputs(B, T, H, D, D, 'diag', seed=320, dtype='bf16')
    x['a'][:, 10] = 1e-33
    x['a'][:, 70, 1] = 1e-33
    g = torch.Generator().manual_seed(321)
    S0 = 0.05 * torch.randn(B, H, D, D, generator=g)
    got = _engine(x, S0)
    torch.cuda.synchronize()
    _check(got, _oracle(x, S0))


def test_engine_resumes_from_its_final_state():
    """T tokens in one call, or 37 then T - 37 from the returned (S, lam):
    the same outputs and state (chunk boundaries differ between the two)."""
    B, T, H = 2, 160, 2
    x = synth.layer_inputs(B, T, H, D, D, 'diag', seed=330, dtype='bf16')
    o, S, lam = _engine(x)
    a = {k: v[:, :37].contiguous() for k, v in x.items()}
    b = {k: v[:, 37:].contiguous() for k, v in x.items()}
    oa, Sa, la = _engine(a)
    ob, Sb, lb = _engine(b, Sa.cpu(), la.cpu())
    assert rel_maxabs(torch.cat([oa, ob], 1), f64(o)) <= O_TOL
    assert rel_maxabs(Sb, f64(S)) <= S_TOL
    np.testing.assert_allclose(f64(lb), f64(lam), rtol=LAM_RTOL)


def test_engine_in_place_and_status():
    """S_out and lam_out may be S0 and lam0; the workspace's error word reads
    KDN_OK after the call."""
    B, T, H = 1, 100, 2
    x = synth.layer_inputs(B, T, H, D, D, 'diag', seed=340, dtype='bf16')
    g = torch.Generator().manual_seed(341)
    S0 = 0.05 * torch.randn(B, H, D, D, generator=g)
    lam0 = torch.rand(B, H, D, generator=g) + 0.5
    o1, S1, l1 = _engine(x, S0, lam0)
    xd = {k: v.cuda() for k, v in x.items()}
    S = S0.cuda()
    lam = lam0.cuda()
    ws = torch.zeros(kdn.kdn_kla_workspace_size(B, T, H, D, D), dtype=torch.uint8, device='cuda')
    o2, _, _ = kdn.kdn_kla_forward(xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'], S, lam,
                                   S_out=S, lam_out=lam, workspace=ws)
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_OK
    assert torch.equal(o1, o2) and torch.equal(S1, S) and torch.equal(l1, lam)


def test_engine_full_width_matches_recurrent_kernel():
    """The benchmark inputs (Diagonal KDN, B8 T4096 H16 d128, bf16): every
    head and token of the engine against the token-recurrent kernel (itself
    checked against the oracle), and sampled heads against the oracle."""
    c = synth.WORKLOADS['diag_1p3b']
    B, T, H = c['B'], c['T'], c['H']
    x = synth.layer_inputs(B, T, H, D, D, 'diag', seed=c['seed'], dtype=c['dtype'])
    o, S, lam = _engine(x)
    o_k, S_k, lam_k = _engine(x, recurrent=True)
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(H):
            assert rel_maxabs(o[b, :, h], o_k[b, :, h]) <= O_TOL, (b, h)
            assert rel_maxabs(S[b, h], S_k[b, h]) <= S_TOL, (b, h)
    np.testing.assert_allclose(f64(lam), f64(lam_k), rtol=LAM_RTOL)
    for b, h in [(0, 0), (6, 13)]:
        sl = {n: x[n][b:b + 1, :, h:h + 1] for n in ('q', 'k', 'v', 'a', 'w', 'r')}
        o_r, S_r, lam_r = _oracle(sl)
        assert rel_maxabs(o[b, :, h], o_r[0, :, 0]) <= O_TOL, (b, h)
        assert rel_maxabs(S[b, h], S_r[0, 0]) <= S_TOL, (b, h)


def test_engine_bounded_wait_reports_timeout_and_context_survives():
    """One V copy is left out: the issuer's bounded wait gives up, every role
    of every CTA leaves through its bounded waits, the workspace reports
    KDN_ERR_TIMEOUT, and the next call on the same context is correct."""
    B, T, H = 1, 256, 2
    x = synth.layer_inputs(B, T, H, D, D, 'diag', seed=350, dtype='bf16')
    xd = {k: v.cuda() for k, v in x.items()}
    ws = torch.zeros(kdn.kdn_kla_workspace_size(B, T, H, D, D), dtype=torch.uint8, device='cuda')
    kdn.kdn_testing_kla_skip_v_copy(xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'], 2, ws)
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_ERR_TIMEOUT
    got = kdn.kdn_kla_forward(xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'], workspace=ws)
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_OK
    _check(got, _oracle(x))
