"""kdn_mobius_scan_noalloc: the scan for callers that cannot allocate device
memory at the call (their host owns all device memory through its own pool,
or hands them only input and output buffers).  Its scratch is a fixed array
inside the library, so the test checks, through the C ABI, that two calls in
a row (the second reusing what the first left in that array) both match the
workspace-taking kdn_mobius_scan, that the first case also matches the fp64
oracle directly, and that a size beyond the array's limit is refused.  This
file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from kalman_filter_linear_b200 import kdn, synth
from oracle import kdn_ref
from gpu_util import SCAN_RTOL, max_rel, f64

pytestmark = pytest.mark.gpu


def _noalloc(x, lam0, kappa, want_aux):
    N, T = x['a'].shape
    lam = torch.empty_like(x['a'])
    prior = torch.empty_like(x['a']) if want_aux else None
    gain = torch.empty_like(x['a']) if want_aux else None
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = kdn.lib().kdn_mobius_scan_noalloc(
        p(x['a']), p(x['w']), p(x['r']), p(x['n']), p(lam0), ctypes.c_float(kappa), p(lam),
        p(prior), p(gain), N, T, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == kdn.KDN_OK, kdn.lib().kdn_status_string(st)
    return lam, prior, gain


def test_noalloc_scan_matches_workspace_scan_twice_in_a_row():
    cases = [(6, 9000, 1 / 64, True), (37, 4099, 1.0, False)]
    inputs = [{k: v.cuda() for k, v in synth.scan_inputs(N, T, seed=40 + i).items()}
              for i, (N, T, _, _) in enumerate(cases)]
    lam0s = [torch.rand(N, device='cuda') + 0.1 for (N, _, _, _) in cases]
    # two no-alloc calls back to back, then the reference calls
    got = [_noalloc(x, l0, kappa, aux) for x, l0, (_, _, kappa, aux) in zip(inputs, lam0s, cases)]
    for x, l0, (N, T, kappa, aux), g in zip(inputs, lam0s, cases, got):
        ref = kdn.kdn_mobius_scan(x['a'], x['w'], x['r'], x['n'], l0, kappa,
                                  want_prior=aux, want_gain=aux)
        torch.cuda.synchronize()
        assert max_rel(g[0], ref[0].double().cpu().numpy()) <= SCAN_RTOL
        if aux:
            assert max_rel(g[1], ref[1].double().cpu().numpy()) <= SCAN_RTOL
            assert max_rel(g[2], ref[2].double().cpu().numpy()) <= SCAN_RTOL
    # the first case against the oracle itself (variances, priors, gains)
    x, l0, (N, T, kappa, _), g = inputs[0], lam0s[0], cases[0], got[0]
    a, w, r, n = (f64(x[k]) for k in 'awrn')
    prior, post = kdn_ref.variance_scan(a, w, r, kappa * n, f64(l0))
    assert max_rel(g[0], post) <= SCAN_RTOL
    assert max_rel(g[1], prior) <= SCAN_RTOL
    assert max_rel(g[2], prior / (prior * n + r)) <= SCAN_RTOL


def test_noalloc_scan_rejects_sizes_beyond_its_scratch():
    limit = kdn.KDN_SCAN_NOALLOC_MAX_TILES
    N, T = limit + 1, 5  # one tile per lane: one tile too many
    x = {k: torch.ones(N, T, device='cuda') for k in 'awrn'}
    lam = torch.empty_like(x['a'])
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = kdn.lib().kdn_mobius_scan_noalloc(p(x['a']), p(x['w']), p(x['r']), p(x['n']), None,
                                           ctypes.c_float(1.0), p(lam), None, None, N, T,
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == kdn.KDN_ERR_WORKSPACE
