"""GPU parity of kdn_mobius_scan against the fp64 oracle (needs a B200)."""
import numpy as np
import pytest
import torch

from kalman_filter_linear_b200 import kdn, synth
from oracle import kdn_ref
from gpu_util import SCAN_RTOL, max_rel, to_dev, f64

pytestmark = pytest.mark.gpu


def _oracle(x, kappa, lam0=None, lanes=None):
    sel = (lambda t: f64(t)) if lanes is None else (lambda t: f64(t[lanes]))
    a, w, r, n = (sel(x[k]) for k in 'awrn')
    lam0 = np.ones(a.shape[0]) if lam0 is None else sel(lam0)
    prior, post = kdn_ref.variance_scan(a, w, r, kappa * n, lam0)
    gain = prior / (prior * n + r)
    return post, prior, gain


@pytest.mark.parametrize("N,T", [(3, 1), (5, 7), (4, 2048), (3, 2049), (2, 10000), (1, 40961),
                                 (37, 4099)])
def test_scan_matches_oracle(N, T):
    x = to_dev(synth.scan_inputs(N, T, seed=N * 7 + T))
    lam0 = torch.rand(N, device='cuda') * 2 + 0.05
    lam, prior, gain, ws = kdn.kdn_mobius_scan(x['a'], x['w'], x['r'], x['n'], lam0, 1 / 64,
                                               want_prior=True, want_gain=True)
    torch.cuda.synchronize()
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_OK
    post_r, prior_r, gain_r = _oracle(x, 1 / 64, lam0)
    assert max_rel(lam, post_r) <= SCAN_RTOL
    assert max_rel(prior, prior_r) <= SCAN_RTOL
    assert max_rel(gain, gain_r) <= SCAN_RTOL


def test_scan_default_lambda0_and_info_scale_one():
    x = to_dev(synth.scan_inputs(6, 3000, seed=5))
    lam, _, _, _ = kdn.kdn_mobius_scan(x['a'], x['w'], x['r'], x['n'], None, 1.0)
    post_r, _, _ = _oracle(x, 1.0)
    assert max_rel(lam, post_r) <= SCAN_RTOL


def test_scan_extreme_coefficients_stay_finite():
    """Tiny decays, huge noise ratios and zero process noise still give
    finite variances within tolerance (renormalisation at work)."""
    N, T = 8, 5000
    g = torch.Generator().manual_seed(3)
    a = torch.rand(N, T, generator=g) * 0.999 + 1e-3
    w = torch.rand(N, T, generator=g) * 10
    w[:, ::7] = 0.0
    r = torch.exp(torch.randn(N, T, generator=g) * 3)
    n = torch.exp(torch.randn(N, T, generator=g) * 3)
    x = to_dev(dict(a=a, w=w, r=r, n=n))
    lam, _, _, _ = kdn.kdn_mobius_scan(x['a'], x['w'], x['r'], x['n'], None, 1.0)
    post_r, _, _ = _oracle(x, 1.0)
    assert torch.isfinite(lam).all()
    assert max_rel(lam, post_r) <= SCAN_RTOL


def test_scan_full_size_sampled_lanes():
    """The 4096 x 65536 workload, in the launch the benchmark times; the
    oracle checks 12 sampled lanes over all 65536 steps."""
    cfg = synth.WORKLOADS['scan']
    x = to_dev(synth.scan_inputs(cfg['N'], cfg['T'], cfg['seed']))
    lam, _, _, ws = kdn.kdn_mobius_scan(x['a'], x['w'], x['r'], x['n'], None, cfg['info_scale'])
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_OK
    lanes = torch.tensor([0, 1, 2, 63, 511, 1000, 2047, 2048, 3001, 4093, 4094, 4095])
    post_r, _, _ = _oracle(x, cfg['info_scale'], lanes=lanes)
    assert max_rel(lam[lanes.cuda()], post_r) <= SCAN_RTOL
    assert bool((lam > 0).all())


def test_scan_bounded_wait_reports_timeout_and_context_survives():
    """A tile that never publishes makes its successor's bounded look-back
    run out; the call still completes, the workspace reports a timeout, and
    the next call on the same context is correct."""
    N, T = 2, 3 * 2048
    x = to_dev(synth.scan_inputs(N, T, seed=9))
    silent = 1 * N + 0  # tile 1 of lane 0
    _, ws = kdn.kdn_testing_mobius_scan_unpublished_tile(x['a'], x['w'], x['r'], x['n'], silent)
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_ERR_TIMEOUT
    lam, _, _, ws2 = kdn.kdn_mobius_scan(x['a'], x['w'], x['r'], x['n'], None, 1.0)
    assert kdn.kdn_read_workspace_status(ws2) == kdn.KDN_OK
    post_r, _, _ = _oracle(x, 1.0)
    assert max_rel(lam, post_r) <= SCAN_RTOL


def test_scan_rejects_small_workspace_on_device():
    x = to_dev(synth.scan_inputs(2, 100, seed=1))
    ws = torch.empty(64, dtype=torch.uint8, device='cuda')
    with pytest.raises(kdn.KdnError) as e:
        kdn.kdn_mobius_scan(x['a'], x['w'], x['r'], x['n'], None, 1.0, workspace=ws)
    assert e.value.status == kdn.KDN_ERR_WORKSPACE
