"""GPU parity of the chunkwise tensor-core engine against the fp64 oracle
(needs a B200).  Tolerances are the layer contract's: outputs to 2e-2 and the
final state to 1e-3 of max-abs error over the RMS; variances to 1e-5."""
import numpy as np
import pytest
import torch

from kalman_filter_linear_b200 import kdn, synth
from oracle import kdn_ref
from gpu_util import OUT_TOL, STATE_TOL, rel_maxabs, to_dev, f64

pytestmark = pytest.mark.gpu
CH = kdn.KDN_CHUNK_64


def _run(variant, x, S0=None, p0=None, chunk=CH, **kw):
    if variant == 'iso':
        return kdn.kdn_iso_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], S0, p0,
                                   chunk=chunk, **kw)
    return kdn.kdn_diag_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], S0, p0,
                                chunk=chunk, **kw)


def _ref(variant, x, S0=None, p0=None, heads=None):
    """Oracle on all heads, or on a list of (b, h) pairs (returned stacked as
    B = 1, H = len(heads))."""
    def pick(t):
        a = f64(t)
        if heads is None:
            return a
        bi = np.array([p[0] for p in heads])
        hi = np.array([p[1] for p in heads])
        return a[bi, :, hi][None].swapaxes(1, 2) if a.ndim >= 3 else a
    args = [pick(x[n]) for n in 'qkvawr']
    fwd = kdn_ref.iso_forward if variant == 'iso' else kdn_ref.diag_forward
    return fwd(*args, S0=None if S0 is None else f64(S0), p0=None if p0 is None else f64(p0))


@pytest.mark.parametrize("variant", ["iso", "diag"])
@pytest.mark.parametrize("T,dv", [(1, 128), (37, 128), (64, 128), (65, 128), (200, 64),
                                  (333, 128)])
def test_chunked_matches_oracle(variant, T, dv):
    B, H, dk = 2, 2, 128
    x = to_dev(synth.layer_inputs(B, T, H, dk, dv, variant, seed=T + dv, dtype='bf16'))
    g = torch.Generator().manual_seed(T)
    S0 = (0.05 * torch.randn(B, H, dv, dk, generator=g)).cuda()
    p0 = (torch.rand((B, H) if variant == 'iso' else (B, H, dk), generator=g) + 0.2).cuda()
    o, S, p = _run(variant, x, S0, p0)
    o_r, S_r, p_r = _ref(variant, x, S0, p0)
    eo, eS = rel_maxabs(o, o_r), rel_maxabs(S, S_r)
    assert eo <= OUT_TOL, eo
    assert eS <= STATE_TOL, eS
    np.testing.assert_allclose(f64(p), p_r, rtol=1e-5)


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_chunked_agrees_with_recurrent_path(variant):
    B, T, H, d = 1, 300, 3, 128
    x = to_dev(synth.layer_inputs(B, T, H, d, d, variant, seed=17, dtype='bf16'))
    o1, S1, p1 = _run(variant, x, chunk=CH)
    o2, S2, p2 = _run(variant, x, chunk=kdn.KDN_CHUNK_RECURRENT)
    assert rel_maxabs(o1, o2) <= OUT_TOL
    assert rel_maxabs(S1, S2) <= STATE_TOL
    torch.testing.assert_close(p1, p2, rtol=1e-5, atol=0)


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_chunked_state_handover_and_p_alias(variant):
    """[0, T) in one call equals [0, h) then [h, T) with the state handed
    over; the second call writes its final variance over its own p0."""
    B, T, H, d = 1, 260, 2, 128
    x = to_dev(synth.layer_inputs(B, T, H, d, d, variant, seed=23, dtype='bf16'))
    o, S, p = _run(variant, x)
    h = 130
    xa = {k: v[:, :h].clone() for k, v in x.items()}
    xb = {k: v[:, h:].clone() for k, v in x.items()}
    oa, Sa, pa = _run(variant, xa)
    ob, Sb, pb = _run(variant, xb, Sa, pa, S_out=Sa, p_out=pa)
    assert Sb.data_ptr() == Sa.data_ptr() and pb.data_ptr() == pa.data_ptr()
    assert rel_maxabs(torch.cat([oa, ob], 1), o) <= OUT_TOL / 4
    assert rel_maxabs(Sb, S) <= STATE_TOL
    torch.testing.assert_close(pb, p, rtol=1e-5, atol=0)


@pytest.mark.parametrize("name", ["iso_1p3b", "diag_1p3b"])
def test_full_size_sampled_heads(name):
    """The benchmark workload in the launch the benchmark times; the oracle
    follows 3 sampled heads over all 4096 tokens."""
    c = synth.WORKLOADS[name]
    x = to_dev(synth.layer_inputs(c['B'], c['T'], c['H'], c['dk'], c['dv'], c['variant'],
                                  c['seed'], c['dtype']))
    o, S, p = _run(c['variant'], x, chunk=kdn.KDN_CHUNK_AUTO)
    heads = [(0, 0), (3, 7), (7, 15)]
    o_r, S_r, p_r = _ref(c['variant'], x, heads=heads)
    for i, (bi, hi) in enumerate(heads):
        assert rel_maxabs(o[bi, :, hi], o_r[0, :, i]) <= OUT_TOL
        assert rel_maxabs(S[bi, hi], S_r[0, i]) <= STATE_TOL
        np.testing.assert_allclose(f64(p[bi, hi]), p_r[0, i], rtol=1e-4)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()


def test_long_context_diag_sampled_heads():
    """Diagonal forward at B1 T65536 H16 d128; the oracle follows 2 heads."""
    c = synth.WORKLOADS['diag_long']
    x = to_dev(synth.layer_inputs(c['B'], c['T'], c['H'], c['dk'], c['dv'], 'diag', c['seed'],
                                  c['dtype']))
    o, S, p = _run('diag', x, chunk=kdn.KDN_CHUNK_AUTO)
    heads = [(0, 0), (0, 11)]
    o_r, S_r, p_r = _ref('diag', x, heads=heads)
    for i, (bi, hi) in enumerate(heads):
        assert rel_maxabs(o[bi, :, hi], o_r[0, :, i]) <= OUT_TOL
        assert rel_maxabs(S[bi, hi], S_r[0, i]) <= STATE_TOL
        np.testing.assert_allclose(f64(p[bi, hi]), p_r[0, i], rtol=1e-4)


def test_chunked_workspace_status_ok_and_small_workspace_rejected():
    x = to_dev(synth.layer_inputs(1, 100, 2, 128, 128, 'iso', seed=5, dtype='bf16'))
    need = kdn.kdn_forward_workspace_size(kdn.KDN_ISO, 1, 100, 2, 128, 128, CH)
    ws = torch.empty(need, dtype=torch.uint8, device='cuda')
    _run('iso', x, workspace=ws)
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_OK
    small = torch.empty(need - 256 if need > 256 else 16, dtype=torch.uint8, device='cuda')
    with pytest.raises(kdn.KdnError) as e:
        _run('iso', x, workspace=small)
    assert e.value.status == kdn.KDN_ERR_WORKSPACE


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_chunked_bounded_wait_reports_timeout_and_context_survives(variant):
    """One V copy is left out: the engine's bounded wait gives up, every CTA
    takes its abort path, the workspace reports KDN_ERR_TIMEOUT, and the next
    call on the same context is correct again."""
    B, T, H, d = 1, 256, 2, 128
    x = to_dev(synth.layer_inputs(B, T, H, d, d, variant, seed=41, dtype='bf16'))
    var = kdn.KDN_ISO if variant == 'iso' else kdn.KDN_DIAG
    ws = torch.empty(kdn.kdn_forward_workspace_size(var, B, T, H, d, d, CH), dtype=torch.uint8,
                     device='cuda')
    kdn.kdn_testing_forward_skip_v_copy(var, x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], 2,
                                        ws)
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_ERR_TIMEOUT
    o, S, p = _run(variant, x, workspace=ws)
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_OK
    o_r, S_r, p_r = _ref(variant, x)
    assert rel_maxabs(o, o_r) <= OUT_TOL
    assert rel_maxabs(S, S_r) <= STATE_TOL


def _per_head_err(o, o_ref, S, S_ref):
    """Per (b, h): max-abs error over the reference's RMS, for o [B,T,H,dv]
    and S [B,H,dv,dk]; computed on the device."""
    eo = (o - o_ref).abs().amax(dim=(1, 3)) / o_ref.pow(2).mean(dim=(1, 3)).sqrt()
    eS = (S - S_ref).abs().amax(dim=(2, 3)) / S_ref.pow(2).mean(dim=(2, 3)).sqrt()
    return eo, eS


@pytest.mark.parametrize("name", ["iso_1p3b", "diag_1p3b", "diag_long"])
def test_engine_full_width_matches_recurrent_kernel(name):
    """Every head and every token of the benchmark launches: the chunked
    engine against the token-recurrent kernel (itself checked against the
    oracle), each head within the layer tolerances."""
    c = synth.WORKLOADS[name]
    x = to_dev(synth.layer_inputs(c['B'], c['T'], c['H'], c['dk'], c['dv'], c['variant'],
                                  c['seed'], c['dtype']))
    o1, S1, p1 = _run(c['variant'], x, chunk=kdn.KDN_CHUNK_AUTO)
    o2, S2, p2 = _run(c['variant'], x, chunk=kdn.KDN_CHUNK_RECURRENT)
    eo, eS = _per_head_err(o1, o2, S1, S2)
    assert float(eo.max()) <= OUT_TOL, float(eo.max())
    assert float(eS.max()) <= STATE_TOL, float(eS.max())
    ep = float(((p1 - p2).abs() / p2.abs()).max())
    assert ep <= 1e-4, ep


@pytest.mark.parametrize("variant", ["iso", "diag"])
@pytest.mark.parametrize("T,dv", [(63, 128), (129, 128), (63, 64), (129, 64)])
def test_engine_extreme_coefficients(variant, T, dv):
    """Decays of 1e-3 and exactly 1, zero process noise, observation noise
    over six decades and key norms away from 1 (the log-space decay prefix,
    the gains and the variance carry at their edges), against the oracle."""
    B, H, dk = 1, 2, 128
    x = to_dev(synth.layer_inputs_extreme(B, T, H, dk, dv, variant, seed=T + dv + 7,
                                          dtype='bf16'))
    g = torch.Generator().manual_seed(T + 1)
    S0 = (0.05 * torch.randn(B, H, dv, dk, generator=g)).cuda()
    p0 = (torch.rand((B, H) if variant == 'iso' else (B, H, dk), generator=g) + 0.2).cuda()
    o, S, p = _run(variant, x, S0, p0, chunk=kdn.KDN_CHUNK_AUTO)
    o_r, S_r, p_r = _ref(variant, x, S0, p0)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    eo, eS = rel_maxabs(o, o_r), rel_maxabs(S, S_r)
    assert eo <= OUT_TOL, eo
    assert eS <= STATE_TOL, eS
    np.testing.assert_allclose(f64(p), p_r, rtol=1e-5)


@pytest.mark.parametrize("variant", ["iso", "diag"])
@pytest.mark.parametrize("extreme", [False, True])
def test_segmented_long_sequence_matches_oracle(variant, extreme):
    """Few heads over a long sequence (B1 H2 T8192) take the segmented
    forward: eight segments of 1024 tokens run as extra heads, from the
    variances their composed Mobius maps give and the states the chained
    segment transitions give.  Against the oracle over the whole sequence,
    with a non-zero initial state and variance."""
    B, T, H, d = 1, 8192, 2, 128
    gen = synth.layer_inputs_extreme if extreme else synth.layer_inputs
    x = to_dev(gen(B, T, H, d, d, variant, seed=81 + extreme, dtype='bf16'))
    g = torch.Generator().manual_seed(82)
    S0 = (0.05 * torch.randn(B, H, d, d, generator=g)).cuda()
    p0 = (torch.rand((B, H) if variant == 'iso' else (B, H, d), generator=g) + 0.2).cuda()
    var = kdn.KDN_ISO if variant == 'iso' else kdn.KDN_DIAG
    ws = torch.empty(kdn.kdn_forward_workspace_size(var, B, T, H, d, d), dtype=torch.uint8,
                     device='cuda')
    # the segmented forward needs more than the engine's own 256-byte workspace
    assert ws.numel() > kdn.kdn_forward_workspace_size(var, B, 300, H, d, d)
    o, S, p = _run(variant, x, S0, p0, chunk=kdn.KDN_CHUNK_AUTO, workspace=ws)
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_OK
    o_r, S_r, p_r = _ref(variant, x, S0, p0)
    eo, eS = rel_maxabs(o, o_r), rel_maxabs(S, S_r)
    assert eo <= OUT_TOL, eo
    assert eS <= STATE_TOL, eS
    np.testing.assert_allclose(f64(p), p_r, rtol=1e-5)
    # the same call split at the middle with the state handed over agrees
    h = T // 2
    xa = {k: v[:, :h].contiguous() for k, v in x.items()}
    xb = {k: v[:, h:].contiguous() for k, v in x.items()}
    _, Sa, pa = _run(variant, xa, S0, p0, chunk=kdn.KDN_CHUNK_AUTO)
    ob, Sb, pb = _run(variant, xb, Sa, pa, chunk=kdn.KDN_CHUNK_AUTO)
    assert rel_maxabs(ob, o_r[:, h:]) <= OUT_TOL
    assert rel_maxabs(Sb, S_r) <= STATE_TOL
