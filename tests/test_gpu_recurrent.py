"""GPU parity of the recurrent forward path and of kdn_decode_step against
the fp64 oracle (needs a B200)."""
import json
import os

import numpy as np
import pytest
import torch

from kalman_filter_linear_b200 import kdn, synth
from oracle import kdn_ref
from gpu_util import OUT_TOL, STATE_TOL, rel_maxabs, to_dev, f64

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
REC = kdn.KDN_CHUNK_RECURRENT


def _run(variant, x, S0=None, p0=None, chunk=REC, kappa=0.0):
    if variant == 'iso':
        return kdn.kdn_iso_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], S0, p0,
                                   info_scale=kappa, chunk=chunk)
    return kdn.kdn_diag_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], S0, p0,
                                chunk=chunk)


def _ref(variant, x, S0=None, p0=None, kappa=None):
    args = [f64(x[n]) for n in 'qkvawr']
    S0 = None if S0 is None else f64(S0)
    p0 = None if p0 is None else f64(p0)
    if variant == 'iso':
        return kdn_ref.iso_forward(*args, S0=S0, p0=p0, info_scale=kappa)
    return kdn_ref.diag_forward(*args, S0=S0, p0=p0)


def test_iso_small_workload_matches_golden_and_oracle():
    cfg = synth.WORKLOADS['iso_small']
    x = to_dev(synth.layer_inputs(cfg['B'], cfg['T'], cfg['H'], cfg['dk'], cfg['dv'], 'iso',
                                  cfg['seed'], cfg['dtype']))
    o, S, p = _run('iso', x, chunk=kdn.KDN_CHUNK_AUTO)
    o_r, S_r, p_r = _ref('iso', x)
    assert rel_maxabs(o, o_r) <= 1e-3   # fp32 inputs: aim well inside the 2e-2 bound
    assert rel_maxabs(S, S_r) <= STATE_TOL
    np.testing.assert_allclose(f64(p), p_r, rtol=1e-5)
    with open(os.path.join(HERE, 'golden', 'iso_small.json')) as f:
        gold = json.load(f)
    oc = f64(o)
    got = np.array([oc[tuple(i)] for i in gold['o_index']])
    assert np.max(np.abs(got - np.array(gold['o_value']))) / gold['o_rms'] <= 1e-3


@pytest.mark.parametrize("variant", ["iso", "diag"])
@pytest.mark.parametrize("dtype,dk,dv,T", [("bf16", 128, 128, 67), ("bf16", 64, 48, 33),
                                           ("f32", 32, 128, 19), ("f32", 128, 7, 5),
                                           ("bf16", 128, 100, 1)])
def test_recurrent_matches_oracle(variant, dtype, dk, dv, T):
    B, H = 2, 3
    x = to_dev(synth.layer_inputs(B, T, H, dk, dv, variant, seed=dk + dv + T, dtype=dtype))
    g = torch.Generator().manual_seed(T)
    S0 = (0.1 * torch.randn(B, H, dv, dk, generator=g)).cuda()
    p0 = (torch.rand((B, H) if variant == 'iso' else (B, H, dk), generator=g) + 0.1).cuda()
    o, S, p = _run(variant, x, S0, p0)
    o_r, S_r, p_r = _ref(variant, x, S0, p0)
    assert rel_maxabs(o, o_r) <= OUT_TOL / 10
    assert rel_maxabs(S, S_r) <= STATE_TOL / 10
    np.testing.assert_allclose(f64(p), p_r, rtol=1e-5)


def test_iso_info_scale_is_honoured():
    x = to_dev(synth.layer_inputs(1, 40, 2, 64, 64, 'iso', seed=3, dtype='f32'))
    o, S, p = _run('iso', x, kappa=1.0)
    o_r, S_r, p_r = _ref('iso', x, kappa=1.0)
    np.testing.assert_allclose(f64(p), p_r, rtol=1e-5)
    assert rel_maxabs(S, S_r) <= STATE_TOL / 10


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_forward_state_handover(variant):
    """A forward over [0, T) equals one over [0, h) then [h, T) with the
    state handed over (in-place S/p aliasing allowed)."""
    B, T, H, d = 1, 50, 2, 64
    x = to_dev(synth.layer_inputs(B, T, H, d, d, variant, seed=11, dtype='bf16'))
    o, S, p = _run(variant, x)
    h = 21
    xa = {k: v[:, :h].clone() for k, v in x.items()}
    xb = {k: v[:, h:].clone() for k, v in x.items()}
    oa, Sa, pa = _run(variant, xa)
    ob, Sb, pb = _run(variant, xb, Sa, pa)
    torch.testing.assert_close(torch.cat([oa, ob], 1), o, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(Sb, S, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_decode_steps_match_oracle(variant):
    B, H, dk, dv = 4, 3, 128, 128
    st = synth.decode_state(B, H, dk, dv, variant, seed=2)
    S = st['S'].cuda()
    p = st['p'].cuda()
    S_r, p_r = f64(S), f64(p)
    for t in range(6):
        x = to_dev(synth.decode_inputs(B, H, dk, dv, variant, seed=100 + t))
        o = kdn.kdn_decode_step(variant, x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], S, p)
        o_r, S_r, p_r = kdn_ref.decode_step(variant, *(f64(x[n]) for n in 'qkvawr'), S_r, p_r)
        assert rel_maxabs(o, o_r) <= OUT_TOL / 10
    assert rel_maxabs(S, S_r) <= STATE_TOL / 10
    np.testing.assert_allclose(f64(p), p_r, rtol=1e-5)


def test_decode_512_steps_full_batch_sampled_heads():
    """512 decode steps at batch 256 x 16 heads (d 128, diagonal), from
    S ~ N(0, 0.02^2), p ~ U(0.1, 1); the oracle follows 6 sampled heads."""
    cfg = synth.WORKLOADS['diag_long']
    B, H, d, steps = cfg['decode_batch'], cfg['H'], cfg['dk'], cfg['decode_steps']
    st = synth.decode_state(B, H, d, d, 'diag', seed=cfg['seed'])
    S, p = st['S'].cuda(), st['p'].cuda()
    heads = [(0, 0), (17, 5), (100, 15), (128, 3), (200, 9), (255, 15)]
    bi = np.array([h[0] for h in heads])
    hi = np.array([h[1] for h in heads])
    S_r = f64(st['S'])[bi, hi][None]
    p_r = f64(st['p'])[bi, hi][None]
    worst_o = 0.0
    for t in range(steps):
        x = synth.decode_inputs(B, H, d, d, 'diag', seed=cfg['seed'] * 100000 + t)
        xd = to_dev(x)
        o = kdn.kdn_decode_step('diag', xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'], S, p)
        xs = [f64(x[n])[bi, hi][None] for n in 'qkvawr']
        o_r, S_r, p_r = kdn_ref.decode_step('diag', *xs, S_r, p_r)
        worst_o = max(worst_o, rel_maxabs(f64(o)[bi, hi], o_r[0]))
    assert worst_o <= OUT_TOL
    assert rel_maxabs(f64(S)[bi, hi], S_r[0]) <= STATE_TOL
    np.testing.assert_allclose(f64(p)[bi, hi], p_r[0], rtol=1e-4)


def test_unsupported_and_misaligned_rejected_on_device():
    x = to_dev(synth.layer_inputs(1, 8, 1, 64, 64, 'iso', seed=1, dtype='bf16'))
    with pytest.raises(kdn.KdnError) as e:
        kdn.kdn_iso_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'],
                            chunk=5)
    assert e.value.status == kdn.KDN_ERR_INVALID_ARG
    buf = torch.zeros(2 * 8 * 64 + 8, dtype=torch.bfloat16, device='cuda')
    kmis = buf[4:4 + 8 * 64].view(1, 8, 1, 64)  # 8-byte offset: not 16-byte aligned
    with pytest.raises(kdn.KdnError) as e:
        kdn.kdn_iso_forward(x['q'], kmis, x['v'], x['a'], x['w'], x['r'])
    assert e.value.status == kdn.KDN_ERR_INVALID_ARG
