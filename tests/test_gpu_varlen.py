"""Packed variable-length sequences (kdn_forward_varlen) against the fp64
oracle run sequence by sequence, and the prefill -> decode handoff (needs a
B200).  Tolerances as the layer contract: outputs 2e-2, final state 1e-3
(max-abs over RMS), variances 1e-5."""
import numpy as np
import pytest
import torch

from kalman_filter_linear_b200 import kdn, synth
from oracle import kdn_ref
from gpu_util import OUT_TOL, STATE_TOL, rel_maxabs, f64

pytestmark = pytest.mark.gpu

LENGTHS = [65, 0, 1, 130, 63, 64, 7, 200]


def _packed(variant, lengths, H, dk, dv, dtype, seed):
    """Seeded inputs of the given lengths, packed along the token axis."""
    total = sum(lengths)
    x = synth.layer_inputs(1, max(total, 1), H, dk, dv, variant, seed=seed, dtype=dtype)
    x = {k: v[0, :total].contiguous() for k, v in x.items()}
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    return x, cu


def _oracle(variant, x, cu, S0, p0):
    fwd = kdn_ref.iso_forward if variant == 'iso' else kdn_ref.diag_forward
    outs, Ss, ps = [], [], []
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        sl = {k: f64(v[lo:hi])[None] for k, v in x.items()}
        o, S, p = fwd(sl['q'], sl['k'], sl['v'], sl['a'], sl['w'], sl['r'],
                      S0=f64(S0[s:s + 1]), p0=f64(p0[s:s + 1]))
        outs.append(o[0])
        Ss.append(S[0])
        ps.append(p[0])
    return np.concatenate(outs, 0), np.stack(Ss), np.stack(ps)


@pytest.mark.parametrize("variant", ["iso", "diag"])
@pytest.mark.parametrize("case", ["chunked", "recurrent"])
def test_varlen_matches_oracle(variant, case):
    """Sequences of mixed lengths (an empty one among them, lengths on both
    sides of the 64-token chunk) each match the oracle run on their own."""
    H = 2
    d, dt = (128, 'bf16') if case == 'chunked' else (64, 'f32')
    x, cu = _packed(variant, LENGTHS, H, d, d, dt, seed=77)
    N = len(LENGTHS)
    g = torch.Generator().manual_seed(3)
    S0 = 0.05 * torch.randn(N, H, d, d, generator=g)
    p0 = torch.rand((N, H) if variant == 'iso' else (N, H, d), generator=g) + 0.2
    xd = {k: v.cuda() for k, v in x.items()}
    var = kdn.KDN_ISO if variant == 'iso' else kdn.KDN_DIAG
    ws = torch.empty(kdn.kdn_forward_varlen_workspace_size(var, N, H, d, d), dtype=torch.uint8,
                     device='cuda')
    o, S, p = kdn.kdn_forward_varlen(var, xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                                     cu.cuda(), S0.cuda(), p0.cuda(), workspace=ws)
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_OK
    o_r, S_r, p_r = _oracle(variant, x, cu, S0, p0)
    assert rel_maxabs(o, o_r) <= OUT_TOL
    assert rel_maxabs(S, S_r) <= STATE_TOL
    np.testing.assert_allclose(f64(p), p_r, rtol=1e-5)
    # the empty sequence hands its initial state through unchanged
    assert torch.equal(S[1].cpu(), S0[1]) and torch.equal(p[1].cpu(), p0[1])


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_varlen_equal_lengths_agree_with_dense(variant):
    """Packed sequences of one length give the dense [B, T] call's results."""
    B, T, H, d = 3, 150, 2, 128
    x = synth.layer_inputs(B, T, H, d, d, variant, seed=9, dtype='bf16')
    xd = {k: v.cuda() for k, v in x.items()}
    fwd = kdn.kdn_iso_forward if variant == 'iso' else kdn.kdn_diag_forward
    o_d, S_d, p_d = fwd(xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'])
    flat = {k: v.reshape(B * T, *v.shape[2:]).contiguous() for k, v in xd.items()}
    cu = torch.arange(0, B * T + 1, T, dtype=torch.int32, device='cuda')
    var = kdn.KDN_ISO if variant == 'iso' else kdn.KDN_DIAG
    o_v, S_v, p_v = kdn.kdn_forward_varlen(var, flat['q'], flat['k'], flat['v'], flat['a'],
                                           flat['w'], flat['r'], cu)
    assert rel_maxabs(o_v.reshape(B, T, H, d), f64(o_d)) <= 1e-5
    assert rel_maxabs(S_v, f64(S_d)) <= 1e-5
    torch.testing.assert_close(p_v, p_d, rtol=1e-6, atol=0)


def _sm_count():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_varlen_many_sequences_longest_first(variant):
    """More (sequence, head) problems than SMs: the engine takes the
    sequences longest first, and every sequence still lands in its own rows
    of o, S_T and p_T.  Lengths mix zeros, ragged tails and full chunks."""
    H, d = 2, 128
    N = _sm_count() // H + 12
    g = np.random.default_rng(41)
    lengths = [int(n) for n in g.integers(0, 150, size=N)]
    lengths[3] = 0
    lengths[N - 1] = 300  # the longest one last in the packing
    x, cu = _packed(variant, lengths, H, d, d, 'bf16', seed=43)
    gt = torch.Generator().manual_seed(44)
    S0 = 0.05 * torch.randn(N, H, d, d, generator=gt)
    p0 = torch.rand((N, H) if variant == 'iso' else (N, H, d), generator=gt) + 0.2
    xd = {k: v.cuda() for k, v in x.items()}
    var = kdn.KDN_ISO if variant == 'iso' else kdn.KDN_DIAG
    ws = torch.empty(kdn.kdn_forward_varlen_workspace_size(var, N, H, d, d), dtype=torch.uint8,
                     device='cuda')
    o, S, p = kdn.kdn_forward_varlen(var, xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                                     cu.cuda(), S0.cuda(), p0.cuda(), workspace=ws)
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_OK
    o_r, S_r, p_r = _oracle(variant, x, cu, S0, p0)
    assert rel_maxabs(o, o_r) <= OUT_TOL
    for s in range(N):  # per sequence, so that a swapped pair of rows fails
        assert rel_maxabs(S[s], S_r[s]) <= STATE_TOL, s
    np.testing.assert_allclose(f64(p), p_r, rtol=1e-5)
    assert torch.equal(S[3].cpu(), S0[3]) and torch.equal(p[3].cpu(), p0[3])


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_varlen_longest_first_is_bitwise_the_dense_result(variant):
    """With the launch order permuted (more problems than SMs, unequal
    lengths), each sequence's results are bit for bit those of the dense
    call on that sequence alone: the order moves work, not arithmetic."""
    H, d = 2, 128
    N = _sm_count() // H + 4
    lengths = [64 + 37 * (i % 5) for i in range(N)]
    x, cu = _packed(variant, lengths, H, d, d, 'bf16', seed=47)
    xd = {k: v.cuda() for k, v in x.items()}
    var = kdn.KDN_ISO if variant == 'iso' else kdn.KDN_DIAG
    o, S, p = kdn.kdn_forward_varlen(var, xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                                     cu.cuda())
    fwd = kdn.kdn_iso_forward if variant == 'iso' else kdn.kdn_diag_forward
    for s in (0, 1, 2, 3, 4, N - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        one = {k: v[lo:hi][None].clone() for k, v in xd.items()}  # aligned copies
        o1, S1, p1 = fwd(one['q'], one['k'], one['v'], one['a'], one['w'], one['r'])
        assert torch.equal(o[lo:hi], o1[0]), s
        assert torch.equal(S[s], S1[0]) and torch.equal(p[s], p1[0]), s


def test_varlen_bad_offsets_are_clamped_and_reported():
    """Offsets out of order are clamped (the sequence is empty) and the
    workspace reports KDN_ERR_INVALID_ARG."""
    H, d = 2, 128
    x, _ = _packed('iso', [100, 50], H, d, d, 'bf16', seed=5)
    cu = torch.tensor([0, 120, 100], dtype=torch.int32, device='cuda')
    xd = {k: v.cuda() for k, v in x.items()}
    ws = torch.empty(kdn.kdn_forward_varlen_workspace_size(kdn.KDN_ISO, 2, H, d, d),
                     dtype=torch.uint8, device='cuda')
    kdn.kdn_forward_varlen(kdn.KDN_ISO, xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                           cu, workspace=ws)
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_ERR_INVALID_ARG


@pytest.mark.parametrize("variant", ["iso", "diag"])
def test_prefill_then_decode_continues_each_sequence(variant):
    """The final states of a packed prefill feed kdn_decode_step; each step's
    output and state match the oracle run over the sequence plus the token."""
    H, d = 2, 128
    lengths = [70, 1, 129]
    N = len(lengths)
    x, cu = _packed(variant, lengths, H, d, d, 'bf16', seed=21)
    xd = {k: v.cuda() for k, v in x.items()}
    var = kdn.KDN_ISO if variant == 'iso' else kdn.KDN_DIAG
    o, S, p = kdn.kdn_forward_varlen(var, xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                                     cu.cuda())
    nxt = synth.layer_inputs(N, 1, H, d, d, variant, seed=22, dtype='bf16')
    nx = {k: v[:, 0].contiguous().cuda() for k, v in nxt.items()}
    o1 = kdn.kdn_decode_step(var, nx['q'], nx['k'], nx['v'], nx['a'], nx['w'], nx['r'], S, p)
    S1, p1 = S, p  # updated in place
    fwd = kdn_ref.iso_forward if variant == 'iso' else kdn_ref.diag_forward
    for s in range(N):
        lo, hi = int(cu[s]), int(cu[s + 1])
        seq = {k: np.concatenate([f64(x[k][lo:hi]), f64(nxt[k][s])], 0)[None] for k in x}
        o_r, S_r, p_r = fwd(seq['q'], seq['k'], seq['v'], seq['a'], seq['w'], seq['r'])
        assert rel_maxabs(o1[s], o_r[0, -1]) <= OUT_TOL
        assert rel_maxabs(S1[s], S_r[0]) <= STATE_TOL
        np.testing.assert_allclose(f64(p1[s]), p_r[0], rtol=1e-5)
