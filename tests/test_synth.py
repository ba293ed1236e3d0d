"""The seeded input generators (CPU): the packed-length mix and the
determinism every parity test relies on."""
import torch

from kalman_filter_linear_b200 import synth


def test_packed_lengths_fill_the_budget_within_bounds():
    for seed in range(5):
        L = synth.packed_lengths(32768, seed, 64, 4096)
        assert sum(L) == 32768
        assert all(64 <= n <= 4096 for n in L[:-1])
        assert 1 <= L[-1] <= 4096
    assert synth.packed_lengths(32768, 5) == synth.packed_lengths(32768, 5)
    assert synth.packed_lengths(32768, 5) != synth.packed_lengths(32768, 6)
    assert synth.packed_lengths(10, 0, 64, 4096) == [10]


def test_layer_inputs_are_seeded_and_in_range():
    a = synth.layer_inputs(1, 20, 2, 32, 16, 'diag', seed=3, dtype='f32')
    b = synth.layer_inputs(1, 20, 2, 32, 16, 'diag', seed=3, dtype='f32')
    for k in a:
        assert torch.equal(a[k], b[k])
    assert a['w'].shape == (1, 20, 2, 32)
    assert torch.all((a['a'] > 0) & (a['a'] < 1))
    assert torch.all(a['w'] > 0) and torch.all(a['r'] > 0)
    torch.testing.assert_close(a['k'].norm(dim=-1), torch.ones(1, 20, 2))


def test_extreme_layer_inputs_are_seeded_and_reach_the_edges():
    a = synth.layer_inputs_extreme(1, 90, 2, 32, 16, 'diag', seed=4, dtype='f32')
    b = synth.layer_inputs_extreme(1, 90, 2, 32, 16, 'diag', seed=4, dtype='f32')
    for k in a:
        assert torch.equal(a[k], b[k])
    dec = a['a']
    assert torch.any(dec == 1.0) and torch.any(torch.isclose(dec, torch.tensor(1e-3)))
    assert torch.all((dec > 0) & (dec <= 1))
    assert torch.all(a['w'][:, ::5] == 0) and torch.all(a['w'] >= 0)
    assert float(a['r'].min()) < 1e-2 and float(a['r'].max()) > 1e2
    n = a['k'].norm(dim=-1) ** 2
    assert float(n.min()) < 0.5 and float(n.max()) > 2.0
