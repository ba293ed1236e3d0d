"""kdn_forward_host (host buffers, batch slices on two streams) gives the
results of the device calls on the same data, and reports its workspace
status (needs a B200)."""
import pytest
import torch

from kalman_filter_linear_b200 import kdn, synth
from gpu_util import to_dev

pytestmark = pytest.mark.gpu


def _host(x):
    return {k: v.contiguous().pin_memory() for k, v in x.items()}


@pytest.mark.parametrize("variant", [kdn.KDN_ISO, kdn.KDN_DIAG])
@pytest.mark.parametrize("slice_b", [0, 2, 5])
def test_host_forward_equals_device_forward(variant, slice_b):
    B, T, H, d = 5, 130, 2, 128
    name = 'iso' if variant == kdn.KDN_ISO else 'diag'
    x = synth.layer_inputs(B, T, H, d, d, name, seed=31, dtype='bf16')
    g = torch.Generator().manual_seed(5)
    S0 = 0.05 * torch.randn(B, H, d, d, generator=g)
    p0 = torch.rand((B, H) if variant == kdn.KDN_ISO else (B, H, d), generator=g) + 0.2
    xd = to_dev(x)
    fwd = kdn.kdn_iso_forward if variant == kdn.KDN_ISO else kdn.kdn_diag_forward
    o_d, S_d, p_d = fwd(xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'], S0.cuda(),
                        p0.cuda())
    xh = _host(x)
    ws = torch.empty(kdn.kdn_forward_host_workspace_size(variant, B, T, H, d, d, kdn.KDN_BF16,
                                                         kdn.KDN_CHUNK_AUTO, slice_b),
                     dtype=torch.uint8, device='cuda')
    o_h, S_h, p_h = kdn.kdn_forward_host(variant, xh['q'], xh['k'], xh['v'], xh['a'], xh['w'],
                                         xh['r'], S0.pin_memory(), p0.pin_memory(),
                                         slice_b=slice_b, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_d.cpu())
    assert torch.equal(S_h, S_d.cpu())
    assert torch.equal(p_h, p_d.cpu())
    assert kdn.kdn_read_workspace_status(ws) == kdn.KDN_OK


def test_host_forward_recurrent_path_and_small_workspace():
    """fp32 inputs at d = 64 take the token-recurrent kernel; a workspace one
    byte short is rejected before anything runs."""
    B, T, H, d = 3, 50, 2, 64
    x = synth.layer_inputs(B, T, H, d, d, 'iso', seed=8, dtype='f32')
    xd = to_dev(x)
    o_d, S_d, p_d = kdn.kdn_iso_forward(xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'])
    xh = _host(x)
    need = kdn.kdn_forward_host_workspace_size(kdn.KDN_ISO, B, T, H, d, d, kdn.KDN_F32)
    ws = torch.empty(need, dtype=torch.uint8, device='cuda')
    o_h, S_h, p_h = kdn.kdn_forward_host(kdn.KDN_ISO, xh['q'], xh['k'], xh['v'], xh['a'],
                                         xh['w'], xh['r'], workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(S_h, S_d.cpu())
    assert torch.equal(p_h, p_d.cpu())
    with pytest.raises(kdn.KdnError) as e:
        kdn.kdn_forward_host(kdn.KDN_ISO, xh['q'], xh['k'], xh['v'], xh['a'], xh['w'], xh['r'],
                             workspace=ws[:need - 1])
    assert e.value.status == kdn.KDN_ERR_WORKSPACE
