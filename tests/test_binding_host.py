"""The Python binding fails loudly and never computes on the CPU (no GPU
needed): CPU tensors are refused before any call, a missing library raises,
and the package never imports the oracle."""
import os
import subprocess
import sys

import pytest
import torch

from kalman_filter_linear_b200 import kdn, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cpu_inputs(variant='iso', d=128):
    return synth.layer_inputs(1, 8, 1, d, d, variant, seed=0, dtype='bf16')


@pytest.mark.parametrize("call", [
    lambda x: kdn.kdn_iso_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r']),
    lambda x: kdn.kdn_exact_forward('iso', x['q'], x['k'], x['v'], x['a'], x['w'], x['r']),
    lambda x: kdn.kdn_backward('iso', x['q'], x['k'], x['v'], x['a'], x['w'], x['r'],
                               torch.zeros(x['v'].shape)),
    lambda x: kdn.kdn_forward_varlen(kdn.KDN_ISO, x['q'][0], x['k'][0], x['v'][0], x['a'][0],
                                     x['w'][0], x['r'][0], torch.tensor([0, 8], dtype=torch.int32)),
])
def test_cpu_tensors_are_refused(call):
    with pytest.raises(TypeError, match='CUDA tensor'):
        call(_cpu_inputs())


def test_cpu_tensors_are_refused_by_the_diagonal_calls():
    x = _cpu_inputs('diag')
    with pytest.raises(TypeError, match='CUDA tensor'):
        kdn.kdn_diag_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'])
    with pytest.raises(TypeError, match='CUDA tensor'):
        kdn.kdn_kla_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'])


def test_missing_library_raises(monkeypatch):
    monkeypatch.setattr(kdn, 'LIB_PATH', os.path.join(ROOT, 'no_such_dir', 'libkdn.so'))
    monkeypatch.setattr(kdn, '_lib', None)
    with pytest.raises(RuntimeError, match='missing'):
        kdn.lib()


def test_package_never_imports_the_oracle():
    code = ('import sys; import kalman_filter_linear_b200, kalman_filter_linear_b200.kdn, '
            'kalman_filter_linear_b200.synth; '
            'sys.exit(1 if any(m == "oracle" or m.startswith("oracle.") for m in sys.modules) '
            'else 0)')
    r = subprocess.run([sys.executable, '-c', code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
