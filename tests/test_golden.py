"""The oracle still reproduces the committed golden values (CPU only)."""
import json
import os

import numpy as np

from kalman_filter_linear_b200 import synth
from oracle import kdn_ref

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_reproduces_iso_small_golden():
    with open(os.path.join(HERE, 'golden', 'iso_small.json')) as f:
        gold = json.load(f)
    cfg = synth.WORKLOADS['iso_small']
    x = synth.layer_inputs(cfg['B'], cfg['T'], cfg['H'], cfg['dk'], cfg['dv'], 'iso',
                           cfg['seed'], cfg['dtype'])
    o, S, p = kdn_ref.iso_forward(*(x[n].double().numpy() for n in 'qkvawr'))
    np.testing.assert_allclose([o[tuple(i)] for i in gold['o_index']], gold['o_value'],
                               rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose([S[tuple(i)] for i in gold['S_index']], gold['S_value'],
                               rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(p, gold['p_T'], rtol=1e-13)
