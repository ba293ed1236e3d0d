"""Write tests/golden/iso_small.json from the fp64 oracle (and nothing else).

The workload is the small isotropic forward (B1 T256 H2 d64, fp32, seed 0,
S0 = 0, p0 = 1, kappa = 1/d_k) drawn by kalman_filter_linear_b200.synth.  The
pages print no worked example, so these values are a regression pin of the
oracle and a fixed anchor for the GPU parity tests, not a value from the pages.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from kalman_filter_linear_b200 import synth  # noqa: E402
from oracle import kdn_ref  # noqa: E402


def main():
    cfg = synth.WORKLOADS['iso_small']
    x = synth.layer_inputs(cfg['B'], cfg['T'], cfg['H'], cfg['dk'], cfg['dv'], 'iso',
                           cfg['seed'], cfg['dtype'])
    o, S, p = kdn_ref.iso_forward(*(x[n].double().numpy() for n in 'qkvawr'))
    rng = np.random.default_rng(1234)
    o_idx = [tuple(int(i) for i in ix) for ix in zip(*(rng.integers(0, s, 64) for s in o.shape))]
    S_idx = [tuple(int(i) for i in ix) for ix in zip(*(rng.integers(0, s, 32) for s in S.shape))]
    out = dict(
        workload='iso_small', source='oracle/kdn_ref.iso_forward (fp64)',
        o_index=o_idx, o_value=[float(o[i]) for i in o_idx],
        S_index=S_idx, S_value=[float(S[i]) for i in S_idx],
        p_T=p.tolist(), o_rms=float(np.sqrt((o ** 2).mean())),
        S_rms=float(np.sqrt((S ** 2).mean())))
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), 'iso_small.json')
    with open(path, 'w') as f:
        json.dump(out, f, indent=1)
    print('wrote', path)


if __name__ == '__main__':
    main()
