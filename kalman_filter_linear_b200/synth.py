"""Seeded synthetic inputs for the KDN layer, its variance scan and decode.

This module only draws random numbers; it holds none of the filter's
arithmetic, so the CUDA path and the fp64 oracle can both take their inputs
from it.  Everything is drawn on the CPU with ``torch.Generator`` in fp32, in
a fixed order, so a (workload, seed) pair names one exact input set.

Distributions (per token and head):
  q, k  ~ N(0, 1), then L2-normalised over the key dimension
  v     ~ N(0, 1)
  a     = sigmoid(N(2, 0.5))          decay
  w     = softplus(N(-2, 0.5))        process-noise variance ([B,T,H] for the
                                      isotropic layer, [B,T,H,d_k] diagonal)
  r     = softplus(N(0, 1))           observation-noise variance
q, k and v are then cast to the requested dtype (k is normalised in fp32
first).  a, w and r stay fp32.

The named workloads mirror the five benchmark configurations of this library:
  'iso_small'   isotropic layer, fp32, B1 T256 H2 d64, seed 0
  'scan'        variance scan alone, 4096 lanes x T 65536, ||k||^2 ~ U(0.5,1.5)
  'iso_1p3b'    isotropic layer, bf16, B8 T4096 H16 d128, seed 2
  'diag_1p3b'   diagonal layer, bf16, B8 T4096 H16 d128, seed 3
  'diag_long'   diagonal layer, bf16, B1 T65536 H16 d128, seed 4, followed by
                512 decode steps at batch 256 from S ~ N(0, 0.02^2),
                p ~ U(0.1, 1)
  'iso_varlen'  isotropic layer, bf16, H16 d128, 32768 tokens packed from
                sequences of log-uniform length in [64, 4096] (``packed_lengths``,
                seed 5), the same token count as 'iso_1p3b'
  'exact_d64'   dense (full-covariance) filter, bf16, B8 T4096 H16 d_k = d_v = 64,
                W = w I, seed 6
"""
from __future__ import annotations

import torch

WORKLOADS = {
    'iso_small': dict(variant='iso', B=1, T=256, H=2, dk=64, dv=64, dtype='f32', seed=0),
    'scan': dict(N=4096, T=65536, seed=1, info_scale=1.0 / 64),
    'iso_1p3b': dict(variant='iso', B=8, T=4096, H=16, dk=128, dv=128, dtype='bf16', seed=2),
    'diag_1p3b': dict(variant='diag', B=8, T=4096, H=16, dk=128, dv=128, dtype='bf16', seed=3),
    'diag_long': dict(variant='diag', B=1, T=65536, H=16, dk=128, dv=128, dtype='bf16', seed=4,
                      decode_batch=256, decode_steps=512),
    'iso_varlen': dict(variant='iso', total=32768, H=16, dk=128, dv=128, dtype='bf16', seed=5,
                       min_len=64, max_len=4096),
    'exact_d64': dict(variant='iso', B=8, T=4096, H=16, dk=64, dv=64, dtype='bf16', seed=6),
}

_DT = {'f32': torch.float32, 'bf16': torch.bfloat16}


def _gen(seed):
    g = torch.Generator(device='cpu')
    g.manual_seed(int(seed))
    return g


def _normal(g, shape, mean=0.0, std=1.0):
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x


def _unit(x):
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def layer_inputs(B, T, H, dk, dv, variant='iso', seed=0, dtype='bf16'):
    """Inputs of one layer forward, as CPU tensors.

    Returns dict q, k [B,T,H,dk] and v [B,T,H,dv] in ``dtype``; a, r [B,T,H]
    fp32; w [B,T,H] (iso) or [B,T,H,dk] (diag) fp32.  Draw order: q, k, v, a,
    w, r.
    """
    g = _gen(seed)
    dt = _DT[dtype] if isinstance(dtype, str) else dtype
    q = _unit(_normal(g, (B, T, H, dk)))
    k = _unit(_normal(g, (B, T, H, dk)))
    v = _normal(g, (B, T, H, dv))
    a = torch.sigmoid(_normal(g, (B, T, H), 2.0, 0.5))
    wshape = (B, T, H) if variant == 'iso' else (B, T, H, dk)
    w = torch.nn.functional.softplus(_normal(g, wshape, -2.0, 0.5))
    r = torch.nn.functional.softplus(_normal(g, (B, T, H)))
    return dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), a=a, w=w, r=r)


def layer_inputs_extreme(B, T, H, dk, dv, variant='iso', seed=0, dtype='bf16'):
    """Layer inputs at the edges of the coefficient range, as CPU tensors,
    shaped as ``layer_inputs``.

    Per token and head: a is 1e-3 (a third of the tokens), exactly 1 (a
    third) or sigmoid(N(2, 0.5)); w = softplus(N(-2, 0.5)) with every fifth
    token's w exactly 0 (the whole vector, diagonal variant); r = 10^U(-3, 3);
    k is a unit direction times a norm 10^U(-0.5, 0.3) (so ||k||^2 spans about
    0.1 to 4); q is a unit direction; v ~ N(0, 1).  Draw order: q, k, the key
    norms, v, the decay kind, the decay, w, r.
    """
    g = _gen(seed)
    dt = _DT[dtype] if isinstance(dtype, str) else dtype
    q = _unit(_normal(g, (B, T, H, dk)))
    k = _unit(_normal(g, (B, T, H, dk)))
    knorm = torch.pow(10.0, torch.rand((B, T, H, 1), generator=g) * 0.8 - 0.5)
    k = k * knorm
    v = _normal(g, (B, T, H, dv))
    kind = torch.randint(0, 3, (B, T, H), generator=g)
    a = torch.sigmoid(_normal(g, (B, T, H), 2.0, 0.5))
    a = torch.where(kind == 0, torch.full_like(a, 1e-3), a)
    a = torch.where(kind == 1, torch.ones_like(a), a)
    wshape = (B, T, H) if variant == 'iso' else (B, T, H, dk)
    w = torch.nn.functional.softplus(_normal(g, wshape, -2.0, 0.5))
    w[:, ::5] = 0.0
    r = torch.pow(10.0, torch.rand((B, T, H), generator=g) * 6.0 - 3.0)
    return dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), a=a, w=w, r=r)


def scan_inputs(N, T, seed=1):
    """Inputs of the standalone variance scan: a, w, r, n each [N, T] fp32.

    n stands for the squared key norm and is drawn U(0.5, 1.5).  Draw order:
    a, w, r, n.
    """
    g = _gen(seed)
    a = torch.sigmoid(_normal(g, (N, T), 2.0, 0.5))
    w = torch.nn.functional.softplus(_normal(g, (N, T), -2.0, 0.5))
    r = torch.nn.functional.softplus(_normal(g, (N, T)))
    n = torch.rand((N, T), generator=g, dtype=torch.float32).add_(0.5)
    return dict(a=a, w=w, r=r, n=n)


def decode_state(B, H, dk, dv, variant='diag', seed=0):
    """A random decoding state: S ~ N(0, 0.02^2) [B,H,dv,dk] fp32 and
    p ~ U(0.1, 1) ([B,H] iso or [B,H,dk] diag) fp32."""
    g = _gen(seed)
    S = _normal(g, (B, H, dv, dk), 0.0, 0.02)
    pshape = (B, H) if variant == 'iso' else (B, H, dk)
    p = torch.rand(pshape, generator=g, dtype=torch.float32).mul_(0.9).add_(0.1)
    return dict(S=S, p=p)


def decode_inputs(B, H, dk, dv, variant='diag', seed=0, dtype='bf16'):
    """One token per (b, h), drawn like ``layer_inputs`` with T = 1 and the
    token axis removed: q, k [B,H,dk], v [B,H,dv], a, r [B,H], w [B,H] or
    [B,H,dk]."""
    x = layer_inputs(B, 1, H, dk, dv, variant, seed, dtype)
    return {name: t[:, 0] for name, t in x.items()}


def packed_lengths(total, seed=0, min_len=64, max_len=4096):
    """Sequence lengths for a packed batch of ``total`` tokens.

    Lengths are drawn log-uniform in [min_len, max_len] (a long-tailed mix of
    short and long documents), rounded down to integers, until the next one
    would pass ``total``; the last sequence takes what is left, so the list
    sums to ``total`` exactly and only its last entry may be below
    ``min_len``.  Returns a list of ints.
    """
    import math
    g = _gen(seed)
    lo, hi = math.log(min_len), math.log(max_len)
    out, left = [], int(total)
    while left > 0:
        u = float(torch.rand((), generator=g, dtype=torch.float64))
        n = min(int(math.exp(lo + u * (hi - lo))), left)
        out.append(n)
        left -= n
    return out
