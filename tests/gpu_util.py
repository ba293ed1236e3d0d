"""Helpers shared by the GPU parity tests (no filter arithmetic here)."""
import numpy as np
import torch

# Tolerances of the layer contract: the fp32 scan to 1e-5 relative; layer
# outputs to 2e-2 of max-abs error over the output RMS; the fp32 final state
# to 1e-3 of max-abs error over its RMS.
SCAN_RTOL = 1e-5
OUT_TOL = 2e-2
STATE_TOL = 1e-3


def rel_maxabs(x, ref):
    """max |x - ref| / rms(ref), both converted to fp64 NumPy."""
    x = np.asarray(x.detach().cpu().double() if isinstance(x, torch.Tensor) else x, np.float64)
    ref = np.asarray(ref.detach().cpu().double() if isinstance(ref, torch.Tensor) else ref,
                     np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(x - ref)) / rms) if rms > 0 else float(np.max(np.abs(x - ref)))


def max_rel(x, ref):
    x = np.asarray(x.detach().cpu().double() if isinstance(x, torch.Tensor) else x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref) / np.abs(ref)))


def to_dev(d, device='cuda'):
    return {k: v.to(device).contiguous() for k, v in d.items()}


def f64(t):
    return t.detach().cpu().double().numpy()
