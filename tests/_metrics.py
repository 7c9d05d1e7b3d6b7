"""Parity metrics and tolerances used by the GPU tests.

y: max|y - y_ref| / max|y_ref| over the whole tensor, at most Y_TOL.
states: ||S - S_ref||_F / ||S_ref||_F over the whole state tensor, at most S_TOL.
gradients: the max-normalised metric of y, per tensor, at most G_TOL.
"""
import numpy as np
import torch

Y_TOL = 1e-2
S_TOL = 1e-3
G_TOL = 1e-2


def _np(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def max_rel(x, ref):
    x, ref = _np(x), _np(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.all(np.isfinite(x)), "non-finite values in GPU output"
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(x - ref)) / (den if den > 0 else 1.0))


def frob_rel(x, ref):
    x, ref = _np(x), _np(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.all(np.isfinite(x)), "non-finite values in GPU output"
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))
