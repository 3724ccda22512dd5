"""Output tolerance used by every GPU-vs-oracle comparison of the layer output.

The layer output is bf16, so the comparison allows, per element, the output's own mandatory
rounding (half a bf16 ulp of the larger of |gpu| and |oracle|) on top of an absolute 2e-2, and
requires a relative RMS error of at most 1e-2 over the whole output.  The oracle value is fp64.
"""
import numpy as np
import torch

ABS_TOL = 2e-2
REL_RMS_TOL = 1e-2


def to_f64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().double().cpu().numpy()
    return np.asarray(t, np.float64)


def ulp_bf16(a):
    a = np.maximum(np.abs(a), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def compare(gpu, ref, abs_tol=ABS_TOL, rel_rms_tol=REL_RMS_TOL):
    g = to_f64(gpu)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), "non-finite GPU output"
    err = np.abs(g - r)
    bound = abs_tol + 0.5 * ulp_bf16(np.maximum(np.abs(g), np.abs(r)))
    nr = np.linalg.norm(r)
    rel_rms = np.linalg.norm(g - r) / nr if nr > 0 else np.linalg.norm(g - r)
    stats = dict(max_abs=float(err.max()) if err.size else 0.0, rel_rms=float(rel_rms),
                 worst_ratio=float((err / bound).max()) if err.size else 0.0)
    assert rel_rms <= rel_rms_tol, stats
    assert (err <= bound).all(), stats
    return stats
