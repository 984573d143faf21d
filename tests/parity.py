"""Shared parity tolerance for bf16 outputs computed with fp32 accumulation.

Pass iff  max|g - r| <= 2e-2  and  max(|g - r| / max(|r|, 1e-2)) <= 1e-2,
g the GPU result (bf16 -> fp64), r the fp64 oracle.  The relative bound uses
a floor of 1e-2 because long-context outputs are small (|r| ~ 1e-2 at 32k
positions), where a pure absolute bound of 2e-2 would say nothing; rounding
the oracle itself to bf16 already costs up to 2^-9 relative.
"""
import numpy as np
import torch

ATOL = 2e-2
RTOL = 1e-2
REL_FLOOR = 1e-2


def errors(got, ref):
    g = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    d = np.abs(g - r)
    rel = d / np.maximum(np.abs(r), REL_FLOOR)
    norm = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))
    return float(d.max(initial=0.0)), float(rel.max(initial=0.0)), norm


def assert_parity(got, ref, what=""):
    mx, rel, norm = errors(got, ref)
    assert np.all(np.isfinite(np.asarray(got.detach().float().cpu() if isinstance(got, torch.Tensor) else got))), what
    assert mx <= ATOL and rel <= RTOL, f"{what}: max-abs {mx:.3e}, max-rel {rel:.3e}, normwise {norm:.3e}"
    return mx, rel, norm
