"""Pins of the oracle's augmented query projection (structured-summary page, section 3.2
"Big-Picture Architecture", item 4: q = q_down(SiLU(q_gate(x)) * q_up(x))) against closed forms
and library routines, never against the oracle's own formula retyped."""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle


def _one_hot_case(gates, ups, d_model=64):
    """x = e_0, so the gate and up sums of output o are exactly gates[o] and ups[o]."""
    n = len(gates)
    x = torch.zeros(1, d_model)
    x[0, 0] = 1.0
    wg = torch.zeros(n, d_model)
    wu = torch.zeros(n, d_model)
    wg[:, 0] = torch.tensor(gates, dtype=torch.float32)
    wu[:, 0] = torch.tensor(ups, dtype=torch.float32)
    return oracle.augq_hidden(x.bfloat16(), wg.bfloat16(), wu.bfloat16())[0]


def test_silu_closed_forms():
    g = [0.0, 0.5, -0.5, 1.0, -1.0, 2.0, -2.0, 8.0, -8.0, 64.0, -64.0, 2.0 ** -20]
    h = _one_hot_case(g, [1.0] * len(g))
    assert h[0] == 0.0                                     # SiLU(0) = 0
    for i in range(1, 11, 2):                              # SiLU(g) - SiLU(-g) = g(s(g) + s(-g)) = g
        assert abs((h[i] - h[i + 1]) - g[i]) <= 1e-15 * abs(g[i])
    assert abs(h[9] - 64.0) <= 64.0 * 1e-27 + 1e-12        # 64 (1 - e^-64 + ...) -> 64
    assert 0 > h[10] > -1e-25                              # -64 e^-64
    assert abs(h[11] / g[11] - 0.5) < 1e-6                 # slope 1/2 at 0
    assert all(np.diff(h[[0, 1, 3, 5, 7, 9]]) > 0)         # increasing for g >= 0
    assert h[4] < 0 and h[4] > -0.28                       # minimum of SiLU is about -0.2785


def test_gate_and_up_roles():
    """SiLU acts on the gate branch only: (gate 64, up 1) gives 64, (gate 1, up 64) gives 64 s(1)."""
    h = _one_hot_case([64.0, 1.0, 0.0, 3.0], [1.0, 64.0, 5.0, 0.0])
    assert abs(h[0] - 64.0) < 1e-12
    assert abs(h[1] - 64.0 * scipy.special.expit(1.0)) < 1e-12
    assert h[2] == 0.0 and h[3] == 0.0                     # a zero gate or a zero up branch zeroes h


def _int_bf16(shape, lo, hi, gen):
    return torch.randint(lo, hi + 1, shape, generator=gen).to(torch.bfloat16)


def test_matches_library_on_integer_inputs():
    """Small integers keep every sum exact, so numpy's integer matmul gives the exact gate and up
    values; scipy's logistic function gives SiLU; numpy's float matmul gives the down projection.
    Every dimension differs, so a transposed operand cannot pass."""
    gen = torch.Generator().manual_seed(41)
    tokens, d_model, d_inter, d_out = 7, 48, 40, 24
    x = _int_bf16((tokens, d_model), -4, 4, gen)
    wg = _int_bf16((d_inter, d_model), -3, 3, gen)
    wu = _int_bf16((d_inter, d_model), -3, 3, gen)
    wd = _int_bf16((d_out, d_inter), -2, 2, gen)
    xi, gi, ui, di = (t.to(torch.int64).numpy() for t in (x, wg, wu, wd))
    g = (xi @ gi.T).astype(np.float64)
    u = (xi @ ui.T).astype(np.float64)
    h_ref = g * scipy.special.expit(g) * u
    q_ref = h_ref @ di.T.astype(np.float64)
    h = oracle.augq_hidden(x, wg, wu)
    np.testing.assert_allclose(h, h_ref, rtol=1e-13, atol=1e-13)
    q = oracle.augq_project(x, wg, wu, wd)
    np.testing.assert_allclose(q, q_ref, rtol=1e-12, atol=1e-9)
    rows = [6, 0, 3]
    np.testing.assert_array_equal(oracle.augq_project(x, wg, wu, wd, rows=rows), q[rows])


def test_down_is_a_matrix_product():
    gen = np.random.default_rng(42)
    h = gen.standard_normal((5, 96))
    wd = torch.from_numpy(gen.integers(-8, 9, (33, 96)).astype(np.float32)).bfloat16()
    np.testing.assert_allclose(oracle.augq_down(h, wd), h @ wd.float().numpy().T.astype(np.float64),
                               rtol=1e-13, atol=1e-12)


def test_bad_rows_are_rejected():
    x = torch.zeros(3, 64).bfloat16()
    w = torch.zeros(8, 64).bfloat16()
    with pytest.raises(RuntimeError):
        oracle.augq_hidden(x, w, w, rows=[3])
