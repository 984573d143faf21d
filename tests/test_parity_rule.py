"""The parity rules themselves: both accept the oracle rounded to bf16 and reject outputs that are
wrong but small (long-context outputs are ~1e-2); the element-wise rule also rejects a single
element off by more than 1e-2 of itself, which the per-vector rule lets through."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity import assert_parity, assert_parity_gemm, assert_parity_gemm_vector, assert_parity_prefill, errors


def _long_context_ref():
    d = wl.random_decode_inputs(2, 4096, wl.DIFFQKV, seed=501)
    return oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])


@pytest.mark.parametrize("rule", [assert_parity, assert_parity_prefill])
def test_bf16_rounded_oracle_passes(rule):
    ref = _long_context_ref()
    got = torch.from_numpy(ref).to(torch.bfloat16)
    rule(got, ref, "bf16(oracle)")


@pytest.mark.parametrize("rule", [assert_parity, assert_parity_prefill])
def test_zero_and_shuffled_outputs_fail(rule):
    ref = _long_context_ref()
    assert np.abs(ref).max() < 2e-1     # small outputs: an absolute bound alone would be vacuous
    with pytest.raises(AssertionError):
        rule(np.zeros_like(ref), ref, "zeros")
    with pytest.raises(AssertionError):
        rule(ref[:, ::-1].copy(), ref, "heads swapped")
    with pytest.raises(AssertionError):
        rule(ref * 1.03, ref, "3% scale error")


def test_element_rule_rejects_one_bad_element():
    ref = _long_context_ref()
    got = ref.copy()
    i = np.unravel_index(np.argmin(np.abs(np.abs(ref) - 0.02)), ref.shape)
    got[i] *= 1.03            # one element of ~0.02 3% off; its vector is still within 1e-2 of itself
    assert errors(got, ref)[1] <= 1e-2
    assert_parity_prefill(got, ref, "one element, per-vector rule")
    with pytest.raises(AssertionError):
        assert_parity(got, ref, "one element, element-wise rule")


def test_element_rule_floor_near_zero():
    ref = np.array([[0.0, 1e-3, 0.5]])
    assert_parity(ref + np.array([[9e-5, -9e-5, 4e-3]]), ref, "inside: 9e-5 below the floor, 0.8% above it")
    with pytest.raises(AssertionError):
        assert_parity(ref + np.array([[2e-4, 0.0, 0.0]]), ref, "2e-4 at a zero element")


def test_vector_rule_zero_reference_rows_must_be_exact():
    ref = np.zeros((2, 3, 8))
    assert errors(np.zeros_like(ref), ref)[1] == 0.0
    with pytest.raises(AssertionError):
        assert_parity_prefill(np.full_like(ref, 1e-6), ref, "nonzero where zero")


def test_gemm_rules_scale_free():
    """GEMM rules: the bf16 rounding of values up to 100 passes (the attention rules' absolute cap
    would not), a 3% scale error or one element 3% off fails the element rule, and the vector rule
    rejects a swapped pair of rows."""
    rng = np.random.default_rng(3)
    ref = rng.standard_normal((40, 64)) * 30.0
    got = torch.from_numpy(ref).to(torch.bfloat16)
    assert errors(got, ref)[0] > 2e-2
    assert_parity_gemm(got, ref, "bf16 of large values")
    assert_parity_gemm_vector(got, ref, "bf16 of large values")
    with pytest.raises(AssertionError):
        assert_parity(got, ref, "attention rule caps the absolute error")
    with pytest.raises(AssertionError):
        assert_parity_gemm(ref * 1.03, ref, "3% scale")
    bad = ref.copy()
    bad[5, 7] *= 1.03
    with pytest.raises(AssertionError):
        assert_parity_gemm(bad, ref, "one element")
    with pytest.raises(AssertionError):
        assert_parity_gemm_vector(ref[[1, 0] + list(range(2, 40))], ref, "rows swapped")
