"""The parity rule itself: it must accept the oracle rounded to bf16 and reject
outputs that are wrong but small (long-context outputs are ~1e-2)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity import assert_parity, errors


def _long_context_ref():
    d = wl.random_decode_inputs(2, 4096, wl.DIFFQKV, seed=501)
    return oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])


def test_bf16_rounded_oracle_passes():
    ref = _long_context_ref()
    got = torch.from_numpy(ref).to(torch.bfloat16)
    assert_parity(got, ref, "bf16(oracle)")


def test_zero_and_shuffled_outputs_fail():
    ref = _long_context_ref()
    assert np.abs(ref).max() < 2e-1     # small outputs: an absolute bound alone would be vacuous
    with pytest.raises(AssertionError):
        assert_parity(np.zeros_like(ref), ref, "zeros")
    with pytest.raises(AssertionError):
        assert_parity(ref[:, ::-1].copy(), ref, "heads swapped")
    with pytest.raises(AssertionError):
        assert_parity(ref * 1.03, ref, "3% scale error")


def test_zero_reference_rows_must_be_exact():
    ref = np.zeros((2, 3, 8))
    assert errors(np.zeros_like(ref), ref)[1] == 0.0
    with pytest.raises(AssertionError):
        assert_parity(np.full_like(ref, 1e-6), ref, "nonzero where zero")
