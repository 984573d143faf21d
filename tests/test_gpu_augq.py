"""GPU parity of the augmented query projection (structured-summary page, section 3.2
"Big-Picture Architecture", item 4) against the fp64 oracle, through the C ABI.

Each stage is checked element by element against the oracle fed the same bf16 inputs: the
gated hidden state h against oracle.augq_hidden, and q against oracle.augq_down of the GPU's
own (bf16-rounded) h, both within 1e-2 of each element (floor 1e-2; no absolute cap, since
GEMM outputs have no fixed scale).  The whole chain against the fp64 oracle, where h stays
unrounded, takes the per-vector rule: the single bf16 rounding of h (2^-9 per element) then
moves elements of q that cancel to nearly zero by more than 1e-2 of themselves."""
import numpy as np
import pytest
import torch

import asymmetric_head_kv_b200 as ak
import oracle
import workloads as wl
from parity import assert_parity_gemm, assert_parity_gemm_vector

pytestmark = pytest.mark.gpu


def _run(d, dev, status=None):
    g = {k: v.to(dev) for k, v in d.items()}
    q, h = ak.augq_project(g["x"], g["w_gate"], g["w_up"], g["w_down"], status=status)
    torch.cuda.synchronize()
    return q, h


def _check(d, dev, what, rows=None):
    q, h = _run(d, dev)
    r = None if rows is None else torch.as_tensor(rows)
    h_cpu = h.cpu() if r is None else h.cpu()[r]
    q_cpu = q.cpu() if r is None else q.cpu()[r]
    h_ref = oracle.augq_hidden(d["x"], d["w_gate"], d["w_up"], rows=rows)
    assert_parity_gemm(h_cpu, h_ref, f"{what}: h")
    q_from_h = oracle.augq_down(h_cpu.double().numpy(), d["w_down"])
    assert_parity_gemm(q_cpu, q_from_h, f"{what}: q from the GPU's h")
    assert_parity_gemm_vector(q_cpu, oracle.augq_down(h_ref, d["w_down"]), f"{what}: chain")
    return q, h


@pytest.mark.parametrize("tokens,d_model,d_inter,d_out", [
    (300, 256, 384, 160),     # a token tail (300 = 2 x 128 + 44) and a partial 256-wide output tile
    (1, 128, 128, 32),        # one decode token, the smallest tiles
    (129, 512, 256, 512),     # one row past a tile; two full output tiles
    (1000, 192, 640, 288),
])
def test_small_shapes(cuda_device, tokens, d_model, d_inter, d_out):
    d = wl.random_augq_inputs(tokens, d_model, d_inter, d_out, seed=tokens + d_out)
    _check(d, cuda_device, f"augq {tokens}x{d_model}x{d_inter}x{d_out}")


def test_zero_tokens_is_a_no_op(cuda_device):
    d = wl.random_augq_inputs(0, 128, 128, 32, seed=1)
    q, h = _run(d, cuda_device)
    assert q.shape == (0, 32) and h.shape == (0, 128)


def test_full_sigma_shape_sampled_rows(cuda_device):
    """16384 tokens of Sigma-1.5B's projection (2048 -> 3072 -> 2048); rows sampled across every
    128-token tile position, the first and the last."""
    w = wl.AUGQ_16K
    d = wl.make_augq_inputs(w)
    gen = np.random.default_rng(7)
    rows = sorted(set([0, 1, 127, 128, w.tokens - 1] + gen.integers(0, w.tokens, 43).tolist()))
    _check(d, cuda_device, w.name, rows=rows)


def test_status_word_and_repeatability(cuda_device):
    d = wl.random_augq_inputs(700, 256, 512, 256, seed=9)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    q1, h1 = _run(d, cuda_device, status=status)
    q2, h2 = _run(d, cuda_device, status=status)
    assert int(status.item()) == 0
    assert torch.equal(q1, q2) and torch.equal(h1, h2)   # fixed accumulation order


def test_rejects_bad_shapes(cuda_device):
    d = {k: v.to(cuda_device) for k, v in wl.random_augq_inputs(8, 128, 128, 32, seed=3).items()}
    with pytest.raises(ValueError):
        ak.augq_project(d["x"], d["w_gate"], d["w_up"][:64], d["w_down"])
    x = torch.zeros(8, 96, dtype=torch.bfloat16, device=cuda_device)
    wg = torch.zeros(128, 96, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(ak.DiffqkvError):
        ak.augq_project(x, wg, wg, d["w_down"])
