"""GPU parity of the query fold for query and key of different widths.

The pages project every cached K row up to the query width before the dot product (the Attend
function of section 3.4 Step 4).  The library folds that projection into the query instead;
expected values come from the fp64 oracle in the pages' order (keys projected up, then the
softmax), and from the fp64 fold itself with an explicit error bound for the fp32 sum and the
bf16 rounding of the folded query."""
import math

import numpy as np
import pytest
import torch

import asymmetric_head_kv_b200 as ak
import oracle
import workloads as wl
from workloads import Shape
from parity import assert_parity, assert_parity_prefill

pytestmark = pytest.mark.gpu


def _inputs(shape, d_q, w_heads, seed, lens, t_max):
    d = wl.random_decode_inputs(len(lens), t_max, shape, seed=seed, seq_lens=lens)
    g = torch.Generator().manual_seed(seed + 1)
    q_aug = torch.randn(len(lens), shape.n_q, d_q, generator=g).to(torch.bfloat16)
    w = (torch.randn(w_heads, d_q, shape.d_k, generator=g) / math.sqrt(shape.d_k)).to(torch.bfloat16)
    return d, q_aug, w


CASES = [
    ("diffqkv_dq192", wl.DIFFQKV, 192, 4),
    ("diffqkv_dq96_shared", wl.DIFFQKV, 96, 1),
    ("gqa_dk128_dq256", wl.GQA_CONTROL, 256, 16),
    ("qpk3_dq40", Shape(12, 4, 4, 64, 64), 40, 4),
    # 16 warps over 5 rows: 3 slices x 5 rows leave one warp without a (row, slice) slot
    ("qpk5_dq72", Shape(20, 4, 4, 64, 64), 72, 4),
    ("mha_dq8", Shape(8, 8, 8, 128, 64), 8, 8),
]


@pytest.mark.parametrize("name,shape,d_q,w_heads", CASES)
def test_fold_matches_oracle_within_rounding(cuda_device, name, shape, d_q, w_heads):
    _, q_aug, w = _inputs(shape, d_q, w_heads, 801, [5, 5, 5], 5)
    ref = oracle.fold_query(q_aug, w, shape.n_k)
    got = ak.fold_query(q_aug.to(cuda_device), w.to(cuda_device), n_k=shape.n_k)
    torch.cuda.synchronize()
    got = got.cpu().double().numpy()
    Wh = w.double().expand(shape.n_k, -1, -1)[torch.arange(shape.n_q) // (shape.n_q // shape.n_k)]
    absum = torch.einsum("bhr,hrc->bhc", q_aug.double().abs(), Wh.abs()).numpy()
    # bf16 rounding of the result (2^-8 relative) plus the fp32 sum's error (d_q roundings of 2^-24)
    bound = 2.0 ** -8 * np.abs(ref) + (d_q + 2) * 2.0 ** -23 * absum
    assert np.all(np.abs(got - ref) <= bound), f"{name}: max excess {np.max(np.abs(got - ref) - bound)}"


@pytest.mark.parametrize("name,shape,d_q,w_heads", CASES[:3])
def test_fold_then_decode_matches_up_projected_attention(cuda_device, name, shape, d_q, w_heads):
    lens = [700, 1, 333, 0]
    d, q_aug, w = _inputs(shape, d_q, w_heads, 811, lens, 700)
    scale = d_q ** -0.5
    ref = oracle.decode_up_projected(q_aug, w, d["k_cache"], d["v_cache"], d["seq_lens"], scale)
    g = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    q = ak.fold_query(q_aug.to(cuda_device), w.to(cuda_device), n_k=shape.n_k)
    ws = ak.decode_workspace(q, g["k_cache"], g["v_cache"])
    out = ak.decode(q, g["k_cache"], g["v_cache"], g["seq_lens"], scale=scale, workspace=ws)
    assert ak.workspace_status(ws) == 0
    # the decode on the folded (bf16) query: element-wise against the oracle on that same query
    q_bf16 = q.cpu()
    assert_parity(out, oracle.decode(q_bf16, d["k_cache"], d["v_cache"], d["seq_lens"], scale), f"decode {name}")
    # end to end against the pages' order (keys projected up in fp64): the folded query is rounded
    # to bf16 (2^-9 relative), which perturbs every score of a row together, like the bf16 weights
    # of the tensor-core prefill, so this comparison takes the per-vector rule
    assert_parity_prefill(out, ref, f"fold + decode {name}")


def test_fold_is_deterministic(cuda_device):
    _, q_aug, w = _inputs(wl.DIFFQKV, 192, 4, 821, [1] * 16, 1)
    qa, wd = q_aug.to(cuda_device), w.to(cuda_device)
    first = ak.fold_query(qa, wd, n_k=4)
    for _ in range(3):
        assert torch.equal(ak.fold_query(qa, wd, n_k=4), first)
