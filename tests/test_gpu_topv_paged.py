"""GPU parity of selective-V decode over paged K/V caches (K and V page pools, one block table).

Expected values: the fp64 oracle over the pools gathered into contiguous caches (index sets bit
for bit, outputs within the element-wise tolerance).  The paged call cuts the work exactly like the
contiguous one, so its indices and output must also equal, bit for bit, the contiguous selective-V
call over the gathered caches with the same capacity."""
import numpy as np
import pytest
import torch

import asymmetric_head_kv_b200 as ak
import oracle
import workloads as wl
from workloads import Shape
from parity import assert_parity

pytestmark = pytest.mark.gpu


def _to(d, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def _dims(d, shape):
    return ak.make_dims(d["q"].shape[0], shape.n_q, shape.n_k, shape.n_v, shape.d_k, shape.d_v, d["scale"])


def _paged(g, d, shape, topk, expect=0, **kw):
    t_max = g["block_table"].shape[1] * g["k_pages"].shape[1]
    ws = ak.decode_topv_workspace(_dims(d, shape), t_max, topk, g["q"].device)
    out, idx = ak.decode_topv_paged(g["q"], g["k_pages"], g["v_pages"], g["block_table"], g["seq_lens"], topk,
                                    scale=d["scale"], workspace=ws, **kw)
    assert ak.workspace_status(ws) == expect
    return out, idx


@pytest.mark.parametrize("page_size", [8, 16, 64, 120])
@pytest.mark.parametrize("name,shape", [("diffqkv", wl.DIFFQKV), ("gqa", wl.GQA_CONTROL),
                                        ("mha64", Shape(8, 8, 8, 64, 64))])
def test_paged_topv_matches_oracle_and_contiguous(cuda_device, name, shape, page_size):
    lens = [2500, 1, 0, 700, page_size, page_size + 1]
    max_blocks = -(-2501 // page_size)
    d = wl.random_paged_inputs(len(lens), max_blocks, page_size, shape, seed=901, seq_lens=lens, spare_pages=3)
    kc = oracle.gather_paged(d["k_pages"], d["block_table"], d["seq_lens"])
    vc = oracle.gather_paged(d["v_pages"], d["block_table"], d["seq_lens"])
    topk = 100
    r_out, r_idx = oracle.decode_topv(d["q"], kc, vc, d["seq_lens"], topk, d["scale"])
    g = _to(d, cuda_device)
    out, idx = _paged(g, d, shape, topk)
    assert np.array_equal(idx.cpu().numpy(), r_idx), f"{name} P={page_size}: index sets"
    assert_parity(out, r_out, f"paged top-v {name} P={page_size}")
    # the contiguous call over the gathered caches (same capacity): identical bits
    flat_out, flat_idx = ak.decode_topv(g["q"], kc.to(cuda_device), vc.to(cuda_device), g["seq_lens"], topk,
                                        scale=d["scale"])
    torch.cuda.synchronize()
    assert torch.equal(idx, flat_idx) and torch.equal(out, flat_out), "paged and contiguous top-v differ"


def test_paged_topv_full_weights_and_large_k(cuda_device):
    shape, page_size = wl.DIFFQKV, 16
    lens = [9000, 3000]
    d = wl.random_paged_inputs(2, 9000 // page_size + 1, page_size, shape, seed=911, seq_lens=lens)
    kc = oracle.gather_paged(d["k_pages"], d["block_table"], d["seq_lens"])
    vc = oracle.gather_paged(d["v_pages"], d["block_table"], d["seq_lens"])
    g = _to(d, cuda_device)
    for topk, full in ((1024, True), (4000, False)):
        r_out, r_idx = oracle.decode_topv(d["q"], kc, vc, d["seq_lens"], topk, d["scale"], full_weights=full)
        out, idx = _paged(g, d, shape, topk, full_weights=full)
        assert np.array_equal(idx.cpu().numpy(), r_idx), f"k={topk} full={full}: index sets"
        assert_parity(out, r_out, f"paged top-v k={topk} full={full}")


def test_paged_topv_units_in_rounds(cuda_device):
    """160 (batch, K head) units over 16-position pages: one part per unit, two rounds; index sets and
    outputs bit for bit those of the contiguous call over the gathered caches."""
    shape, page_size = wl.DIFFQKV, 16
    lens = [600, 37, 600, 1, 420, 50, 599, 64] * 5
    max_blocks = -(-600 // page_size)
    d = wl.random_paged_inputs(len(lens), max_blocks, page_size, shape, seed=931, seq_lens=lens)
    kc = oracle.gather_paged(d["k_pages"], d["block_table"], d["seq_lens"])
    vc = oracle.gather_paged(d["v_pages"], d["block_table"], d["seq_lens"])
    r_out, r_idx = oracle.decode_topv(d["q"], kc, vc, d["seq_lens"], 50, d["scale"])
    g = _to(d, cuda_device)
    out, idx = _paged(g, d, shape, 50)
    assert np.array_equal(idx.cpu().numpy(), r_idx), "index sets"
    assert_parity(out, r_out, "paged top-v in rounds")
    flat_out, flat_idx = ak.decode_topv(g["q"], kc.to(cuda_device), vc.to(cuda_device), g["seq_lens"], 50,
                                        scale=d["scale"])
    torch.cuda.synchronize()
    assert torch.equal(idx, flat_idx) and torch.equal(out, flat_out), "paged and contiguous top-v differ"


def test_paged_topv_bad_entry_is_flagged(cuda_device):
    """A used block-table entry past the pool: flagged DIFFQKV_ERR_DEVICE_PAGE, pool page 0 read in its
    place (every load stays in the pools); the other sequence is unaffected."""
    shape, page_size = wl.DIFFQKV, 16
    lens = [200, 200]
    d = wl.random_paged_inputs(2, 13, page_size, shape, seed=921, seq_lens=lens)
    kc = oracle.gather_paged(d["k_pages"], d["block_table"], d["seq_lens"])
    vc = oracle.gather_paged(d["v_pages"], d["block_table"], d["seq_lens"])
    r_out, r_idx = oracle.decode_topv(d["q"], kc, vc, d["seq_lens"], 32, d["scale"])
    d["block_table"][0, 3] = d["num_pages"] + 7
    g = _to(d, cuda_device)
    out, idx = _paged(g, d, shape, 32, expect=ak._capi.DEVICE_PAGE)
    assert np.array_equal(idx[1].cpu().numpy(), r_idx[1])
    assert_parity(out[1], r_out[1], "paged top-v, other sequence")


def test_paged_topv_rejects_page_sizes_off_the_swizzle_atom(cuda_device):
    shape = wl.DIFFQKV
    d = wl.random_paged_inputs(1, 20, 12, shape, seed=931, seq_lens=[100])
    g = _to(d, cuda_device)
    with pytest.raises(ak.DiffqkvError) as e:
        ak.decode_topv_paged(g["q"], g["k_pages"], g["v_pages"], g["block_table"], g["seq_lens"], 8,
                             scale=d["scale"])
    assert e.value.status == ak._capi.UNSUPPORTED
