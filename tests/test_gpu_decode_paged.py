"""GPU parity of decode over paged K/V caches (separate K and V page pools, one block table).

Expected values: the fp64 oracle decode over the pools gathered into contiguous caches.  The
paged call cuts the work exactly like the contiguous one, so its output must also equal, bit for
bit, the contiguous decode over the gathered caches with the same capacity."""
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


def _paged(g, scale, expect=0, **kw):
    """Paged decode through the C ABI; the workspace's error word must read `expect`."""
    B, n_q, d_k = g["q"].shape
    dims = ak.make_dims(B, n_q, g["k_pages"].shape[2], g["v_pages"].shape[2], d_k, g["v_pages"].shape[3], scale)
    ws = ak.decode_workspace(dims, device=g["q"].device)
    out = ak.decode_paged(g["q"], g["k_pages"], g["v_pages"], g["block_table"], g["seq_lens"], scale=scale,
                          workspace=ws, **kw)
    assert ak.workspace_status(ws) == expect
    return out


def _gathered(d):
    return (oracle.gather_paged(d["k_pages"], d["block_table"], d["seq_lens"]),
            oracle.gather_paged(d["v_pages"], d["block_table"], d["seq_lens"]))


SHAPES = {
    "diffqkv": wl.DIFFQKV,
    "gqa_control": wl.GQA_CONTROL,
    "mha64": Shape(8, 8, 8, 64, 64),
    "straddling_v_heads": Shape(24, 12, 8, 64, 128),
}


@pytest.mark.parametrize("page_size", [16, 5, 64, 256])
@pytest.mark.parametrize("name", list(SHAPES))
def test_paged_matches_oracle(cuda_device, name, page_size):
    shape = SHAPES[name]
    lens = [0, 1, 333, 1000, 64, page_size, page_size + 1]
    max_blocks = -(-1001 // page_size)
    d = wl.random_paged_inputs(len(lens), max_blocks, page_size, shape, seed=601, seq_lens=lens, spare_pages=3)
    ref = oracle.decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], d["scale"])
    g = _to(d, cuda_device)
    out = _paged(g, d["scale"])
    assert_parity(out, ref, f"paged {name} P={page_size}")
    kc, vc = _gathered(d)
    flat = ak.decode(g["q"], kc.to(cuda_device), vc.to(cuda_device), g["seq_lens"], scale=d["scale"])
    assert torch.equal(out, flat), "paged and contiguous decode differ"


def test_paged_mid_size_against_contiguous(cuda_device):
    """4 x 8192 positions in 16-position pages dealt out in random order: every output equals the
    contiguous decode bit for bit, and sampled rows match the oracle."""
    shape, page_size, T = wl.DIFFQKV, 16, 8192
    d = wl.random_paged_inputs(4, T // page_size + 1, page_size, shape, seed=611, seq_lens=[T, T - 5, 4097, 16])
    g = _to(d, cuda_device)
    out = _paged(g, d["scale"])
    kc, vc = _gathered(d)
    flat = ak.decode(g["q"], kc.to(cuda_device), vc.to(cuda_device), g["seq_lens"], scale=d["scale"])
    torch.cuda.synchronize()
    assert torch.equal(out, flat)
    rows = [(0, 0), (0, 15), (1, 7), (2, 3), (3, 12)]
    ref = oracle.decode(d["q"], kc, vc, d["seq_lens"], d["scale"], rows=rows)
    assert_parity(torch.stack([out[b, h] for b, h in rows]), ref, "paged 4 x 8192 sampled rows")


@pytest.mark.parametrize("page_size", [16, 7])
def test_paged_append(cuda_device, page_size):
    """Append mode: the new rows land in row p % P of page table[b][p // P]; output attends over p + 1."""
    shape = wl.DIFFQKV
    lens = [0, 15, 16, 100, 2 * page_size - 1]
    max_blocks = -(-(max(lens) + 1) // page_size)
    d = wl.random_paged_inputs(len(lens), max_blocks, page_size, shape, seed=621, seq_lens=lens, spare_pages=2)
    gen = torch.Generator().manual_seed(622)
    k_new = torch.randn(len(lens), shape.n_k, shape.d_k, generator=gen).to(torch.bfloat16)
    v_new = torch.randn(len(lens), shape.n_v, shape.d_v, generator=gen).to(torch.bfloat16)
    k_after, v_after = d["k_pages"].clone(), d["v_pages"].clone()
    for b, p in enumerate(lens):
        page = int(d["block_table"][b, p // page_size])
        k_after[page, p % page_size] = k_new[b]
        v_after[page, p % page_size] = v_new[b]
    new_lens = d["seq_lens"] + 1
    ref = oracle.decode_paged(d["q"], k_after, v_after, d["block_table"], new_lens, d["scale"])
    g = _to(d, cuda_device)
    out = _paged(g, d["scale"], k_new=k_new.to(cuda_device), v_new=v_new.to(cuda_device))
    assert torch.equal(g["k_pages"].cpu(), k_after) and torch.equal(g["v_pages"].cpu(), v_after)
    assert_parity(out, ref, f"paged append P={page_size}")


def test_bad_page_entry_is_flagged(cuda_device):
    """A used block-table entry past the pool: flagged DIFFQKV_ERR_DEVICE_PAGE, page 0 read in its place,
    nothing appended into it; the other sequences are unaffected."""
    shape, page_size = wl.DIFFQKV, 16
    lens = [40, 40]
    d = wl.random_paged_inputs(2, 4, page_size, shape, seed=631, seq_lens=lens)
    ref = oracle.decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], d["scale"])
    d["block_table"][0, 1] = d["num_pages"] + 5
    g = _to(d, cuda_device)
    out = _paged(g, d["scale"], expect=ak._capi.DEVICE_PAGE)
    assert_parity(out[1:], ref[1:], "paged, other sequence")
    # append into a position whose page entry is bad: nothing written anywhere
    d["block_table"][0, 1] = -3
    g = _to(d, cuda_device)
    kn = torch.ones(2, shape.n_k, shape.d_k, dtype=torch.bfloat16, device=cuda_device)
    vn = torch.ones(2, shape.n_v, shape.d_v, dtype=torch.bfloat16, device=cuda_device)
    g["seq_lens"][0] = 20  # position 20 lives in logical page 1
    before = g["k_pages"].clone()
    _paged(g, d["scale"], expect=ak._capi.DEVICE_PAGE, k_new=kn, v_new=vn)
    page1 = int(d["block_table"][1, 40 // page_size])
    changed = (g["k_pages"] != before).flatten(1).any(1).nonzero().flatten().tolist()
    assert changed == [page1]  # only sequence 1's append
