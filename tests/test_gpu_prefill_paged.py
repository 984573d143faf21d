"""GPU parity of the causal prefill over paged K/V pools (chunked prefill whose prefix sits in a
paged cache).  Pools start as NaN and only the sequences' rows are written, in pages dealt out in
random order; the result must equal the contiguous-cache prefill over the same rows bit for bit
(rows past the sequence, NaN here, must read as zeros) and the fp64 oracle within the per-vector
rule of the tensor-core prefill."""
import numpy as np
import pytest
import torch

import asymmetric_head_kv_b200 as ak
import oracle
import workloads as wl
from parity import assert_parity_prefill

pytestmark = pytest.mark.gpu


def _paged(k, v, page_size, seed, extra_blocks=2, spare_pages=3):
    """Scatter contiguous caches [B, T, heads, d] into NaN-filled pools sharing one block table."""
    B, T = k.shape[:2]
    per_seq = -(-T // page_size)
    num_pages = B * per_seq + spare_pages
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g)
    table = torch.full((B, per_seq + extra_blocks), -1, dtype=torch.int32)
    kp = torch.full((num_pages, page_size) + tuple(k.shape[2:]), float("nan")).to(torch.bfloat16)
    vp = torch.full((num_pages, page_size) + tuple(v.shape[2:]), float("nan")).to(torch.bfloat16)
    for b in range(B):
        for p in range(per_seq):
            pg = int(perm[b * per_seq + p])
            table[b, p] = pg
            rows = slice(p * page_size, min(T, (p + 1) * page_size))
            n = rows.stop - rows.start
            kp[pg, :n] = k[b, rows]
            vp[pg, :n] = v[b, rows]
    return kp, vp, table


def _case(shape, B, P0, S, page_size, seed, dev):
    d = wl.random_prefill_inputs(B, P0 + S, shape, seed=seed)
    q = d["q"][:, P0:].contiguous()
    kp, vp, table = _paged(d["k"], d["v"], page_size, seed + 1)
    g = lambda t: t.to(dev)  # noqa: E731
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    got = ak.prefill_causal_paged(g(q), g(kp), g(vp), g(table), P0, scale=d["scale"], status=status)
    ref = ak.prefill_causal_prefix(g(q), g(d["k"]), g(d["v"]), P0, scale=d["scale"])
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return d, q, got, ref


@pytest.mark.parametrize("name,shape", [("diffqkv", wl.DIFFQKV), ("gqa", wl.GQA_CONTROL)])
@pytest.mark.parametrize("page_size", [8, 16, 24, 64, 128, 256])
@pytest.mark.parametrize("P0,S", [(0, 200), (300, 77), (1000, 129)])
def test_paged_equals_contiguous(cuda_device, name, shape, page_size, P0, S):
    _, _, got, ref = _case(shape, 2, P0, S, page_size, seed=900 + P0 + page_size, dev=cuda_device)
    assert torch.isfinite(got.float()).all(), "a NaN row past the sequence reached the output"
    assert torch.equal(got, ref), f"{name} P={page_size} prefix {P0} seq {S}: paged differs from contiguous"


@pytest.mark.parametrize("name,shape", [("diffqkv", wl.DIFFQKV), ("gqa", wl.GQA_CONTROL)])
def test_paged_against_oracle(cuda_device, name, shape):
    P0, S = 700, 333
    d, q, got, _ = _case(shape, 2, P0, S, 16, seed=950, dev=cuda_device)
    ref = oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"])[:, P0:]
    assert_parity_prefill(got, ref, f"paged prefill {name}")


def test_bad_table_entries_are_flagged(cuda_device):
    d = wl.random_prefill_inputs(2, 300, wl.DIFFQKV, seed=960)
    kp, vp, table = _paged(d["k"], d["v"], 16, 961)
    table[1, 3] = kp.shape[0] + 5       # past the pool
    table[0, 0] = -7                    # negative
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = ak.prefill_causal_paged(d["q"][:, 100:].contiguous().to(cuda_device), kp.to(cuda_device),
                                  vp.to(cuda_device), table.to(cuda_device), 100, scale=d["scale"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == ak._capi.DEVICE_PAGE
    assert out.shape == (2, 200, 16, 128)
