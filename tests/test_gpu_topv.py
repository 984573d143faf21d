"""GPU parity of selective-V decode (through the C ABI) against the fp64 oracle.

Index sets must match bit-exactly (exact dot products, ties toward the lower
position); outputs within the bf16 parity tolerance."""
import numpy as np
import pytest
import torch

import asymmetric_head_kv_b200 as ak
import oracle
import workloads as wl
from workloads import Shape
from parity import assert_parity

pytestmark = pytest.mark.gpu


def _a256(x):
    return -(-x // 256) * 256


def _counter_region(batch, n_q, n_k):
    """Byte range of the counters that every completed call leaves zero (the header's layout)."""
    rows, units = batch * n_q, batch * n_k
    return 256, 256 + _a256(_a256(units * 16) + _a256(rows * 16) + rows * 2048 * 4)


def _gpu(d, topk, dev, expect=0, **kw):
    """Selective-V decode through the C ABI; the workspace's error word must read `expect`."""
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    dims = ak.make_dims(*g["q"].shape[:2], g["k_cache"].shape[2], g["v_cache"].shape[2], g["q"].shape[2],
                        g["v_cache"].shape[3], d["scale"])
    ws = ak.decode_topv_workspace(dims, g["k_cache"].shape[1], topk, dev)
    out, idx = ak.decode_topv(g["q"], g["k_cache"], g["v_cache"], g["seq_lens"], topk, scale=d["scale"],
                              workspace=ws, **kw)
    assert ak.workspace_status(ws) == expect
    return out, idx


def _check(d, topk, dev, what, **kw):
    out, idx = _gpu(d, topk, dev, **kw)
    r_out, r_idx = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], topk, d["scale"])
    got = idx.cpu().numpy()
    bad = np.argwhere((got != r_idx).any(axis=-1))
    assert bad.size == 0, f"{what}: index sets differ for (b, h) {bad[:5].tolist()}"
    assert_parity(out, r_out, what)
    return out, idx


@pytest.mark.parametrize("name,shape", [("diffqkv", wl.DIFFQKV), ("gqa", wl.GQA_CONTROL),
                                        ("paper", wl.SIGMA_1P5B_PAPER), ("mha64", Shape(8, 8, 8, 64, 64)),
                                        ("k_more_than_v", Shape(16, 8, 2, 64, 128))])
def test_ragged_shapes(cuda_device, name, shape):
    lens = [3000, 1, 100, 101, 2500]
    d = wl.random_decode_inputs(len(lens), 3000, shape, seed=301, seq_lens=lens)
    _check(d, 100, cuda_device, name)


def test_more_units_than_ctas_run_in_rounds(cuda_device):
    """40 sequences x 4 K heads = 160 (batch, K head) units: more than one CTA per SM can hold, so one
    part per unit, each CTA selecting all four rows of its unit, units taken in two rounds (ragged
    lengths, some at or below k)."""
    lens = [600, 37, 600, 1, 420, 50, 599, 64] * 5
    d = wl.random_decode_inputs(len(lens), 600, wl.DIFFQKV, seed=313, seq_lens=lens)
    _check(d, 50, cuda_device, "160 units in rounds")


@pytest.mark.parametrize("topk", [1, 2, 7, 64, 1024, 2999, 3000, 5000])
def test_topk_sizes(cuda_device, topk):
    d = wl.random_decode_inputs(2, 3000, wl.DIFFQKV, seed=302, seq_lens=[3000, 1500])
    out, idx = _check(d, topk, cuda_device, f"k={topk}")
    if topk >= 3000:   # every position kept: plain decode, indices 0..T-1 then -1
        full = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])
        assert_parity(out, full, "k >= T")
        assert idx[0, 0, :3000].tolist() == list(range(3000))
        assert torch.all(idx[1, :, 1500:] == -1)


def test_empty_rows(cuda_device):
    d = wl.random_decode_inputs(3, 200, wl.DIFFQKV, seed=303, seq_lens=[0, 200, 0])
    out, idx = _check(d, 16, cuda_device, "empty rows")
    assert torch.all(idx[0] == -1) and torch.all(out[0] == 0)


def test_exact_ties_choose_lower_positions(cuda_device):
    """Every cached key identical: all scores tie exactly; the kept set is 0..k-1
    (thousands of ambiguous positions: the radix path of the exact select)."""
    d = wl.random_decode_inputs(1, 5000, wl.DIFFQKV, seed=304)
    d["k_cache"][:] = d["k_cache"][:, :1]
    _, idx = _check(d, 1000, cuda_device, "all ties")
    assert torch.all(idx[0, :, :] == torch.arange(1000, dtype=torch.int32, device=idx.device))


def test_duplicate_rows_at_the_boundary(cuda_device):
    d = wl.random_decode_inputs(1, 4000, wl.DIFFQKV, seed=305)
    # copy a few rows many times so exact ties straddle the k-th position (pairwise path)
    for src, dsts in ((11, range(100, 4000, 400)), (500, range(7, 4000, 333)), (1234, range(2, 4000, 97))):
        for j in dsts:
            d["k_cache"][0, j] = d["k_cache"][0, src]
    for k in (5, 33, 40, 200):
        _check(d, k, cuda_device, f"dup k={k}")


def _near_tie_inputs(n_rows, seed):
    """Keys whose exact dots differ by ~2^-30 relative: fp32 scores tie, exact order does not."""
    s = wl.DIFFQKV
    d = wl.random_decode_inputs(1, n_rows, s, seed=seed)
    g = torch.Generator().manual_seed(seed)
    q = d["q"][0].float()
    q[:, 1] = 2.0 ** -30                    # tiny weight on component 1 for every head
    d["q"][0] = q.to(torch.bfloat16)
    base = d["k_cache"][0, 0].clone()
    k = base.repeat(n_rows, 1, 1)
    # component 1 takes small integer values: differences of 2^-30 .. 2^-27 in the dot
    k[:, :, 1] = torch.randint(-8, 9, (n_rows, s.n_k), generator=g).to(torch.bfloat16)
    d["k_cache"][0] = k
    return d


@pytest.mark.parametrize("n_rows,topk", [(50, 10), (3000, 700)])
def test_near_ties_ordered_by_exact_value(cuda_device, n_rows, topk):
    d = _near_tie_inputs(n_rows, 306)
    _check(d, topk, cuda_device, f"near ties {n_rows}")


def test_workspace_too_small_is_rejected(cuda_device):
    d = wl.random_decode_inputs(1, 100, wl.DIFFQKV, seed=307)
    g = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    ws = torch.empty(64, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(ak.DiffqkvError) as e:
        ak.decode_topv(g["q"], g["k_cache"], g["v_cache"], g["seq_lens"], 8, workspace=ws)
    assert e.value.status == ak._capi.WORKSPACE


def test_full_topv_workload(cuda_device):
    w = wl.TOPV_64K
    d = wl.make_decode_inputs(w, cuda_device)
    dims = ak.make_dims(w.batch, w.shape.n_q, w.shape.n_k, w.shape.n_v, w.shape.d_k, w.shape.d_v, d["scale"])
    ws = ak.decode_topv_workspace(dims, w.t_max, w.topk, cuda_device)
    out, idx = ak.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], w.topk, scale=d["scale"],
                              workspace=ws)
    assert ak.workspace_status(ws) == 0
    cpu = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    r_out, r_idx = oracle.decode_topv(cpu["q"], cpu["k_cache"], cpu["v_cache"], cpu["seq_lens"], w.topk, d["scale"])
    assert np.array_equal(idx.cpu().numpy(), r_idx)
    assert_parity(out, r_out, w.name)


@pytest.mark.parametrize("topk", [64, 1024, 4000])
def test_workspace_reuse_is_bitwise_stable(cuda_device, topk):
    """Two calls on one workspace (every counter must come back to zero) give identical bits:
    the parts of a row are added in a fixed order."""
    d = wl.random_decode_inputs(3, 6000, wl.DIFFQKV, seed=308, seq_lens=[6000, 2500, 4100])
    g = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    dims = ak.make_dims(3, 16, 4, 16, 64, 128, d["scale"])
    ws = ak.decode_topv_workspace(dims, 6000, topk, cuda_device)
    runs = []
    for _ in range(2):
        out, idx = ak.decode_topv(g["q"], g["k_cache"], g["v_cache"], g["seq_lens"], topk, scale=d["scale"],
                                  workspace=ws)
        assert ak.workspace_status(ws) == 0
        runs.append((out.clone(), idx.clone()))
    assert torch.equal(runs[0][0], runs[1][0]) and torch.equal(runs[0][1], runs[1][1])
    c0, c1 = _counter_region(3, 16, 4)
    assert torch.count_nonzero(ws[c0:c1]) == 0, "counters not returned to zero"
    r_out, r_idx = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], topk, d["scale"])
    assert np.array_equal(runs[0][1].cpu().numpy(), r_idx)
    assert_parity(runs[0][0], r_out, f"reuse k={topk}")


@pytest.mark.parametrize("name,shape,topk", [("diffqkv", wl.DIFFQKV, 100), ("diffqkv_k1", wl.DIFFQKV, 1),
                                             ("gqa", wl.GQA_CONTROL, 64), ("mha64", Shape(8, 8, 8, 64, 64), 300)])
def test_full_softmax_weights(cuda_device, name, shape, topk):
    """The pages' formula: kept rows weighted by the full-softmax alpha_j of every cached position
    (rows of 9000 positions span two filter chunks; a 200-position row keeps everything)."""
    lens = [9000, 200, 0, 4100]
    d = wl.random_decode_inputs(len(lens), 9000, shape, seed=309, seq_lens=lens)
    out, idx = _gpu(d, topk, cuda_device, full_weights=True)
    r_out, r_idx = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], topk, d["scale"],
                                      full_weights=True)
    assert np.array_equal(idx.cpu().numpy(), r_idx), f"{name}: index sets"
    assert_parity(out, r_out, f"full weights {name}")
    _, idx_renorm = _gpu(d, topk, cuda_device)
    assert torch.equal(idx, idx_renorm)  # the selection does not depend on the weighting


def test_out_of_range_lengths_are_clamped_and_flagged(cuda_device):
    """Lengths outside [0, t_max] are clamped, as in the decode, and flagged
    DIFFQKV_ERR_DEVICE_SEQLEN in the workspace's error word."""
    d = wl.random_decode_inputs(3, 800, wl.DIFFQKV, seed=310, seq_lens=[800, 300, 800])
    bad = dict(d, seq_lens=torch.tensor([900, 300, -4], dtype=torch.int32))
    out, idx = _gpu(bad, 50, cuda_device, expect=ak._capi.DEVICE_SEQLEN)
    clamped = dict(d, seq_lens=torch.tensor([800, 300, 0], dtype=torch.int32))
    r_out, r_idx = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], clamped["seq_lens"], 50, d["scale"])
    assert np.array_equal(idx.cpu().numpy(), r_idx)
    assert_parity(out, r_out, "clamped lengths")
    _gpu(d, 50, cuda_device)   # in-range lengths: nothing flagged


@pytest.mark.parametrize("topk", [1, 100, 1024])
def test_poisoned_workspace_is_never_read_before_written(cuda_device, topk):
    """Every byte of the scratch after the counters (candidate lists, ambiguous lists, kept scores,
    per-row words, per-part sums) starts as 0xFF: a kernel that read scratch this call did not
    write would change the index sets or the output.  The counters are zero again afterwards."""
    lens = [5000, 1, 2047, 0, 3000]
    d = wl.random_decode_inputs(len(lens), 5000, wl.DIFFQKV, seed=311, seq_lens=lens)
    g = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    dims = ak.make_dims(len(lens), 16, 4, 16, 64, 128, d["scale"])
    ws = ak.decode_topv_workspace(dims, 5000, topk, cuda_device)
    c0, c1 = _counter_region(len(lens), 16, 4)
    ws[c1:] = 0xFF
    out, idx = ak.decode_topv(g["q"], g["k_cache"], g["v_cache"], g["seq_lens"], topk, scale=d["scale"],
                              workspace=ws)
    assert ak.workspace_status(ws) == 0
    r_out, r_idx = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], topk, d["scale"])
    assert np.array_equal(idx.cpu().numpy(), r_idx)
    assert torch.isfinite(out.float()).all()
    assert_parity(out, r_out, f"poisoned workspace k={topk}")
    assert torch.count_nonzero(ws[c0:c1]) == 0, "counters not returned to zero"


def _candidate_lists(ws, batch, n_q, n_k, d_v, t_max):
    """Views of the workspace's candidate positions and scores ([rows][t_pad] each; the header's layout)."""
    rows, units, t_pad = batch * n_q, batch * n_k, -(-t_max // 64) * 64
    off = 256 + _a256(_a256(units * 16) + _a256(rows * 16) + rows * 2048 * 4)
    off += _a256(rows * 8 * 4) + _a256(rows * 256 * 8)
    cj = ws[off:off + rows * t_pad * 4].view(torch.int32).view(rows, t_pad)
    off += _a256(rows * t_pad * 4)
    cs = ws[off:off + rows * t_pad * 4].view(torch.float32).view(rows, t_pad)
    return cj, cs


@pytest.mark.parametrize("kind", ["normal", "outliers", "wide"])
def test_tensor_core_score_error_within_model(cuda_device, kind):
    """The scores come from tcgen05 MMAs, whose addition order and rounding the PTX documentation
    leaves open.  The selection's bound is the truncating block-addition model,
    n (1 + 1/16) 2^-23 sum|q k| per score; this measures the candidates' fp32 scores against the
    exact dot products and requires a margin of 4 below it (inputs: normal, normal with 256x
    outliers, exponents spread over 2^+-20)."""
    s = wl.DIFFQKV
    B, T, topk = 2, 6000, 300
    d = wl.random_decode_inputs(B, T, s, seed=312)
    g = torch.Generator().manual_seed(312)
    if kind != "normal":
        k = d["k_cache"].float()
        if kind == "outliers":
            k = k * torch.where(torch.rand(k.shape, generator=g) < 0.05, 256.0, 1.0)
        else:
            k = k * torch.exp2(torch.randint(-20, 21, k.shape, generator=g).float())
        d["k_cache"] = k.to(torch.bfloat16)
    gdev = {kk: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for kk, v in d.items()}
    dims = ak.make_dims(B, s.n_q, s.n_k, s.n_v, s.d_k, s.d_v, d["scale"])
    ws = ak.decode_topv_workspace(dims, T, topk, cuda_device)
    cj, cs = _candidate_lists(ws, B, s.n_q, s.n_k, s.d_v, T)
    cj.fill_(-1)
    out, idx = ak.decode_topv(gdev["q"], gdev["k_cache"], gdev["v_cache"], gdev["seq_lens"], topk,
                              scale=d["scale"], workspace=ws)
    assert ak.workspace_status(ws) == 0
    r_out, r_idx = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], topk, d["scale"])
    assert np.array_equal(idx.cpu().numpy(), r_idx)
    assert_parity(out, r_out, f"tensor-core scores, {kind}")
    q = d["q"].double().numpy()
    kc = d["k_cache"].double().numpy()
    cj_h, cs_h = cj.cpu().numpy(), cs.cpu().numpy().astype(np.float64)
    qpk, worst, checked = s.n_q // s.n_k, 0.0, 0
    for row in range(B * s.n_q):
        b, h = divmod(row, s.n_q)
        sel = cj_h[row] >= 0
        pos = cj_h[row][sel]
        krow = kc[b, pos, h // qpk]                        # [n, d_k]
        exact = krow @ q[b, h]                             # exact: 64 products of bf16 in fp64
        mag = np.abs(krow) @ np.abs(q[b, h])
        err = np.abs(cs_h[row][sel] - exact)
        model = s.d_k * (1 + 1 / 16) * 2.0 ** -23 * mag + s.d_k * 2.0 ** -126
        assert np.all(err <= model / 4), f"{kind}: row {row} error {err.max():.3e} within 4x of the model"
        rn = s.d_k * 2.0 ** -24 * mag                      # the round-to-nearest gamma_n, for the record
        worst = max(worst, float(np.max(err / np.maximum(rn, 1e-300))))
        checked += int(sel.sum())
    assert checked > 1000
    print(f"{kind}: {checked} candidate scores, worst error {worst:.3f} x the round-to-nearest bound")
