"""GPU parity of the tcgen05 causal prefill (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import asymmetric_head_kv_b200 as ak
import oracle
import workloads as wl
from workloads import Shape
from parity import assert_parity, assert_parity_prefill

pytestmark = pytest.mark.gpu

SHAPES = {
    "diffqkv": wl.DIFFQKV,
    "gqa_control": wl.GQA_CONTROL,
    "mha64": Shape(8, 8, 8, 64, 64),
    "paper_1p5b": wl.SIGMA_1P5B_PAPER,
    "k_more_than_v": Shape(16, 8, 2, 64, 128),
    "dk128_dv64": Shape(16, 4, 16, 128, 64),
}


def _gpu(d, dev):
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    out = ak.prefill_causal(g["q"], g["k"], g["v"], scale=d["scale"])
    torch.cuda.synchronize()
    assert ak.device_status() == 0
    return out


@pytest.mark.parametrize("seq", [1, 5, 64, 127, 128, 129, 300, 1000])
def test_lengths_diffqkv(cuda_device, seq):
    d = wl.random_prefill_inputs(2, seq, wl.DIFFQKV, seed=400 + seq)
    out = _gpu(d, cuda_device)
    assert_parity_prefill(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), f"S={seq}")
    # row 0 attends to position 0 only: exactly V_0 (weight 2^0 = 1)
    assert torch.equal(out[:, 0].cpu(), d["v"][:, 0].repeat_interleave(wl.DIFFQKV.n_q // wl.DIFFQKV.n_v, dim=1))


@pytest.mark.parametrize("shape_name", ["diffqkv", "gqa"])
def test_many_sequences(cuda_device, shape_name):
    """33 sequences of 191 positions: more CTAs than the GPU holds at once in both tilings, each
    with a ragged last query tile."""
    s = wl.DIFFQKV if shape_name == "diffqkv" else wl.GQA_CONTROL
    d = wl.random_prefill_inputs(33, 191, s, seed=480)
    out = _gpu(d, cuda_device)
    assert_parity_prefill(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), f"33 x 191 {shape_name}")


@pytest.mark.parametrize("name", list(SHAPES))
def test_shapes(cuda_device, name):
    d = wl.random_prefill_inputs(2, 333, SHAPES[name], seed=410)
    out = _gpu(d, cuda_device)
    assert_parity_prefill(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), name)


@pytest.mark.parametrize("seq", [1, 5, 127, 128, 129, 255, 256, 257, 300, 600])
def test_lengths_dk128(cuda_device, seq):
    """The d_k = 128 tiling runs two 128-row query tiles per CTA over 128-position K/V tiles:
    lengths around those boundaries put the second tile partly or wholly past the end and
    give the two tiles different K/V tile counts."""
    s = wl.GQA_CONTROL
    d = wl.random_prefill_inputs(1, seq, s, seed=440 + seq)
    out = _gpu(d, cuda_device)
    assert_parity_prefill(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), f"d_k 128, S={seq}")
    assert torch.equal(out[:, 0].cpu(), d["v"][:, 0].repeat_interleave(s.n_q // s.n_v, dim=1))


def test_sharp_softmax_rescaling(cuda_device):
    """Large score growth along the sequence forces the in-TMEM output rescaling path."""
    d = wl.random_prefill_inputs(1, 700, wl.DIFFQKV, seed=420)
    ramp = torch.linspace(0.1, 6.0, 700).to(torch.bfloat16)
    d["k"] = (d["k"].float() * ramp[None, :, None, None].float()).to(torch.bfloat16)
    out = _gpu(d, cuda_device)
    assert_parity_prefill(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), "rescale")


def test_sharp_softmax_rescaling_dk128(cuda_device):
    """The same ramp on the d_k = 128 tiling (its own rescale path, one per query tile)."""
    d = wl.random_prefill_inputs(1, 700, wl.GQA_CONTROL, seed=421)
    ramp = torch.linspace(0.1, 6.0, 700).to(torch.bfloat16)
    d["k"] = (d["k"].float() * ramp[None, :, None, None].float()).to(torch.bfloat16)
    out = _gpu(d, cuda_device)
    assert_parity_prefill(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), "rescale d_k 128")


def test_prefill_rows_match_gpu_decode(cuda_device):
    """Row i of causal prefill is decode over positions 0..i (two different kernels)."""
    s = wl.DIFFQKV
    d = wl.random_prefill_inputs(1, 400, s, seed=430)
    out = _gpu(d, cuda_device)
    k = d["k"].to(cuda_device)
    v = d["v"].to(cuda_device)
    for i in (0, 63, 64, 200, 399):
        q = d["q"][:, i].contiguous().to(cuda_device)
        dec = ak.decode(q, k, v, torch.tensor([i + 1], dtype=torch.int32, device=cuda_device), scale=d["scale"])
        ref = oracle.decode(d["q"][:, i].contiguous(), d["k"], d["v"], torch.tensor([i + 1], dtype=torch.int32),
                            d["scale"])
        assert_parity_prefill(out[:, i], ref, f"row {i}")
        assert_parity(dec, ref, f"decode {i}")


def _full_check_rows(w, n_heads_full):
    """Every query position of one (batch, head) per covered K head, plus every head of both
    sequences on every 64th position (and the last one).  The covered heads are spread over the K
    heads (and so over the tile scheduler's (batch, head) order) and alternate between sequences."""
    s = w.shape
    qpk = s.n_q // s.n_k
    stride = max(1, s.n_k // n_heads_full)
    full = []
    for i, g in enumerate(range(0, s.n_k, stride)):
        h = g * qpk + (i % qpk)          # a different member of each group, so V heads vary too
        full.append((i % w.batch, h))
    rows = [(b, pos, h) for b, h in full for pos in range(w.seq)]
    strided = sorted(set(list(range(0, w.seq, 64)) + [w.seq - 1]))
    rows += [(b, pos, h) for b in range(w.batch) for pos in strided for h in range(s.n_q)
             if (b, h) not in full]
    return full, rows


@pytest.mark.parametrize("w,n_heads_full", [(wl.PREFILL_8K, 4), (wl.PREFILL_8K_GQA, 4)], ids=lambda x: getattr(x, "name", str(x)))
def test_full_prefill_every_row_of_covered_heads(cuda_device, w, n_heads_full):
    """The full 2 x 8192 causal prefill: all 8192 query positions of one (batch, head) per K head
    (for the DiffQKV shape; four spread K heads of the 16 of the GQA control), and every head on
    every 64th position, against the fp64 oracle."""
    d = wl.make_prefill_inputs(w, cuda_device)
    out = ak.prefill_causal(d["q"], d["k"], d["v"], scale=d["scale"])
    torch.cuda.synchronize()
    assert ak.device_status() == 0
    assert torch.isfinite(out.float()).all()
    full, rows = _full_check_rows(w, n_heads_full)
    assert len(full) == n_heads_full
    ref = oracle.prefill_causal(d["q"].cpu(), d["k"].cpu(), d["v"].cpu(), d["scale"], rows=rows)
    idx = torch.tensor(rows)
    got = out[idx[:, 0], idx[:, 1], idx[:, 2]]
    assert_parity_prefill(got, ref, w.name)


def _prefix_expected(q, k, v, scale, P):
    """Rows P.. of a causal prefill over the whole P+S sequence (rows are independent, so the
    prefix rows' queries can be anything: zeros here)."""
    B, S, n_q, d_k = q.shape
    q_full = torch.cat([torch.zeros(B, P, n_q, d_k, dtype=q.dtype), q], dim=1)
    return oracle.prefill_causal(q_full, k, v, scale)[:, P:]


@pytest.mark.parametrize("shape_name", ["diffqkv", "gqa_control"])
@pytest.mark.parametrize("P,S", [(1, 5), (64, 130), (100, 257), (128, 1), (300, 300)])
def test_prefix_prefill(cuda_device, shape_name, P, S):
    """Chunked prefill: S new rows at positions P.. attend over the P cached and the new keys
    (both tilings; prefixes and lengths straddle the 64- and 128-position tile edges)."""
    shape = SHAPES[shape_name]
    d = wl.random_prefill_inputs(2, P + S, shape, seed=450 + P + S)
    q = d["q"][:, P:].contiguous()
    g = {k: d[k].to(cuda_device) for k in ("k", "v")}
    out = ak.prefill_causal_prefix(q.to(cuda_device), g["k"], g["v"], P, scale=d["scale"])
    torch.cuda.synchronize()
    assert ak.device_status() == 0
    assert_parity_prefill(out, _prefix_expected(q, d["k"], d["v"], d["scale"], P), f"{shape_name} P={P} S={S}")


def test_prefix_zero_is_plain_prefill_and_chunks_compose(cuda_device):
    s = wl.DIFFQKV
    d = wl.random_prefill_inputs(1, 600, s, seed=460)
    g = {k: d[k].to(cuda_device) for k in ("q", "k", "v")}
    whole = ak.prefill_causal(g["q"], g["k"], g["v"], scale=d["scale"])
    zero = ak.prefill_causal_prefix(g["q"], g["k"], g["v"], 0, scale=d["scale"])
    torch.cuda.synchronize()
    assert torch.equal(whole, zero)
    # three chunks of 200 rows, each over its prefix, equal the whole prefill
    parts = [ak.prefill_causal_prefix(g["q"][:, c:c + 200].contiguous(), g["k"][:, :c + 200].contiguous(),
                                      g["v"][:, :c + 200].contiguous(), c, scale=d["scale"]) for c in (0, 200, 400)]
    torch.cuda.synchronize()
    assert ak.device_status() == 0
    ref = oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"])
    assert_parity_prefill(torch.cat(parts, dim=1), ref, "chunked prefill")


def test_prefill_reports_into_the_callers_status_word(cuda_device):
    """diffqkv_prefill_causal_ex: the call's device-side errors go to the word the caller passes,
    not to the per-device word (a clean call leaves both at zero and computes the same bits)."""
    d = wl.random_prefill_inputs(1, 200, wl.DIFFQKV, seed=470)
    g = {k: d[k].to(cuda_device) for k in ("q", "k", "v")}
    word = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = ak.prefill_causal(g["q"], g["k"], g["v"], scale=d["scale"], status=word)
    plain = ak.prefill_causal(g["q"], g["k"], g["v"], scale=d["scale"])
    torch.cuda.synchronize()
    assert int(word.item()) == 0 and ak.device_status() == 0
    assert torch.equal(out, plain)
    assert_parity_prefill(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), "prefill with status word")
