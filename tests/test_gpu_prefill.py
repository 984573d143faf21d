"""GPU parity of the tcgen05 causal prefill (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import asymmetric_head_kv_b200 as ak
import oracle
import workloads as wl
from workloads import Shape
from parity import assert_parity

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
    assert_parity(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), f"S={seq}")
    # row 0 attends to position 0 only: exactly V_0 (weight 2^0 = 1)
    assert torch.equal(out[:, 0].cpu(), d["v"][:, 0].repeat_interleave(wl.DIFFQKV.n_q // wl.DIFFQKV.n_v, dim=1))


@pytest.mark.parametrize("name", list(SHAPES))
def test_shapes(cuda_device, name):
    d = wl.random_prefill_inputs(2, 333, SHAPES[name], seed=410)
    out = _gpu(d, cuda_device)
    assert_parity(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), name)


@pytest.mark.parametrize("seq", [1, 5, 127, 128, 129, 255, 256, 257, 300, 600])
def test_lengths_dk128(cuda_device, seq):
    """The d_k = 128 tiling runs two 128-row query tiles per CTA over 128-position K/V tiles:
    lengths around those boundaries put the second tile partly or wholly past the end and
    give the two tiles different K/V tile counts."""
    s = wl.GQA_CONTROL
    d = wl.random_prefill_inputs(1, seq, s, seed=440 + seq)
    out = _gpu(d, cuda_device)
    assert_parity(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), f"d_k 128, S={seq}")
    assert torch.equal(out[:, 0].cpu(), d["v"][:, 0].repeat_interleave(s.n_q // s.n_v, dim=1))


def test_sharp_softmax_rescaling(cuda_device):
    """Large score growth along the sequence forces the in-TMEM output rescaling path."""
    d = wl.random_prefill_inputs(1, 700, wl.DIFFQKV, seed=420)
    ramp = torch.linspace(0.1, 6.0, 700).to(torch.bfloat16)
    d["k"] = (d["k"].float() * ramp[None, :, None, None].float()).to(torch.bfloat16)
    out = _gpu(d, cuda_device)
    assert_parity(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), "rescale")


def test_sharp_softmax_rescaling_dk128(cuda_device):
    """The same ramp on the d_k = 128 tiling (its own rescale path, one per query tile)."""
    d = wl.random_prefill_inputs(1, 700, wl.GQA_CONTROL, seed=421)
    ramp = torch.linspace(0.1, 6.0, 700).to(torch.bfloat16)
    d["k"] = (d["k"].float() * ramp[None, :, None, None].float()).to(torch.bfloat16)
    out = _gpu(d, cuda_device)
    assert_parity(out, oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"]), "rescale d_k 128")


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
        assert_parity(out[:, i], ref, f"row {i}")
        assert_parity(dec, ref, f"decode {i}")


def _sample_rows(B, S, n_q, seed):
    rng = np.random.default_rng(seed)
    pos = sorted(set([0, 1, 2, 63, 64, 65, 127, 128, 129, 1000, S // 2 - 1, S // 2, S - 2, S - 1] +
                     rng.integers(0, S, 16).tolist()))
    return [(b, i, h) for b in range(B) for i in pos for h in range(n_q)]


@pytest.mark.parametrize("w", [wl.PREFILL_8K, wl.PREFILL_8K_GQA], ids=lambda w: w.name)
def test_full_prefill_sampled_rows(cuda_device, w):
    d = wl.make_prefill_inputs(w, cuda_device)
    out = ak.prefill_causal(d["q"], d["k"], d["v"], scale=d["scale"])
    torch.cuda.synchronize()
    assert ak.device_status() == 0
    assert torch.isfinite(out.float()).all()
    rows = _sample_rows(w.batch, w.seq, w.shape.n_q, 440)
    ref = oracle.prefill_causal(d["q"].cpu(), d["k"].cpu(), d["v"].cpu(), d["scale"], rows=rows)
    idx = torch.tensor(rows)
    got = out[idx[:, 0], idx[:, 1], idx[:, 2]]
    assert_parity(got, ref, w.name)


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
    assert_parity(out, _prefix_expected(q, d["k"], d["v"], d["scale"], P), f"{shape_name} P={P} S={S}")


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
    assert_parity(torch.cat(parts, dim=1), ref, "chunked prefill")
