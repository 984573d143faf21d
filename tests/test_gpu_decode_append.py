"""GPU parity of the decode step with the KV-cache append fused in.

Expected values: the fp64 oracle decode over a CPU copy of the caches with the
new K/V rows placed at position seq_lens[b], attending over seq_lens[b] + 1
positions; the device caches must equal that copy bit for bit."""
import pytest
import torch

import asymmetric_head_kv_b200 as ak
import oracle
import workloads as wl
from workloads import Shape
from parity import assert_parity

pytestmark = pytest.mark.gpu


def _new_rows(shape, batch, seed):
    g = torch.Generator().manual_seed(seed)
    k_new = torch.randn(batch, shape.n_k, shape.d_k, generator=g).to(torch.bfloat16)
    v_new = torch.randn(batch, shape.n_v, shape.d_v, generator=g).to(torch.bfloat16)
    return k_new, v_new


def _expected(d, k_new, v_new, t_max):
    """Caches after the append, and the oracle output over the appended positions."""
    k_after, v_after = d["k_cache"].clone(), d["v_cache"].clone()
    lens = d["seq_lens"].tolist()
    for b, p in enumerate(lens):
        if 0 <= p < t_max:
            k_after[b, p] = k_new[b]
            v_after[b, p] = v_new[b]
    new_lens = torch.tensor([min(max(p, 0) + 1, t_max) if p < t_max else t_max for p in lens], dtype=torch.int32)
    out = oracle.decode(d["q"], k_after, v_after, new_lens, d["scale"])
    return k_after, v_after, out


def _run(d, k_new, v_new, dev, expect=0):
    """The fused append through the C ABI; the workspace's error word must read `expect`."""
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    kn, vn = k_new.to(dev), v_new.to(dev)
    ws = ak.decode_workspace(g["q"], g["k_cache"], g["v_cache"])
    out = ak.decode_append(g["q"], kn, vn, g["k_cache"], g["v_cache"], g["seq_lens"], scale=d["scale"],
                           workspace=ws)
    assert ak.workspace_status(ws) == expect
    return out, g["k_cache"], g["v_cache"]


SHAPES = {
    "diffqkv": wl.DIFFQKV,
    "gqa_control": wl.GQA_CONTROL,
    "mha64": Shape(8, 8, 8, 64, 64),
    "k_more_than_v": Shape(16, 8, 2, 64, 128),
    "straddling_v_heads": Shape(24, 12, 8, 64, 128),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_append_matches_oracle(cuda_device, name):
    shape = SHAPES[name]
    t_max = 700
    lens = [0, 1, 333, 699, 64, 65]
    d = wl.random_decode_inputs(len(lens), t_max, shape, seed=501, seq_lens=lens)
    k_new, v_new = _new_rows(shape, len(lens), 502)
    k_after, v_after, ref = _expected(d, k_new, v_new, t_max)
    out, kc, vc = _run(d, k_new, v_new, cuda_device)
    assert torch.equal(kc.cpu(), k_after) and torch.equal(vc.cpu(), v_after), f"{name}: cache contents"
    assert_parity(out, ref, f"append {name}")
    # an empty cache attends to the new token alone: exactly its V row
    vh = torch.arange(shape.n_q) // (shape.n_q // shape.n_v)
    assert torch.equal(out[0].cpu(), v_new[0, vh])


def test_append_consecutive_steps(cuda_device):
    """Three generation steps on one cache, advancing seq_lens between calls."""
    shape, t_max = wl.DIFFQKV, 2000
    lens = [1500, 7, 0]
    d = wl.random_decode_inputs(len(lens), t_max, shape, seed=511, seq_lens=lens)
    g = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    k_cpu, v_cpu = d["k_cache"].clone(), d["v_cache"].clone()
    ws = ak.decode_workspace(g["q"], g["k_cache"], g["v_cache"])
    for step in range(3):
        k_new, v_new = _new_rows(shape, len(lens), 520 + step)
        q = torch.randn(len(lens), shape.n_q, shape.d_k, generator=torch.Generator().manual_seed(530 + step))
        q = q.to(torch.bfloat16)
        cur = g["seq_lens"].cpu()
        out = ak.decode_append(q.to(cuda_device), k_new.to(cuda_device), v_new.to(cuda_device), g["k_cache"],
                               g["v_cache"], g["seq_lens"], scale=d["scale"], workspace=ws)
        assert ak.workspace_status(ws) == 0
        for b, p in enumerate(cur.tolist()):
            k_cpu[b, p] = k_new[b]
            v_cpu[b, p] = v_new[b]
        ref = oracle.decode(q, k_cpu, v_cpu, cur + 1, d["scale"])
        assert_parity(out, ref, f"step {step}")
        g["seq_lens"] += 1
    assert torch.equal(g["k_cache"].cpu(), k_cpu) and torch.equal(g["v_cache"].cpu(), v_cpu)


def test_append_full_cache_is_flagged(cuda_device):
    """No free slot (seq_len == t_max): nothing is written, the step attends over the cache, and the
    workspace's error word reports DIFFQKV_ERR_DEVICE_SEQLEN."""
    shape, t_max = wl.DIFFQKV, 300
    lens = [300, 120]
    d = wl.random_decode_inputs(len(lens), t_max, shape, seed=541, seq_lens=lens)
    k_new, v_new = _new_rows(shape, len(lens), 542)
    k_after, v_after, ref = _expected(d, k_new, v_new, t_max)
    out, kc, vc = _run(d, k_new, v_new, cuda_device, expect=ak._capi.DEVICE_SEQLEN)
    assert torch.equal(kc.cpu(), k_after) and torch.equal(vc.cpu(), v_after)
    assert torch.equal(kc.cpu()[0], d["k_cache"][0])  # the full row is untouched
    assert_parity(out, ref, "full cache")
