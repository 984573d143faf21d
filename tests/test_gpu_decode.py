"""GPU parity of the split/combine decode (through the C ABI) against the fp64 oracle."""
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
    "mqa": Shape(16, 1, 1, 128, 64),
    "paper_1p5b": wl.SIGMA_1P5B_PAPER,
    "k_more_than_v": Shape(16, 8, 2, 64, 128),
    "uneven_v_span": Shape(24, 12, 8, 64, 128),
    "qpk16": Shape(16, 1, 16, 64, 128),
}


def _run(d, dev, expect=0, **kw):
    """Decode through the C ABI; the call's workspace error word must read `expect`."""
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    ws = kw.pop("workspace", None)
    if ws is None:
        ws = ak.decode_workspace(g["q"], g["k_cache"], g["v_cache"])
    out = ak.decode(g["q"], g["k_cache"], g["v_cache"], g["seq_lens"], scale=d["scale"], workspace=ws, **kw)
    assert ak.workspace_status(ws) == expect
    return out


def _oracle(d, **kw):
    return oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"], **kw)


def test_small_workload_full(cuda_device):
    d = wl.make_decode_inputs(wl.DECODE_SMALL, "cpu")
    out = _run(d, cuda_device)
    assert_parity(out, _oracle(d), "decode B=1 T=512")


@pytest.mark.parametrize("name", list(SHAPES))
def test_shapes_ragged(cuda_device, name):
    shape = SHAPES[name]
    lens = [1, 2, 17, 63, 64, 65, 300, 1000]
    d = wl.random_decode_inputs(len(lens), 1000, shape, seed=101, seq_lens=lens)
    out = _run(d, cuda_device)
    assert_parity(out, _oracle(d), name)


def test_many_short_sequences(cuda_device):
    """96 sequences x 4 K heads = 384 (batch, K head) units, more than the CTAs, with ragged lengths
    from 0 to 700 (empty rows, single positions, tile edges)."""
    g = torch.Generator().manual_seed(109)
    lens = torch.randint(0, 701, (96,), generator=g).tolist()
    lens[:6] = [0, 1, 47, 48, 49, 700]
    d = wl.random_decode_inputs(len(lens), 700, wl.DIFFQKV, seed=109, seq_lens=lens)
    out = _run(d, cuda_device)
    assert_parity(out, _oracle(d), "decode 96 short sequences")


@pytest.mark.parametrize("grid", [1, 2, 3, 7, 64, 148, 333, 2048])
def test_split_points_do_not_change_result(cuda_device, grid):
    """Forcing the split-kernel grid moves every split boundary; the combined result must not move."""
    d = wl.random_decode_inputs(3, 2000, wl.DIFFQKV, seed=102, seq_lens=[2000, 5, 1311])
    ref = _oracle(d)
    out = _run(d, cuda_device, tuning={"grid_ctas": grid, "stages": 0, "ctas_per_sm": 0})
    assert_parity(out, ref, f"grid={grid}")


@pytest.mark.parametrize("stages", [2, 3, 4, 5, 8])
def test_pipeline_depth(cuda_device, stages):
    d = wl.random_decode_inputs(2, 3000, wl.DIFFQKV, seed=103, seq_lens=[3000, 1777])
    tuning = {"grid_ctas": 0, "stages": stages, "ctas_per_sm": 0}
    dims = ak.make_dims(2, 16, 4, 16, 64, 128, 0.125)
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    try:
        ak.decode_plan(dims, 3000, 3000, sms, tuning)
    except ak.DiffqkvError as e:
        # a ring that does not fit in 227 KiB of shared memory is rejected before launch
        assert e.status == ak._capi.UNSUPPORTED
        with pytest.raises(ak.DiffqkvError) as e2:
            _run(d, cuda_device, tuning=tuning)
        assert e2.value.status == ak._capi.UNSUPPORTED
        return
    out = _run(d, cuda_device, tuning=tuning)
    assert_parity(out, _oracle(d), f"stages={stages}")


def test_empty_and_out_of_range_lengths(cuda_device):
    d = wl.random_decode_inputs(4, 100, wl.DIFFQKV, seed=104, seq_lens=[0, 100, 0, 7])
    out = _run(d, cuda_device)
    assert torch.all(out[0] == 0) and torch.all(out[2] == 0)
    assert_parity(out, _oracle(d), "empty rows")
    # a negative or too-long length is clamped and flagged in the workspace's error word
    bad = dict(d, seq_lens=torch.tensor([-3, 100, 150, 7], dtype=torch.int32))
    out = _run(bad, cuda_device, expect=ak._capi.DEVICE_SEQLEN)
    clamped = dict(d, seq_lens=torch.tensor([0, 100, 100, 7], dtype=torch.int32))
    assert_parity(out, _oracle(clamped), "clamped lengths")


def test_workspace_reuse_across_shapes(cuda_device):
    """Counters are left zeroed by every call, so one workspace serves many calls."""
    big = wl.DecodeWorkload("ws", wl.DIFFQKV, 8, 4096, seed=105)
    dims = ak.make_dims(8, 16, 4, 16, 64, 128, 0.125)
    ws = ak.decode_workspace(dims, device=cuda_device)
    for lens in ([4096] * 8, [1, 4096, 2, 3000, 17, 0, 4095, 64], [33] * 8):
        d = wl.make_decode_inputs(big, "cpu")
        d["seq_lens"] = torch.tensor(lens, dtype=torch.int32)
        out = _run(d, cuda_device, workspace=ws)
        assert_parity(out, _oracle(d), f"lens={lens[:3]}")
    # the per-unit counters (after a 256-byte header, one uint32 per (batch, K head)) are zero again,
    # and so is the header (its first word is the error word, read and cleared by _run)
    assert torch.count_nonzero(ws[:256 + 8 * 4 * 4]) == 0


def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    ak.selftest_wait_timeout(2_000_000)   # 2 ms wait on a barrier nothing signals
    assert ak.device_status() == ak._capi.DEVICE_TIMEOUT
    assert ak.device_status() == 0         # read-and-clear
    d = wl.make_decode_inputs(wl.DECODE_SMALL, "cpu")
    assert_parity(_run(d, cuda_device), _oracle(d), "after timeout")


# ---------------------------------------------------------------- full-size workloads
@pytest.mark.parametrize("w", [wl.DECODE_32K, wl.DECODE_32K_GQA], ids=lambda w: w.name)
def test_full_decode_32k(cuda_device, w):
    d = wl.make_decode_inputs(w, cuda_device)
    ws = ak.decode_workspace(d["q"], d["k_cache"], d["v_cache"])
    out = ak.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], scale=d["scale"], workspace=ws)
    assert ak.workspace_status(ws) == 0
    ref = oracle.decode(d["q"].cpu(), d["k_cache"].cpu(), d["v_cache"].cpu(), d["seq_lens"].cpu(), d["scale"])
    assert_parity(out, ref, w.name)


@pytest.mark.parametrize("w", [wl.DECODE_RAGGED, wl.DECODE_RAGGED_GQA], ids=lambda w: w.name)
def test_full_decode_ragged(cuda_device, w):
    d = wl.make_decode_inputs(w, cuda_device)
    ws = ak.decode_workspace(d["q"], d["k_cache"], d["v_cache"])
    out = ak.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], scale=d["scale"],
                    max_seq_len=int(d["seq_lens"].max()), workspace=ws)
    assert ak.workspace_status(ws) == 0
    ref = oracle.decode(d["q"].cpu(), d["k_cache"].cpu(), d["v_cache"].cpu(), d["seq_lens"].cpu(), d["scale"])
    assert_parity(out, ref, w.name)


def test_decode_from_host_matches_device_path(cuda_device):
    d = wl.make_decode_inputs(wl.DecodeWorkload("e2e", wl.DIFFQKV, 4, 2048, seed=106), "cpu")
    host = {k: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    out_host = torch.empty((4, 16, 128), dtype=torch.bfloat16).pin_memory()
    dev = {k: torch.empty_like(host[k], device=cuda_device) for k in ("q", "k_cache", "v_cache", "seq_lens")}
    dev["out"] = torch.empty((4, 16, 128), dtype=torch.bfloat16, device=cuda_device)
    dev["workspace"] = ak.decode_workspace(ak.make_dims(4, 16, 4, 16, 64, 128, 0.125), device=cuda_device)
    ak.decode_from_host(host["q"], host["k_cache"], host["v_cache"], host["seq_lens"], out_host, dev,
                        scale=d["scale"])
    torch.cuda.synchronize()
    ref_dev = _run(d, cuda_device)
    assert torch.equal(out_host, ref_dev.cpu())
    assert_parity(out_host, _oracle(d), "from host")


def test_error_words_are_per_workspace(cuda_device):
    """Two decodes on two streams, each with its own workspace: the one given out-of-range lengths
    reports DIFFQKV_ERR_DEVICE_SEQLEN in its workspace, the other reports nothing, and reading one
    word clears neither the other nor the per-device word."""
    good = wl.random_decode_inputs(2, 500, wl.DIFFQKV, seed=107, seq_lens=[500, 3])
    bad = dict(good, seq_lens=torch.tensor([600, -1], dtype=torch.int32))
    gg = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in good.items()}
    gb = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in bad.items()}
    ws_good, ws_bad = (ak.decode_workspace(gg["q"], gg["k_cache"], gg["v_cache"]) for _ in range(2))
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    out_b = ak.decode(gb["q"], gb["k_cache"], gb["v_cache"], gb["seq_lens"], scale=good["scale"],
                      workspace=ws_bad, stream=s1)
    out_g = ak.decode(gg["q"], gg["k_cache"], gg["v_cache"], gg["seq_lens"], scale=good["scale"],
                      workspace=ws_good, stream=s2)
    torch.cuda.synchronize()
    assert ak.workspace_status(ws_good, stream=s2) == 0
    assert ak.device_status() == 0
    assert ak.workspace_status(ws_bad, stream=s1) == ak._capi.DEVICE_SEQLEN
    assert ak.workspace_status(ws_bad, stream=s1) == 0     # read-and-clear of that word only
    assert_parity(out_g, _oracle(good), "good stream")
    clamped = dict(good, seq_lens=torch.tensor([500, 0], dtype=torch.int32))
    assert_parity(out_b, _oracle(clamped), "bad stream, clamped")


@pytest.mark.parametrize("grid", [0, 7, 2048])
def test_poisoned_partials_are_never_read_before_written(cuda_device, grid):
    """Every byte of the split-partial region starts as 0xFF (a NaN pattern): a combine that read a
    partial no CTA of this call wrote would turn the output NaN or wrong."""
    lens = [2000, 5, 1311, 0, 48, 49]
    d = wl.random_decode_inputs(len(lens), 2000, wl.DIFFQKV, seed=108, seq_lens=lens)
    g = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    ws = ak.decode_workspace(g["q"], g["k_cache"], g["v_cache"])
    counters_end = 256 + -(-len(lens) * wl.DIFFQKV.n_k * 4 // 256) * 256
    ws[counters_end:] = 0xFF
    tuning = {"grid_ctas": grid, "stages": 0, "ctas_per_sm": 0} if grid else None
    out = _run(d, cuda_device, workspace=ws, tuning=tuning)
    assert torch.isfinite(out.float()).all()
    assert_parity(out, _oracle(d), f"poisoned partials, grid {grid}")
