"""Edge shapes of every kernel run through the checked build (device-side index checks on).

Run as a script with DIFFQKV_BOUNDS_CHECK=1 by tests/test_gpu_checked_build.py: every call must
match the fp64 oracle and leave every status word at DIFFQKV_OK (no index check fired).  Prints
one line per case and "all cases ok" at the end."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import asymmetric_head_kv_b200 as ak  # noqa: E402
from asymmetric_head_kv_b200 import _capi  # noqa: E402
import oracle  # noqa: E402
import workloads as wl  # noqa: E402
from parity import assert_parity, assert_parity_gemm, assert_parity_prefill  # noqa: E402


def to(d, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def main():
    assert _capi.CHECKED and _capi.LIB_PATH.endswith("libdiffqkv_checked.so"), "not the checked build"
    dev = torch.device("cuda", 0)
    s = wl.DIFFQKV
    # decode: lengths around the 48-position tile and tiny contexts, plus the fused append
    lens = [1, 2, 17, 47, 48, 49, 63, 65, 0]
    d = wl.random_decode_inputs(len(lens), 130, s, seed=71, seq_lens=lens)
    g = to(d, dev)
    ws = ak.decode_workspace(g["q"], g["k_cache"], g["v_cache"])
    out = ak.decode(g["q"], g["k_cache"], g["v_cache"], g["seq_lens"], scale=d["scale"], workspace=ws)
    assert ak.workspace_status(ws) == 0
    assert_parity(out, oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"]), "checked decode")
    kn = torch.randn(len(lens), s.n_k, s.d_k, generator=torch.Generator().manual_seed(72)).to(torch.bfloat16)
    vn = torch.randn(len(lens), s.n_v, s.d_v, generator=torch.Generator().manual_seed(73)).to(torch.bfloat16)
    ak.decode_append(g["q"], kn.to(dev), vn.to(dev), g["k_cache"], g["v_cache"], g["seq_lens"], scale=d["scale"],
                     workspace=ws)
    assert ak.workspace_status(ws) == 0
    print("decode and append ok")
    # allocation-free decode
    out = ak.decode_noalloc(g["q"], g["k_cache"], g["v_cache"], g["seq_lens"], scale=d["scale"])
    torch.cuda.synchronize()
    assert ak.device_status() == 0
    print("allocation-free decode ok")
    # paged decode and paged selective V (8-position pages)
    p = wl.random_paged_inputs(3, 40, 8, s, seed=74, seq_lens=[1, 121, 300])
    gp = to(p, dev)
    pws = ak.decode_workspace(ak.make_dims(3, 16, 4, 16, 64, 128, p["scale"]), device=dev)
    out = ak.decode_paged(gp["q"], gp["k_pages"], gp["v_pages"], gp["block_table"], gp["seq_lens"],
                          scale=p["scale"], workspace=pws)
    assert ak.workspace_status(pws) == 0
    assert_parity(out, oracle.decode_paged(p["q"], p["k_pages"], p["v_pages"], p["block_table"], p["seq_lens"],
                                           p["scale"]), "checked paged decode")
    tws = ak.decode_topv_workspace(ak.make_dims(3, 16, 4, 16, 64, 128, p["scale"]), 320, 50, dev)
    out, idx = ak.decode_topv_paged(gp["q"], gp["k_pages"], gp["v_pages"], gp["block_table"], gp["seq_lens"], 50,
                                    scale=p["scale"], workspace=tws)
    assert ak.workspace_status(tws) == 0
    kc = oracle.gather_paged(p["k_pages"], p["block_table"], p["seq_lens"])
    vc = oracle.gather_paged(p["v_pages"], p["block_table"], p["seq_lens"])
    r_out, r_idx = oracle.decode_topv(p["q"], kc, vc, p["seq_lens"], 50, p["scale"])
    assert np.array_equal(idx.cpu().numpy(), r_idx)
    assert_parity(out, r_out, "checked paged top-v")
    print("paged decode and paged selective V ok")
    # selective V: lengths around the 128-position tile
    t = wl.random_decode_inputs(4, 300, s, seed=75, seq_lens=[127, 128, 129, 300])
    gt = to(t, dev)
    tws = ak.decode_topv_workspace(ak.make_dims(4, 16, 4, 16, 64, 128, t["scale"]), 300, 100, dev)
    out, idx = ak.decode_topv(gt["q"], gt["k_cache"], gt["v_cache"], gt["seq_lens"], 100, scale=t["scale"],
                              workspace=tws)
    assert ak.workspace_status(tws) == 0
    r_out, r_idx = oracle.decode_topv(t["q"], t["k_cache"], t["v_cache"], t["seq_lens"], 100, t["scale"])
    assert np.array_equal(idx.cpu().numpy(), r_idx)
    assert_parity(out, r_out, "checked top-v")
    print("selective V ok")
    # prefill, both tilings, lengths around the tiles, with the call's own status word
    for shape, seq in ((wl.DIFFQKV, 129), (wl.GQA_CONTROL, 257)):
        pr = wl.random_prefill_inputs(1, seq, shape, seed=76)
        gpr = to(pr, dev)
        word = torch.zeros(1, dtype=torch.int32, device=dev)
        out = ak.prefill_causal(gpr["q"], gpr["k"], gpr["v"], scale=pr["scale"], status=word)
        torch.cuda.synchronize()
        assert int(word.item()) == 0
        assert_parity_prefill(out, oracle.prefill_causal(pr["q"], pr["k"], pr["v"], pr["scale"]), "checked prefill")
    print("prefill ok")
    # prefill over paged pools (16-position pages) and a prefix
    pr = wl.random_prefill_inputs(2, 300, wl.DIFFQKV, seed=77)
    per = -(-300 // 16)
    perm = torch.randperm(2 * per, generator=torch.Generator().manual_seed(78)).to(torch.int32).view(2, per)
    kp = torch.zeros((2 * per, 16, s.n_k, s.d_k), dtype=torch.bfloat16)
    vp = torch.zeros((2 * per, 16, s.n_v, s.d_v), dtype=torch.bfloat16)
    for b in range(2):
        for pg in range(per):
            n = min(16, 300 - pg * 16)
            kp[perm[b, pg], :n] = pr["k"][b, pg * 16:pg * 16 + n]
            vp[perm[b, pg], :n] = pr["v"][b, pg * 16:pg * 16 + n]
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    out = ak.prefill_causal_paged(pr["q"][:, 100:].contiguous().to(dev), kp.to(dev), vp.to(dev), perm.to(dev), 100,
                                  scale=pr["scale"], status=word)
    torch.cuda.synchronize()
    assert int(word.item()) == 0
    assert_parity_prefill(out, oracle.prefill_causal(pr["q"], pr["k"], pr["v"], pr["scale"])[:, 100:],
                          "checked paged prefill")
    print("paged prefill ok")
    # augmented query projection: a token tail and a partial output tile
    a = wl.random_augq_inputs(300, 256, 384, 160, seed=79)
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    q, h = ak.augq_project(*(a[k].to(dev) for k in ("x", "w_gate", "w_up", "w_down")), status=word)
    torch.cuda.synchronize()
    assert int(word.item()) == 0
    assert_parity_gemm(h, oracle.augq_hidden(a["x"], a["w_gate"], a["w_up"]), "checked augmented Q: h")
    assert_parity_gemm(q, oracle.augq_down(h.cpu().double().numpy(), a["w_down"]), "checked augmented Q: q")
    print("augmented query projection ok")
    print("all cases ok")


if __name__ == "__main__":
    main()
