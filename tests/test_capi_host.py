"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, plans launches, and rejects bad arguments before launching."""
import ctypes

import pytest

import asymmetric_head_kv_b200 as ak
from asymmetric_head_kv_b200 import _capi
from asymmetric_head_kv_b200.build import build


@pytest.fixture(scope="module", autouse=True)
def _built():
    build()


def test_exports_every_declared_symbol():
    lib = _capi.lib()
    names = _capi.header_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_capi.SIGNATURES), "binding and header disagree"


def test_status_strings_and_version():
    lib = _capi.lib()
    for code, name in _capi.STATUS.items():
        assert lib.diffqkv_status_string(code).decode() == name
    assert lib.diffqkv_status_string(999).decode() == "DIFFQKV_ERR_UNKNOWN"
    assert lib.diffqkv_version() >= 10000


def dims(**kw):
    base = dict(batch=16, n_q=16, n_k=4, n_v=16, d_k=64, d_v=128, scale=0.125)
    base.update(kw)
    return ak.make_dims(**base)


def test_workspace_size_depends_only_on_dims():
    lib = _capi.lib()
    d = dims()
    n = lib.diffqkv_decode_workspace_size(ctypes.byref(d))
    assert n > 0 and n % 16 == 0
    assert lib.diffqkv_decode_workspace_size(ctypes.byref(dims(batch=32))) > n
    assert lib.diffqkv_decode_workspace_size(ctypes.byref(dims(n_k=3))) == 0   # 16 % 3 != 0
    assert lib.diffqkv_decode_workspace_size(None) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(n_k=3), _capi.INVALID_ARG),
    (dict(n_v=5), _capi.INVALID_ARG),
    (dict(batch=0), _capi.INVALID_ARG),
    (dict(scale=0.0), _capi.INVALID_ARG),
    (dict(scale=float("nan")), _capi.INVALID_ARG),
    (dict(d_k=96), _capi.UNSUPPORTED),
    (dict(n_q=64, n_k=2, n_v=16), _capi.UNSUPPORTED),   # 32 query heads per K head
])
def test_plan_rejects_bad_shapes(kw, code):
    with pytest.raises(ak.DiffqkvError) as e:
        ak.decode_plan(dims(**kw), 32768, 32768, 148)
    assert e.value.status == code


@pytest.mark.parametrize("shape", [
    dict(), dict(n_k=16, d_k=128), dict(n_q=32, n_k=4, n_v=16, d_v=64), dict(n_k=16, n_v=16, d_k=64, d_v=64),
    dict(n_k=1, n_v=1), dict(n_k=8, n_v=2), dict(n_q=24, n_k=12, n_v=8),
])
def test_plan_fits_b200(shape):
    p = ak.decode_plan(dims(**shape), 32768, 32768, 148)
    assert 2 <= p["stages"] <= 8
    assert p["smem_bytes"] <= 227 * 1024
    assert 1 <= p["grid_ctas"] <= 148
    assert 4 <= p["tile_tokens"] <= 128
    assert p["threads"] % 32 == 0 and p["threads"] <= 1024


def test_plan_grid_follows_context_and_override():
    p = ak.decode_plan(dims(batch=1), 512, 512, 148)
    assert p["grid_ctas"] == 4 * -(-512 // p["tile_tokens"])    # fewer tiles than SMs
    p = ak.decode_plan(dims(), 32768, 32768, 148, {"grid_ctas": 7, "stages": 3, "ctas_per_sm": 0})
    assert p["grid_ctas"] == 7 and p["stages"] == 3
    with pytest.raises(ak.DiffqkvError):
        ak.decode_plan(dims(), 32768, 32768, 148, {"grid_ctas": 5000, "stages": 0, "ctas_per_sm": 0})


def test_v_heads_per_tile():
    assert ak.decode_plan(dims(), 1024, 1024, 148)["v_heads_per_tile"] == 4
    assert ak.decode_plan(dims(n_k=16, d_k=128), 1024, 1024, 148)["v_heads_per_tile"] == 1
    assert ak.decode_plan(dims(n_k=8, n_v=2), 1024, 1024, 148)["v_heads_per_tile"] == 1
    # n_q=24, n_k=12 (2 q-heads per K head), n_v=8 (3 per V head): group 1 spans V heads 0 and 1
    assert ak.decode_plan(dims(n_q=24, n_k=12, n_v=8), 1024, 1024, 148)["v_heads_per_tile"] == 2
    with pytest.raises(ak.DiffqkvError):   # 3 query heads per K head has no kernel
        ak.decode_plan(dims(n_q=12, n_k=4, n_v=6), 1024, 1024, 148)


def _decode_raw(d, q=0x1000, k=0x2000, v=0x3000, sl=0x4000, t_max=128, out=0x5000, ws=0x6000, ws_bytes=1 << 30):
    return _capi.lib().diffqkv_decode(ctypes.byref(d), q, k, v, sl, t_max, t_max, out, ws, ws_bytes, None)


def test_decode_rejects_before_launch():
    d = dims()
    assert _decode_raw(d, q=None) == _capi.INVALID_ARG
    assert _decode_raw(d, t_max=0) == _capi.INVALID_ARG
    assert _decode_raw(d, q=0x1008) == _capi.MISALIGNED
    assert _decode_raw(d, out=0x5004) == _capi.MISALIGNED
    assert _decode_raw(d, ws=None) == _capi.WORKSPACE
    assert _decode_raw(d, ws_bytes=16) == _capi.WORKSPACE
    assert _decode_raw(dims(n_k=3)) == _capi.INVALID_ARG


def test_prefill_and_topv_reject_null():
    lib = _capi.lib()
    d = dims()
    assert lib.diffqkv_prefill_causal(ctypes.byref(d), None, None, None, 16, None, None) != _capi.OK
    assert lib.diffqkv_decode_topv(ctypes.byref(d), None, None, None, None, 16, 16, 4, None, None, None, 0,
                                   None) != _capi.OK


def test_selftest_and_status_reject_bad_args():
    lib = _capi.lib()
    assert lib.diffqkv_selftest_wait_timeout(10, None) == _capi.INVALID_ARG
    assert lib.diffqkv_get_device_status(None, None) == _capi.INVALID_ARG


def _topv_raw(d, t_max=128, topk=4, q=0x1000, idx=0x7000, ws=0x6000, ws_bytes=1 << 34):
    return _capi.lib().diffqkv_decode_topv(ctypes.byref(d), q, 0x2000, 0x3000, 0x4000, t_max, t_max, topk, 0x5000,
                                           idx, ws, ws_bytes, None)


def test_topv_rejects_before_launch():
    d = dims()
    assert _topv_raw(d, topk=0) == _capi.INVALID_ARG
    assert _topv_raw(d, t_max=0) == _capi.INVALID_ARG
    assert _topv_raw(d, t_max=131073) == _capi.UNSUPPORTED  # kept-position bitmap holds 131072 positions
    assert _topv_raw(d, q=0x1008) == _capi.MISALIGNED
    assert _topv_raw(d, idx=0x7002) == _capi.MISALIGNED
    assert _topv_raw(d, ws_bytes=16) == _capi.WORKSPACE
    assert _capi.lib().diffqkv_decode_topv_workspace_size(ctypes.byref(d), 131072, 1024) > 0
    # 14 bytes per (row, position): candidate position and score, ambiguous position, two state bytes
    small = _capi.lib().diffqkv_decode_topv_workspace_size(ctypes.byref(d), 1024, 8)
    large = _capi.lib().diffqkv_decode_topv_workspace_size(ctypes.byref(d), 2048, 8)
    assert large - small == d.batch * d.n_q * 1024 * 14


def test_decode_append_rejects_before_launch():
    lib = _capi.lib()
    d = dims()

    def call(kn=0x8000, vn=0x9000, q=0x1000):
        return lib.diffqkv_decode_append(ctypes.byref(d), q, kn, vn, 0x2000, 0x3000, 0x4000, 128, 128, 0x5000,
                                         0x6000, 1 << 30, None)
    assert call(kn=None) == _capi.INVALID_ARG
    assert call(vn=None) == _capi.INVALID_ARG
    assert call(kn=0x8008) == _capi.MISALIGNED
    assert call(q=None) == _capi.INVALID_ARG


def test_topv_ex_rejects_unknown_flags():
    d = dims()
    st = _capi.lib().diffqkv_decode_topv_ex(ctypes.byref(d), 0x1000, 0x2000, 0x3000, 0x4000, 128, 128, 4, 2,
                                             0x5000, 0x7000, 0x6000, 1 << 34, None)
    assert st == _capi.INVALID_ARG


def test_prefill_prefix_rejects_negative_prefix():
    d = dims()
    st = _capi.lib().diffqkv_prefill_causal_prefix(ctypes.byref(d), 0x1000, 0x2000, 0x3000, -1, 16, 0x5000, None)
    assert st == _capi.INVALID_ARG


def test_decode_paged_rejects_before_launch():
    lib = _capi.lib()
    d = dims()

    def call(bt=0x7000, max_blocks=8, page_size=16, num_pages=10, kn=None, vn=None, q=0x1000):
        return lib.diffqkv_decode_paged(ctypes.byref(d), q, kn, vn, 0x2000, 0x3000, bt, max_blocks, page_size,
                                        num_pages, 0x4000, 128, 0x5000, 0x6000, 1 << 30, None)
    assert call(bt=None) == _capi.INVALID_ARG
    assert call(bt=0x7002) == _capi.MISALIGNED
    assert call(page_size=0) == _capi.INVALID_ARG
    assert call(max_blocks=0) == _capi.INVALID_ARG
    assert call(num_pages=0) == _capi.INVALID_ARG
    assert call(max_blocks=1 << 20, page_size=1 << 12) == _capi.INVALID_ARG  # capacity past int32
    assert call(kn=0x8000) == _capi.INVALID_ARG                               # k_new without v_new
    assert call(q=0x1008) == _capi.MISALIGNED


def test_fold_query_rejects_before_launch():
    lib = _capi.lib()
    d = dims()

    def call(d_q=192, w_heads=4, q=0x1000, dd=d):
        return lib.diffqkv_fold_query(ctypes.byref(dd), d_q, w_heads, q, 0x2000, 0x3000, None)
    assert call(d_q=100) == _capi.INVALID_ARG     # not a multiple of 8
    assert call(d_q=0) == _capi.INVALID_ARG
    assert call(w_heads=2) == _capi.INVALID_ARG   # neither 1 nor n_k
    assert call(q=None) == _capi.INVALID_ARG
    assert call(q=0x1008) == _capi.MISALIGNED
    assert call(dd=dims(d_k=96)) == _capi.UNSUPPORTED


def test_paged_input_recipe_deals_distinct_pages():
    """Each sequence holds ceil((seq_len + 1) / page_size) distinct pool pages, none shared, -1 elsewhere."""
    import workloads as wl
    d = wl.random_paged_inputs(4, 10, 16, wl.DIFFQKV, seed=5, seq_lens=[0, 15, 16, 150], spare_pages=2)
    table = d["block_table"]
    held = [(t + 1 + 15) // 16 for t in (0, 15, 16, 150)]
    assert d["num_pages"] == sum(held) + 2
    used = []
    for b, n in enumerate(held):
        assert (table[b, :n] >= 0).all() and (table[b, n:] == -1).all()
        used += table[b, :n].tolist()
    assert len(set(used)) == len(used) and max(used) < d["num_pages"]
    assert d["k_pages"].shape == (d["num_pages"], 16, 4, 64) and d["v_pages"].shape == (d["num_pages"], 16, 16, 128)


def test_python_bindings_reject_host_tensors_and_bad_shapes():
    import torch
    q = torch.zeros(2, 16, 64, dtype=torch.bfloat16)
    kp = torch.zeros(8, 16, 4, 64, dtype=torch.bfloat16)
    vp = torch.zeros(8, 16, 16, 128, dtype=torch.bfloat16)
    bt = torch.zeros(2, 4, dtype=torch.int32)
    lens = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        ak.decode_paged(q, kp, vp, bt, lens)
    with pytest.raises(TypeError, match="bfloat16"):
        ak.decode_paged(q.float(), kp, vp, bt, lens)
    with pytest.raises(TypeError, match="bfloat16"):
        ak.fold_query(q.float(), torch.zeros(4, 64, 64), n_k=4)
    with pytest.raises(ValueError, match="CUDA"):
        ak.fold_query(q, torch.zeros(4, 64, 64, dtype=torch.bfloat16), n_k=4)


def test_header_is_plain_c_and_a_c_program_links(tmp_path):
    """include/diffqkv.h compiles as strict C99 (no C++ in the ABI) and a C program links and calls the library."""
    import os
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "abi.c"
    src.write_text('#include "diffqkv.h"\n#include <stdio.h>\n'
                   'int main(void) { printf("%s %d\\n", diffqkv_status_string(DIFFQKV_ERR_DEVICE_PAGE), '
                   'diffqkv_version() >= 10000); return 0; }\n')
    pkg = os.path.dirname(_capi.LIB_PATH)
    exe = tmp_path / "abi"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(root, "include"),
                        str(src), "-L", pkg, "-ldiffqkv", "-Wl,-rpath," + pkg, "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "DIFFQKV_ERR_DEVICE_PAGE 1"


def _from_host_raw(d, q_dev=0x11000, out_dev=0x15000, ws=0x16000, ws_bytes=1 << 30, t_max=128):
    # host buffers are never touched when an argument is rejected
    return _capi.lib().diffqkv_decode_from_host(ctypes.byref(d), 0x1000, 0x2000, 0x3000, 0x4000, t_max, t_max,
                                                0x5000, q_dev, 0x12000, 0x13000, 0x14000, out_dev, ws, ws_bytes,
                                                None)


def test_from_host_checks_every_argument_before_any_copy():
    """Without a GPU, an enqueued copy would fail with DIFFQKV_ERR_CUDA; these specific codes show
    that the decode's checks ran before the first cudaMemcpyAsync."""
    d = dims()
    assert _from_host_raw(d, q_dev=0x11008) == _capi.MISALIGNED
    assert _from_host_raw(d, out_dev=0x15004) == _capi.MISALIGNED
    assert _from_host_raw(d, ws=None) == _capi.WORKSPACE
    assert _from_host_raw(d, ws_bytes=64) == _capi.WORKSPACE
    assert _from_host_raw(d, t_max=0) == _capi.INVALID_ARG
    assert _from_host_raw(dims(n_k=3)) == _capi.INVALID_ARG
    assert _from_host_raw(dims(d_k=96)) == _capi.UNSUPPORTED


def test_workspace_status_and_prefill_word_reject_bad_args():
    lib = _capi.lib()
    v = ctypes.c_int32(0)
    assert lib.diffqkv_workspace_status(None, 1 << 20, None, ctypes.byref(v)) == _capi.INVALID_ARG
    assert lib.diffqkv_workspace_status(0x1000, 255, None, ctypes.byref(v)) == _capi.INVALID_ARG
    assert lib.diffqkv_workspace_status(0x1000, 1 << 20, None, None) == _capi.INVALID_ARG
    assert lib.diffqkv_workspace_status(0x1008, 1 << 20, None, ctypes.byref(v)) == _capi.MISALIGNED
    d = dims()
    # a misaligned status word is rejected before any device work
    assert lib.diffqkv_prefill_causal_ex(ctypes.byref(d), 0x1000, 0x2000, 0x3000, 0, 16, 0x5000, 0x6002,
                                         None) == _capi.MISALIGNED
    assert lib.diffqkv_prefill_causal_ex(ctypes.byref(d), 0x1000, 0x2000, 0x3000, -1, 16, 0x5000, None,
                                         None) == _capi.INVALID_ARG


def test_decode_topv_paged_rejects_before_launch():
    lib = _capi.lib()
    d = dims()

    def call(bt=0x7000, max_blocks=8, page_size=16, num_pages=10, q=0x1000, flags=0):
        return lib.diffqkv_decode_topv_paged(ctypes.byref(d), q, 0x2000, 0x3000, bt, max_blocks, page_size, num_pages,
                                             0x4000, 128, 4, flags, 0x5000, 0x7000, 0x6000, 1 << 34, None)
    assert call(bt=None) == _capi.INVALID_ARG
    assert call(bt=0x7002) == _capi.MISALIGNED
    assert call(page_size=0) == _capi.INVALID_ARG
    assert call(num_pages=0) == _capi.INVALID_ARG
    assert call(page_size=12) == _capi.UNSUPPORTED          # not a multiple of 8
    assert call(max_blocks=2048, page_size=128) == _capi.UNSUPPORTED  # capacity past 131072
    assert call(flags=2) == _capi.INVALID_ARG
    assert call(q=0x1008) == _capi.MISALIGNED


def test_checked_build_exports_every_declared_symbol_and_nvtx_switch_is_harmless():
    """The checked library exports the same C ABI; with DIFFQKV_NVTX set, calls still return their
    status (here without a GPU) through the NVTX-ranged entry points."""
    import subprocess
    import sys
    code = (
        "import ctypes, asymmetric_head_kv_b200 as ak\n"
        "from asymmetric_head_kv_b200 import _capi\n"
        "lib = _capi.lib()\n"
        "assert _capi.LIB_PATH.endswith('libdiffqkv_checked.so')\n"
        "for n in _capi.header_symbols(): getattr(lib, n)\n"
        "d = ak.make_dims(1, 16, 4, 16, 64, 128, 0.125)\n"
        "st = lib.diffqkv_decode(ctypes.byref(d), None, 0, 0, 0, 16, 16, 0, 0, 0, None)\n"
        "assert st == _capi.INVALID_ARG, st\n"
        "assert lib.diffqkv_status_string(11).decode() == 'DIFFQKV_ERR_DEVICE_BOUNDS'\n"
        "print('ok')\n")
    import os
    env = dict(os.environ, DIFFQKV_BOUNDS_CHECK="1", DIFFQKV_NVTX="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], env=env, cwd=root, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr


def test_augq_project_rejects_before_launch():
    """The augmented query projection checks pointers, alignment and tile multiples on the host;
    zero tokens launch nothing (no device needed for any of these)."""
    lib = _capi.lib()

    def call(x=0x1000, wg=0x2000, wu=0x3000, wd=0x4000, tokens=300, d_model=2048, d_inter=3072, d_out=2048,
             h=0x5000, q=0x6000, status=None):
        return lib.diffqkv_augq_project(x, wg, wu, wd, tokens, d_model, d_inter, d_out, h, q, status, None)
    assert call(x=None) == _capi.INVALID_ARG
    assert call(h=None) == _capi.INVALID_ARG
    assert call(tokens=-1) == _capi.INVALID_ARG
    assert call(d_model=32) == _capi.INVALID_ARG
    assert call(d_model=2048 + 32) == _capi.UNSUPPORTED   # reduction in whole 64-element steps
    assert call(d_inter=3072 + 64) == _capi.UNSUPPORTED   # gate/up tiles of 128 features
    assert call(d_out=2048 + 16) == _capi.UNSUPPORTED     # 32-column epilogue chunks
    assert call(wd=0x4008) == _capi.MISALIGNED
    assert call(status=0x7002) == _capi.MISALIGNED
    assert call(tokens=1 << 20) == _capi.UNSUPPORTED      # tokens * 3072 >= 2^31
    assert call(tokens=0) == _capi.OK                     # nothing to do
    assert call(tokens=0, x=None, h=None, q=None) == _capi.OK  # empty tensors have no storage
    assert call(tokens=0, wg=None) == _capi.INVALID_ARG


def test_prefill_causal_paged_rejects_before_launch():
    lib = _capi.lib()
    d = dims(batch=2)

    def call(bt=0x7000, max_blocks=8, page_size=16, num_pages=10, prefix=64, seq=64, status=None):
        return lib.diffqkv_prefill_causal_paged(ctypes.byref(d), 0x1000, 0x2000, 0x3000, bt, max_blocks, page_size,
                                                num_pages, prefix, seq, 0x5000, status, None)
    assert call(bt=None) == _capi.INVALID_ARG
    assert call(bt=0x7002) == _capi.MISALIGNED
    assert call(page_size=12) == _capi.UNSUPPORTED        # boxes need whole 8-row swizzle atoms
    assert call(max_blocks=7) == _capi.INVALID_ARG        # 128 positions need 8 pages of 16
    assert call(num_pages=0) == _capi.INVALID_ARG
    assert call(seq=0) == _capi.INVALID_ARG
    assert call(prefix=-1) == _capi.INVALID_ARG
    assert call(status=0x6002) == _capi.MISALIGNED
