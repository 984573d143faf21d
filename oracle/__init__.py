"""fp64 CPU oracle for DiffQKV attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding in ``asymmetric_head_kv_b200``) never imports, links or
executes anything here, and this package imports nothing from it.

The arithmetic lives in ``oracle.c`` (plain C, fp64) and follows "Sigma:
Differential Rescaling of Query, Key and Value for Efficient Language Models"
(structured summary page), section 3.4 "DiffQKV Attention: Generalized
Formulation" Steps 2-5, "Selective V Cache Fetching", "FlexHeadFA Kernel
and Deployment Infrastructure", and section 3.2 "Big-Picture Architecture"
item 4 (augmented Q with SwiGLU gating).  This module only marshals arrays.

Inputs are bf16 tensors (torch) or uint16 arrays holding bf16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from fractions import Fraction

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (no CUDA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    c_i, c_d, c_p, c_i64 = ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_int64
    lib.oracle_head_map.argtypes = [c_i, c_i, c_i]
    lib.oracle_head_map.restype = c_i
    lib.oracle_decode.argtypes = [c_i] * 6 + [c_d] + [c_p] * 4 + [c_i, c_i, c_p, c_i64, c_p, c_i]
    lib.oracle_decode.restype = c_i
    lib.oracle_prefill_causal.argtypes = [c_i] * 7 + [c_d] + [c_p] * 4 + [c_i64, c_p, c_i]
    lib.oracle_prefill_causal.restype = c_i
    lib.oracle_exact_dot.argtypes = [c_p, c_p, c_i, c_p, ctypes.POINTER(c_i)]
    lib.oracle_exact_dot.restype = c_i
    lib.oracle_decode_topv.argtypes = (
        [c_i] * 6 + [c_d] + [c_p] * 4 + [c_i, c_i, c_p, c_i64, c_p, c_p, c_i]
    )
    lib.oracle_decode_topv.restype = c_i
    lib.oracle_decode_topv_ex.argtypes = (
        [c_i] * 6 + [c_d] + [c_p] * 4 + [c_i, c_i, c_i, c_p, c_i64, c_p, c_p, c_i]
    )
    lib.oracle_decode_topv_ex.restype = c_i
    lib.oracle_gather_paged.argtypes = [c_i] * 6 + [c_p] * 4
    lib.oracle_gather_paged.restype = c_i
    lib.oracle_decode_up_projected.argtypes = [c_i] * 8 + [c_d] + [c_p] * 5 + [c_i, c_p]
    lib.oracle_decode_up_projected.restype = c_i
    lib.oracle_fold_query.argtypes = [c_i] * 6 + [c_p] * 3
    lib.oracle_fold_query.restype = c_i
    lib.oracle_augq_hidden.argtypes = [c_i] * 3 + [c_p] * 4 + [c_i, c_p, c_i]
    lib.oracle_augq_hidden.restype = c_i
    lib.oracle_augq_down.argtypes = [c_i] * 3 + [c_p] * 3 + [c_i]
    lib.oracle_augq_down.restype = c_i
    _lib = lib
    return lib


def _bits(x) -> np.ndarray:
    """bf16 tensor / uint16 array -> C-contiguous uint16 numpy view of the bits."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            if x.dtype != torch.bfloat16:
                raise TypeError(f"expected bfloat16, got {x.dtype}")
            x = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError(f"expected bf16 bit patterns (uint16), got {x.dtype}")
    return x


def _i32(x) -> np.ndarray:
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc < 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


def head_map(n_q: int, n_kv: int, h: int) -> int:
    """GroupSharing: query head h reads K/V head floor(h * n_kv / n_q)."""
    r = _load().oracle_head_map(n_q, n_kv, h)
    if r < 0:
        raise ValueError("bad head-map arguments")
    return r


def decode(q, k_cache, v_cache, seq_lens, scale: float, *, num_splits: int = 0,
           rows=None, threads: int = 0) -> np.ndarray:
    """fp64 decode attention.

    q [B, n_q, d_k], k_cache [B, t_max, n_k, d_k], v_cache [B, t_max, n_v, d_v]
    (bf16), seq_lens [B].  ``num_splits`` > 0 runs the split/combine form.
    Returns [B, n_q, d_v] float64, or [len(rows), d_v] for ``rows`` = (b, h) pairs.
    """
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    B, n_q, d_k = qb.shape
    _, t_max, n_k, d_k2 = kb.shape
    _, t_max2, n_v, d_v = vb.shape
    assert d_k == d_k2 and t_max == t_max2 and kb.shape[0] == B and vb.shape[0] == B
    sl = _i32(seq_lens)
    assert sl.shape == (B,)
    if rows is None:
        out = np.empty((B * n_q, d_v), np.float64)
        rp, nr = None, B * n_q
    else:
        rr = _i32(rows).reshape(-1, 2)
        out = np.empty((rr.shape[0], d_v), np.float64)
        rp, nr = _ptr(rr), rr.shape[0]
    rc = _load().oracle_decode(B, n_q, n_k, n_v, d_k, d_v, float(scale), _ptr(qb), _ptr(kb), _ptr(vb),
                               _ptr(sl), t_max, num_splits, rp, nr, _ptr(out), threads)
    _check(rc, "decode")
    return out.reshape(B, n_q, d_v) if rows is None else out


def prefill_causal(q, k, v, scale: float, *, rows=None, threads: int = 0) -> np.ndarray:
    """fp64 causal prefill.

    q [B, S, n_q, d_k], k [B, S, n_k, d_k], v [B, S, n_v, d_v] (bf16).
    Returns [B, S, n_q, d_v] float64, or [len(rows), d_v] for ``rows`` = (b, i, h).
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, S, n_q, d_k = qb.shape
    n_k, n_v, d_v = kb.shape[2], vb.shape[2], vb.shape[3]
    assert kb.shape == (B, S, n_k, d_k) and vb.shape[:2] == (B, S)
    if rows is None:
        out = np.empty((B * S * n_q, d_v), np.float64)
        rp, nr = None, B * S * n_q
    else:
        rr = _i32(rows).reshape(-1, 3)
        out = np.empty((rr.shape[0], d_v), np.float64)
        rp, nr = _ptr(rr), rr.shape[0]
    rc = _load().oracle_prefill_causal(B, S, n_q, n_k, n_v, d_k, d_v, float(scale), _ptr(qb), _ptr(kb),
                                       _ptr(vb), rp, nr, _ptr(out), threads)
    _check(rc, "prefill_causal")
    return out.reshape(B, S, n_q, d_v) if rows is None else out


def exact_dot(a, b) -> Fraction:
    """Exact value of sum_i a_i * b_i for bf16 vectors, as a Fraction."""
    ab, bb = _bits(a).reshape(-1), _bits(b).reshape(-1)
    assert ab.shape == bb.shape
    digits = np.zeros(32, np.int64)
    lsb = ctypes.c_int(0)
    nd = _load().oracle_exact_dot(_ptr(ab), _ptr(bb), ab.shape[0], _ptr(digits), ctypes.byref(lsb))
    _check(nd, "exact_dot")
    total = sum(int(digits[i]) << (32 * i) for i in range(nd))
    return Fraction(total, 1) * Fraction(2) ** lsb.value


def decode_topv(q, k_cache, v_cache, seq_lens, topk: int, scale: float, *, rows=None,
                threads: int = 0, full_weights: bool = False):
    """fp64 selective-V decode over the top-k exact-scoring positions per query head.

    The kept V rows are weighted by the softmax renormalised over the kept set, or with
    ``full_weights`` by the full-softmax weights alpha_j (the other positions counting as zero).
    Returns (out float64 [B, n_q, d_v], idx int32 [B, n_q, topk]) -- idx ascending,
    padded with -1 when topk exceeds the context -- or row-major [len(rows), ...].
    """
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    B, n_q, d_k = qb.shape
    _, t_max, n_k, _ = kb.shape
    _, _, n_v, d_v = vb.shape
    sl = _i32(seq_lens)
    if rows is None:
        nr, rp = B * n_q, None
    else:
        rr = _i32(rows).reshape(-1, 2)
        nr, rp = rr.shape[0], _ptr(rr)
    out = np.empty((nr, d_v), np.float64)
    idx = np.empty((nr, max(topk, 0)), np.int32)
    rc = _load().oracle_decode_topv_ex(B, n_q, n_k, n_v, d_k, d_v, float(scale), _ptr(qb), _ptr(kb),
                                       _ptr(vb), _ptr(sl), t_max, topk, 1 if full_weights else 0, rp, nr,
                                       _ptr(out), _ptr(idx), threads)
    _check(rc, "decode_topv")
    if rows is None:
        return out.reshape(B, n_q, d_v), idx.reshape(B, n_q, max(topk, 0))
    return out, idx


def gather_paged(pool, block_table, seq_lens):
    """Contiguous cache [B, max_blocks * page_size, heads, d] (bf16 bits as a torch bf16 tensor)
    holding the first seq_lens[b] positions of each sequence of a paged pool
    [num_pages, page_size, heads, d] under block_table [B, max_blocks]; zeros elsewhere."""
    import torch

    pb = _bits(pool)
    num_pages, page_size, heads, d = pb.shape
    bt = _i32(block_table)
    B, max_blocks = bt.shape
    sl = _i32(seq_lens)
    assert sl.shape == (B,)
    out = np.empty((B, max_blocks * page_size, heads, d), np.uint16)
    rc = _load().oracle_gather_paged(B, heads, d, page_size, max_blocks, num_pages, _ptr(pb), _ptr(bt),
                                     _ptr(sl), _ptr(out))
    _check(rc, "gather_paged")
    return torch.from_numpy(out.view(np.int16)).view(torch.bfloat16)


def decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale: float, *, rows=None,
                 threads: int = 0) -> np.ndarray:
    """fp64 decode over paged K/V pools: the pools gathered into contiguous caches, then :func:`decode`."""
    k = gather_paged(k_pages, block_table, seq_lens)
    v = gather_paged(v_pages, block_table, seq_lens)
    return decode(q, k, v, seq_lens, scale, rows=rows, threads=threads)


def decode_up_projected(q_aug, w_up, k_cache, v_cache, seq_lens, scale: float) -> np.ndarray:
    """fp64 decode whose keys are first projected up to the query width: q_aug [B, n_q, d_q],
    w_up [w_heads, d_q, d_k] (w_heads 1 or n_k), caches as in :func:`decode`.  [B, n_q, d_v]."""
    qb, wb, kb, vb = _bits(q_aug), _bits(w_up), _bits(k_cache), _bits(v_cache)
    B, n_q, d_q = qb.shape
    w_heads, d_q2, d_k = wb.shape
    _, t_max, n_k, d_k2 = kb.shape
    _, _, n_v, d_v = vb.shape
    assert d_q == d_q2 and d_k == d_k2
    sl = _i32(seq_lens)
    out = np.empty((B, n_q, d_v), np.float64)
    rc = _load().oracle_decode_up_projected(B, n_q, n_k, n_v, d_q, d_k, d_v, w_heads, float(scale), _ptr(qb),
                                            _ptr(wb), _ptr(kb), _ptr(vb), _ptr(sl), t_max, _ptr(out))
    _check(rc, "decode_up_projected")
    return out


def fold_query(q_aug, w_up, n_k: int) -> np.ndarray:
    """fp64 W^T q for every query head (its K head's matrix): [B, n_q, d_k]."""
    qb, wb = _bits(q_aug), _bits(w_up)
    B, n_q, d_q = qb.shape
    w_heads, d_q2, d_k = wb.shape
    assert d_q == d_q2
    out = np.empty((B, n_q, d_k), np.float64)
    rc = _load().oracle_fold_query(B, n_q, n_k, d_q, d_k, w_heads, _ptr(qb), _ptr(wb), _ptr(out))
    _check(rc, "fold_query")
    return out


def augq_hidden(x, w_gate, w_up, *, rows=None, threads: int = 0) -> np.ndarray:
    """fp64 gated hidden state of the augmented query projection, SiLU(x W_gate^T) * (x W_up^T):
    x [tokens, d_model], w_gate / w_up [d_inter, d_model] (bf16).  ``rows``: token indices to
    evaluate (all when None).  [n_rows, d_inter]."""
    xb, gb, ub = _bits(x), _bits(w_gate), _bits(w_up)
    tokens, d_model = xb.shape
    d_inter, d_model2 = gb.shape
    assert ub.shape == gb.shape and d_model == d_model2
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, np.int32))
    n = tokens if r is None else len(r)
    out = np.empty((n, d_inter), np.float64)
    rc = _load().oracle_augq_hidden(tokens, d_model, d_inter, _ptr(xb), _ptr(gb), _ptr(ub),
                                    None if r is None else _ptr(r), n, _ptr(out), threads)
    _check(rc, "augq_hidden")
    return out


def augq_down(h, w_down, *, threads: int = 0) -> np.ndarray:
    """fp64 down projection h W_down^T: h [n_rows, d_inter] (any float array, e.g. a rounded
    hidden state), w_down [d_out, d_inter] (bf16).  [n_rows, d_out]."""
    hd = np.ascontiguousarray(np.asarray(h, np.float64))
    wb = _bits(w_down)
    n, d_inter = hd.shape
    d_out, d_inter2 = wb.shape
    assert d_inter == d_inter2
    out = np.empty((n, d_out), np.float64)
    rc = _load().oracle_augq_down(n, d_inter, d_out, _ptr(hd), _ptr(wb), _ptr(out), threads)
    _check(rc, "augq_down")
    return out


def augq_project(x, w_gate, w_up, w_down, *, rows=None, threads: int = 0) -> np.ndarray:
    """fp64 augmented query q = q_down(SiLU(q_gate(x)) * q_up(x)) for the token rows ``rows``
    (all when None): [n_rows, d_out]."""
    return augq_down(augq_hidden(x, w_gate, w_up, rows=rows, threads=threads), w_down, threads=threads)
