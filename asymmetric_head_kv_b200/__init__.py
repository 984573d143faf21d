"""DiffQKV attention on NVIDIA B200 (sm_100a): Python binding of libdiffqkv.so.

DiffQKV attention (Sigma paper, structured summary page, section 3.4) lets the
K and V caches have different head counts and head dims; query head h reads K
head h/(n_q/n_k) and V head h/(n_q/n_v).  Every function below only marshals
torch tensors into the C ABI declared in include/diffqkv.h: shapes become a
``diffqkv_dims_t``, tensors become device pointers, and the current torch CUDA
stream is passed through.  All arithmetic runs in the library's CUDA kernels;
torch provides device memory and streams.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _capi
from ._capi import DiffqkvError, Dims, DecodePlan, DecodeTuning, check, lib

__all__ = [
    "decode", "decode_workspace", "decode_plan", "decode_from_host", "decode_topv", "decode_topv_workspace",
    "prefill_causal", "device_status", "selftest_wait_timeout", "DiffqkvError", "Dims", "library_path",
    "decode_noalloc", "decode_append", "decode_paged", "prefill_causal_prefix", "fold_query", "workspace_status",
    "decode_topv_paged", "augq_project", "prefill_causal_paged",
]

library_path = _capi.LIB_PATH


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _bf16_dev(t: torch.Tensor, name: str, ndim: int):
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-D tensor, got shape {tuple(t.shape)}")


def make_dims(batch, n_q, n_k, n_v, d_k, d_v, scale) -> Dims:
    return Dims(batch, n_q, n_k, n_v, d_k, d_v, float(scale))


def _decode_dims(q, k_cache, v_cache, scale):
    B, n_q, d_k = q.shape
    Bk, t_max, n_k, d_k2 = k_cache.shape
    Bv, t_max2, n_v, d_v = v_cache.shape
    if B != Bk or B != Bv or d_k != d_k2 or t_max != t_max2:
        raise ValueError("q / k_cache / v_cache shapes disagree")
    if scale is None:
        scale = d_k ** -0.5
    return make_dims(B, n_q, n_k, n_v, d_k, d_v, scale), t_max


def decode_workspace(q_or_dims, k_cache=None, v_cache=None, device=None) -> torch.Tensor:
    """Zero-filled workspace for :func:`decode` (reusable across calls of one shape)."""
    dims = q_or_dims if isinstance(q_or_dims, Dims) else _decode_dims(q_or_dims, k_cache, v_cache, 1.0)[0]
    n = lib().diffqkv_decode_workspace_size(ctypes.byref(dims))
    if n == 0:
        raise DiffqkvError(_capi.INVALID_ARG, "decode_workspace_size")
    dev = device if device is not None else (q_or_dims.device if isinstance(q_or_dims, torch.Tensor) else "cuda")
    return torch.zeros(n, dtype=torch.uint8, device=dev)


def decode_plan(dims: Dims, t_max: int, max_seq_len: int, num_sms: int, tuning: Optional[dict] = None) -> dict:
    """Host-side launch plan of :func:`decode` (no GPU needed)."""
    plan = DecodePlan()
    tun = DecodeTuning(**tuning) if tuning else None
    st = lib().diffqkv_decode_plan(ctypes.byref(dims), t_max, max_seq_len, num_sms,
                                   ctypes.byref(tun) if tun else None, ctypes.byref(plan))
    check(st, "decode_plan")
    return {f: getattr(plan, f) for f, _ in DecodePlan._fields_}


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, seq_lens: torch.Tensor, *,
           scale: Optional[float] = None, max_seq_len: Optional[int] = None, out: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None, tuning: Optional[dict] = None,
           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Split/combine DiffQKV decode: out[b, h] = softmax(scale q.K^T) V over seq_lens[b] positions.

    q [B, n_q, d_k], k_cache [B, t_max, n_k, d_k], v_cache [B, t_max, n_v, d_v] (bf16, CUDA),
    seq_lens int32 [B] (CUDA).  Returns bf16 [B, n_q, d_v].
    """
    _bf16_dev(q, "q", 3)
    _bf16_dev(k_cache, "k_cache", 4)
    _bf16_dev(v_cache, "v_cache", 4)
    if seq_lens.dtype != torch.int32 or not seq_lens.is_cuda:
        raise TypeError("seq_lens must be an int32 CUDA tensor")
    dims, t_max = _decode_dims(q, k_cache, v_cache, scale)
    if out is None:
        out = torch.empty((dims.batch, dims.n_q, dims.d_v), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        workspace = decode_workspace(dims, device=q.device)
    msl = t_max if max_seq_len is None else int(max_seq_len)
    if tuning:
        tun = DecodeTuning(**tuning)
        st = lib().diffqkv_decode_ex(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
                                     t_max, msl, _ptr(out), _ptr(workspace), workspace.numel(), ctypes.byref(tun),
                                     _stream_ptr(stream))
    else:
        st = lib().diffqkv_decode(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), t_max,
                                  msl, _ptr(out), _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    check(st, "diffqkv_decode")
    return out


def decode_append(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor,
                  v_cache: torch.Tensor, seq_lens: torch.Tensor, *, scale: Optional[float] = None,
                  max_seq_len: Optional[int] = None, out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Decode step with the KV-cache append fused in: writes k_new [B, n_k, d_k] and v_new [B, n_v, d_v]
    into the caches at position seq_lens[b] (the cached count before the step; not modified) and
    returns attention over positions 0..seq_lens[b] of the updated caches, bf16 [B, n_q, d_v]."""
    _bf16_dev(q, "q", 3)
    _bf16_dev(k_new, "k_new", 3)
    _bf16_dev(v_new, "v_new", 3)
    _bf16_dev(k_cache, "k_cache", 4)
    _bf16_dev(v_cache, "v_cache", 4)
    if seq_lens.dtype != torch.int32 or not seq_lens.is_cuda:
        raise TypeError("seq_lens must be an int32 CUDA tensor")
    dims, t_max = _decode_dims(q, k_cache, v_cache, scale)
    if tuple(k_new.shape) != (dims.batch, dims.n_k, dims.d_k) or tuple(v_new.shape) != (dims.batch, dims.n_v, dims.d_v):
        raise ValueError("k_new must be [B, n_k, d_k] and v_new [B, n_v, d_v]")
    if out is None:
        out = torch.empty((dims.batch, dims.n_q, dims.d_v), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        workspace = decode_workspace(dims, device=q.device)
    msl = t_max if max_seq_len is None else int(max_seq_len)
    st = lib().diffqkv_decode_append(ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                     _ptr(v_cache), _ptr(seq_lens), t_max, msl, _ptr(out), _ptr(workspace),
                                     workspace.numel(), _stream_ptr(stream))
    check(st, "diffqkv_decode_append")
    return out


def decode_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, block_table: torch.Tensor,
                 seq_lens: torch.Tensor, *, k_new: Optional[torch.Tensor] = None, v_new: Optional[torch.Tensor] = None,
                 scale: Optional[float] = None, max_seq_len: Optional[int] = None, out: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Decode over paged caches: k_pages [num_pages, page_size, n_k, d_k], v_pages [num_pages, page_size, n_v, d_v]
    and block_table int32 [B, max_blocks]; position j of sequence b is row j % page_size of page
    block_table[b, j // page_size].  With k_new / v_new given the step's token is appended at
    position seq_lens[b] first (as in :func:`decode_append`).  Returns bf16 [B, n_q, d_v]."""
    _bf16_dev(q, "q", 3)
    _bf16_dev(k_pages, "k_pages", 4)
    _bf16_dev(v_pages, "v_pages", 4)
    for t, name in ((block_table, "block_table"), (seq_lens, "seq_lens")):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous int32 CUDA tensor")
    B, n_q, d_k = q.shape
    num_pages, page_size, n_k, d_k2 = k_pages.shape
    num_pages2, page_size2, n_v, d_v = v_pages.shape
    if d_k != d_k2 or num_pages != num_pages2 or page_size != page_size2:
        raise ValueError("q / k_pages / v_pages shapes disagree")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B, max_blocks]")
    max_blocks = block_table.shape[1]
    dims = make_dims(B, n_q, n_k, n_v, d_k, d_v, d_k ** -0.5 if scale is None else scale)
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new, or neither")
    if k_new is not None:
        _bf16_dev(k_new, "k_new", 3)
        _bf16_dev(v_new, "v_new", 3)
        if tuple(k_new.shape) != (B, n_k, d_k) or tuple(v_new.shape) != (B, n_v, d_v):
            raise ValueError("k_new must be [B, n_k, d_k] and v_new [B, n_v, d_v]")
    if out is None:
        out = torch.empty((B, n_q, d_v), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        workspace = decode_workspace(dims, device=q.device)
    t_max = max_blocks * page_size
    msl = t_max if max_seq_len is None else int(max_seq_len)
    st = lib().diffqkv_decode_paged(ctypes.byref(dims), _ptr(q), _ptr(k_new),
                                    _ptr(v_new), _ptr(k_pages), _ptr(v_pages),
                                    _ptr(block_table), max_blocks, page_size, num_pages, _ptr(seq_lens), msl,
                                    _ptr(out), _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    check(st, "diffqkv_decode_paged")
    return out


def fold_query(q_aug: torch.Tensor, w_up: torch.Tensor, *, n_k: int, out: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Folds the K up-projection into the query: q_aug [B, n_q, d_q] and w_up [w_heads, d_q, d_k]
    (w_heads 1 or n_k) give the d_k-wide query W[h // (n_q // n_k)]^T q_aug[b, h], bf16 [B, n_q, d_k]."""
    _bf16_dev(q_aug, "q_aug", 3)
    _bf16_dev(w_up, "w_up", 3)
    B, n_q, d_q = q_aug.shape
    w_heads, d_q2, d_k = w_up.shape
    if d_q != d_q2:
        raise ValueError("q_aug and w_up disagree on d_q")
    dims = make_dims(B, n_q, n_k, n_k, d_k, d_k, 1.0)
    if out is None:
        out = torch.empty((B, n_q, d_k), dtype=torch.bfloat16, device=q_aug.device)
    st = lib().diffqkv_fold_query(ctypes.byref(dims), d_q, w_heads, _ptr(q_aug), _ptr(w_up), _ptr(out),
                                  _stream_ptr(stream))
    check(st, "diffqkv_fold_query")
    return out


def augq_project(x: torch.Tensor, w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor, *,
                 h_out: Optional[torch.Tensor] = None, q_out: Optional[torch.Tensor] = None,
                 status: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
    """Augmented query projection q = (SiLU(x W_gate^T) * (x W_up^T)) W_down^T.

    x [tokens, d_model]; w_gate, w_up [d_inter, d_model]; w_down [d_out, d_inter] (bf16, CUDA).
    Returns (q [tokens, d_out], h [tokens, d_inter]), h being the gated hidden state the second
    GEMM read.  ``status``: an int32 CUDA tensor of one element, zero, for this call's device-side
    error (else the per-device word)."""
    _bf16_dev(x, "x", 2)
    _bf16_dev(w_gate, "w_gate", 2)
    _bf16_dev(w_up, "w_up", 2)
    _bf16_dev(w_down, "w_down", 2)
    tokens, d_model = x.shape
    d_inter = w_gate.shape[0]
    d_out = w_down.shape[0]
    if w_gate.shape != (d_inter, d_model) or w_up.shape != (d_inter, d_model) or w_down.shape != (d_out, d_inter):
        raise ValueError("x / w_gate / w_up / w_down shapes disagree")
    if h_out is None:
        h_out = torch.empty((tokens, d_inter), dtype=torch.bfloat16, device=x.device)
    if q_out is None:
        q_out = torch.empty((tokens, d_out), dtype=torch.bfloat16, device=x.device)
    _bf16_dev(h_out, "h_out", 2)
    _bf16_dev(q_out, "q_out", 2)
    if h_out.shape != (tokens, d_inter) or q_out.shape != (tokens, d_out):
        raise ValueError("h_out / q_out shapes disagree")
    if status is not None:
        _status_word(status)
    st = lib().diffqkv_augq_project(_ptr(x), _ptr(w_gate), _ptr(w_up), _ptr(w_down), tokens, d_model, d_inter,
                                    d_out, _ptr(h_out), _ptr(q_out), None if status is None else _ptr(status),
                                    _stream_ptr(stream))
    check(st, "diffqkv_augq_project")
    return q_out, h_out


def decode_from_host(q_host, k_host, v_host, seq_lens_host, out_host, dev_buffers: dict, *,
                     scale: Optional[float] = None, max_seq_len: Optional[int] = None,
                     stream: Optional[torch.cuda.Stream] = None) -> None:
    """End-to-end decode from (pinned) host tensors through one C-ABI call.

    ``dev_buffers`` holds preallocated CUDA tensors q, k_cache, v_cache, seq_lens, out, workspace
    of the same shapes.  Host->device copies, the decode and the device->host copy of the
    output are all enqueued on the stream; synchronise before reading ``out_host``.
    """
    dims, t_max = _decode_dims(q_host, k_host, v_host, scale)
    d = dev_buffers
    msl = t_max if max_seq_len is None else int(max_seq_len)
    st = lib().diffqkv_decode_from_host(
        ctypes.byref(dims), _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(seq_lens_host), t_max, msl,
        _ptr(out_host), _ptr(d["q"]), _ptr(d["k_cache"]), _ptr(d["v_cache"]), _ptr(d["seq_lens"]), _ptr(d["out"]),
        _ptr(d["workspace"]), d["workspace"].numel(), _stream_ptr(stream))
    check(st, "diffqkv_decode_from_host")


def decode_topv_workspace(dims: Dims, t_max: int, topk: int, device="cuda") -> torch.Tensor:
    """Workspace for :func:`decode_topv`; zero-filled (its 256-byte header holds the error word)."""
    n = lib().diffqkv_decode_topv_workspace_size(ctypes.byref(dims), t_max, topk)
    if n == 0:
        raise DiffqkvError(_capi.INVALID_ARG, "decode_topv_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def decode_topv(q, k_cache, v_cache, seq_lens, topk: int, *, scale: Optional[float] = None,
                max_seq_len: Optional[int] = None, out=None, idx_out=None, workspace=None,
                full_weights: bool = False, stream: Optional[torch.cuda.Stream] = None):
    """Selective-V decode over the top-k exact-scoring positions of each query head.

    The kept V rows are weighted by the softmax renormalised over them, or with ``full_weights`` by
    the full-softmax weights of every cached position (the others counting as zero).
    Returns (out bf16 [B, n_q, d_v], idx int32 [B, n_q, topk] ascending, -1 padded).
    """
    _bf16_dev(q, "q", 3)
    _bf16_dev(k_cache, "k_cache", 4)
    _bf16_dev(v_cache, "v_cache", 4)
    if seq_lens.dtype != torch.int32 or not seq_lens.is_cuda:
        raise TypeError("seq_lens must be an int32 CUDA tensor")
    dims, t_max = _decode_dims(q, k_cache, v_cache, scale)
    if out is None:
        out = torch.empty((dims.batch, dims.n_q, dims.d_v), dtype=torch.bfloat16, device=q.device)
    if idx_out is None:
        idx_out = torch.empty((dims.batch, dims.n_q, topk), dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = decode_topv_workspace(dims, t_max, topk, q.device)
    msl = t_max if max_seq_len is None else int(max_seq_len)
    if full_weights:
        st = lib().diffqkv_decode_topv_ex(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(seq_lens), t_max, msl, topk, _capi.TOPV_FULL_SOFTMAX_WEIGHTS,
                                          _ptr(out), _ptr(idx_out), _ptr(workspace), workspace.numel(),
                                          _stream_ptr(stream))
    else:
        st = lib().diffqkv_decode_topv(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
                                       t_max, msl, topk, _ptr(out), _ptr(idx_out), _ptr(workspace),
                                       workspace.numel(), _stream_ptr(stream))
    check(st, "diffqkv_decode_topv")
    return out, idx_out


def decode_topv_paged(q, k_pages, v_pages, block_table, seq_lens, topk: int, *, scale: Optional[float] = None,
                      max_seq_len: Optional[int] = None, out=None, idx_out=None, workspace=None,
                      full_weights: bool = False, stream: Optional[torch.cuda.Stream] = None):
    """:func:`decode_topv` over paged caches: K and V page pools [num_pages, page_size, heads, d] and an
    int32 block table [B, max_blocks] of pool pages (position j of sequence b is row j % page_size of pool
    page block_table[b, j // page_size]).  Returns (out, idx) as :func:`decode_topv`."""
    _bf16_dev(q, "q", 3)
    _bf16_dev(k_pages, "k_pages", 4)
    _bf16_dev(v_pages, "v_pages", 4)
    for t, name in ((seq_lens, "seq_lens"), (block_table, "block_table")):
        if t.dtype != torch.int32 or not t.is_cuda:
            raise TypeError(f"{name} must be an int32 CUDA tensor")
    if block_table.dim() != 2 or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous [B, max_blocks] tensor")
    B, n_q, d_k = q.shape
    num_pages, page_size, n_k, _ = k_pages.shape
    n_v, d_v = v_pages.shape[2], v_pages.shape[3]
    max_blocks = block_table.shape[1]
    t_max = max_blocks * page_size
    dims = make_dims(B, n_q, n_k, n_v, d_k, d_v, d_k ** -0.5 if scale is None else scale)
    if out is None:
        out = torch.empty((B, n_q, d_v), dtype=torch.bfloat16, device=q.device)
    if idx_out is None:
        idx_out = torch.empty((B, n_q, topk), dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = decode_topv_workspace(dims, t_max, topk, q.device)
    msl = t_max if max_seq_len is None else int(max_seq_len)
    flags = _capi.TOPV_FULL_SOFTMAX_WEIGHTS if full_weights else 0
    st = lib().diffqkv_decode_topv_paged(ctypes.byref(dims), _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                         max_blocks, page_size, num_pages, _ptr(seq_lens), msl, topk, flags, _ptr(out),
                                         _ptr(idx_out), _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    check(st, "diffqkv_decode_topv_paged")
    return out, idx_out


def prefill_causal(q, k, v, *, scale: Optional[float] = None, out=None, status: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Causal prefill: q [B,S,n_q,d_k], k [B,S,n_k,d_k], v [B,S,n_v,d_v] -> out [B,S,n_q,d_v] (bf16).

    ``status``: an int32 CUDA tensor of one element, zero, that receives this call's device-side
    error instead of the per-device word (``diffqkv_prefill_causal_ex``)."""
    _bf16_dev(q, "q", 4)
    _bf16_dev(k, "k", 4)
    _bf16_dev(v, "v", 4)
    B, S, n_q, d_k = q.shape
    n_k, n_v, d_v = k.shape[2], v.shape[2], v.shape[3]
    if k.shape != (B, S, n_k, d_k) or v.shape[:2] != (B, S):
        raise ValueError("q / k / v shapes disagree")
    dims = make_dims(B, n_q, n_k, n_v, d_k, d_v, d_k ** -0.5 if scale is None else scale)
    if out is None:
        out = torch.empty((B, S, n_q, d_v), dtype=torch.bfloat16, device=q.device)
    if status is not None:
        _status_word(status)
        st = lib().diffqkv_prefill_causal_ex(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), 0, S, _ptr(out),
                                             _ptr(status), _stream_ptr(stream))
    else:
        st = lib().diffqkv_prefill_causal(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), S, _ptr(out),
                                          _stream_ptr(stream))
    check(st, "diffqkv_prefill_causal")
    return out


def prefill_causal_paged(q, k_pages, v_pages, block_table, prefix_len: int, *, scale: Optional[float] = None,
                         out=None, status: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Causal prefill over paged K/V pools: q [B,S,n_q,d_k] for positions prefix_len..prefix_len+S-1;
    k_pages [num_pages, page_size, n_k, d_k], v_pages [num_pages, page_size, n_v, d_v] holding every
    sequence's prefix_len + S positions through block_table [B, max_blocks] (int32) -> [B,S,n_q,d_v]."""
    _bf16_dev(q, "q", 4)
    _bf16_dev(k_pages, "k_pages", 4)
    _bf16_dev(v_pages, "v_pages", 4)
    if block_table.dtype != torch.int32 or not block_table.is_cuda or block_table.dim() != 2 \
            or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous int32 CUDA tensor [B, max_blocks]")
    B, S, n_q, d_k = q.shape
    num_pages, page_size, n_k, d_k2 = k_pages.shape
    n_v, d_v = v_pages.shape[2], v_pages.shape[3]
    if d_k2 != d_k or v_pages.shape[:2] != (num_pages, page_size) or block_table.shape[0] != B:
        raise ValueError("q / k_pages / v_pages / block_table shapes disagree")
    dims = make_dims(B, n_q, n_k, n_v, d_k, d_v, d_k ** -0.5 if scale is None else scale)
    if out is None:
        out = torch.empty((B, S, n_q, d_v), dtype=torch.bfloat16, device=q.device)
    if status is not None:
        _status_word(status)
    st = lib().diffqkv_prefill_causal_paged(ctypes.byref(dims), _ptr(q), _ptr(k_pages), _ptr(v_pages),
                                            _ptr(block_table), block_table.shape[1], page_size, num_pages,
                                            int(prefix_len), S, _ptr(out), _ptr(status), _stream_ptr(stream))
    check(st, "diffqkv_prefill_causal_paged")
    return out


def _status_word(t: torch.Tensor):
    if t.dtype != torch.int32 or not t.is_cuda or t.numel() < 1:
        raise TypeError("status must be an int32 CUDA tensor with at least one element")


def prefill_causal_prefix(q, k, v, prefix_len: int, *, scale: Optional[float] = None, out=None,
                          stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Causal prefill over an existing prefix: q [B,S,n_q,d_k] for positions prefix_len..prefix_len+S-1,
    k [B,P+S,n_k,d_k] and v [B,P+S,n_v,d_v] holding the prefix and the new rows -> out [B,S,n_q,d_v]."""
    _bf16_dev(q, "q", 4)
    _bf16_dev(k, "k", 4)
    _bf16_dev(v, "v", 4)
    B, S, n_q, d_k = q.shape
    n_k, n_v, d_v = k.shape[2], v.shape[2], v.shape[3]
    P = int(prefix_len)
    if k.shape != (B, P + S, n_k, d_k) or v.shape[:2] != (B, P + S):
        raise ValueError("k / v must hold prefix_len + S positions")
    dims = make_dims(B, n_q, n_k, n_v, d_k, d_v, d_k ** -0.5 if scale is None else scale)
    if out is None:
        out = torch.empty((B, S, n_q, d_v), dtype=torch.bfloat16, device=q.device)
    st = lib().diffqkv_prefill_causal_prefix(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), P, S, _ptr(out),
                                             _stream_ptr(stream))
    check(st, "diffqkv_prefill_causal_prefix")
    return out


def workspace_status(workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronises the stream and returns (and clears) the error word of a decode or top-v workspace:
    the first device-side error of the calls that used it since the last read."""
    if workspace.dtype != torch.uint8 or not workspace.is_cuda:
        raise TypeError("workspace must be a uint8 CUDA tensor")
    v = ctypes.c_int32(0)
    check(lib().diffqkv_workspace_status(_ptr(workspace), workspace.numel(), _stream_ptr(stream), ctypes.byref(v)),
          "diffqkv_workspace_status")
    return v.value


def device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronises the stream and returns (and clears) the per-device error word (the calls without a
    word of their own: prefill without ``status``, the allocation-free decode, the wait self-test)."""
    v = ctypes.c_int32(0)
    check(lib().diffqkv_get_device_status(_stream_ptr(stream), ctypes.byref(v)), "diffqkv_get_device_status")
    return v.value


def selftest_wait_timeout(timeout_ns: int, stream: Optional[torch.cuda.Stream] = None) -> None:
    check(lib().diffqkv_selftest_wait_timeout(int(timeout_ns), _stream_ptr(stream)), "diffqkv_selftest_wait_timeout")


def decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, seq_lens: torch.Tensor, *,
                   scale: Optional[float] = None, max_seq_len: Optional[int] = None,
                   out: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """:func:`decode` through ``diffqkv_decode_noalloc``: no workspace argument.

    For callers that cannot hand the library device memory (plugin interfaces
    that only pass inputs and outputs, servers that forbid device allocation
    after start-up).  The library's built-in scratch array is shared by every
    call: calls that can overlap on the GPU must be serialised.  Pass ``out``
    to make the call itself allocate nothing on the Python side either.
    """
    _bf16_dev(q, "q", 3)
    _bf16_dev(k_cache, "k_cache", 4)
    _bf16_dev(v_cache, "v_cache", 4)
    if seq_lens.dtype != torch.int32 or not seq_lens.is_cuda:
        raise TypeError("seq_lens must be an int32 CUDA tensor")
    dims, t_max = _decode_dims(q, k_cache, v_cache, scale)
    if out is None:
        out = torch.empty((dims.batch, dims.n_q, dims.d_v), dtype=torch.bfloat16, device=q.device)
    msl = t_max if max_seq_len is None else int(max_seq_len)
    st = lib().diffqkv_decode_noalloc(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
                                      t_max, msl, _ptr(out), _stream_ptr(stream))
    check(st, "diffqkv_decode_noalloc")
    return out
