"""Seeded synthetic inputs for DiffQKV attention workloads.

This module holds shapes and random-number recipes only -- none of the
attention arithmetic.  Both the CUDA path (through tests and the benchmark) and
the fp64 oracle read the very same bytes produced here.

Workload shapes follow the Sigma paper's efficiency study (structured summary
page, "Efficiency Analysis: SIGMA vs. Standard GQA Model"): a DiffQKV layer
with 4 K heads and 16 V heads against a symmetric GQA control with 16/16
heads, here at d_k = 64 / d_v = 128 (GQA control: 128 / 128).  The paper's
timings used activations of a trained model, which are not available;
i.i.d. N(0, 1) bf16 tensors stand in for them.

Recipe (per workload, ``seed`` fixed per workload):
  * seq_lens: uniform context, or -- for the ragged workload -- drawn first
    with ``torch.randint(lo, hi + 1, (B,))`` on a CPU generator seeded ``seed``;
  * q, then K, then V: ``torch.randn(..., dtype=float32)`` on a generator
    seeded ``seed`` on the chosen device, K and V drawn one batch element at a
    time ([t_max, heads, dim] per element), each rounded to bf16 (RNE);
  * optional K scale (the ragged workload uses 0.5, exact in bf16);
  * paged caches: q, then the K pool, then the V pool (one draw each, the
    whole [num_pages, page_size, heads, dim] pool), then a random permutation of the pool pages
    (``torch.randperm`` on the CPU generator seeded ``seed + 1``) dealt out
    in sequence order, ceil((seq_len + 1) / page_size) pages per sequence
    (one spare position for an append) and -1 in the unused table entries.
  * augmented query projection: x [tokens, d_model] ~ N(0, 1) (hidden states
    after the layer's RMSNorm have unit scale), then W_gate, W_up
    [d_inter, d_model] and W_down [d_out, d_inter] ~ N(0, 1 / fan_in) (the usual
    initialisation scale, so the gate and up sums are ~ N(0, 1)), drawn in that
    order on a generator seeded ``seed``, each rounded to bf16.
The CPU and CUDA generators produce different streams; each run feeds the
bytes it generated to both sides.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Shape:
    n_q: int = 16
    n_k: int = 4
    n_v: int = 16
    d_k: int = 64
    d_v: int = 128

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_k)

    @property
    def kv_elems_per_token(self) -> int:
        """Cache elements per cached position: n_k*d_k + n_v*d_v."""
        return self.n_k * self.d_k + self.n_v * self.d_v


DIFFQKV = Shape(16, 4, 16, 64, 128)
GQA_CONTROL = Shape(16, 16, 16, 128, 128)
# The paper's own Sigma-1.5B attention shape (32 query heads, 4 K, 16 V, d = 64).
SIGMA_1P5B_PAPER = Shape(32, 4, 16, 64, 64)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    shape: Shape
    batch: int
    t_max: int
    seed: int
    ragged: Optional[tuple] = None  # (lo, hi) inclusive context lengths
    k_scale: float = 1.0
    topk: int = 0                    # >0: selective-V decode
    page_size: int = 0               # >0: paged caches (random_paged_inputs)

    def seq_lens(self) -> torch.Tensor:
        if self.ragged is None:
            return torch.full((self.batch,), self.t_max, dtype=torch.int32)
        g = torch.Generator().manual_seed(self.seed)
        lo, hi = self.ragged
        return torch.randint(lo, hi + 1, (self.batch,), generator=g).to(torch.int32)

    def with_shape(self, shape: Shape, suffix: str) -> "DecodeWorkload":
        return dataclasses.replace(self, shape=shape, name=self.name + suffix)


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    name: str
    shape: Shape
    batch: int
    seq: int
    seed: int

    def with_shape(self, shape: Shape, suffix: str) -> "PrefillWorkload":
        return dataclasses.replace(self, shape=shape, name=self.name + suffix)


# The five reference workloads.
DECODE_SMALL = DecodeWorkload("decode_b1_t512", DIFFQKV, 1, 512, seed=0)
DECODE_32K = DecodeWorkload("decode_b16_t32768", DIFFQKV, 16, 32768, seed=1)
DECODE_RAGGED = DecodeWorkload("decode_ragged_b8_t16k_131k", DIFFQKV, 8, 131072, seed=2,
                               ragged=(16384, 131072), k_scale=0.5)
PREFILL_8K = PrefillWorkload("prefill_causal_b2_s8192", DIFFQKV, 2, 8192, seed=3)
TOPV_64K = DecodeWorkload("decode_topv_b4_t65536_k1024", DIFFQKV, 4, 65536, seed=4, topk=1024)

DECODE_32K_GQA = DECODE_32K.with_shape(GQA_CONTROL, "_gqa")
DECODE_RAGGED_GQA = DECODE_RAGGED.with_shape(GQA_CONTROL, "_gqa")
PREFILL_8K_GQA = PREFILL_8K.with_shape(GQA_CONTROL, "_gqa")


def _randn_bf16(shape, g: torch.Generator, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, dtype=torch.float32, device=device).to(torch.bfloat16)


def _per_batch(batch: int, inner, g, device) -> torch.Tensor:
    out = torch.empty((batch,) + tuple(inner), dtype=torch.bfloat16, device=device)
    for b in range(batch):
        out[b] = _randn_bf16(inner, g, device)
    return out


def make_decode_inputs(w: DecodeWorkload, device="cpu"):
    """Returns dict(q, k_cache, v_cache, seq_lens, scale, topk) on ``device``.

    q [B, n_q, d_k], k_cache [B, t_max, n_k, d_k], v_cache [B, t_max, n_v, d_v]
    bf16; seq_lens int32 [B]."""
    s = w.shape
    seq_lens = w.seq_lens()
    g = torch.Generator(device=device).manual_seed(w.seed)
    q = _randn_bf16((w.batch, s.n_q, s.d_k), g, device)
    k = _per_batch(w.batch, (w.t_max, s.n_k, s.d_k), g, device)
    if w.k_scale != 1.0:
        k.mul_(w.k_scale)
    v = _per_batch(w.batch, (w.t_max, s.n_v, s.d_v), g, device)
    return dict(q=q, k_cache=k, v_cache=v, seq_lens=seq_lens.to(device), scale=s.scale, topk=w.topk)


def make_prefill_inputs(w: PrefillWorkload, device="cpu"):
    """Returns dict(q, k, v, scale) -- [B, S, heads, dim] bf16 on ``device``."""
    s = w.shape
    g = torch.Generator(device=device).manual_seed(w.seed)
    q = _per_batch(w.batch, (w.seq, s.n_q, s.d_k), g, device)
    k = _per_batch(w.batch, (w.seq, s.n_k, s.d_k), g, device)
    v = _per_batch(w.batch, (w.seq, s.n_v, s.d_v), g, device)
    return dict(q=q, k=k, v=v, scale=s.scale)


def random_decode_inputs(batch, t_max, shape: Shape, seed: int, device="cpu", seq_lens=None,
                         k_scale: float = 1.0):
    """Small ad-hoc decode inputs for tests (same recipe, caller-chosen sizes)."""
    w = DecodeWorkload("adhoc", shape, batch, t_max, seed, k_scale=k_scale)
    d = make_decode_inputs(w, device)
    if seq_lens is not None:
        d["seq_lens"] = torch.as_tensor(seq_lens, dtype=torch.int32).to(device)
    return d


def random_paged_inputs(batch, max_blocks, page_size, shape: Shape, seed: int, seq_lens, device="cpu",
                        spare_pages: int = 0):
    """Paged decode inputs: dict(q, k_pages, v_pages, block_table, seq_lens, scale, num_pages).

    k_pages [num_pages, page_size, n_k, d_k] and v_pages [num_pages, page_size, n_v, d_v] bf16;
    block_table int32 [B, max_blocks] of distinct pool pages in random order, -1 where unused.
    num_pages = the pages the sequences hold plus ``spare_pages`` never referenced."""
    s = shape
    lens = torch.as_tensor(seq_lens, dtype=torch.int32)
    t_max = max_blocks * page_size
    held = [min(max_blocks, (int(t) + 1 + page_size - 1) // page_size) for t in lens.clamp(0, t_max).tolist()]
    num_pages = max(1, sum(held) + spare_pages)
    g = torch.Generator(device=device).manual_seed(seed)
    q = _randn_bf16((batch, s.n_q, s.d_k), g, device)
    k = _randn_bf16((num_pages, page_size, s.n_k, s.d_k), g, device)
    v = _randn_bf16((num_pages, page_size, s.n_v, s.d_v), g, device)
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(seed + 1)).to(torch.int32)
    table = torch.full((batch, max_blocks), -1, dtype=torch.int32)
    at = 0
    for b, n in enumerate(held):
        table[b, :n] = perm[at:at + n]
        at += n
    return dict(q=q, k_pages=k, v_pages=v, block_table=table.to(device), seq_lens=lens.to(device),
                scale=s.scale, num_pages=num_pages)


def random_prefill_inputs(batch, seq, shape: Shape, seed: int, device="cpu"):
    return make_prefill_inputs(PrefillWorkload("adhoc", shape, batch, seq, seed), device)


@dataclasses.dataclass(frozen=True)
class AugQWorkload:
    """Augmented query projection of ``tokens`` hidden states (section 3.2, item 4)."""
    name: str
    tokens: int
    d_model: int
    d_inter: int
    d_out: int
    seed: int


# Sigma-1.5B's attention block: hidden 2048, Q intermediate 3072 (1.5x the hidden size), 32 query heads
# of 64 = 2048 outputs; 16384 tokens = the 2 x 8192 prefill rows.
AUGQ_16K = AugQWorkload("augq_proj_t16384_d2048_i3072_o2048", 16384, 2048, 3072, 2048, seed=5)


def make_augq_inputs(w: AugQWorkload, device="cpu"):
    """Returns dict(x, w_gate, w_up, w_down) on ``device`` (bf16)."""
    g = torch.Generator(device=device).manual_seed(w.seed)
    x = _randn_bf16((w.tokens, w.d_model), g, device)
    out = {"x": x}
    for name, rows, fan_in in (("w_gate", w.d_inter, w.d_model), ("w_up", w.d_inter, w.d_model),
                               ("w_down", w.d_out, w.d_inter)):
        v = torch.randn((rows, fan_in), generator=g, dtype=torch.float32, device=device) * fan_in ** -0.5
        out[name] = v.to(torch.bfloat16)
    return out


def random_augq_inputs(tokens, d_model, d_inter, d_out, seed: int, device="cpu"):
    return make_augq_inputs(AugQWorkload("adhoc", tokens, d_model, d_inter, d_out, seed), device)


def augq_flops(w: AugQWorkload) -> int:
    """FLOPs of the two GEMMs: 2 T d_model (2 d_inter) + 2 T d_inter d_out."""
    return 2 * w.tokens * w.d_model * 2 * w.d_inter + 2 * w.tokens * w.d_inter * w.d_out


# Measurement units (algorithmic traffic/work per step), used by the benchmark.
BF16_BYTES = 2


def decode_kv_bytes(shape: Shape, seq_lens) -> int:
    """Bytes of K and V cache a decode step must read: sum_b T_b * (n_k d_k + n_v d_v) * 2."""
    total = int(torch.as_tensor(seq_lens, dtype=torch.int64).clamp(min=0).sum())
    return total * shape.kv_elems_per_token * BF16_BYTES


def prefill_causal_flops(shape: Shape, batch: int, seq: int) -> int:
    """Causal FLOPs: 2 * B * n_q * S(S+1)/2 * (d_k + d_v)."""
    return 2 * batch * shape.n_q * (seq * (seq + 1) // 2) * (shape.d_k + shape.d_v)
