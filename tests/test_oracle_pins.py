"""Pins for the fp64 oracle against things other than itself.

Each pin is chosen so that a plausible slip in the oracle (a swapped K/V head
map, a wrong scale, a dropped max-shift term, a split chunk lost in the
combine, an off-by-one causal bound, a wrong tie order) fails at least one:
  * the worked head-map example and floor rule printed on the Sigma pages;
  * closed forms (one position, two positions, identical keys, q = 0);
  * PyTorch's fp64 SDPA (math backend) on K/V expanded with repeat_interleave
    -- MHA, MQA, GQA and full DiffQKV shapes;
  * the kv_group_sharing equivalence (duplicate K heads up to n_v);
  * split-count independence of the split/combine form;
  * causal SDPA for prefill, and prefill row i == decode over i+1 positions;
  * exact rational arithmetic (fractions.Fraction) for the superaccumulator and
    brute-force top-k on tiny inputs, with ties built on purpose.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads as wl
from workloads import Shape

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def _sdpa_decode(d, shape: Shape):
    """Library reference: fp64 SDPA over heads expanded with repeat_interleave."""
    q = d["q"].double()                       # [B, n_q, d_k]
    k = d["k_cache"].double()                 # [B, T, n_k, d_k]
    v = d["v_cache"].double()
    B = q.shape[0]
    outs = []
    for b in range(B):
        T = int(d["seq_lens"][b])
        kb = k[b, :T].permute(1, 0, 2).repeat_interleave(shape.n_q // shape.n_k, dim=0)
        vb = v[b, :T].permute(1, 0, 2).repeat_interleave(shape.n_q // shape.n_v, dim=0)
        o = F.scaled_dot_product_attention(q[b][:, None, :], kb, vb, scale=d["scale"])
        outs.append(o[:, 0, :])
    return torch.stack(outs).numpy()


# ---------------------------------------------------------------- head map
def test_head_map_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "head_map_sigma_1p5b.json")))
    s = g["shape"]
    for row in g["worked_example"]:
        assert oracle.head_map(s["n_q"], s["n_k"], row["idx_q"]) == row["idx_k"]
        assert oracle.head_map(s["n_q"], s["n_v"], row["idx_q"]) == row["idx_v"]
    for i in range(s["n_q"]):
        assert oracle.head_map(s["n_q"], s["n_k"], i) == i // g["k_group_size"]
        assert oracle.head_map(s["n_q"], s["n_v"], i) == i // g["v_group_size"]


@pytest.mark.parametrize("n_q", [1, 2, 4, 8, 12, 16, 24, 32, 64])
def test_head_map_floor_equals_group_division(n_q):
    # floor(h * n_kv / n_q) equals h // (n_q // n_kv) whenever n_kv divides n_q
    for n_kv in range(1, n_q + 1):
        if n_q % n_kv:
            continue
        for h in range(n_q):
            assert oracle.head_map(n_q, n_kv, h) == h // (n_q // n_kv)


def test_kv_cache_element_counts():
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_elements.json")))
    for key in ("sigma_1p5b", "gqa_std"):
        c = g[key]
        s = Shape(32, c["n_k"], c["n_v"], c["d_k"], c["d_v"])
        assert s.kv_elems_per_token == c["elements_per_token"]
    red = 1 - g["sigma_1p5b"]["elements_per_token"] / g["gqa_std"]["elements_per_token"]
    assert red == pytest.approx(g["reduction"], abs=0)


# ---------------------------------------------------------------- closed forms
def test_single_position_returns_v0():
    d = wl.random_decode_inputs(2, 5, wl.DIFFQKV, seed=11, seq_lens=[1, 1])
    o = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])
    for b in range(2):
        for h in range(16):
            vh = h * 16 // 16
            assert np.array_equal(o[b, h], d["v_cache"][b, 0, vh].double().numpy())


def test_two_positions_sigmoid_form():
    d = wl.random_decode_inputs(1, 2, wl.DIFFQKV, seed=12)
    o = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])
    q, k, v = d["q"].double(), d["k_cache"].double(), d["v_cache"].double()
    for h in range(16):
        kh, vh = h // 4, h
        s0 = float(q[0, h] @ k[0, 0, kh]) * d["scale"]
        s1 = float(q[0, h] @ k[0, 1, kh]) * d["scale"]
        a0 = 1.0 / (1.0 + math.exp(s1 - s0))
        want = a0 * v[0, 0, vh].numpy() + (1 - a0) * v[0, 1, vh].numpy()
        np.testing.assert_allclose(o[0, h], want, rtol=0, atol=1e-12)


def test_identical_keys_and_zero_query_give_mean_of_values():
    d = wl.random_decode_inputs(1, 37, wl.DIFFQKV, seed=13)
    d["k_cache"][:] = d["k_cache"][:, :1]      # every cached key identical
    o = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])
    mean = d["v_cache"][0].double().mean(dim=0).numpy()  # [n_v, d_v]
    np.testing.assert_allclose(o[0], mean, rtol=0, atol=1e-12)
    d2 = wl.random_decode_inputs(1, 37, wl.DIFFQKV, seed=14)
    d2["q"].zero_()
    o2 = oracle.decode(d2["q"], d2["k_cache"], d2["v_cache"], d2["seq_lens"], d2["scale"])
    np.testing.assert_allclose(o2[0], d2["v_cache"][0].double().mean(dim=0).numpy(), atol=1e-12)


def test_weights_sum_to_one():
    d = wl.random_decode_inputs(2, 300, wl.DIFFQKV, seed=15, seq_lens=[300, 123])
    d["v_cache"].fill_(1.0)
    o = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-12)


def test_empty_context_gives_zero_row():
    d = wl.random_decode_inputs(2, 8, wl.DIFFQKV, seed=16, seq_lens=[0, 8])
    o = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])
    assert np.all(o[0] == 0.0) and np.all(np.isfinite(o[1]))


# ---------------------------------------------------------------- library SDPA
SHAPES = {
    "mha": Shape(8, 8, 8, 64, 64),
    "mqa": Shape(8, 1, 1, 64, 64),
    "gqa": Shape(16, 4, 4, 128, 128),
    "diffqkv": wl.DIFFQKV,
    "diffqkv_paper_1p5b": wl.SIGMA_1P5B_PAPER,
    "k_more_than_v": Shape(16, 8, 2, 64, 128),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_decode_matches_fp64_sdpa(name):
    shape = SHAPES[name]
    d = wl.random_decode_inputs(3, 97, shape, seed=21, seq_lens=[97, 1, 50])
    o = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])
    np.testing.assert_allclose(o, _sdpa_decode(d, shape), rtol=0, atol=1e-12)


def test_wrong_scale_would_be_caught():
    # guards the SDPA pin itself: a different scale must move the output
    d = wl.random_decode_inputs(1, 64, wl.DIFFQKV, seed=22)
    o = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"] * 1.01)
    assert np.max(np.abs(o - _sdpa_decode(d, wl.DIFFQKV))) > 1e-6


def test_kv_group_sharing_equivalence():
    """Duplicating each K head n_v/n_k times (the pages' compatibility wrapper)
    turns DiffQKV into GQA with n_k = n_v; the outputs must agree."""
    s = wl.DIFFQKV
    d = wl.random_decode_inputs(2, 80, s, seed=23, seq_lens=[80, 41])
    native = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])
    k_dup = d["k_cache"].repeat_interleave(s.n_v // s.n_k, dim=2).contiguous()
    wrapped = oracle.decode(d["q"], k_dup, d["v_cache"], d["seq_lens"], d["scale"])
    np.testing.assert_allclose(native, wrapped, rtol=0, atol=1e-12)


@pytest.mark.parametrize("splits", [1, 2, 7, 64, 211, 300])
def test_split_count_independence(splits):
    d = wl.random_decode_inputs(2, 211, wl.DIFFQKV, seed=24, seq_lens=[211, 5])
    ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])
    got = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"], num_splits=splits)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_rows_subset_matches_full():
    d = wl.random_decode_inputs(2, 50, wl.DIFFQKV, seed=25)
    full = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])
    rows = [(1, 15), (0, 3), (1, 0)]
    sub = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"], rows=rows)
    for r, (b, h) in enumerate(rows):
        assert np.array_equal(sub[r], full[b, h])


# ---------------------------------------------------------------- prefill
@pytest.mark.parametrize("name", ["diffqkv", "gqa", "mha", "k_more_than_v"])
def test_prefill_matches_causal_sdpa(name):
    shape = SHAPES[name]
    d = wl.random_prefill_inputs(2, 45, shape, seed=31)
    o = oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"])
    q = d["q"].double().permute(0, 2, 1, 3)
    k = d["k"].double().permute(0, 2, 1, 3).repeat_interleave(shape.n_q // shape.n_k, dim=1)
    v = d["v"].double().permute(0, 2, 1, 3).repeat_interleave(shape.n_q // shape.n_v, dim=1)
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=d["scale"])
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def test_prefill_row_equals_decode_over_prefix():
    s = wl.DIFFQKV
    d = wl.random_prefill_inputs(1, 33, s, seed=32)
    o = oracle.prefill_causal(d["q"], d["k"], d["v"], d["scale"])
    assert np.array_equal(o[0, 0], np.repeat(d["v"][0, 0].double().numpy(), s.n_q // s.n_v, axis=0))
    for i in (0, 1, 17, 32):
        dec = oracle.decode(d["q"][:, i], d["k"], d["v"], torch.tensor([i + 1], dtype=torch.int32),
                            d["scale"])
        assert np.array_equal(dec[0], o[0, i])


# ---------------------------------------------------------------- superaccumulator
def _frac(x):
    return Fraction(float(torch.as_tensor(x).float()))


def _frac_dot(a, b):
    return sum((_frac(x) * _frac(y) for x, y in zip(a, b)), Fraction(0))


def _bits_to_bf16(bits):
    return torch.from_numpy(np.asarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def test_superaccumulator_random_vectors():
    g = torch.Generator().manual_seed(41)
    for n in (1, 7, 64, 128, 1000):
        a = torch.randn(n, generator=g).to(torch.bfloat16)
        b = torch.randn(n, generator=g).to(torch.bfloat16)
        assert oracle.exact_dot(a, b) == _frac_dot(a, b)


def test_superaccumulator_adversarial_exponents():
    rng = np.random.default_rng(42)
    for trial in range(200):
        n = int(rng.integers(1, 80))
        # any finite bf16 pattern: exponent fields 0..254, random signs/mantissas
        e = rng.integers(0, 255, size=(2, n))
        m = rng.integers(0, 128, size=(2, n))
        sgn = rng.integers(0, 2, size=(2, n))
        bits = (sgn << 15) | (e << 7) | m
        a, b = _bits_to_bf16(bits[0]), _bits_to_bf16(bits[1])
        assert oracle.exact_dot(a, b) == _frac_dot(a, b), trial
    # exact cancellation: huge + tiny - huge leaves the tiny term
    huge, tiny = 2.0 ** 120, 2.0 ** -130
    a = _bf([huge, tiny, -huge])
    b = _bf([1.0, 2.0 ** -3, 1.0])
    assert oracle.exact_dot(a, b) == Fraction(2) ** -133


# ---------------------------------------------------------------- selective V (top-k)
def _brute_topk(d, b, h, k, shape):
    T = int(d["seq_lens"][b])
    kh = h // (shape.n_q // shape.n_k)
    keys = [(_frac_dot(d["q"][b, h], d["k_cache"][b, j, kh]), j) for j in range(T)]
    keys.sort(key=lambda t: (-t[0], t[1]))
    return sorted(j for _, j in keys[:k])


def _masked_sdpa(d, b, h, sel, shape):
    kh, vh = h // (shape.n_q // shape.n_k), h // (shape.n_q // shape.n_v)
    T = int(d["seq_lens"][b])
    q = d["q"][b, h].double()[None, None, None]
    k = d["k_cache"][b, :T, kh].double()[None, None]
    v = d["v_cache"][b, :T, vh].double()[None, None]
    mask = torch.full((T,), float("-inf"), dtype=torch.float64)
    mask[list(sel)] = 0.0
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask[None, None, None], scale=d["scale"])[0, 0, 0].numpy()


def test_topv_index_sets_match_brute_force_and_masked_sdpa():
    s = wl.DIFFQKV
    d = wl.random_decode_inputs(2, 90, s, seed=51, seq_lens=[90, 33])
    k = 10
    out, idx = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], k, d["scale"])
    for b in range(2):
        for h in range(s.n_q):
            want = _brute_topk(d, b, h, k, s)
            assert idx[b, h].tolist() == want
            np.testing.assert_allclose(out[b, h], _masked_sdpa(d, b, h, want, s), atol=1e-12, rtol=0)


def test_topv_ties_go_to_lower_index():
    s = wl.DIFFQKV
    d = wl.random_decode_inputs(1, 40, s, seed=52)
    # positions 5, 9, 20 and 33 share one key; position 7 another, duplicated at 30
    for j in (9, 20, 33):
        d["k_cache"][0, j] = d["k_cache"][0, 5]
    d["k_cache"][0, 30] = d["k_cache"][0, 7]
    for k in (1, 2, 3, 5, 8):
        _, idx = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], k, d["scale"])
        for h in range(s.n_q):
            assert idx[0, h].tolist() == _brute_topk(d, 0, h, k, s)


def test_topv_k_at_least_context_equals_full_decode():
    s = wl.DIFFQKV
    d = wl.random_decode_inputs(2, 64, s, seed=53, seq_lens=[64, 20])
    full = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], d["scale"])
    out, idx = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], 70, d["scale"])
    np.testing.assert_allclose(out, full, rtol=0, atol=1e-12)
    assert idx[0, 0].tolist() == list(range(64)) + [-1] * 6
    assert idx[1, 3].tolist() == list(range(20)) + [-1] * 50


def test_topv_k1_is_argmax_row_and_weights_renormalise():
    s = wl.DIFFQKV
    d = wl.random_decode_inputs(1, 77, s, seed=54)
    out, idx = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], 1, d["scale"])
    for h in range(s.n_q):
        j = _brute_topk(d, 0, h, 1, s)[0]
        assert idx[0, h, 0] == j
        assert np.array_equal(out[0, h], d["v_cache"][0, j, h].double().numpy())
    d["v_cache"].fill_(1.0)
    out, _ = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], 9, d["scale"])
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-12)


def _zeroed_v_sdpa(d, b, h, sel, shape):
    """Full softmax over every cached position, with the V rows outside `sel` set to zero."""
    kh, vh = h // (shape.n_q // shape.n_k), h // (shape.n_q // shape.n_v)
    T = int(d["seq_lens"][b])
    q = d["q"][b, h].double()[None, None, None]
    k = d["k_cache"][b, :T, kh].double()[None, None]
    v = d["v_cache"][b, :T, vh].double().clone()
    keep = torch.zeros(T, dtype=torch.bool)
    keep[list(sel)] = True
    v[~keep] = 0.0
    return F.scaled_dot_product_attention(q, k, v[None, None], scale=d["scale"])[0, 0, 0].numpy()


def test_topv_full_weights_equals_full_softmax_with_other_v_rows_zeroed():
    """The pages' formula: kept rows weighted by the full-softmax alpha_j, the rest counting as zero."""
    s = wl.DIFFQKV
    d = wl.random_decode_inputs(2, 90, s, seed=55, seq_lens=[90, 41])
    k = 12
    out, idx = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], k, d["scale"],
                                  full_weights=True)
    _, idx_renorm = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], k, d["scale"])
    assert np.array_equal(idx, idx_renorm)
    for b in range(2):
        for h in range(s.n_q):
            want = _brute_topk(d, b, h, k, s)
            assert idx[b, h].tolist() == want
            np.testing.assert_allclose(out[b, h], _zeroed_v_sdpa(d, b, h, want, s), atol=1e-12, rtol=0)


def test_topv_full_weights_sum_to_the_kept_mass():
    s = wl.DIFFQKV
    d = wl.random_decode_inputs(1, 60, s, seed=56)
    d["v_cache"].fill_(1.0)
    out, _ = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], 5, d["scale"], full_weights=True)
    assert np.all(out < 1.0) and np.all(out > 0.0)  # 5 of 60 positions: a strict part of the mass
    out, _ = oracle.decode_topv(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], 60, d["scale"], full_weights=True)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- paged caches

def _scatter_to_pages(cache, seq_lens, page_size, max_blocks, perm):
    """Test-side inverse of the paged layout: cache [B, T, H, D] into a pool whose page for logical
    page p of sequence b is perm[b * max_blocks + p], written position by position."""
    B, T, H, D = cache.shape
    pool = torch.zeros(B * max_blocks, page_size, H, D, dtype=cache.dtype)
    table = torch.full((B, max_blocks), -1, dtype=torch.int32)
    for b in range(B):
        for j in range(int(seq_lens[b])):
            page = int(perm[b * max_blocks + j // page_size])
            table[b, j // page_size] = page
            pool[page, j % page_size] = cache[b, j]
    return pool, table


@pytest.mark.parametrize("page_size", [1, 3, 16, 40])
def test_gather_paged_inverts_a_scatter(page_size):
    s = wl.DIFFQKV
    t_max = 120
    max_blocks = -(-t_max // page_size)
    d = wl.random_decode_inputs(3, max_blocks * page_size, s, seed=61, seq_lens=[120, 0, 47])
    perm = torch.randperm(3 * max_blocks, generator=torch.Generator().manual_seed(62))
    for name in ("k_cache", "v_cache"):
        pool, table = _scatter_to_pages(d[name], d["seq_lens"], page_size, max_blocks, perm)
        got = oracle.gather_paged(pool, table, d["seq_lens"])
        assert got.shape == d[name].shape
        for b, T in enumerate(d["seq_lens"].tolist()):
            assert torch.equal(got[b, :T], d[name][b, :T])
            assert not got[b, T:].float().any()


def test_gather_paged_one_page_per_sequence_is_the_pool():
    """page_size = t_max with table[b] = [b]: the pool already is the contiguous cache."""
    s = wl.DIFFQKV
    d = wl.random_decode_inputs(2, 33, s, seed=63)
    table = torch.arange(2, dtype=torch.int32)[:, None]
    assert torch.equal(oracle.gather_paged(d["v_cache"], table, d["seq_lens"]), d["v_cache"])


def test_gather_paged_rejects_a_bad_entry():
    pool = torch.zeros(4, 8, 1, 8, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError):
        oracle.gather_paged(pool, torch.tensor([[0, 4]], dtype=torch.int32), torch.tensor([9], dtype=torch.int32))
    # an entry past the sequence's pages is never read
    oracle.gather_paged(pool, torch.tensor([[0, -7]], dtype=torch.int32), torch.tensor([8], dtype=torch.int32))


def test_decode_paged_matches_sdpa_over_the_pages():
    """Paged decode against library SDPA on K/V rows looked up straight from the pools."""
    s = wl.DIFFQKV
    d = wl.random_paged_inputs(2, 5, 16, s, seed=64, seq_lens=[70, 33])
    out = oracle.decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], d["scale"])
    for b, T in enumerate(d["seq_lens"].tolist()):
        pages = d["block_table"][b].long()
        pos = torch.arange(T)
        k = d["k_pages"][pages[pos // 16], pos % 16].double()   # [T, n_k, d_k]
        v = d["v_pages"][pages[pos // 16], pos % 16].double()
        k = k.repeat_interleave(s.n_q // s.n_k, dim=1).transpose(0, 1)[:, None]   # [n_q, 1, T, d_k]
        v = v.repeat_interleave(s.n_q // s.n_v, dim=1).transpose(0, 1)[:, None]
        ref = F.scaled_dot_product_attention(d["q"][b].double()[:, None, None], k, v, scale=d["scale"])
        np.testing.assert_allclose(out[b], ref[:, 0, 0].numpy(), atol=1e-12, rtol=0)


# ---------------------------------------------------------------- query and key of different widths

def _up_inputs(seed, d_q, w_heads, shape=wl.DIFFQKV, T=40):
    d = wl.random_decode_inputs(2, T, shape, seed=seed, seq_lens=[T, T // 2 + 1])
    g = torch.Generator().manual_seed(seed + 1)
    q_aug = torch.randn(2, shape.n_q, d_q, generator=g).to(torch.bfloat16)
    w = (torch.randn(w_heads, d_q, shape.d_k, generator=g) / math.sqrt(shape.d_k)).to(torch.bfloat16)
    return d, q_aug, w


@pytest.mark.parametrize("w_heads", [1, 4])
def test_up_projected_decode_matches_sdpa_on_projected_keys(w_heads):
    """The pages' order: every K row projected up to d_q, then SDPA in fp64 (library routine)."""
    s, d_q = wl.DIFFQKV, 96
    d, q_aug, w = _up_inputs(71, d_q, w_heads)
    scale = d_q ** -0.5
    out = oracle.decode_up_projected(q_aug, w, d["k_cache"], d["v_cache"], d["seq_lens"], scale)
    Wg = w.double().expand(s.n_k, -1, -1)                      # [n_k, d_q, d_k]
    for b, T in enumerate(d["seq_lens"].tolist()):
        kup = torch.einsum("grc,tgc->tgr", Wg, d["k_cache"][b, :T].double())          # [T, n_k, d_q]
        kup = kup.repeat_interleave(s.n_q // s.n_k, dim=1).transpose(0, 1)[:, None]  # [n_q, 1, T, d_q]
        v = d["v_cache"][b, :T].double().repeat_interleave(s.n_q // s.n_v, dim=1).transpose(0, 1)[:, None]
        ref = F.scaled_dot_product_attention(q_aug[b].double()[:, None, None], kup, v, scale=scale)
        np.testing.assert_allclose(out[b], ref[:, 0, 0].numpy(), atol=1e-12, rtol=0)


def test_fold_query_moves_the_projection_onto_the_query():
    """fold = einsum over each query head's K-head matrix, and <W^T q, k> = <q, W k> for every key."""
    s, d_q = wl.DIFFQKV, 96
    d, q_aug, w = _up_inputs(72, d_q, 4)
    f = oracle.fold_query(q_aug, w, s.n_k)                     # [B, n_q, d_k]
    Wh = w.double()[torch.arange(s.n_q) // (s.n_q // s.n_k)]  # [n_q, d_q, d_k]
    np.testing.assert_allclose(f, torch.einsum("bhr,hrc->bhc", q_aug.double(), Wh).numpy(), atol=1e-12, rtol=0)
    kk = d["k_cache"].double()[:, :, torch.arange(s.n_q) // (s.n_q // s.n_k)]   # [B, T, n_q, d_k]
    folded = torch.einsum("bhc,bthc->bth", torch.from_numpy(f), kk)
    projected = torch.einsum("bhr,bthr->bth", q_aug.double(), torch.einsum("hrc,bthc->bthr", Wh, kk))
    np.testing.assert_allclose(folded.numpy(), projected.numpy(), atol=1e-10, rtol=0)


def test_fold_query_identity_and_shared_matrix():
    s = wl.DIFFQKV
    q = wl.random_decode_inputs(2, 1, s, seed=73)["q"]
    eye = torch.eye(s.d_k).to(torch.bfloat16)[None]
    np.testing.assert_array_equal(oracle.fold_query(q, eye, s.n_k), q.double().numpy())
    _, q_aug, w = _up_inputs(74, 40, 1)
    shared = oracle.fold_query(q_aug, w, s.n_k)
    np.testing.assert_array_equal(shared, oracle.fold_query(q_aug, w.expand(s.n_k, -1, -1).contiguous(), s.n_k))
