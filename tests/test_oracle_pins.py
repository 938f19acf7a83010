"""Pins for the fp64 oracle: facts the pages and the mathematics fix, checked
against formulations that share nothing with the oracle's code.

The pages (arXiv 2604.15464 abstract; RPA talk summary, 00:06:36 and the
FlashAttention / PagedAttention glossary entries) define the method as exact
softmax attention over a paged, ragged batch after the new K/V are written
into the cache.  They print no worked example, so the pins are invariants,
closed forms, special cases, a library reduction (torch SDPA in fp64) and a
brute-force masked softmax.
"""
import math

import numpy as np
import pytest
import torch

from ragged_paged_attention_03_b200 import inputs as I


def run(oracle, prob, causal=None, threads=2):
    kc = I.to_storage(prob.k_cache).copy()
    vc = I.to_storage(prob.v_cache).copy()
    out, lse = oracle.forward(I.to_storage(prob.q), I.to_storage(prob.k_new),
                              I.to_storage(prob.v_new), kc, vc, prob.page_table.numpy(),
                              prob.cu_q_lens, prob.kv_lens, prob.scale,
                              prob.causal if causal is None else causal, prob.dtype, threads)
    return out, lse, kc, vc


def f64(t):
    return t.detach().to(torch.float64).cpu()


def logical_kv(prob, s):
    """Contiguous K/V of sequence s (context then new tokens), fp64, from the
    generator's logical arrays -- never through the page table."""
    a, b = int(prob.cu_q_lens[s]), int(prob.cu_q_lens[s + 1])
    k = torch.cat([f64(prob.ctx_k[s]), f64(prob.k_new[a:b])], 0)
    v = torch.cat([f64(prob.ctx_v[s]), f64(prob.v_new[a:b])], 0)
    return k, v


MIXES = [
    ([1, 1, 50, 17], [37, 100, 50, 80]),   # the tiny mixed workload's lengths
    ([3, 0, 16, 1], [3, 5, 40, 1]),        # q_len 0, kv_len 1, page-aligned
    ([33], [129]),                         # ragged chunked prefill
]


@pytest.mark.parametrize("dtype", [I.F32, I.BF16])
@pytest.mark.parametrize("mix", range(len(MIXES)))
@pytest.mark.parametrize("causal", [True, False])
def test_equals_contiguous_sdpa(oracle_mod, dtype, mix, causal):
    """Library reduction: per sequence, the oracle equals torch SDPA in fp64
    on the contiguous (never paged) K/V, with a bottom-right causal mask
    (standard is_causal when there is no prior context), GQA by repeating
    each KV head over its G query heads; lse equals torch.logsumexp of the
    masked scaled scores."""
    ql, kv = MIXES[mix]
    prob = I.make_problem(ql, kv, num_q_heads=4, num_kv_heads=2, head_dim=32, page_size=8,
                          dtype=dtype, causal=causal, seed=11 + mix, pool=2.0)
    out, lse, _, _ = run(oracle_mod, prob)
    g = prob.num_q_heads // prob.num_kv_heads
    for s in range(prob.num_seqs):
        a, b = int(prob.cu_q_lens[s]), int(prob.cu_q_lens[s + 1])
        if a == b:
            continue
        k, v = logical_kv(prob, s)
        q = f64(prob.q[a:b]).transpose(0, 1)                 # [Hq, q, D]
        k = k.transpose(0, 1).repeat_interleave(g, 0)        # [Hq, kv, D]
        v = v.transpose(0, 1).repeat_interleave(g, 0)
        c = int(prob.kv_lens[s]) - (b - a)
        if causal and c == 0:
            ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True,
                                                                   scale=prob.scale)
            mask = torch.ones(b - a, k.shape[1], dtype=torch.bool).tril()
        else:
            mask = torch.ones(b - a, k.shape[1], dtype=torch.bool)
            if causal:
                mask = mask.tril(diagonal=c)
            ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                                   scale=prob.scale)
        sc = (q @ k.transpose(1, 2)) * prob.scale
        ref_lse = torch.logsumexp(sc.masked_fill(~mask, float("-inf")), dim=-1)
        np.testing.assert_allclose(out[a:b], ref.transpose(0, 1).numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[a:b], ref_lse.transpose(0, 1).numpy(), rtol=0, atol=1e-12)


def test_brute_force_explicit_mask(oracle_mod):
    """An explicit [q_len x kv_len] mask matrix with -inf entries and a
    row-by-row softmax written with Python loops agrees to 1e-12."""
    prob = I.make_problem([1, 5, 3], [6, 5, 9], num_q_heads=2, num_kv_heads=1, head_dim=8,
                          page_size=4, dtype=I.F32, causal=True, seed=5, pool=9)
    out, lse, _, _ = run(oracle_mod, prob)
    for s in range(prob.num_seqs):
        a, b = int(prob.cu_q_lens[s]), int(prob.cu_q_lens[s + 1])
        kvl = int(prob.kv_lens[s])
        c = kvl - (b - a)
        k, v = logical_kv(prob, s)
        k, v = k.numpy(), v.numpy()
        for i in range(b - a):
            mask = [0.0 if j <= c + i else -math.inf for j in range(kvl)]
            for h in range(prob.num_q_heads):
                qrow = f64(prob.q[a + i, h]).numpy()
                sc = [prob.scale * float(sum(qrow[t] * k[j, 0, t] for t in range(8))) + mask[j]
                      for j in range(kvl)]
                mx = max(sc)
                e = [math.exp(x - mx) for x in sc]
                tot = sum(e)
                o = [sum(e[j] * v[j, 0, t] for j in range(kvl)) / tot for t in range(8)]
                np.testing.assert_allclose(out[a + i, h], o, rtol=0, atol=1e-12)
                assert abs(lse[a + i, h] - (mx + math.log(tot))) < 1e-12


@pytest.mark.parametrize("dtype", [I.F32, I.BF16])
def test_page_permutation_invariance(oracle_mod, dtype):
    """Moving every physical page elsewhere in the pool and rewriting the
    page table to match leaves out and lse bit-identical, and the updated
    caches are the same permutation of each other."""
    prob = I.make_problem([1, 7, 20], [30, 7, 45], num_q_heads=4, num_kv_heads=2, head_dim=16,
                          page_size=8, dtype=dtype, causal=True, seed=3, pool=2.0)
    out1, lse1, kc1, vc1 = run(oracle_mod, prob)
    perm = torch.randperm(prob.num_pages, generator=torch.Generator().manual_seed(99))
    k2 = torch.empty_like(prob.k_cache)
    v2 = torch.empty_like(prob.v_cache)
    k2[perm] = prob.k_cache
    v2[perm] = prob.v_cache
    pt2 = perm[prob.page_table.long()].to(torch.int32)
    prob2 = I.Problem(**{**prob.__dict__, "k_cache": k2, "v_cache": v2, "page_table": pt2})
    out2, lse2, kc2, vc2 = run(oracle_mod, prob2)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)
    p = perm.numpy()
    assert np.array_equal(kc2[p].view(np.uint8), kc1.view(np.uint8))
    assert np.array_equal(vc2[p].view(np.uint8), vc1.view(np.uint8))


@pytest.mark.parametrize("dtype", [I.F32, I.BF16])
def test_scatter_logical_view(oracle_mod, dtype):
    """After the call, reading each sequence through its page table gives
    exactly its context followed by its new K/V (bit for bit), and every
    slot outside the sequences' [0, kv_len) ranges is untouched."""
    prob = I.make_problem([1, 1, 50, 17, 0], [37, 100, 50, 80, 9], num_q_heads=4,
                          num_kv_heads=2, head_dim=16, page_size=16, dtype=dtype, seed=1, pool=40)
    pre_k = I.to_storage(prob.k_cache).copy()
    _, _, kc, vc = run(oracle_mod, prob)
    p = prob.page_size
    touched = np.zeros(prob.num_pages * p, dtype=bool)
    flat_k = kc.reshape(prob.num_pages * p, -1)
    flat_v = vc.reshape(prob.num_pages * p, -1)
    for s in range(prob.num_seqs):
        kvl = int(prob.kv_lens[s])
        table = prob.page_table[s].numpy()
        slots = np.array([table[j // p] * p + j % p for j in range(kvl)], dtype=np.int64)
        touched[slots] = True
        a, b = int(prob.cu_q_lens[s]), int(prob.cu_q_lens[s + 1])
        want_k = torch.cat([prob.ctx_k[s], prob.k_new[a:b]], 0).reshape(kvl, -1)
        want_v = torch.cat([prob.ctx_v[s], prob.v_new[a:b]], 0).reshape(kvl, -1)
        assert np.array_equal(flat_k[slots].view(np.uint8), I.to_storage(want_k).view(np.uint8))
        assert np.array_equal(flat_v[slots].view(np.uint8), I.to_storage(want_v).view(np.uint8))
    pre = pre_k.reshape(prob.num_pages * p, -1)
    assert np.array_equal(flat_k[~touched].view(np.uint8), pre[~touched].view(np.uint8))


def test_single_key_gives_v(oracle_mod):
    """kv_len = 1 (a one-token prompt): the only key is the new token, so
    out = its V exactly and lse = scale * q.k."""
    prob = I.make_problem([1, 1], [1, 1], num_q_heads=4, num_kv_heads=2, head_dim=16,
                          page_size=8, dtype=I.BF16, seed=4, pool=4)
    out, lse, _, _ = run(oracle_mod, prob)
    for t in range(2):
        for h in range(4):
            hk = h // 2
            assert np.array_equal(out[t, h], f64(prob.v_new[t, hk]).numpy())
            want = prob.scale * float(np.dot(f64(prob.q[t, h]).numpy(), f64(prob.k_new[t, hk]).numpy()))
            assert abs(lse[t, h] - want) < 1e-12


@pytest.mark.parametrize("causal", [True, False])
def test_constant_scores_give_mean(oracle_mod, causal):
    """q = 0 makes every score 0: out is the plain mean of the visible V rows
    and lse = ln(number of visible keys)."""
    prob = I.make_problem([1, 6, 4], [10, 6, 13], num_q_heads=2, num_kv_heads=1, head_dim=8,
                          page_size=4, dtype=I.F32, causal=causal, seed=8, pool=12)
    prob.q.zero_()
    out, lse, _, _ = run(oracle_mod, prob)
    for s in range(prob.num_seqs):
        a, b = int(prob.cu_q_lens[s]), int(prob.cu_q_lens[s + 1])
        c = int(prob.kv_lens[s]) - (b - a)
        _, v = logical_kv(prob, s)
        for i in range(b - a):
            n = c + i + 1 if causal else int(prob.kv_lens[s])
            for h in range(2):
                np.testing.assert_allclose(out[a + i, h], v[:n, 0].mean(0).numpy(), rtol=0, atol=1e-14)
                assert abs(lse[a + i, h] - math.log(n)) < 1e-14


def test_rows_sum_to_one(oracle_mod):
    """Every row of softmax weights sums to 1, and keys past the causal
    bound get weight exactly 0."""
    prob = I.make_problem([1, 12], [25, 30], num_q_heads=2, num_kv_heads=1, head_dim=16,
                          page_size=8, dtype=I.BF16, causal=True, seed=9, pool=10)
    kc = I.to_storage(prob.k_cache).copy()
    vc = I.to_storage(prob.v_cache).copy()
    pt = prob.page_table.numpy()
    oracle_mod.scatter(I.to_storage(prob.k_new), I.to_storage(prob.v_new), kc, vc, pt,
                       prob.cu_q_lens, prob.kv_lens, 2, prob.dtype)
    for s, i in [(0, 0), (1, 0), (1, 5), (1, 11)]:
        for h in range(2):
            w = oracle_mod.row_weights(I.to_storage(prob.q), kc, vc, pt, prob.cu_q_lens,
                                       prob.kv_lens, prob.scale, True, prob.dtype, s, i, h)
            c = int(prob.kv_lens[s]) - int(prob.q_lens[s])
            assert abs(w.sum() - 1.0) < 1e-12
            assert np.all(w[c + i + 1:] == 0.0) and np.all(w[:c + i + 1] > 0.0)


def test_gqa_equals_mha_with_repeated_heads(oracle_mod):
    """GQA with G = 4 equals plain multi-head attention whose cache and new
    K/V repeat each KV head G times (bit-identical results)."""
    prob = I.make_problem([1, 9, 4], [20, 9, 17], num_q_heads=8, num_kv_heads=2, head_dim=16,
                          page_size=8, dtype=I.BF16, causal=True, seed=12, pool=2.0)
    out1, lse1, _, _ = run(oracle_mod, prob)
    rep = lambda t: t.repeat_interleave(4, dim=-2).contiguous()
    prob2 = I.Problem(**{**prob.__dict__, "num_kv_heads": 8, "k_cache": rep(prob.k_cache),
                         "v_cache": rep(prob.v_cache), "k_new": rep(prob.k_new),
                         "v_new": rep(prob.v_new)})
    out2, lse2, _, _ = run(oracle_mod, prob2)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


def test_affine_in_v(oracle_mod):
    """Softmax weights sum to one, so V -> a V + b maps out -> a out + b and
    leaves lse unchanged."""
    prob = I.make_problem([1, 7], [19, 12], num_q_heads=2, num_kv_heads=1, head_dim=8,
                          page_size=4, dtype=I.F32, causal=True, seed=13, pool=12)
    out1, lse1, _, _ = run(oracle_mod, prob)
    a, b = 2.0, 0.75
    prob2 = I.Problem(**{**prob.__dict__, "v_cache": prob.v_cache * a + b,
                         "v_new": prob.v_new * a + b})
    out2, lse2, _, _ = run(oracle_mod, prob2)
    np.testing.assert_allclose(out2, a * out1 + b, rtol=0, atol=1e-6)
    assert np.array_equal(lse1, lse2)


def test_decode_causal_equals_noncausal(oracle_mod):
    """A single new token sits at the last position, so the causal mask hides
    nothing: causal and non-causal decode agree bit for bit."""
    prob = I.make_problem([1, 1, 1], [5, 33, 64], num_q_heads=4, num_kv_heads=1, head_dim=16,
                          page_size=16, dtype=I.BF16, seed=14, pool=2.0)
    o1, l1, _, _ = run(oracle_mod, prob, causal=True)
    o2, l2, _, _ = run(oracle_mod, prob, causal=False)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_attend_rows_matches_forward(oracle_mod):
    """The sampled-row entry point gives the same bits as the full pass."""
    prob = I.make_workload("tiny_mixed_f32")
    out, lse, kc, vc = run(oracle_mod, prob)
    rows = np.array([0, 1, 2, 30, 51, 68], dtype=np.int32)
    heads = np.array([0, 3, 1, 2, 0, 3], dtype=np.int32)
    o, l = oracle_mod.attend_rows(I.to_storage(prob.q), kc, vc, prob.page_table.numpy(),
                                  prob.cu_q_lens, prob.kv_lens, prob.scale, True, prob.dtype,
                                  rows, heads)
    assert np.array_equal(o, out[rows, heads]) and np.array_equal(l, lse[rows, heads])


def test_rejects_bad_lengths(oracle_mod):
    prob = I.make_problem([2], [5], num_q_heads=1, num_kv_heads=1, head_dim=8, page_size=4,
                          dtype=I.F32, seed=1, pool=4)
    kc = I.to_storage(prob.k_cache).copy()
    vc = I.to_storage(prob.v_cache).copy()
    args = (I.to_storage(prob.q), I.to_storage(prob.k_new), I.to_storage(prob.v_new), kc, vc)
    with pytest.raises(ValueError):   # kv_len < q_len
        oracle_mod.forward(*args, prob.page_table.numpy(), prob.cu_q_lens,
                           np.array([1], np.int32), 1.0, True, I.F32)
    with pytest.raises(ValueError):   # page index outside the pool
        oracle_mod.forward(*args, np.array([[0, 9]], np.int32), prob.cu_q_lens, prob.kv_lens,
                           1.0, True, I.F32)
