"""rpa_forward_host: host buffers in and out, copies overlapped with the
kernels group by group.

Against the oracle: outputs within the bf16 / fp32 tolerances and the cache
bit for bit, on batches that stay one group and on batches the library cuts
into several (decode run first, then prefill and chunked sequences one per
group).  Against rpa_forward: the host call must give, bit for bit, what
rpa_forward gives when called on each group of rpa_host_groups with device
tensors, which pins every row / page-table offset of the marshalling.
"""
import numpy as np
import pytest
import torch

from ragged_paged_attention_03_b200 import inputs as I

from harness import check_close, f64, oracle_full, same_bits, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ragged_paged_attention_03_b200 import build
    build.build()


def run_host(prob, pinned=True, lse=True, use_distribution=True):
    """rpa_forward_host over `prob` (host tensors; the caches on the GPU)."""
    from ragged_paged_attention_03_b200 import binding

    def host(t):
        t = t.cpu().contiguous()
        return t.pin_memory() if pinned else t

    q, kn, vn, pt = host(prob.q), host(prob.k_new), host(prob.v_new), host(prob.page_table)
    out = host(torch.full(prob.q.shape, float("nan"), dtype=prob.q.dtype))
    lse_t = host(torch.full((prob.q.shape[0], prob.q.shape[1]), float("nan"))) if lse else None
    kc, vc = prob.k_cache.cuda().clone(), prob.v_cache.cuda().clone()
    stream = torch.cuda.Stream()
    binding.rpa_forward_host(q, kn, vn, kc, vc, pt, prob.cu_q_lens, prob.kv_lens,
                             prob.distribution if use_distribution else None, prob.scale,
                             prob.causal, out, lse_t, stream=stream)
    flags = binding.rpa_device_status(stream)
    return out, lse_t, kc, vc, flags


def groups_of(prob, lse=True):
    from ragged_paged_attention_03_b200 import binding
    dims = binding.make_dims(prob.q, prob.k_cache, prob.page_table)
    return binding.rpa_host_groups(prob.cu_q_lens, dims, lse)


def per_group_device(prob, bounds, use_distribution=True):
    """rpa_forward on each group of `bounds`, device tensors, one stream."""
    from ragged_paged_attention_03_b200 import binding
    dp = to_device(prob)
    out = torch.full_like(dp.q, float("nan"))
    lse = torch.full((dp.q.shape[0], dp.q.shape[1]), float("nan"), device="cuda")
    cu = np.asarray(prob.cu_q_lens, dtype=np.int64)
    kv = np.asarray(prob.kv_lens)
    dist = prob.distribution if use_distribution else None
    for g in range(len(bounds) - 1):
        s0, s1 = int(bounds[g]), int(bounds[g + 1])
        t0, t1 = int(cu[s0]), int(cu[s1])
        if t1 == t0:
            continue
        d = None
        if dist is not None:
            d = [min(max(int(dist[0]), s0), s1) - s0, min(max(int(dist[1]), s0), s1) - s0, s1 - s0]
        binding.rpa_forward(dp.q[t0:t1], dp.k_new[t0:t1], dp.v_new[t0:t1], dp.k_cache, dp.v_cache,
                            dp.page_table[s0:s1].contiguous(), cu[s0:s1 + 1] - t0, kv[s0:s1], d,
                            prob.scale, prob.causal, out[t0:t1], lse[t0:t1])
    assert binding.rpa_device_status() == 0
    return out, lse, dp.k_cache, dp.v_cache


def pipelined_problem(causal=True, seed=31, dtype=I.BF16):
    """20 decode sequences, 2 fresh prefill and 2 chunked sequences of
    900-1100 rows (in that order, so the batch has a distribution): about
    20 MB of copies at 8/2 heads, D 128, which the library cuts into a
    decode group and one group per long sequence."""
    ql = [1] * 20 + [900, 1000, 1100, 950]
    kv = [int(x) for x in np.random.default_rng(seed).integers(40, 3000, 20)] + [900, 1000, 1600, 2100]
    return I.make_problem(ql, kv, num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=16,
                          dtype=dtype, causal=causal, seed=seed, pool=1.3, name="host_pipelined")


def check_vs_oracle(oracle_mod, prob, **kw):
    out_ref, lse_ref, kc_ref, vc_ref = oracle_full(oracle_mod, prob)
    out, lse, kc, vc, flags = run_host(prob, **kw)
    assert flags == 0, f"device error flags {flags:#x}"
    check_close(f64(out), out_ref, None if lse is None else f64(lse),
                None if lse is None else lse_ref, prob.dtype, prob.name)
    assert same_bits(kc, kc_ref) and same_bits(vc, vc_ref), "cache differs from the oracle's"


def test_groups_of_the_pipelined_batch():
    prob = pipelined_problem()
    b = groups_of(prob)
    assert list(b) == [0, 20, 21, 22, 23, 24], b


@pytest.mark.parametrize("causal", [True, False])
def test_pipelined_batch_vs_oracle(oracle_mod, causal):
    check_vs_oracle(oracle_mod, pipelined_problem(causal=causal, seed=31 + causal))


def test_pipelined_batch_f32_vs_oracle(oracle_mod):
    check_vs_oracle(oracle_mod, pipelined_problem(seed=40, dtype=I.F32))


def test_single_group_small_mix_vs_oracle(oracle_mod):
    prob = I.make_problem([1, 1, 1, 200, 40], [300, 17, 1000, 200, 170], num_q_heads=32,
                          num_kv_heads=8, head_dim=128, page_size=16, dtype=I.BF16, seed=2024,
                          pool=1.5, name="host_small")
    assert len(groups_of(prob)) == 2   # one group
    check_vs_oracle(oracle_mod, prob)


def test_pageable_memory_and_no_lse(oracle_mod):
    prob = pipelined_problem(seed=44)
    check_vs_oracle(oracle_mod, prob, pinned=False, lse=False)


@pytest.mark.parametrize("use_distribution", [True, False])
def test_same_bits_as_rpa_forward_per_group(use_distribution):
    prob = pipelined_problem(seed=50)
    if not use_distribution:
        prob.distribution = None
    bounds = groups_of(prob)
    assert len(bounds) > 2
    out, lse, kc, vc, flags = run_host(prob, use_distribution=use_distribution)
    assert flags == 0
    out_d, lse_d, kc_d, vc_d = per_group_device(prob, bounds, use_distribution)
    assert torch.equal(out.view(torch.int16), out_d.cpu().view(torch.int16))
    assert torch.equal(lse.view(torch.int32), lse_d.cpu().view(torch.int32))
    assert same_bits(kc, I.to_storage(kc_d)) and same_bits(vc, I.to_storage(vc_d))


def test_repeated_calls_and_growth(oracle_mod):
    """A small call, then a larger one (the staging buffer grows), then the
    small one again on another stream: every result stays correct."""
    small = I.make_problem([1, 30], [50, 30], num_q_heads=8, num_kv_heads=2, head_dim=128,
                           page_size=16, dtype=I.BF16, seed=60, pool=1.5, name="host_rep_small")
    big = pipelined_problem(seed=61)
    for prob in (small, big, small):
        check_vs_oracle(oracle_mod, prob)


def test_empty_and_zero_length_groups(oracle_mod):
    """q_len = 0 sequences inside a pipelined batch (the last group holds
    only one, so nothing runs or is read back for it), and an empty batch."""
    from ragged_paged_attention_03_b200 import binding
    ql = [1] * 10 + [0, 0] + [900, 0, 800, 0]
    kv = [100] * 10 + [5, 7] + [900, 9, 1200, 3]
    prob = I.make_problem(ql, kv, num_q_heads=16, num_kv_heads=4, head_dim=128, page_size=16,
                          dtype=I.BF16, seed=70, pool=1.3, name="host_zero_len")
    assert list(groups_of(prob)) == [0, 12, 13, 15, 16]
    check_vs_oracle(oracle_mod, prob)
    empty = I.make_problem([], [], num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=16,
                           dtype=I.BF16, seed=71, pool=4, name="host_empty")
    kc = empty.k_cache.cuda()
    binding.rpa_forward_host(empty.q, empty.k_new, empty.v_new, kc, empty.v_cache.cuda(),
                             empty.page_table, empty.cu_q_lens, empty.kv_lens, None, empty.scale,
                             True, empty.q.clone(), None)


def test_calls_on_two_streams(oracle_mod):
    """Two pipelined calls queued back to back on different streams share
    the library's staging buffers; the second must wait for the first, and
    both results must be the oracle's."""
    from ragged_paged_attention_03_b200 import binding
    probs = [pipelined_problem(seed=80), pipelined_problem(seed=81, causal=False)]
    refs = [oracle_full(oracle_mod, p) for p in probs]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    res = []
    for prob, st in zip(probs, streams):
        q, kn, vn, pt = (t.cpu().contiguous().pin_memory() for t in (prob.q, prob.k_new, prob.v_new, prob.page_table))
        out = torch.full(prob.q.shape, float("nan"), dtype=prob.q.dtype).pin_memory()
        lse = torch.full((prob.q.shape[0], prob.q.shape[1]), float("nan")).pin_memory()
        kc, vc = prob.k_cache.cuda().clone(), prob.v_cache.cuda().clone()
        torch.cuda.synchronize()
        binding.rpa_forward_host(q, kn, vn, kc, vc, pt, prob.cu_q_lens, prob.kv_lens, prob.distribution,
                                 prob.scale, prob.causal, out, lse, stream=st)
        res.append((out, lse, kc, vc, (q, kn, vn, pt)))
    for st in streams:
        st.synchronize()
    assert binding.rpa_device_status() == 0
    for prob, (out_ref, lse_ref, kc_ref, vc_ref), (out, lse, kc, vc, _) in zip(probs, refs, res):
        check_close(f64(out), out_ref, f64(lse), lse_ref, prob.dtype, prob.name + " two streams")
        assert same_bits(kc, kc_ref) and same_bits(vc, vc_ref)


def test_serial_groups_option(oracle_mod):
    """RPA_OPT_CONCURRENT_MIXED < 0: every group in order on the caller's
    stream; the results are the oracle's all the same."""
    from ragged_paged_attention_03_b200 import binding
    old = binding.rpa_set_option(binding.RPA_OPT_CONCURRENT_MIXED, -1)
    try:
        check_vs_oracle(oracle_mod, pipelined_problem(seed=90))
    finally:
        binding.rpa_set_option(binding.RPA_OPT_CONCURRENT_MIXED, old)
