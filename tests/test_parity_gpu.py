"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small problems: every output row and the whole cache pool compared with the
oracle on the same seeded inputs (outputs within the stated tolerances, the
cache bit for bit).  Full-size workloads, in the launch configuration the
benchmark times: sampled sequences against the oracle (rows and their
pages of the cache), plus whole-pool cache properties that hold at any size.
Unused pages, tail slots and the new tokens' destination slots hold NaN
before the call, so a read of any slot the method must not read shows up.
"""
import numpy as np
import pytest
import torch

from ragged_paged_attention_03_b200 import inputs as I

from harness import (TOL, check_cache_property, check_close, f64, oracle_full, run_gpu,
                      same_bits, to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ragged_paged_attention_03_b200 import build
    build.build()


def full_check(oracle_mod, prob, use_distribution=True):
    out_ref, lse_ref, kc_ref, vc_ref = oracle_full(oracle_mod, prob)
    dp = to_device(prob)
    out, lse, flags = run_gpu(dp, use_distribution=use_distribution)
    assert flags == 0, f"device error flags {flags:#x}"
    errs = check_close(f64(out), out_ref, f64(lse), lse_ref, prob.dtype, prob.name)
    assert same_bits(dp.k_cache, kc_ref), "k_cache differs from the oracle's"
    assert same_bits(dp.v_cache, vc_ref), "v_cache differs from the oracle's"
    return errs


def test_tiny_mixed_f32(oracle_mod):
    """The 4-sequence fp32 mix (decode, decode, prefill, chunked)."""
    full_check(oracle_mod, I.make_workload("tiny_mixed_f32"))


SMALL = [
    # (q_lens, kv_lens, Hq, Hkv, D, P, causal)
    ([1] * 7, [1, 15, 16, 17, 100, 1000, 2049], 32, 8, 128, 16, True),
    ([1] * 5, [1, 7, 8, 9, 300], 16, 4, 256, 64, True),
    ([1] * 4, [63, 64, 65, 700], 8, 8, 64, 8, True),
    ([1] * 3, [50, 513, 1200], 16, 1, 128, 32, True),
    ([2, 127, 128, 129, 300], [2, 127, 128, 129, 300], 32, 8, 128, 16, True),
    ([2, 127, 129, 300], [2, 127, 129, 300], 32, 8, 128, 16, False),
    ([33, 200, 128, 1], [129, 1000, 256, 77], 32, 8, 128, 16, True),
    ([33, 200, 128], [129, 1000, 256], 8, 2, 128, 16, False),
    ([1, 1, 50, 17], [37, 100, 50, 80], 4, 1, 64, 16, True),
    ([130, 1, 64], [130, 900, 200], 16, 4, 256, 64, True),
    ([5, 1, 0, 40], [5, 20, 9, 41], 8, 4, 128, 256, True),
]


@pytest.mark.parametrize("case", range(len(SMALL)))
@pytest.mark.parametrize("dtype", [I.BF16, I.F32])
def test_small_mixes(oracle_mod, case, dtype):
    ql, kv, hq, hkv, d, p, causal = SMALL[case]
    prob = I.make_problem(ql, kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                          dtype=dtype, causal=causal, seed=100 + case, pool=1.5,
                          name=f"small{case}")
    full_check(oracle_mod, prob)


@pytest.mark.parametrize("case,seed", [(10, s) for s in (710, 711, 712, 713, 714, 715)] +
                         [(9, s) for s in (710, 711, 712)] + [(4, s) for s in (710, 711)])
def test_dominant_key_after_context_block(oracle_mod, case, seed):
    """Chunked rows with a few keys, the first in a context block and a
    dominant one among the new tokens: the running max stays at the context
    key (the lazy rescale waits for a 2^8 jump), so the dominant weight is
    above 1 when it is rounded to bf16 for the PV MMA.  The row sum must be
    taken over the same rounded weights for O / l to stay within one bf16
    step of the oracle (these seeds put outputs near 4 on such rows)."""
    ql, kv, hq, hkv, d, p, causal = SMALL[case]
    prob = I.make_problem(ql, kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                          dtype=I.BF16, causal=causal, seed=seed, pool=1.5,
                          name=f"small{case}-seed{seed}")
    full_check(oracle_mod, prob)


def test_without_distribution_and_shuffled_order(oracle_mod):
    """Sequence order and the absence of a distribution change nothing."""
    prob = I.make_problem([40, 1, 1, 300, 17], [90, 33, 1, 300, 17], num_q_heads=32,
                          num_kv_heads=8, head_dim=128, page_size=16, dtype=I.BF16, seed=7,
                          pool=1.3)
    assert prob.distribution is None
    full_check(oracle_mod, prob, use_distribution=False)


@pytest.mark.parametrize("concurrent,sms", [(1, 20), (-1, 0)])
def test_mixed_batch_schedules(oracle_mod, concurrent, sms):
    """A mixed batch with its prefill kernel limited to 20 CTAs on the side
    stream (decode on the caller's stream around it), and the same batch run
    one kernel after the other (RPA_OPT_CONCURRENT_MIXED < 0): both give the
    oracle's results (the default, concurrent on every SM, runs in the other
    mixed tests)."""
    from ragged_paged_attention_03_b200 import binding
    old_c = binding.rpa_set_option(binding.RPA_OPT_CONCURRENT_MIXED, concurrent)
    old_k = binding.rpa_set_option(binding.RPA_OPT_PREFILL_SMS, sms)
    try:
        prob = I.make_problem([1] * 6 + [300, 77], [40, 900, 2100, 1, 17, 300, 300, 500],
                              num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=16,
                              dtype=I.BF16, seed=21, pool=1.3)
        full_check(oracle_mod, prob)
    finally:
        binding.rpa_set_option(binding.RPA_OPT_CONCURRENT_MIXED, old_c)
        binding.rpa_set_option(binding.RPA_OPT_PREFILL_SMS, old_k)


@pytest.mark.parametrize("chunk", [1, 3])
def test_decode_heavy_split_kv(oracle_mod, chunk):
    """Decode sequences cut into many small work items (1 or 3 blocks of 16
    tokens each) merged by the log-sum-exp combine."""
    from ragged_paged_attention_03_b200 import binding
    old = binding.rpa_set_option(binding.RPA_OPT_DECODE_CHUNK_BLOCKS, chunk)
    try:
        prob = I.make_problem([1] * 5, [1, 16, 33, 500, 1000], num_q_heads=16, num_kv_heads=2,
                              head_dim=128, page_size=8, dtype=I.BF16, seed=22, pool=1.3)
        full_check(oracle_mod, prob)
    finally:
        binding.rpa_set_option(binding.RPA_OPT_DECODE_CHUNK_BLOCKS, old)


@pytest.mark.parametrize("chunk,inline", [(1, False), (16, True)])
def test_decode_only_plan_in_or_beyond_launch_parameters(oracle_mod, chunk, inline):
    """A decode-only batch whose work items fit in the launch parameters
    (the inline plan, no upload) and the same batch cut into more items than
    those hold (the plan uploaded to device memory): both paths against the
    oracle."""
    from ragged_paged_attention_03_b200 import binding
    old = binding.rpa_set_option(binding.RPA_OPT_DECODE_CHUNK_BLOCKS, chunk)
    try:
        prob = I.make_problem([1] * 4, [4000, 5000, 3000, 3500], num_q_heads=16, num_kv_heads=2,
                              head_dim=128, page_size=16, dtype=I.BF16, seed=23, pool=1.3)
        d = binding.rpa_dims(num_q_heads=16, num_kv_heads=2, head_dim=128, page_size=16,
                             num_pages=prob.k_cache.shape[0], max_pages_per_seq=prob.page_table.shape[1],
                             total_q_tokens=prob.q.shape[0], dtype=binding.RPA_BF16)
        info = binding.rpa_plan(np.asarray(prob.cu_q_lens, dtype=np.int32),
                                np.asarray(prob.kv_lens, dtype=np.int32), prob.distribution, d)
        assert (info.decode_items <= 900 and info.combine_rows <= 1800) == inline, \
            (info.decode_items, info.combine_rows)
        full_check(oracle_mod, prob)
    finally:
        binding.rpa_set_option(binding.RPA_OPT_DECODE_CHUNK_BLOCKS, old)


@pytest.mark.parametrize("loaders", [1, 2])
@pytest.mark.parametrize("case", [4, 5, 6, 7, 8])
def test_prefill_loader_builds(oracle_mod, loaders, case):
    """Both builds of the head_dim <= 128 prefill kernel (K and V sharing one
    producer warp, or one each), forced through RPA_OPT_PREFILL_LOADERS, on
    fresh and chunked prefill mixes with ragged tails."""
    from ragged_paged_attention_03_b200 import binding
    old = binding.rpa_set_option(binding.RPA_OPT_PREFILL_LOADERS, loaders)
    try:
        ql, kv, hq, hkv, d, p, causal = SMALL[case]
        prob = I.make_problem(ql, kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                              dtype=I.BF16, causal=causal, seed=300 + case, pool=1.5)
        full_check(oracle_mod, prob)
    finally:
        binding.rpa_set_option(binding.RPA_OPT_PREFILL_LOADERS, old)


@pytest.mark.parametrize("loaders", [1, 2])
def test_chunked_prefill_long_context(oracle_mod, loaders):
    """Chunked prefill after a long paged context (the batch shape that picks
    one producer warp per operand), page size 8, with partial blocks at the
    end of the context and of the new rows."""
    from ragged_paged_attention_03_b200 import binding
    old = binding.rpa_set_option(binding.RPA_OPT_PREFILL_LOADERS, loaders)
    try:
        prob = I.make_problem([300, 77, 1], [2100, 1000, 500], num_q_heads=16, num_kv_heads=4,
                              head_dim=128, page_size=8, dtype=I.BF16, seed=41, pool=1.3)
        full_check(oracle_mod, prob)
    finally:
        binding.rpa_set_option(binding.RPA_OPT_PREFILL_LOADERS, old)


MORE = [
    # chunked prefill after a cache, both prefill builds forced below: page 8 and 256, D 64 / 128
    ([300, 1, 129], [1500, 4000, 700], 16, 4, 64, 8, True),
    ([257, 64, 1], [3000, 64, 9000], 32, 8, 128, 256, True),
    ([200, 17], [2600, 900], 8, 8, 128, 32, False),
    # head_dim 256: chunked rows after context, ragged tails, page 64 and 16
    ([130, 3, 1], [1000, 260, 5000], 16, 4, 256, 64, True),
    ([65, 1], [65, 300], 8, 2, 256, 16, False),
    # decode: G = 1 and G = 16 (two 8-head groups per tile), long and short mixed
    ([1] * 6, [1, 2, 4096, 5000, 31, 12000], 8, 8, 128, 16, True),
    ([1] * 4, [9000, 17, 3000, 128], 32, 2, 128, 16, True),
    ([1] * 5, [1, 777, 8000, 64, 20000], 16, 1, 64, 32, True),
]


@pytest.mark.parametrize("loaders", [0, 2])
@pytest.mark.parametrize("case", range(len(MORE)))
def test_more_shapes(oracle_mod, case, loaders):
    """Page sizes, head dims, GQA ratios and length mixes beyond the small
    set, with the prefill kernel build chosen by the planner (0) or the one
    producer warp per operand build forced (2)."""
    from ragged_paged_attention_03_b200 import binding
    ql, kv, hq, hkv, d, p, causal = MORE[case]
    old = binding.rpa_set_option(binding.RPA_OPT_PREFILL_LOADERS, loaders)
    try:
        prob = I.make_problem(ql, kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                              dtype=I.BF16, causal=causal, seed=500 + case, pool=1.3)
        full_check(oracle_mod, prob)
    finally:
        binding.rpa_set_option(binding.RPA_OPT_PREFILL_LOADERS, old)


@pytest.mark.parametrize("pack", [0, -1])
@pytest.mark.parametrize("shape", [(16, 1, 64, 8), (32, 8, 128, 16), (64, 4, 256, 64)])
def test_packed_short_decode(oracle_mod, pack, shape):
    """Short decode sequences run four per CTA (one per warp; the last CTA
    holds one), against the same batch with packing off."""
    from ragged_paged_attention_03_b200 import binding
    hq, hkv, d, p = shape
    old = binding.rpa_set_option(binding.RPA_OPT_DECODE_PACK_BLOCKS, pack)
    try:
        # enough short sequences to be packed (>= 296 packed CTAs); the last CTA holds one
        base = [1, 2, 15, 16, 17, 31, 100, 200, 255, 256, 257, 400, 511]
        n = 4 * (296 // hkv + 1) + 1
        kv = [base[i % len(base)] for i in range(n)]
        prob = I.make_problem([1] * len(kv), kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                              page_size=p, dtype=I.BF16, seed=700 + d, pool=1.5)
        if pack == 0:
            from ragged_paged_attention_03_b200 import binding as rb
            info = rb.rpa_plan(prob.cu_q_lens, prob.kv_lens, None,
                               rb.rpa_dims(num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                                           num_pages=prob.num_pages, max_pages_per_seq=prob.page_table.shape[1],
                                           total_q_tokens=len(kv), dtype=I.BF16))
            assert info.decode_packed == len(kv)
        full_check(oracle_mod, prob)
    finally:
        binding.rpa_set_option(binding.RPA_OPT_DECODE_PACK_BLOCKS, old)


def test_bad_page_is_flagged_not_read(oracle_mod):
    """A page-table entry outside the pool is reported through the device
    error word; the kernels never dereference it."""
    from ragged_paged_attention_03_b200 import binding
    prob = to_device(I.make_problem([1, 3], [40, 3], num_q_heads=8, num_kv_heads=2, head_dim=128,
                                    page_size=16, dtype=I.BF16, seed=3, pool=2.0))
    prob.page_table[0, 1] = prob.num_pages + 5
    out, lse, flags = run_gpu(prob)
    assert flags & binding.RPA_DEV_BAD_PAGE


def sampled_check(oracle_mod, prob_dev, pre_k, pre_v, out, lse, seqs, rows_per_seq=48, seed=0):
    """Oracle on a sub-problem holding only `seqs` (their pages in pre-call
    state), at sampled rows and all heads; plus those pages after the call."""
    sub = I.sub_problem(I.Problem(**{**prob_dev.__dict__, "k_cache": pre_k, "v_cache": pre_v}), seqs)
    kc = I.to_storage(sub.k_cache).copy()
    vc = I.to_storage(sub.v_cache).copy()
    pt = sub.page_table.numpy()
    oracle_mod.scatter(I.to_storage(sub.k_new), I.to_storage(sub.v_new), kc, vc, pt,
                       sub.cu_q_lens, sub.kv_lens, sub.num_q_heads, sub.dtype)
    rng = np.random.default_rng(seed)
    rows, heads, grows = [], [], []
    for j, s in enumerate(seqs):
        a, b = int(sub.cu_q_lens[j]), int(sub.cu_q_lens[j + 1])
        n = b - a
        pick = sorted(set([0, n - 1] + rng.integers(0, n, size=min(n, rows_per_seq)).tolist()))
        for r in pick:
            for h in range(sub.num_q_heads):
                rows.append(a + r)
                heads.append(h)
                grows.append(int(prob_dev.cu_q_lens[s]) + r)
    rows, heads, grows = map(lambda x: np.array(x, np.int32), (rows, heads, grows))
    o_ref, l_ref = oracle_mod.attend_rows(I.to_storage(sub.q), kc, vc, pt, sub.cu_q_lens,
                                          sub.kv_lens, sub.scale, sub.causal, sub.dtype, rows, heads)
    gi = torch.from_numpy(grows.astype(np.int64)).to(out.device)
    hi = torch.from_numpy(heads.astype(np.int64)).to(out.device)
    errs = check_close(f64(out[gi, hi]), o_ref, f64(lse[gi, hi]), l_ref, sub.dtype, prob_dev.name)
    # the sampled sequences' pages after the call equal the oracle's scatter
    p = prob_dev.page_size
    pages = []
    for s in seqs:
        n = (int(prob_dev.kv_lens[s]) + p - 1) // p
        pages += prob_dev.page_table[s, :n].tolist()
    pidx = torch.tensor(pages, dtype=torch.long, device=out.device)
    assert same_bits(prob_dev.k_cache.index_select(0, pidx), kc)
    assert same_bits(prob_dev.v_cache.index_select(0, pidx), vc)
    return errs


FULL = [("decode_128", None), ("prefill_8x2048", True), ("prefill_8x2048", False),
        ("mixed_96d_4c", None), ("long_d256", None)]


@pytest.mark.parametrize("name,causal", FULL, ids=[f"{n}-{c}" for n, c in FULL])
def test_full_size_workloads(oracle_mod, name, causal):
    prob = I.make_workload(name, device="cuda", causal=causal)
    pre_k = prob.k_cache.clone()
    pre_v = prob.v_cache.clone()
    out, lse, flags = run_gpu(prob)
    assert flags == 0, f"device error flags {flags:#x}"
    q_lens = prob.q_lens
    dec = [s for s in range(prob.num_seqs) if q_lens[s] == 1]
    pre = [s for s in range(prob.num_seqs) if q_lens[s] > 1]
    seqs = []
    if dec:
        kvs = prob.kv_lens[dec]
        seqs += sorted({dec[int(np.argmax(kvs))], dec[int(np.argmin(kvs))], dec[len(dec) // 2]})
    if pre:
        seqs += [pre[0], pre[-1]] if len(pre) > 1 else pre
    sampled_check(oracle_mod, prob, pre_k, pre_v, out, lse, seqs)
    check_cache_property(pre_k, pre_v, prob)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
