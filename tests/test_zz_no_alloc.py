"""rpa_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (an allocator or memory pool servicing a request, a process
whose device memory is reserved up front, a hard memory budget).  It keeps
its plan and split-KV partials in a fixed device array inside the library
instead of the workspace rpa_forward grows with cudaMalloc.

The GPU test calls it through the C ABI twice in a row, on different
batches, and checks each result against rpa_forward on the same inputs
within the parity tolerance (bf16: max-abs 1.5e-2, mean-abs 2e-3, lse 2e-3),
plus bit-identical caches; both batches are also checked against the fp64
oracle (outputs within that tolerance, the cache equal to the oracle's
scatter bit for bit), so that a planning defect both entry points share
would still fail.  The second batch runs without a caller error word, so the
array's own error word (cleared by each call) is used.  This file sorts last
so that a run stopping at the first failure has already run every other
test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from ragged_paged_attention_03_b200 import inputs as I

from harness import TOL, check_close, oracle_full


@pytest.fixture(scope="module")
def rb():
    from ragged_paged_attention_03_b200 import build
    build.build()
    from ragged_paged_attention_03_b200 import binding
    return binding


def _call_host_only(rb, kv, dims):
    """A call whose sizes are rejected before any device is touched (fake
    device pointers, no stream): runs without a GPU."""
    fake = ctypes.c_void_p(0x1000)
    return rb.library().rpa_decode_noalloc(fake, fake, fake, fake, fake, fake,
                                           kv.ctypes.data_as(ctypes.c_void_p), len(kv), 1.0, fake, None,
                                           ctypes.byref(dims), None, None)


def test_rejects_batches_beyond_the_scratch(rb):
    """Too many work items for the fixed array: RPA_ERR_SCRATCH_LIMIT."""
    n = 9000
    kv = np.full(n, 5, np.int32)
    dims = rb.rpa_dims(num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=16, num_pages=n,
                       max_pages_per_seq=1, total_q_tokens=n, dtype=1)
    rc = _call_host_only(rb, kv, dims)
    assert rc == rb.RPA_ERR_SCRATCH_LIMIT
    assert "scratch" in rb.rpa_status_string(rc)


def test_rejects_partials_beyond_the_scratch(rb):
    """Few work items but too many split-KV partial results: with 16 KV heads
    of 16 query heads each at head_dim 256, one split item needs 16 * 16 *
    257 floats, and 10 sequences of 30000 tokens cut into 10 items each
    need 100 of them, more than the ~15.6 MiB of the array hold."""
    kv = np.full(10, 30000, np.int32)
    dims = rb.rpa_dims(num_q_heads=256, num_kv_heads=16, head_dim=256, page_size=16,
                       num_pages=10 * 1875, max_pages_per_seq=1875, total_q_tokens=10, dtype=1)
    assert _call_host_only(rb, kv, dims) == rb.RPA_ERR_SCRATCH_LIMIT
    # the same sequences at 4 KV heads fit (the call would then need a GPU)
    small = rb.rpa_dims(num_q_heads=64, num_kv_heads=4, head_dim=256, page_size=16,
                        num_pages=10 * 1875, max_pages_per_seq=1875, total_q_tokens=10, dtype=1)
    per_partial = 4 * 16 * 257
    assert 100 * per_partial * 4 < (16 << 20) - (1 << 20)   # fits: the size check passes
    assert rb.rpa_plan(np.arange(11, dtype=np.int32), kv, None, small).decode_items == 100


def _run(rb, prob, noalloc, with_flags=True):
    kc, vc = prob.k_cache.clone(), prob.v_cache.clone()
    out = torch.full_like(prob.q, float("nan"))
    lse = torch.full((prob.q.shape[0], prob.num_q_heads), float("nan"), device="cuda")
    if noalloc:
        flags = torch.zeros(1, dtype=torch.int32, device="cuda") if with_flags else None
        rb.rpa_decode_noalloc(prob.q, prob.k_new, prob.v_new, kc, vc, prob.page_table,
                              prob.kv_lens, prob.scale, out, lse, dev_flags=flags)
        torch.cuda.synchronize()
        if flags is not None:
            assert int(flags.item()) == 0
    else:
        rb.rpa_forward(prob.q, prob.k_new, prob.v_new, kc, vc, prob.page_table, prob.cu_q_lens,
                       prob.kv_lens, None, prob.scale, True, out, lse)
        assert rb.rpa_device_status() == 0
    return out, lse, kc, vc


@pytest.mark.gpu
def test_noalloc_matches_forward_on_two_calls_in_a_row(rb):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tol = TOL[I.BF16]
    batches = [
        # long sequences (split into several work items, so the combine and
        # the partial buffers in the fixed array are used), short ones too
        dict(kv=[1, 17, 1500, 4100, 9000, 300, 2048], hq=32, hkv=8, d=128, p=16, seed=31, flags=True),
        # a smaller batch right after: stale scratch contents must not leak;
        # no caller error word, so the array's own one is cleared and used
        dict(kv=[3000, 64, 1025], hq=16, hkv=4, d=256, p=64, seed=32, flags=False),
    ]
    for b in batches:
        prob = I.make_problem([1] * len(b["kv"]), b["kv"], num_q_heads=b["hq"],
                              num_kv_heads=b["hkv"], head_dim=b["d"], page_size=b["p"],
                              dtype=I.BF16, seed=b["seed"], pool=1.25, device="cuda",
                              logical=False)
        o_ref, l_ref, kc_ref, vc_ref = _run(rb, prob, noalloc=False)
        o, l, kc, vc = _run(rb, prob, noalloc=True, with_flags=b["flags"])
        err = (o.float() - o_ref.float()).abs()
        assert torch.isfinite(o.float()).all() and torch.isfinite(l).all()
        assert err.max().item() <= tol["max_abs"] and err.mean().item() <= tol["mean_abs"]
        assert (l - l_ref).abs().max().item() <= tol["lse"]
        assert torch.equal(kc.view(torch.int16), kc_ref.view(torch.int16))
        assert torch.equal(vc.view(torch.int16), vc_ref.view(torch.int16))
        # against the fp64 oracle on the same (pre-call) inputs
        o_or, l_or, kc_or, vc_or = oracle_full(oracle, prob)
        check_close(o.float().cpu().numpy(), o_or, l.cpu().numpy(), l_or, I.BF16,
                    what=f"noalloc vs oracle, batch {b['seed']}")
        assert np.array_equal(I.to_storage(kc), kc_or)
        assert np.array_equal(I.to_storage(vc), vc_or)


@pytest.mark.gpu
def test_noalloc_refuses_stream_capture(rb):
    """The plan is staged in host arrays that later calls rewrite, so a call
    on a capturing stream is refused (before any device work) rather than
    recorded."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    prob = I.make_problem([1, 1], [40, 500], num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=16,
                          dtype=I.BF16, seed=33, pool=1.25, device="cuda", logical=False)
    out = torch.empty_like(prob.q)
    side = torch.cuda.Stream()
    x = torch.zeros(1, device="cuda")
    graph = torch.cuda.CUDAGraph()
    codes = []
    with torch.cuda.graph(graph, stream=side):
        x.add_(1)
        try:
            rb.rpa_decode_noalloc(prob.q, prob.k_new, prob.v_new, prob.k_cache, prob.v_cache,
                                  prob.page_table, prob.kv_lens, prob.scale, out, None, stream=side)
        except rb.RpaError as e:
            codes.append(e.code)
    del graph
    torch.cuda.synchronize()
    assert codes == [1]   # RPA_ERR_INVALID_ARG
