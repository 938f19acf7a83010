"""rpa_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (an allocator or memory pool servicing a request, a process
whose device memory is reserved up front, a hard memory budget).  It keeps
its plan and split-KV partials in a fixed device array inside the library
instead of the workspace rpa_forward grows with cudaMalloc.

The GPU test calls it through the C ABI twice in a row, on different
batches, and checks each result against rpa_forward on the same inputs
within the parity tolerance (bf16: max-abs 1.5e-2, mean-abs 2e-3, lse 2e-3),
plus bit-identical caches.  This file sorts last so that a run stopping at
the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from ragged_paged_attention_03_b200 import inputs as I

from harness import TOL


@pytest.fixture(scope="module")
def rb():
    from ragged_paged_attention_03_b200 import build
    build.build()
    from ragged_paged_attention_03_b200 import binding
    return binding


def test_rejects_batches_beyond_the_scratch(rb):
    """Too many work items for the fixed array: RPA_ERR_SCRATCH_LIMIT, before
    any device is touched (runs without a GPU)."""
    n = 9000
    kv = np.full(n, 5, np.int32)
    dims = rb.rpa_dims(num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=16, num_pages=n,
                       max_pages_per_seq=1, total_q_tokens=n, dtype=1)
    fake = ctypes.c_void_p(0x1000)
    rc = rb.library().rpa_decode_noalloc(fake, fake, fake, fake, fake, fake,
                                         kv.ctypes.data_as(ctypes.c_void_p), n, 1.0, fake, None,
                                         ctypes.byref(dims), None, None)
    assert rc == rb.RPA_ERR_SCRATCH_LIMIT
    assert "scratch" in rb.rpa_status_string(rc)


def _run(rb, prob, noalloc):
    kc, vc = prob.k_cache.clone(), prob.v_cache.clone()
    out = torch.full_like(prob.q, float("nan"))
    lse = torch.full((prob.q.shape[0], prob.num_q_heads), float("nan"), device="cuda")
    if noalloc:
        flags = torch.zeros(1, dtype=torch.int32, device="cuda")
        rb.rpa_decode_noalloc(prob.q, prob.k_new, prob.v_new, kc, vc, prob.page_table,
                              prob.kv_lens, prob.scale, out, lse, dev_flags=flags)
        torch.cuda.synchronize()
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
        dict(kv=[1, 17, 1500, 4100, 9000, 300, 2048], hq=32, hkv=8, d=128, p=16, seed=31),
        # a smaller batch right after: stale scratch contents must not leak
        dict(kv=[3000, 64, 1025], hq=16, hkv=4, d=256, p=64, seed=32),
    ]
    for b in batches:
        prob = I.make_problem([1] * len(b["kv"]), b["kv"], num_q_heads=b["hq"],
                              num_kv_heads=b["hkv"], head_dim=b["d"], page_size=b["p"],
                              dtype=I.BF16, seed=b["seed"], pool=1.25, device="cuda",
                              logical=False)
        o_ref, l_ref, kc_ref, vc_ref = _run(rb, prob, noalloc=False)
        o, l, kc, vc = _run(rb, prob, noalloc=True)
        err = (o.float() - o_ref.float()).abs()
        assert torch.isfinite(o.float()).all() and torch.isfinite(l).all()
        assert err.max().item() <= tol["max_abs"] and err.mean().item() <= tol["mean_abs"]
        assert (l - l_ref).abs().max().item() <= tol["lse"]
        assert torch.equal(kc.view(torch.int16), kc_ref.view(torch.int16))
        assert torch.equal(vc.view(torch.int16), vc_ref.view(torch.int16))
