"""Host-side checks of the C ABI (no GPU needed): the library loads and
exports every function include/rpa.h declares, validation returns the
documented codes, and the planner's classification and work lists match the
lengths it was given."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from ragged_paged_attention_03_b200 import build as B
from ragged_paged_attention_03_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def rb():
    B.build()
    from ragged_paged_attention_03_b200 import binding
    return binding


def declared_functions():
    src = open(os.path.join(ROOT, "include", "rpa.h")).read()
    return sorted(set(re.findall(r"RPA_API\s+[\w\s\*]*?\b(rpa_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(rb):
    names = declared_functions()
    assert {"rpa_forward", "rpa_device_status", "rpa_status_string", "rpa_plan",
            "rpa_set_option"} <= set(names)
    lib = rb.library()
    for n in names:
        assert hasattr(lib, n), n


def dims(**kw):
    from ragged_paged_attention_03_b200 import binding
    base = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=16, num_pages=1000,
                max_pages_per_seq=64, total_q_tokens=0, dtype=1)
    base.update(kw)
    return binding.rpa_dims(**base)


def plan(rb, q_lens, kv_lens, dist=None, **kw):
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    return rb.rpa_plan(cu, np.array(kv_lens, np.int32), dist,
                       dims(total_q_tokens=int(cu[-1]), **kw))


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), 2), (dict(page_size=12), 2), (dict(page_size=4), 2),
    (dict(num_kv_heads=5), 2), (dict(num_q_heads=64, num_kv_heads=2), 2),
    (dict(dtype=7), 1), (dict(num_pages=0), 1),
])
def test_bad_dims(rb, kw, code):
    with pytest.raises(rb.RpaError) as e:
        plan(rb, [1], [10], **kw)
    assert e.value.code == code


def test_bad_lengths(rb):
    with pytest.raises(rb.RpaError) as e:
        plan(rb, [5], [4])                      # kv_len < q_len
    assert e.value.code == 3
    with pytest.raises(rb.RpaError) as e:
        plan(rb, [1], [64 * 16 + 1])            # more pages than a table row holds
    assert e.value.code == 3
    with pytest.raises(rb.RpaError) as e:       # T disagrees with cu_q_lens
        rb.rpa_plan(np.array([0, 3], np.int32), np.array([3], np.int32), None,
                    dims(total_q_tokens=4))
    assert e.value.code == 3
    with pytest.raises(rb.RpaError) as e:       # cu_q_lens must start at 0
        rb.rpa_plan(np.array([1, 3], np.int32), np.array([3], np.int32), None,
                    dims(total_q_tokens=3))
    assert e.value.code == 3


def test_bad_distribution(rb):
    with pytest.raises(rb.RpaError) as e:       # a 5-token sequence in the decode range
        plan(rb, [1, 5], [9, 5], dist=np.array([2, 2, 2], np.int32))
    assert e.value.code == 4
    with pytest.raises(rb.RpaError) as e:       # chunked sequence in the prefill range
        plan(rb, [1, 5], [9, 9], dist=np.array([1, 2, 2], np.int32))
    assert e.value.code == 4
    with pytest.raises(rb.RpaError) as e:       # counts do not cover the batch
        plan(rb, [1, 5], [9, 9], dist=np.array([1, 1, 3], np.int32))
    assert e.value.code == 4
    info = plan(rb, [1, 5, 3], [9, 5, 9], dist=np.array([1, 2, 3], np.int32))
    assert info.num_decode + info.num_generic + info.num_prefill == 3


def test_empty_batches(rb):
    info = plan(rb, [], [])
    assert info.plan_bytes == 0
    info = plan(rb, [0, 0], [5, 9])
    assert info.num_empty == 2 and info.plan_bytes == 0


def test_fp32_routes_to_generic(rb):
    info = plan(rb, [1, 50, 17], [37, 50, 80], dtype=0)
    assert info.num_generic == 3 and info.num_decode == 0 and info.num_prefill == 0


def test_force_generic_option(rb):
    old = rb.rpa_set_option(rb.RPA_OPT_FORCE_GENERIC, 1)
    try:
        info = plan(rb, [1, 50], [37, 50])
        assert info.num_generic == 2
    finally:
        rb.rpa_set_option(rb.RPA_OPT_FORCE_GENERIC, old)


def test_decode_chunking(rb):
    """Decode work items: ceil(kv_len / 16) blocks per sequence, cut into
    near-equal chunks of at most the chunk size; sequences cut more than
    once need the combine."""
    old = rb.rpa_set_option(rb.RPA_OPT_DECODE_CHUNK_BLOCKS, 8)
    try:
        info = plan(rb, [1, 1, 1], [16 * 8, 16 * 8 + 1, 5])
    finally:
        rb.rpa_set_option(rb.RPA_OPT_DECODE_CHUNK_BLOCKS, old)
    if info.num_decode == 0:
        pytest.skip("decode kernel not routed")
    assert info.decode_items == 1 + 2 + 1
    assert info.combine_rows == 1 and info.decode_max_splits == 2
    # three sequences are too few to pack (they would not fill the GPU)
    assert info.decode_packed == 0


def test_decode_packing(rb):
    """Whole sequences of at most RPA_OPT_DECODE_PACK_BLOCKS blocks (default
    64) run four per CTA, one per warp, when there are enough of them to
    fill 296 CTAs (two per SM); < 0 turns packing off."""
    # 150 of each: 1, 64, 65 and 119 blocks; 8 KV heads -> 38 * 8 = 304 packed CTAs
    kv = [5] * 150 + [16 * 64] * 150 + [16 * 64 + 1] * 150 + [1900] * 150
    info = plan(rb, [1] * len(kv), kv, max_pages_per_seq=128)
    if info.num_decode == 0:
        pytest.skip("decode kernel not routed")
    assert info.decode_packed == 300 and info.decode_items == 600
    # too few short sequences: they stay in the main decode launch
    info = plan(rb, [1] * 4, [5, 16 * 64, 16 * 64 + 1, 1900], max_pages_per_seq=128)
    assert info.decode_packed == 0 and info.decode_items == 4
    old = rb.rpa_set_option(rb.RPA_OPT_DECODE_PACK_BLOCKS, -1)
    try:
        info = plan(rb, [1] * len(kv), kv, max_pages_per_seq=128)
        assert info.decode_packed == 0 and info.decode_items == 600
        rb.rpa_set_option(rb.RPA_OPT_DECODE_PACK_BLOCKS, 1000)     # clamped to 120 blocks
        info = plan(rb, [1] * len(kv), kv, max_pages_per_seq=128)
        assert info.decode_packed == 600
    finally:
        rb.rpa_set_option(rb.RPA_OPT_DECODE_PACK_BLOCKS, old)


def test_workload_plans(rb):
    """Every named workload plans, and each sequence lands in exactly one class."""
    for name in I.WORKLOADS:
        dtype, hq, hkv, d, p, _, _, seed, _ = I.WORKLOADS[name]
        q_lens, kv_lens = I._lengths(name, torch.Generator().manual_seed(seed))
        pages = max((k + p - 1) // p for k in kv_lens)
        cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
        info = rb.rpa_plan(cu, np.array(kv_lens, np.int32), I.classify(q_lens, kv_lens),
                           dims(num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                                max_pages_per_seq=pages, total_q_tokens=int(cu[-1]),
                                num_pages=10 ** 7, dtype=dtype))
        assert info.num_decode + info.num_prefill + info.num_generic + info.num_empty == len(q_lens)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_forward_without_gpu_fails_loudly(rb):
    """Without a usable device rpa_forward returns RPA_ERR_CUDA (nothing is
    computed anywhere else)."""
    lib = rb.library()
    cu = np.array([0, 1], np.int32)
    kv = np.array([4], np.int32)
    d = dims(total_q_tokens=1)
    fake = ctypes.c_void_p(0x1000)
    rc = lib.rpa_forward(fake, fake, fake, fake, fake, fake, cu.ctypes.data_as(ctypes.c_void_p),
                         kv.ctypes.data_as(ctypes.c_void_p), 1, None, 1.0, 1, fake, None,
                         ctypes.byref(d), None)
    assert rc == 6


def test_forward_rejects_before_touching_device(rb):
    lib = rb.library()
    cu = np.array([0, 2], np.int32)
    kv = np.array([1], np.int32)     # kv_len < q_len
    d = dims(total_q_tokens=2)
    fake = ctypes.c_void_p(0x1000)
    rc = lib.rpa_forward(fake, fake, fake, fake, fake, fake, cu.ctypes.data_as(ctypes.c_void_p),
                         kv.ctypes.data_as(ctypes.c_void_p), 1, None, 1.0, 1, fake, None,
                         ctypes.byref(d), None)
    assert rc == 3
    assert rb.rpa_status_string(3) == "invalid sequence lengths"


@pytest.mark.parametrize("scale", [0.0, -0.125, float("nan"), float("inf")])
def test_forward_rejects_non_positive_scale(rb, scale):
    """The scale must be positive and finite (the kernels take row maxima of
    the unscaled scores); anything else is rejected before device work."""
    lib = rb.library()
    cu = np.array([0, 1], np.int32)
    kv = np.array([4], np.int32)
    d = dims(total_q_tokens=1)
    fake = ctypes.c_void_p(0x1000)
    rc = lib.rpa_forward(fake, fake, fake, fake, fake, fake, cu.ctypes.data_as(ctypes.c_void_p),
                         kv.ctypes.data_as(ctypes.c_void_p), 1, None, ctypes.c_float(scale), 1, fake, None,
                         ctypes.byref(d), None)
    assert rc == 1
    rc = lib.rpa_decode_noalloc(fake, fake, fake, fake, fake, fake, kv.ctypes.data_as(ctypes.c_void_p), 1,
                                ctypes.c_float(scale), fake, None, ctypes.byref(d), None, None)
    assert rc == 1


def test_device_workspace_size(rb):
    """The device-planned call's workspace depends on the geometry, the
    sequence capacity and the decode options only, and grows with each."""
    d = dims(total_q_tokens=128, max_pages_per_seq=512)
    assert rb.rpa_device_workspace_size(d, 0) == 256            # the header alone
    sizes = [rb.rpa_device_workspace_size(d, n) for n in (1, 16, 128)]
    assert sizes[0] < sizes[1] < sizes[2]
    assert all(s % 256 == 0 for s in sizes)
    # longer contexts allow more split-KV chunks, hence more partial slots
    assert rb.rpa_device_workspace_size(dims(total_q_tokens=128, max_pages_per_seq=2048), 128) > sizes[2]
    # fp32 runs on the generic kernel: no decode items, no partials
    assert rb.rpa_device_workspace_size(dims(total_q_tokens=128, max_pages_per_seq=512, dtype=0), 128) < sizes[2]
    old = rb.rpa_set_option(rb.RPA_OPT_DECODE_CHUNK_BLOCKS, 16)
    try:
        assert rb.rpa_device_workspace_size(d, 128) > sizes[2]
    finally:
        rb.rpa_set_option(rb.RPA_OPT_DECODE_CHUNK_BLOCKS, old)
    with pytest.raises(rb.RpaError) as e:
        rb.rpa_device_workspace_size(d, -1)
    assert e.value.code == 1
    with pytest.raises(rb.RpaError) as e:
        rb.rpa_device_workspace_size(dims(head_dim=96), 4)
    assert e.value.code == 2


def test_forward_device_host_checks(rb):
    """rpa_forward_device rejects bad scale, pointers and workspaces on the
    host, before anything is queued; an empty capacity is a no-op."""
    lib = rb.library()
    d = dims(total_q_tokens=8)
    need = rb.rpa_device_workspace_size(d, 4)
    fake = ctypes.c_void_p(0x10000)

    def call(ws=fake, ws_bytes=need, scale=1.0, max_seqs=4, cu=fake, dd=d):
        return lib.rpa_forward_device(fake, fake, fake, fake, fake, fake, cu, fake, fake, max_seqs,
                                      ctypes.c_float(scale), 1, fake, None, ctypes.byref(dd), ws, ws_bytes,
                                      None, None)
    assert call(ws_bytes=need - 1) == rb.RPA_ERR_WORKSPACE
    assert call(ws=ctypes.c_void_p(0x10000 + 64)) == rb.RPA_ERR_WORKSPACE    # not 256-byte aligned
    assert call(ws=None) == 1
    assert call(cu=None) == 1
    assert call(scale=0.0) == 1
    assert call(max_seqs=-1) == 1
    assert call(dd=dims(head_dim=96, total_q_tokens=8)) == 2
    assert call(max_seqs=0) == 0                  # no sequence slot: nothing to do
    assert call(dd=dims(total_q_tokens=0)) == 0   # no token row: nothing to do
    assert rb.rpa_status_string(rb.RPA_ERR_WORKSPACE) == "workspace too small or misaligned"


def test_host_groups(rb):
    """The sequence groups rpa_forward_host pipelines: one group under 8 MiB
    of copies, one per long sequence, a decode run kept apart from the long
    sequences after it, in order, covering every sequence."""
    assert list(rb.rpa_host_groups(np.arange(129), dims(total_q_tokens=128))) == [0, 128]
    cu = np.arange(9) * 2048
    assert list(rb.rpa_host_groups(cu, dims(total_q_tokens=16384))) == list(range(9))
    cu = np.concatenate([np.arange(97), 96 + np.arange(1, 5) * 512])
    assert list(rb.rpa_host_groups(cu, dims(total_q_tokens=int(cu[-1])))) == [0, 96, 97, 98, 99, 100]
    cu = np.concatenate([[0], np.cumsum(np.random.default_rng(3).integers(0, 3000, 1000))])
    b = rb.rpa_host_groups(cu, dims(total_q_tokens=int(cu[-1])))
    assert 1 < len(b) - 1 <= rb.RPA_HOST_MAX_GROUPS and b[0] == 0 and b[-1] == 1000
    assert (np.diff(b) > 0).all()
    # 1000 tokens at 8/2 heads: ~5 MB of copies in bf16 (one group), twice
    # that in fp32 (two); lse adds Hq floats per token
    small, d8 = np.array([0, 500, 1000]), dict(total_q_tokens=1000, num_q_heads=8, num_kv_heads=2)
    assert len(rb.rpa_host_groups(small, dims(**d8))) == 2
    assert len(rb.rpa_host_groups(small, dims(dtype=0, **d8))) == 3
    edge = np.array([0, 815, 1630])     # 8 MiB with lse, just under without
    assert len(rb.rpa_host_groups(edge, dims(**dict(d8, total_q_tokens=1630)), True)) == 3
    assert len(rb.rpa_host_groups(edge, dims(**dict(d8, total_q_tokens=1630)), False)) == 2
    with pytest.raises(rb.RpaError) as e:
        rb.rpa_host_groups(np.array([1, 2]), dims(total_q_tokens=2))
    assert e.value.code == 3
    with pytest.raises(rb.RpaError) as e:
        rb.rpa_host_groups(np.array([0, 5, 4]), dims(total_q_tokens=4))
    assert e.value.code == 3


def test_forward_host_checks(rb):
    """rpa_forward_host validates the whole batch on the host before any
    device work, and without a usable device fails with RPA_ERR_CUDA."""
    lib = rb.library()
    fake = ctypes.c_void_p(0x1000)

    def call(q_lens, kv_lens, scale=1.0, ptr=fake, dist=None):
        cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
        kv = np.array(kv_lens, np.int32)
        d = dims(total_q_tokens=int(cu[-1]))
        dp = None if dist is None else np.array(dist, np.int32).ctypes.data_as(ctypes.c_void_p)
        return lib.rpa_forward_host(ptr, fake, fake, fake, fake, fake, cu.ctypes.data_as(ctypes.c_void_p),
                                    kv.ctypes.data_as(ctypes.c_void_p), len(kv_lens), dp, ctypes.c_float(scale),
                                    1, fake, None, ctypes.byref(d), None)
    assert call([2], [1]) == 3                    # kv_len < q_len
    assert call([1], [4], scale=0.0) == 1
    assert call([1], [4], ptr=None) == 1
    assert call([1, 3], [4, 3], dist=[0, 2, 2]) == 4   # sequence 0 is not a fresh prefill
    assert call([], []) == 0                      # empty batch: a no-op
    if not torch.cuda.is_available():
        assert call([1], [4]) == 6
