"""rpa_forward_device: the planner on the GPU, lengths in device memory,
kernels launched with capacity-sized grids.

Parity with the fp64 oracle on the small mixes (rows past the batch's last
token and sequences past num_seqs must stay untouched), replay of one
captured CUDA graph over batches of different shapes, the device-side
length checks, and bit-for-bit agreement with the host-planned rpa_forward
on the full-size workloads (both paths make the same per-sequence splits and
tiles, so every output element goes through the same arithmetic).
"""
import numpy as np
import pytest
import torch

from ragged_paged_attention_03_b200 import inputs as I

from harness import check_close, f64, oracle_full, run_gpu, same_bits, to_device
from test_parity_gpu import MORE, SMALL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ragged_paged_attention_03_b200 import build
    build.build()


class Slots:
    """Capacity-sized device buffers of one captured call: T rows of tokens,
    S sequence slots, the page pool and page table of `proto`."""

    def __init__(self, proto: I.Problem, cap_tokens: int, cap_seqs: int, max_pages: int):
        from ragged_paged_attention_03_b200 import binding as rb
        dev = "cuda"
        hq, hkv, d = proto.q.shape[1], proto.k_new.shape[1], proto.q.shape[2]
        dt = proto.q.dtype
        self.q = torch.zeros(cap_tokens, hq, d, dtype=dt, device=dev)
        self.k_new = torch.zeros(cap_tokens, hkv, d, dtype=dt, device=dev)
        self.v_new = torch.zeros(cap_tokens, hkv, d, dtype=dt, device=dev)
        self.k_cache = proto.k_cache.to(dev).clone()
        self.v_cache = proto.v_cache.to(dev).clone()
        self.page_table = torch.zeros(cap_seqs, max_pages, dtype=torch.int32, device=dev)
        self.cu = torch.zeros(cap_seqs + 1, dtype=torch.int32, device=dev)
        self.kv = torch.zeros(cap_seqs, dtype=torch.int32, device=dev)
        self.n = torch.zeros(1, dtype=torch.int32, device=dev)
        self.out = torch.empty(cap_tokens, hq, d, dtype=dt, device=dev)
        self.lse = torch.empty(cap_tokens, hq, dtype=torch.float32, device=dev)
        self.flags = torch.zeros(1, dtype=torch.int32, device=dev)
        dims = rb.make_dims(self.q, self.k_cache, self.page_table)
        self.ws = torch.empty(rb.rpa_device_workspace_size(dims, cap_seqs), dtype=torch.uint8, device=dev)
        self.scale, self.causal = proto.scale, proto.causal

    def load(self, prob: I.Problem):
        """Copy one batch into the slots; out / lse are poisoned with NaN."""
        t, s = prob.q.shape[0], prob.num_seqs
        for dst, src in ((self.q, prob.q), (self.k_new, prob.k_new), (self.v_new, prob.v_new)):
            dst.zero_()
            dst[:t].copy_(src)
        self.k_cache.copy_(prob.k_cache)
        self.v_cache.copy_(prob.v_cache)
        self.page_table.zero_()
        mp = prob.page_table.shape[1]
        self.page_table[:s, :mp].copy_(prob.page_table)
        cu = torch.as_tensor(np.asarray(prob.cu_q_lens), dtype=torch.int32)
        self.cu.fill_(int(cu[-1]))
        self.cu[:s + 1].copy_(cu)
        self.kv.zero_()
        self.kv[:s].copy_(torch.as_tensor(np.asarray(prob.kv_lens), dtype=torch.int32))
        self.n.fill_(s)
        self.out.fill_(float("nan"))
        self.lse.fill_(float("nan"))
        self.flags.zero_()

    def call(self):
        from ragged_paged_attention_03_b200 import binding as rb
        rb.rpa_forward_device(self.q, self.k_new, self.v_new, self.k_cache, self.v_cache, self.page_table,
                              self.cu, self.kv, self.n, self.scale, self.causal, self.out, self.ws,
                              lse=self.lse, dev_flags=self.flags)


def check_slots(oracle_mod, slots: Slots, prob: I.Problem):
    torch.cuda.synchronize()
    t = prob.q.shape[0]
    assert int(slots.flags.item()) == 0, f"device flags {int(slots.flags.item()):#x}"
    out_ref, lse_ref, kc_ref, vc_ref = oracle_full(oracle_mod, prob)
    check_close(f64(slots.out[:t]), out_ref, f64(slots.lse[:t]), lse_ref, prob.dtype, prob.name)
    assert torch.isnan(slots.out[t:].float()).all() and torch.isnan(slots.lse[t:]).all(), \
        "rows past the batch were written"
    assert same_bits(slots.k_cache, kc_ref) and same_bits(slots.v_cache, vc_ref), "cache differs from the oracle's"


def one_shot(oracle_mod, prob, extra_tokens=7, extra_seqs=3):
    slots = Slots(prob, prob.q.shape[0] + extra_tokens, prob.num_seqs + extra_seqs, prob.page_table.shape[1])
    slots.load(prob)
    slots.call()
    check_slots(oracle_mod, slots, prob)


@pytest.mark.parametrize("case", range(len(SMALL)))
@pytest.mark.parametrize("dtype", [I.BF16, I.F32])
def test_small_mixes(oracle_mod, case, dtype):
    ql, kv, hq, hkv, d, p, causal = SMALL[case]
    prob = I.make_problem(ql, kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                          dtype=dtype, causal=causal, seed=800 + case, pool=1.5, name=f"dev-small{case}")
    one_shot(oracle_mod, prob)


@pytest.mark.parametrize("case", range(len(MORE)))
def test_more_shapes(oracle_mod, case):
    ql, kv, hq, hkv, d, p, causal = MORE[case]
    prob = I.make_problem(ql, kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                          dtype=I.BF16, causal=causal, seed=900 + case, pool=1.3, name=f"dev-more{case}")
    one_shot(oracle_mod, prob)


def test_serial_schedule(oracle_mod):
    """RPA_OPT_CONCURRENT_MIXED < 0: the device-planned call queues every
    kernel on the caller's stream (no side-stream branch)."""
    from ragged_paged_attention_03_b200 import binding as rb
    ql, kv, hq, hkv, d, p, causal = SMALL[6]
    prob = I.make_problem(ql, kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                          dtype=I.BF16, causal=causal, seed=990, pool=1.5, name="dev-serial")
    old = rb.rpa_set_option(rb.RPA_OPT_CONCURRENT_MIXED, -1)
    try:
        one_shot(oracle_mod, prob)
    finally:
        rb.rpa_set_option(rb.RPA_OPT_CONCURRENT_MIXED, old)


def test_split_kv_and_packed_decode(oracle_mod):
    """Enough short decode sequences to be packed four per CTA, next to long
    ones cut into chunks (1-block chunks force many partials)."""
    from ragged_paged_attention_03_b200 import binding as rb
    base = [1, 5, 16, 17, 200, 511, 1000]
    kv = [base[i % len(base)] for i in range(4 * 75)] + [3000, 5000]
    prob = I.make_problem([1] * len(kv), kv, num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=16,
                          dtype=I.BF16, seed=950, pool=1.2, name="dev-pack")
    one_shot(oracle_mod, prob, extra_tokens=0, extra_seqs=0)
    old = rb.rpa_set_option(rb.RPA_OPT_DECODE_CHUNK_BLOCKS, 3)
    try:
        one_shot(oracle_mod, prob)
    finally:
        rb.rpa_set_option(rb.RPA_OPT_DECODE_CHUNK_BLOCKS, old)


def test_graph_replay_with_new_lengths(oracle_mod):
    """One call captured in a CUDA graph, replayed over three batches of
    different sizes and kinds loaded into the same device buffers."""
    geo = dict(num_q_heads=16, num_kv_heads=4, head_dim=128, page_size=16, dtype=I.BF16)
    batches = [
        I.make_problem([1, 1, 300, 40, 1], [700, 90, 300, 1500, 2100], seed=961, pool=600, **geo, name="A"),
        I.make_problem([1] * 9, [1, 33, 4000, 16, 17, 900, 1200, 5, 2600], seed=962, pool=600, **geo, name="B"),
        I.make_problem([513, 2], [513, 700], seed=963, pool=600, **geo, name="C"),
    ]
    max_pages = max(b.page_table.shape[1] for b in batches)
    slots = Slots(batches[0], 600, 12, max_pages)
    slots.load(batches[0])
    slots.call()                       # plain run first (also the warm-up)
    check_slots(oracle_mod, slots, batches[0])
    graph = torch.cuda.CUDAGraph()
    slots.load(batches[0])
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        slots.call()
    for prob in (batches[1], batches[2], batches[0]):
        slots.load(prob)
        graph.replay()
        check_slots(oracle_mod, slots, prob)
    del graph


def test_bad_device_lengths_write_nothing(oracle_mod):
    from ragged_paged_attention_03_b200 import binding as rb
    prob = I.make_problem([1, 20, 1], [50, 20, 9], num_q_heads=8, num_kv_heads=2, head_dim=64, page_size=16,
                          dtype=I.BF16, seed=970, pool=1.5)
    slots = Slots(prob, 30, 4, prob.page_table.shape[1])
    pre_k, pre_v = prob.k_cache.clone(), prob.v_cache.clone()
    for breakage in ("kv_below_q", "past_capacity", "too_many_seqs", "cu_start"):
        slots.load(prob)
        if breakage == "kv_below_q":
            slots.kv[1] = 10                       # q_len 20 > kv_len 10
        elif breakage == "past_capacity":
            slots.kv[0] = slots.page_table.shape[1] * 16 + 1
        elif breakage == "too_many_seqs":
            slots.n.fill_(5)                       # max_seqs is 4
        else:
            slots.cu[0] = 1
        slots.call()
        torch.cuda.synchronize()
        assert int(slots.flags.item()) & rb.RPA_DEV_BAD_LENGTHS, breakage
        assert torch.isnan(slots.out.float()).all() and torch.isnan(slots.lse).all(), breakage
        assert same_bits(slots.k_cache.cpu(), pre_k) and same_bits(slots.v_cache.cpu(), pre_v), breakage
    # zero sequences: nothing written, nothing flagged
    slots.load(prob)
    slots.n.fill_(0)
    slots.call()
    torch.cuda.synchronize()
    assert int(slots.flags.item()) == 0
    assert torch.isnan(slots.out.float()).all()
    assert same_bits(slots.k_cache.cpu(), pre_k)


FULL = [("decode_128", True), ("mixed_96d_4c", True), ("prefill_8x2048", True), ("prefill_8x2048", False),
        ("long_d256", True)]


@pytest.mark.parametrize("name,causal", FULL, ids=[f"{n}-{c}" for n, c in FULL])
def test_full_size_same_bits_as_host_plan(name, causal):
    """At the benchmark's sizes the device-planned call gives exactly the
    host-planned call's out, lse and cache (the host path itself is checked
    against the oracle by the sampled full-size parity tests)."""
    prob = I.make_workload(name, device="cuda", causal=causal)
    pre_k, pre_v = prob.k_cache.clone(), prob.v_cache.clone()
    out_h, lse_h, flags = run_gpu(prob)
    assert flags == 0
    kc_h, vc_h = prob.k_cache.clone(), prob.v_cache.clone()
    prob.k_cache.copy_(pre_k)
    prob.v_cache.copy_(pre_v)
    slots = Slots(prob, prob.q.shape[0], prob.num_seqs, prob.page_table.shape[1])
    del pre_k, pre_v
    slots.load(prob)
    slots.call()
    torch.cuda.synchronize()
    assert int(slots.flags.item()) == 0
    assert torch.equal(slots.out.view(torch.int16), out_h.view(torch.int16)), "out differs from the host plan's"
    assert torch.equal(slots.lse.view(torch.int32), lse_h.view(torch.int32)), "lse differs from the host plan's"
    assert torch.equal(slots.k_cache.view(torch.int16), kc_h.view(torch.int16))
    assert torch.equal(slots.v_cache.view(torch.int16), vc_h.view(torch.int16))
