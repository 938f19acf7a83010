"""Prefill kernels other than each head dim's default, forced through
RPA_OPT_PREFILL_KERNEL, against the fp64 oracle: the CTA-pair kernel (tcgen05
MMAs of M = 256 across two SMs, a separate epilogue warpgroup; the default at
head_dim 256) at head_dim 128 and its one-CTA form, and the one-tile-per-CTA
head_dim-256 kernel.  Every output row and the whole cache pool on small
mixes (fresh and chunked prefill with ragged tails, page sizes 8 to 256,
causal and not), and sampled rows plus whole-pool cache properties on a
full-size causal prefill batch of each head dim.
"""
import numpy as np
import pytest
import torch

from ragged_paged_attention_03_b200 import inputs as I

from harness import check_cache_property
from test_parity_gpu import SMALL, MORE, full_check, sampled_check

pytestmark = pytest.mark.gpu

KERNELS = {2: "pair", 3: "single"}
# head_dim 256: the pair kernel is the default; the one-tile kernel is forced with 1
CASES = [("small", i) for i in (0, 4, 5, 6, 7, 10)] + [("more", i) for i in (1, 2)]
CASES_256 = [("small", 9), ("more", 3), ("more", 4)]   # head_dim 256: pairs only


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ragged_paged_attention_03_b200 import build
    build.build()


@pytest.fixture
def kernel_option(request):
    from ragged_paged_attention_03_b200 import binding
    old = binding.rpa_set_option(binding.RPA_OPT_PREFILL_KERNEL, request.param)
    yield request.param
    binding.rpa_set_option(binding.RPA_OPT_PREFILL_KERNEL, old)


@pytest.mark.parametrize("kernel_option", list(KERNELS), ids=list(KERNELS.values()), indirect=True)
@pytest.mark.parametrize("table,case", CASES, ids=[f"{t}{c}" for t, c in CASES])
def test_forced_prefill_kernel(oracle_mod, kernel_option, table, case):
    # the inputs of the default kernel's tests of the same cases
    ql, kv, hq, hkv, d, p, causal = (SMALL if table == "small" else MORE)[case]
    seed, pool = (100 + case, 1.5) if table == "small" else (500 + case, 1.3)
    prob = I.make_problem(ql, kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                          dtype=I.BF16, causal=causal, seed=seed, pool=pool)
    full_check(oracle_mod, prob)


@pytest.mark.parametrize("kernel_option", list(KERNELS), ids=list(KERNELS.values()), indirect=True)
@pytest.mark.parametrize("seed", [710, 711, 712, 714])
def test_forced_dominant_key_after_context_block(oracle_mod, kernel_option, seed):
    """The rows of test_parity_gpu's test_dominant_key_after_context_block on
    the forced kernels: their row sums also take the bf16-rounded weights."""
    ql, kv, hq, hkv, d, p, causal = SMALL[10]
    prob = I.make_problem(ql, kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                          dtype=I.BF16, causal=causal, seed=seed, pool=1.5)
    full_check(oracle_mod, prob)


@pytest.mark.parametrize("kernel_option", [2, 1], ids=["pair", "one-tile"], indirect=True)
@pytest.mark.parametrize("table,case", CASES_256, ids=[f"{t}{c}" for t, c in CASES_256])
def test_forced_head_dim_256(oracle_mod, kernel_option, table, case):
    ql, kv, hq, hkv, d, p, causal = (SMALL if table == "small" else MORE)[case]
    assert d == 256
    seed, pool = (100 + case, 1.5) if table == "small" else (500 + case, 1.3)
    prob = I.make_problem(ql, kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=p,
                          dtype=I.BF16, causal=causal, seed=seed, pool=pool)
    full_check(oracle_mod, prob)


@pytest.mark.parametrize("kernel_option,name", [(2, "prefill_8x2048"), (1, "prefill_4x4096_d256")],
                         ids=["pair-d128", "one-tile-d256"], indirect=["kernel_option"])
def test_forced_full_causal_prefill(oracle_mod, kernel_option, name):
    prob = I.make_workload(name, device="cuda")
    pre_k, pre_v = prob.k_cache.clone(), prob.v_cache.clone()
    from harness import run_gpu
    out, lse, flags = run_gpu(prob)
    assert flags == 0, f"device error flags {flags:#x}"
    sampled_check(oracle_mod, prob, pre_k, pre_v, out, lse, [0, prob.num_seqs - 1], rows_per_seq=32)
    check_cache_property(pre_k, pre_v, prob)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
