"""A wide seeded sweep of random batches through rpa_forward against the
oracle, beyond the 100 cases of test_random_gpu.py.  Off by default (about
1,500 cases take four minutes): set RPA_RANDOM_SWEEP=N to run N cases,
RPA_RANDOM_SWEEP_BASE to move the seeds and RPA_RANDOM_SWEEP_KERNEL to force
an RPA_OPT_PREFILL_KERNEL value.  Every case must meet the tolerances with
the cache bit-exact; the worst case's share of each bound is printed.
"""
import os

import numpy as np
import pytest
import torch

from ragged_paged_attention_03_b200 import inputs as I

from harness import TOL, f64, oracle_full, run_gpu, same_bits, to_device
from test_random_gpu import draw_case

pytestmark = pytest.mark.gpu

N = int(os.environ.get("RPA_RANDOM_SWEEP", "0"))
BASE = int(os.environ.get("RPA_RANDOM_SWEEP_BASE", "50000"))
KERNEL = int(os.environ.get("RPA_RANDOM_SWEEP_KERNEL", "0"))


@pytest.mark.skipif(N <= 0, reason="set RPA_RANDOM_SWEEP=N to run the wide random sweep")
def test_random_sweep(oracle_mod):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ragged_paged_attention_03_b200 import binding, build
    build.build()
    old = binding.rpa_set_option(binding.RPA_OPT_PREFILL_KERNEL, KERNEL)
    failures, worst = [], (0.0, None)
    try:
        for i in range(N):
            c = draw_case(BASE + i)
            prob = I.make_problem(c["q_lens"], c["kv_lens"], num_q_heads=c["num_q_heads"],
                                  num_kv_heads=c["num_kv_heads"], head_dim=c["head_dim"],
                                  page_size=c["page_size"], dtype=c["dtype"], causal=c["causal"],
                                  seed=BASE + 100000 + i, pool=1.5)
            out_ref, lse_ref, kc_ref, vc_ref = oracle_full(oracle_mod, prob)
            dp = to_device(prob)
            out, lse, flags = run_gpu(dp, use_distribution=False)
            if out.numel() == 0:
                continue
            tol = TOL[prob.dtype]
            err = np.abs(f64(out) - out_ref)
            lerr = np.abs(f64(lse) - lse_ref)
            share = max(err.max() / tol["max_abs"], err.mean() / tol["mean_abs"], lerr.max() / tol["lse"])
            if share > worst[0]:
                worst = (share, (i, c))
            if flags != 0 or share > 1.0 or not (same_bits(dp.k_cache, kc_ref) and same_bits(dp.v_cache, vc_ref)):
                failures.append((i, c, float(err.max()), float(err.mean()), float(lerr.max()), flags))
    finally:
        binding.rpa_set_option(binding.RPA_OPT_PREFILL_KERNEL, old)
    print(f"\n{N} cases from seed {BASE}, kernel option {KERNEL}: worst case at {worst[0]:.3f} of a bound: {worst[1]}")
    assert not failures, failures[:5]
