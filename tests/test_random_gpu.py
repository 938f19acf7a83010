"""Seeded random batches against the oracle, through all three entry points.

Each case draws a geometry (head_dim 64/128/256, G = Hq/Hkv from 1 to 8,
page size 8..256, causal or not, bf16 or fp32) and a batch that mixes
decode, fresh-prefill, chunked-prefill and empty sequences with lengths
across block and page boundaries.  rpa_forward (host planner),
rpa_forward_device (planner kernel) and rpa_forward_host (host buffers,
split into copy-overlapped groups when the batch's copies reach 8 MiB) must
each match the oracle within the stated tolerances, with the cache
bit-exact.
"""
import numpy as np
import pytest
import torch

from ragged_paged_attention_03_b200 import inputs as I

from harness import check_close, f64, oracle_full, run_gpu, same_bits, to_device
from test_device_plan_gpu import Slots, check_slots
from test_host_io_gpu import run_host

pytestmark = pytest.mark.gpu

N_CASES = 100


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ragged_paged_attention_03_b200 import build
    build.build()


def draw_case(seed):
    rng = np.random.default_rng(seed)
    d = int(rng.choice([64, 128, 256]))
    hkv = int(rng.choice([1, 2, 4]))
    g = int(rng.choice([1, 2, 4, 8]))
    p = int(rng.choice([8, 16, 32, 64, 128, 256]))
    dtype = I.F32 if rng.random() < 0.15 else I.BF16
    causal = bool(rng.random() < 0.7)
    q_lens, kv_lens = [], []
    for _ in range(int(rng.integers(1, 9))):
        kind = rng.choice(["decode", "prefill", "chunked", "empty"], p=[0.4, 0.25, 0.3, 0.05])
        kv = int(rng.choice([1, 15, 16, 17, 63, 64, 65, 127, 128, 129, 255, 256, 257])
                 if rng.random() < 0.5 else rng.integers(1, 1500))
        if kind == "decode":
            q = 1
        elif kind == "prefill":
            q = kv
        elif kind == "chunked":
            q = int(rng.integers(1, kv + 1))
        else:
            q = 0
        q_lens.append(q)
        kv_lens.append(max(kv, q))
    if sum(q_lens) == 0:
        q_lens[0] = 1
    return dict(q_lens=q_lens, kv_lens=kv_lens, num_q_heads=hkv * g, num_kv_heads=hkv, head_dim=d,
                page_size=p, dtype=dtype, causal=causal)


@pytest.mark.parametrize("seed", range(N_CASES))
def test_random_batch(oracle_mod, seed):
    c = draw_case(2000 + seed)
    prob = I.make_problem(c["q_lens"], c["kv_lens"], num_q_heads=c["num_q_heads"], num_kv_heads=c["num_kv_heads"],
                          head_dim=c["head_dim"], page_size=c["page_size"], dtype=c["dtype"], causal=c["causal"],
                          seed=3000 + seed, pool=1.5, name=f"random{seed}")
    out_ref, lse_ref, kc_ref, vc_ref = oracle_full(oracle_mod, prob)
    # host-planned call (classification from the lengths, no distribution)
    dp = to_device(prob)
    out, lse, flags = run_gpu(dp, use_distribution=False)
    assert flags == 0, f"device error flags {flags:#x}"
    check_close(f64(out), out_ref, f64(lse), lse_ref, prob.dtype, f"{prob.name} {c}")
    assert same_bits(dp.k_cache, kc_ref) and same_bits(dp.v_cache, vc_ref), f"{prob.name}: cache differs"
    # device-planned call, with spare capacity
    slots = Slots(prob, prob.q.shape[0] + 3, prob.num_seqs + 2, prob.page_table.shape[1])
    slots.load(prob)
    slots.call()
    check_slots(oracle_mod, slots, prob)
    # host buffers in and out
    out_h, lse_h, kc_h, vc_h, flags = run_host(prob, use_distribution=False)
    assert flags == 0, f"device error flags {flags:#x}"
    check_close(f64(out_h), out_ref, f64(lse_h), lse_ref, prob.dtype, f"{prob.name} host {c}")
    assert same_bits(kc_h, kc_ref) and same_bits(vc_h, vc_ref), f"{prob.name}: host-call cache differs"
