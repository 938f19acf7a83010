"""KV-head shards of one batch (the multi-GPU split of `bench.py --shard
heads`), run one after another on one GPU.

Attention never mixes heads, so rank r's shard (KV heads [r Hkv/n, (r+1)
Hkv/n) with their query heads, every sequence and page) must give exactly the
full call's out, lse and cache slices: the test demands them bit for bit, and
checks sampled rows of the last shard against the fp64 oracle as well.
"""
import pytest
import torch

from ragged_paged_attention_03_b200 import inputs as I

from harness import run_gpu, same_bits
from test_parity_gpu import sampled_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ragged_paged_attention_03_b200 import build
    build.build()


CASES = [("mixed_96d_4c", 2), ("mixed_96d_4c", 8), ("prefill_4x4096_d256", 4)]


@pytest.mark.parametrize("name,n", CASES, ids=[f"{a}-x{b}" for a, b in CASES])
def test_head_shards_equal_the_full_call(oracle_mod, name, n):
    full = I.make_workload(name, device="cuda")
    pre = I.Problem(**{**full.__dict__, "k_cache": full.k_cache.clone(), "v_cache": full.v_cache.clone()})
    out, lse, flags = run_gpu(full)
    assert flags == 0, f"device error flags {flags:#x}"
    g = full.num_q_heads // full.num_kv_heads
    for r in range(n):
        sh = I.head_slice(pre, r, n)
        sh_pre_k, sh_pre_v = sh.k_cache.clone(), sh.v_cache.clone()
        s_out, s_lse, s_flags = run_gpu(sh)
        assert s_flags == 0, f"shard {r}: device error flags {s_flags:#x}"
        kv0, kv1 = r * full.num_kv_heads // n, (r + 1) * full.num_kv_heads // n
        q0, q1 = kv0 * g, kv1 * g
        assert same_bits(s_out, out[:, q0:q1].contiguous()), f"shard {r}: out differs from the full call"
        assert same_bits(s_lse, lse[:, q0:q1].contiguous()), f"shard {r}: lse differs from the full call"
        assert same_bits(sh.k_cache, full.k_cache[:, :, kv0:kv1].contiguous()), f"shard {r}: k_cache"
        assert same_bits(sh.v_cache, full.v_cache[:, :, kv0:kv1].contiguous()), f"shard {r}: v_cache"
        if r == n - 1:
            q_lens = sh.q_lens
            dec = [s for s in range(sh.num_seqs) if q_lens[s] == 1]
            pfx = [s for s in range(sh.num_seqs) if q_lens[s] > 1]
            seqs = sorted(set(dec[:1] + dec[-1:] + pfx[:1] + pfx[-1:]))
            sampled_check(oracle_mod, sh, sh_pre_k, sh_pre_v, s_out, s_lse, seqs, rows_per_seq=16)
        del sh, sh_pre_k, sh_pre_v
