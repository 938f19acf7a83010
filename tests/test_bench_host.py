"""Host-side logic of bench.py, on CPU: the multi-rank aggregation (two gloo
ranks, as torchrun would launch two replicas), the algorithmic work counts
and the roofline arithmetic.  No GPU and no kernel call."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from ragged_paged_attention_03_b200 import inputs as I  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms_by_rank, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))

    class Args:
        impl = "ours"

    try:
        got_world, got_rank, _ = bench.dist_setup(Args, backend="gloo")
        ms = bench.max_over_ranks(ms_by_rank[rank], "cpu")
        e2e = bench.max_over_ranks(2.0 * ms_by_rank[rank], "cpu")
        work = {"bytes": 10 ** 9, "flops": 10 ** 12, "tokens": 1000}
        v = bench.value_of("decode_128", work, ms, got_world)
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
        out_q.put((rank, got_world, got_rank, ms, e2e, v))
    except Exception as e:  # report instead of hanging the parent
        out_q.put((rank, "error", repr(e)))


def test_two_replicas_take_the_slowest_rank():
    """Each replica times its own steps; the job's step time is the max over
    ranks and the value counts the work of every rank (weak scaling)."""
    world, port = 2, _free_port()
    ms_by_rank = [0.40, 0.55]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, ms_by_rank, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in res:
        assert r[1] != "error", r
        rank, got_world, got_rank, ms, e2e, v = r
        assert got_world == 2 and got_rank == rank
        assert ms == pytest.approx(0.55)
        assert e2e == pytest.approx(1.10)
        # 2 ranks x 1 GB each in 0.55 ms
        assert v == pytest.approx(2 * 1e9 / 0.55e-3 / 1e9)


def test_single_process_max_is_identity():
    assert not torch.distributed.is_initialized()
    assert bench.max_over_ranks(0.123, "cpu") == 0.123


def test_algorithmic_counts_tiny_workload():
    """Bytes and FLOPs of the tiny fp32 mix, counted by hand from its lengths:
    (q, kv) = (1,37), (1,100), (50,50), (17,80); Hq 4, Hkv 1, D 64, page 16."""
    prob = I.make_workload("tiny_mixed_f32", device="cpu")
    w = bench.algorithmic(prob)
    e, hq, hkv, d = 4, 4, 1, 64
    q = np.array([1, 1, 50, 17])
    k = np.array([37, 100, 50, 80])
    assert list(prob.q_lens) == list(q) and list(prob.kv_lens) == list(k)
    t = int(q.sum())
    pages = int(((k + 15) // 16).sum())
    want_bytes = (k.sum() * hkv * d * 2 * e + t * hkv * d * 2 * e + 2 * t * hq * d * e + 4 * t * hq
                  + 4 * pages)
    assert w["bytes"] == want_bytes
    # causal visible pairs: decode rows see everything; prefill rows see c + i + 1 keys
    pairs = 37 + 100 + sum(i + 1 for i in range(50)) + sum(63 + i + 1 for i in range(17))
    assert w["flops"] == 4 * d * hq * pairs
    assert w["tokens"] == t
    assert w["prefill_flops"] == 4 * d * hq * (pairs - 37 - 100)


def test_roofline_uses_the_dominant_kernel():
    work = {"bytes": 3 * 10 ** 9, "flops": 4 * 10 ** 12, "tokens": 10, "decode_kernel_bytes": 2 * 10 ** 9,
            "prefill_flops": 10 ** 12}
    pk = {"hbm": 8000.0, "tc": 2000.0, "tc_sustained": 1500.0, "source": "test"}
    # decode dominates: 2 launches of 0.25 ms each move 2 GB per launch
    r = bench.roofline("decode_128", work, {"decode": (2, 0.5), "combine": (2, 0.05)}, pk, 2)
    assert r["kernel"] == "decode" and r["bound"] == "hbm"
    assert r["achieved"] == pytest.approx(2e9 / 0.25e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 8000.0)
    # prefill dominates: 1 launch of 1 ms does 1 TFLOP
    r = bench.roofline("mixed_96d_4c", work, {"decode": (1, 0.2), "prefill": (1, 1.0)}, pk, 1)
    assert r["kernel"] == "prefill" and r["bound"] == "tensor"
    assert r["achieved"] == pytest.approx(1000.0)
    assert r["kernel_share"]["prefill"] == pytest.approx(1.0 / 1.2, abs=1e-4)


def test_head_shards_split_heads_not_sequences():
    """--shard heads: each rank gets the same sequences, lengths and pages
    with Hkv / n KV heads and their query heads, sliced from the one batch
    (concatenated along the head axis, the shards give back the whole draw);
    n must divide Hkv."""
    full = I.make_workload("tiny_mixed_f32", device="cpu")
    shards = [I.make_workload("mixed_96d_4c", device="cpu", poison=False, head_shard=(r, 4), max_seqs=6)
              for r in range(4)]
    ref = I.make_workload("mixed_96d_4c", device="cpu", poison=False, max_seqs=6)
    for sh in shards:
        assert list(sh.q_lens) == list(ref.q_lens) and list(sh.kv_lens) == list(ref.kv_lens)
        assert torch.equal(sh.page_table, ref.page_table)
        assert sh.q.shape == (ref.q.shape[0], ref.q.shape[1] // 4, ref.q.shape[2])
        assert sh.k_cache.shape[2] == ref.k_cache.shape[2] // 4
        assert sh.q.is_contiguous() and sh.k_cache.is_contiguous()
    for name, axis in (("q", 1), ("k_new", 1), ("v_new", 1), ("k_cache", 2), ("v_cache", 2)):
        whole = torch.cat([getattr(sh, name) for sh in shards], dim=axis)
        assert torch.equal(whole.view(torch.int16), getattr(ref, name).view(torch.int16)), name
    with pytest.raises(ValueError):
        I.make_workload("tiny_mixed_f32", device="cpu", head_shard=(0, 2))   # 1 KV head
    assert full.q.shape[1] == 4


def test_head_shard_job_value():
    """Value of a head-sharded job: bytes / FLOPs are summed over the ranks,
    the batch's tokens are counted once."""
    work = {"bytes": 10 ** 9, "flops": 10 ** 12, "tokens": 1000}
    w = bench.rank_work(work, 4, "heads")
    assert bench.value_of("mixed_96d_4c", w, 1.0, 4) == pytest.approx(1000 / 1e-3)
    assert bench.value_of("decode_128", w, 1.0, 4) == pytest.approx(4 * 1e9 / 1e-3 / 1e9)
    assert bench.rank_work(work, 4, "replicas") is work
    assert bench.value_of("mixed_96d_4c", work, 1.0, 4) == pytest.approx(4 * 1000 / 1e-3)


def test_traffic_records_only_for_the_captured_source_and_kernel(tmp_path, monkeypatch):
    """A DRAM-traffic record is reported only while its kernel source is the
    one that was captured and the run uses the captured kernel option."""
    import hashlib
    import json
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"prefill/w": {"dram_bytes_per_launch": 123, "source": "k.cu",
                         "source_sha256": hashlib.sha256(b"kernel v1\n").hexdigest(),
                         "prefill_kernel_option": 0}}
    (prof / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "PREFILL_KERNEL_OPTION", 0)
    assert bench.traffic_for("prefill", "w") == 123
    assert bench.traffic_for("decode", "w") is None
    monkeypatch.setattr(bench, "PREFILL_KERNEL_OPTION", 2)
    assert bench.traffic_for("prefill", "w") is None
    monkeypatch.setattr(bench, "PREFILL_KERNEL_OPTION", 0)
    src.write_text("kernel v2\n")
    assert bench.traffic_for("prefill", "w") is None


def test_committed_traffic_records_match_their_sources():
    """Every committed record names an existing kernel source; a record whose
    source has changed since the capture is reported as null by the bench
    (this only lists them, it does not fail: recapturing needs a GPU)."""
    import hashlib
    import json
    recs = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for key, rec in recs.items():
        path = os.path.join(bench.ROOT, rec["source"])
        assert os.path.exists(path), key
        assert rec["dram_bytes_per_launch"] > 0, key
        fresh = hashlib.sha256(open(path, "rb").read()).hexdigest() == rec["source_sha256"]
        print(key, "current" if fresh else "stale (reported as null)")
