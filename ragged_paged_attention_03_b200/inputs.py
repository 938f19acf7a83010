"""Seeded synthetic workloads for ragged paged attention.

This module only draws inputs: sequence lengths, a shuffled page pool, a page
table, and N(0,1) values for Q, the new K/V and the cached context.  It holds
none of the attention arithmetic, so the CUDA path and the fp64 oracle can
both consume what it produces without sharing any of the method's code.

Recipes (the shapes are those of a Llama-3-8B attention layer: 32 query heads,
8 KV heads, head_dim 128; no weights are involved):

* ``tiny_mixed_f32``   fp32, seed 0: (q_len, kv_len) = (1,37), (1,100),
  (50,50), (17,80); 4/1 heads, D 64, page 16, 32 physical pages in a random
  permutation, pages given to sequences consecutively from that permutation.
* ``decode_128``       bf16: 128 sequences, q_len 1, kv_len uniform in
  [1024, 8192]; 32/8 heads, D 128, page 16; pool 1.25x the pages needed,
  shuffled; all values 0.5 * N(0,1).
* ``prefill_8x2048``   bf16: 8 fresh sequences, q_len = kv_len = 2048; 32/8
  heads, D 128, page 16, shuffled 1.25x pool, N(0,1); causal or not.
* ``mixed_96d_4c``     bf16, causal: 96 decode sequences with kv_len
  log-uniform in [512, 16384] and 4 chunked-prefill sequences with q_len 512
  over a prior context log-uniform in [1024, 8192]; 32/8 heads, D 128, page 16.
* ``long_d256``        bf16, causal: 32 decode sequences with kv_len 131072
  and 4 fresh prefill sequences with q_len = kv_len = 4096; 16/4 heads,
  D 256, page 64, shuffled 1.25x pool.

Cache contents before the call: every context slot (positions < kv_len -
q_len of its sequence) holds a drawn value; every other slot (unused pages,
the slots the new tokens will be written to, tail slots past kv_len) holds
NaN when ``poison`` is set, so any read of a slot the method must not read
shows up in the outputs.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

F32, BF16 = 0, 1


@dataclass
class Problem:
    name: str
    dtype: int                      # F32 or BF16
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    num_pages: int
    q: torch.Tensor                 # [T, Hq, D]
    k_new: torch.Tensor             # [T, Hkv, D]
    v_new: torch.Tensor             # [T, Hkv, D]
    k_cache: torch.Tensor           # [num_pages, P, Hkv, D], state before the call
    v_cache: torch.Tensor
    page_table: torch.Tensor        # [S, max_pages] int32 (same device as the cache)
    cu_q_lens: np.ndarray           # [S+1] int32, host
    kv_lens: np.ndarray             # [S] int32, host
    distribution: Optional[np.ndarray]  # [3] int32 or None
    scale: float
    causal: bool
    ctx_k: Optional[list] = None    # per sequence [c, Hkv, D] logical context (small problems)
    ctx_v: Optional[list] = None
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return len(self.kv_lens)

    @property
    def total_q(self) -> int:
        return int(self.cu_q_lens[-1]) if len(self.cu_q_lens) else 0

    @property
    def q_lens(self) -> np.ndarray:
        return np.diff(self.cu_q_lens).astype(np.int32)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == F32 else torch.bfloat16


def to_storage(t: torch.Tensor) -> np.ndarray:
    """Host numpy view of a tensor's stored elements: float32, or the uint16
    bit patterns of bf16 (what the oracle reads)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def classify(q_lens: Sequence[int], kv_lens: Sequence[int]) -> Optional[np.ndarray]:
    """Distribution triple {d, p, S} if the sequences are already ordered as
    decode, then fresh prefill, then chunked; None otherwise."""
    kinds = []
    for ql, kv in zip(q_lens, kv_lens):
        kinds.append(0 if ql <= 1 else (1 if ql == kv else 2))
    if kinds != sorted(kinds):
        return None
    d = sum(1 for k in kinds if k == 0)
    p = d + sum(1 for k in kinds if k == 1)
    return np.array([d, p, len(kinds)], dtype=np.int32)


def _lengths(name: str, gen: torch.Generator):
    """(q_lens, kv_lens) for a named workload, drawn from ``gen`` (CPU)."""
    if name == "tiny_mixed_f32":
        return [1, 1, 50, 17], [37, 100, 50, 80]
    if name == "decode_128":
        kv = torch.randint(1024, 8193, (128,), generator=gen).tolist()
        return [1] * 128, kv
    if name == "prefill_8x2048":
        return [2048] * 8, [2048] * 8
    if name == "mixed_96d_4c":
        u = torch.rand(96, generator=gen, dtype=torch.float64)
        dec = [int(round(math.exp(math.log(512) + x * (math.log(16384) - math.log(512)))))
               for x in u.tolist()]
        u = torch.rand(4, generator=gen, dtype=torch.float64)
        prior = [int(round(math.exp(math.log(1024) + x * (math.log(8192) - math.log(1024)))))
                 for x in u.tolist()]
        return [1] * 96 + [512] * 4, dec + [p + 512 for p in prior]
    if name == "long_d256":
        return [1] * 32 + [4096] * 4, [131072] * 32 + [4096] * 4
    if name == "prefill_4x4096_d256":
        return [4096] * 4, [4096] * 4
    raise KeyError(name)


WORKLOADS = {
    # name: (dtype, Hq, Hkv, D, P, causal, value scale, seed, pool)
    "tiny_mixed_f32": (F32, 4, 1, 64, 16, True, 1.0, 0, 32),
    "decode_128": (BF16, 32, 8, 128, 16, True, 0.5, 2, 1.25),
    "prefill_8x2048": (BF16, 32, 8, 128, 16, True, 1.0, 3, 1.25),
    "mixed_96d_4c": (BF16, 32, 8, 128, 16, True, 1.0, 4, 1.25),
    "long_d256": (BF16, 16, 4, 256, 64, True, 1.0, 5, 1.25),
    # the prefill sequences of long_d256 alone (a size a profiler capture fits)
    "prefill_4x4096_d256": (BF16, 16, 4, 256, 64, True, 1.0, 6, 1.25),
}


def make_workload(name: str, device="cpu", causal: Optional[bool] = None, poison: bool = True,
                  logical: Optional[bool] = None, max_seqs: Optional[int] = None,
                  head_shard: Optional[Tuple[int, int]] = None) -> Problem:
    """One of the named workloads (see the module docstring).  ``max_seqs``
    keeps only the first sequences (smaller cases for profiler captures).
    ``head_shard = (rank, n)``: rank's share of a KV-head split of the same
    batch over n GPUs (``head_slice`` of the whole draw): Hkv / n KV heads with
    their Hq / n query heads, every sequence, length and page (heads never
    interact, so the shards need no exchange)."""
    dtype, hq, hkv, d, p, causal_default, vscale, seed, pool = WORKLOADS[name]
    if head_shard is not None:
        rank, n = head_shard
        if n < 1 or hkv % n != 0 or not 0 <= rank < n:
            raise ValueError(f"{name}: {hkv} KV heads do not split over {n} GPUs")
    gen = torch.Generator().manual_seed(seed)
    q_lens, kv_lens = _lengths(name, gen)
    if max_seqs is not None:
        q_lens, kv_lens = q_lens[:max_seqs], kv_lens[:max_seqs]
    if logical is None:
        logical = name == "tiny_mixed_f32"
    prob = make_problem(q_lens, kv_lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                        page_size=p, dtype=dtype, causal=causal_default if causal is None else causal,
                        seed=seed, pool=pool, value_scale=vscale, device=device, poison=poison,
                        logical=logical, name=name, gen=gen)
    if head_shard is None or head_shard[1] == 1:
        return prob
    shard = head_slice(prob, *head_shard)
    del prob
    return shard


def head_slice(prob: Problem, rank: int, n: int) -> Problem:
    """KV heads [rank * Hkv / n, (rank + 1) * Hkv / n) of a problem, with
    their query heads (query head h reads KV head h // G, so they are the
    matching contiguous range): q, k_new, v_new and both caches sliced along
    the head axis into contiguous copies; lengths, pages, page table, scale
    and mask unchanged."""
    hkv, hq = prob.num_kv_heads, prob.num_q_heads
    if n < 1 or hkv % n != 0 or not 0 <= rank < n:
        raise ValueError(f"{hkv} KV heads do not split {n} ways")
    kv0, kv1 = rank * hkv // n, (rank + 1) * hkv // n
    g = hq // hkv
    q0, q1 = kv0 * g, kv1 * g

    def cut(t, a, b, axis):
        return t.narrow(axis, a, b - a).contiguous()

    d = dict(prob.__dict__)
    d.update(num_q_heads=q1 - q0, num_kv_heads=kv1 - kv0,
             q=cut(prob.q, q0, q1, 1), k_new=cut(prob.k_new, kv0, kv1, 1), v_new=cut(prob.v_new, kv0, kv1, 1),
             k_cache=cut(prob.k_cache, kv0, kv1, 2), v_cache=cut(prob.v_cache, kv0, kv1, 2),
             ctx_k=None if prob.ctx_k is None else [cut(t, kv0, kv1, 1) for t in prob.ctx_k],
             ctx_v=None if prob.ctx_v is None else [cut(t, kv0, kv1, 1) for t in prob.ctx_v],
             meta={**prob.meta, "head_shard": (rank, n)})
    return Problem(**d)


def make_problem(q_lens: Sequence[int], kv_lens: Sequence[int], *, num_q_heads: int,
                 num_kv_heads: int, head_dim: int, page_size: int, dtype: int = BF16,
                 causal: bool = True, seed: int = 0, pool=1.25, value_scale: float = 1.0,
                 device="cpu", poison: bool = True, logical: bool = True, name: str = "custom",
                 gen: Optional[torch.Generator] = None, scale: Optional[float] = None,
                 max_pages_extra: int = 0, pad_value: int = 0) -> Problem:
    """A seeded problem with the given per-sequence (q_len, kv_len).

    ``pool``: an int is an exact physical page count; a float is a multiple of
    the pages the sequences need.  Physical pages are a random permutation of
    the pool, given to the sequences consecutively.  ``logical``: draw each
    sequence's context as a contiguous array first, then place it into its
    pages (kept in ``ctx_k``/``ctx_v``); otherwise draw the whole pool at once
    (large problems).  Unused page-table entries hold ``pad_value``."""
    q_lens = [int(x) for x in q_lens]
    kv_lens = [int(x) for x in kv_lens]
    assert len(q_lens) == len(kv_lens)
    for ql, kv in zip(q_lens, kv_lens):
        assert 0 <= ql <= kv, (ql, kv)
    if gen is None:
        gen = torch.Generator().manual_seed(seed)
    tdt = torch.float32 if dtype == F32 else torch.bfloat16
    npages_seq = [(kv + page_size - 1) // page_size for kv in kv_lens]
    need = sum(npages_seq)
    num_pages = int(pool) if isinstance(pool, int) else max(1, int(math.ceil(need * float(pool))))
    assert num_pages >= need, (num_pages, need)
    max_pages = max([1] + npages_seq) + max_pages_extra
    perm = torch.randperm(num_pages, generator=gen).tolist()
    table = np.full((len(kv_lens), max_pages), pad_value, dtype=np.int32)
    pos = 0
    for s, n in enumerate(npages_seq):
        table[s, :n] = perm[pos:pos + n]
        pos += n
    cu = np.zeros(len(q_lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(q_lens)
    t_total = int(cu[-1])
    s_count = len(q_lens)

    dev_gen = torch.Generator(device=device).manual_seed(seed + 1000)

    def randn(*shape):
        x = torch.randn(*shape, generator=dev_gen, device=device, dtype=torch.float32)
        if value_scale != 1.0:
            x = x * value_scale
        return x.to(tdt)

    q = randn(t_total, num_q_heads, head_dim)
    k_new = randn(t_total, num_kv_heads, head_dim)
    v_new = randn(t_total, num_kv_heads, head_dim)
    shape = (num_pages, page_size, num_kv_heads, head_dim)
    ctx_k = ctx_v = None
    if logical:
        k_cache = torch.full(shape, float("nan") if poison else 0.0, dtype=tdt, device=device)
        v_cache = torch.full(shape, float("nan") if poison else 0.0, dtype=tdt, device=device)
        ctx_k, ctx_v = [], []
        kc = k_cache.view(num_pages * page_size, num_kv_heads, head_dim)
        vc = v_cache.view(num_pages * page_size, num_kv_heads, head_dim)
        for s in range(s_count):
            c = kv_lens[s] - q_lens[s]
            ck = randn(c, num_kv_heads, head_dim)
            cv = randn(c, num_kv_heads, head_dim)
            ctx_k.append(ck)
            ctx_v.append(cv)
            if c:
                slots = _context_slots(table[s], c, page_size)
                idx = torch.from_numpy(slots).to(device)
                kc[idx] = ck
                vc[idx] = cv
    else:
        k_cache = randn(*shape)
        v_cache = randn(*shape)
        if poison:
            valid = np.zeros(num_pages * page_size, dtype=bool)
            for s in range(s_count):
                c = kv_lens[s] - q_lens[s]
                if c:
                    valid[_context_slots(table[s], c, page_size)] = True
            bad = torch.from_numpy(np.nonzero(~valid)[0].astype(np.int64)).to(device)
            nan = float("nan")
            k_cache.view(num_pages * page_size, -1)[bad] = nan
            v_cache.view(num_pages * page_size, -1)[bad] = nan
    dist = classify(q_lens, kv_lens)
    return Problem(name=name, dtype=dtype, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                   head_dim=head_dim, page_size=page_size, num_pages=num_pages, q=q, k_new=k_new,
                   v_new=v_new, k_cache=k_cache, v_cache=v_cache,
                   page_table=torch.from_numpy(table).to(device), cu_q_lens=cu,
                   kv_lens=np.array(kv_lens, dtype=np.int32), distribution=dist,
                   scale=float(scale if scale is not None else 1.0 / math.sqrt(head_dim)),
                   causal=bool(causal), ctx_k=ctx_k, ctx_v=ctx_v,
                   meta={"seed": seed, "value_scale": value_scale})


def _context_slots(table_row: np.ndarray, c: int, page_size: int) -> np.ndarray:
    """Flat slot ids (page * P + slot) of logical positions 0..c-1."""
    n = (c + page_size - 1) // page_size
    ids = (table_row[:n].astype(np.int64)[:, None] * page_size
           + np.arange(page_size, dtype=np.int64)[None, :]).reshape(-1)
    return ids[:c]


def sub_problem(prob: Problem, seqs: Sequence[int]) -> Problem:
    """The problem restricted to a subset of sequences, on the host, with a
    compact pool holding only their pages (renumbered in order) plus the
    pre-call cache state of those pages.  Used to check sampled sequences of
    large workloads against the oracle without copying a whole pool."""
    seqs = list(seqs)
    p = prob.page_size
    q_lens = prob.q_lens
    tables, rows_q = [], []
    pages = []
    for s in seqs:
        n = (int(prob.kv_lens[s]) + p - 1) // p
        row = prob.page_table[s, :n].cpu().numpy().astype(np.int64)
        tables.append(np.arange(len(pages), len(pages) + n, dtype=np.int32))
        pages.extend(row.tolist())
        rows_q.append((int(prob.cu_q_lens[s]), int(prob.cu_q_lens[s + 1])))
    max_pages = max([1] + [len(t) for t in tables])
    table = np.zeros((len(seqs), max_pages), dtype=np.int32)
    for i, t in enumerate(tables):
        table[i, :len(t)] = t
    pidx = torch.tensor(pages if pages else [0], dtype=torch.int64, device=prob.k_cache.device)
    k_cache = prob.k_cache.index_select(0, pidx).cpu()
    v_cache = prob.v_cache.index_select(0, pidx).cpu()
    tok = torch.cat([torch.arange(a, b) for a, b in rows_q]) if rows_q else torch.zeros(0, dtype=torch.long)
    tok = tok.to(prob.q.device)
    cu = np.zeros(len(seqs) + 1, dtype=np.int32)
    cu[1:] = np.cumsum([int(q_lens[s]) for s in seqs])
    return Problem(name=prob.name + "[sub]", dtype=prob.dtype, num_q_heads=prob.num_q_heads,
                   num_kv_heads=prob.num_kv_heads, head_dim=prob.head_dim, page_size=p,
                   num_pages=max(1, len(pages)), q=prob.q.index_select(0, tok).cpu(),
                   k_new=prob.k_new.index_select(0, tok).cpu(),
                   v_new=prob.v_new.index_select(0, tok).cpu(), k_cache=k_cache, v_cache=v_cache,
                   page_table=torch.from_numpy(table), cu_q_lens=cu,
                   kv_lens=np.array([int(prob.kv_lens[s]) for s in seqs], dtype=np.int32),
                   distribution=None, scale=prob.scale, causal=prob.causal)
