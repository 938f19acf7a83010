"""Shared helpers for the parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, compare."""
from __future__ import annotations

import numpy as np
import torch

from ragged_paged_attention_03_b200 import inputs as I

# Tolerances.  bf16 I/O with fp32 accumulation: max-abs 1.5e-2, mean-abs
# 2e-3, lse 2e-3 (the stated bar for this method).  fp32 I/O (no tensor
# cores, no TF32): fp32 rounding of a D-term dot product and of the softmax
# sum stays far below 1e-4 for N(0,1) data of these sizes.
TOL = {I.BF16: dict(max_abs=1.5e-2, mean_abs=2e-3, lse=2e-3),
       I.F32: dict(max_abs=1e-4, mean_abs=1e-5, lse=1e-4)}


def to_device(prob: I.Problem, device="cuda") -> I.Problem:
    d = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in prob.__dict__.items()}
    d["k_cache"] = prob.k_cache.to(device).clone()
    d["v_cache"] = prob.v_cache.to(device).clone()
    return I.Problem(**d)


def run_gpu(prob: I.Problem, use_distribution=True, lse=True):
    """One rpa_forward over `prob` (device tensors, caches updated in place)."""
    from ragged_paged_attention_03_b200 import binding
    out = torch.empty_like(prob.q)
    lse_t = torch.empty(prob.q.shape[0], prob.q.shape[1], dtype=torch.float32,
                        device=prob.q.device) if lse else None
    if out.numel():
        out.fill_(float("nan"))
    if lse_t is not None and lse_t.numel():
        lse_t.fill_(float("nan"))
    binding.rpa_forward(prob.q, prob.k_new, prob.v_new, prob.k_cache, prob.v_cache,
                        prob.page_table, prob.cu_q_lens, prob.kv_lens,
                        prob.distribution if use_distribution else None, prob.scale, prob.causal,
                        out, lse_t)
    flags = binding.rpa_device_status()
    return out, lse_t, flags


def oracle_full(oracle, prob: I.Problem, threads=0):
    kc = I.to_storage(prob.k_cache).copy()
    vc = I.to_storage(prob.v_cache).copy()
    out, lse = oracle.forward(I.to_storage(prob.q), I.to_storage(prob.k_new),
                              I.to_storage(prob.v_new), kc, vc, prob.page_table.cpu().numpy(),
                              prob.cu_q_lens, prob.kv_lens, prob.scale, prob.causal, prob.dtype,
                              threads)
    return out, lse, kc, vc


def check_close(out_gpu: np.ndarray, out_ref: np.ndarray, lse_gpu, lse_ref, dtype, what=""):
    tol = TOL[dtype]
    assert np.isfinite(out_gpu).all(), f"{what}: non-finite outputs"
    err = np.abs(out_gpu.astype(np.float64) - out_ref)
    assert err.max() <= tol["max_abs"], f"{what}: max-abs {err.max():.3e} > {tol['max_abs']}"
    assert err.mean() <= tol["mean_abs"], f"{what}: mean-abs {err.mean():.3e} > {tol['mean_abs']}"
    if lse_gpu is not None:
        assert np.isfinite(lse_gpu).all(), f"{what}: non-finite lse"
        lerr = np.abs(lse_gpu.astype(np.float64) - lse_ref)
        assert lerr.max() <= tol["lse"], f"{what}: lse err {lerr.max():.3e} > {tol['lse']}"
    return float(err.max()), float(err.mean())


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def same_bits(a, b) -> bool:
    if isinstance(a, torch.Tensor):
        a = I.to_storage(a)
    if isinstance(b, torch.Tensor):
        b = I.to_storage(b)
    return a.shape == b.shape and np.array_equal(a.view(np.uint8), b.view(np.uint8))


def new_slot_ids(prob: I.Problem) -> torch.Tensor:
    """Flat cache slot (page * P + slot) of every new token, in token order."""
    ids = []
    p = prob.page_size
    table = prob.page_table.cpu().numpy().astype(np.int64)
    for s in range(prob.num_seqs):
        a, b = int(prob.cu_q_lens[s]), int(prob.cu_q_lens[s + 1])
        c = int(prob.kv_lens[s]) - (b - a)
        pos = np.arange(c, c + b - a)
        ids.append(table[s, pos // p] * p + pos % p)
    return torch.from_numpy(np.concatenate(ids) if ids else np.zeros(0, np.int64))


def check_cache_property(prob_pre_k, prob_pre_v, prob: I.Problem):
    """Whole-pool bit-exact check that holds at any size: the new tokens'
    slots hold exactly k_new / v_new, and every other slot kept its bits."""
    ids = new_slot_ids(prob).to(prob.k_cache.device)
    n = prob.num_pages * prob.page_size
    for pre, post, new in ((prob_pre_k, prob.k_cache, prob.k_new), (prob_pre_v, prob.v_cache, prob.v_new)):
        ib = torch.int16 if post.dtype == torch.bfloat16 else torch.int32
        post_f = post.view(ib).view(n, -1)
        pre_f = pre.view(ib).view(n, -1)
        assert torch.equal(post_f[ids], new.view(ib).reshape(len(ids), -1)), "new slots differ"
        keep = torch.ones(n, dtype=torch.bool, device=post.device)
        keep[ids] = False
        assert torch.equal(post_f[keep], pre_f[keep]), "slots outside the new tokens changed"
