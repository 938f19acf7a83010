"""fp64 CPU oracle for ragged paged attention -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and it shares no code
with them.  The arithmetic lives in ``rpa_oracle.c`` (plain C, fp64, OpenMP
over sequence x head); this module only builds that file with gcc and
marshals numpy arrays into it.

Every function here follows "Ragged Paged Attention: A High-Performance and
Flexible LLM Inference Kernel for TPU" (arXiv 2604.15464), abstract, and the
RPA talk summary (rocketrecap.com), 00:06:36 (fused cache update, then
attention) and its glossary entries FlashAttention (exact attention) and
PagedAttention (page table).  Pins for every part are in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rpa_oracle.c")
_LIB = os.path.join(_HERE, "librpa_oracle.so")

F32, BF16 = 0, 1
_ERRORS = {-1: "invalid argument", -2: "invalid lengths", -3: "page index out of range"}


def build(force: bool = False) -> str:
    """Compile rpa_oracle.c into librpa_oracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32 = ctypes.c_int32
        lib.rpa_oracle_scatter.argtypes = [P, P, P, P, P, i32, P, P, i32, i32, i32, i32, i32, i32, i32]
        lib.rpa_oracle_forward.argtypes = [P, P, P, P, P, P, i32, P, P, i32, i32, i32, i32, i32, i32,
                                           i32, ctypes.c_double, i32, P, P, i32]
        lib.rpa_oracle_attend_rows.argtypes = [P, P, P, P, i32, P, P, i32, i32, i32, i32, i32, i32,
                                               i32, ctypes.c_double, i32, i32, P, P, P, P, i32]
        lib.rpa_oracle_row_weights.argtypes = [P, P, P, P, i32, P, P, i32, i32, i32, i32, i32, i32,
                                               i32, ctypes.c_double, i32, i32, i32, i32, P]
        for f in ("rpa_oracle_scatter", "rpa_oracle_forward", "rpa_oracle_attend_rows",
                  "rpa_oracle_row_weights", "rpa_oracle_num_threads"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _raw(a: np.ndarray, dtype: int) -> np.ndarray:
    """Stored elements as a C-contiguous array: float32, or uint16 bf16 bits."""
    want = np.float32 if dtype == F32 else np.uint16
    if a.dtype != want:
        raise TypeError(f"expected {want} storage, got {a.dtype}")
    return np.ascontiguousarray(a)


def _check(rc: int):
    if rc != 0:
        raise ValueError(f"oracle rejected the problem: {_ERRORS.get(rc, rc)}")


def _geom(k_cache: np.ndarray, q: np.ndarray, page_table: np.ndarray):
    num_pages, page_size, hkv, d = k_cache.shape
    hq = q.shape[1]
    return num_pages, page_size, hkv, d, hq, page_table.shape[1]


def num_threads() -> int:
    return int(_load().rpa_oracle_num_threads())


def scatter(k_new, v_new, k_cache, v_cache, page_table, cu_q_lens, kv_lens, hq, dtype):
    """Fused cache update only, in place on host caches (talk summary 00:06:36)."""
    lib = _load()
    k_new, v_new = _raw(k_new, dtype), _raw(v_new, dtype)
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    cu = np.ascontiguousarray(cu_q_lens, dtype=np.int32)
    kv = np.ascontiguousarray(kv_lens, dtype=np.int32)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    num_pages, page_size, hkv, d = k_cache.shape
    _check(lib.rpa_oracle_scatter(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(pt),
                                  pt.shape[1], _ptr(cu), _ptr(kv), len(kv), hq, hkv, d, page_size,
                                  num_pages, dtype))


def forward(q, k_new, v_new, k_cache, v_cache, page_table, cu_q_lens, kv_lens, scale, causal,
            dtype, threads: int = 0):
    """Scatter then attend every row.  Caches are host arrays updated in place.

    Returns (out [T, Hq, D] float64, lse [T, Hq] float64)."""
    lib = _load()
    q, k_new, v_new = _raw(q, dtype), _raw(k_new, dtype), _raw(v_new, dtype)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    cu = np.ascontiguousarray(cu_q_lens, dtype=np.int32)
    kv = np.ascontiguousarray(kv_lens, dtype=np.int32)
    num_pages, page_size, hkv, d, hq, max_pages = _geom(k_cache, q, pt)
    t = q.shape[0]
    out = np.zeros((t, hq, d), dtype=np.float64)
    lse = np.zeros((t, hq), dtype=np.float64)
    _check(lib.rpa_oracle_forward(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(pt), max_pages, _ptr(cu), _ptr(kv), len(kv), hq, hkv, d,
                                  page_size, num_pages, dtype, float(scale), int(bool(causal)),
                                  _ptr(out), _ptr(lse), threads))
    return out, lse


def attend_rows(q, k_cache, v_cache, page_table, cu_q_lens, kv_lens, scale, causal, dtype, rows,
                heads, threads: int = 0):
    """Attention of selected (token row, query head) pairs over an already
    updated cache (call ``scatter`` first).  Returns (out [n, D], lse [n])."""
    lib = _load()
    q = _raw(q, dtype)
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    cu = np.ascontiguousarray(cu_q_lens, dtype=np.int32)
    kv = np.ascontiguousarray(kv_lens, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    num_pages, page_size, hkv, d, hq, max_pages = _geom(k_cache, q, pt)
    n = len(rows)
    out = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    _check(lib.rpa_oracle_attend_rows(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(pt), max_pages,
                                      _ptr(cu), _ptr(kv), len(kv), hq, hkv, d, page_size, num_pages,
                                      dtype, float(scale), int(bool(causal)), n, _ptr(rows),
                                      _ptr(heads), _ptr(out), _ptr(lse), threads))
    return out, lse


def row_weights(q, k_cache, v_cache, page_table, cu_q_lens, kv_lens, scale, causal, dtype, seq, i,
                h):
    """Softmax weights of one query row over its kv_len keys (0 where masked)."""
    lib = _load()
    q = _raw(q, dtype)
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    cu = np.ascontiguousarray(cu_q_lens, dtype=np.int32)
    kv = np.ascontiguousarray(kv_lens, dtype=np.int32)
    num_pages, page_size, hkv, d, hq, max_pages = _geom(k_cache, q, pt)
    w = np.zeros((int(kv[seq]),), dtype=np.float64)
    _check(lib.rpa_oracle_row_weights(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(pt), max_pages,
                                      _ptr(cu), _ptr(kv), len(kv), hq, hkv, d, page_size, num_pages,
                                      dtype, float(scale), int(bool(causal)), seq, i, h, _ptr(w)))
    return w
