"""ctypes binding of include/rpa.h -- argument marshalling only.

Every function here has the name of the C entry point it calls and does no
computation of its own: it checks types and shapes, turns torch tensors into
device pointers and numpy arrays into host pointers, and raises on a non-zero
return code.  The library must have been built in-tree
(``python -m ragged_paged_attention_03_b200.build``); importing this module
without it raises, so nothing can silently run without the CUDA path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# RPA_ABLATE_CACHE_WRITE=1 selects the timing-only build without the fused
# cache stores (bench.py --ablate-write runs it in a child process); its
# caches are not updated, so nothing else may use it.
LIB_PATH = os.path.join(_HERE, "librpa_b200_nowrite.so" if os.environ.get("RPA_ABLATE_CACHE_WRITE") == "1"
                        else "librpa_b200.so")

RPA_F32, RPA_BF16 = 0, 1
RPA_OK = 0
RPA_DEV_BAD_PAGE = 0x1
RPA_DEV_TIMEOUT = 0x2
RPA_OPT_DECODE_CHUNK_BLOCKS = 0
RPA_OPT_FORCE_GENERIC = 1
RPA_OPT_DISABLE_PREFILL_TC = 2
RPA_OPT_PREFILL_SMS = 3
RPA_OPT_CONCURRENT_MIXED = 4
RPA_OPT_PREFILL_LOADERS = 5
RPA_OPT_DECODE_PACK_BLOCKS = 6
RPA_OPT_PREFILL_KERNEL = 7


class rpa_dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_q_heads", "num_kv_heads", "head_dim", "page_size", "num_pages",
        "max_pages_per_seq", "total_q_tokens", "dtype")]


class rpa_plan_info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_decode", "num_prefill", "num_generic", "num_empty", "decode_items",
        "decode_max_splits", "combine_rows", "prefill_tiles")] + [("plan_bytes", ctypes.c_int64)] + [
        ("decode_packed", ctypes.c_int32), ("pad", ctypes.c_int32)]


class RpaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {rpa_status_string(code)} (code {code})")
        self.code = code


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m ragged_paged_attention_03_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)
_P = ctypes.c_void_p
_i32 = ctypes.c_int32
_lib.rpa_forward.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _i32, _P, ctypes.c_float, _i32, _P,
                             _P, ctypes.POINTER(rpa_dims), _P]
_lib.rpa_forward.restype = ctypes.c_int
_lib.rpa_device_status.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32)]
_lib.rpa_device_status.restype = ctypes.c_int
_lib.rpa_status_string.argtypes = [ctypes.c_int]
_lib.rpa_status_string.restype = ctypes.c_char_p
_lib.rpa_plan.argtypes = [_P, _P, _i32, _P, ctypes.POINTER(rpa_dims), ctypes.POINTER(rpa_plan_info)]
_lib.rpa_plan.restype = ctypes.c_int
_lib.rpa_set_option.argtypes = [_i32, ctypes.c_int64]
_lib.rpa_set_option.restype = ctypes.c_int64
_lib.rpa_profile_enable.argtypes = [_i32]
_lib.rpa_profile_enable.restype = ctypes.c_int32
_lib.rpa_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
_lib.rpa_profile_read.restype = ctypes.c_int
KERNEL_CLASSES = ("generic", "decode", "combine", "prefill")
_lib.rpa_decode_noalloc.argtypes = [_P, _P, _P, _P, _P, _P, _P, _i32, ctypes.c_float, _P, _P,
                                    ctypes.POINTER(rpa_dims), _P, _P]
_lib.rpa_decode_noalloc.restype = ctypes.c_int
RPA_ERR_SCRATCH_LIMIT = 7
RPA_ERR_WORKSPACE = 8
RPA_DEV_BAD_LENGTHS = 0x4
_lib.rpa_device_workspace_size.argtypes = [ctypes.POINTER(rpa_dims), _i32, ctypes.POINTER(ctypes.c_int64)]
_lib.rpa_device_workspace_size.restype = ctypes.c_int
_lib.rpa_forward_device.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _i32, ctypes.c_float, _i32, _P, _P,
                                    ctypes.POINTER(rpa_dims), _P, ctypes.c_int64, _P, _P]
_lib.rpa_forward_device.restype = ctypes.c_int


def library() -> ctypes.CDLL:
    return _lib


def rpa_status_string(code: int) -> str:
    return _lib.rpa_status_string(int(code)).decode()


def rpa_set_option(option: int, value: int) -> int:
    return int(_lib.rpa_set_option(int(option), int(value)))


def _host_i32(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        a = a.cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _hp(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(_P)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RPA_F32
    if t.dtype == torch.bfloat16:
        return RPA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def make_dims(q: torch.Tensor, k_cache: torch.Tensor, page_table: torch.Tensor) -> rpa_dims:
    num_pages, page_size, hkv, d = k_cache.shape
    return rpa_dims(num_q_heads=q.shape[1], num_kv_heads=hkv, head_dim=d, page_size=page_size,
                    num_pages=num_pages, max_pages_per_seq=page_table.shape[1],
                    total_q_tokens=q.shape[0], dtype=_dtype_code(q))


def rpa_plan(cu_q_lens, kv_lens, distribution, dims: rpa_dims) -> rpa_plan_info:
    cu, kv, dist = _host_i32(cu_q_lens), _host_i32(kv_lens), _host_i32(distribution)
    info = rpa_plan_info()
    rc = _lib.rpa_plan(_hp(cu), _hp(kv), len(kv), _hp(dist), ctypes.byref(dims), ctypes.byref(info))
    if rc != RPA_OK:
        raise RpaError(rc, "rpa_plan")
    return info


def _dev(t: Optional[torch.Tensor], name: str, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def rpa_forward(q, k_new, v_new, k_cache, v_cache, page_table, cu_q_lens, kv_lens, distribution,
                scale: float, causal: bool, out, lse=None, stream=None) -> None:
    """Calls rpa_forward on `stream` (default: torch's current stream).

    Device tensors: q [T,Hq,D], k_new/v_new [T,Hkv,D], k_cache/v_cache
    [pages,P,Hkv,D], page_table [S,max_pages] int32, out [T,Hq,D], lse [T,Hq]
    float32 or None.  Host arrays: cu_q_lens [S+1], kv_lens [S], distribution
    [3] or None (int32)."""
    dt = q.dtype
    for name, t in (("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache),
                    ("v_cache", v_cache), ("out", out)):
        if t.dtype != dt:
            raise TypeError(f"{name} dtype {t.dtype} != q dtype {dt}")
    cu, kv, dist = _host_i32(cu_q_lens), _host_i32(kv_lens), _host_i32(distribution)
    dims = make_dims(q, k_cache, page_table)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    sptr = ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))
    rc = _lib.rpa_forward(_dev(q, "q"), _dev(k_new, "k_new"), _dev(v_new, "v_new"),
                          _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                          _dev(page_table, "page_table", torch.int32), _hp(cu), _hp(kv), len(kv),
                          _hp(dist), float(scale), int(bool(causal)), _dev(out, "out"),
                          _dev(lse, "lse", torch.float32), ctypes.byref(dims), sptr)
    if rc != RPA_OK:
        raise RpaError(rc, "rpa_forward")


def rpa_device_status(stream=None) -> int:
    """Synchronises `stream` and returns (and clears) the device error bits."""
    if stream is None:
        stream = torch.cuda.current_stream()
    sptr = ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))
    flags = ctypes.c_uint32(0)
    rc = _lib.rpa_device_status(sptr, ctypes.byref(flags))
    if rc != RPA_OK:
        raise RpaError(rc, "rpa_device_status")
    return int(flags.value)


def rpa_profile_enable(on: bool) -> bool:
    return bool(_lib.rpa_profile_enable(int(bool(on))))


def rpa_profile_read() -> dict:
    """{kernel class: (launches, total ms)} since the last read."""
    ms = (ctypes.c_double * 4)()
    n = (ctypes.c_int64 * 4)()
    rc = _lib.rpa_profile_read(ms, n)
    if rc != RPA_OK:
        raise RpaError(rc, "rpa_profile_read")
    return {k: (int(n[i]), float(ms[i])) for i, k in enumerate(KERNEL_CLASSES)}


def rpa_decode_noalloc(q, k_new, v_new, k_cache, v_cache, page_table, kv_lens, scale: float, out,
                       lse=None, dev_flags=None, stream=None) -> None:
    """Calls rpa_decode_noalloc: a decode-only batch (token s is sequence s's
    one new token) run entirely in the library's fixed scratch array, for
    callers that must not allocate device memory.  dev_flags: optional int32
    CUDA tensor of one element that receives the device error bits."""
    kv = _host_i32(kv_lens)
    dims = make_dims(q, k_cache, page_table)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    sptr = ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))
    rc = _lib.rpa_decode_noalloc(_dev(q, "q"), _dev(k_new, "k_new"), _dev(v_new, "v_new"),
                                 _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                 _dev(page_table, "page_table", torch.int32), _hp(kv), len(kv),
                                 float(scale), _dev(out, "out"), _dev(lse, "lse", torch.float32),
                                 ctypes.byref(dims), _dev(dev_flags, "dev_flags", torch.int32), sptr)
    if rc != RPA_OK:
        raise RpaError(rc, "rpa_decode_noalloc")


def rpa_device_workspace_size(dims: rpa_dims, max_seqs: int) -> int:
    """Bytes of device workspace rpa_forward_device needs for these dims and
    at most `max_seqs` sequences."""
    n = ctypes.c_int64(0)
    rc = _lib.rpa_device_workspace_size(ctypes.byref(dims), int(max_seqs), ctypes.byref(n))
    if rc != RPA_OK:
        raise RpaError(rc, "rpa_device_workspace_size")
    return int(n.value)


def rpa_forward_device(q, k_new, v_new, k_cache, v_cache, page_table, cu_q_lens, kv_lens, num_seqs,
                       scale: float, causal: bool, out, workspace, lse=None, dev_flags=None,
                       stream=None) -> None:
    """Calls rpa_forward_device: the lengths stay on the device and the
    planning runs in a kernel, so the call can be captured in a CUDA graph.

    cu_q_lens [max_seqs+1], kv_lens [max_seqs], num_seqs [1]: int32 CUDA
    tensors (max_seqs = kv_lens.numel()); page_table has max_seqs rows; q's
    row count is the token capacity T.  workspace: uint8 CUDA tensor of at
    least rpa_device_workspace_size bytes.  dev_flags: optional int32 CUDA
    tensor of one element that receives the device error bits."""
    dt = q.dtype
    for name, t in (("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache),
                    ("v_cache", v_cache), ("out", out)):
        if t.dtype != dt:
            raise TypeError(f"{name} dtype {t.dtype} != q dtype {dt}")
    max_seqs = kv_lens.numel()
    if cu_q_lens.numel() < max_seqs + 1 or num_seqs.numel() < 1 or page_table.shape[0] < max_seqs:
        raise ValueError("cu_q_lens needs max_seqs + 1 entries, num_seqs one, page_table max_seqs rows")
    dims = make_dims(q, k_cache, page_table)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    sptr = ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))
    rc = _lib.rpa_forward_device(_dev(q, "q"), _dev(k_new, "k_new"), _dev(v_new, "v_new"),
                                 _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                 _dev(page_table, "page_table", torch.int32),
                                 _dev(cu_q_lens, "cu_q_lens", torch.int32), _dev(kv_lens, "kv_lens", torch.int32),
                                 _dev(num_seqs, "num_seqs", torch.int32), max_seqs, float(scale),
                                 int(bool(causal)), _dev(out, "out"), _dev(lse, "lse", torch.float32),
                                 ctypes.byref(dims), _dev(workspace, "workspace", torch.uint8),
                                 workspace.numel(), _dev(dev_flags, "dev_flags", torch.int32), sptr)
    if rc != RPA_OK:
        raise RpaError(rc, "rpa_forward_device")


RPA_HOST_MAX_GROUPS = 32
_lib.rpa_forward_host.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _i32, _P, ctypes.c_float, _i32, _P, _P,
                                  ctypes.POINTER(rpa_dims), _P]
_lib.rpa_forward_host.restype = ctypes.c_int
_lib.rpa_host_groups.argtypes = [_P, _i32, ctypes.POINTER(rpa_dims), _i32, _P, ctypes.POINTER(ctypes.c_int32)]
_lib.rpa_host_groups.restype = ctypes.c_int


def _host(t: Optional[torch.Tensor], name: str, dtype=None):
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def rpa_forward_host(q, k_new, v_new, k_cache, v_cache, page_table, cu_q_lens, kv_lens, distribution,
                     scale: float, causal: bool, out, lse=None, stream=None) -> None:
    """Calls rpa_forward_host: q, k_new, v_new, page_table, out and lse are
    host (CPU, preferably pinned) tensors; k_cache / v_cache are CUDA tensors.
    Asynchronous on `stream` (default: the current stream of the caches'
    device): synchronise it before reading out / lse."""
    dt = q.dtype
    for name, t in (("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache),
                    ("v_cache", v_cache), ("out", out)):
        if t.dtype != dt:
            raise TypeError(f"{name} dtype {t.dtype} != q dtype {dt}")
    cu, kv, dist = _host_i32(cu_q_lens), _host_i32(kv_lens), _host_i32(distribution)
    dims = make_dims(q, k_cache, page_table)
    if stream is None:
        stream = torch.cuda.current_stream(k_cache.device)
    sptr = ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))
    rc = _lib.rpa_forward_host(_host(q, "q"), _host(k_new, "k_new"), _host(v_new, "v_new"),
                               _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                               _host(page_table, "page_table", torch.int32), _hp(cu), _hp(kv), len(kv),
                               _hp(dist), float(scale), int(bool(causal)), _host(out, "out"),
                               _host(lse, "lse", torch.float32), ctypes.byref(dims), sptr)
    if rc != RPA_OK:
        raise RpaError(rc, "rpa_forward_host")


def rpa_host_groups(cu_q_lens, dims: rpa_dims, with_lse: bool = True) -> np.ndarray:
    """Sequence group boundaries rpa_forward_host uses for this batch."""
    cu = _host_i32(cu_q_lens)
    bounds = np.zeros(RPA_HOST_MAX_GROUPS + 1, dtype=np.int32)
    n = ctypes.c_int32(0)
    rc = _lib.rpa_host_groups(_hp(cu), len(cu) - 1, ctypes.byref(dims), int(bool(with_lse)), _hp(bounds),
                              ctypes.byref(n))
    if rc != RPA_OK:
        raise RpaError(rc, "rpa_host_groups")
    return bounds[:n.value + 1].copy()
