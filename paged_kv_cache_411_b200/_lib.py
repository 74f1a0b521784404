"""ctypes binding of libpagedkv.so: argument marshalling only.

Every function here converts its arguments (torch tensors -> device pointers,
Python ints -> C ints) and calls the C entry point of the same name; all the
work runs in the library.  Loading fails loudly if the library is missing:
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int32, c_int64, c_size_t, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_OOM = 2
PA_ERR_NOT_FOUND = 3
PA_ERR_EXISTS = 4
PA_ERR_UNSUPPORTED = 5
PA_ERR_CUDA = 6
PA_ERR_DEVICE_CHECK = 7

PA_DEVCHK_BLOCK_ID = 1
PA_DEVCHK_SLOT = 2
PA_DEVCHK_SEQ_LEN = 4
PA_DEVCHK_QUERY_RANGE = 8
PA_DEVCHK_TIMEOUT = 16

PA_KERNEL_DECODE = 1
PA_KERNEL_PREFILL = 2

STATUS_NAMES = {
    PA_OK: "ok", PA_ERR_INVALID_ARG: "invalid_arg", PA_ERR_OOM: "oom", PA_ERR_NOT_FOUND: "not_found",
    PA_ERR_EXISTS: "exists", PA_ERR_UNSUPPORTED: "unsupported", PA_ERR_CUDA: "cuda",
    PA_ERR_DEVICE_CHECK: "device_check",
}


class PagedKVError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class AllocStats(ctypes.Structure):
    _fields_ = [
        ("num_blocks", c_int32), ("block_size", c_int32), ("num_free", c_int32), ("num_used", c_int32),
        ("total_refs", c_int64), ("num_requests", c_int64), ("oom_count", c_int64), ("waste_tokens", c_int64),
    ]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


class CacheStats(ctypes.Structure):
    _fields_ = [("cached_blocks", c_int64), ("evictable_blocks", c_int64), ("hit_blocks", c_int64),
                ("evictions", c_int64), ("prefix_nodes", c_int64)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


class SchedConfig(ctypes.Structure):
    _fields_ = [("max_num_seqs", c_int32), ("max_num_tokens", c_int32), ("chunked_prefill", c_int32),
                ("watermark_blocks", c_int32)]


class StepInfo(ctypes.Structure):
    _fields_ = [("step", c_int64), ("num_prefill", c_int32), ("num_decode", c_int32), ("num_tokens", c_int32),
                ("num_admitted", c_int32), ("num_preempted", c_int32), ("num_finished", c_int32)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


class RequestInfo(ctypes.Structure):
    _fields_ = [("state", c_int32), ("prompt_len", c_int32), ("max_new_tokens", c_int32), ("prefilled", c_int32),
                ("to_prefill", c_int32), ("generated", c_int32), ("preemptions", c_int32), ("pad_", c_int32),
                ("first_token_step", c_int64), ("finish_step", c_int64)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_ if k != "pad_"}


class SchedStats(ctypes.Structure):
    _fields_ = [(k, c_int64) for k in ("steps", "waiting", "running", "finished", "preemptions",
                                        "prefill_tokens", "decode_tokens", "cached_tokens", "swapped", "swap_outs",
                                        "swap_ins")]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


_P = c_void_p
_I32P = POINTER(c_int32)
_I64P = POINTER(c_int64)

# name -> (restype, argtypes); must match include/pagedkv.h.
SIGNATURES = {
    "pa_abi_version": (c_int32, []),
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_status_string": (ctypes.c_char_p, [c_int32]),
    "pa_check_device_flag": (c_int32, [c_int32]),
    "pa_debug_inject_stall": (c_int32, [c_int32, ctypes.c_uint64]),
    "pa_alloc_create": (c_int32, [c_int32, c_int32, _I32P, POINTER(c_void_p)]),
    "pa_alloc_destroy": (None, [_P]),
    "pa_alloc_allocate": (c_int32, [_P, c_int64, c_int32]),
    "pa_alloc_append_token": (c_int32, [_P, c_int64, _I64P]),
    "pa_alloc_append_tokens": (c_int32, [_P, c_int64, c_int32, _I64P]),
    "pa_alloc_fork": (c_int32, [_P, c_int64, c_int64, c_int32]),
    "pa_alloc_free": (c_int32, [_P, c_int64]),
    "pa_alloc_get_block_table": (c_int32, [_P, c_int64, _I32P, c_int32, _I32P]),
    "pa_alloc_seq_len": (c_int32, [_P, c_int64, _I32P]),
    "pa_alloc_slots": (c_int32, [_P, c_int64, c_int32, c_int32, _I64P]),
    "pa_alloc_pack": (c_int32, [_P, _I64P, c_int32, c_int32, _I32P, _I32P]),
    "pa_alloc_stats": (c_int32, [_P, POINTER(AllocStats)]),
    "pa_alloc_available": (c_int32, [_P, _I64P]),
    "pa_alloc_refcount": (c_int32, [_P, c_int32, _I32P]),
    "pa_alloc_free_list": (c_int32, [_P, _I32P, c_int32, _I32P]),
    "pa_alloc_allocate_cached": (c_int32, [_P, c_int64, _I32P, c_int32, _I32P]),
    "pa_alloc_cache_stats": (c_int32, [_P, POINTER(CacheStats)]),
    "pa_alloc_cached_prefix": (c_int32, [_P, _I32P, c_int32, _I32P, _I32P]),
    "pa_alloc_begin_cached": (c_int32, [_P, c_int64, _I32P, c_int32, _I32P]),
    "pa_alloc_extend_tokens": (c_int32, [_P, c_int64, _I32P, c_int32]),
    "pa_alloc_evictable_list": (c_int32, [_P, _I32P, c_int32, _I32P]),
    "pa_alloc_serialize": (c_int32, [_P, _P, c_size_t, POINTER(c_size_t)]),
    "pa_alloc_deserialize": (c_int32, [_P, c_size_t, POINTER(c_void_p)]),
    "pa_swap_blocks": (c_int32, [_P, _P, _P, _P, _I64P, c_int32, c_int64, c_int32, c_int32, _P]),
    "pa_alloc_swap_out": (c_int32, [_P, _P, c_int64, _P, _P, _P, _P, c_int64, _P]),
    "pa_alloc_swap_in": (c_int32, [_P, _P, c_int64, _P, _P, _P, _P, c_int64, _P]),
    "pa_sched_create": (c_int32, [_P, POINTER(SchedConfig), POINTER(c_void_p)]),
    "pa_sched_destroy": (None, [_P]),
    "pa_sched_add_request": (c_int32, [_P, c_int64, c_int32, c_int32]),
    "pa_sched_step": (c_int32, [_P, POINTER(StepInfo), _I64P, _I32P, _I32P, _I64P, _I32P, _I64P]),
    "pa_sched_complete": (c_int32, [_P]),
    "pa_sched_complete_tokens": (c_int32, [_P, _I32P, c_int32]),
    "pa_sched_add_request_tokens": (c_int32, [_P, c_int64, _I32P, c_int32, c_int32]),
    "pa_sched_enable_swap": (c_int32, [_P, _P]),
    "pa_sched_last_swaps": (c_int32, [_P, _I64P, c_int32, _I32P, _I64P, c_int32, _I32P]),
    "pa_sched_request_info": (c_int32, [_P, c_int64, POINTER(RequestInfo)]),
    "pa_sched_stats": (c_int32, [_P, POINTER(SchedStats)]),
    "pa_reshape_and_cache": (c_int32, [_P, _P, _P, _P, _P, c_int32, c_int32, c_int32, c_int32, c_int32, _P, _P]),
    "pa_decode_workspace_bytes": (c_size_t, [c_int32, c_int32, c_int32, c_int32, c_int32]),
    "pa_paged_attention_decode": (c_int32, [_P, _P, _P, _P, _P, _P, c_int32, c_int32, c_int32, c_int32, c_int32,
                                            c_int32, c_float, _P, c_size_t, _P, _P]),
    "pa_paged_attention_decode_noalloc": (c_int32, [_P, _P, _P, _P, _P, _P, c_int32, c_int32, c_int32, c_int32,
                                                    c_int32, c_int32, c_float, _P, _P]),
    "pa_paged_attention_prefill_chunk": (c_int32, [_P, _P, _P, _P, _P, _P, _P, c_int32, c_int32, c_int32, c_int32,
                                                   c_int32, c_int32, c_int32, c_float, _P, _P]),
}

_lib = None


def lib():
    """The loaded library (raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with `python -m paged_kv_cache_411_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def last_error() -> str:
    return (lib().pa_last_error() or b"").decode()


def check(status: int) -> None:
    if status != PA_OK:
        raise PagedKVError(status, last_error())
