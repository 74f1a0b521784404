"""Paged-KV attention for NVIDIA B200 (sm_100a): the Python face of libpagedkv.so.

The functions and the ``BlockAllocator`` class carry the names of the C entry
points in ``include/pagedkv.h`` and only marshal arguments: torch tensors are
used for device memory and streams, every computation runs in the library.

    reshape_and_cache(k_new, v_new, k_cache, v_cache, slot_mapping)
    paged_attention_decode(out, q, k_cache, v_cache, block_tables, seq_lens, scale, workspace)
    paged_attention_prefill_chunk(out, q, k_cache, v_cache, block_tables, q_start, ctx_before, scale)
    BlockAllocator(num_blocks, block_size, free_order=None)
"""
from __future__ import annotations

import ctypes
from ctypes import POINTER, byref, c_int32, c_int64, c_size_t, c_void_p

import numpy as np

from ._lib import (PA_DEVCHK_BLOCK_ID, PA_DEVCHK_QUERY_RANGE, PA_DEVCHK_SEQ_LEN, PA_DEVCHK_SLOT,
                   PA_DEVCHK_TIMEOUT, PA_KERNEL_DECODE, PA_KERNEL_PREFILL, PA_ERR_CUDA, PA_ERR_DEVICE_CHECK, PA_ERR_EXISTS, PA_ERR_INVALID_ARG,
                   PA_ERR_NOT_FOUND, PA_ERR_OOM, PA_ERR_UNSUPPORTED, PA_OK, STATUS_NAMES, AllocStats,
                   CacheStats, PagedKVError, check, last_error, lib)

__all__ = [
    "BlockAllocator", "Scheduler", "reshape_and_cache", "paged_attention_decode", "paged_attention_prefill_chunk",
    "decode_workspace_bytes", "paged_attention_decode_noalloc", "swap_blocks", "swap_out", "swap_in",
    "PagedKVError", "lib", "STATUS_NAMES", "PA_OK", "PA_ERR_INVALID_ARG",
    "PA_ERR_OOM", "PA_ERR_NOT_FOUND", "PA_ERR_EXISTS", "PA_ERR_UNSUPPORTED", "PA_ERR_CUDA",
    "PA_ERR_DEVICE_CHECK", "PA_DEVCHK_BLOCK_ID", "PA_DEVCHK_SLOT", "PA_DEVCHK_SEQ_LEN",
    "PA_DEVCHK_QUERY_RANGE", "PA_DEVCHK_TIMEOUT", "PA_KERNEL_DECODE", "PA_KERNEL_PREFILL",
]


def _i32p(a: np.ndarray):
    return a.ctypes.data_as(POINTER(c_int32))


def _i64p(a: np.ndarray):
    return a.ctypes.data_as(POINTER(c_int64))


class BlockAllocator:
    """Host block allocator (pa_alloc_*).  Methods return the C status code
    (``PA_OK`` ...) plus their outputs, exactly as the C calls report them."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self._h = c_void_p()
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int32)
        check(lib().pa_alloc_create(num_blocks, block_size, None if order is None else _i32p(order),
                                    byref(self._h)))
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)

    def close(self):
        if self._h:
            lib().pa_alloc_destroy(self._h)
            self._h = c_void_p()

    def serialize(self) -> bytes:
        """pa_alloc_serialize: the allocator's whole host state as bytes (equal states, equal bytes)."""
        n = c_size_t(0)
        check(lib().pa_alloc_serialize(self._h, None, 0, byref(n)))
        buf = (ctypes.c_uint8 * max(n.value, 1))()
        check(lib().pa_alloc_serialize(self._h, ctypes.cast(buf, c_void_p), n.value, byref(n)))
        return bytes(buf)[:n.value]

    @classmethod
    def deserialize(cls, data: bytes) -> "BlockAllocator":
        """pa_alloc_deserialize: a new allocator holding a state written by serialize() (raises on bad bytes)."""
        raw = (ctypes.c_uint8 * max(len(data), 1)).from_buffer_copy(data if data else b"\0")
        h = c_void_p()
        check(lib().pa_alloc_deserialize(ctypes.cast(raw, c_void_p), len(data), byref(h)))
        obj = cls.__new__(cls)
        obj._h = h
        hdr = np.frombuffer(bytes(data[8:16]), dtype=np.int32)
        obj.num_blocks, obj.block_size = int(hdr[0]), int(hdr[1])
        return obj

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def allocate(self, req: int, num_tokens: int) -> int:
        return lib().pa_alloc_allocate(self._h, req, num_tokens)

    def append_token(self, req: int):
        slot = c_int64(-1)
        st = lib().pa_alloc_append_token(self._h, req, byref(slot))
        return st, (slot.value if st == PA_OK else None)

    def append_tokens(self, req: int, n: int):
        out = np.empty(max(n, 0), dtype=np.int64)
        st = lib().pa_alloc_append_tokens(self._h, req, n, _i64p(out))
        return st, (out if st == PA_OK else np.empty(0, np.int64))

    def fork(self, src: int, dst: int, prefix_tokens: int) -> int:
        return lib().pa_alloc_fork(self._h, src, dst, prefix_tokens)

    def free(self, req: int) -> int:
        return lib().pa_alloc_free(self._h, req)

    def get_block_table(self, req: int):
        n = c_int32(0)
        st = lib().pa_alloc_get_block_table(self._h, req, None, 0, byref(n))
        if st == PA_ERR_NOT_FOUND:
            return st, np.empty(0, np.int32)
        out = np.empty(n.value, dtype=np.int32)
        st = lib().pa_alloc_get_block_table(self._h, req, _i32p(out), n.value, byref(n))
        return st, out

    def seq_len(self, req: int):
        n = c_int32(0)
        st = lib().pa_alloc_seq_len(self._h, req, byref(n))
        return st, (n.value if st == PA_OK else None)

    def slots(self, req: int, pos_begin: int, n: int):
        out = np.empty(max(n, 0), dtype=np.int64)
        st = lib().pa_alloc_slots(self._h, req, pos_begin, n, _i64p(out))
        return st, out

    def pack(self, reqs, max_blocks: int, tables=None, lens=None):
        """Block tables [n, max_blocks] (padding -1) and lengths [n] of the requests; written into the given
        C-contiguous int32 arrays when passed (e.g. views of a pinned staging buffer), else into new ones."""
        r = np.ascontiguousarray(reqs, dtype=np.int64)
        n = len(r)
        if tables is None:
            tables = np.empty((n, max_blocks), dtype=np.int32)
        if lens is None:
            lens = np.empty(n, dtype=np.int32)
        if (tables.dtype != np.int32 or tables.shape != (n, max_blocks) or not tables.flags.c_contiguous
                or not tables.flags.writeable or lens.dtype != np.int32 or lens.shape != (n,)
                or not lens.flags.c_contiguous or not lens.flags.writeable):
            raise ValueError("pack: tables must be int32 [n, max_blocks] and lens int32 [n], C-contiguous and "
                             "writeable")
        st = lib().pa_alloc_pack(self._h, _i64p(r), n, max_blocks, _i32p(tables), _i32p(lens))
        return st, tables, lens

    def stats(self) -> dict:
        s = AllocStats()
        check(lib().pa_alloc_stats(self._h, byref(s)))
        return s.as_dict()

    def available(self) -> int:
        n = c_int64(0)
        check(lib().pa_alloc_available(self._h, byref(n)))
        return n.value

    def refcount(self, block: int):
        n = c_int32(0)
        st = lib().pa_alloc_refcount(self._h, block, byref(n))
        return st, n.value

    def free_list(self) -> np.ndarray:
        n = c_int32(0)
        lib().pa_alloc_free_list(self._h, None, 0, byref(n))
        out = np.empty(n.value, dtype=np.int32)
        check(lib().pa_alloc_free_list(self._h, _i32p(out), n.value, byref(n)))
        return out

    # ---- automatic prefix caching
    def allocate_cached(self, req: int, tokens):
        """Returns (status, cached_tokens): blocks of the longest cached prefix are reused."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        n = c_int32(0)
        st = lib().pa_alloc_allocate_cached(self._h, req, _i32p(t), len(t), byref(n))
        return st, (n.value if st == PA_OK else 0)

    def cached_prefix(self, tokens):
        """(cached blocks begin_cached would reuse for tokens, of which parked in the LRU)."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        h, p = c_int32(0), c_int32(0)
        check(lib().pa_alloc_cached_prefix(self._h, _i32p(t), len(t), byref(h), byref(p)))
        return h.value, p.value

    def begin_cached(self, req: int, tokens):
        """Returns (status, cached_tokens): the request starts with its cached prefix only and is tracked."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        n = c_int32(0)
        st = lib().pa_alloc_begin_cached(self._h, req, _i32p(t), len(t), byref(n))
        return st, (n.value if st == PA_OK else 0)

    def extend_tokens(self, req: int, ids) -> int:
        t = np.ascontiguousarray(ids, dtype=np.int32)
        return lib().pa_alloc_extend_tokens(self._h, req, _i32p(t), len(t))

    def cache_stats(self) -> dict:
        s = CacheStats()
        check(lib().pa_alloc_cache_stats(self._h, byref(s)))
        return s.as_dict()

    def evictable_list(self) -> np.ndarray:
        n = c_int32(0)
        lib().pa_alloc_evictable_list(self._h, None, 0, byref(n))
        out = np.empty(n.value, dtype=np.int32)
        check(lib().pa_alloc_evictable_list(self._h, _i32p(out), n.value, byref(n)))
        return out


# ------------------------------------------------------------------ scheduler
class Scheduler:
    """Continuous-batching step driver (pa_sched_*) over a BlockAllocator."""

    def __init__(self, alloc: "BlockAllocator", max_num_seqs: int, max_num_tokens: int, chunked_prefill: bool = True,
                 watermark_blocks: int = 0):
        from ._lib import SchedConfig
        self._alloc = alloc                       # the C scheduler borrows it
        self._cpu = None
        self.max_num_seqs, self.max_num_tokens = int(max_num_seqs), int(max_num_tokens)
        cfg = SchedConfig(self.max_num_seqs, self.max_num_tokens, int(bool(chunked_prefill)), int(watermark_blocks))
        self._h = c_void_p()
        check(lib().pa_sched_create(alloc._h, byref(cfg), byref(self._h)))
        # output buffers of pa_sched_step and their ctypes pointers, made once (a step copies out its slices)
        n, t = self.max_num_seqs, self.max_num_tokens + self.max_num_seqs
        self._bufs = (np.empty(n, np.int64), np.empty(n, np.int32), np.empty(n, np.int32),
                      np.empty(n, np.int64), np.empty(n, np.int32), np.empty(t, np.int64))
        conv = (_i64p, _i32p, _i32p, _i64p, _i32p, _i64p)
        self._ptrs = tuple(f(b) for f, b in zip(conv, self._bufs))

    def close(self):
        if self._h:
            lib().pa_sched_destroy(self._h)
            self._h = c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_request(self, req: int, prompt_len: int, max_new_tokens: int, tokens=None) -> int:
        """Queue a request; with its prompt's token ids it goes through the prefix cache."""
        if tokens is None:
            return lib().pa_sched_add_request(self._h, req, prompt_len, max_new_tokens)
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        if len(t) != prompt_len:
            raise ValueError("add_request: len(tokens) must equal prompt_len")
        return lib().pa_sched_add_request_tokens(self._h, req, _i32p(t), prompt_len, max_new_tokens)

    def step(self) -> dict:
        """Schedule one step; returns info plus the prefill/decode entries and the slot mapping."""
        from ._lib import StepInfo
        pr, pc, pl, dr, dl, sm = self._bufs
        info = StepInfo()
        check(lib().pa_sched_step(self._h, byref(info), *self._ptrs))
        d = info.as_dict()
        P, D, T = info.num_prefill, info.num_decode, info.num_tokens
        d.update(prefill_reqs=pr[:P].copy(), prefill_ctx=pc[:P].copy(), prefill_len=pl[:P].copy(),
                 decode_reqs=dr[:D].copy(), decode_seq_lens=dl[:D].copy(), slot_mapping=sm[:T].copy())
        if self._cpu is not None:
            d["swap_out"], d["swap_in"] = self.last_swaps()
        return d

    def enable_swap(self, cpu: "BlockAllocator") -> int:
        """Preempt by swapping to `cpu` (a BlockAllocator over the host pool; None: recompute)."""
        st = lib().pa_sched_enable_swap(self._h, None if cpu is None else cpu._h)
        if st == PA_OK:
            self._cpu = cpu                       # the C scheduler borrows it
        return st

    def last_swaps(self):
        """Block moves of the last step: (swap-out pairs [n, 2] GPU -> CPU, swap-in pairs [m, 2] CPU -> GPU)."""
        no, ni = c_int32(0), c_int32(0)
        check(lib().pa_sched_last_swaps(self._h, None, 0, byref(no), None, 0, byref(ni)))
        out = np.empty((no.value, 2), np.int64)
        inn = np.empty((ni.value, 2), np.int64)
        check(lib().pa_sched_last_swaps(self._h, _i64p(out), no.value, byref(no), _i64p(inn), ni.value, byref(ni)))
        return out, inn

    def complete(self, sampled=None) -> None:
        """Apply the step; `sampled` (optional) = the ids of the tokens it emitted, in emission order."""
        if sampled is None:
            check(lib().pa_sched_complete(self._h))
            return
        t = np.ascontiguousarray(sampled, dtype=np.int32)
        check(lib().pa_sched_complete_tokens(self._h, _i32p(t), len(t)))

    def request_info(self, req: int):
        from ._lib import RequestInfo
        r = RequestInfo()
        st = lib().pa_sched_request_info(self._h, req, byref(r))
        return st, (r.as_dict() if st == PA_OK else None)

    def stats(self) -> dict:
        from ._lib import SchedStats
        s = SchedStats()
        check(lib().pa_sched_stats(self._h, byref(s)))
        return s.as_dict()


# ------------------------------------------------------------------ swapping
def _ptr_any(t):
    if t is None:
        return None
    return c_void_p(t.data_ptr() if hasattr(t, "data_ptr") else int(t))


def _stream_handle(stream):
    if stream is None:
        try:
            import torch
            if torch.cuda.is_available():
                return c_void_p(torch.cuda.current_stream().cuda_stream)
        except ImportError:
            pass
        return None
    return c_void_p(stream.cuda_stream)


def swap_blocks(src_k, src_v, dst_k, dst_v, mapping, block_bytes, src_num_blocks, dst_num_blocks, stream=None):
    """pa_swap_blocks: mapping is an int64 [n, 2] host array of (source block, destination block)."""
    m = np.ascontiguousarray(mapping, dtype=np.int64).reshape(-1, 2)
    check(lib().pa_swap_blocks(_ptr_any(src_k), _ptr_any(src_v), _ptr_any(dst_k), _ptr_any(dst_v), _i64p(m),
                               len(m), int(block_bytes), src_num_blocks, dst_num_blocks, _stream_handle(stream)))


def swap_out(gpu_alloc, cpu_alloc, req, gpu_k, gpu_v, cpu_k, cpu_v, block_bytes, stream=None) -> int:
    """pa_alloc_swap_out; returns the status (PA_ERR_OOM when the host pool is full)."""
    return lib().pa_alloc_swap_out(gpu_alloc._h, cpu_alloc._h, req, _ptr_any(gpu_k), _ptr_any(gpu_v),
                                   _ptr_any(cpu_k), _ptr_any(cpu_v), int(block_bytes), _stream_handle(stream))


def swap_in(gpu_alloc, cpu_alloc, req, gpu_k, gpu_v, cpu_k, cpu_v, block_bytes, stream=None) -> int:
    """pa_alloc_swap_in; returns the status (PA_ERR_OOM when the GPU pool is full)."""
    return lib().pa_alloc_swap_in(gpu_alloc._h, cpu_alloc._h, req, _ptr_any(gpu_k), _ptr_any(gpu_v),
                                  _ptr_any(cpu_k), _ptr_any(cpu_v), int(block_bytes), _stream_handle(stream))


# ------------------------------------------------------------------ kernels
def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return c_void_p(stream.cuda_stream)


def _need(cond, msg):
    if not cond:
        raise PagedKVError(PA_ERR_INVALID_ARG, msg)


def _on_device(*ts):
    """The kernels dereference every pointer on the current device: refuse host tensors and tensors of
    another GPU here, before the C call (the library itself does not inspect pointers)."""
    import torch
    ts = [t for t in ts if t is not None]
    for t in ts:
        _need(t.is_cuda, f"CUDA tensors expected; got one on {t.device}")
    dev = torch.cuda.current_device()
    for t in ts:
        _need(t.get_device() == dev, f"tensors must be on the current CUDA device (cuda:{dev}); got one on {t.device}")


def reshape_and_cache(k_new, v_new, k_cache, v_cache, slot_mapping, err_flag=None, stream=None):
    """pa_reshape_and_cache on torch tensors: k_new/v_new [T,H,D] fp16, caches [NB,bs,H,D] fp16,
    slot_mapping [T] int64 (device)."""
    import torch
    _need(k_new.dtype == torch.float16 and k_cache.dtype == torch.float16, "fp16 tensors expected")
    _need(slot_mapping.dtype == torch.int64, "slot_mapping must be int64")
    _need(all(t.is_contiguous() for t in (k_new, v_new, k_cache, v_cache, slot_mapping)), "contiguous tensors expected")
    _on_device(k_new, v_new, k_cache, v_cache, slot_mapping, err_flag)
    T, H, D = k_new.shape
    NB, bs = k_cache.shape[:2]
    check(lib().pa_reshape_and_cache(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
                                     T, H, D, bs, NB, _ptr(err_flag), _stream(stream)))


def decode_workspace_bytes(num_seqs: int, num_heads: int, head_dim: int, max_blocks: int, block_size: int) -> int:
    return int(lib().pa_decode_workspace_bytes(num_seqs, num_heads, head_dim, max_blocks, block_size))


def paged_attention_decode(out, q, k_cache, v_cache, block_tables, seq_lens, scale, workspace,
                           err_flag=None, stream=None):
    """pa_paged_attention_decode on torch tensors: out/q [S,H,D] fp16, caches [NB,bs,H,D] fp16,
    block_tables [S,max_blocks] int32, seq_lens [S] int32, workspace uint8 (device)."""
    import torch
    _need(q.dtype == torch.float16 and out.dtype == torch.float16, "fp16 tensors expected")
    _need(block_tables.dtype == torch.int32 and seq_lens.dtype == torch.int32, "int32 tables expected")
    _need(all(t.is_contiguous() for t in (out, q, k_cache, v_cache, block_tables, seq_lens)), "contiguous tensors expected")
    _on_device(out, q, k_cache, v_cache, block_tables, seq_lens, workspace, err_flag)
    S, H, D = q.shape
    NB, bs = k_cache.shape[:2]
    max_blocks = block_tables.shape[1] if block_tables.dim() == 2 else 0
    check(lib().pa_paged_attention_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                          _ptr(seq_lens), S, H, D, bs, max_blocks, NB, float(scale),
                                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          _ptr(err_flag), _stream(stream)))


def paged_attention_decode_noalloc(out, q, k_cache, v_cache, block_tables, seq_lens, scale, err_flag=None,
                                   stream=None):
    """pa_paged_attention_decode_noalloc on torch tensors: as paged_attention_decode, with the
    library's fixed device scratch instead of a caller workspace (for callers that cannot allocate)."""
    import torch
    _need(q.dtype == torch.float16 and out.dtype == torch.float16, "fp16 tensors expected")
    _need(block_tables.dtype == torch.int32 and seq_lens.dtype == torch.int32, "int32 tables expected")
    _need(all(t.is_contiguous() for t in (out, q, k_cache, v_cache, block_tables, seq_lens)), "contiguous tensors expected")
    _on_device(out, q, k_cache, v_cache, block_tables, seq_lens, err_flag)
    S, H, D = q.shape
    NB, bs = k_cache.shape[:2]
    check(lib().pa_paged_attention_decode_noalloc(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                                  _ptr(block_tables), _ptr(seq_lens), S, H, D, bs,
                                                  block_tables.shape[1], NB, float(scale), _ptr(err_flag),
                                                  _stream(stream)))


def paged_attention_prefill_chunk(out, q, k_cache, v_cache, block_tables, q_start, ctx_before, scale,
                                  err_flag=None, stream=None):
    """pa_paged_attention_prefill_chunk on torch tensors: out/q [T,H,D] fp16, caches [NB,bs,H,D] fp16,
    block_tables [B,max_blocks] int32, q_start [B+1] int32, ctx_before [B] int32 (device)."""
    import torch
    _need(q.dtype == torch.float16 and out.dtype == torch.float16, "fp16 tensors expected")
    _need(all(t.is_contiguous() for t in (out, q, k_cache, v_cache, block_tables, q_start, ctx_before)),
          "contiguous tensors expected")
    _on_device(out, q, k_cache, v_cache, block_tables, q_start, ctx_before, err_flag)
    T, H, D = q.shape
    NB, bs = k_cache.shape[:2]
    B = ctx_before.shape[0]
    check(lib().pa_paged_attention_prefill_chunk(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                                 _ptr(block_tables), _ptr(q_start), _ptr(ctx_before), B, T, H, D,
                                                 bs, block_tables.shape[1], NB, float(scale), _ptr(err_flag),
                                                 _stream(stream)))
