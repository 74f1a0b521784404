"""Builds one synthetic paged-attention step on the GPU through libpagedkv.

The recipe: a pool sized from the requests' demand, optional allocate/append/
free churn to fragment it, an optional shared prefix forked into every
decode sequence, an optional chunked-prefill request, each decode sequence's
cached context, then the step's appends (prefill chunk rows first, then one
token per decode sequence), whose slots form the step's slot mapping.  All
block bookkeeping runs in the C++ allocator (``BlockAllocator``); the cached
context is written into the pool with the library's ``reshape_and_cache``
kernel.  Random draws come from ``synth_inputs``; unused pool rows hold NaN so
that a read of a row outside a sequence shows up in the output.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import synth_inputs as si

from . import PA_OK, BlockAllocator, reshape_and_cache

try:
    import torch
except ImportError:  # the host replay needs no torch
    torch = None


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def demand_blocks(w: si.Workload) -> int:
    bs = w.block_size
    if w.shared_prefix:
        shared = (w.shared_prefix // bs) * bs
        d = _ceil_div(w.shared_prefix, bs) + sum(_ceil_div(n - shared, bs) for n in w.decode_lens)
    else:
        d = sum(_ceil_div(n, bs) for n in w.decode_lens)
    if w.prefill is not None:
        d += _ceil_div(w.prefill.ctx_before + w.prefill.chunk, bs)
    return d


def pool_blocks(w: si.Workload) -> int:
    return w.pool_blocks if w.pool_blocks is not None else int(math.ceil(w.pool_factor * demand_blocks(w)))


@dataclasses.dataclass
class DeviceStep:
    workload: si.Workload
    alloc: BlockAllocator
    num_blocks: int
    max_blocks: int
    k_cache: torch.Tensor            # [N, bs, H, D] fp16, state before the step
    v_cache: torch.Tensor
    q: torch.Tensor                  # [S, H, D] decode queries
    k_step: torch.Tensor             # [T, H, D] rows the step writes (prefill chunk, then decode)
    v_step: torch.Tensor
    slot_mapping: torch.Tensor       # [T] int64
    block_tables: torch.Tensor       # [S, max_blocks] int32
    seq_lens: torch.Tensor           # [S] int32
    tables_host: np.ndarray
    seq_lens_host: np.ndarray
    slots_host: np.ndarray
    cap_hits: int = 0
    prefill_q: Optional[torch.Tensor] = None
    prefill_table: Optional[torch.Tensor] = None     # [1, blocks] int32
    prefill_q_start: Optional[torch.Tensor] = None   # [2] int32
    prefill_ctx_before: Optional[torch.Tensor] = None

    @property
    def decode_kv_bytes(self) -> int:
        """Algorithmic K+V bytes decode reads: sum of seq_len * H * D * 2 tensors * 2 bytes."""
        w = self.workload
        return int(self.seq_lens_host.astype(np.int64).sum()) * w.num_heads * w.head_dim * 4


def _ok(st):
    if st != PA_OK:
        raise RuntimeError(f"workload replay failed with status {st}")


@dataclasses.dataclass
class HostReplay:
    """The recipe replayed through the C++ allocator (no GPU needed)."""
    workload: si.Workload
    alloc: BlockAllocator
    num_blocks: int
    cap_hits: int
    segments: list                  # (slots int64[n], source, seq index, first position)
    step_slots: np.ndarray          # [T] int64: prefill chunk rows, then one per decode sequence
    prefill_table: Optional[np.ndarray]


def replay(w: si.Workload) -> HostReplay:
    """Run the allocation side of the recipe (pool, churn, prefix, prefill, context, step appends)."""
    bs = w.block_size
    N = pool_blocks(w)
    demand = demand_blocks(w)
    alloc = BlockAllocator(N, bs, w.free_order(N))

    cap_hits = 0
    if w.churn is not None:
        cap = N - demand
        kind, u, tokens = w.churn_ops()
        live = []
        for i in range(w.churn.n_ops):
            used = N - alloc.stats()["num_free"]
            k = int(kind[i])
            if k == 0:
                if used + _ceil_div(int(tokens[i]), bs) > cap:
                    cap_hits += 1
                    continue
                req = si.CHURN_REQ_BASE + i
                _ok(alloc.allocate(req, int(tokens[i])))
                live.append(req)
            elif k == 1:
                if not live:
                    continue
                req = live[int(u[i] * len(live))]
                if alloc.seq_len(req)[1] % bs == 0 and used + 1 > cap:
                    cap_hits += 1
                    continue
                _ok(alloc.append_token(req)[0])
            else:
                if not live:
                    continue
                _ok(alloc.free(live.pop(int(u[i] * len(live)))))
        for j in w.churn_final_order(len(live)):
            _ok(alloc.free(live[int(j)]))

    segments = []

    def record(req, pos0, n, source, index):
        st, sl = alloc.slots(req, pos0, n)
        _ok(st)
        segments.append((sl, source, index, pos0))

    if w.shared_prefix:
        _ok(alloc.allocate(si.PREFIX_REQ, w.shared_prefix))
        record(si.PREFIX_REQ, 0, w.shared_prefix, "prefix", -1)
    if w.prefill is not None:
        _ok(alloc.allocate(si.PREFILL_REQ, w.prefill.ctx_before))
        record(si.PREFILL_REQ, 0, w.prefill.ctx_before, "prefill_ctx", -1)
    for s, n in enumerate(w.decode_lens):
        if w.shared_prefix:
            _ok(alloc.fork(si.PREFIX_REQ, s, w.shared_prefix))
            start = alloc.seq_len(s)[1]
            _ok(alloc.append_tokens(s, n - 1 - start)[0])
        else:
            start = 0
            _ok(alloc.allocate(s, n - 1))
        record(s, start, n - 1 - start, "context", s)

    step = []
    prefill_table = None
    if w.prefill is not None:
        st, ps = alloc.append_tokens(si.PREFILL_REQ, w.prefill.chunk)
        _ok(st)
        step.append(ps)
        prefill_table = alloc.get_block_table(si.PREFILL_REQ)[1][None].copy()
    dec = np.empty(w.num_seqs, dtype=np.int64)
    for s in range(w.num_seqs):
        st, slot = alloc.append_token(s)
        _ok(st)
        dec[s] = slot
    step.append(dec)
    if w.shared_prefix:
        _ok(alloc.free(si.PREFIX_REQ))
    return HostReplay(workload=w, alloc=alloc, num_blocks=N, cap_hits=cap_hits, segments=segments,
                      step_slots=np.concatenate(step), prefill_table=prefill_table)


def build(w: si.Workload, device="cuda", pad="neg1", max_blocks: Optional[int] = None) -> DeviceStep:
    """Replay ``w`` and return the step's device tensors.

    pad: "neg1" fills block-table padding with -1; "garbage" with in-range
    wrong block ids (a kernel that reads past ceil(seq_len / bs) then reads
    NaN rows or another sequence's rows)."""
    bs, H, D = w.block_size, w.num_heads, w.head_dim
    r = replay(w)
    N = r.num_blocks
    k_cache = torch.full((N, bs, H, D), float("nan"), dtype=torch.float16, device=device)
    v_cache = torch.full((N, bs, H, D), float("nan"), dtype=torch.float16, device=device)
    for sl, source, index, pos0 in r.segments:
        if source == "prefix":
            k, v = w.prefix_kv()
        elif source == "prefill_ctx":
            k, v = w.prefill_context_kv()
        else:
            k, v = w.context_kv(index, len(sl))
        if len(sl) == 0:
            continue
        reshape_and_cache(torch.from_numpy(k).to(device), torch.from_numpy(v).to(device), k_cache, v_cache,
                          torch.from_numpy(sl).to(device))

    k_parts, v_parts = [], []
    prefill_q = prefill_table = q_start = ctx_before = None
    if w.prefill is not None:
        qc, kq, vq = w.prefill_qkv()
        k_parts.append(kq)
        v_parts.append(vq)
        prefill_q = torch.from_numpy(qc).to(device)
        prefill_table = torch.from_numpy(r.prefill_table).to(device)
        q_start = torch.tensor([0, w.prefill.chunk], dtype=torch.int32, device=device)
        ctx_before = torch.tensor([w.prefill.ctx_before], dtype=torch.int32, device=device)
    k_parts.append(w.k_new())
    v_parts.append(w.v_new())

    need = max((_ceil_div(n, bs) for n in w.decode_lens), default=1)
    mb = need if max_blocks is None else max(need, max_blocks)
    st, tables, lens = r.alloc.pack(np.arange(w.num_seqs), mb)
    _ok(st)
    if pad == "garbage":
        g = si.garbage_block_ids(w.seed, tables.shape, N)
        tables = np.where(tables >= 0, tables, g)
    return DeviceStep(
        workload=w, alloc=r.alloc, num_blocks=N, max_blocks=mb, k_cache=k_cache, v_cache=v_cache,
        q=torch.from_numpy(w.q()).to(device),
        k_step=torch.from_numpy(np.concatenate(k_parts)).to(device),
        v_step=torch.from_numpy(np.concatenate(v_parts)).to(device),
        slot_mapping=torch.from_numpy(r.step_slots).to(device),
        block_tables=torch.from_numpy(tables).to(device), seq_lens=torch.from_numpy(lens).to(device),
        tables_host=tables, seq_lens_host=lens, slots_host=r.step_slots, cap_hits=r.cap_hits,
        prefill_q=prefill_q, prefill_table=prefill_table, prefill_q_start=q_start,
        prefill_ctx_before=ctx_before)
