"""Replays a seeded workload recipe through the oracle (test infrastructure only).

The recipe (pool size, churn, request order, which tokens exist before the
step) is stated once here and once, independently, in the CUDA side's
builder; both consume the same draws from ``synth_inputs``.  The order of
operations is:

1. Pool of N blocks, N = ceil(pool_factor * demand) (or fixed), demand being
   the blocks the step's requests need; free list in the recipe's order.
2. Churn (if any): op i allocates request CHURN_REQ_BASE + i with its drawn
   token count, appends one token to, or frees, the live churn request at
   index floor(u * #live) (creation order).  Churn holdings are capped at
   N - demand blocks; an op that would cross the cap is skipped.  The churn
   requests still live at the end are freed in the drawn order.
3. Shared prefix (if any): allocate it and write its K/V.
4. Prefill request (if any): allocate its cached prefix and write its K/V.
5. Decode sequence s = 0..S-1: fork the shared prefix then append its private
   context, or allocate its context of seq_len - 1 tokens; write its K/V.
6. The step: append the prefill chunk's tokens, then one token per decode
   sequence; these slots form the step's slot mapping (chunk rows first).
7. The shared-prefix request itself is freed (its blocks stay referenced).

The cache content written here is the state *before* the step's
reshape_and_cache.  Positions are written through the block manager's slot
mapping (page "LLM 推理引擎 Continuous Batching 与 PagedAttention", §3.3).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

import synth_inputs as si

from . import attention
from .block_manager import OK, BlockManager
from .sizes import blocks_needed


class _NanBlocks(dict):
    """Sparse cache: block id -> fp16 [bs, H, D], created as NaN on first touch."""

    def __init__(self, shape):
        super().__init__()
        self._shape = shape

    def __missing__(self, key):
        arr = np.full(self._shape, np.nan, dtype=np.float16)
        self[key] = arr
        return arr


@dataclasses.dataclass
class OracleStep:
    workload: si.Workload
    num_blocks: int
    bm: BlockManager
    cap_hits: int
    max_blocks: int
    block_tables: np.ndarray          # [S, max_blocks] int32, pad -1
    seq_lens: np.ndarray              # [S] int32, incl. the step's token
    slot_mapping: np.ndarray          # [T] int64: prefill chunk rows, then decode rows
    k_step: np.ndarray                # [T, H, D] fp16
    v_step: np.ndarray
    q: np.ndarray                     # [S, H, D] fp16 decode queries
    k_cache: object                   # before the step: ndarray [N,bs,H,D] or sparse dict
    v_cache: object
    prefill_q: Optional[np.ndarray] = None
    prefill_table: Optional[np.ndarray] = None   # [1, max_blocks_prefill]
    prefill_ctx_before: int = 0
    sampled: Optional[list] = None    # decode sequences whose cache content exists (None = all)


def demand_blocks(w: si.Workload) -> int:
    bs = w.block_size
    if w.shared_prefix:
        shared = (w.shared_prefix // bs) * bs
        d = blocks_needed(w.shared_prefix, bs) + sum(blocks_needed(n - shared, bs) for n in w.decode_lens)
    else:
        d = sum(blocks_needed(n, bs) for n in w.decode_lens)
    if w.prefill is not None:
        d += blocks_needed(w.prefill.ctx_before + w.prefill.chunk, bs)
    return d


def pool_blocks(w: si.Workload) -> int:
    if w.pool_blocks is not None:
        return w.pool_blocks
    return int(math.ceil(w.pool_factor * demand_blocks(w)))


def _check(st):
    if st != OK:
        raise RuntimeError(f"oracle workload replay failed: {st}")


def _write(bm, k_cache, v_cache, req, pos0, k, v):
    st, slots = bm.slots(req, pos0, len(k))
    _check(st)
    attention.reshape_and_cache(k_cache, v_cache, k, v, slots, bm.block_size)


def build(w: si.Workload, seqs=None) -> OracleStep:
    """Replay ``w``.  ``seqs`` limits the cache content to those decode sequences
    (plus the shared prefix and prefill request) and switches to a sparse cache."""
    bs, H, D = w.block_size, w.num_heads, w.head_dim
    N = pool_blocks(w)
    demand = demand_blocks(w)
    bm = BlockManager(N, bs, w.free_order(N))

    # 2. churn
    cap_hits = 0
    if w.churn is not None:
        cap = N - demand
        kind, u, tokens = w.churn_ops()
        live: list[int] = []
        for i in range(w.churn.n_ops):
            used = N - len(bm.free_blocks)
            if kind[i] == 0:
                if used + blocks_needed(int(tokens[i]), bs) > cap:
                    cap_hits += 1
                    continue
                req = si.CHURN_REQ_BASE + i
                _check(bm.allocate(req, int(tokens[i])))
                live.append(req)
            elif kind[i] == 1:
                if not live:
                    continue
                req = live[int(u[i] * len(live))]
                if bm.seq_lens[req] % bs == 0 and used + 1 > cap:
                    cap_hits += 1
                    continue
                _check(bm.append_token(req)[0])
            else:
                if not live:
                    continue
                _check(bm.free(live.pop(int(u[i] * len(live)))))
        for j in w.churn_final_order(len(live)):
            _check(bm.free(live[int(j)]))

    sparse = seqs is not None
    want = set(range(w.num_seqs)) if seqs is None else set(int(s) for s in seqs)
    if sparse:
        k_cache, v_cache = _NanBlocks((bs, H, D)), _NanBlocks((bs, H, D))
    else:
        k_cache = np.full((N, bs, H, D), np.nan, dtype=np.float16)
        v_cache = np.full((N, bs, H, D), np.nan, dtype=np.float16)

    # 3. shared prefix
    if w.shared_prefix:
        _check(bm.allocate(si.PREFIX_REQ, w.shared_prefix))
        kp, vp = w.prefix_kv()
        _write(bm, k_cache, v_cache, si.PREFIX_REQ, 0, kp, vp)

    # 4. prefill request's cached prefix
    if w.prefill is not None:
        _check(bm.allocate(si.PREFILL_REQ, w.prefill.ctx_before))
        kc, vc = w.prefill_context_kv()
        _write(bm, k_cache, v_cache, si.PREFILL_REQ, 0, kc, vc)

    # 5. decode sequences' context
    for s, n in enumerate(w.decode_lens):
        if w.shared_prefix:
            _check(bm.fork(si.PREFIX_REQ, s, w.shared_prefix))
            start = bm.seq_lens[s]
            _check(bm.append_tokens(s, n - 1 - start)[0])
        else:
            start = 0
            _check(bm.allocate(s, n - 1))
        if s in want:
            k, v = w.context_kv(s, n - 1 - start)
            _write(bm, k_cache, v_cache, s, start, k, v)

    # 6. the step's appends
    step_slots = []
    k_parts, v_parts = [], []
    prefill_q = prefill_table = None
    if w.prefill is not None:
        st, slots = bm.append_tokens(si.PREFILL_REQ, w.prefill.chunk)
        _check(st)
        step_slots += slots
        prefill_q, kq, vq = w.prefill_qkv()
        k_parts.append(kq)
        v_parts.append(vq)
        t = bm.block_tables[si.PREFILL_REQ]
        prefill_table = np.asarray([t], dtype=np.int32)
    for s in range(w.num_seqs):
        st, slot = bm.append_token(s)
        _check(st)
        step_slots.append(slot)
    k_parts.append(w.k_new())
    v_parts.append(w.v_new())

    # 7. drop the prefix owner
    if w.shared_prefix:
        _check(bm.free(si.PREFIX_REQ))

    max_blocks = max((blocks_needed(n, bs) for n in w.decode_lens), default=1)
    st, tables, lens = bm.pack(list(range(w.num_seqs)), max_blocks)
    _check(st)
    return OracleStep(
        workload=w, num_blocks=N, bm=bm, cap_hits=cap_hits, max_blocks=max_blocks,
        block_tables=np.asarray(tables, dtype=np.int32).reshape(-1, max_blocks), seq_lens=np.asarray(lens, dtype=np.int32),
        slot_mapping=np.asarray(step_slots, dtype=np.int64),
        k_step=np.concatenate(k_parts), v_step=np.concatenate(v_parts), q=w.q(),
        k_cache=k_cache, v_cache=v_cache, prefill_q=prefill_q, prefill_table=prefill_table,
        prefill_ctx_before=0 if w.prefill is None else w.prefill.ctx_before,
        sampled=sorted(want) if sparse else None)


def run_step(step: OracleStep):
    """The step on the oracle: reshape_and_cache, then decode (and the prefill chunk).

    Returns (decode_out [S,H,D] f64, prefill_out [L,H,D] f64 or None, k_cache, v_cache after).
    Sparse caches hold only the sampled sequences, so only their rows are meaningful."""
    w = step.workload
    if isinstance(step.k_cache, np.ndarray):
        kc, vc = step.k_cache.copy(), step.v_cache.copy()
    else:
        kc, vc = _NanBlocks(step.k_cache._shape), _NanBlocks(step.v_cache._shape)
        for b, a in step.k_cache.items():
            kc[b] = a.copy()
        for b, a in step.v_cache.items():
            vc[b] = a.copy()
    attention.reshape_and_cache(kc, vc, step.k_step, step.v_step, step.slot_mapping, w.block_size)
    dec = paged_decode_subset(step, kc, vc, step.sampled)
    pre = None
    if w.prefill is not None:
        L = w.prefill.chunk
        pre = attention.paged_attention_prefill_chunk(
            step.prefill_q, kc, vc, step.prefill_table, [0, L], [step.prefill_ctx_before],
            w.block_size, w.scale)
    return dec, pre, kc, vc


def paged_decode_subset(step: OracleStep, kc, vc, seqs=None):
    """Decode outputs for ``seqs`` (None = all); the other rows are NaN."""
    w = step.workload
    S = w.num_seqs
    out = np.full((S, w.num_heads, w.head_dim), np.nan)
    seqs = list(range(S)) if seqs is None else list(seqs)
    if seqs:
        idx = np.asarray(seqs)
        out[idx] = attention.paged_attention_decode(
            step.q[idx], kc, vc, step.block_tables[idx], step.seq_lens[idx], w.block_size, w.scale)
    return out
