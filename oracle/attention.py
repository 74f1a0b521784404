"""Oracle paged attention in float64 (test infrastructure only).

Restates what the page "LLM 推理引擎 Continuous Batching 与 PagedAttention"
defines:

* §3.3 (GPU Kernel 中的分页读取): a sequence's token j lives in physical
  block ``block_table[j // block_size]`` at row ``j % block_size``; the
  kernel scores ``q . k_j * scale`` with a softmax over all positions of
  the sequence and (the step the page leaves out as "省略") weights V by it.
  Cache layout read here: ``[num_blocks, block_size, num_heads, head_dim]``
  for K and V separately (the page's pointer arithmetic
  ``+ head_idx * head_dim`` puts heads inside a token row).
* §1.1 / §4.3: decode attends one new query per sequence over the whole
  cached sequence including the new token; a prefill chunk of queries at
  absolute positions ``ctx_before + i`` attends causally to keys
  ``0 .. ctx_before + i``.
* The step's new K/V is written into the cache at the slots of the slot
  mapping (``block = slot // block_size``, ``row = slot % block_size``);
  a negative slot is a padding token and is skipped.

The cache arguments may be NumPy arrays or any mapping ``block -> [bs, H, D]``
(used for full-size workloads where only sampled sequences are built).
fp16 inputs are widened to float64 exactly; no arithmetic runs below fp64.
"""
from __future__ import annotations

import numpy as np


def reshape_and_cache(k_cache, v_cache, k_new, v_new, slot_mapping, block_size: int) -> None:
    """Write token t's K/V rows [H, D] at slot_mapping[t] (in place; slot < 0 skipped)."""
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        block, row = divmod(int(slot), block_size)
        k_cache[block][row] = k_new[t]
        v_cache[block][row] = v_new[t]


def gather_sequence(cache, block_table, seq_len: int, block_size: int) -> np.ndarray:
    """Logical rows 0..seq_len-1 of one sequence, widened to float64 ([seq_len, H, D])."""
    table = np.asarray(block_table)
    if seq_len == 0:
        first = cache[0] if isinstance(cache, np.ndarray) else next(iter(cache.values()))
        return np.zeros((0,) + tuple(first.shape[1:]), dtype=np.float64)
    pos = np.arange(seq_len)
    blocks = table[pos // block_size]
    rows = pos % block_size
    if isinstance(cache, np.ndarray):
        return cache[blocks, rows].astype(np.float64)
    return np.stack([cache[int(b)][int(r)] for b, r in zip(blocks, rows)]).astype(np.float64)


def softmax_attention(q, k, v, scale: float, allowed=None) -> np.ndarray:
    """softmax(scale * q k^T) v per head, float64 with max subtraction.

    q [L, H, D], k and v [n, H, D]; ``allowed`` [L, n] bool masks keys per
    query (None = all).  A query row with no key returns zeros.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L, H, D = q.shape
    if k.shape[0] == 0:
        return np.zeros((L, H, D), dtype=np.float64)
    qh = q.transpose(1, 0, 2)                      # [H, L, D]
    kh = k.transpose(1, 0, 2)                      # [H, n, D]
    vh = v.transpose(1, 0, 2)                      # [H, n, D]
    s = scale * np.matmul(qh, kh.transpose(0, 2, 1))   # [H, L, n]
    if allowed is not None:
        s = np.where(np.asarray(allowed)[None], s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    empty = ~np.isfinite(m)
    m = np.where(empty, 0.0, m)
    p = np.exp(s - m)
    l = p.sum(axis=-1, keepdims=True)
    o = np.matmul(p, vh) / np.where(l == 0, 1.0, l)    # [H, L, D]
    return o.transpose(1, 0, 2)


def paged_attention_decode(q, k_cache, v_cache, block_tables, seq_lens, block_size: int,
                           scale: float) -> np.ndarray:
    """Decode: out[s] = attention of q[s] over sequence s's cached rows 0..seq_lens[s]-1."""
    q = np.asarray(q)
    S, H, D = q.shape
    out = np.zeros((S, H, D), dtype=np.float64)
    for s in range(S):
        n = int(seq_lens[s])
        if n == 0:
            continue
        k = gather_sequence(k_cache, block_tables[s], n, block_size)
        v = gather_sequence(v_cache, block_tables[s], n, block_size)
        out[s] = softmax_attention(q[s][None], k, v, scale)[0]
    return out


def paged_attention_prefill_chunk(q, k_cache, v_cache, block_tables, q_start, ctx_before,
                                  block_size: int, scale: float) -> np.ndarray:
    """Causal chunk: query row i of request b sits at position ctx_before[b] + i and sees
    keys 0 .. ctx_before[b] + i of its own sequence."""
    q = np.asarray(q)
    out = np.zeros(q.shape, dtype=np.float64)
    for b in range(len(ctx_before)):
        lo, hi = int(q_start[b]), int(q_start[b + 1])
        L = hi - lo
        if L == 0:
            continue
        c = int(ctx_before[b])
        n = c + L
        k = gather_sequence(k_cache, block_tables[b], n, block_size)
        v = gather_sequence(v_cache, block_tables[b], n, block_size)
        allowed = np.arange(n)[None, :] <= (c + np.arange(L))[:, None]
        out[lo:hi] = softmax_attention(q[lo:hi], k, v, scale, allowed)
    return out
