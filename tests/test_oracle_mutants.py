"""Plants plausible mistakes in the CPU oracle and checks that a pin catches each one.

Each mutant replaces one oracle function (on the CPU, for the duration of one
test) with a copy carrying a single mistake: a dropped scale, swapped
operands, a wrong block index, an off-by-one causal bound, a FIFO free list,
and so on.  The pins in ``test_oracle_pins`` must fail on every mutant.
"""
import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import attention as oatt
from oracle import block_manager as obm
from oracle import sizes

_orig_softmax = oatt.softmax_attention
_orig_gather = oatt.gather_sequence
_orig_prefill = oatt.paged_attention_prefill_chunk


def _no_scale(q, k, v, scale, allowed=None):
    return _orig_softmax(q, k, v, 1.0, allowed)


def _swap_kv(q, k, v, scale, allowed=None):
    return _orig_softmax(q, v, k, scale, allowed)


def _no_max_guard_wrong_sign(q, k, v, scale, allowed=None):
    return _orig_softmax(q, k, v, -scale, allowed)


def _gather_mod_index(cache, block_table, seq_len, block_size):
    table = np.asarray(block_table)
    pos = np.arange(seq_len)
    blocks = table[pos % len(table)] if len(table) else table
    rows = pos % block_size
    return np.asarray(cache)[blocks, rows].astype(np.float64)


def _gather_ignores_table(cache, block_table, seq_len, block_size):
    pos = np.arange(seq_len)
    first = int(np.asarray(block_table)[0])
    return np.asarray(cache)[first + pos // block_size, pos % block_size].astype(np.float64)


def _prefill_strict_causal(q, k_cache, v_cache, block_tables, q_start, ctx_before, block_size, scale):
    out = np.zeros(np.asarray(q).shape)
    for b in range(len(ctx_before)):
        lo, hi = int(q_start[b]), int(q_start[b + 1])
        L, c = hi - lo, int(ctx_before[b])
        k = oatt.gather_sequence(k_cache, block_tables[b], c + L, block_size)
        v = oatt.gather_sequence(v_cache, block_tables[b], c + L, block_size)
        allowed = np.arange(c + L)[None, :] < (c + np.arange(L))[:, None] + (np.arange(L)[:, None] == 0)
        out[lo:hi] = oatt.softmax_attention(q[lo:hi], k, v, scale, allowed)
    return out


def _prefill_ignores_context(q, k_cache, v_cache, block_tables, q_start, ctx_before, block_size, scale):
    return _orig_prefill(q, k_cache, v_cache, block_tables, q_start, [0] * len(ctx_before), block_size, scale)


class _FifoBM(obm.BlockManager):
    def allocate(self, req, num_tokens):
        self.free_blocks.reverse()
        st = super().allocate(req, num_tokens)
        self.free_blocks.reverse()
        return st


class _EarlyAppendBM(obm.BlockManager):
    def append_token(self, req):
        if req not in self.block_tables:
            return obm.NOT_FOUND, None
        cur = self.seq_lens[req]
        if cur % self.block_size == self.block_size - 1 or not self.block_tables[req]:
            if not self.free_blocks:
                return obm.OOM, None
            b = self.free_blocks.pop()
            self.refcount[b] += 1
            self.block_tables[req].append(b)
        self.seq_lens[req] = cur + 1
        t = self.block_tables[req]
        return obm.OK, t[min(cur // self.block_size, len(t) - 1)] * self.block_size + cur % self.block_size


class _ReverseFreeBM(obm.BlockManager):
    def free(self, req):
        if req in self.block_tables:
            self.block_tables[req] = self.block_tables[req][::-1]
        return super().free(req)


class _CeilForkBM(obm.BlockManager):
    def fork(self, src, dst, prefix_tokens):
        st = super().fork(src, dst, 0)
        if st != obm.OK:
            return st
        blocks = list(self.block_tables[src][:-(-prefix_tokens // self.block_size)])
        for b in blocks:
            self.refcount[b] += 1
        self.block_tables[dst] = blocks
        self.seq_lens[dst] = prefix_tokens
        return obm.OK


class _NoRefcountBM(obm.BlockManager):
    def free(self, req):
        if req not in self.block_tables:
            return obm.OK
        for b in self.block_tables[req]:
            self.refcount[b] = 0
            if b not in self.free_blocks:
                self.free_blocks.append(b)
        del self.block_tables[req]
        del self.seq_lens[req]
        return obm.OK


def _floor_blocks(n, bs):
    return n // bs


def _kv_no_two(layers, heads, head_dim, b):
    return layers * heads * head_dim * b


MUTANTS = [
    ("attention drops scale", oatt, "softmax_attention", _no_scale,
     [lambda: pins.test_decode_matches_torch_sdpa(4, 64, 16, [5, 16, 17, 33])]),
    ("attention swaps K and V", oatt, "softmax_attention", _swap_kv,
     [lambda: pins.test_decode_matches_torch_sdpa(2, 128, 16, [1, 64, 100])]),
    ("attention flips score sign", oatt, "softmax_attention", _no_max_guard_wrong_sign,
     [lambda: pins.test_decode_scale_is_honoured()]),
    ("gather indexes table by j % len", oatt, "gather_sequence", _gather_mod_index,
     [lambda: pins.test_decode_matches_torch_sdpa(3, 32, 32, [31, 32, 33, 200])]),
    ("gather ignores the table", oatt, "gather_sequence", _gather_ignores_table,
     [lambda: pins.test_decode_matches_torch_sdpa(4, 64, 16, [5, 16, 17, 33])]),
    ("prefill excludes the diagonal", oatt, "paged_attention_prefill_chunk", _prefill_strict_causal,
     [lambda: pins.test_prefill_without_context_is_causal_sdpa()]),
    ("prefill ignores cached context", oatt, "paged_attention_prefill_chunk", _prefill_ignores_context,
     [lambda: pins.test_prefill_chunk_split_and_last_row_match_decode()]),
    ("free list is FIFO", obm, "BlockManager", _FifoBM,
     [lambda: pins.test_allocator_matches_hand_trace()]),
    ("append takes a block one token early", obm, "BlockManager", _EarlyAppendBM,
     [lambda: pins.test_append_takes_block_only_at_boundary()]),
    ("free pushes blocks in reverse order", obm, "BlockManager", _ReverseFreeBM,
     [lambda: pins.test_allocator_matches_hand_trace()]),
    ("fork shares a partial block", obm, "BlockManager", _CeilForkBM,
     [lambda: pins.test_shared_prefix_stored_once_and_refcounted()]),
    ("free ignores refcounts", obm, "BlockManager", _NoRefcountBM,
     [lambda: pins.test_shared_prefix_stored_once_and_refcounted()]),
    ("blocks_needed floors", sizes, "blocks_needed", _floor_blocks,
     [lambda: pins.test_blocks_needed_is_smallest_cover(16)]),
    ("kv bytes drop the K+V factor", sizes, "kv_bytes_per_token", _kv_no_two,
     [lambda: pins.test_kv_bytes_per_token_matches_page()]),
]


@pytest.mark.parametrize("name,module,attr,mutant,checks", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(monkeypatch, name, module, attr, mutant, checks):
    monkeypatch.setattr(module, attr, mutant)
    if module is sizes and attr == "blocks_needed":
        monkeypatch.setattr(obm, "blocks_needed", mutant)
    for check in checks:
        with pytest.raises(Exception):
            check()
