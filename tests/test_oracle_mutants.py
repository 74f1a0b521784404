"""Plants plausible mistakes in the CPU oracle and checks that a pin catches each one.

Each mutant replaces one oracle function (on the CPU, for the duration of one
test) with a copy carrying a single mistake: a dropped scale, swapped
operands, a wrong block index, an off-by-one causal bound, a FIFO free list,
and so on.  The pins in ``test_oracle_pins`` must fail on every mutant.
"""
import numpy as np
import pytest

import test_oracle_pins as pins
import test_oracle_serving_pins as spins
import test_prefix_cache as ppins
from oracle import attention as oatt
from oracle import block_manager as obm
from oracle import prefix_cache as opc
from oracle import scheduler as osch
from oracle import sizes
from oracle import swap as oswap

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


# ---- step driver ([CB-PA] §2.2, §4.3, §5.3, §5.4)
_Sched = osch.Scheduler


class _DecodesUseBudget(_Sched):
    def _schedule_prefills(self, budget):
        return super()._schedule_prefills(budget - len(self.last_decode))


class _PrefillBeforeDecode(_Sched):
    def step(self):
        info = dict(step=self.steps, num_admitted=0, num_preempted=0, num_finished=0)
        self._free_finished(info)
        need = self._preempt(info)
        self._admit(info, need)
        self.last_prefill, self.last_decode = [], []
        pre_slots = self._schedule_prefills(self.max_num_tokens)
        dec_slots = self._schedule_decodes()
        info.update(num_prefill=len(self.last_prefill), num_decode=len(self.last_decode),
                    num_tokens=len(pre_slots) + len(dec_slots), prefill=list(self.last_prefill),
                    decode=list(self.last_decode), slot_mapping=pre_slots + dec_slots)
        return info


class _AdmitPastMaxSeqs(_Sched):
    def _admit(self, info, need):
        self.max_num_seqs += 1
        try:
            super()._admit(info, need)
        finally:
            self.max_num_seqs -= 1


class _WatermarkOffByOne(_Sched):
    def _admit(self, info, need):
        super()._admit(info, need + 1)


class _WatermarkIgnoresDecodes(_Sched):
    def _admit(self, info, need):
        super()._admit(info, 0)


class _PreemptOldest(_Sched):
    def _preempt(self, info):
        self.running.reverse()
        try:
            return super()._preempt(info)
        finally:
            self.running.reverse()


class _PreemptedToBack(_Sched):
    def _preempt(self, info):
        n = len(self.waiting)
        need = super()._preempt(info)
        k = info["num_preempted"]
        if k:
            victims = [self.waiting.popleft() for _ in range(k)]
            self.waiting.extend(reversed(victims))
        assert len(self.waiting) == n + k
        return need


class _RecomputePromptOnly(_Sched):
    def _preempt(self, info):
        need = super()._preempt(info)
        for r in list(self.waiting)[:info["num_preempted"]]:
            self.reqs[r].to_prefill = self.reqs[r].prompt_len
        return need


# ---- swap ([CB-PA] §4.4)
_orig_move = oswap._move


def _free_before_allocate(src, dst, req, src_k, src_v, dst_k, dst_v):
    if req not in src.block_tables:
        return obm.NOT_FOUND
    table, n = list(src.block_tables[req]), src.seq_lens[req]
    src.free(req)
    st = dst.allocate(req, n)
    if st == obm.OK and src_k is not None:
        for s_, d in zip(table, dst.block_tables[req]):
            dst_k[d] = src_k[s_]
            dst_v[d] = src_v[s_]
    return st


def _whole_blocks_length(src, dst, req, src_k, src_v, dst_k, dst_v):
    st = _orig_move(src, dst, req, src_k, src_v, dst_k, dst_v)
    if st == obm.OK:
        dst.seq_lens[req] = len(dst.block_tables[req]) * dst.block_size
    return st


def _copies_reversed(src, dst, req, src_k, src_v, dst_k, dst_v):
    if req not in src.block_tables:
        return obm.NOT_FOUND
    if req in dst.block_tables:
        return obm.EXISTS
    st = dst.allocate(req, src.seq_lens[req])
    if st != obm.OK:
        return st
    if src_k is not None:
        for s_, d in zip(src.block_tables[req], reversed(dst.block_tables[req])):
            dst_k[d] = src_k[s_]
            dst_v[d] = src_v[s_]
    return src.free(req)


def _k_only(src, dst, req, src_k, src_v, dst_k, dst_v):
    if req not in src.block_tables:
        return obm.NOT_FOUND
    if req in dst.block_tables:
        return obm.EXISTS
    st = dst.allocate(req, src.seq_lens[req])
    if st != obm.OK:
        return st
    if src_k is not None:
        for s_, d in zip(src.block_tables[req], dst.block_tables[req]):
            dst_k[d] = src_k[s_]
    return src.free(req)


# ---- prefix cache ([CB-PA] §4.1, §4.2)
_PC = opc.PrefixCachingBlockManager


class _EvictMru(_PC):
    def _take(self):
        if self.free_blocks:
            return super()._take()
        b, _ = self.lru.popitem(last=True)
        del self.cache[self.block_node[b]]
        self.block_node[b] = -1
        self.evictions += 1
        self.refcount[b] += 1
        return b


class _ParkInTableOrder(_PC):
    def _release(self, table):
        zero = []
        for b in table:
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                zero.append(b)
        for b in zero:
            if self.block_node[b] < 0:
                self.free_blocks.append(b)
            else:
                self.lru[b] = None


class _HashBlockAlone(_PC):
    def _node(self, parent, block_tokens, create):
        return super()._node(-1, block_tokens, create)


class _RegisterPartialBlock(_PC):
    def allocate_cached(self, req, tokens):
        st, cached = super().allocate_cached(req, tokens)
        n, bs = len(tokens), self.block_size
        if st == obm.OK and n % bs:
            parent = -1
            for i in range(n // bs):
                parent = self._node(parent, [int(t) for t in tokens[i * bs:(i + 1) * bs]], create=True)
            node = self._node(parent, [int(t) for t in tokens[(n // bs) * bs:]], create=True)
            b = self.block_tables[req][-1]
            if node not in self.cache:
                self.cache[node] = b
                self.block_node[b] = node
        return st, cached


class _NoPrune(_PC):
    def _prune(self, node):
        return None


class _BeginTakesAll(_PC):
    def _lookup(self, tokens, max_blocks):
        return super()._lookup(tokens, len(tokens) // self.block_size)


class _AppendsDoNotRegister(_PC):
    def append_token(self, req):
        return obm.BlockManager.append_token(self, req)


class _PrefixIgnored(_Sched):
    def add_request(self, req, prompt_len, max_new, tokens=None):
        return super().add_request(req, prompt_len, max_new, None)


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
    ("scheduler counts decodes against the prefill budget", osch, "Scheduler", _DecodesUseBudget,
     [lambda: spins.run_oracle_scheduler_trace(spins._case("timeline"))]),
    ("scheduler gives prefills their blocks before decodes", osch, "Scheduler", _PrefillBeforeDecode,
     [lambda: spins.run_oracle_scheduler_trace(spins._case("timeline"))]),
    ("scheduler admits past max_num_seqs", osch, "Scheduler", _AdmitPastMaxSeqs,
     [lambda: spins.run_oracle_scheduler_trace(spins._case("timeline"))]),
    ("watermark needs one block more", osch, "Scheduler", _WatermarkOffByOne,
     [lambda: spins.run_oracle_scheduler_trace(spins._case("watermark_boundary_admits"))]),
    ("watermark ignores the decodes' blocks", osch, "Scheduler", _WatermarkIgnoresDecodes,
     [lambda: spins.run_oracle_scheduler_trace(spins._case("watermark_counts_decode_needs"))]),
    ("preemption takes the oldest request", osch, "Scheduler", _PreemptOldest,
     [lambda: spins.run_oracle_scheduler_trace(spins._case("preemption"))]),
    ("preempted request goes to the back of the queue", osch, "Scheduler", _PreemptedToBack,
     [lambda: spins.run_oracle_scheduler_trace(spins._case("preemption"))]),
    ("preempted request recomputes only its prompt", osch, "Scheduler", _RecomputePromptOnly,
     [lambda: spins.run_oracle_scheduler_trace(spins._case("preemption"))]),
    ("swap frees the source before allocating", oswap, "_move", _free_before_allocate,
     [lambda: spins.run_oracle_swap_trace()]),
    ("swap gives the destination whole blocks of tokens", oswap, "_move", _whole_blocks_length,
     [lambda: spins.run_oracle_swap_trace()]),
    ("swap copies blocks in reverse order", oswap, "_move", _copies_reversed,
     [lambda: spins.run_oracle_swap_trace()]),
    ("swap leaves V behind", oswap, "_move", _k_only,
     [lambda: spins.run_oracle_swap_trace()]),
    ("prefix cache evicts the most recent block", opc, "PrefixCachingBlockManager", _EvictMru,
     [lambda: ppins.test_oracle_follows_hand_trace()]),
    ("prefix cache parks blocks in table order", opc, "PrefixCachingBlockManager", _ParkInTableOrder,
     [lambda: ppins.test_oracle_follows_hand_trace()]),
    ("prefix cache hashes a block without its prefix", opc, "PrefixCachingBlockManager", _HashBlockAlone,
     [lambda: ppins.test_shared_system_prompt_is_stored_once()]),
    ("prefix cache registers the partial last block", opc, "PrefixCachingBlockManager", _RegisterPartialBlock,
     [lambda: ppins.test_oracle_follows_hand_trace()]),
    ("prefix trie is never pruned", opc, "PrefixCachingBlockManager", _NoPrune,
     [lambda: ppins.test_oracle_follows_tracked_hand_trace()]),
    ("begin_cached reuses every full block", opc, "PrefixCachingBlockManager", _BeginTakesAll,
     [lambda: ppins.test_oracle_follows_tracked_hand_trace()]),
    ("filled blocks are not registered", opc, "PrefixCachingBlockManager", _AppendsDoNotRegister,
     [lambda: ppins.test_oracle_follows_tracked_hand_trace()]),
    ("scheduler ignores the prompt's token ids", osch, "Scheduler", _PrefixIgnored,
     [lambda: _shared_prompt_pin()]),
]


def _shared_prompt_pin():
    """Oracle-only copy of the shared-prompt check: the second and third requests start at 32 cached tokens."""
    system = list(range(100, 132))
    prompts = [system + [1, 2, 3], system + [4, 5], system + [6] * 9]
    sched = osch.Scheduler(opc.PrefixCachingBlockManager(64, 8), 4, 64)
    ctx = []
    for step in range(3):
        sched.add_request(step, len(prompts[step]), 3, tokens=prompts[step])
        info = sched.step()
        ctx.append([c for _, c, _ in info["prefill"]])
        sched.complete(sampled=[0] * (len(info["decode"]) + sum(
            1 for r, c, n in info["prefill"] if sched.reqs[r].prefilled + n == sched.reqs[r].to_prefill)))
    assert ctx == [[0], [32], [32]] and sched.cached_tokens == 64


@pytest.mark.parametrize("name,module,attr,mutant,checks", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(monkeypatch, name, module, attr, mutant, checks):
    monkeypatch.setattr(module, attr, mutant)
    if module is sizes and attr == "blocks_needed":
        monkeypatch.setattr(obm, "blocks_needed", mutant)
    for check in checks:
        with pytest.raises(Exception):
            check()
