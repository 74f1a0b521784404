"""Oracle continuous-batching scheduler (test infrastructure only).

Page "LLM 推理引擎 Continuous Batching 与 PagedAttention": §2.2
(``ContinuousBatchingScheduler.step``: free finished requests, admit waiting
ones while ``_can_allocate``, build a batch with prefill first under
``max_num_tokens`` and one token per decode), §4.3 (chunked prefill), §5.3
(admission keeps a block watermark), §5.4 (preemption: the newest running
request goes back to the front of the waiting queue and its blocks are freed;
"recompute" redoes its tokens).  Chapter "动态批处理算法" §4.4 gives the same
loop.  Readings where the sketch leaves a step open:

* preemption happens before admission, only as far as the running decodes
  need new blocks that are not available (the sketch preempts while no block is
  free); a preempted request recomputes its prompt plus the tokens it
  generated;
* ``_can_allocate`` admits a request when the blocks of its whole prefill, the
  decodes' needs and the watermark are available;
* decodes get their token before prefills get chunks (so admission can never
  starve them of blocks); prefill chunks go in running order, at most the
  remaining token budget each (whole prompts only without chunking); a chunk
  that cannot get its blocks waits; the step's slot mapping lists the prefill
  rows, then the decode rows;
* finishing: a request emits a token when its prefill completes and at each
  decode; at ``max_new_tokens`` it finishes and is freed at the next step.

§5.4 also names a second preemption strategy, swapping the victim's KV to CPU
memory (§4.4's ``SwappingManager``).  With a CPU block manager given
(``swap_cpu``), a victim is moved to the CPU pool instead of being freed
(``oracle.swap``: destination allocated first, block i to block i, source
freed); when the CPU pool cannot take it, it is recomputed as above.  Readings
where the page leaves the strategy open:

* a swapped request keeps its progress (prefilled and generated tokens) and
  waits in a swapped queue, the most recently preempted at the front;
* swapped requests come back before any waiting request is admitted, in queue
  order, while seats are free and the blocks of their table (plus one if their
  next decode opens a block), the decodes' needs and the watermark are
  available; no waiting request is admitted while a request is still swapped;
* the step reports its block moves (GPU to CPU for the swap-outs, then CPU to
  GPU for the swap-ins), which the caller performs before the step's kernels.

§4.2's automatic prefix caching inside the §2.2 loop, for requests whose token
ids are given (``add_request(..., tokens=)``):

* admission looks up the longest cached prefix of the ids it knows (prompt,
  then generated tokens reported by ``complete(sampled=)``), needs new blocks
  only for the rest (``blocks_needed(to_prefill) - hits``, with parked hits
  no longer counted as available), and starts the request there
  (``begin_cached``): the cached tokens are not prefilled again;
* the blocks its prefill chunks and decodes fill are registered as they fill
  (the allocator's tracked requests), and its generated ids are reported to
  the allocator as they are emitted, so decoded text becomes cacheable too; a
  request preempted by recomputation finds its own blocks in the cache when it
  comes back;
* ``complete(sampled)`` takes one id per emitted token, in emission order:
  requests whose prefill completed (prefill order), then the decodes.
"""
from __future__ import annotations

from collections import deque

from .block_manager import OK, OOM
from .sizes import blocks_needed
from .swap import SwappingManager

WAITING, RUNNING, FINISHED, SWAPPED = 0, 1, 2, 3


class _Req:
    def __init__(self, prompt_len, max_new, tokens=None):
        self.tokens = None if tokens is None else [int(t) for t in tokens]
        self.prompt_len = prompt_len
        self.max_new = max_new
        self.to_prefill = prompt_len
        self.prefilled = 0
        self.generated = 0
        self.state = WAITING
        self.first_token_step = -1
        self.finish_step = -1
        self.preemptions = 0


class Scheduler:
    def __init__(self, bm, max_num_seqs, max_num_tokens, chunked_prefill=True, watermark_blocks=0,
                 swap_cpu=None):
        self.bm = bm
        self.swapper = SwappingManager(bm, swap_cpu) if swap_cpu is not None else None
        self.swapped: deque = deque()
        self.swap_out_pairs: list = []
        self.swap_in_pairs: list = []
        self.max_num_seqs = max_num_seqs
        self.max_num_tokens = max_num_tokens
        self.chunked = bool(chunked_prefill)
        self.watermark = watermark_blocks
        self.reqs: dict = {}
        self.waiting: deque = deque()
        self.running: list = []
        self.steps = 0
        self.cached_tokens = 0
        self.last_prefill: list = []
        self.last_decode: list = []

    def add_request(self, req, prompt_len, max_new, tokens=None):
        self.reqs[req] = _Req(prompt_len, max_new, tokens)
        self.waiting.append(req)
        return OK

    def _decoding(self, q):
        return q.state == RUNNING and q.prefilled == q.to_prefill and q.generated < q.max_new

    def _need(self):
        bs = self.bm.block_size
        return sum(1 for r in self.running
                   if self._decoding(self.reqs[r]) and self.bm.seq_lens[r] % bs == 0)

    def step(self):
        info = dict(step=self.steps, num_admitted=0, num_preempted=0, num_finished=0)
        self.swap_out_pairs, self.swap_in_pairs = [], []
        self._free_finished(info)
        need = self._preempt(info)
        need = self._swap_in(info, need)
        if not self.swapped:
            self._admit(info, need)
        self.last_prefill, self.last_decode = [], []
        dec_slots = self._schedule_decodes()
        pre_slots = self._schedule_prefills(self.max_num_tokens)
        info.update(num_prefill=len(self.last_prefill), num_decode=len(self.last_decode),
                    num_tokens=len(pre_slots) + len(dec_slots),
                    prefill=list(self.last_prefill), decode=list(self.last_decode),
                    slot_mapping=pre_slots + dec_slots, swap_out=list(self.swap_out_pairs),
                    swap_in=list(self.swap_in_pairs))
        return info

    # §2.2 step 1: requests that emitted their last token give their blocks back
    def _free_finished(self, info):
        keep = []
        for r in self.running:
            if self.reqs[r].state == FINISHED:
                self.bm.free(r)
                info["num_finished"] += 1
            else:
                keep.append(r)
        self.running = keep

    # §5.4: preempt the newest running request while the decodes lack blocks; strategy 2 (swap its KV
    # to the CPU pool) when a CPU pool is given and has room, else strategy 1 (recompute)
    def _preempt(self, info):
        need = self._need()
        while need > self.bm._available() and self.running:
            v = self.running.pop()
            q = self.reqs[v]
            q.preemptions += 1
            info["num_preempted"] += 1
            if self.swapper is not None:
                gpu_table = list(self.bm.block_tables[v])
                if self.swapper.swap_out(v) == OK:
                    self.swap_out_pairs += list(zip(gpu_table, self.swapper.cpu.block_tables[v]))
                    q.state = SWAPPED
                    self.swapped.appendleft(v)
                    need = self._need()
                    continue
            self.bm.free(v)
            q.to_prefill = q.prompt_len + q.generated
            q.prefilled = 0
            q.state = WAITING
            self.waiting.appendleft(v)
            need = self._need()
        return need

    # swapped requests come back first (§4.4 swap_in), while seats and blocks last
    def _swap_in(self, info, need):
        bs = self.bm.block_size
        while self.swapped and len(self.running) < self.max_num_seqs:
            r = self.swapped[0]
            q = self.reqs[r]
            cpu_table = list(self.swapper.cpu.block_tables[r])
            opens = 1 if (q.prefilled == q.to_prefill and q.generated < q.max_new
                          and self.swapper.cpu.seq_lens[r] % bs == 0) else 0
            if self.bm._available() - need - self.watermark < len(cpu_table) + opens:
                break
            self.swapped.popleft()
            assert self.swapper.swap_in(r) == OK
            self.swap_in_pairs += list(zip(cpu_table, self.bm.block_tables[r]))
            q.state = RUNNING
            self.running.append(r)
            need += opens
        return need

    # §2.2 step 2 with §5.3's watermark: admit in arrival order while seats and blocks last
    def _admit(self, info, need):
        bs = self.bm.block_size
        while len(self.running) < self.max_num_seqs and self.waiting:
            r = self.waiting[0]
            q = self.reqs[r]
            hits, parked = 0, 0
            if q.tokens is not None:
                known = q.tokens[:q.to_prefill]
                hits, parked = self.bm.cached_prefix(known)
            if self.bm._available() - parked - need - self.watermark < blocks_needed(q.to_prefill, bs) - hits:
                break
            self.waiting.popleft()
            q.prefilled = 0
            if q.tokens is not None:
                st, q.prefilled = self.bm.begin_cached(r, known)
                self.cached_tokens += q.prefilled
            else:
                st = self.bm.allocate(r, 0)
            assert st == OK
            q.state = RUNNING
            self.running.append(r)
            info["num_admitted"] += 1

    # §2.2 step 3, decode half: one token for every fully prefilled request
    def _schedule_decodes(self):
        slots = []
        for r in self.running:
            if not self._decoding(self.reqs[r]):
                continue
            st, slot = self.bm.append_token(r)
            assert st == OK
            slots.append(slot)
            self.last_decode.append((r, self.bm.seq_lens[r]))
        return slots

    # §2.2 step 3, prefill half, with §4.3's chunks: prefill tokens share the step's budget
    def _schedule_prefills(self, budget):
        slots = []
        for r in self.running:
            q = self.reqs[r]
            if q.state != RUNNING or q.prefilled >= q.to_prefill:
                continue
            remaining = q.to_prefill - q.prefilled
            chunk = min(remaining, budget) if self.chunked else (remaining if remaining <= budget else 0)
            if chunk <= 0:
                continue
            st, s = self.bm.append_tokens(r, chunk)
            if st == OOM:
                continue
            slots += s
            self.last_prefill.append((r, q.prefilled, chunk))
            budget -= chunk
        return slots

    def complete(self, sampled=None):
        now = self.steps
        emitting = [r for r, ctx, chunk in self.last_prefill if self.reqs[r].prefilled + chunk == self.reqs[r].to_prefill]
        emitting += [r for r, _ in self.last_decode]
        if sampled is not None:
            assert len(sampled) == len(emitting)
            for r, t in zip(emitting, sampled):
                q = self.reqs[r]
                if q.tokens is not None:
                    q.tokens.append(int(t))
                    self.bm.extend_tokens(r, [int(t)])

        def emit(q):
            q.generated += 1
            if q.first_token_step < 0:
                q.first_token_step = now
            if q.generated >= q.max_new:
                q.state = FINISHED
                q.finish_step = now

        for r, ctx, chunk in self.last_prefill:
            q = self.reqs[r]
            q.prefilled += chunk
            if q.prefilled == q.to_prefill:
                emit(q)
        for r, _ in self.last_decode:
            emit(self.reqs[r])
        self.steps += 1
