"""Oracle block manager (test infrastructure only).

A plain restatement of ``BlockManager`` from the page "LLM 推理引擎
Continuous Batching 与 PagedAttention", §3.2 (核心数据结构), with the
refcounted shared-prefix blocks of §4.1 (KV Cache 的 Shared Prefix).

Readings taken where the page's sketch is silent or garbled:

* The free list starts as ``0 .. N-1`` (or a given order) and every take is
  a pop from its END; ``allocate`` pops its blocks one after another.
* ``allocate`` is all-or-nothing: ceil(n / block_size) blocks or OOM with no
  change.  Allocating an id that already exists is refused (the page's
  sketch would silently overwrite and leak it).
* ``append_token``: ``current_len`` is the number of tokens stored before
  the append; the new token goes at position ``current_len``; a block is
  popped iff ``current_len % block_size == 0`` (including length 0).  OOM
  leaves the state unchanged.
* ``free`` (the sketch's ``block_blocks`` is a typo for ``block_tables``)
  decrements every block of the table, in table order, and pushes onto the
  free list the ones whose refcount reaches zero.  Freeing an unknown id is
  a no-op, as the sketch's ``if ... in`` makes it.
* ``fork`` shares only whole blocks (§4.1 hashes the token content of whole
  blocks): the first floor(prefix / block_size) blocks of the source, each
  refcount + 1; the child starts with that many full blocks.
* A token's slot is ``table[pos // block_size] * block_size + pos %
  block_size``, the address form of §3.3 (GPU Kernel 中的分页读取).
"""
from __future__ import annotations

from .sizes import blocks_needed

OK = "ok"
INVALID_ARG = "invalid_arg"
OOM = "oom"
NOT_FOUND = "not_found"
EXISTS = "exists"


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks < 0 or block_size <= 0:
            raise ValueError("bad pool")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        if free_order is None:
            self.free_blocks = list(range(self.num_blocks))
        else:
            self.free_blocks = [int(b) for b in free_order]
            if sorted(self.free_blocks) != list(range(self.num_blocks)):
                raise ValueError("free_order must be a permutation of 0..N-1")
        self.block_tables: dict[int, list[int]] = {}
        self.seq_lens: dict[int, int] = {}
        self.refcount = [0] * self.num_blocks
        self.oom_count = 0

    # ---- §3.2 allocate ----------------------------------------------------
    def allocate(self, req: int, num_tokens: int) -> str:
        if num_tokens < 0:
            return INVALID_ARG
        if req in self.block_tables:
            return EXISTS
        n = blocks_needed(num_tokens, self.block_size)
        if self._available() < n:
            self.oom_count += 1
            return OOM
        blocks = [self._take() for _ in range(n)]
        self.block_tables[req] = blocks
        self.seq_lens[req] = num_tokens
        return OK

    # ---- §3.2 append_token ------------------------------------------------
    def append_token(self, req: int):
        """Returns (status, slot of the appended token or None)."""
        if req not in self.block_tables:
            return NOT_FOUND, None
        table = self.block_tables[req]
        cur = self.seq_lens[req]
        if cur % self.block_size == 0:
            if self._available() == 0:
                self.oom_count += 1
                return OOM, None
            table.append(self._take())
        self.seq_lens[req] = cur + 1
        return OK, self.slot(req, cur)

    def append_tokens(self, req: int, n: int):
        """n appends as one all-or-nothing step.  Returns (status, slots)."""
        if n < 0:
            return INVALID_ARG, []
        if req not in self.block_tables:
            return NOT_FOUND, []
        cur = self.seq_lens[req]
        extra = blocks_needed(cur + n, self.block_size) - len(self.block_tables[req])
        if extra > self._available():
            self.oom_count += 1
            return OOM, []
        slots = []
        for _ in range(n):
            st, s = self.append_token(req)
            assert st == OK
            slots.append(s)
        return OK, slots

    # ---- §4.1 shared prefix -----------------------------------------------
    def fork(self, src: int, dst: int, prefix_tokens: int) -> str:
        if src not in self.block_tables:
            return NOT_FOUND
        if dst in self.block_tables:
            return EXISTS
        if prefix_tokens < 0 or prefix_tokens > self.seq_lens[src]:
            return INVALID_ARG
        shared = prefix_tokens // self.block_size
        blocks = list(self.block_tables[src][:shared])
        for b in blocks:
            self.refcount[b] += 1
        self.block_tables[dst] = blocks
        self.seq_lens[dst] = shared * self.block_size
        return OK

    # ---- §3.2 free --------------------------------------------------------
    def free(self, req: int) -> str:
        if req not in self.block_tables:
            return OK
        self._release(self.block_tables[req])
        del self.block_tables[req]
        del self.seq_lens[req]
        return OK

    # ---- free-list primitives (the prefix cache overrides them) -------------
    def _available(self) -> int:
        return len(self.free_blocks)

    def _take(self) -> int:
        b = self.free_blocks.pop()
        self.refcount[b] += 1
        return b

    def _release(self, table) -> None:
        for b in table:
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                self.free_blocks.append(b)

    # ---- queries ----------------------------------------------------------
    def get_block_table(self, req: int):
        if req not in self.block_tables:
            return NOT_FOUND, []
        return OK, list(self.block_tables[req])

    def seq_len(self, req: int):
        if req not in self.seq_lens:
            return NOT_FOUND, None
        return OK, self.seq_lens[req]

    def slot(self, req: int, pos: int) -> int:
        """Slot of logical position ``pos`` (address form of §3.3)."""
        table = self.block_tables[req]
        return table[pos // self.block_size] * self.block_size + pos % self.block_size

    def slots(self, req: int, pos_begin: int, n: int):
        """Slots of positions pos_begin .. pos_begin+n-1 (all below seq_len)."""
        if req not in self.block_tables:
            return NOT_FOUND, []
        if pos_begin < 0 or n < 0 or pos_begin + n > self.seq_lens[req]:
            return INVALID_ARG, []
        return OK, [self.slot(req, p) for p in range(pos_begin, pos_begin + n)]

    def pack(self, reqs, max_blocks: int):
        """Padded block tables [n, max_blocks] (pad -1) and seq_lens [n]."""
        tables, lens = [], []
        for r in reqs:
            if r not in self.block_tables:
                return NOT_FOUND, None, None
            t = self.block_tables[r]
            if len(t) > max_blocks:
                return INVALID_ARG, None, None
            tables.append(list(t) + [-1] * (max_blocks - len(t)))
            lens.append(self.seq_lens[r])
        return OK, tables, lens

    def stats(self) -> dict:
        return {
            "num_blocks": self.num_blocks,
            "num_free": len(self.free_blocks),
            "num_used": sum(1 for c in self.refcount if c > 0),
            "total_refs": sum(self.refcount),
            "num_requests": len(self.block_tables),
            "oom_count": self.oom_count,
            "waste_tokens": sum(len(t) * self.block_size - self.seq_lens[r]
                                for r, t in self.block_tables.items()),
        }
