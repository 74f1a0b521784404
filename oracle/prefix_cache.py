"""Oracle automatic prefix caching (test infrastructure only).

Page "LLM 推理引擎 Continuous Batching 与 PagedAttention", §4.1 (KV Cache 的
Shared Prefix: the token content of every block is hashed, identical blocks
are stored once, refcounts govern their lifetime) and §4.2 (Automatic Prefix
Caching: ``PrefixCachingBlockManager`` keeps a table from token content to
physical blocks plus an LRU ``eviction_queue``).  The page's sketch is
garbled (``new_blocks`` is never defined); the plainest complete reading,
taken here:

* A full block's content is its whole token prefix: block i of a request is
  identified by the pair (identity of block i-1, tokens of block i), interned
  into a prefix trie whose node numbers are never reused.  Two blocks match
  only if every token up to their end matches, which is what reusing KV needs.
* ``allocate_cached(req, tokens)`` walks the request's full blocks from the
  first one and reuses the cached block of each prefix node until the first
  miss; the remaining blocks are taken fresh and the new full ones are
  registered (a node already cached elsewhere keeps its block).  The partial
  last block is private.  All-or-nothing, like ``allocate``.
* A registered block whose refcount reaches zero is parked at the back of the
  LRU (``OrderedDict``) instead of the free list; the blocks a request frees
  are parked last block first, so a prefix stays at least as recent as its
  extensions.  Unregistered blocks go to the free list in table order.
* A take pops the free list; when it is empty it evicts the LRU's front
  block, whose cache entry is dropped.
"""
from __future__ import annotations

from collections import OrderedDict

from .block_manager import EXISTS, INVALID_ARG, OK, OOM, BlockManager
from .sizes import blocks_needed


class PrefixCachingBlockManager(BlockManager):
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        super().__init__(num_blocks, block_size, free_order)
        self.trie: dict = {}                 # (parent node, tuple of tokens) -> node
        self.cache: dict = {}                # node -> block
        self.block_node = [-1] * self.num_blocks
        self.lru: OrderedDict = OrderedDict()   # parked blocks, least recently parked first
        self.hit_blocks = 0
        self.evictions = 0

    def _available(self) -> int:
        return len(self.free_blocks) + len(self.lru)

    def _take(self) -> int:
        if self.free_blocks:
            b = self.free_blocks.pop()
        else:
            b, _ = self.lru.popitem(last=False)
            del self.cache[self.block_node[b]]
            self.block_node[b] = -1
            self.evictions += 1
        self.refcount[b] += 1
        return b

    def _release(self, table) -> None:
        zero = []
        for b in table:
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                zero.append(b)
        for b in zero:
            if self.block_node[b] < 0:
                self.free_blocks.append(b)
        for b in reversed(zero):
            if self.block_node[b] >= 0:
                self.lru[b] = None

    def _node(self, parent, block_tokens, create):
        key = (parent, tuple(block_tokens))
        if key not in self.trie:
            if not create:
                return None
            self.trie[key] = len(self.trie)
        return self.trie[key]

    def allocate_cached(self, req, tokens):
        """Returns (status, cached_tokens)."""
        tokens = [int(t) for t in tokens]
        if req in self.block_tables:
            return EXISTS, 0
        bs = self.block_size
        n = len(tokens)
        nfull = n // bs
        hits, parent = [], -1
        for i in range(nfull):
            node = self._node(parent, tokens[i * bs:(i + 1) * bs], create=False)
            if node is None or node not in self.cache:
                break
            hits.append(self.cache[node])
            parent = node
        need = blocks_needed(n, bs) - len(hits)
        parked_hits = sum(1 for b in hits if b in self.lru)
        if need > self._available() - parked_hits:
            self.oom_count += 1
            return OOM, 0
        table = []
        for b in hits:
            self.lru.pop(b, None)
            self.refcount[b] += 1
            table.append(b)
        table += [self._take() for _ in range(need)]
        parent = -1
        for i in range(nfull):
            node = self._node(parent, tokens[i * bs:(i + 1) * bs], create=True)
            if i >= len(hits) and node not in self.cache:
                self.cache[node] = table[i]
                self.block_node[table[i]] = node
            parent = node
        self.block_tables[req] = table
        self.seq_lens[req] = n
        self.hit_blocks += len(hits)
        return OK, len(hits) * bs

    def cache_stats(self) -> dict:
        return {"cached_blocks": len(self.cache), "evictable_blocks": len(self.lru),
                "hit_blocks": self.hit_blocks, "evictions": self.evictions, "prefix_nodes": len(self.trie)}


__all__ = ["PrefixCachingBlockManager", "OK", "OOM", "EXISTS", "INVALID_ARG"]
