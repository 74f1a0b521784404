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

§4.2 keeps its table of blocks by content for as long as the blocks live; read
with §4.1's refcounted lifetime, an entry lives as long as its block, so the
trie does not grow with every prefix ever seen:

* when an evicted block's node has no children, the node is dropped, and so,
  walking up, is every ancestor left without a block and without children
  (node numbers are never reused).

The §2.2 loop reuses cached blocks at admission and makes the blocks it fills
cacheable, which needs the request's token ids:

* ``begin_cached(req, tokens)`` starts a request with only the cached blocks
  of the longest cached prefix of ``tokens`` (at most ``(n - 1) // bs`` whole
  blocks, so at least one token is left to compute), taking nothing new;
  ``cached_prefix(tokens)`` answers the same lookup without taking anything;
* a request started by ``begin_cached`` or ``allocate_cached`` is tracked: its
  known token ids (``extend_tokens`` adds the ones it generates) register
  each block its appends fill, under the node of the block before it;
  tracking stops when a filled block's ids are not known, or its content is
  already cached in another block (the request's chain then ends there).
"""
from __future__ import annotations

from collections import OrderedDict

from .block_manager import EXISTS, INVALID_ARG, NOT_FOUND, OK, OOM, BlockManager
from .sizes import blocks_needed


class PrefixCachingBlockManager(BlockManager):
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        super().__init__(num_blocks, block_size, free_order)
        self.trie: dict = {}                 # (parent node, tuple of tokens) -> node
        self.node_key: dict = {}             # node -> its key in the trie
        self.children: dict = {}             # node -> number of child nodes
        self.next_node = 0
        self.cache: dict = {}                # node -> block
        self.tokens: dict = {}               # tracked request -> its known token ids
        self.last_node: dict = {}            # tracked request -> node of its last registered block
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
            node = self.block_node[b]
            del self.cache[node]
            self.block_node[b] = -1
            self.evictions += 1
            self._prune(node)
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
            node = self.next_node
            self.next_node += 1
            self.trie[key] = node
            self.node_key[node] = key
            self.children[node] = 0
            if parent >= 0:
                self.children[parent] += 1
        return self.trie[key]

    def _prune(self, node):
        """Drop `node` and then its ancestors while they hold no block and have no children."""
        while node >= 0 and node not in self.cache and self.children[node] == 0:
            key = self.node_key.pop(node)
            del self.trie[key]
            del self.children[node]
            node = key[0]
            if node >= 0:
                self.children[node] -= 1

    def _lookup(self, tokens, max_blocks):
        """Cached blocks (and their nodes) of the longest cached prefix of whole blocks, at most max_blocks."""
        bs = self.block_size
        hits, nodes, parent = [], [], -1
        for i in range(max_blocks):
            node = self._node(parent, tokens[i * bs:(i + 1) * bs], create=False)
            if node is None or node not in self.cache:
                break
            hits.append(self.cache[node])
            nodes.append(node)
            parent = node
        return hits, nodes

    def _take_hits(self, hits):
        for b in hits:
            self.lru.pop(b, None)
            self.refcount[b] += 1

    # ---- tracked requests: blocks their appends fill become cacheable
    def append_token(self, req):
        st, slot = super().append_token(req)
        if st == OK and req in self.tokens:
            n, bs = self.seq_lens[req], self.block_size
            if n % bs == 0:
                toks = self.tokens[req]
                node = None
                if len(toks) >= n:
                    node = self._node(self.last_node[req], toks[n - bs:n], create=True)
                    if node in self.cache:
                        node = None          # the content lives in another block: the chain ends here
                    else:
                        b = self.block_tables[req][-1]
                        self.cache[node] = b
                        self.block_node[b] = node
                if node is None:
                    del self.tokens[req], self.last_node[req]
                else:
                    self.last_node[req] = node
        return st, slot

    def free(self, req):
        self.tokens.pop(req, None)
        self.last_node.pop(req, None)
        return super().free(req)

    def extend_tokens(self, req, ids):
        if req not in self.block_tables:
            return NOT_FOUND
        if req in self.tokens:
            self.tokens[req] += [int(t) for t in ids]
        return OK

    def cached_prefix(self, tokens):
        """(cached blocks, of which parked) that begin_cached would reuse for tokens."""
        tokens = [int(t) for t in tokens]
        hits, _ = self._lookup(tokens, max(0, (len(tokens) - 1) // self.block_size))
        return len(hits), sum(1 for b in hits if b in self.lru)

    def begin_cached(self, req, tokens):
        """Returns (status, cached_tokens)."""
        tokens = [int(t) for t in tokens]
        if req in self.block_tables:
            return EXISTS, 0
        hits, nodes = self._lookup(tokens, max(0, (len(tokens) - 1) // self.block_size))
        self._take_hits(hits)
        self.block_tables[req] = list(hits)
        self.seq_lens[req] = len(hits) * self.block_size
        self.tokens[req] = tokens
        self.last_node[req] = nodes[-1] if nodes else -1
        self.hit_blocks += len(hits)
        return OK, len(hits) * self.block_size

    def allocate_cached(self, req, tokens):
        """Returns (status, cached_tokens)."""
        tokens = [int(t) for t in tokens]
        if req in self.block_tables:
            return EXISTS, 0
        bs = self.block_size
        n = len(tokens)
        nfull = n // bs
        hits, _ = self._lookup(tokens, nfull)
        need = blocks_needed(n, bs) - len(hits)
        parked_hits = sum(1 for b in hits if b in self.lru)
        if need > self._available() - parked_hits:
            self.oom_count += 1
            return OOM, 0
        self._take_hits(hits)
        table = list(hits) + [self._take() for _ in range(need)]
        parent, chain = -1, True
        for i in range(nfull):
            node = self._node(parent, tokens[i * bs:(i + 1) * bs], create=True)
            if i >= len(hits) and node not in self.cache:
                self.cache[node] = table[i]
                self.block_node[table[i]] = node
            chain = chain and self.cache.get(node) == table[i]
            parent = node
        self.block_tables[req] = table
        self.seq_lens[req] = n
        self.hit_blocks += len(hits)
        if chain:                        # every full block is its own node's block: keep registering
            self.tokens[req] = tokens
            self.last_node[req] = parent
        return OK, len(hits) * bs

    def cache_stats(self) -> dict:
        return {"cached_blocks": len(self.cache), "evictable_blocks": len(self.lru),
                "hit_blocks": self.hit_blocks, "evictions": self.evictions, "prefix_nodes": len(self.trie)}


__all__ = ["PrefixCachingBlockManager", "OK", "OOM", "EXISTS", "INVALID_ARG"]
