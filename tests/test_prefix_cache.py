"""Automatic prefix caching: the oracle against a hand-traced golden log and the page's
shared system-prompt example, then the C++ allocator against the oracle, bit for bit, on
random logs of prefix-sharing requests (no GPU)."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import paged_kv_cache_411_b200 as pk
from conftest import golden
from oracle import block_manager as obm
from oracle import prefix_cache as opc
from oracle.prefix_cache import PrefixCachingBlockManager

_NAMES = {pk.PA_OK: obm.OK, pk.PA_ERR_OOM: obm.OOM, pk.PA_ERR_NOT_FOUND: obm.NOT_FOUND,
          pk.PA_ERR_EXISTS: obm.EXISTS, pk.PA_ERR_INVALID_ARG: obm.INVALID_ARG}


def test_oracle_follows_hand_trace():
    g = golden("prefix_cache_trace.json")
    bm = opc.PrefixCachingBlockManager(g["num_blocks"], g["block_size"])
    for op in g["ops"]:
        kind = op[0]
        if kind == "allocate_cached":
            st_, cached = bm.allocate_cached(op[1], op[2])
            assert (st_, cached) == (op[3], op[4]), op
            if op[5] is not None:
                assert bm.block_tables[op[1]] == op[5], op
        elif kind == "allocate":
            assert bm.allocate(op[1], op[2]) == op[3]
            assert bm.block_tables[op[1]] == op[4]
        elif kind == "free":
            assert bm.free(op[1]) == op[2]
        elif kind == "check_lru":
            assert list(bm.lru) == op[1], op
        elif kind == "check_free":
            assert bm.free_blocks == op[1], op
        elif kind == "check_refcount":
            assert bm.refcount == op[1], op


def _cached_prefixes(bm):
    """Each cached block's whole token prefix (ids joined by commas) -> block."""
    out = {}
    for node, b in bm.cache.items():
        toks, n = [], node
        while n >= 0:
            parent, blk = bm.node_key[n]
            toks = list(blk) + toks
            n = parent
        out[",".join(map(str, toks))] = b
    return out


def run_tracked_trace(make):
    """Replays the tracked-request golden through an allocator made by make(num_blocks, block_size); the
    prefix-to-block checks need the oracle's trie, the rest runs on either side."""
    g = golden("prefix_cache_tracked_trace.json")
    bm = make(g["num_blocks"], g["block_size"])
    ids = {"A": 1, "B": 2, "C": 3, "D": 4}
    oracle = isinstance(bm, opc.PrefixCachingBlockManager)
    names = (lambda x: x) if oracle else (lambda x: _NAMES[x])
    for op in g["ops"]:
        r = ids[op["req"]]
        kind = op["op"]
        if kind == "begin_cached":
            st, cached = bm.begin_cached(r, op["tokens"])
            assert (names(st), cached) == (op["status"], op["cached"]), op["why"]
        elif kind == "append_tokens":
            st, slots = bm.append_tokens(r, op["n"])
            assert names(st) == op["status"] and list(slots) == op["slots"], op["why"]
        elif kind == "append_token":
            st, slot = bm.append_token(r)
            assert names(st) == op["status"] and slot == op["slot"], op["why"]
        elif kind == "extend_tokens":
            assert names(bm.extend_tokens(r, op["ids"])) == op["status"]
        elif kind == "allocate":
            assert names(bm.allocate(r, op["tokens"])) == op["status"], op["why"]
        else:
            assert names(bm.free(r)) == op["status"]
        tab = (lambda q: bm.block_tables[q]) if oracle else (lambda q: bm.get_block_table(q)[1].tolist())
        if "table" in op:
            assert tab(r) == op["table"], op["why"]
        if "lru" in op:
            assert (list(bm.lru) if oracle else bm.evictable_list().tolist()) == op["lru"], op["why"]
        if "free" in op:
            assert (bm.free_blocks if oracle else bm.free_list().tolist()) == op["free"], op["why"]
        if "prefix_nodes" in op:
            assert (len(bm.trie) if oracle else bm.cache_stats()["prefix_nodes"]) == op["prefix_nodes"], op["why"]
        if "cached_prefixes" in op:
            if oracle:
                assert _cached_prefixes(bm) == op["cached_prefixes"], op["why"]
            else:
                assert bm.cache_stats()["cached_blocks"] == len(op["cached_prefixes"]), op["why"]


def test_oracle_follows_tracked_hand_trace():
    run_tracked_trace(opc.PrefixCachingBlockManager)


def test_cpp_follows_tracked_hand_trace():
    run_tracked_trace(pk.BlockAllocator)


def test_shared_system_prompt_is_stored_once():
    """The page's figure: a 3-block system prompt shared by two requests with 2 private blocks
    each occupies 7 blocks; the second request finds all 3 prompt blocks in the cache."""
    bs = 16
    rng = np.random.default_rng(0)
    system = rng.integers(0, 32000, 3 * bs).tolist()
    q1 = rng.integers(0, 32000, 20).tolist()
    q2 = rng.integers(0, 32000, 25).tolist()
    bm = opc.PrefixCachingBlockManager(32, bs)
    assert bm.allocate_cached(1, system + q1) == (obm.OK, 0)
    assert bm.allocate_cached(2, system + q2) == (obm.OK, 3 * bs)
    assert bm.block_tables[1][:3] == bm.block_tables[2][:3]
    assert not set(bm.block_tables[1][3:]) & set(bm.block_tables[2][3:])
    assert bm.stats()["num_used"] == 7 and bm.cache_stats()["hit_blocks"] == 3
    assert all(bm.refcount[b] == 2 for b in bm.block_tables[1][:3])
    # a different prompt shares nothing; the same prompt after both left is still cached
    bm.free(1)
    bm.free(2)
    assert bm.allocate_cached(3, rng.integers(0, 32000, 48).tolist()) == (obm.OK, 0)
    assert bm.allocate_cached(4, system + [7]) == (obm.OK, 3 * bs)
    # identical block content after a different prefix is a different block
    other = rng.integers(0, 32000, bs).tolist()
    assert bm.allocate_cached(5, other + system[bs:2 * bs]) == (obm.OK, 0)
    # and a block seen only after a prefix is no hit at the start of a prompt
    assert bm.allocate_cached(6, system[bs:2 * bs] + [1]) == (obm.OK, 0)


def _trie_is_pruned(om):
    """Every prefix node holds a block or has a child (nothing dead is kept)."""
    for node in om.node_key:
        assert node in om.cache or om.children[node] > 0, node


def _toks(fam, vocab, b, n):
    base = [fam * 1000 + i for i in range(n)]
    return base[: n - (b % 3)] + [(vocab * b + i) % 7 for i in range(b % 3)]


def _replay(N, bs, log, vocab):
    ca = pk.BlockAllocator(N, bs)
    om = PrefixCachingBlockManager(N, bs)
    for kind, a, b, fam, n in log:
        if kind == 0:
            toks = _toks(fam, vocab, b, n)
            st, cached = ca.allocate_cached(a, toks)
            ost, ocached = om.allocate_cached(a, toks)
            assert (_NAMES[st], cached) == (ost, ocached)
        elif kind == 1:
            assert _NAMES[ca.allocate(a, n)] == om.allocate(a, n)
        elif kind == 2:
            st, slot = ca.append_token(a)
            ost, oslot = om.append_token(a)
            assert _NAMES[st] == ost and slot == oslot
        elif kind == 3:
            p = min(n, om.seq_lens.get(a, 0))
            assert _NAMES[ca.fork(a, b, p)] == om.fork(a, b, p)
        elif kind == 4:
            assert _NAMES[ca.free(a)] == om.free(a)
        elif kind == 5:
            toks = _toks(fam, vocab, b, n)
            assert ca.cached_prefix(toks) == om.cached_prefix(toks)
            st, cached = ca.begin_cached(a, toks)
            ost, ocached = om.begin_cached(a, toks)
            assert (_NAMES[st], cached) == (ost, ocached)
        elif kind == 6:
            ids = [fam * 1000 + om.seq_lens.get(a, 0) + i for i in range(b + 1)]
            assert _NAMES[ca.extend_tokens(a, ids)] == om.extend_tokens(a, ids)
        else:
            k = b % 4 + 1
            st, slots = ca.append_tokens(a, k)
            ost, oslots = om.append_tokens(a, k)
            assert _NAMES[st] == ost and list(slots) == list(oslots)
        assert ca.free_list().tolist() == om.free_blocks
        assert ca.evictable_list().tolist() == list(om.lru)
        assert ca.cache_stats()["prefix_nodes"] == len(om.trie)
        _trie_is_pruned(om)
    for r in range(6):
        st, t = ca.get_block_table(r)
        assert t.tolist() == om.get_block_table(r)[1]
    assert [ca.refcount(b)[1] for b in range(N)] == om.refcount
    assert ca.cache_stats() == om.cache_stats()
    s1, s2 = ca.stats(), om.stats()
    assert all(s1[k] == s2[k] for k in s2)


ops = st.lists(st.tuples(st.integers(0, 7), st.integers(0, 5), st.integers(0, 5), st.integers(0, 2),
                         st.integers(0, 40)), min_size=1, max_size=120)


@settings(max_examples=300, deadline=None)
@given(st.integers(1, 24), st.sampled_from([1, 2, 4, 8]), st.integers(1, 5), ops)
def test_cpp_prefix_cache_matches_oracle(N, bs, vocab, log):
    _replay(N, bs, log, vocab)


def test_prefix_cache_errors():
    ca = pk.BlockAllocator(4, 2)
    assert ca.allocate_cached(1, [1, 2, 3]) == (pk.PA_OK, 0)
    assert ca.allocate_cached(1, [1, 2]) == (pk.PA_ERR_EXISTS, 0)
    assert ca.allocate_cached(2, [1, 2, 9, 9, 9, 9, 9]) == (pk.PA_ERR_OOM, 0)
    assert ca.stats()["oom_count"] == 1 and ca.cache_stats()["cached_blocks"] == 1
    assert ca.allocate_cached(3, []) == (pk.PA_OK, 0)


def test_available_counts_free_and_parked_blocks():
    a = pk.BlockAllocator(6, 2)
    assert a.available() == 6
    assert a.allocate_cached(1, [1, 2, 3, 4, 5]) == (pk.PA_OK, 0)     # 3 blocks, 2 registered
    assert a.available() == 3
    a.free(1)                                                          # 2 parked, 1 freed
    assert a.available() == 6 and len(a.evictable_list()) == 2 and len(a.free_list()) == 4
