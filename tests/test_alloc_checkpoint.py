"""Checkpoint / resume of the host allocator (pa_alloc_serialize / pa_alloc_deserialize; no GPU).

A seeded log of allocator operations -- plain allocations, appends, forks, frees, and the prefix-cache
calls that register, park and evict blocks -- is cut at a random point: the state is written to bytes,
read back into a second allocator, and the rest of the log runs on both.  The two must report the same
status for every operation and end with byte-identical states.  Malformed bytes are refused without
creating anything."""
import numpy as np
import pytest

import paged_kv_cache_411_b200 as pk


def _run_ops(rng, n_ops, num_blocks, bs):
    """A seeded op log over a small pool (so that OOM, parking and eviction all happen)."""
    systems = [rng.integers(0, 50, int(rng.integers(bs, 4 * bs))).tolist() for _ in range(3)]
    ops, live, next_id = [], [], 0
    for _ in range(n_ops):
        kind = rng.choice(["alloc", "cached", "begin", "append", "extend", "fork", "free"],
                          p=[.12, .16, .12, .3, .1, .05, .15])
        if kind in ("alloc", "cached", "begin") or not live:
            toks = systems[int(rng.integers(3))] + rng.integers(0, 50, int(rng.integers(0, 3 * bs))).tolist()
            ops.append((kind if kind in ("alloc", "cached", "begin") else "cached", next_id, toks))
            live.append(next_id)
            next_id += 1
        elif kind == "append":
            ops.append(("append", live[int(rng.integers(len(live)))], int(rng.integers(1, 2 * bs))))
        elif kind == "extend":
            ops.append(("extend", live[int(rng.integers(len(live)))], rng.integers(0, 50, int(rng.integers(1, bs))).tolist()))
        elif kind == "fork":
            ops.append(("fork", live[int(rng.integers(len(live)))], next_id, int(rng.integers(0, 3 * bs))))
            live.append(next_id)
            next_id += 1
        else:
            r = live.pop(int(rng.integers(len(live))))
            ops.append(("free", r))
    return ops


def _apply(a, op):
    kind = op[0]
    if kind == "alloc":
        return a.allocate(op[1], len(op[2]))
    if kind == "cached":
        return a.allocate_cached(op[1], op[2])[0]
    if kind == "begin":
        return a.begin_cached(op[1], op[2])[0]
    if kind == "append":
        return a.append_tokens(op[1], op[2])[0]
    if kind == "extend":
        return a.extend_tokens(op[1], op[2])
    if kind == "fork":
        return a.fork(op[1], op[2], op[3])
    return a.free(op[1])


@pytest.mark.parametrize("seed", range(12))
def test_resume_continues_identically(seed):
    rng = np.random.default_rng(seed)
    bs = int(rng.choice([2, 4, 16]))
    num_blocks = int(rng.integers(8, 40))
    ops = _run_ops(rng, 300, num_blocks, bs)
    cut = int(rng.integers(0, len(ops)))
    a = pk.BlockAllocator(num_blocks, bs, free_order=rng.permutation(num_blocks))
    for op in ops[:cut]:
        _apply(a, op)
    state = a.serialize()
    b = pk.BlockAllocator.deserialize(state)
    assert b.serialize() == state                      # read back unchanged
    assert (b.num_blocks, b.block_size) == (num_blocks, bs)
    for op in ops[cut:]:
        assert _apply(a, op) == _apply(b, op), op
    assert a.serialize() == b.serialize()
    assert a.free_list().tolist() == b.free_list().tolist()
    assert a.cache_stats() == b.cache_stats() and a.evictable_list().tolist() == b.evictable_list().tolist()


def test_equal_states_give_equal_bytes():
    """Equal states serialise to equal bytes even when the requests' hash map got there by another path
    (extra requests created and freed first): maps are written in key order."""
    a, b = pk.BlockAllocator(16, 4), pk.BlockAllocator(16, 4)
    for r in (100, 7, 42):                   # zero-token requests take no block; freeing them changes nothing else
        assert b.allocate(r, 0) == pk.PA_OK
    for r in (42, 100, 7):
        assert b.free(r) == pk.PA_OK
    for x in (a, b):
        for r in (5, 1, 9):
            assert x.allocate(r, 6) == pk.PA_OK
        assert x.append_token(1)[0] == pk.PA_OK
    assert a.serialize() == b.serialize()


def test_malformed_state_is_refused():
    rng = np.random.default_rng(3)
    a = pk.BlockAllocator(24, 4)
    for op in _run_ops(rng, 120, 24, 4):
        _apply(a, op)
    good = a.serialize()
    for cut in [0, 3, 8, 20, len(good) // 2, len(good) - 1]:
        with pytest.raises(pk.PagedKVError):
            pk.BlockAllocator.deserialize(good[:cut])
    with pytest.raises(pk.PagedKVError):
        pk.BlockAllocator.deserialize(b"XXXX" + good[4:])            # magic
    with pytest.raises(pk.PagedKVError):
        pk.BlockAllocator.deserialize(good + b"\0")                 # trailing bytes
    # random single-byte corruptions: refused, or read as some well-formed state; never a crash
    for _ in range(400):
        bad = bytearray(good)
        i = int(rng.integers(len(bad)))
        bad[i] = int(rng.integers(256))
        try:
            pk.BlockAllocator.deserialize(bytes(bad)).close()
        except pk.PagedKVError:
            pass


@pytest.mark.parametrize("seed", range(4))
def test_every_reachable_state_is_accepted(seed):
    """The consistency checks of the reader (refcounts against the tables, free and parked blocks,
    child counts) hold in every state the operations reach: each one reads back to the same bytes."""
    rng = np.random.default_rng(100 + seed)
    bs = int(rng.choice([2, 4]))
    a = pk.BlockAllocator(20, bs, free_order=rng.permutation(20))
    for op in _run_ops(rng, 150, 20, bs):
        _apply(a, op)
        state = a.serialize()
        b = pk.BlockAllocator.deserialize(state)
        assert b.serialize() == state
        b.close()


# byte offset of the first free-list entry: magic, version, num_blocks, block_size (4 x 4 bytes), four i64
# counters, the u64 free-list length; the refcounts follow the free list
FREE_LIST_AT = 16 + 32 + 8


def test_inconsistent_state_is_refused():
    """Well-formed bytes that describe an impossible state are refused: a refcount that disagrees with
    the block tables, and a block that is both free and held by a request."""
    a = pk.BlockAllocator(12, 4)
    assert a.allocate(1, 9) == pk.PA_OK                  # 3 blocks held
    assert a.allocate(2, 4) == pk.PA_OK                  # 1 block held
    good = a.serialize()
    nf = len(a.free_list())
    assert nf == 8
    off = FREE_LIST_AT + 4 * nf                          # refcount[0]
    st, table = a.get_block_table(1)
    assert st == pk.PA_OK
    held = int(table[0])
    # one more reference than the tables hold
    bad = bytearray(good)
    rc = int.from_bytes(bad[off + 4 * held: off + 4 * held + 4], "little")
    assert rc == 1
    bad[off + 4 * held: off + 4 * held + 4] = (2).to_bytes(4, "little")
    with pytest.raises(pk.PagedKVError):
        pk.BlockAllocator.deserialize(bytes(bad))
    # the top of the free stack replaced by a block that request 1 holds
    bad = bytearray(good)
    top = FREE_LIST_AT + 4 * (nf - 1)                    # the last free-list entry
    bad[top: top + 4] = held.to_bytes(4, "little")
    with pytest.raises(pk.PagedKVError):
        pk.BlockAllocator.deserialize(bytes(bad))
    pk.BlockAllocator.deserialize(good).close()           # the untouched bytes still read
