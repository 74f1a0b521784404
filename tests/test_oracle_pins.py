"""Pins of the CPU oracle against facts fixed outside it (no GPU).

Each test checks the oracle against something other than itself: numbers the
pages print (``tests/golden``), closed forms, brute force, ``torch``'s
scaled-dot-product attention on CPU in float64, invariances the paging
definition implies, and special cases with known answers.
"""
import math

import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import synth_inputs as si
from conftest import golden
from oracle import attention as oatt
from oracle import block_manager as obm
from oracle import sizes
from oracle import workloads as owl

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# --------------------------------------------------------------------- sizes
def test_kv_bytes_per_token_matches_page():
    g = golden("kv_size_llama2_7b.json")
    b = sizes.kv_bytes_per_token(g["layers"], g["heads"], g["head_dim"], g["bytes_per_elem"])
    assert b == g["bytes_per_token"]
    assert b / 2**20 == g["approx_mb_per_token"]
    assert g["tokens"] * b == g["approx_gb"] * 2**30


def test_pool_arrays_hold_closed_form_bytes():
    """A 4096-token Llama-2-7B pool in the cache layout [blocks, 16, heads, head_dim], K and V,
    32 layers, measured from NumPy's own array sizes."""
    g = golden("kv_size_llama2_7b.json")
    layer_k = np.zeros((g["tokens"] // 16, 16, g["heads"], g["head_dim"]), np.float16)
    total = g["layers"] * 2 * layer_k.nbytes
    assert total == g["tokens"] * sizes.kv_bytes_per_token(32, 32, 128, 2) == 2147483648


@pytest.mark.parametrize("bs", [1, 8, 16, 32, 48])
def test_blocks_needed_is_smallest_cover(bs):
    for n in range(0, 201):
        k = 0
        while k * bs < n:
            k += 1
        assert sizes.blocks_needed(n, bs) == k


def test_tiny_workload_demand():
    assert [sizes.blocks_needed(n, 16) for n in (5, 16, 17, 33)] == [1, 1, 2, 3]
    assert owl.demand_blocks(si.tiny()) == 7


def test_block_size_table_max_waste():
    g = golden("block_size_tradeoff.json")
    for bs, w in g["max_waste_tokens"].items():
        assert max(sizes.internal_waste(n, int(bs)) for n in range(1, 2000)) == w


def test_waste_rate_formula():
    g = golden("block_size_tradeoff.json")["example"]
    # uniform residues: mean waste is (bs - 1) / 2 exactly; the page rounds it to bs / 2
    for bs in (8, 16, 32):
        lens = range(1024, 1024 + 64 * bs)
        assert np.mean([sizes.internal_waste(n, bs) for n in lens]) == (bs - 1) / 2
    frac = sizes.expected_waste_fraction(g["block_size"], g["avg_seq_len"])
    assert frac == g["half_block"] / g["avg_seq_len"]
    assert abs(100 * frac - g["approx_waste_percent"]) < 0.01


# ------------------------------------------------------------- block manager
def test_allocator_matches_hand_trace():
    g = golden("allocator_sketch_trace.json")
    bm = obm.BlockManager(g["num_blocks"], g["block_size"])
    for i, op in enumerate(g["ops"]):
        if op[0] == "allocate":
            assert bm.allocate(op[1], op[2]) == op[3]
        elif op[0] == "append_token":
            st_, slot = bm.append_token(op[1])
            assert st_ == op[2] and slot == op[3]
        elif op[0] == "free":
            assert bm.free(op[1]) == op[2]
        if i == 0:
            assert bm.block_tables[1] == g["after_allocate_1_table"]
        if i == 1:
            assert bm.block_tables[2] == g["after_allocate_2_table"]
    assert {str(k): v for k, v in bm.block_tables.items()} == g["final_tables"]
    assert bm.free_blocks == g["final_free_list"]
    assert {str(k): v for k, v in bm.seq_lens.items()} == g["final_seq_lens"]


def test_page_table_figure():
    """The chapter's figure: A -> pages 0, 2, 5; B -> pages 1, 4; page 3 free.  With a page
    size of 48 and a free list whose pops come out in the figure's order, the block manager
    reproduces it and the paged gather walks A's pages in logical order."""
    g = golden("page_table_diagram.json")
    bs = 48
    order = [3, 4, 1, 5, 2, 0]         # popped from the end: 0, 2, 5 then 1, 4
    bm = obm.BlockManager(g["num_pages"], bs, order)
    for name in ("A", "B"):
        assert bm.allocate(name, g["requests"][name]["tokens"]) == obm.OK
        assert bm.block_tables[name] == g["requests"][name]["pages"]
    assert bm.free_blocks == g["free_pages"]
    cache = np.zeros((g["num_pages"], bs, 1, 2), np.float16)
    for p in range(g["num_pages"]):
        cache[p, :, 0, 0] = p
        cache[p, :, 0, 1] = np.arange(bs)
    rows = oatt.gather_sequence(cache, bm.block_tables["A"], 128, bs)
    assert rows[:, 0, 0].tolist() == [0] * 48 + [2] * 48 + [5] * 32
    assert rows[:, 0, 1].tolist() == list(range(48)) * 2 + list(range(32))


def _snapshot(bm):
    return (list(bm.free_blocks), {k: list(v) for k, v in bm.block_tables.items()},
            dict(bm.seq_lens), list(bm.refcount))


def _check_invariants(bm):
    N, bs = bm.num_blocks, bm.block_size
    free = bm.free_blocks
    assert len(set(free)) == len(free) and all(0 <= b < N for b in free)
    count = [0] * N
    for t in bm.block_tables.values():
        for b in t:
            count[b] += 1
    assert count == bm.refcount
    used = {b for b in range(N) if count[b] > 0}
    assert not used & set(free)
    assert len(free) + len(used) == N
    for r, t in bm.block_tables.items():
        n = bm.seq_lens[r]
        assert len(t) * bs >= n > (len(t) - 1) * bs or (n == 0 and not t)
        assert len(t) * bs - n < bs or not t
    s = bm.stats()
    assert s["num_free"] == len(free) and s["num_used"] == len(used)
    assert s["total_refs"] == sum(count)


op_strategy = st.lists(st.tuples(st.integers(0, 5), st.integers(0, 5), st.integers(0, 5),
                                 st.integers(0, 70)), min_size=1, max_size=120)


@settings(max_examples=300, deadline=None)
@given(st.integers(1, 24), st.sampled_from([1, 4, 16]), op_strategy)
def test_block_manager_invariants(N, bs, ops):
    bm = obm.BlockManager(N, bs)
    for kind, a, b, n in ops:
        before = _snapshot(bm)
        if kind == 0:
            st_ = bm.allocate(a, n)
        elif kind == 1:
            st_, _ = bm.append_token(a)
        elif kind == 2:
            st_, slots = bm.append_tokens(a, n % 7)
            if st_ == obm.OK:
                assert len(slots) == n % 7
        elif kind == 3:
            src_len = bm.seq_lens.get(a, 0)
            st_ = bm.fork(a, b, min(n, src_len))
        else:
            st_ = bm.free(a)
        if st_ in (obm.OOM, obm.EXISTS, obm.NOT_FOUND, obm.INVALID_ARG):
            assert _snapshot(bm) == before
        _check_invariants(bm)


def test_append_takes_block_only_at_boundary():
    bm = obm.BlockManager(10, 4)
    assert bm.allocate(0, 0) == obm.OK and bm.block_tables[0] == []
    taken = []
    for pos in range(13):
        free_before = len(bm.free_blocks)
        st_, slot = bm.append_token(0)
        assert st_ == obm.OK
        taken.append(free_before - len(bm.free_blocks))
        t = bm.block_tables[0]
        assert slot == t[pos // 4] * 4 + pos % 4
    assert taken == [1, 0, 0, 0] * 3 + [1]


def test_oom_keeps_state_and_counts():
    bm = obm.BlockManager(3, 16)
    assert bm.allocate(0, 40) == obm.OK
    snap = _snapshot(bm)
    assert bm.allocate(1, 17) == obm.OOM
    assert bm.append_tokens(0, 9)[0] == obm.OOM       # 49 tokens need a 4th block
    assert _snapshot(bm) == snap and bm.oom_count == 2
    assert bm.append_tokens(0, 8)[0] == obm.OK        # 48 tokens fit in 3 blocks
    assert bm.append_token(0)[0] == obm.OOM


def test_shared_prefix_stored_once_and_refcounted():
    """The page's shared system prompt: three blocks stored once, two requests pointing at
    them, each with private blocks; blocks return to the free list only at refcount zero."""
    bm = obm.BlockManager(16, 16)
    assert bm.allocate("sys", 48) == obm.OK
    sys_blocks = list(bm.block_tables["sys"])
    for r in ("r1", "r2"):
        assert bm.fork("sys", r, 48) == obm.OK
        assert bm.append_tokens(r, 20)[0] == obm.OK
        assert bm.block_tables[r][:3] == sys_blocks
    assert all(bm.refcount[b] == 3 for b in sys_blocks)
    private = set(bm.block_tables["r1"][3:]) | set(bm.block_tables["r2"][3:])
    assert len(private) == 4 and not private & set(sys_blocks)
    assert bm.stats()["num_used"] == 7
    bm.free("sys")
    bm.free("r1")
    assert not set(sys_blocks) & set(bm.free_blocks)
    bm.free("r2")
    assert set(sys_blocks) <= set(bm.free_blocks)
    assert len(bm.free_blocks) == 16
    # a fork shares whole blocks only: 40 tokens -> 2 blocks, child length 32
    assert bm.allocate("p", 40) == obm.OK
    assert bm.fork("p", "c", 40) == obm.OK
    assert bm.seq_lens["c"] == 32 and bm.block_tables["c"] == bm.block_tables["p"][:2]


def test_free_unknown_and_errors():
    bm = obm.BlockManager(4, 16)
    assert bm.free(123) == obm.OK
    assert bm.append_token(5)[0] == obm.NOT_FOUND
    assert bm.allocate(1, -1) == obm.INVALID_ARG
    assert bm.allocate(1, 16) == obm.OK
    assert bm.allocate(1, 16) == obm.EXISTS
    assert bm.fork(1, 2, 17) == obm.INVALID_ARG
    assert bm.fork(9, 2, 0) == obm.NOT_FOUND
    st_, t, l = bm.pack([1], 0)
    assert st_ == obm.INVALID_ARG
    st_, t, l = bm.pack([1], 3)
    assert st_ == obm.OK and t == [[bm.block_tables[1][0], -1, -1]] and l == [16]


# ----------------------------------------------------------------- attention
def _place(rng, logical, bs, num_blocks, order):
    """Put each sequence's logical rows into a NaN cache at blocks taken from ``order``."""
    H, D = logical[0].shape[1:]
    cache = np.full((num_blocks, bs, H, D), np.nan, np.float16)
    tables, nxt = [], 0
    for rows in logical:
        nb = sizes.blocks_needed(len(rows), bs)
        t = [int(b) for b in order[nxt:nxt + nb]]
        nxt += nb
        for j, row in enumerate(rows):
            cache[t[j // bs], j % bs] = row
        tables.append(t)
    maxb = max(len(t) for t in tables)
    return cache, np.asarray([t + [-1] * (maxb - len(t)) for t in tables], np.int32)


def _sdpa(q, k, v, scale, causal=False):
    """torch's scaled_dot_product_attention in float64 on CPU; q [L,H,D], k/v [n,H,D]."""
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64)).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=scale, is_causal=causal)
    return o[0].permute(1, 0, 2).numpy()


def _random_case(seed, S, H, D, bs, lens, extra_blocks=3, shuffle=True):
    rng = np.random.default_rng(seed)
    logical_k = [rng.standard_normal((n, H, D)).astype(np.float16) for n in lens]
    logical_v = [rng.standard_normal((n, H, D)).astype(np.float16) for n in lens]
    q = rng.standard_normal((S, H, D)).astype(np.float16)
    N = sum(sizes.blocks_needed(n, bs) for n in lens) + extra_blocks
    order = rng.permutation(N) if shuffle else np.arange(N)
    kc, tables = _place(rng, logical_k, bs, N, order)
    vc, _ = _place(rng, logical_v, bs, N, order)
    return q, logical_k, logical_v, kc, vc, tables


@pytest.mark.parametrize("H,D,bs,lens", [
    (4, 64, 16, [5, 16, 17, 33]),
    (2, 128, 16, [1, 64, 100]),
    (3, 32, 32, [31, 32, 33, 200]),
    (2, 16, 1, [7, 3]),
    (1, 8, 8, [250]),
])
def test_decode_matches_torch_sdpa(H, D, bs, lens):
    S = len(lens)
    q, lk, lv, kc, vc, tables = _random_case(7, S, H, D, bs, lens)
    scale = 1 / math.sqrt(D)
    out = oatt.paged_attention_decode(q, kc, vc, tables, lens, bs, scale)
    for s in range(S):
        ref = _sdpa(q[s][None], lk[s], lv[s], scale)[0]
        np.testing.assert_allclose(out[s], ref, rtol=1e-12, atol=1e-12)


def test_decode_scale_is_honoured():
    q, lk, lv, kc, vc, tables = _random_case(3, 2, 2, 64, 16, [40, 9])
    for scale in (0.05, 0.3, 1.0):
        out = oatt.paged_attention_decode(q, kc, vc, tables, [40, 9], 16, scale)
        for s in range(2):
            np.testing.assert_allclose(out[s], _sdpa(q[s][None], lk[s], lv[s], scale)[0], atol=1e-12)


def test_decode_invariant_under_block_permutation():
    lens = [37, 16, 1, 90]
    q, lk, lv, kc, vc, tables = _random_case(11, 4, 4, 64, 16, lens, extra_blocks=5)
    base = oatt.paged_attention_decode(q, kc, vc, tables, lens, 16, 0.125)
    for seed in range(3):
        perm = np.random.default_rng(seed).permutation(kc.shape[0])
        kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
        kc2[perm], vc2[perm] = kc, vc
        t2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1)
        out = oatt.paged_attention_decode(q, kc2, vc2, t2, lens, 16, 0.125)
        assert np.array_equal(out, base)


def test_decode_special_cases():
    rng = np.random.default_rng(5)
    H, D, bs = 2, 64, 16
    # one token: the output is that token's V exactly
    q, lk, lv, kc, vc, tables = _random_case(1, 1, H, D, bs, [1])
    out = oatt.paged_attention_decode(q, kc, vc, tables, [1], bs, 0.125)
    assert np.array_equal(out[0], lv[0][0].astype(np.float64))
    # all keys equal: the output is the mean of V
    n = 45
    k = np.repeat(rng.standard_normal((1, H, D)).astype(np.float16), n, axis=0)
    v = rng.standard_normal((n, H, D)).astype(np.float16)
    kc, tables = _place(rng, [k], bs, 4, [2, 0, 3, 1])
    vc, _ = _place(rng, [v], bs, 4, [2, 0, 3, 1])
    out = oatt.paged_attention_decode(rng.standard_normal((1, H, D)).astype(np.float16), kc, vc,
                                      tables, [n], bs, 0.125)
    np.testing.assert_allclose(out[0], v.astype(np.float64).mean(0), atol=1e-13)
    # one dominant key: the output is that key's V
    k = rng.standard_normal((n, H, D)).astype(np.float16)
    k[17] = 0
    k[17, :, 0] = 100
    qd = np.zeros((1, H, D), np.float16)
    qd[0, :, 0] = 100
    kc, tables = _place(rng, [k], bs, 4, [1, 3, 0, 2])
    vc, _ = _place(rng, [v], bs, 4, [1, 3, 0, 2])
    out = oatt.paged_attention_decode(qd, kc, vc, tables, [n], bs, 1 / 8)
    np.testing.assert_allclose(out[0], v[17].astype(np.float64), atol=1e-12)
    # an empty sequence gives zeros
    out = oatt.paged_attention_decode(qd, kc, vc, tables, [0], bs, 1 / 8)
    assert not out.any()


def test_prefill_without_context_is_causal_sdpa():
    L, H, D, bs = 70, 3, 64, 16
    q, lk, lv, kc, vc, tables = _random_case(4, 1, H, D, bs, [L])
    rng = np.random.default_rng(9)
    qc = rng.standard_normal((L, H, D)).astype(np.float16)
    out = oatt.paged_attention_prefill_chunk(qc, kc, vc, tables, [0, L], [0], bs, 0.125)
    np.testing.assert_allclose(out, _sdpa(qc, lk[0], lv[0], 0.125, causal=True), atol=1e-12)


def test_prefill_chunk_split_and_last_row_match_decode():
    c, L, H, D, bs = 50, 40, 2, 64, 16
    q, lk, lv, kc, vc, tables = _random_case(8, 1, H, D, bs, [c + L])
    qc = np.random.default_rng(2).standard_normal((L, H, D)).astype(np.float16)
    whole = oatt.paged_attention_prefill_chunk(qc, kc, vc, tables, [0, L], [c], bs, 0.125)
    a = oatt.paged_attention_prefill_chunk(qc[:13], kc, vc, tables, [0, 13], [c], bs, 0.125)
    b = oatt.paged_attention_prefill_chunk(qc[13:], kc, vc, tables, [0, L - 13], [c + 13], bs, 0.125)
    np.testing.assert_allclose(whole, np.concatenate([a, b]), rtol=0, atol=1e-13)
    dec = oatt.paged_attention_decode(qc[-1:], kc, vc, tables, [c + L], bs, 0.125)
    np.testing.assert_allclose(whole[-1], dec[0], atol=1e-13)
    # row i sees exactly c + i + 1 keys: it must differ from the decode over c + i keys
    d2 = oatt.paged_attention_decode(qc[5:6], kc, vc, tables, [c + 5], bs, 0.125)
    assert not np.allclose(whole[5], d2[0])
    # two requests in one call give the same rows as two calls
    two = oatt.paged_attention_prefill_chunk(np.concatenate([qc, qc[:7]]), kc, vc,
                                             np.concatenate([tables, tables]), [0, L, L + 7], [c, 3], bs, 0.125)
    one = oatt.paged_attention_prefill_chunk(qc[:7], kc, vc, tables, [0, 7], [3], bs, 0.125)
    np.testing.assert_allclose(two[:L], whole, atol=0)
    np.testing.assert_allclose(two[L:], one, atol=0)


def test_reshape_then_gather_round_trip():
    """Write rows at the block manager's slots, read them back through the block table."""
    rng = np.random.default_rng(0)
    H, D, bs = 2, 8, 4
    bm = obm.BlockManager(9, bs, list(rng.permutation(9)))
    assert bm.allocate(0, 0) == obm.OK and bm.allocate(1, 3) == obm.OK
    kc = np.full((9, bs, H, D), np.nan, np.float16)
    vc = kc.copy()
    k = rng.standard_normal((11, H, D)).astype(np.float16)
    v = rng.standard_normal((11, H, D)).astype(np.float16)
    st_, slots = bm.append_tokens(0, 11)
    oatt.reshape_and_cache(kc, vc, k, v, slots, bs)
    np.testing.assert_array_equal(oatt.gather_sequence(kc, bm.block_tables[0], 11, bs), k.astype(np.float64))
    np.testing.assert_array_equal(oatt.gather_sequence(vc, bm.block_tables[0], 11, bs), v.astype(np.float64))
    # padding tokens (slot < 0) are skipped and nothing else changes
    before = kc.copy()
    oatt.reshape_and_cache(kc, vc, k[:2], v[:2], [-1, -7], bs)
    assert np.array_equal(np.isnan(kc), np.isnan(before))
    assert np.array_equal(np.nan_to_num(kc), np.nan_to_num(before))
    assert int((~np.isnan(kc)).sum()) == 11 * H * D


# ------------------------------------------------------------------ workloads
def test_tiny_workload_against_logical_sdpa():
    """The whole replay (allocation, placement, step slot mapping, new-token write, paged
    read) agrees with SDPA over the logical sequences drawn directly from the recipe."""
    w = si.tiny()
    step = owl.build(w)
    assert step.num_blocks == 16 and step.bm.stats()["num_used"] == 7
    assert [len([b for b in t if b >= 0]) for t in step.block_tables] == [1, 1, 2, 3]
    dec, _, kc, vc = owl.run_step(step)
    qn, kn, vn = w.q(), w.k_new(), w.v_new()
    for s, n in enumerate(w.decode_lens):
        k_ctx, v_ctx = w.context_kv(s, n - 1)
        k = np.concatenate([k_ctx, kn[s][None]])
        v = np.concatenate([v_ctx, vn[s][None]])
        np.testing.assert_allclose(dec[s], _sdpa(qn[s][None], k, v, w.scale)[0], atol=1e-12)
    # used slots are finite, every other slot is still poison
    finite = ~np.isnan(kc[..., 0, 0])
    assert finite.sum() == sum(w.decode_lens)


def test_mixed_workload_prefill_against_logical_sdpa():
    w = si.mixed_prefill_decode()
    small = si.Workload(name="mixed_small", seed=w.seed, num_heads=2, head_dim=64, block_size=16,
                        decode_lens=(130, 17), pool_factor=1.1, prefill=si.PrefillSpec(ctx_before=40, chunk=24))
    step = owl.build(small)
    assert len(step.slot_mapping) == 24 + 2
    dec, pre, kc, vc = owl.run_step(step)
    qc, kq, vq = small.prefill_qkv()
    kctx, vctx = small.prefill_context_kv()
    k = np.concatenate([kctx, kq])
    v = np.concatenate([vctx, vq])
    for i in range(24):
        ref = _sdpa(qc[i][None], k[:40 + i + 1], v[:40 + i + 1], small.scale)[0]
        np.testing.assert_allclose(pre[i], ref, atol=1e-12)


def test_shared_prefix_workload_refcounts():
    w = si.long_shared_prefix()
    small = si.Workload(name="prefix_small", seed=5, num_heads=2, head_dim=16, block_size=32,
                        decode_lens=(200,) * 3, pool_factor=1.1, shared_prefix=64)
    step = owl.build(small)
    bm = step.bm
    shared = step.block_tables[0][:2]
    assert all(bm.refcount[b] == 3 for b in shared)
    assert all((step.block_tables[s][:2] == shared).all() for s in range(3))
    assert bm.stats()["num_used"] == 2 + 3 * sizes.blocks_needed(200 - 64, 32)
    dec, _, kc, vc = owl.run_step(step)
    kp, vp = small.prefix_kv()
    for s in range(3):
        kx, vx = small.context_kv(s, 200 - 1 - 64)
        k = np.concatenate([kp, kx, small.k_new()[s][None]])
        v = np.concatenate([vp, vx, small.v_new()[s][None]])
        np.testing.assert_allclose(dec[s], _sdpa(small.q()[s][None], k, v, small.scale)[0], atol=1e-12)
    # the full-size recipe's demand in closed form: 32 shared prefix blocks + 8 x 992 private ones
    assert owl.demand_blocks(w) == 32 + 8 * 992
    assert owl.pool_blocks(w) == math.ceil(1.1 * (32 + 8 * 992))


def test_churn_workload_fragments_pool():
    w = si.llama7b_b256_ragged()
    small = si.Workload(name="churn_small", seed=3, num_heads=1, head_dim=8, block_size=16,
                        decode_lens=w.decode_lens[:32], pool_factor=1.5, shuffle_free_list=False,
                        churn=si.ChurnSpec(n_ops=2000, max_tokens=512))
    step = owl.build(small, seqs=[0, 5])
    _check_invariants(step.bm)
    tables = [t[t >= 0] for t in step.block_tables]
    runs = sum(int(np.all(np.diff(t) == 1)) for t in tables if len(t) > 2)
    multi = sum(1 for t in tables if len(t) > 2)
    assert runs < multi           # churn left the targets' blocks scattered
    assert min(w.decode_lens) >= 16 and max(w.decode_lens) <= 4096
