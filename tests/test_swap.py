"""Swapping requests between a GPU pool and a host pool: the C++ bookkeeping against the
oracle's SwappingManager bit for bit (no GPU; block_bytes 0 moves no data), and the data
round trip on the GPU (marked gpu)."""
import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import paged_kv_cache_411_b200 as pk
import synth_inputs as si
from oracle import attention as oatt
from oracle import block_manager as obm
from oracle.swap import SwappingManager
from paged_kv_cache_411_b200 import workload as pwl

_NAMES = {pk.PA_OK: obm.OK, pk.PA_ERR_OOM: obm.OOM, pk.PA_ERR_NOT_FOUND: obm.NOT_FOUND,
          pk.PA_ERR_EXISTS: obm.EXISTS, pk.PA_ERR_INVALID_ARG: obm.INVALID_ARG}

ops = st.lists(st.tuples(st.integers(0, 5), st.integers(0, 4), st.integers(0, 60)), min_size=1, max_size=100)


@settings(max_examples=200, deadline=None)
@given(st.integers(1, 20), st.integers(1, 12), st.sampled_from([1, 4, 16]), ops)
def test_swap_bookkeeping_matches_oracle(ng, nc, bs, log):
    g, c = pk.BlockAllocator(ng, bs), pk.BlockAllocator(nc, bs)
    og, oc = obm.BlockManager(ng, bs), obm.BlockManager(nc, bs)
    sm = SwappingManager(og, oc)
    for kind, r, n in log:
        if kind == 0:
            assert _NAMES[g.allocate(r, n)] == og.allocate(r, n)
        elif kind == 1:
            assert _NAMES[g.append_token(r)[0]] == og.append_token(r)[0]
        elif kind == 2:
            assert _NAMES[pk.swap_out(g, c, r, None, None, None, None, 0)] == sm.swap_out(r)
        elif kind == 3:
            assert _NAMES[pk.swap_in(g, c, r, None, None, None, None, 0)] == sm.swap_in(r)
        elif kind == 4:
            assert _NAMES[g.free(r)] == og.free(r)
        else:
            assert _NAMES[c.free(r)] == oc.free(r)
    for a, o in ((g, og), (c, oc)):
        assert a.free_list().tolist() == o.free_blocks
        for r in range(5):
            assert a.get_block_table(r)[1].tolist() == o.get_block_table(r)[1]
            assert a.seq_len(r)[1] == o.seq_len(r)[1]
        assert a.stats()["oom_count"] == o.oom_count


def test_swap_argument_errors():
    g, c = pk.BlockAllocator(4, 16), pk.BlockAllocator(4, 8)
    assert g.allocate(1, 5) == pk.PA_OK
    assert pk.swap_out(g, c, 1, None, None, None, None, 0) == pk.PA_ERR_INVALID_ARG      # block sizes differ
    c2 = pk.BlockAllocator(4, 16)
    assert pk.swap_out(g, c2, 9, None, None, None, None, 0) == pk.PA_ERR_NOT_FOUND
    assert c2.allocate(1, 1) == pk.PA_OK
    assert pk.swap_out(g, c2, 1, None, None, None, None, 0) == pk.PA_ERR_EXISTS
    with pytest.raises(pk.PagedKVError):
        pk.swap_blocks(None, None, None, None, [[0, 5]], 16, 4, 4)     # pair outside the pools


def _bits(a):
    return np.ascontiguousarray(a).view(np.int16)


@pytest.mark.gpu
def test_swap_round_trip_matches_oracle(cuda_ready):
    """Swap three sequences of a batch out to a pinned host pool and back into different GPU blocks,
    moving the same requests with the oracle's SwappingManager on NumPy copies of the same starting
    pools ([CB-PA] §4.4).  After every move the GPU pool and the host pool equal the oracle's pools
    bit for bit (NaN-poisoned spare rows included), and the tables and free lists match; decode over
    the moved blocks then matches oracle attention over the oracle's pool and is bitwise the decode
    from before the round trip."""
    from oracle import workloads as owl
    w = si.Workload(name="swap", seed=12, num_heads=8, head_dim=128, block_size=16,
                    decode_lens=(100, 37, 513, 16, 260, 1), pool_factor=2.0)
    ds = pwl.build(w)
    o = owl.build(w)
    bs = w.block_size
    kc, vc = o.k_cache.copy(), o.v_cache.copy()
    oatt.reshape_and_cache(kc, vc, o.k_step, o.v_step, o.slot_mapping, bs)
    pk.reshape_and_cache(ds.k_step, ds.v_step, ds.k_cache, ds.v_cache, ds.slot_mapping)
    S, H, D = ds.q.shape
    mb = ds.max_blocks
    ws = torch.empty(pk.decode_workspace_bytes(S, H, D, mb, bs), dtype=torch.uint8, device="cuda")
    ref = torch.empty_like(ds.q)
    pk.paged_attention_decode(ref, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.seq_lens, w.scale, ws)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(ds.k_cache.cpu().numpy()), _bits(kc))

    gpu, ogpu = ds.alloc, o.bm
    NC = 64
    cpu, ocpu = pk.BlockAllocator(NC, bs), obm.BlockManager(NC, bs)
    sm = SwappingManager(ogpu, ocpu)
    ck = torch.zeros((NC, bs, H, D), dtype=torch.float16).pin_memory()
    cv = torch.zeros_like(ck).pin_memory()
    ock, ocv = np.zeros((NC, bs, H, D), np.float16), np.zeros((NC, bs, H, D), np.float16)
    block_bytes = bs * H * D * 2

    def check_same(what):
        torch.cuda.synchronize()
        assert np.array_equal(_bits(ds.k_cache.cpu().numpy()), _bits(kc)), what
        assert np.array_equal(_bits(ds.v_cache.cpu().numpy()), _bits(vc)), what
        assert np.array_equal(_bits(ck.numpy()), _bits(ock)), what
        assert np.array_equal(_bits(cv.numpy()), _bits(ocv)), what
        assert gpu.free_list().tolist() == ogpu.free_blocks, what
        assert cpu.free_list().tolist() == ocpu.free_blocks, what
        for r in list(range(S)) + [99]:
            assert gpu.get_block_table(r)[1].tolist() == ogpu.get_block_table(r)[1], (what, r)
            assert cpu.get_block_table(r)[1].tolist() == ocpu.get_block_table(r)[1], (what, r)

    before = {r: gpu.get_block_table(r)[1] for r in (0, 2, 4)}
    for r in (0, 2, 4):
        assert pk.swap_out(gpu, cpu, r, ds.k_cache, ds.v_cache, ck, cv, block_bytes) == pk.PA_OK
        assert sm.swap_out(r, kc, vc, ock, ocv) == obm.OK
        check_same(f"swap_out {r}")
        assert gpu.seq_len(r)[0] == pk.PA_ERR_NOT_FOUND
    # reuse the freed GPU blocks for a filler request, then swap back in: new physical blocks
    filler_tokens = sum(len(v) for v in before.values()) * bs // 2
    assert gpu.allocate(99, filler_tokens) == pk.PA_OK
    assert ogpu.allocate(99, filler_tokens) == obm.OK
    for r in (0, 2, 4):
        assert pk.swap_in(gpu, cpu, r, ds.k_cache, ds.v_cache, ck, cv, block_bytes) == pk.PA_OK
        assert sm.swap_in(r, kc, vc, ock, ocv) == obm.OK
        check_same(f"swap_in {r}")
    st_, tables, lens = gpu.pack(np.arange(S), mb)
    assert st_ == pk.PA_OK
    assert any(not np.array_equal(tables[r][:len(before[r])], before[r]) for r in (0, 2, 4))
    out = torch.empty_like(ds.q)
    pk.paged_attention_decode(out, ds.q, ds.k_cache, ds.v_cache, torch.from_numpy(tables).cuda(),
                              torch.from_numpy(lens).cuda(), w.scale, ws)
    torch.cuda.synchronize()
    want = oatt.paged_attention_decode(o.q, kc, vc, tables, lens, bs, w.scale)
    assert float(np.abs(out.float().cpu().numpy() - want).max()) <= 2e-3
    assert torch.equal(out, ref)
    assert cpu.stats()["num_free"] == NC
