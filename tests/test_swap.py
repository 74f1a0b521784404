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


@pytest.mark.gpu
def test_swap_round_trip_on_gpu(cuda_ready):
    """Swap three sequences of a batch out to pinned host memory (bit-exact copies), decode the
    others, swap them back into different GPU blocks, and decode all: identical outputs."""
    w = si.Workload(name="swap", seed=12, num_heads=8, head_dim=128, block_size=16,
                    decode_lens=(100, 37, 513, 16, 260, 1), pool_factor=2.0)
    ds = pwl.build(w)
    pk.reshape_and_cache(ds.k_step, ds.v_step, ds.k_cache, ds.v_cache, ds.slot_mapping)
    S, H, D = ds.q.shape
    bs = w.block_size
    mb = ds.max_blocks
    ws = torch.empty(pk.decode_workspace_bytes(S, H, D, mb, bs), dtype=torch.uint8, device="cuda")
    ref = torch.empty_like(ds.q)
    pk.paged_attention_decode(ref, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.seq_lens, w.scale, ws)
    gpu = ds.alloc
    NC = 64
    cpu = pk.BlockAllocator(NC, bs)
    ck = torch.zeros((NC, bs, H, D), dtype=torch.float16).pin_memory()
    cv = torch.zeros_like(ck).pin_memory()
    block_bytes = bs * H * D * 2
    before = {r: gpu.get_block_table(r)[1] for r in (0, 2, 4)}
    gk_host, gv_host = ds.k_cache.cpu().numpy(), ds.v_cache.cpu().numpy()
    for r in (0, 2, 4):
        assert pk.swap_out(gpu, cpu, r, ds.k_cache, ds.v_cache, ck, cv, block_bytes) == pk.PA_OK
    torch.cuda.synchronize()
    for r in (0, 2, 4):
        ct = cpu.get_block_table(r)[1]
        assert np.array_equal(ck.numpy()[ct].view(np.int16), gk_host[before[r]].view(np.int16))
        assert np.array_equal(cv.numpy()[ct].view(np.int16), gv_host[before[r]].view(np.int16))
        assert gpu.seq_len(r)[0] == pk.PA_ERR_NOT_FOUND
    # reuse the freed GPU blocks for a filler request, then swap back in: new physical blocks
    filler_tokens = sum(len(v) for v in before.values()) * bs // 2
    assert gpu.allocate(99, filler_tokens) == pk.PA_OK
    for r in (0, 2, 4):
        assert pk.swap_in(gpu, cpu, r, ds.k_cache, ds.v_cache, ck, cv, block_bytes) == pk.PA_OK
    st_, tables, lens = gpu.pack(np.arange(S), mb)
    assert st_ == pk.PA_OK
    assert any(not np.array_equal(tables[r][:len(before[r])], before[r]) for r in (0, 2, 4))
    out = torch.empty_like(ds.q)
    pk.paged_attention_decode(out, ds.q, ds.k_cache, ds.v_cache, torch.from_numpy(tables).cuda(),
                              torch.from_numpy(lens).cuda(), w.scale, ws)
    assert torch.equal(out, ref)
    assert cpu.stats()["num_free"] == NC
