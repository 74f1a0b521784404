"""Host-side checks of libpagedkv (no GPU): the library loads, exports every
entry point the header declares, rejects bad arguments before touching a
device, and its C++ block allocator matches the oracle bit for bit."""
import os
import re

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

import paged_kv_cache_411_b200 as pk
import synth_inputs as si
from conftest import ROOT
from oracle import block_manager as obm
from oracle import workloads as owl
from paged_kv_cache_411_b200 import _lib
from paged_kv_cache_411_b200 import workload as pwl

HEADER = os.path.join(ROOT, "include", "pagedkv.h")


def _declared():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = pk.lib()
    names = _declared()
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), "ctypes signatures out of sync with the header"
    assert lib.pa_abi_version() == 2


def test_header_serves_a_plain_c_program(tmp_path):
    """include/pagedkv.h compiles as strict C11 and a C program linked against libpagedkv.so follows a
    hand-traced allocator sequence (tests/c_consumer/alloc_from_c.c) with no Python in between."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = os.path.join(ROOT, "tests", "c_consumer", "alloc_from_c.c")
    exe = str(tmp_path / "alloc_from_c")
    libdir = os.path.dirname(_lib.LIB_PATH)
    r = subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                        src, "-o", exe, "-L", libdir, "-lpagedkv", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr


def test_status_strings_and_device_flag():
    lib = pk.lib()
    assert lib.pa_status_string(pk.PA_ERR_OOM) == b"PA_ERR_OOM"
    assert lib.pa_check_device_flag(0) == pk.PA_OK
    assert lib.pa_check_device_flag(pk.PA_DEVCHK_BLOCK_ID) == pk.PA_ERR_DEVICE_CHECK


def test_device_entry_points_reject_bad_arguments_on_host():
    """Argument errors come back before anything is enqueued (no GPU needed)."""
    lib = pk.lib()
    # unsupported head_dim
    assert lib.pa_paged_attention_decode(None, None, None, None, None, None, 1, 4, 96, 16, 4, 4, 0.1,
                                         None, 0, None, None) == pk.PA_ERR_UNSUPPORTED
    # unsupported block size
    assert lib.pa_paged_attention_decode(None, None, None, None, None, None, 1, 4, 64, 12, 4, 4, 0.1,
                                         None, 0, None, None) == pk.PA_ERR_UNSUPPORTED
    # NULL pointers with work to do
    assert lib.pa_paged_attention_decode(None, None, None, None, None, None, 1, 4, 64, 16, 4, 4, 0.1,
                                         None, 0, None, None) == pk.PA_ERR_INVALID_ARG
    assert lib.pa_reshape_and_cache(None, None, None, None, None, 3, 4, 64, 16, 4, None, None) == pk.PA_ERR_INVALID_ARG
    assert lib.pa_reshape_and_cache(None, None, None, None, None, -1, 4, 64, 16, 4, None, None) == pk.PA_ERR_INVALID_ARG
    # nothing to do is fine even without buffers
    assert lib.pa_reshape_and_cache(None, None, None, None, None, 0, 4, 64, 16, 4, None, None) == pk.PA_OK
    assert lib.pa_paged_attention_decode(None, None, None, None, None, None, 0, 4, 64, 16, 4, 4, 0.1,
                                         None, 0, None, None) == pk.PA_OK
    assert pk.decode_workspace_bytes(4, 4, 64, 3, 16) > 0
    assert pk.decode_workspace_bytes(-1, 4, 64, 3, 16) == 0


# Stand-in addresses: every call below fails a host-side check before anything is launched, so these
# are never dereferenced (the checks look only at their values).
_A = 1 << 20            # 256-byte aligned
_BUF = [_A + i * (1 << 16) for i in range(6)]


def _decode_call(ws, ws_bytes, scale=0.125, S=4, H=4, D=64, bs=16, mb=3, nb=16):
    return pk.lib().pa_paged_attention_decode(*_BUF, S, H, D, bs, mb, nb, scale, ws, ws_bytes, None, None)


def test_decode_rejects_misaligned_or_small_workspace():
    need = pk.decode_workspace_bytes(4, 4, 64, 3, 16)
    assert _decode_call(_A + 64, need) == pk.PA_ERR_INVALID_ARG
    assert "256-byte aligned" in pk.last_error()
    assert _decode_call(_A, need - 1) == pk.PA_ERR_INVALID_ARG
    assert f"< {need}" in pk.last_error()
    assert _decode_call(None, need) == pk.PA_ERR_INVALID_ARG
    assert "NULL" in pk.last_error()
    # a misaligned fp16 buffer is refused before the workspace is looked at
    bad = list(_BUF)
    bad[1] += 2
    assert pk.lib().pa_paged_attention_decode(*bad, 4, 4, 64, 16, 3, 16, 0.125, _A, need, None, None) == \
        pk.PA_ERR_INVALID_ARG
    assert "16-byte aligned" in pk.last_error()


@pytest.mark.parametrize("scale", [0.0, -0.125, float("nan"), float("inf")])
def test_attention_entry_points_refuse_bad_scale(scale):
    """The softmax temperature must be finite and positive: decode and prefill refuse anything else
    before launching (the prefill kernel takes its row maximum on unscaled scores)."""
    need = pk.decode_workspace_bytes(4, 4, 64, 3, 16)
    assert _decode_call(_A, need, scale=scale) == pk.PA_ERR_INVALID_ARG
    assert "scale" in pk.last_error()
    st = pk.lib().pa_paged_attention_prefill_chunk(*_BUF, _A, 1, 32, 4, 64, 16, 3, 16, scale, None, None)
    assert st == pk.PA_ERR_INVALID_ARG
    assert "scale" in pk.last_error()


def test_workspace_bytes_grow_with_shape():
    a = pk.decode_workspace_bytes(32, 32, 128, 64, 16)
    b = pk.decode_workspace_bytes(64, 32, 128, 64, 16)
    c = pk.decode_workspace_bytes(32, 32, 128, 256, 16)
    assert 0 < a < b and a < c
    assert a % 256 == 0


# ------------------------------------------------------------ allocator parity
_NAMES = {pk.PA_OK: obm.OK, pk.PA_ERR_OOM: obm.OOM, pk.PA_ERR_NOT_FOUND: obm.NOT_FOUND,
          pk.PA_ERR_EXISTS: obm.EXISTS, pk.PA_ERR_INVALID_ARG: obm.INVALID_ARG}


def _compare_state(ca: pk.BlockAllocator, om: obm.BlockManager, reqs):
    assert ca.free_list().tolist() == om.free_blocks
    for r in reqs:
        st, t = ca.get_block_table(r)
        ost, ot = om.get_block_table(r)
        assert _NAMES[st] == ost
        assert t.tolist() == ot
        st, n = ca.seq_len(r)
        assert _NAMES[st] == om.seq_len(r)[0] and n == om.seq_len(r)[1]
    for b in range(om.num_blocks):
        assert ca.refcount(b) == (pk.PA_OK, om.refcount[b])
    cs, os_ = ca.stats(), om.stats()
    for k in ("num_blocks", "num_free", "num_used", "total_refs", "num_requests", "oom_count", "waste_tokens"):
        assert cs[k] == os_[k], k


ops = st.lists(st.tuples(st.integers(0, 6), st.integers(0, 5), st.integers(0, 5), st.integers(0, 80)),
               min_size=1, max_size=150)


@settings(max_examples=200, deadline=None)
@given(st.integers(0, 30), st.sampled_from([1, 3, 8, 16]), st.booleans(), ops)
def test_cpp_allocator_matches_oracle_on_random_logs(N, bs, shuffled, log):
    order = list(np.random.default_rng(N * 31 + bs).permutation(N)) if shuffled else None
    ca = pk.BlockAllocator(N, bs, order)
    om = obm.BlockManager(N, bs, order)
    for kind, a, b, n in log:
        if kind == 0:
            assert _NAMES[ca.allocate(a, n)] == om.allocate(a, n)
        elif kind == 1:
            st, slot = ca.append_token(a)
            ost, oslot = om.append_token(a)
            assert _NAMES[st] == ost and slot == oslot
        elif kind == 2:
            st, slots = ca.append_tokens(a, n % 9)
            ost, oslots = om.append_tokens(a, n % 9)
            assert _NAMES[st] == ost and slots.tolist() == oslots
        elif kind == 3:
            p = min(n, om.seq_lens.get(a, 0)) if n % 5 else n + 1000
            assert _NAMES[ca.fork(a, b, p)] == om.fork(a, b, p)
        elif kind == 4:
            assert _NAMES[ca.free(a)] == om.free(a)
        elif kind == 5:
            if a in om.seq_lens:
                L = om.seq_lens[a]
                p0, cnt = min(n, L), max(0, L - min(n, L))
                st, sl = ca.slots(a, p0, cnt)
                ost, osl = om.slots(a, p0, cnt)
                assert _NAMES[st] == ost and sl.tolist() == osl
        else:
            reqs = sorted(om.block_tables)[:3]
            mb = max([len(om.block_tables[r]) for r in reqs] + [0]) + (n % 3)
            st, t, l = ca.pack(reqs, mb)
            ost, ot, ol = om.pack(reqs, mb)
            assert _NAMES[st] == ost
            if ost == obm.OK:
                assert t.tolist() == ot and l.tolist() == ol
    _compare_state(ca, om, range(6))


def test_binding_refuses_host_tensors():
    """The kernel wrappers refuse tensors that are not on the GPU before any C call, since the kernels
    would dereference them on the device."""
    import torch
    H, D, bs, nb = 4, 64, 16, 4
    q = torch.zeros(1, H, D, dtype=torch.float16)
    kc = torch.zeros(nb, bs, H, D, dtype=torch.float16)
    tables = torch.zeros(1, 2, dtype=torch.int32)
    lens = torch.ones(1, dtype=torch.int32)
    with pytest.raises(pk.PagedKVError, match="CUDA tensors expected"):
        pk.paged_attention_decode(q.clone(), q, kc, kc, tables, lens, 0.125, torch.zeros(1 << 12, dtype=torch.uint8))
    with pytest.raises(pk.PagedKVError, match="CUDA tensors expected"):
        pk.paged_attention_decode_noalloc(q.clone(), q, kc, kc, tables, lens, 0.125)
    with pytest.raises(pk.PagedKVError, match="CUDA tensors expected"):
        pk.paged_attention_prefill_chunk(q.clone(), q, kc, kc, tables, torch.tensor([0, 1], dtype=torch.int32),
                                         torch.zeros(1, dtype=torch.int32), 0.125)
    with pytest.raises(pk.PagedKVError, match="CUDA tensors expected"):
        pk.reshape_and_cache(q, q, kc, kc, torch.zeros(1, dtype=torch.int64))


def test_cpp_allocator_error_paths():
    with pytest.raises(pk.PagedKVError):
        pk.BlockAllocator(4, 16, [0, 1, 1, 2])
    with pytest.raises(pk.PagedKVError):
        pk.BlockAllocator(4, 0)
    a = pk.BlockAllocator(4, 16)
    assert a.allocate(1, 10) == pk.PA_OK
    assert a.refcount(4)[0] == pk.PA_ERR_INVALID_ARG
    assert a.slots(1, 5, 6)[0] == pk.PA_ERR_INVALID_ARG
    assert a.get_block_table(9)[0] == pk.PA_ERR_NOT_FOUND
    st, t, l = a.pack([1, 9], 2)
    assert st == pk.PA_ERR_NOT_FOUND


@pytest.mark.parametrize("name", ["tiny", "b32", "b256", "mixed", "longctx", "prefill8k"])
def test_workload_replay_matches_oracle(name):
    """Every workload's allocation replay through the C++ allocator is bit-identical to the
    oracle's: pool size, churn cap hits, tables, free list, refcounts, step slot mapping."""
    w = si.get(name)
    r = pwl.replay(w)
    o = owl.build(w, seqs=[])
    assert r.num_blocks == o.num_blocks and r.cap_hits == o.cap_hits
    assert np.array_equal(r.step_slots, o.slot_mapping)
    _compare_state(r.alloc, o.bm, list(range(w.num_seqs)) + [si.PREFILL_REQ, si.PREFIX_REQ])
    mb = o.max_blocks
    st, t, l = r.alloc.pack(np.arange(w.num_seqs), mb)
    assert st == pk.PA_OK and np.array_equal(t, o.block_tables) and np.array_equal(l, o.seq_lens)
    if w.prefill is not None:
        assert np.array_equal(r.prefill_table, o.prefill_table)
    # the context segments land on the oracle's slots
    for sl, source, index, pos0 in r.segments:
        if source == "context":
            ot = o.block_tables[index]
            pos = np.arange(pos0, pos0 + len(sl))
            assert np.array_equal(sl, ot[pos // w.block_size].astype(np.int64) * w.block_size + pos % w.block_size)


@pytest.mark.parametrize("bs", [8, 16, 32, 64])
def test_internal_waste_matches_page_estimate(bs):
    """Block-size trade-off (page §3.4): each request wastes < block_size slots of its last block;
    on the ragged batch-256 lengths the mean waste per request is close to (bs - 1) / 2, the page's
    bs / 2 estimate, measured from the C++ allocator's counters."""
    w = si.with_block_size(si.get("b256"), bs)
    r = pwl.replay(w)
    st = r.alloc.stats()
    S = w.num_seqs
    per_req = st["waste_tokens"] / S
    assert abs(per_req - (bs - 1) / 2) < 0.15 * bs
    _, t, lens = r.alloc.pack(np.arange(S), max(-(-n // bs) for n in w.decode_lens))
    waste = (t >= 0).sum(axis=1) * bs - lens
    assert (waste >= 0).all() and (waste < bs).all() and waste.sum() == st["waste_tokens"]


def test_stall_hook_arguments():
    lib = pk.lib()
    assert lib.pa_debug_inject_stall(3, 1000) == pk.PA_ERR_INVALID_ARG
    assert lib.pa_debug_inject_stall(pk.PA_KERNEL_DECODE, 0) == pk.PA_ERR_INVALID_ARG
    assert lib.pa_debug_inject_stall(pk.PA_KERNEL_PREFILL, 3_000_000_000) == pk.PA_ERR_INVALID_ARG


def test_pack_into_caller_arrays_matches_allocating_path():
    """pack(tables=, lens=) writes into the caller's (e.g. pinned staging) arrays exactly what the
    allocating form returns, -1 padding included; wrong dtypes, shapes, layouts and read-only views
    are refused before the C call can write through them."""
    a = pk.BlockAllocator(32, 4)
    for r, n in ((1, 9), (2, 1), (3, 16), (4, 0)):
        assert a.allocate(r, n) == pk.PA_OK
    reqs = [3, 1, 4, 2]
    st, t0, l0 = a.pack(reqs, 6)
    assert st == pk.PA_OK
    buf = np.full(4 * 6 + 4 + 3, 12345, dtype=np.int32)
    tv, lv = buf[:24].reshape(4, 6), buf[24:28]
    st, t1, l1 = a.pack(reqs, 6, tables=tv, lens=lv)
    assert st == pk.PA_OK and t1 is tv and l1 is lv
    assert np.array_equal(tv, t0) and np.array_equal(lv, l0)
    assert (tv[2] == -1).all() and tv[1, 3:].tolist() == [-1, -1, -1]
    assert buf[28:].tolist() == [12345] * 3                       # nothing written past the views
    with pytest.raises(ValueError):
        a.pack(reqs, 6, tables=np.zeros((4, 6), np.int64))
    with pytest.raises(ValueError):
        a.pack(reqs, 6, tables=np.zeros((4, 5), np.int32))
    with pytest.raises(ValueError):
        a.pack(reqs, 6, tables=np.zeros((6, 4), np.int32).T)
    with pytest.raises(ValueError):
        a.pack(reqs, 6, lens=np.broadcast_to(np.zeros(1, np.int32), (4,)))
    ro = np.zeros((4, 6), np.int32)
    ro.flags.writeable = False
    with pytest.raises(ValueError):
        a.pack(reqs, 6, tables=ro)
