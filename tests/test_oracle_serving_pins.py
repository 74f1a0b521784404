"""Pins of the serving-side oracles against hand traces of the pages (no GPU).

The step driver (``oracle.scheduler``) is run through the page's own
continuous-batching timeline, a preemption trace and three watermark cases
(``tests/golden/scheduler_traces.json``), and the swap manager
(``oracle.swap``) through a hand-traced sequence of moves between a GPU and a
CPU pool (``tests/golden/swap_trace.json``).  Every expected number in those
files was worked out by hand from the cited passages; none comes from running
the oracle or the library.  The C++ scheduler and swap bookkeeping are run
through the same traces.
"""
import numpy as np
import pytest

import paged_kv_cache_411_b200 as pk
from conftest import golden
from oracle import block_manager as obm
from oracle import scheduler as osch
from oracle import swap as oswap
from oracle.prefix_cache import PrefixCachingBlockManager

_CASES = golden("scheduler_traces.json")["cases"]
_NAMES = {pk.PA_OK: obm.OK, pk.PA_ERR_OOM: obm.OOM, pk.PA_ERR_NOT_FOUND: obm.NOT_FOUND,
          pk.PA_ERR_EXISTS: obm.EXISTS, pk.PA_ERR_INVALID_ARG: obm.INVALID_ARG}


def _case(name):
    return next(c for c in _CASES if c["name"] == name)


def run_oracle_scheduler_trace(case):
    """Replays one golden case through the oracle scheduler and checks every step and the end state."""
    cfg = case["config"]
    bm = PrefixCachingBlockManager(cfg["num_blocks"], cfg["block_size"])
    cpu = obm.BlockManager(cfg["swap_cpu_blocks"], cfg["block_size"]) if "swap_cpu_blocks" in cfg else None
    sched = osch.Scheduler(bm, cfg["max_num_seqs"], cfg["max_num_tokens"], cfg["chunked_prefill"],
                           cfg["watermark_blocks"], swap_cpu=cpu)
    for i, want in enumerate(case["steps"]):
        for r in case["requests"]:
            if r["arrival"] == i:
                sched.add_request(r["id"], r["prompt"], r["max_new"])
        got = sched.step()
        assert got["num_finished"] == want["finished"], (case["name"], i, "finished")
        assert got["num_preempted"] == want["preempted"], (case["name"], i, "preempted")
        assert got["num_admitted"] == want["admitted"], (case["name"], i, "admitted")
        assert [list(p) for p in got["prefill"]] == want["prefill"], (case["name"], i, "prefill")
        assert [list(d) for d in got["decode"]] == want["decode"], (case["name"], i, "decode")
        assert got["slot_mapping"] == want["slot_mapping"], (case["name"], i, "slots")
        if "swap_out" in want:
            assert [list(x) for x in got["swap_out"]] == want["swap_out"], (case["name"], i, "swap_out")
            assert [list(x) for x in got["swap_in"]] == want["swap_in"], (case["name"], i, "swap_in")
        sched.complete()
    fin = case["final"]
    assert bm.free_blocks == fin["free_list"]
    if cpu is not None:
        assert cpu.free_blocks == fin["cpu_free_list"]
    assert {str(r): t for r, t in bm.block_tables.items()} == fin["tables"]
    for rid, want in fin["requests"].items():
        q = sched.reqs[int(rid)]
        got = {"state": q.state, "generated": q.generated, "first_token_step": q.first_token_step,
               "finish_step": q.finish_step, "preemptions": q.preemptions, "to_prefill": q.to_prefill}
        assert {k: got[k] for k in want} == want, (case["name"], rid)


@pytest.mark.parametrize("name", [c["name"] for c in _CASES])
def test_oracle_scheduler_follows_hand_trace(name):
    run_oracle_scheduler_trace(_case(name))


@pytest.mark.parametrize("name", [c["name"] for c in _CASES])
def test_cpp_scheduler_follows_hand_trace(name):
    case = _case(name)
    cfg = case["config"]
    alloc = pk.BlockAllocator(cfg["num_blocks"], cfg["block_size"])
    sched = pk.Scheduler(alloc, max_num_seqs=cfg["max_num_seqs"], max_num_tokens=cfg["max_num_tokens"],
                         chunked_prefill=cfg["chunked_prefill"], watermark_blocks=cfg["watermark_blocks"])
    cpu = None
    if "swap_cpu_blocks" in cfg:
        cpu = pk.BlockAllocator(cfg["swap_cpu_blocks"], cfg["block_size"])
        assert sched.enable_swap(cpu) == pk.PA_OK
    for i, want in enumerate(case["steps"]):
        for r in case["requests"]:
            if r["arrival"] == i:
                assert sched.add_request(r["id"], r["prompt"], r["max_new"]) == pk.PA_OK
        got = sched.step()
        assert (got["num_finished"], got["num_preempted"], got["num_admitted"]) == \
            (want["finished"], want["preempted"], want["admitted"]), (name, i)
        assert [[int(a), int(b), int(c)] for a, b, c in
                zip(got["prefill_reqs"], got["prefill_ctx"], got["prefill_len"])] == want["prefill"], (name, i)
        assert [[int(a), int(b)] for a, b in zip(got["decode_reqs"], got["decode_seq_lens"])] == want["decode"]
        assert got["slot_mapping"].tolist() == want["slot_mapping"], (name, i)
        if "swap_out" in want:
            assert got["swap_out"].tolist() == want["swap_out"] and got["swap_in"].tolist() == want["swap_in"], (name, i)
        sched.complete()
    fin = case["final"]
    assert alloc.free_list().tolist() == fin["free_list"]
    if cpu is not None:
        assert cpu.free_list().tolist() == fin["cpu_free_list"]
    for rid, t in fin["tables"].items():
        assert alloc.get_block_table(int(rid))[1].tolist() == t
    for rid, want in fin["requests"].items():
        st, info = sched.request_info(int(rid))
        assert st == pk.PA_OK
        assert {k: int(info[k]) for k in want} == want, (name, rid)


# ------------------------------------------------------------------ swap (§4.4)
def _tag_pools(n, bs, tags):
    """K pool whose block b holds tags[b] everywhere, and a V pool holding 100 + tags[b]."""
    k = np.empty((n, bs, 1, 2), np.float64)
    for b, t in enumerate(tags):
        k[b] = t
    return k, k + 100.0


def _tags_of(k, v):
    """The tag each block holds (asserting it is uniform and that V carries the same block)."""
    out = []
    for b in range(k.shape[0]):
        t = k[b].flat[0]
        assert np.all(k[b] == t) and np.all(v[b] == t + 100.0), b
        out.append(int(t))
    return out


def run_oracle_swap_trace():
    g = golden("swap_trace.json")
    bs = g["block_size"]
    gpu = obm.BlockManager(g["gpu_blocks"], bs)
    cpu = obm.BlockManager(g["cpu_blocks"], bs, g["cpu_free_order"])
    sm = oswap.SwappingManager(gpu, cpu)
    gk, gv = _tag_pools(g["gpu_blocks"], bs, range(g["gpu_blocks"]))
    ck, cv = _tag_pools(g["cpu_blocks"], bs, [-1] * g["cpu_blocks"])
    for op in g["ops"]:
        kind = op["op"]
        if kind == "gpu_allocate":
            st = gpu.allocate(op["req"], op["tokens"])
        elif kind == "gpu_fork":
            st = gpu.fork(op["src"], op["dst"], op["prefix"])
        elif kind == "swap_out":
            st = sm.swap_out(op["req"], gk, gv, ck, cv)
        else:
            st = sm.swap_in(op["req"], gk, gv, ck, cv)
        assert st == op["status"], op
        if "gpu_free" in op:
            assert gpu.free_blocks == op["gpu_free"], op["why"]
            assert cpu.free_blocks == op["cpu_free"], op["why"]
            assert {str(r): t for r, t in gpu.block_tables.items()} == op["gpu_tables"], op["why"]
            assert {str(r): t for r, t in cpu.block_tables.items()} == op["cpu_tables"], op["why"]
            for r, n in op.get("cpu_seq_lens", {}).items():
                assert cpu.seq_lens[int(r)] == n, op["why"]
            for r, n in op.get("gpu_seq_lens", {}).items():
                assert gpu.seq_lens[int(r)] == n, op["why"]
            assert gpu.refcount == op["gpu_refcount"], op["why"]
            assert _tags_of(gk, gv) == op["gpu_tags"], op["why"]
            assert _tags_of(ck, cv) == op["cpu_tags"], op["why"]


def test_oracle_swap_follows_hand_trace():
    run_oracle_swap_trace()


def test_cpp_swap_bookkeeping_follows_hand_trace():
    """The C++ moves on the same trace with block_bytes 0 (bookkeeping only; the data moves are
    checked against the oracle on the GPU)."""
    g = golden("swap_trace.json")
    bs = g["block_size"]
    gpu = pk.BlockAllocator(g["gpu_blocks"], bs)
    cpu = pk.BlockAllocator(g["cpu_blocks"], bs, free_order=g["cpu_free_order"])
    for op in g["ops"]:
        kind = op["op"]
        if kind == "gpu_allocate":
            st = gpu.allocate(op["req"], op["tokens"])
        elif kind == "gpu_fork":
            st = gpu.fork(op["src"], op["dst"], op["prefix"])
        elif kind == "swap_out":
            st = pk.swap_out(gpu, cpu, op["req"], None, None, None, None, 0)
        else:
            st = pk.swap_in(gpu, cpu, op["req"], None, None, None, None, 0)
        assert _NAMES[st] == op["status"], op
        if "gpu_free" in op:
            assert gpu.free_list().tolist() == op["gpu_free"], op["why"]
            assert cpu.free_list().tolist() == op["cpu_free"], op["why"]
            for tables, a in ((op["gpu_tables"], gpu), (op["cpu_tables"], cpu)):
                for r, t in tables.items():
                    assert a.get_block_table(int(r))[1].tolist() == t, op["why"]
            for r, n in op.get("cpu_seq_lens", {}).items():
                assert cpu.seq_len(int(r))[1] == n
            assert [gpu.refcount(b)[1] for b in range(g["gpu_blocks"])] == op["gpu_refcount"]
