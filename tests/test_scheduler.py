"""Continuous-batching step driver: the C++ scheduler against the oracle scheduler, plan for
plan, on seeded arrival traces (no GPU), plus hand-checked behaviours of the page's loop."""
import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

import paged_kv_cache_411_b200 as pk
from oracle import block_manager as obm
from oracle import scheduler as osch
from oracle.prefix_cache import PrefixCachingBlockManager


def _pair(N, bs, cpu_blocks=None, **cfg):
    ca = pk.BlockAllocator(N, bs)
    cs = pk.Scheduler(ca, **cfg)
    om = PrefixCachingBlockManager(N, bs)
    ocpu = None
    if cpu_blocks is not None:
        cs._keep_cpu = pk.BlockAllocator(cpu_blocks, bs)
        assert cs.enable_swap(cs._keep_cpu) == pk.PA_OK
        ocpu = obm.BlockManager(cpu_blocks, bs)
    os_ = osch.Scheduler(om, cfg["max_num_seqs"], cfg["max_num_tokens"], cfg.get("chunked_prefill", True),
                         cfg.get("watermark_blocks", 0), swap_cpu=ocpu)
    return ca, cs, om, os_


def _sampled(r, k):
    """The id a request emits as its k-th token (deterministic, from a small vocabulary)."""
    return (r * 7919 + k * 31) % 11


def _run(trace, N, bs, steps, cpu_blocks=None, prompts=None, **cfg):
    """trace: [(arrival_step, prompt_len, max_new)], request ids = index; prompts: token ids per request
    (prefix caching) or None."""
    ca, cs, om, os_ = _pair(N, bs, cpu_blocks, **cfg)
    pending = sorted(range(len(trace)), key=lambda i: trace[i][0])
    k = 0
    log = []
    for step in range(steps):
        while k < len(pending) and trace[pending[k]][0] <= step:
            i = pending[k]
            toks = None if prompts is None else prompts[i]
            assert cs.add_request(i, trace[i][1], trace[i][2], tokens=toks) == pk.PA_OK
            os_.add_request(i, trace[i][1], trace[i][2], tokens=toks)
            k += 1
        a = cs.step()
        b = os_.step()
        for key in ("num_prefill", "num_decode", "num_tokens", "num_admitted", "num_preempted", "num_finished"):
            assert a[key] == b[key], (step, key, a[key], b[key])
        assert [(int(r), int(c), int(n)) for r, c, n in zip(a["prefill_reqs"], a["prefill_ctx"], a["prefill_len"])] \
            == b["prefill"]
        assert [(int(r), int(n)) for r, n in zip(a["decode_reqs"], a["decode_seq_lens"])] == b["decode"]
        assert a["slot_mapping"].tolist() == b["slot_mapping"]
        if cpu_blocks is not None:
            assert a["swap_out"].tolist() == [list(x) for x in b["swap_out"]], step
            assert a["swap_in"].tolist() == [list(x) for x in b["swap_in"]], step
        if prompts is None:
            cs.complete()
            os_.complete()
        else:
            emit = [int(r) for r, c, n in b["prefill"] if os_.reqs[r].prefilled + n == os_.reqs[r].to_prefill]
            emit += [int(r) for r, _ in b["decode"]]
            ids = [_sampled(r, os_.reqs[r].generated) for r in emit]
            cs.complete(sampled=ids)
            os_.complete(sampled=ids)
            assert ca.cache_stats()["prefix_nodes"] == len(om.trie)
            assert ca.evictable_list().tolist() == list(om.lru)
        log.append(a)
    assert ca.free_list().tolist() == om.free_blocks
    assert cs.stats()["cached_tokens"] == os_.cached_tokens
    for i in range(len(trace)):
        st_, info = cs.request_info(i)
        if st_ == pk.PA_OK:
            q = os_.reqs[i]
            assert (info["state"], info["generated"], info["prefilled"], info["to_prefill"], info["preemptions"],
                    info["first_token_step"], info["finish_step"]) == \
                (q.state, q.generated, q.prefilled, q.to_prefill, q.preemptions, q.first_token_step, q.finish_step)
    return cs, os_, log


trace_st = st.lists(st.tuples(st.integers(0, 12), st.integers(1, 90), st.integers(1, 12)), min_size=1, max_size=14)


@settings(max_examples=200, deadline=None)
@given(trace_st, st.integers(4, 40), st.sampled_from([1, 4, 16]), st.integers(1, 6), st.integers(1, 64),
       st.booleans(), st.integers(0, 2))
def test_cpp_scheduler_matches_oracle(trace, N, bs, max_seqs, max_tokens, chunked, watermark):
    _run(trace, N, bs, 40, max_num_seqs=max_seqs, max_num_tokens=max_tokens, chunked_prefill=chunked,
         watermark_blocks=watermark)


@settings(max_examples=200, deadline=None)
@given(trace_st, st.integers(4, 40), st.integers(0, 30), st.sampled_from([1, 4, 16]), st.integers(1, 6),
       st.integers(1, 64), st.booleans(), st.integers(0, 2))
def test_cpp_swap_scheduler_matches_oracle(trace, N, ncpu, bs, max_seqs, max_tokens, chunked, watermark):
    """Swap preemption ([CB-PA] §5.4 strategy 2): plans, block moves and end states agree, including CPU
    pools too small to take a victim (recompute fallback)."""
    _run(trace, N, bs, 40, cpu_blocks=ncpu, max_num_seqs=max_seqs, max_num_tokens=max_tokens,
         chunked_prefill=chunked, watermark_blocks=watermark)


prefix_trace_st = st.lists(st.tuples(st.integers(0, 12), st.integers(0, 2), st.integers(0, 40), st.integers(1, 12)),
                          min_size=1, max_size=14)


@settings(max_examples=200, deadline=None)
@given(prefix_trace_st, st.integers(4, 40), st.sampled_from([1, 2, 4]), st.integers(1, 6), st.integers(1, 64),
       st.booleans(), st.integers(0, 2), st.sampled_from([None, 0, 12]))
def test_cpp_prefix_caching_scheduler_matches_oracle(trace, N, bs, max_seqs, max_tokens, chunked, watermark, ncpu):
    """Requests with token ids ([CB-PA] §4.2 in the §2.2 loop): prompts share family prefixes, emitted
    ids are reported each step; plans, cached-token counts, the LRU and the trie agree, with recompute
    or swap preemption."""
    prompts = [[fam * 100 + (i % 9) for i in range(12)] + [(r * 13 + i) % 17 for i in range(tail)]
               for r, (_, fam, tail, _) in enumerate(trace)]
    t = [(arr, len(prompts[r]), new) for r, (arr, _, _, new) in enumerate(trace)]
    _run(t, N, bs, 40, cpu_blocks=ncpu, prompts=prompts, max_num_seqs=max_seqs, max_num_tokens=max_tokens,
         chunked_prefill=chunked, watermark_blocks=watermark)


def test_shared_prompt_is_prefilled_once():
    """Three requests with one 32-token system prompt, arriving one step apart: the second and third
    find its blocks in the cache and prefill only their own tails; a recomputed request after preemption
    finds its own blocks again."""
    system = list(range(100, 132))
    prompts = [system + [1, 2, 3], system + [4, 5], system + [6] * 9]
    cs, os_, log = _run([(0, 35, 3), (1, 34, 3), (2, 41, 3)], 64, 8, 20, prompts=prompts, max_num_seqs=4,
                        max_num_tokens=64)
    assert os_.cached_tokens == 64 and cs.stats()["cached_tokens"] == 64
    assert [int(x) for x in log[1]["prefill_ctx"]] == [32] and [int(x) for x in log[2]["prefill_ctx"]] == [32]


def test_swap_preemption_keeps_progress():
    """A pool too small for two long generations, with a CPU pool: the newer request is swapped out and
    back instead of recomputed, every request finishes, and nothing stays on the CPU."""
    cs, os_, log = _run([(0, 16, 40), (0, 16, 40)], 10, 8, 200, cpu_blocks=8, max_num_seqs=2, max_num_tokens=64)
    st = cs.stats()
    assert st["swap_outs"] >= 1 and st["swap_ins"] == st["swap_outs"] and st["swapped"] == 0
    assert os_.reqs[1].to_prefill == 16 and os_.reqs[1].preemptions >= 1     # nothing recomputed
    assert cs._keep_cpu.stats()["num_free"] == 8


def test_seeded_trace_serves_everything():
    """A seeded trace (lognormal prompt/output lengths, Poisson arrivals) on a pool large enough:
    every request finishes, each emits exactly max_new tokens, and prefill/decode mix in steps."""
    rng = np.random.default_rng(4)
    n = 40
    arrivals = np.cumsum(rng.poisson(0.7, n))
    prompts = np.clip(rng.lognormal(4.0, 0.8, n).astype(int), 1, 600)
    outs = np.clip(rng.lognormal(3.0, 0.7, n).astype(int), 1, 120)
    trace = list(zip(arrivals.tolist(), prompts.tolist(), outs.tolist()))
    cs, os_, log = _run(trace, 400, 16, 400, max_num_seqs=16, max_num_tokens=256)
    stats = cs.stats()
    assert stats["finished"] == n and stats["decode_tokens"] + n == int(outs.sum())
    assert any(s["num_prefill"] and s["num_decode"] for s in log)      # mixed steps ([CB-PA] §2.2)
    assert all(s["num_tokens"] - s["num_decode"] <= 256 for s in log)   # prefill budget


def test_preemption_recomputes_newest_first():
    """A pool too small for two long generations: the newer request is preempted, goes back to the
    front of the waiting queue, and later recomputes its prompt plus what it had generated."""
    cs, os_, log = _run([(0, 16, 40), (0, 16, 40)], 10, 8, 200, max_num_seqs=2, max_num_tokens=64)
    assert sum(s["num_preempted"] for s in log) >= 1
    q = os_.reqs[1]
    assert q.preemptions >= 1 and q.state == osch.FINISHED and os_.reqs[0].state == osch.FINISHED
    assert q.to_prefill > 16                                              # prompt + generated tokens


def test_whole_prompt_mode_skips_prompts_that_do_not_fit():
    cs, os_, log = _run([(0, 100, 2), (0, 10, 2)], 64, 16, 10, max_num_seqs=4, max_num_tokens=64,
                        chunked_prefill=False)
    first = log[0]
    assert first["prefill_reqs"].tolist() == [1]      # the 100-token prompt never fits a 64-token budget
    assert os_.reqs[0].prefilled == 0


def test_scheduler_errors():
    a = pk.BlockAllocator(8, 16)
    s = pk.Scheduler(a, max_num_seqs=2, max_num_tokens=32)
    assert s.add_request(1, 0, 5) == pk.PA_ERR_INVALID_ARG
    assert s.add_request(1, 5, 5) == pk.PA_OK
    assert s.add_request(1, 5, 5) == pk.PA_ERR_EXISTS
    s.step()
    with pytest.raises(pk.PagedKVError):
        s.step()                                        # previous step not completed
    s.complete()
    with pytest.raises(pk.PagedKVError):
        s.complete()
    with pytest.raises(pk.PagedKVError):
        pk.Scheduler(a, max_num_seqs=0, max_num_tokens=32)


def test_step_results_are_the_callers_own():
    """The binding reuses its output buffers between steps; what a step returns must not change when
    the next step runs or when the caller writes into it."""
    alloc = pk.BlockAllocator(64, 16)
    sched = pk.Scheduler(alloc, max_num_seqs=4, max_num_tokens=64)
    sched.add_request(1, 40, 3)
    sched.add_request(2, 10, 2)
    first = sched.step()
    kept = {k: v.copy() for k, v in first.items() if isinstance(v, np.ndarray)}
    sched.complete()
    second = sched.step()
    for k, v in kept.items():
        assert np.array_equal(first[k], v), k
    first["slot_mapping"][:] = -7
    assert not np.any(second["slot_mapping"] == -7)
