"""The continuous-batching step driver running the kernels (GPU).

The C++ scheduler plans every step of a seeded arrival trace (mixed prefill
chunks and decodes, preemption by recomputation -- or by swapping to a host
pool -- under a small pool); each
step writes its rows with reshape_and_cache and runs the prefill and decode
kernels on the planned tables.  Every output row is checked against the
float64 oracle's attention over the request's logical K/V (a recomputed
position gets the same K/V, as recomputation would give)."""
import zlib

import numpy as np
import pytest
import torch

import paged_kv_cache_411_b200 as pk
from oracle import attention as oatt

pytestmark = pytest.mark.gpu
TOL = 2e-3


def test_scheduler_drives_kernels(cuda_ready):
    _serve(swap=False)


def test_scheduler_with_swap_preemption_drives_kernels(cuda_ready):
    """[CB-PA] §5.4 strategy 2: preempted requests move to a pinned host pool and back.  Each step the
    block moves the scheduler reports run first (GPU to host, then host to GPU, pa_swap_blocks on the
    stream), then the step's kernels.  A swapped-in request's blocks hold its K/V bit for bit, it is
    never recomputed, and every output row matches the oracle."""
    _serve(swap=True)


def test_scheduler_with_prefix_caching_drives_kernels(cuda_ready):
    """[CB-PA] §4.2 inside the §2.2 loop: requests share three system prompts and report the ids they
    generate.  A token's K/V is a function of its whole token prefix (as a model's would be), so a cached
    block serves every request whose prefix matches; admission skips the cached tokens, and every output
    row still matches the oracle over each request's own logical K/V."""
    _serve(swap=False, prefix=True)


class _PrefixKV:
    """Logical K (or V) rows of one request whose row p depends only on its token ids 0..p."""

    def __init__(self, toks, H, D, salt):
        self.toks, self.H, self.D, self.salt = toks, H, D, salt
        self.rows = {}

    def row(self, p):
        key = zlib.crc32(np.asarray(self.toks[:p + 1], np.int32).tobytes())
        if (p, key) not in self.rows:
            g = np.random.default_rng([self.salt, p, key])
            self.rows[(p, key)] = g.standard_normal((self.H, self.D)).astype(np.float16)
        return self.rows[(p, key)]

    def __getitem__(self, idx):
        if isinstance(idx, slice):
            return np.stack([self.row(p) for p in range(*idx.indices(len(self.toks)))])
        return self.row(idx)


def _serve(swap, prefix=False):
    H, D, bs, N = 4, 128, 16, 14            # a pool that forces preemptions
    scale = 1 / np.sqrt(D)
    rng = np.random.default_rng(30)
    n = 10
    prompts = rng.integers(5, 150, n)
    outs = rng.integers(2, 24, n)
    arrivals = np.sort(rng.integers(0, 6, n))
    toks = None
    if prefix:
        systems = [rng.integers(0, 1000, int(m)).tolist() for m in (40, 57, 64)]
        toks = [systems[r % 3] + rng.integers(0, 1000, int(rng.integers(1, 40))).tolist() for r in range(n)]
        prompts = np.asarray([len(t) for t in toks])
    maxlen = int((prompts + outs).max()) + 1
    if prefix:
        K = {r: _PrefixKV(toks[r], H, D, 1) for r in range(n)}
        V = {r: _PrefixKV(toks[r], H, D, 2) for r in range(n)}
    else:
        K = {r: rng.standard_normal((maxlen, H, D)).astype(np.float16) for r in range(n)}
        V = {r: rng.standard_normal((maxlen, H, D)).astype(np.float16) for r in range(n)}
    alloc = pk.BlockAllocator(N, bs)
    sched = pk.Scheduler(alloc, max_num_seqs=6, max_num_tokens=64)
    kc = torch.full((N, bs, H, D), float("nan"), dtype=torch.float16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    NC = 40
    block_bytes = bs * H * D * 2
    if swap:
        cpu = pk.BlockAllocator(NC, bs)
        assert sched.enable_swap(cpu) == pk.PA_OK
        ck = torch.full((NC, bs, H, D), float("nan"), dtype=torch.float16).pin_memory()
        cv = torch.full_like(ck, float("nan")).pin_memory()
    swapped_in = 0
    mb = -(-maxlen // bs)
    ws = torch.empty(pk.decode_workspace_bytes(6, H, D, mb, bs), dtype=torch.uint8, device="cuda")
    added, checked_rows, preempted, mixed = 0, 0, 0, 0
    for step in range(400):
        while added < n and arrivals[added] <= step:
            assert sched.add_request(added, int(prompts[added]), int(outs[added]),
                                     tokens=None if toks is None else list(toks[added])) == pk.PA_OK
            added += 1
        plan = sched.step()
        preempted += plan["num_preempted"]
        emitted = []                                        # requests emitting a token this step, in order
        for r, c, L in zip(plan["prefill_reqs"], plan["prefill_ctx"], plan["prefill_len"]):
            info = sched.request_info(int(r))[1]
            if int(c) + int(L) == info["to_prefill"]:
                emitted.append(int(r))
        emitted += [int(r) for r in plan["decode_reqs"]]

        def complete():
            if toks is None:
                sched.complete()
                return
            ids = [int(rng.integers(0, 1000)) for _ in emitted]
            sched.complete(sampled=ids)
            for r, t in zip(emitted, ids):
                toks[r].append(t)
        if swap:
            if len(plan["swap_out"]):
                pk.swap_blocks(kc, vc, ck, cv, plan["swap_out"], block_bytes, N, NC)
            if len(plan["swap_in"]):
                pk.swap_blocks(ck, cv, kc, vc, plan["swap_in"], block_bytes, NC, N)
                torch.cuda.synchronize()
                moved = {int(b) for b in plan["swap_in"][:, 1]}
                for r in range(n):
                    st, t = alloc.get_block_table(r)
                    if st != pk.PA_OK or not moved & set(t.tolist()):
                        continue
                    # positions already cached: the step's own rows (a decode token, a chunk) come later
                    n_kv = alloc.seq_len(r)[1] - int((plan["decode_reqs"] == r).sum()) \
                        - int(plan["prefill_len"][plan["prefill_reqs"] == r].sum())
                    idx = np.arange(n_kv)
                    got_k = kc[torch.from_numpy(t[idx // bs]).cuda(), torch.from_numpy(idx % bs).cuda()]
                    got_v = vc[torch.from_numpy(t[idx // bs]).cuda(), torch.from_numpy(idx % bs).cuda()]
                    assert np.array_equal(got_k.cpu().numpy().view(np.int16), K[r][:n_kv].view(np.int16)), r
                    assert np.array_equal(got_v.cpu().numpy().view(np.int16), V[r][:n_kv].view(np.int16)), r
                    swapped_in += 1
        if plan["num_tokens"] == 0:
            complete()
            if sched.stats()["finished"] == n:
                break
            continue
        mixed += bool(plan["num_prefill"] and plan["num_decode"])
        rows = []                                           # (request, position) of each slot-mapping row
        for r, c, L in zip(plan["prefill_reqs"], plan["prefill_ctx"], plan["prefill_len"]):
            rows += [(int(r), p) for p in range(int(c), int(c) + int(L))]
        for r, sl in zip(plan["decode_reqs"], plan["decode_seq_lens"]):
            rows.append((int(r), int(sl) - 1))
        k_rows = np.stack([K[r][p] for r, p in rows])
        v_rows = np.stack([V[r][p] for r, p in rows])
        pk.reshape_and_cache(torch.from_numpy(k_rows).cuda(), torch.from_numpy(v_rows).cuda(), kc, vc,
                             torch.from_numpy(plan["slot_mapping"]).cuda())
        P, S = plan["num_prefill"], plan["num_decode"]
        if P:
            T = int(plan["prefill_len"].sum())
            qp = rng.standard_normal((T, H, D)).astype(np.float16)
            st, tables, _ = alloc.pack(plan["prefill_reqs"], mb)
            assert st == pk.PA_OK
            q_start = np.concatenate([[0], np.cumsum(plan["prefill_len"])]).astype(np.int32)
            out = torch.empty(T, H, D, dtype=torch.float16, device="cuda")
            pk.paged_attention_prefill_chunk(out, torch.from_numpy(qp).cuda(), kc, vc, torch.from_numpy(tables).cuda(),
                                             torch.from_numpy(q_start).cuda(),
                                             torch.from_numpy(plan["prefill_ctx"]).cuda(), scale)
            got = out.float().cpu().numpy()
            for i, (r, c, L) in enumerate(zip(plan["prefill_reqs"], plan["prefill_ctx"], plan["prefill_len"])):
                r, c, L = int(r), int(c), int(L)
                allowed = np.arange(c + L)[None, :] <= (c + np.arange(L))[:, None]
                ref = oatt.softmax_attention(qp[q_start[i]:q_start[i + 1]], K[r][:c + L], V[r][:c + L], scale, allowed)
                assert np.abs(got[q_start[i]:q_start[i + 1]] - ref).max() <= TOL, (step, r)
                checked_rows += L
        if S:
            qd = rng.standard_normal((S, H, D)).astype(np.float16)
            st, tables, lens = alloc.pack(plan["decode_reqs"], mb)
            assert st == pk.PA_OK and lens.tolist() == plan["decode_seq_lens"].tolist()
            out = torch.empty(S, H, D, dtype=torch.float16, device="cuda")
            pk.paged_attention_decode(out, torch.from_numpy(qd).cuda(), kc, vc, torch.from_numpy(tables).cuda(),
                                      torch.from_numpy(lens).cuda(), scale, ws)
            got = out.float().cpu().numpy()
            for i, (r, sl) in enumerate(zip(plan["decode_reqs"], plan["decode_seq_lens"])):
                r, sl = int(r), int(sl)
                ref = oatt.softmax_attention(qd[i][None], K[r][:sl], V[r][:sl], scale)[0]
                assert np.abs(got[i] - ref).max() <= TOL, (step, r)
                checked_rows += 1
        complete()
        if sched.stats()["finished"] == n:
            break
    stats = sched.stats()
    assert stats["finished"] == n and preempted > 0 and mixed > 0 and checked_rows > 500
    for r in range(n):
        st, info = sched.request_info(r)
        assert info["generated"] == outs[r]
    if prefix:
        assert stats["cached_tokens"] > 0 and alloc.cache_stats()["hit_blocks"] > 0
    if swap:
        assert stats["swap_outs"] > 0 and stats["swap_ins"] == stats["swap_outs"] and swapped_in > 0
        assert stats["prefill_tokens"] == int(prompts.sum())      # nothing was recomputed
        assert cpu.stats()["num_free"] == NC
