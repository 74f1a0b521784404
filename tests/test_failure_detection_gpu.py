"""Device-side failure detection on the GPU, without faulting it.

Every wait inside the attention kernels is bounded.  pa_debug_inject_stall makes
the next launch's softmax role wait on a barrier that nothing completes, with
a 1 ms limit on that launch's pipeline waits: the wait runs out, the kernel
sets PA_DEVCHK_TIMEOUT, its other roles run out of their own waits and unwind
(copies and tensor-core work drain under the normal 2 s bound), and the launch
returns.  The context must stay usable: the next, normal launch matches the
oracle and reports no error.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_411_b200 as pk
import synth_inputs as si
from oracle import workloads as owl
from paged_kv_cache_411_b200 import workload as pwl

pytestmark = pytest.mark.gpu
TOL = 2e-3
LIMIT_NS = 1_000_000


def test_decode_wait_timeout_is_reported_and_recovered(cuda_ready):
    w = si.get("b32")
    ds = pwl.build(w)
    pk.reshape_and_cache(ds.k_step, ds.v_step, ds.k_cache, ds.v_cache, ds.slot_mapping)
    S, H, D = ds.q.shape
    ws = torch.empty(pk.decode_workspace_bytes(S, H, D, ds.max_blocks, w.block_size), dtype=torch.uint8,
                     device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(ds.q)
    assert pk.lib().pa_debug_inject_stall(pk.PA_KERNEL_DECODE, LIMIT_NS) == pk.PA_OK
    pk.paged_attention_decode(out, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.seq_lens, w.scale, ws,
                              err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pk.PA_DEVCHK_TIMEOUT
    # the context is intact and the hook was one-shot: a normal call matches the oracle
    err.zero_()
    out.fill_(float("nan"))
    pk.paged_attention_decode(out, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.seq_lens, w.scale, ws,
                              err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    dec, _, _, _ = owl.run_step(owl.build(w))
    assert float(np.abs(out.float().cpu().numpy() - dec).max()) <= TOL


def test_prefill_wait_timeout_is_reported_and_recovered(cuda_ready):
    w = si.Workload(name="timeout_prefill", seed=8, num_heads=4, head_dim=128, block_size=16, decode_lens=(),
                    pool_factor=1.2, prefill=si.PrefillSpec(ctx_before=300, chunk=500))
    ds = pwl.build(w)
    pk.reshape_and_cache(ds.k_step, ds.v_step, ds.k_cache, ds.v_cache, ds.slot_mapping)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(ds.prefill_q)

    def call():
        pk.paged_attention_prefill_chunk(out, ds.prefill_q, ds.k_cache, ds.v_cache, ds.prefill_table,
                                         ds.prefill_q_start, ds.prefill_ctx_before, w.scale, err_flag=err)
        torch.cuda.synchronize()
        return int(err.item())

    assert pk.lib().pa_debug_inject_stall(pk.PA_KERNEL_PREFILL, LIMIT_NS) == pk.PA_OK
    assert call() & pk.PA_DEVCHK_TIMEOUT
    err.zero_()
    out.fill_(float("nan"))
    assert call() == 0
    _, pre, _, _ = owl.run_step(owl.build(w))
    assert float(np.abs(out.float().cpu().numpy() - pre).max()) <= TOL
