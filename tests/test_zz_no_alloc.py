"""The no-allocation decode entry point against the workspace one (GPU).

pa_paged_attention_decode_noalloc serves callers that cannot call cudaMalloc
(they were handed fixed buffers, or their host forbids allocation after
start-up): it takes its scratch from a fixed array the library keeps in device
memory.  Called twice in a row through the C ABI, it must give what
pa_paged_attention_decode gives with a caller workspace, and it must refuse a
batch whose scratch would not fit.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_411_b200 as pk
import synth_inputs as si
from paged_kv_cache_411_b200 import workload as pwl

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_decode_twice(cuda_ready):
    """Shapes in decreasing order (the 64-sequence mixed decode set, then 32 sequences of 32 heads x
    128, then the tiny set with head_dim 64), two calls each: a call that follows a larger one must
    not pick up the header, items or partials the larger one left in the shared scratch.  The
    kernels are deterministic and the workspace path runs the same kernels, so the outputs must be
    bitwise equal."""
    lib = pk.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for name in ("mixed", "b32", "tiny"):
        w = si.get(name)
        ds = pwl.build(w)
        pk.reshape_and_cache(ds.k_step, ds.v_step, ds.k_cache, ds.v_cache, ds.slot_mapping)
        S, H, D = ds.q.shape
        mb = ds.block_tables.shape[1]
        ws = torch.empty(pk.decode_workspace_bytes(S, H, D, mb, w.block_size), dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(ds.q)
        pk.paged_attention_decode(ref, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.seq_lens, w.scale, ws)
        for call in range(2):
            out = torch.full_like(ds.q, float("nan"))
            st = lib.pa_paged_attention_decode_noalloc(
                _p(out), _p(ds.q), _p(ds.k_cache), _p(ds.v_cache), _p(ds.block_tables), _p(ds.seq_lens),
                S, H, D, w.block_size, mb, ds.num_blocks, ctypes.c_float(w.scale), _p(err), stream)
            assert st == pk.PA_OK, pk.last_error()
            torch.cuda.synchronize()
            assert int(err.item()) == 0
            assert torch.equal(out, ref), f"{name} call {call}: max abs difference " \
                f"{(out.float() - ref.float()).abs().max().item()}"


def test_noalloc_rejects_batches_beyond_its_scratch(cuda_ready):
    S, H, D, bs, mb = 256, 32, 128, 16, 256
    assert pk.decode_workspace_bytes(S, H, D, mb, bs) > 64 * 2**20
    q = torch.zeros(S, H, D, dtype=torch.float16, device="cuda")
    kc = torch.zeros(mb, bs, H, D, dtype=torch.float16, device="cuda")
    tables = torch.zeros(S, mb, dtype=torch.int32, device="cuda")
    lens = torch.ones(S, dtype=torch.int32, device="cuda")
    st = pk.lib().pa_paged_attention_decode_noalloc(
        _p(q), _p(q), _p(kc), _p(kc), _p(tables), _p(lens), S, H, D, bs, mb, mb, ctypes.c_float(0.1), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pk.PA_ERR_INVALID_ARG
    assert "static scratch" in pk.last_error()
