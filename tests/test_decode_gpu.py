"""GPU parity of reshape_and_cache and paged decode against the CPU oracle.

Inputs come from the same seeded recipes on both sides; the CUDA side builds
its step through the C++ allocator and the library's kernels, the oracle
through its own block manager and NumPy.  Cache writes must match bit for bit;
attention outputs within 2e-3 absolute (fp16 in, fp32 accumulate, fp16 out).
"""
import dataclasses

import numpy as np
import pytest
import torch

import paged_kv_cache_411_b200 as pk
import synth_inputs as si
from oracle import attention as oatt
from oracle import workloads as owl
from paged_kv_cache_411_b200 import workload as pwl

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _bits(a):
    return np.asarray(a).view(np.int16)


def _run_decode(ds, out=None, workspace=None, err=None):
    w = ds.workload
    S, H, D = ds.q.shape
    if out is None:
        out = torch.full_like(ds.q, float("nan"))
    if workspace is None:
        nbytes = pk.decode_workspace_bytes(S, H, D, ds.block_tables.shape[1], w.block_size)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    pk.paged_attention_decode(out, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.seq_lens, w.scale,
                              workspace, err_flag=err)
    return out


def _step(ds, err=None):
    pk.reshape_and_cache(ds.k_step, ds.v_step, ds.k_cache, ds.v_cache, ds.slot_mapping, err_flag=err)
    return _run_decode(ds, err=err)


def _custom(name, seed, H, D, bs, lens, pool_factor=1.3, **kw):
    return si.Workload(name=name, seed=seed, num_heads=H, head_dim=D, block_size=bs, decode_lens=tuple(lens),
                       pool_factor=pool_factor, **kw)


def _check_decode(w, pad="neg1"):
    ds = pwl.build(w, pad=pad)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _step(ds, err).float().cpu().numpy()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    o = owl.build(w)
    dec, _, kc, vc = owl.run_step(o)
    # the whole pool, context and step rows, bit-exact (NaN poison included)
    assert np.array_equal(_bits(ds.k_cache.cpu().numpy()), _bits(kc))
    assert np.array_equal(_bits(ds.v_cache.cpu().numpy()), _bits(vc))
    assert np.isfinite(out).all()
    diff = np.abs(out - dec)
    assert diff.max() <= TOL, f"max abs error {diff.max():.3g}"
    return ds, out, dec


@pytest.mark.parametrize("name", ["tiny", "b32"])
def test_decode_workloads_match_oracle(cuda_ready, name):
    _check_decode(si.get(name))


def test_mixed_workload_decode_part(cuda_ready):
    """The mixed step's 576-row reshape and its 64-sequence decode."""
    w = si.get("mixed")
    ds = pwl.build(w)
    out = _step(ds).float().cpu().numpy()
    o = owl.build(w)
    dec, _, kc, vc = owl.run_step(o)
    assert np.array_equal(_bits(ds.k_cache.cpu().numpy()), _bits(kc))
    assert np.array_equal(_bits(ds.v_cache.cpu().numpy()), _bits(vc))
    assert np.abs(out - dec).max() <= TOL


SHAPES = [
    # (H, D, bs, lens): ragged tails, block and stage boundaries, several partitions
    (4, 64, 16, [1, 2, 15, 16, 17, 31, 32, 33, 100]),
    (8, 64, 16, [5, 64, 65, 300, 1023]),
    (32, 128, 16, [1, 17, 129, 700, 2049]),
    (8, 128, 8, [1, 7, 8, 9, 250, 1500]),
    (8, 128, 32, [31, 32, 33, 1000, 5000]),
    (4, 128, 64, [63, 64, 65, 777]),
    (2, 128, 16, [3, 90, 513]),
    (12, 128, 48, [47, 48, 49, 960]),
    (16, 64, 8, [9, 400]),
]


@pytest.mark.parametrize("H,D,bs,lens", SHAPES)
def test_decode_shapes_match_oracle(cuda_ready, H, D, bs, lens):
    _check_decode(_custom(f"shape_{H}_{D}_{bs}", 7, H, D, bs, lens))


def test_many_sequences_ragged(cuda_ready):
    rng = np.random.default_rng(11)
    lens = rng.integers(1, 600, size=300).tolist()
    _check_decode(_custom("many", 9, 8, 128, 16, lens))


def test_padding_is_never_read(cuda_ready):
    """Block-table entries past ceil(seq_len / bs) hold wrong but valid block ids: same output."""
    w = _custom("pad", 5, 8, 128, 16, [3, 40, 17, 250])
    a = pwl.build(w, pad="neg1", max_blocks=40)
    b = pwl.build(w, pad="garbage", max_blocks=40)
    assert (b.block_tables.cpu().numpy() >= 0).all()
    oa, ob = _step(a), _step(b)
    assert torch.equal(oa, ob)


def test_invariant_under_physical_block_permutation(cuda_ready):
    w = _custom("perm", 6, 8, 128, 16, [33, 1, 700, 129, 64])
    ds = pwl.build(w)
    base = _step(ds).clone()
    N = ds.num_blocks
    for seed in range(3):
        perm = torch.from_numpy(np.random.default_rng(seed).permutation(N)).cuda()
        k2 = torch.empty_like(ds.k_cache)
        v2 = torch.empty_like(ds.v_cache)
        k2[perm] = ds.k_cache
        v2[perm] = ds.v_cache
        t = ds.block_tables.long()
        t2 = torch.where(t >= 0, perm[t.clamp(min=0)], t).int()
        ds2 = dataclasses.replace(ds, k_cache=k2, v_cache=v2, block_tables=t2.contiguous())
        assert torch.equal(_run_decode(ds2), base)


def test_repeated_calls_reuse_workspace(cuda_ready):
    w = _custom("repeat", 8, 8, 128, 16, [100, 2000, 5])
    ds = pwl.build(w)
    pk.reshape_and_cache(ds.k_step, ds.v_step, ds.k_cache, ds.v_cache, ds.slot_mapping)
    S, H, D = ds.q.shape
    ws = torch.empty(pk.decode_workspace_bytes(S, H, D, ds.max_blocks, w.block_size), dtype=torch.uint8, device="cuda")
    ws.fill_(0xAB)
    a = _run_decode(ds, workspace=ws).clone()
    b = _run_decode(ds, workspace=ws)
    assert torch.equal(a, b)


def test_empty_and_single_token_sequences(cuda_ready):
    """seq_len 0 gives zeros; seq_len 1 gives that token's V (rounded to fp16: exact)."""
    H, D, bs = 8, 128, 16
    kc = torch.randn(4, bs, H, D, device="cuda").half()
    vc = torch.randn(4, bs, H, D, device="cuda").half()
    q = torch.randn(3, H, D, device="cuda").half()
    tables = torch.tensor([[2, -1], [1, -1], [3, 0]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([0, 1, 20], dtype=torch.int32, device="cuda")
    out = torch.full_like(q, float("nan"))
    ws = torch.empty(pk.decode_workspace_bytes(3, H, D, 2, bs), dtype=torch.uint8, device="cuda")
    pk.paged_attention_decode(out, q, kc, vc, tables, lens, 0.088, ws)
    assert torch.equal(out[0], torch.zeros_like(out[0]))
    assert torch.equal(out[1], vc[1, 0])
    ref = oatt.paged_attention_decode(q.cpu().numpy(), kc.cpu().numpy(), vc.cpu().numpy(),
                                      tables.cpu().numpy(), [0, 1, 20], bs, 0.088)
    assert np.abs(out.float().cpu().numpy() - ref).max() <= TOL


def test_device_checks_flag_and_skip(cuda_ready):
    """Bad block ids, slots and lengths set err_flag bits; the kernels stay in bounds."""
    H, D, bs = 8, 128, 16
    kc = torch.randn(4, bs, H, D, device="cuda").half()
    vc = torch.randn(4, bs, H, D, device="cuda").half()
    q = torch.randn(2, H, D, device="cuda").half()
    ws = torch.empty(pk.decode_workspace_bytes(2, H, D, 2, bs), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tables = torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device="cuda")
    pk.paged_attention_decode(out, q, kc, vc, tables, torch.tensor([20, 30], dtype=torch.int32, device="cuda"),
                              0.1, ws, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pk.PA_DEVCHK_BLOCK_ID
    err.zero_()
    pk.paged_attention_decode(out, q, kc, vc, tables, torch.tensor([20, 33], dtype=torch.int32, device="cuda"),
                              0.1, ws, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pk.PA_DEVCHK_SEQ_LEN
    err.zero_()
    slots = torch.tensor([5, 4 * bs + 3, -1], dtype=torch.int64, device="cuda")
    kn = torch.randn(3, H, D, device="cuda").half()
    before = kc.clone()
    pk.reshape_and_cache(kn, kn, kc, vc, slots, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == pk.PA_DEVCHK_SLOT
    assert torch.equal(kc[0, 5], kn[0])
    changed = (kc != before).any(dim=-1).any(dim=-1).nonzero().tolist()
    assert changed == [[0, 5]]
    assert pk.lib().pa_check_device_flag(int(err.item())) == pk.PA_ERR_DEVICE_CHECK


def _full_size(name):
    """A full-size workload in the bench's launch configuration, every sequence against the oracle."""
    w = si.get(name)
    ds = pwl.build(w)
    out = _step(ds).float().cpu().numpy()
    assert np.isfinite(out).all()
    o = owl.build(w, seqs=list(range(w.num_seqs)))
    assert np.array_equal(o.block_tables, ds.tables_host) and np.array_equal(o.slot_mapping, ds.slots_host)
    dec, _, _, _ = owl.run_step(o)
    diff = np.abs(out - dec)
    assert diff.max() <= TOL, f"max abs error {diff.max():.3g}"
    return ds, out


def test_full_size_b256_every_sequence(cuda_ready):
    _full_size("b256")


def test_full_size_long_context_every_sequence(cuda_ready):
    _full_size("longctx")


def test_decode_over_prefix_cached_blocks(cuda_ready):
    """Requests sharing a system prompt through the allocator's prefix cache: later requests
    write only their uncached tail, and decode reads the cached blocks written by the first."""
    H, D, bs, N = 8, 128, 16, 40
    rng = np.random.default_rng(21)
    sys_tokens = rng.integers(0, 32000, 64).tolist()
    sys_k = rng.standard_normal((64, H, D)).astype(np.float16)
    sys_v = rng.standard_normal((64, H, D)).astype(np.float16)
    alloc = pk.BlockAllocator(N, bs)
    kc = torch.full((N, bs, H, D), float("nan"), dtype=torch.float16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    logical = {}
    expect_cached = {"A": 0, "B": 64, "C": 64}
    reqs = {"A": 0, "B": 1, "C": 2}
    for name, n_suffix in (("A", 37), ("B", 50), ("C", 3)):
        toks = sys_tokens + rng.integers(0, 32000, n_suffix).tolist()
        st, cached = alloc.allocate_cached(reqs[name], toks)
        assert st == pk.PA_OK and cached == expect_cached[name]
        n = len(toks)
        sk = rng.standard_normal((n_suffix, H, D)).astype(np.float16)
        sv = rng.standard_normal((n_suffix, H, D)).astype(np.float16)
        k_all, v_all = np.concatenate([sys_k, sk]), np.concatenate([sys_v, sv])
        logical[name] = (k_all, v_all)
        st, slots = alloc.slots(reqs[name], cached, n - cached)
        pk.reshape_and_cache(torch.from_numpy(k_all[cached:]).cuda(), torch.from_numpy(v_all[cached:]).cuda(),
                             kc, vc, torch.from_numpy(slots).cuda())
        if name == "B":
            alloc.free(reqs["A"])          # A leaves: its system blocks stay referenced by B
            del logical["A"]
    names = sorted(logical)
    ids = [reqs[n] for n in names]
    mb = 8
    st, tables, lens = alloc.pack(ids, mb)
    assert st == pk.PA_OK
    q = rng.standard_normal((len(ids), H, D)).astype(np.float16)
    out = torch.empty(len(ids), H, D, dtype=torch.float16, device="cuda")
    ws = torch.empty(pk.decode_workspace_bytes(len(ids), H, D, mb, bs), dtype=torch.uint8, device="cuda")
    pk.paged_attention_decode(out, torch.from_numpy(q).cuda(), kc, vc, torch.from_numpy(tables).cuda(),
                              torch.from_numpy(lens).cuda(), 1 / np.sqrt(D), ws)
    got = out.float().cpu().numpy()
    for i, n in enumerate(names):
        k_all, v_all = logical[n]
        ref = oatt.softmax_attention(q[i][None], k_all, v_all, 1 / np.sqrt(D))[0]
        assert np.abs(got[i] - ref).max() <= TOL
    assert tables[0][:4].tolist() == tables[1][:4].tolist()      # B and C share the 4 prompt blocks
    assert alloc.cache_stats()["hit_blocks"] == 8


@pytest.mark.parametrize("qmul", [8.0, 16.0])
def test_decode_sharp_softmax(cuda_ready, qmul):
    """Scaled-up queries make a few keys dominate each row: the split-K partitions then carry very
    different maxima and the combine's rescaling decides the result."""
    rng = np.random.default_rng(41)
    H, D, bs = 4, 128, 16
    lens = [1, 15, 16, 17, 300, 777, 1500, 2047]
    need = [-(-n // bs) for n in lens]
    N = sum(need) + 7
    order = rng.permutation(N)
    kc = np.full((N, bs, H, D), np.nan, np.float16)
    vc = np.full((N, bs, H, D), np.nan, np.float16)
    maxb = max(need) + 1
    tables = rng.integers(0, N, size=(len(lens), maxb)).astype(np.int32)      # wrong-but-valid padding
    nxt = 0
    for s, n in enumerate(lens):
        t = order[nxt:nxt + need[s]]
        nxt += need[s]
        tables[s, :len(t)] = t
        k = rng.standard_normal((n, H, D)).astype(np.float16)
        v = rng.standard_normal((n, H, D)).astype(np.float16)
        for j in range(n):
            kc[t[j // bs], j % bs] = k[j]
            vc[t[j // bs], j % bs] = v[j]
    q = (rng.standard_normal((len(lens), H, D)) * qmul).astype(np.float16)
    seq_lens = np.asarray(lens, np.int32)
    scale = 1 / np.sqrt(D)
    d = {k_: torch.from_numpy(v_).cuda() for k_, v_ in dict(q=q, kc=kc, vc=vc, t=tables, l=seq_lens).items()}
    ws = torch.empty(pk.decode_workspace_bytes(len(lens), H, D, maxb, bs), dtype=torch.uint8, device="cuda")
    out = torch.full_like(d["q"], float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.paged_attention_decode(out, d["q"], d["kc"], d["vc"], d["t"], d["l"], scale, ws, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = oatt.paged_attention_decode(q, kc, vc, tables, seq_lens, bs, scale)
    diff = np.abs(out.float().cpu().numpy() - ref)
    assert diff.max() <= TOL, f"max abs error {diff.max():.3g}"
