"""GPU parity of the tcgen05 chunked-prefill kernel against the CPU oracle.

Max abs error <= 2e-3 against the float64 oracle (fp16 operands, fp32 TMEM
accumulation, P rounded to fp16 for the second MMA, fp16 output)."""
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


def make_case(seed, H, D, bs, reqs, extra_blocks=5, garbage_pad=True):
    """reqs: [(ctx_before, chunk_len)].  The pool holds every request's ctx + chunk rows at
    shuffled blocks; unused rows are NaN.  Returns numpy and device views."""
    rng = np.random.default_rng(seed)
    need = [-(-(c + L) // bs) for c, L in reqs]
    N = sum(need) + extra_blocks
    order = rng.permutation(N)
    kc = np.full((N, bs, H, D), np.nan, np.float16)
    vc = np.full((N, bs, H, D), np.nan, np.float16)
    maxb = max(need + [1]) + 2
    tables = rng.integers(0, N, size=(len(reqs), maxb)).astype(np.int32) if garbage_pad else \
        np.full((len(reqs), maxb), -1, np.int32)
    nxt = 0
    for b, (c, L) in enumerate(reqs):
        t = order[nxt:nxt + need[b]]
        nxt += need[b]
        tables[b, :len(t)] = t
        n = c + L
        k = rng.standard_normal((n, H, D)).astype(np.float16)
        v = rng.standard_normal((n, H, D)).astype(np.float16)
        for j in range(n):
            kc[t[j // bs], j % bs] = k[j]
            vc[t[j // bs], j % bs] = v[j]
    T = sum(L for _, L in reqs)
    q = rng.standard_normal((T, H, D)).astype(np.float16)
    q_start = np.concatenate([[0], np.cumsum([L for _, L in reqs])]).astype(np.int32)
    ctx = np.asarray([c for c, _ in reqs], np.int32)
    dev = {k_: torch.from_numpy(v_).cuda() for k_, v_ in
           dict(q=q, kc=kc, vc=vc, tables=tables, q_start=q_start, ctx=ctx).items()}
    return dict(q=q, kc=kc, vc=vc, tables=tables, q_start=q_start, ctx=ctx, dev=dev)


def run_prefill(case, scale, err=None):
    d = case["dev"]
    out = torch.full_like(d["q"], float("nan"))
    pk.paged_attention_prefill_chunk(out, d["q"], d["kc"], d["vc"], d["tables"], d["q_start"], d["ctx"], scale,
                                     err_flag=err)
    return out


def oracle_prefill(case, bs, scale):
    return oatt.paged_attention_prefill_chunk(case["q"], case["kc"], case["vc"], case["tables"],
                                              case["q_start"], case["ctx"], bs, scale)


CASES = [
    # (H, D, bs, [(ctx_before, chunk)])
    (2, 128, 16, [(0, 128)]),
    (2, 128, 16, [(0, 70)]),
    (2, 128, 16, [(1536, 512)]),
    (4, 128, 16, [(37, 200)]),
    (3, 64, 16, [(0, 300)]),
    (2, 64, 32, [(100, 129)]),
    (2, 128, 8, [(55, 90)]),
    (2, 128, 64, [(130, 260)]),
    (2, 128, 48, [(47, 81)]),
    (4, 128, 16, [(0, 1), (300, 40), (17, 256), (5, 0), (1000, 130)]),
    (8, 64, 16, [(64, 64), (0, 2), (129, 383)]),
    # more (query block, head) pairs than SMs: the unsplit kernel, whose CTAs walk several pairs each
    (16, 128, 16, [(0, 700), (300, 513), (17, 1000), (1000, 130)]),
    (24, 64, 32, [(64, 300), (0, 1), (129, 900), (5000, 257)]),
]


@pytest.mark.parametrize("H,D,bs,reqs", CASES)
def test_prefill_matches_oracle(cuda_ready, H, D, bs, reqs):
    case = make_case(hash((H, D, bs, len(reqs))) % 1000, H, D, bs, reqs)
    scale = 1 / np.sqrt(D)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_prefill(case, scale, err).float().cpu().numpy()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = oracle_prefill(case, bs, scale)
    assert np.isfinite(out).all()
    diff = np.abs(out - ref)
    assert diff.max() <= TOL, f"max abs error {diff.max():.3g}"


def test_prefill_without_split_matches_oracle(cuda_ready):
    """The same cases through the two-query-tile kernel.  The cases above are small launches, which the
    launcher gives to the one-query-tile kernel; PAGEDKV_PREFILL_SPLIT=0 turns that off (the launcher reads
    it once per process, hence the child process), so the two-query-tile kernel gets the ragged tails, head
    dims, block sizes and multi-request chunks too, and its bounded-wait timeout path."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, PAGEDKV_PREFILL_SPLIT="0")
    stall = os.path.join(os.path.dirname(__file__), "test_failure_detection_gpu.py")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        f"{__file__}::test_prefill_matches_oracle",
                        f"{stall}::test_prefill_wait_timeout_is_reported_and_recovered"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert f"{len(CASES) + 1} passed" in r.stdout, r.stdout[-2000:]


def test_mixed_workload_prefill(cuda_ready):
    """The 512-row chunk after 1536 cached tokens of the mixed step, 32 heads x 128."""
    w = si.get("mixed")
    ds = pwl.build(w)
    pk.reshape_and_cache(ds.k_step, ds.v_step, ds.k_cache, ds.v_cache, ds.slot_mapping)
    out = torch.empty_like(ds.prefill_q)
    pk.paged_attention_prefill_chunk(out, ds.prefill_q, ds.k_cache, ds.v_cache, ds.prefill_table,
                                     ds.prefill_q_start, ds.prefill_ctx_before, w.scale)
    got = out.float().cpu().numpy()
    o = owl.build(w, seqs=[0])
    _, pre, _, _ = owl.run_step(o)
    diff = np.abs(got - pre)
    assert diff.max() <= TOL, f"max abs error {diff.max():.3g}"


def test_chunk_split_and_decode_agree(cuda_ready):
    """Chunking is a scheduling split: two chunks give the rows one chunk gives, and the last
    row equals the decode kernel's output at the same context (within the tolerance)."""
    H, D, bs, c, L = 4, 128, 16, 300, 200
    case = make_case(3, H, D, bs, [(c, L)])
    scale = 1 / np.sqrt(D)
    whole = run_prefill(case, scale).float()
    d = case["dev"]
    parts = []
    for lo, hi in ((0, 77), (77, L)):
        out = torch.empty(hi - lo, H, D, dtype=torch.float16, device="cuda")
        pk.paged_attention_prefill_chunk(out, d["q"][lo:hi].contiguous(), d["kc"], d["vc"], d["tables"],
                                         torch.tensor([0, hi - lo], dtype=torch.int32, device="cuda"),
                                         torch.tensor([c + lo], dtype=torch.int32, device="cuda"), scale)
        parts.append(out.float())
    assert (whole - torch.cat(parts)).abs().max().item() <= TOL
    ws = torch.empty(pk.decode_workspace_bytes(1, H, D, d["tables"].shape[1], bs), dtype=torch.uint8, device="cuda")
    dec = torch.empty(1, H, D, dtype=torch.float16, device="cuda")
    pk.paged_attention_decode(dec, d["q"][L - 1:L].contiguous(), d["kc"], d["vc"], d["tables"],
                              torch.tensor([c + L], dtype=torch.int32, device="cuda"), scale, ws)
    assert (whole[L - 1] - dec[0].float()).abs().max().item() <= TOL


def test_prefill_device_checks(cuda_ready):
    case = make_case(4, 2, 128, 16, [(20, 40)])
    d = case["dev"]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(d["q"])
    bad_start = torch.tensor([0, 41], dtype=torch.int32, device="cuda")     # past num_tokens
    pk.paged_attention_prefill_chunk(out, d["q"], d["kc"], d["vc"], d["tables"], bad_start, d["ctx"], 0.1,
                                     err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pk.PA_DEVCHK_QUERY_RANGE
    err.zero_()
    tables = d["tables"].clone()
    tables[0, 1] = 10_000
    pk.paged_attention_prefill_chunk(out, d["q"], d["kc"], d["vc"], tables, d["q_start"], d["ctx"], 0.1,
                                     err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == pk.PA_DEVCHK_BLOCK_ID
    err.zero_()
    big_ctx = torch.tensor([10_000], dtype=torch.int32, device="cuda")
    pk.paged_attention_prefill_chunk(out, d["q"], d["kc"], d["vc"], d["tables"], d["q_start"], big_ctx, 0.1,
                                     err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pk.PA_DEVCHK_SEQ_LEN


@pytest.mark.parametrize("qmul", [4.0, 8.0, 16.0])
def test_prefill_sharp_softmax(cuda_ready, qmul):
    """Sharper score distributions (q scaled up): the exponent arguments span a wide range, which
    exercises the fp16 exp2 of P; the output must still be within the tolerance."""
    H, D, bs = 4, 128, 16
    case = make_case(17, H, D, bs, [(300, 200), (0, 129)])
    case["q"] = (case["q"].astype(np.float32) * qmul).astype(np.float16)
    case["dev"]["q"] = torch.from_numpy(case["q"]).cuda()
    scale = 1 / np.sqrt(D)
    out = run_prefill(case, scale).float().cpu().numpy()
    ref = oracle_prefill(case, bs, scale)
    diff = np.abs(out - ref)
    assert diff.max() <= TOL, f"max abs error {diff.max():.3g}"


def test_prefill_many_requests(cuda_ready):
    """Sixteen requests of random cached lengths and chunk sizes in one launch: every CTA finds its
    (request, q-tile) among uneven neighbours."""
    rng = np.random.default_rng(53)
    reqs = [(int(rng.integers(0, 700)), int(rng.integers(1, 300))) for _ in range(16)]
    case = make_case(54, 4, 128, 16, reqs)
    scale = 1 / np.sqrt(128)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_prefill(case, scale, err).float().cpu().numpy()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = oracle_prefill(case, 16, scale)
    assert np.isfinite(out).all()
    diff = np.abs(out - ref)
    assert diff.max() <= TOL, f"max abs error {diff.max():.3g}"


def test_causal_prefill_8192_every_row(cuda_ready):
    """The 8192-token causal prefill the benchmark times (one request, nothing cached, 32 heads x 128),
    in the bench's launch configuration.  Every row of every head is compared with the oracle, which
    computes the prompt as 256-row chunks at their absolute positions (the chunk-split identity its
    pins establish), so its float64 score matrices stay within host memory."""
    w = si.get("prefill8k")
    ds = pwl.build(w)
    pk.reshape_and_cache(ds.k_step, ds.v_step, ds.k_cache, ds.v_cache, ds.slot_mapping)
    out = torch.full_like(ds.prefill_q, float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.paged_attention_prefill_chunk(out, ds.prefill_q, ds.k_cache, ds.v_cache, ds.prefill_table,
                                     ds.prefill_q_start, ds.prefill_ctx_before, w.scale, err_flag=err)
    got = out.float().cpu().numpy()
    assert int(err.item()) == 0
    o = owl.build(w)
    kc, vc = o.k_cache.copy(), o.v_cache.copy()
    oatt.reshape_and_cache(kc, vc, o.k_step, o.v_step, o.slot_mapping, w.block_size)
    assert np.array_equal(ds.k_cache.cpu().numpy().view(np.int16), kc.view(np.int16))
    L, step = w.prefill.chunk, 256
    worst = 0.0
    for lo in range(0, L, step):
        hi = min(L, lo + step)
        ref = oatt.paged_attention_prefill_chunk(o.prefill_q[lo:hi], kc, vc, o.prefill_table, [0, hi - lo], [lo],
                                                 w.block_size, w.scale)
        worst = max(worst, float(np.abs(got[lo:hi] - ref).max()))
    assert worst <= TOL, f"max abs error {worst:.3g}"
