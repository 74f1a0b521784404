"""Host-side logic of bench.py (no GPU): algorithmic byte and FLOP counts, the oracle
sample bound, reference-arm rank gating, and the multi-rank reduction (max of times,
sum of bytes) run as two gloo ranks on the CPU."""
import io
import json
import os
import socket
from contextlib import redirect_stdout

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth_inputs as si


def test_step_bytes_tiny():
    w = si.tiny()
    dec, rs, pre = bench.step_bytes(w, w.decode_lens, 3, 4)
    H, D = 4, 64
    kv = sum(w.decode_lens) * H * D * 2 * 2
    assert dec == kv + 2 * 4 * H * D * 2 + (1 + 1 + 2 + 3) * 4 + 4 * 4
    assert rs == 4 * H * D * 2 * 2 * 2 + 4 * 8
    assert pre == 0


def test_prefill_flops_mixed():
    # 512 rows after 1536 cached tokens: 917,760 visible pairs per head, 4 * 32 * 128 flops each
    w = si.get("mixed")
    assert bench.prefill_flops(w) == 917_760 * 4 * 32 * 128 == 15_036_579_840


def test_shared_prefix_counted_once_in_unique_bytes():
    # 8 sequences share a 1024-token prefix (32 whole blocks of 32): 7 of the 8 reads of it are not unique
    w = si.get("longctx")
    extra = bench.shared_prefix_rereads(w, w.decode_lens)
    assert extra == 7 * 1024 * 32 * 128 * 2 * 2
    dec, _, _ = bench.step_bytes(w, w.decode_lens, 1024, 8)
    assert dec - extra == dec - 7 * 16 * 2**20     # 16 MiB of K+V per 1024 tokens x 32 heads x 128
    assert bench.shared_prefix_rereads(si.get("b256"), si.get("b256").decode_lens) == 0


def test_prefill_8k_flops():
    w = si.get("prefill8k")
    assert bench.prefill_flops(w) == 4 * 32 * 128 * (8192 * 8193 // 2)


def test_packed_views_stage_a_step_in_one_buffer():
    """The end-to-end loop's staging: every tensor of a step in one buffer, 256-byte aligned, disjoint,
    typed and contiguous, and a byte copy of the whole buffer carries every tensor."""
    specs = [("q", (3, 4, 64), torch.float16), ("slots", (3,), torch.int64), ("tables", (3, 5), torch.int32),
             ("empty", (0, 5), torch.int32), ("lens", (3,), torch.int32)]
    buf, v = bench.packed_views(specs, lambda n: torch.zeros(n, dtype=torch.uint8))
    base = buf.data_ptr()
    spans = []
    for name, shape, dtype in specs:
        t = v[name]
        assert tuple(t.shape) == shape and t.dtype == dtype and t.is_contiguous()
        if t.numel() == 0:
            continue                                   # an empty view may report a null pointer
        assert (t.data_ptr() - base) % 256 == 0
        spans.append((t.data_ptr() - base, t.numel() * t.element_size()))
    spans.sort()
    for (o0, n0), (o1, _) in zip(spans, spans[1:]):
        assert o0 + n0 <= o1
    assert spans[-1][0] + spans[-1][1] <= buf.numel()
    g = torch.Generator().manual_seed(0)
    v["q"].copy_(torch.randn(3, 4, 64, generator=g).half())
    v["slots"].copy_(torch.tensor([7, -1, 2**40]))
    v["tables"].copy_(torch.arange(15, dtype=torch.int32).view(3, 5))
    v["lens"].copy_(torch.tensor([1, 2, 3], dtype=torch.int32))
    buf2, v2 = bench.packed_views(specs, lambda n: torch.zeros(n, dtype=torch.uint8))
    buf2.copy_(buf)
    for name, _, _ in specs:
        assert torch.equal(v2[name], v[name])


def test_timing_distribution():
    d = bench.dist_ms([1.0, 2.0, 3.0, 4.0, 100.0])
    assert d["median"] == 3.0 and d["n"] == 5 and d["mean"] == 22.0
    assert d["p10"] == pytest.approx(1.4) and d["p90"] == pytest.approx(61.6)


def test_oracle_sample_is_bounded_and_seeded():
    w = si.get("b256")
    a = bench.oracle_sample_seqs(w, 12000)
    b = bench.oracle_sample_seqs(w, 12000)
    assert a == b and a == sorted(a)
    tot = sum(w.decode_lens[s] for s in a)
    assert tot <= 12000 + max(w.decode_lens)


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    f = io.StringIO()
    with redirect_stdout(f):
        rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0", "--workload", "tiny"])
    assert rc == 0 and f.getvalue() == ""


def test_reference_arm_line_on_rank0(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    f = io.StringIO()
    with redirect_stdout(f):
        rc = bench.main(["--impl", "reference", "--steps", "2", "--warmup", "1", "--workload", "tiny"])
    line = json.loads(f.getvalue().strip().splitlines()[-1])
    assert rc == 0 and line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["unit"] == "GB/s" and line["higher_is_better"] is True


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx, sm = bench.reduce_max_sum(10.0 + 5 * rank, 100.0 * (rank + 1), torch.device("cpu"))
        q.put((rank, mx, sm))
    finally:
        dist.destroy_process_group()


def test_reduce_max_sum_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    # every rank sees the max of the times and the sum of the bytes
    assert res == [(0, 15.0, 300.0), (1, 15.0, 300.0)]


def test_reduce_is_identity_without_process_group():
    assert bench.reduce_max_sum(3.0, 7.0, torch.device("cpu")) == (3.0, 7.0)


def test_clock_summary_keeps_the_timed_window():
    """Only nvidia-smi samples taken while the timed region ran count; throttle reasons seen outside it do
    not; lines that cannot be placed in time fall back to all samples."""
    import datetime
    c = bench.ClockSampler(0)
    t = datetime.datetime(2026, 1, 2, 3, 4, 5, 600000)
    fmt = lambda d: d.strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    row = lambda d, mhz, cap: (f"{fmt(d)}, 0, {mhz}, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, "
                               + ("Active" if cap else "Not Active"))
    c.lines = [row(t - datetime.timedelta(seconds=1), 600, True),          # before: idle, capped
               row(t, 1965, False), row(t + datetime.timedelta(milliseconds=50), 1900, False),
               row(t + datetime.timedelta(seconds=2), 700, True),          # after
               "garbage"]
    c.window = [t - datetime.timedelta(milliseconds=10), t + datetime.timedelta(milliseconds=60)]
    assert c.summary() == {"sm_mhz": 1932.5, "sm_max_mhz": 1965.0, "reasons": [], "samples": 2}
    c.window = [None, None]
    s = c.summary()
    assert s["samples"] == 4 and s["reasons"] == ["sw_power_cap"] and s["sm_mhz"] == (700 + 1900) / 2


def test_pool_stats_against_page_estimate():
    """kv_pool: measured waste of the allocator beside the page's (bs/2)/avg_len estimate."""
    import types
    import paged_kv_cache_411_b200 as pk
    bs = 16
    alloc = pk.BlockAllocator(64, bs)
    lens = np.array([10, 16, 33, 100], np.int32)
    for r, n in enumerate(lens):
        assert alloc.allocate(r, int(n)) == pk.PA_OK
    ds = types.SimpleNamespace(alloc=alloc, seq_lens_host=lens,
                               workload=types.SimpleNamespace(block_size=bs, num_seqs=len(lens)))
    st = bench.pool_stats(ds)
    waste = sum(-(-int(n) // bs) * bs - int(n) for n in lens)          # 6 + 0 + 15 + 12
    assert st["waste_tokens"] == waste and st["used_blocks"] == sum(-(-int(n) // bs) for n in lens)
    assert st["waste_frac"] == round(waste / lens.sum(), 5)
    assert st["page_estimate_frac"] == round((bs / 2) / (lens.sum() / len(lens)), 5)
