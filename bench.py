"""Paged-attention decode benchmark: GB/s (and % of HBM peak) and decode tokens/s per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload b256] [--impl ours|reference]

A step is one pass of the hot path over one batch: reshape_and_cache of the
step's new K/V rows, then paged decode attention over every sequence (and,
for the mixed workload, the chunked-prefill kernel).  ``value`` is the
algorithmic bytes of the step (K/V read by decode, q/out, block tables, the
rows written by reshape_and_cache) over the device time of the step, summed
over ranks.  With N > 1 (torchrun) every rank runs its own replica of the
workload on its own GPU (weak scaling, no collective on the data path); the
time is the max over ranks.

At N = 1 the line also carries ``graph``: the same step captured once in a
CUDA graph and replayed (and the decode call alone), which takes the host's
per-call launch path out of the timing; ``--no-graph`` skips it.

``--impl reference`` times the float64 CPU oracle on the host cores instead
(a bounded sample of the same workload per step); under torchrun only rank 0
runs it.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth_inputs as si  # noqa: E402

METRIC = "paged-attn decode GB/s (% of B200 HBM peak) and decode tokens/s at 1 GPU"
FALLBACK_HBM_GBS = 6650.0


FALLBACK_TFLOPS = 1590.0


def measured_peaks():
    """(HBM GB/s, dense fp16/bf16 tensor TFLOP/s burst, kind)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_TFLOPS, "fallback"


def packed_views(specs, make):
    """One uint8 buffer holding a tensor per (name, shape, dtype) of ``specs``, each at a 256-byte aligned
    offset, so that a step's inputs (or outputs) cross between host and device in ONE copy.  ``make(n)``
    allocates the n-byte buffer; returns it and a typed, contiguous view per name."""
    import torch
    offs, n = {}, 0
    for name, shape, dtype in specs:
        nbytes = int(np.prod(shape, dtype=np.int64)) * torch.empty((), dtype=dtype).element_size()
        offs[name] = (n, nbytes)
        n = (n + nbytes + 255) // 256 * 256
    buf = make(max(n, 256))
    views = {name: buf[offs[name][0]:offs[name][0] + offs[name][1]].view(dtype).view(shape)
             for name, shape, dtype in specs}
    return buf, views


def prefill_flops(w):
    """Algorithmic FLOPs of the causal chunk: 4 * H * D per visible (query, key) pair."""
    if w.prefill is None:
        return 0
    L, c = w.prefill.chunk, w.prefill.ctx_before
    pairs = L * c + L * (L + 1) // 2
    return 4 * w.num_heads * w.head_dim * pairs


def shared_prefix_rereads(w, seq_lens):
    """K/V bytes the decode reads more than once: a prefix shared by all sequences (whole blocks) is
    stored once but every sequence reads it, so its bytes beyond the first read are not unique."""
    if not w.shared_prefix or len(seq_lens) == 0:
        return 0
    shared_tokens = (w.shared_prefix // w.block_size) * w.block_size
    return (len(seq_lens) - 1) * shared_tokens * w.num_heads * w.head_dim * 2 * 2


def dist_ms(xs):
    """Median, 10th and 90th percentile (and mean) of per-step times in ms."""
    a = np.asarray(xs, dtype=np.float64)
    return {"median": round(float(np.median(a)), 5), "p10": round(float(np.percentile(a, 10)), 5),
            "p90": round(float(np.percentile(a, 90)), 5), "mean": round(float(a.mean()), 5), "n": int(a.size)}


def step_bytes(w, seq_lens, tables_cols, n_step_rows):
    """Algorithmic bytes of one step (see the module docstring)."""
    H, D, bs = w.num_heads, w.head_dim, w.block_size
    lens = np.asarray(seq_lens, dtype=np.int64)
    kv = int(lens.sum()) * H * D * 2 * 2
    qo = 2 * len(lens) * H * D * 2
    meta = int(((lens + bs - 1) // bs).sum()) * 4 + len(lens) * 4
    reshape = n_step_rows * H * D * 2 * 2 * 2 + n_step_rows * 8
    decode = kv + qo + meta
    prefill = 0
    if w.prefill is not None:
        L, c = w.prefill.chunk, w.prefill.ctx_before
        prefill = (c + L) * H * D * 2 * 2 + 2 * L * H * D * 2
    return decode, reshape, prefill


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms while running; summary() keeps the samples
    taken between mark_start() and mark_end() (the timed region), or all of them if none can be placed."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 50

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.window = [None, None]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.PERIOD_MS)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        return self

    def mark_start(self):
        self.window[0] = datetime.datetime.now()

    def mark_end(self):
        self.window[1] = datetime.datetime.now()

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    @staticmethod
    def _parse(line):
        """(time or None, sm MHz, max MHz, {reason: active}) of one CSV line, or None."""
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 10:
            return None
        try:
            sm, mx = float(parts[2]), float(parts[3])
        except ValueError:
            return None
        try:
            ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
        except ValueError:
            ts = None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        return ts, sm, mx, {n: v.lower() == "active" for n, v in zip(names, parts[6:10])}

    def summary(self):
        rows = [r for r in (self._parse(l) for l in getattr(self, "lines", [])) if r is not None]
        lo, hi = self.window
        if lo is not None and hi is not None:
            pad = datetime.timedelta(milliseconds=self.PERIOD_MS)
            inside = [r for r in rows if r[0] is not None and lo - pad <= r[0] <= hi + pad]
            if inside:
                rows = inside
        sm = [r[1] for r in rows]
        reasons = sorted({n for r in rows for n, on in r[3].items() if on})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": rows[-1][2] if rows else None,
                "reasons": reasons, "samples": len(sm)}


def pool_stats(ds):
    """Measured internal fragmentation of the pool vs the page's (block_size / 2) / avg_len estimate."""
    st = ds.alloc.stats()
    w = ds.workload
    ctx = int(ds.seq_lens_host.astype(np.int64).sum())
    return {"block_size": w.block_size, "num_blocks": st["num_blocks"], "used_blocks": st["num_used"],
            "waste_tokens": st["waste_tokens"], "waste_frac": round(st["waste_tokens"] / max(1, ctx), 5),
            "page_estimate_frac": round((w.block_size / 2) / (ctx / w.num_seqs), 5) if w.num_seqs and ctx else None}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max_sum(value_max, value_sum, device):
    """Max of the first value and sum of the second over all ranks (identity at N = 1)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value_max, value_sum
    t = torch.tensor([value_max], dtype=torch.float64, device=device)
    u = torch.tensor([value_sum], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def oracle_sample_seqs(w, budget_tokens):
    """A seeded sample of decode sequences whose context totals about budget_tokens."""
    rng = np.random.default_rng(1234)
    order = rng.permutation(w.num_seqs)
    pick, tot = [], 0
    for s in order:
        if pick and tot + w.decode_lens[s] > budget_tokens:
            continue
        pick.append(int(s))
        tot += w.decode_lens[s]
        if tot >= budget_tokens:
            break
    return sorted(pick)


def _oracle_case(w, budget_tokens):
    from oracle import attention as oatt
    from oracle import workloads as owl
    sample = oracle_sample_seqs(w, budget_tokens)
    o = owl.build(w, seqs=sample)
    kc, vc = o.k_cache, o.v_cache
    oatt.reshape_and_cache(kc, vc, o.k_step, o.v_step, o.slot_mapping, w.block_size)
    idx = np.asarray(sample)
    args = (o.q[idx], kc, vc, o.block_tables[idx], o.seq_lens[idx], w.block_size, w.scale)
    tokens = int(o.seq_lens[idx].astype(np.int64).sum())
    return sample, args, tokens


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu capture of the current
# kernels on each workload at its default block size; the decode entry sums the plan, streaming and combine
# launches of one call.  Workloads without a capture report None, and so must any entry whose kernel has
# changed since it was taken.
NCU_TRAFFIC_BYTES = {
    "b256": {"decode": 2_812_032_000},
    "b32": {"decode": 276_752_000},
    "mixed": {"decode": 1_104_322_000, "prefill": 37_870_000},
    "prefill8k": {"prefill": 600_975_000},
}


def ncu_traffic(w, args, kernel):
    if args.block_size:
        return None
    return NCU_TRAFFIC_BYTES.get(args.workload, {}).get(kernel)


def time_oracle(w, steps, warmup, budget_tokens, min_seconds=0.0, max_steps=None):
    """Times the CPU oracle's decode on a bounded sample of the workload's sequences.

    Runs ``warmup`` untimed calls, then ``steps`` timed ones (or, with min_seconds, as many as
    fit in min_seconds up to max_steps).  Returns (GB/s, seconds per step, description, threads)."""
    from oracle import attention as oatt
    sample, args, tokens = _oracle_case(w, budget_tokens)
    for _ in range(warmup):
        oatt.paged_attention_decode(*args)
    n = 0
    t0 = time.perf_counter()
    while True:
        oatt.paged_attention_decode(*args)
        n += 1
        el = time.perf_counter() - t0
        if n >= steps and el >= min_seconds:
            break
        if max_steps is not None and n >= max_steps:
            break
    dt = el / n
    nbytes = tokens * w.num_heads * w.head_dim * 4
    desc = (f"oracle float64 decode of {len(sample)} of {w.num_seqs} sequences ({tokens} cached tokens) per "
            f"step, {n} timed steps; GB/s counts those sequences' K/V bytes")
    return nbytes / dt / 1e9, dt, desc, _blas_threads()


def oracle_tokens_for(w, total_steps, target_seconds):
    """Tokens per oracle step so that total_steps steps take about target_seconds on this host."""
    from oracle import attention as oatt
    _, args, tokens = _oracle_case(w, 2000)
    t0 = time.perf_counter()
    oatt.paged_attention_decode(*args)
    rate = tokens / max(time.perf_counter() - t0, 1e-6)
    return int(max(64, min(sum(w.decode_lens), rate * target_seconds / max(1, total_steps))))


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def time_oracle_prefill(w, steps, target_seconds):
    """Times the oracle's causal prefill on the chunk's last rows (the heaviest ones), as many rows as fit
    about target_seconds over all steps.  Returns (step GB/s estimated from the sampled share of the
    chunk's FLOPs, seconds per sampled call, description, threads)."""
    from oracle import attention as oatt
    from oracle import workloads as owl
    o = owl.build(w)
    kc, vc = o.k_cache.copy(), o.v_cache.copy()
    oatt.reshape_and_cache(kc, vc, o.k_step, o.v_step, o.slot_mapping, w.block_size)
    L, c = w.prefill.chunk, w.prefill.ctx_before

    def call(rows):
        lo = L - rows
        t0 = time.perf_counter()
        oatt.paged_attention_prefill_chunk(o.prefill_q[lo:], kc, vc, o.prefill_table, [0, rows], [c + lo],
                                           w.block_size, w.scale)
        return time.perf_counter() - t0

    rows = max(1, min(L, int(16 * target_seconds / max(1, steps) / max(call(16), 1e-6))))
    dts = [call(rows) for _ in range(steps)]
    dt = float(np.mean(dts))
    pairs = rows * c + sum(L - i for i in range(rows))               # visible (query, key) pairs sampled
    share = pairs / (L * c + L * (L + 1) // 2)
    _, rs_b, pre_b = step_bytes(w, [], 0, o.slot_mapping.shape[0])
    desc = (f"oracle float64 causal prefill of the last {rows} of {L} rows ({100 * share:.2f}% of the chunk's "
            f"FLOPs) per step, {steps} timed steps; GB/s = the step's bytes over the time scaled to the whole chunk")
    return (rs_b + pre_b) / (dt / share) / 1e9, dt, desc, _blas_threads()


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    w = si.get(args.workload)
    if args.block_size:
        w = si.with_block_size(w, args.block_size)
    if w.num_seqs == 0:
        gbs, dt, desc, threads = time_oracle_prefill(w, args.steps, 120.0)
        line = {
            "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "num_heads": w.num_heads, "head_dim": w.head_dim,
                       "block_size": w.block_size, "parallelism": "host cores"},
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return 0
    per_step = oracle_tokens_for(w, args.steps + args.warmup, 120.0)
    gbs, dt, desc, threads = time_oracle(w, args.steps, args.warmup, per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "num_seqs": w.num_seqs, "num_heads": w.num_heads, "head_dim": w.head_dim,
                   "block_size": w.block_size, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    import paged_kv_cache_411_b200 as pk
    from paged_kv_cache_411_b200 import workload as pwl

    world, rank, local = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    w = si.get(args.workload)
    if args.block_size:
        w = si.with_block_size(w, args.block_size)
    ds = pwl.build(w, device=device)
    S, H, D = ds.q.shape
    T = ds.k_step.shape[0]
    ws = torch.empty(pk.decode_workspace_bytes(S, H, D, ds.max_blocks, w.block_size), dtype=torch.uint8,
                     device=device)
    out = torch.empty_like(ds.q)
    pout = torch.empty_like(ds.prefill_q) if ds.prefill_q is not None else None
    stream = torch.cuda.current_stream(device)
    dec_b, rs_b, pre_b = step_bytes(w, ds.seq_lens_host, ds.max_blocks, T)
    step_b = dec_b + rs_b + pre_b

    def step(ev=None, pev=None, st=None):
        st = stream if st is None else st
        pk.reshape_and_cache(ds.k_step, ds.v_step, ds.k_cache, ds.v_cache, ds.slot_mapping, stream=st)
        if pout is not None:
            if pev is not None:
                pev[0].record(st)
            pk.paged_attention_prefill_chunk(pout, ds.prefill_q, ds.k_cache, ds.v_cache, ds.prefill_table,
                                             ds.prefill_q_start, ds.prefill_ctx_before, w.scale, stream=st)
            if pev is not None:
                pev[1].record(st)
        if S == 0:
            return
        if ev is not None:
            ev[0].record(st)
        pk.paged_attention_decode(out, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.seq_lens, w.scale, ws,
                                  stream=st)
        if ev is not None:
            ev[1].record(st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)

    dec_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
    step_events = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    pre_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)] if pout is not None else [None] * args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.25)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        clk.mark_start()
        t0.record(stream)
        for i in range(args.steps):
            step_events[i].record(stream)
            step(dec_events[i], pre_events[i])
        step_events[args.steps].record(stream)
        t1.record(stream)
        torch.cuda.synchronize(device)
        clk.mark_end()
        if world > 1:
            dist.barrier()
    local_ms = t0.elapsed_time(t1)
    dec_ms = [a.elapsed_time(b) for a, b in dec_events] if S > 0 else []
    step_ms = [step_events[i].elapsed_time(step_events[i + 1]) for i in range(args.steps)]
    pre_ms = [e[0].elapsed_time(e[1]) for e in pre_events] if pout is not None else []
    total_ms, total_bytes = reduce_max_sum(local_ms, step_b * args.steps, device)
    ms_per_step = total_ms / args.steps
    value = total_bytes / (total_ms / 1e3) / 1e9
    peak, peak_tf, peak_kind = measured_peaks()

    # end to end: every step copies its inputs from pinned host memory to the device, runs, and copies its
    # output back to pinned host memory, as a serving loop would: the inputs of step i+1 go up on a copy
    # stream (into the other of two device input sets) while step i computes, and the host reads the
    # output of each step one step later.  The timed region covers all of it.
    names = ("q", "k_step", "v_step", "slot_mapping", "block_tables", "seq_lens")
    if pout is not None:
        names += ("prefill_q", "prefill_table", "prefill_q_start", "prefill_ctx_before")
    # every input of a step in one pinned buffer and every output in another (one copy each way per step,
    # as the serving loop stages its tables, slots and lengths)
    in_specs = [(k, tuple(getattr(ds, k).shape), getattr(ds, k).dtype) for k in names]
    out_specs = [("out", tuple(out.shape), out.dtype)] + \
        ([("pout", tuple(pout.shape), pout.dtype)] if pout is not None else [])
    host_in, host_v = packed_views(in_specs, lambda n: torch.empty(n, dtype=torch.uint8).pin_memory())
    for k in names:
        host_v[k].copy_(getattr(ds, k).cpu())
    host_out = [packed_views(out_specs, lambda n: torch.empty(n, dtype=torch.uint8).pin_memory())[0]
                for _ in range(2)]
    dev_sets = [packed_views(in_specs, lambda n: torch.empty(n, dtype=torch.uint8, device=device))
                for _ in range(2)]
    dev_outs = [packed_views(out_specs, lambda n: torch.empty(n, dtype=torch.uint8, device=device))
                for _ in range(2)]
    h2d = host_in.numel()
    d2h = host_out[0].numel()
    copy_stream = torch.cuda.Stream(device)
    ready = [torch.cuda.Event() for _ in range(2)]      # inputs of the set are on the device
    done = [torch.cuda.Event() for _ in range(2)]       # the step that used the set has finished
    fetched = [torch.cuda.Event() for _ in range(2)]    # its output is back on the host

    def e2e_upload(b):
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(done[b])              # the step before last has finished with set b
            dev_sets[b][0].copy_(host_in, non_blocking=True)
            ready[b].record(copy_stream)

    def e2e_compute(b):
        d, o = dev_sets[b][1], dev_outs[b][1]
        stream.wait_event(ready[b])
        pk.reshape_and_cache(d["k_step"], d["v_step"], ds.k_cache, ds.v_cache, d["slot_mapping"], stream=stream)
        if pout is not None:
            pk.paged_attention_prefill_chunk(o["pout"], d["prefill_q"], ds.k_cache, ds.v_cache,
                                             d["prefill_table"], d["prefill_q_start"], d["prefill_ctx_before"],
                                             w.scale, stream=stream)
        if S > 0:
            pk.paged_attention_decode(o["out"], d["q"], ds.k_cache, ds.v_cache, d["block_tables"],
                                      d["seq_lens"], w.scale, ws, stream=stream)
        done[b].record(stream)
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(done[b])
            host_out[b].copy_(dev_outs[b][0], non_blocking=True)
            fetched[b].record(copy_stream)

    def e2e_run(n):
        e2e_upload(0)
        for i in range(n):
            b = i & 1
            if i + 1 < n:
                e2e_upload(b ^ 1)
            e2e_compute(b)
            if i > 0:
                fetched[b ^ 1].synchronize()             # the host reads the previous step's output
        fetched[(n - 1) & 1].synchronize()

    for e in done:
        e.record(stream)
    e2e_run(max(1, args.warmup))
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    t_a = time.perf_counter()
    e2e_run(args.steps)
    e2e_s = time.perf_counter() - t_a
    e2e_max, e2e_bytes = reduce_max_sum(e2e_s, step_b * args.steps, device)
    e2e_value = e2e_bytes / e2e_max / 1e9

    # the same step captured once in a CUDA graph and replayed: the kernels and their programmatic-launch
    # edges as above, without the host's per-launch cost (1 GPU; reported beside the stream-launched step)
    graph = None
    if world == 1 and not args.no_graph:
        try:
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(device)               # capture needs a stream other than the default one
            torch.cuda.synchronize(device)
            with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
                step(st=cap)
            with torch.cuda.stream(stream):
                for _ in range(args.warmup):
                    g.replay()
                g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize(device)
                g0.record(stream)
                for _ in range(args.steps):
                    g.replay()
                g1.record(stream)
            torch.cuda.synchronize(device)
            g_ms = g0.elapsed_time(g1) / args.steps
            graph = {"value": round(step_b / (g_ms / 1e3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(g_ms, 5),
                     "steps": args.steps}
            del g
        except Exception as exc:                     # reported, not fatal: the stream-launched figures stand
            torch.cuda.synchronize(device)
            graph = {"error": f"{type(exc).__name__}: {exc}"[:200]}
    # the decode call alone (plan, streaming kernel, combine) as a graph replayed back to back: its device
    # time without the host's launch path between the kernels
    graph_dec_ms = None
    if world == 1 and not args.no_graph and S > 0 and graph is not None and "error" not in graph:
        try:
            gd = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(device)
            torch.cuda.synchronize(device)
            with torch.cuda.graph(gd, stream=cap, capture_error_mode="thread_local"):
                pk.paged_attention_decode(out, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.seq_lens, w.scale,
                                          ws, stream=cap)
            with torch.cuda.stream(stream):
                for _ in range(args.warmup):
                    gd.replay()
                d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize(device)
                d0.record(stream)
                for _ in range(args.steps):
                    gd.replay()
                d1.record(stream)
            torch.cuda.synchronize(device)
            graph_dec_ms = d0.elapsed_time(d1) / args.steps
            del gd
        except Exception as exc:
            torch.cuda.synchronize(device)
            graph["decode_error"] = f"{type(exc).__name__}: {exc}"[:200]

    if rank == 0:
        has_decode = S > 0
        dec_avg_ms = float(np.mean(dec_ms)) if has_decode else 0.0
        unique_b = dec_b - shared_prefix_rereads(w, ds.seq_lens_host)
        dec_gbs = unique_b / (dec_avg_ms / 1e3) / 1e9 if has_decode else 0.0
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {
                "workload": w.name, "num_seqs": S, "num_heads": H, "head_dim": D, "block_size": w.block_size,
                "context_tokens": int(ds.seq_lens_host.sum()), "step_rows_written": T,
                "bytes_per_step": step_b, "accumulate": "f32",
                "l2": f"inputs larger than L2 ({dec_b / 1e9:.2f} GB of K/V per step), no flush",
                "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
            },
            "pct_of_hbm_peak": round(100 * value / world / peak, 2),
            "pct_of_nominal_8tbs": round(100 * value / world / 8000.0, 2),
            "decode_tokens_per_s": round(S * world / (ms_per_step / 1e3), 1),
            "decode_tokens_per_s_32_layers": round(S * world / (32 * ms_per_step / 1e3), 1),
            "roofline": {"kernel": "paged_attention_decode (plan + streaming kernel + combine)", "bound": "hbm",
                         "achieved": round(dec_gbs, 2), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": round(dec_gbs / peak, 4), "traffic": ncu_traffic(w, args, "decode"),
                         "algorithmic_bytes_per_launch": unique_b, "avg_launch_ms": round(dec_avg_ms, 5)},
            "step_ms": dist_ms(step_ms),
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": round(1e3 * e2e_max / args.steps, 4)},
            "gpu_launches": args.steps * (1 + (3 if S > 0 else 0) + (1 if pout is not None else 0)),
            "graph": graph,
            "kv_pool": pool_stats(ds),
            "clocks": clk.summary(),
        }
        if graph_dec_ms is not None:
            ach = unique_b / (graph_dec_ms / 1e3) / 1e9
            graph.update({"decode_ms": round(graph_dec_ms, 5), "decode_achieved": round(ach, 2),
                          "decode_frac": round(ach / peak, 4)})
        if has_decode:
            line["decode_ms"] = dist_ms(dec_ms)
            if unique_b != dec_b:
                # a shared prefix is read by every sequence but stored once: the roofline counts it once
                line["roofline"]["logical_bytes_per_launch"] = dec_b
                line["roofline"]["logical_achieved"] = round(dec_b / (dec_avg_ms / 1e3) / 1e9, 2)
        if pout is not None:
            pre_avg = float(np.mean(pre_ms))
            tf = prefill_flops(w) / (pre_avg / 1e3) / 1e12
            line["prefill_ms"] = dist_ms(pre_ms)
            line["roofline_prefill"] = {
                "kernel": "paged_attention_prefill_chunk (tcgen05)", "bound": "tensor", "achieved": round(tf, 2),
                "peak": peak_tf, "peak_kind": peak_kind + " bf16 burst (fp16 has the same nominal rate)",
                "unit": "TFLOP/s", "frac": round(tf / peak_tf, 4), "traffic": ncu_traffic(w, args, "prefill"),
                "algorithmic_flops_per_launch": prefill_flops(w), "avg_launch_ms": round(pre_avg, 5)}
            if not has_decode:
                # a prefill-only step: its tensor-bound kernel is the dominant one
                line["roofline"] = line.pop("roofline_prefill")
        if world == 1 and not args.no_cpu_baseline and has_decode:
            gbs, dt, desc, threads = time_oracle(w, 1, 1, args.oracle_tokens, min_seconds=10.0, max_steps=30)
            line["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                                    "sample": desc}
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1, user_api="blas"):
                gbs1, _, desc1, threads1 = time_oracle(w, 1, 1, args.oracle_tokens // 4, min_seconds=10.0,
                                                       max_steps=30)
            line["cpu_baseline_1thread"] = {"value": round(gbs1, 4), "unit": "GB/s", "cores": threads1,
                                            "kind": "oracle", "sample": desc1}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def serve_trace(n, seed=2060):
    """Seeded serving trace: all requests arrive at once (request rate inf); prompt and output lengths
    lognormal with means near 223 and 198 tokens (the totals of the page's ShareGPT run, 223,417 input and
    198,203 output tokens over 1000 prompts)."""
    rng = np.random.default_rng(seed)
    sigma = 1.0
    prompts = np.clip(rng.lognormal(np.log(223) - sigma ** 2 / 2, sigma, n), 4, 2048).astype(int)
    outs = np.clip(rng.lognormal(np.log(198) - sigma ** 2 / 2, sigma, n), 1, 1024).astype(int)
    return prompts, outs


def shared_prompt_tokens(prompts, n_systems, system_len, seed=4383):
    """Token ids for the trace's prompts: request r starts with one of n_systems shared system prompts of
    system_len tokens (round robin) and continues with its own ids; its prompt length grows by system_len."""
    rng = np.random.default_rng(seed)
    systems = [rng.integers(0, 32000, system_len).astype(np.int32) for _ in range(n_systems)]
    return [np.concatenate([systems[r % n_systems], rng.integers(0, 32000, int(p)).astype(np.int32)])
            for r, p in enumerate(prompts)]


def run_serve(args):
    """Continuous batching over a seeded trace: the C++ scheduler plans every step, the step runs
    reshape_and_cache, the chunked-prefill kernel and the decode kernel for one attention layer.  With
    --serve-system-prompt L, every prompt starts with one of 8 shared L-token system prompts and goes
    through the prefix cache (its token ids are given; emitted ids are reported each step)."""
    import torch

    import paged_kv_cache_411_b200 as pk

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    H, D, bs = 32, 128, 16
    n = args.serve_requests
    prompts, outs = serve_trace(n)
    toks = None
    if args.serve_system_prompt:
        toks = shared_prompt_tokens(prompts, 8, args.serve_system_prompt)
        prompts = prompts + args.serve_system_prompt
    max_seqs, max_tokens = 256, 8192
    N = args.serve_blocks
    alloc = pk.BlockAllocator(N, bs)
    sched = pk.Scheduler(alloc, max_num_seqs=max_seqs, max_num_tokens=max_tokens)
    for r in range(n):
        sched.add_request(r, int(prompts[r]), int(outs[r]), tokens=None if toks is None else toks[r])
    id_rng = np.random.default_rng(198203)
    kc = torch.zeros((N, bs, H, D), dtype=torch.float16, device=dev)
    vc = torch.zeros_like(kc)
    g = torch.Generator(device=dev).manual_seed(7)
    rows = max_tokens + max_seqs
    kpool = torch.randn((rows, H, D), generator=g, device=dev).half()
    vpool = torch.randn((rows, H, D), generator=g, device=dev).half()
    qpool = torch.randn((rows, H, D), generator=g, device=dev).half()
    mb = -(-int((prompts + outs).max()) // bs)
    ws = torch.empty(pk.decode_workspace_bytes(max_seqs, H, D, mb, bs), dtype=torch.uint8, device=dev)
    out_d = torch.empty((max_seqs, H, D), dtype=torch.float16, device=dev)
    out_p = torch.empty((max_tokens, H, D), dtype=torch.float16, device=dev)
    scale = 1 / np.sqrt(D)
    stream = torch.cuda.current_stream(dev)
    # per-step inputs go up through one pinned staging buffer allocated once at its largest size and sent
    # with one copy per step (an engine reuses it; pinning memory every step would cost more than the
    # scheduling itself)
    layout = [("slots", torch.int64, (rows,)), ("pt", torch.int32, (max_seqs, mb)), ("qs", torch.int32, (max_seqs + 1,)),
              ("ctx", torch.int32, (max_seqs,)), ("dt", torch.int32, (max_seqs, mb)), ("dl", torch.int32, (max_seqs,))]
    offs, total = {}, 0
    for name, dtype, shape in layout:
        nbytes = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        total = (total + 255) // 256 * 256
        offs[name] = (total, nbytes, dtype, shape)
        total += nbytes
    host_buf = torch.empty(total, dtype=torch.uint8).pin_memory()
    dev_buf = torch.empty(total, dtype=torch.uint8, device=dev)
    host_v = {k: host_buf[o:o + nb].view(dt).view(sh).numpy() for k, (o, nb, dt, sh) in offs.items()}
    dev_v = {k: dev_buf[o:o + nb].view(dt).view(sh) for k, (o, nb, dt, sh) in offs.items()}

    def stage(key, arr):
        host_v[key][:arr.shape[0]] = arr
        return dev_v[key][:arr.shape[0]]

    ends, gpu_ms, host_s = [], [], 0.0
    t_start = time.perf_counter()
    while sched.stats()["finished"] < n:
        h0 = time.perf_counter()
        plan = sched.step()
        P, S, T = plan["num_prefill"], plan["num_decode"], plan["num_tokens"]
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if T:
            slots = stage("slots", plan["slot_mapping"])
            if P:
                st, _, _ = alloc.pack(plan["prefill_reqs"], mb, tables=host_v["pt"][:P])   # straight into staging
                if st != pk.PA_OK:
                    raise SystemExit(f"serve: packing the prefill tables failed: {pk.last_error()}")
                q_start = np.concatenate([[0], np.cumsum(plan["prefill_len"])]).astype(np.int32)
                pt_d = dev_v["pt"][:P]
                qs_d = stage("qs", q_start)
                ctx_d = stage("ctx", plan["prefill_ctx"])
            if S:
                st, _, _ = alloc.pack(plan["decode_reqs"], mb, tables=host_v["dt"][:S], lens=host_v["dl"][:S])
                if st != pk.PA_OK:
                    raise SystemExit(f"serve: packing the decode tables failed: {pk.last_error()}")
                dt_d, dl_d = dev_v["dt"][:S], dev_v["dl"][:S]
            dev_buf.copy_(host_buf, non_blocking=True)       # the step's inputs, one copy
            host_s += time.perf_counter() - h0
            ev0.record(stream)
            pk.reshape_and_cache(kpool[:T], vpool[:T], kc, vc, slots, stream=stream)
            if P:
                Tp = int(q_start[-1])
                pk.paged_attention_prefill_chunk(out_p[:Tp], qpool[:Tp], kc, vc, pt_d, qs_d, ctx_d, scale,
                                                 stream=stream)
            if S:
                pk.paged_attention_decode(out_d[:S], qpool[:S], kc, vc, dt_d, dl_d, scale, ws, stream=stream)
            ev1.record(stream)
            stream.synchronize()                     # the step's result goes back to the host
            gpu_ms.append(ev0.elapsed_time(ev1))
        if toks is None:
            sched.complete()
        else:
            # one id per emitted token (requests whose prefill completed, then the decodes)
            n_emit = S + int(sum(1 for r, c, L in zip(plan["prefill_reqs"], plan["prefill_ctx"], plan["prefill_len"])
                                 if c + L == sched.request_info(int(r))[1]["to_prefill"]))
            sched.complete(sampled=id_rng.integers(0, 32000, n_emit))
        ends.append(time.perf_counter() - t_start)
    wall = time.perf_counter() - t_start
    ends = np.asarray(ends)
    ttft, tpot = [], []
    for r in range(n):
        _, info = sched.request_info(r)
        ttft.append(ends[info["first_token_step"]] * 1e3)
        if info["generated"] > 1:
            tpot.append((ends[info["finish_step"]] - ends[info["first_token_step"]]) * 1e3 / (info["generated"] - 1))
    st = sched.stats()

    def dist(x):
        x = np.asarray(x)
        return {"mean": round(float(x.mean()), 3), "median": round(float(np.median(x)), 3),
                "p99": round(float(np.percentile(x, 99)), 3)}

    line = {
        "metric": "serve: output tokens/s of continuous batching over one attention layer", "impl": "ours",
        "value": round(float(outs.sum()) / wall, 1), "unit": "tok/s", "higher_is_better": True,
        "data": "synthetic", "dtype": "f16",
        "config": {"workload": f"serve_trace_{n}req_rate_inf_lognormal223_198"
                   + (f"_system_prompt{args.serve_system_prompt}x8" if toks is not None else ""),
                   "num_heads": H, "head_dim": D,
                   "block_size": bs, "num_blocks": N, "max_num_seqs": max_seqs, "max_num_batched_tokens": max_tokens,
                   "chunked_prefill": True, "input_tokens": int(prompts.sum()), "output_tokens": int(outs.sum())},
        "wall_s": round(wall, 3), "req_per_s": round(n / wall, 2), "steps": st["steps"],
        "preemptions": st["preemptions"], "prefill_tokens": st["prefill_tokens"],
        "gpu_ms_total": round(float(np.sum(gpu_ms)), 2), "host_schedule_s": round(host_s, 3),
        "ttft_ms": dist(ttft), "tpot_ms": dist(tpot),
    }
    if toks is not None:
        cs = alloc.cache_stats()
        # every admission (a preempted request is admitted again) either finds a token's K/V in the cache or
        # prefills it: the hit rate is the cached share of those admitted tokens
        admitted = st["cached_tokens"] + st["prefill_tokens"]
        line["prefix_cache"] = {"cached_prompt_tokens": st["cached_tokens"], "prompt_tokens": int(prompts.sum()),
                                "admitted_prompt_tokens": admitted,
                                "hit_rate": round(st["cached_tokens"] / float(max(1, admitted)), 4),
                                "hit_blocks": cs["hit_blocks"], "evictions": cs["evictions"],
                                "prefix_nodes_at_end": cs["prefix_nodes"], "cached_blocks_at_end": cs["cached_blocks"]}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="b256", choices=sorted(si.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--block-size", type=int, default=0,
                    help="run the workload's requests with this block size instead (block-size sweep)")
    ap.add_argument("--oracle-tokens", type=int, default=40000,
                    help="cached tokens in the cpu_baseline leg's bounded sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay of the step")
    ap.add_argument("--serve", action="store_true",
                    help="continuous-batching run over a seeded trace instead of the single-step benchmark")
    ap.add_argument("--serve-requests", type=int, default=1000)
    ap.add_argument("--serve-blocks", type=int, default=7680)
    ap.add_argument("--serve-system-prompt", type=int, default=0,
                    help="serve: prefix every prompt with one of 8 shared system prompts of this many tokens")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.serve:
        return run_serve(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
