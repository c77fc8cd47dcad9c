"""Benchmark of the MISA token indexer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload chunk_128k] [--h 8]

One step = the whole indexer over one long-context prefill chunk: pool the
131072 keys into 1024 blocks, route every (query, head) against them and keep
the top-8 heads, score the causal prefix of all 8192 queries with their routed
heads and select the top-2048 tokens per query (one fused call: sampled per-row
thresholds, tensor-core scoring with the ReLU * w head-sum and threshold test in
the epilogue, exact selection among the kept logits).  Inputs are seeded synthetic arrays
of the chunk's shape (clustered keys, head-specific query mixtures), resident in
HBM when the timed region starts.  L2 is flushed before every timed step (a
256 MiB write, then a 256 MiB read of another buffer, so no input and no dirty
line is left in it); all times are CUDA events on the launching stream.

N > 1 (torchrun, one process per GPU): every rank indexes its own chunk
(independent problems, no data-path collective), timing is the max over ranks
and `value` is the whole-job milliseconds per chunk (max step time / N).

--impl reference times the CPU oracle (the fp64 restatement of the method) on a
bounded sample of the same workload and extrapolates to the chunk.
"""
from __future__ import annotations

import argparse
import json
import math
import multiprocessing as mp
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from long_context_sparse_block_b200 import workloads as W  # noqa: E402

METRIC = "MISA indexer ms per 8192x131072 chunk; scoring TFLOP/s vs B200 tensor peak"

def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ------------------------------------------------------------------ clocks

class L2Flush:
    """Empties L2 between timed steps: a 256 MiB write (evicts every input line),
    then a 256 MiB read of a second buffer, which writes the first one's dirty
    lines back before the timed region instead of inside it."""

    def __init__(self):
        import torch
        self.w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        self.r = torch.zeros(32 * 1024 * 1024, dtype=torch.int64, device="cuda")

    def __call__(self):
        self.w.zero_()
        self.r.max()


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def wait_first(self, timeout=5.0):
        """Blocks until nvidia-smi has produced its first sample (it starts slowly)."""
        t0 = time.monotonic()
        while self.proc is not None and not self.lines and time.monotonic() - t0 < timeout:
            time.sleep(0.01)

    def mark(self):
        return time.monotonic()

    def stop(self, t_begin=None, t_end=None):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = [ln for t, ln in self.lines
                 if t_begin is None or (t_begin <= t <= t_end + 0.05)]
        if not lines and self.lines:  # nothing inside: the sample nearest the region
            lines = [min(self.lines, key=lambda x: abs(x[0] - (t_begin or 0.0)))[1]]
        for ln in lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        loaded = [x for x in sm if mx and x > 0.3 * mx] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle baseline

_SHARED = {}


def _oracle_worker(rows):
    """One single-threaded oracle over query rows (route + score + top-k each)."""
    import oracle
    wl, h = _SHARED["wl"], _SHARED["h"]
    Kd, kbar, inp = _SHARED["Kd"], _SHARED["kbar"], _SHARED["inp"]
    Qd_rows = oracle.bf16_to_f64(inp["Q"][rows])
    wd = inp["w"][rows].astype(np.float64)
    t0 = time.perf_counter()
    for i, t in enumerate(rows):
        pos = wl.q_pos0 + int(t)
        r, hd = oracle.route(Qd_rows[i:i + 1], wd[i:i + 1], kbar, pos, wl.n_k, wl.B, h)
        lg = oracle.score(Qd_rows[i:i + 1], wd[i:i + 1], hd, Kd, pos)
        oracle.topk(lg, pos, wl.n_k, wl.k)
    return time.perf_counter() - t0, len(rows)


def _oracle_setup(wl: W.Workload, h: int, inp: dict) -> int:
    """Builds the oracle, pools the keys once and returns the worker count (one
    single-threaded oracle process per host core, at most 32)."""
    import oracle
    oracle.build()
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    Kd = oracle.bf16_to_f64(inp["K"])
    _SHARED.update(wl=wl, h=h, inp=inp, Kd=Kd, kbar=oracle.pool_keys(Kd, wl.B))
    return max(1, min(cores, 32))


def _oracle_step(pool, workers: int, rows) -> tuple:
    """One sample: the rows split over the worker processes.  Returns (wall s,
    summed single-thread s, rows)."""
    parts = [rows[i::workers].tolist() for i in range(workers)]
    t0 = time.perf_counter()
    res = pool.map(_oracle_worker, [p for p in parts if p])
    return time.perf_counter() - t0, sum(t for t, _ in res), sum(n for _, n in res)


def cpu_baseline(wl: W.Workload, h: int, inp: dict, budget_s: float = 15.0) -> dict:
    """Times the oracle as it stands (route + score + top-k per query; keys pooled
    once) on a seeded sample of query rows, one single-threaded oracle process per
    core, and extrapolates to milliseconds per chunk.  Must run before any CUDA
    call: the worker processes are forked."""
    workers = _oracle_setup(wl, h, inp)
    rng = np.random.default_rng(12345)
    cal_t, _ = _oracle_worker([wl.n_q - 1])
    per_worker = max(1, min(64, int(budget_s / max(cal_t, 1e-3))))
    n_rows = min(wl.n_q, per_worker * workers)
    rows = np.sort(rng.choice(wl.n_q, size=n_rows, replace=False))
    with mp.get_context("fork").Pool(workers) as pool:
        wall, busy, done = _oracle_step(pool, workers, rows)
    per_query = busy / done   # single-thread s/query
    ms_chunk = per_query * wl.n_q / workers * 1e3
    return {"value": round(ms_chunk, 1), "unit": "ms", "cores": workers, "kind": "oracle",
            "sample": f"{n_rows} of {wl.n_q} query rows of {wl.name} (route + score + top-k "
                      f"each), {workers} single-threaded oracle processes, {wall:.1f} s wall; "
                      f"extrapolated to the whole chunk",
            "per_query_s": round(per_query, 4)}


# ------------------------------------------------------------------ GPU arm

def _workload(args):
    """The named workload, cut to its first --queries queries when given (for
    small profiling captures; the keys and query positions are unchanged)."""
    import dataclasses
    wl = W.WORKLOADS[args.workload]
    if args.queries and args.queries < wl.n_q:
        wl = dataclasses.replace(wl, n_q=args.queries)
    return wl


def _workload_name(wl, h: int) -> str:
    return (f"{wl.name}: {wl.n_q} queries at {wl.q_pos0}..{wl.q_pos0 + wl.n_q - 1} "
            f"x {wl.n_k} keys, H_I={wl.H}, d={wl.d}, B={wl.B}, h={h}, k={wl.k}")


def rank_inputs(inp: dict, rank: int, world: int) -> dict:
    """Every rank indexes its own chunk of the same shape: the shared keys and its
    own seeded permutation of the queries (and their head weights)."""
    if world <= 1:
        return inp
    perm = np.random.default_rng(1000 + rank).permutation(inp["Q"].shape[0])
    out = dict(inp)
    out["Q"], out["w"] = inp["Q"][perm].copy(), inp["w"][perm].copy()
    return out


def max_over_ranks(x: float, device) -> float:
    """The largest value over the ranks of the process group (x itself alone)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_ms(ms_max: float, world: int) -> float:
    """Whole-job milliseconds per chunk: `world` chunks finish in the slowest
    rank's time."""
    return ms_max / world


def run_ours(args, rank, world, local_rank, inp):
    import torch
    import torch.distributed as dist

    from long_context_sparse_block_b200 import _lib
    from long_context_sparse_block_b200.indexer import IndexerShape, MisaIndexer

    torch.cuda.set_device(local_rank)
    wl = _workload(args)
    h = args.h or wl.h
    inp = rank_inputs(inp, rank, world)

    def d16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()

    Q, K, w = d16(inp["Q"]), d16(inp["K"]), torch.from_numpy(inp["w"]).cuda()
    shape = IndexerShape(wl.n_q, wl.q_pos0, wl.n_k, wl.H, wl.d, wl.B, h, wl.k,
                         sub_chunk=args.sub_chunk)
    ix = MisaIndexer(shape)
    stream = torch.cuda.current_stream()
    flush = L2Flush()

    # per-stage events: pool and route from torch events around their calls;
    # the stages inside the fused score + top-k call from the library's own
    # profiler (events recorded on the same stream between its launches)
    stage_events = []

    def step(record):
        ev = []
        s = shape
        e0 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        _lib.misa_pool_keys(K, s.B, kbar_hl=ix.kbar_hl, want_kbar=False)
        e1 = torch.cuda.Event(enable_timing=True)
        e1.record(stream)
        _lib.misa_route_heads(Q, w, ix.kbar_hl, s.q_pos0, s.n_k, s.B, s.h, heads=ix.heads)
        e2 = torch.cuda.Event(enable_timing=True)
        e2.record(stream)
        ev += [("pool", e0, e1), ("route", e1, e2)]
        for c0 in range(0, s.n_q, ix.sub):
            c1 = min(s.n_q, c0 + ix.sub)
            _lib.misa_score_topk(Q[c0:c1], w[c0:c1], ix.heads[c0:c1], K, s.q_pos0 + c0, s.k,
                                 h=s.h, idx=ix.sel[c0:c1], logits=ix.logits[:c1 - c0],
                                 ws=ix.ws_sel)
        e3 = torch.cuda.Event(enable_timing=True)
        e3.record(stream)
        ev += [("score_topk", e2, e3)]
        if record:
            stage_events.append(ev)
        return e0, e3

    fused = _lib.misa_workspace_size("score_topk", ix.sub, wl.n_k, wl.k, 0) > 0
    launches_per_step = 2 + (7 if fused else 2) * math.ceil(wl.n_q / ix.sub)
    for _ in range(args.warmup):
        flush()
        step(False)
    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
        clocks.wait_first()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_begin = time.monotonic()
    _lib.misa_profile_start()
    spans = []
    for _ in range(args.steps):
        flush()
        spans.append(step(True))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_end = time.monotonic()
    clk = clocks.stop(t_begin, t_end) if rank == 0 else None
    fused_stages = _lib.misa_profile_stop()
    repaired = int(ix.ws_sel[4:4 * (ix.sub + 1)].view(torch.int32).sum()) if fused else None
    assert _lib.misa_last_device_status() == 0, "device status"
    step_ms = [a.elapsed_time(b) for a, b in spans]
    variants = None
    if rank == 0 and world == 1 and not args.no_variants and args.workload == "chunk_128k":
        del ix
        variants = run_variants(wl, inp, stream, flush)
        ix = MisaIndexer(shape)
        assert _lib.misa_last_device_status() == 0, "device status"
    stage_ms = {}
    for ev in stage_events:
        for name, a, b in ev:
            stage_ms[name] = stage_ms.get(name, 0.0) + a.elapsed_time(b)
    stage_ms = {k: v / args.steps for k, v in stage_ms.items()}
    for name, (tot, cnt) in fused_stages.items():
        if cnt:
            stage_ms[name] = tot / args.steps
    ms = max_over_ranks(statistics.mean(step_ms), "cuda")

    # ---- end to end through the public API from pinned host buffers
    Qh = torch.from_numpy(inp["Q"].view(np.int16)).pin_memory()
    Kh = torch.from_numpy(inp["K"].view(np.int16)).pin_memory()
    wh = torch.from_numpy(inp["w"]).pin_memory()
    idx_h = torch.empty(ix.final.shape, dtype=torch.int32).pin_memory()
    e2e_ms = []
    for i in range(0 if args.no_e2e else args.warmup + args.steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        ix.run_host(Qh, Kh, wh, out=idx_h)   # copies in, indexes, copies out (overlapped)
        b.record(stream)
        b.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e = max_over_ranks(statistics.mean(e2e_ms) if e2e_ms else float("nan"), "cuda")
    if rank != 0:
        return None

    peaks = _peaks()
    pairs = wl.causal_pairs()
    score_flops = 2.0 * h * wl.d * pairs
    score_key = "select_score" if "select_score" in stage_ms else "score_topk"
    score_ms = stage_ms[score_key]
    tflops = score_flops / (score_ms * 1e-3) / 1e12
    pool_gbs = (wl.n_k * wl.d * 2 + 2 * wl.M * wl.d * 2) / (stage_ms["pool"] * 1e-3) / 1e9
    # router: the method's work is H_I * d multiply-adds per (query, complete
    # causal block); the kernel runs that contraction twice (the hi and lo bf16
    # halves of the pooled keys), reported separately
    blocks = sum(min((p + 1) // wl.B, wl.n_k // wl.B) for p in wl.positions().tolist())
    route_flops = 2.0 * wl.H * wl.d * blocks
    route_tflops = route_flops / (stage_ms["route"] * 1e-3) / 1e12
    h2d = inp["Q"].nbytes + inp["K"].nbytes + inp["w"].nbytes
    d2h = idx_h.numel() * 4
    out = {
        "metric": METRIC,
        "value": round(whole_job_ms(ms, world), 4),
        "unit": "ms",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": _workload_name(wl, h),
            "query_sub_chunk": ix.sub,
            "fused_score_topk": fused,
            "rows_repaired_last_subchunk": repaired,
            "l2": "flushed before every timed step: a 256 MiB write, then a 256 MiB read of another buffer (no input and no dirty line left in L2)",
            "parallelism": f"independent chunks per rank x{world}",
        },
        "roofline": {
            "bound": "tensor",
            "kernel": ("score_tokens select mode (tcgen05, fused ReLU*w head-sum, "
                       "threshold + pass-mask epilogue)"),
            "achieved": round(tflops, 1),
            "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s",
            "frac": round(tflops / peaks["bf16_tflops"], 4),
            "peak_source": f"{peaks['source']} bf16 burst (cuBLAS)",
            "traffic": None,
            "algorithmic": f"2*h*d*pairs = {score_flops:.4g} flop per step, {pairs} causal pairs",
            "launches_per_step": math.ceil(wl.n_q / ix.sub),
        },
        "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "stage_rates": {
            "score_tflops": round(tflops, 1),
            "route_tflops": round(route_tflops, 1),
            "route_frac": round(route_tflops / peaks["bf16_tflops"], 4),
            "route_tflops_issued_hi_lo": round(2.0 * route_tflops, 1),
            "pool_gbs": round(pool_gbs, 1),
            "hbm_peak_gbs": peaks["hbm_gbs"],
            "pairs_per_s": round(pairs / (ms * 1e-3), 1),
        },
        "e2e": {"value": round(whole_job_ms(e2e, world), 4) if e2e_ms else None, "unit": "ms", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if variants is not None:
        out["variants"] = variants
    return out


def _time_ms(fn, stream, flush, reps=5, warm=2):
    import torch
    ts = []
    for i in range(warm + reps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        if i >= warm:
            ts.append(a.elapsed_time(b))
    return statistics.mean(ts)


def _recall(sel, ref, n_k):
    """Mean over rows of |sel & ref| / |ref| (token sets, -1 padding ignored)."""
    import torch
    hit = tot = 0
    for r0 in range(0, ref.shape[0], 512):
        a, b = sel[r0:r0 + 512].long(), ref[r0:r0 + 512].long()
        mark = torch.zeros((b.shape[0], n_k + 1), dtype=torch.bool, device=b.device)
        mark.scatter_(1, torch.where(b >= 0, b, n_k), True)
        mark[:, n_k] = False
        hit += int(mark.gather(1, torch.where(a >= 0, a, n_k)).sum())
        tot += int((b >= 0).sum())
    return hit / max(tot, 1)


class DecodeBatch:
    """A batched decode step: n_seq sequences of the chunk's n_k keys each in one
    page pool (every sequence its own copy of the chunk's keys, in its own
    seeded page order), one new query each (rows of the chunk's queries)."""

    def __init__(self, wl, Q, K, w, n_seq: int = 64, ps: int = 64, k_scale=None):
        """K: bf16 codes [n_k, d], or e4m3 codes (uint8) with k_scale [n_k]."""
        import torch

        from long_context_sparse_block_b200 import _lib
        from long_context_sparse_block_b200 import workloads as Wm
        self.lib, self.wl, self.n_seq = _lib, wl, n_seq
        nb = wl.n_k // ps
        table, n_pages = Wm.page_table(n_seq * wl.n_k, ps, seed=65)
        self.pages = torch.empty((n_pages, ps, wl.d), dtype=K.dtype, device="cuda")
        self.bts = torch.from_numpy(table.reshape(n_seq, nb).copy()).cuda()
        self.ks = None
        if k_scale is not None:
            self.ks = torch.ones((n_pages, ps), dtype=torch.float32, device="cuda")
        Kp = K.view(nb, ps, wl.d)
        for b in range(n_seq):
            self.pages[self.bts[b].long()] = Kp
            if self.ks is not None:
                self.ks[self.bts[b].long()] = k_scale.view(nb, ps)
        self.lens = torch.full((n_seq,), wl.n_k, dtype=torch.int32, device="cuda")
        self.Q = Q[-n_seq:].contiguous()
        self.w = w[-n_seq:].contiguous()
        self.M_max = -(-wl.n_k // wl.B)
        _, self.hl = _lib.misa_decode_pool_keys(self.pages, self.bts, self.lens, wl.B, self.M_max,
                                                self.M_max, k_scale=self.ks)
        self.heads = torch.empty((n_seq, wl.h), dtype=torch.int32, device="cuda")
        self.idx = torch.empty((n_seq, wl.k), dtype=torch.int32, device="cuda")
        self.lg = torch.empty((n_seq, wl.n_k), dtype=torch.float32, device="cuda")
        self.key_bytes = n_seq * wl.n_k * wl.d * K.element_size()
        self.step()

    def score_topk(self):
        self.lib.misa_decode_score_topk(self.Q, self.w, self.heads, self.pages, self.bts,
                                        self.lens, self.wl.k, idx=self.idx, logits=self.lg,
                                        k_scale=self.ks)

    def step(self):
        wl = self.wl
        self.lib.misa_decode_pool_keys(self.pages, self.bts, self.lens, wl.B, self.M_max, 1,
                                       kbar_hl=self.hl, k_scale=self.ks)
        self.lib.misa_decode_route_heads(self.Q, self.w, self.hl, self.lens, wl.B, wl.h,
                                         heads=self.heads)
        self.score_topk()


def run_decode_part(args):
    """--part decode: only the batched decode step, for profiling captures."""
    import torch
    wl = W.WORKLOADS["chunk_128k"]
    inp = W.generate(wl)

    def d16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()

    dec = DecodeBatch(wl, d16(inp["Q"]), d16(inp["K"]), torch.from_numpy(inp["w"]).cuda())
    flush = L2Flush()
    ms = _time_ms(dec.step, torch.cuda.current_stream(), flush, reps=args.steps, warm=args.warmup)
    return {"part": "decode", "n_seq": dec.n_seq, "n_k": wl.n_k, "h": wl.h, "k": wl.k,
            "ms_per_step": round(ms, 4), "key_gbs": round(dec.key_bytes / (ms * 1e-3) / 1e9, 1)}


def run_topk_part(args):
    """--part topk: only the standalone top-k over the chunk's fused logits (the
    unfused path's selection), for profiling captures; --queries cuts the rows."""
    import torch
    from long_context_sparse_block_b200 import _lib
    wl = _workload(args)
    inp = W.generate(wl)

    def d16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()

    Q, K, w = d16(inp["Q"]), d16(inp["K"]), torch.from_numpy(inp["w"]).cuda()
    _, hl = _lib.misa_pool_keys(K, wl.B)
    heads, _ = _lib.misa_route_heads(Q, w, hl, wl.q_pos0, wl.n_k, wl.B, wl.h)
    lg = _lib.misa_score_tokens(Q, w, heads, K, wl.q_pos0)
    del Q
    idx = torch.empty((wl.n_q, wl.k), dtype=torch.int32, device="cuda")
    ms = _time_ms(lambda: _lib.misa_topk(lg, wl.q_pos0, wl.n_k, wl.k, idx=idx),
                  torch.cuda.current_stream(), L2Flush(), reps=args.steps, warm=args.warmup)
    # bytes: every visible logit of every row, read once
    n_vis = sum(min(wl.q_pos0 + t + 1, wl.n_k) for t in range(wl.n_q))
    gbs = n_vis * 4 / (ms * 1e-3) / 1e9
    return {"part": "topk", "n_q": wl.n_q, "n_k": wl.n_k, "k": wl.k, "ms_per_step": round(ms, 4),
            "logit_gbs": round(gbs, 1), "hbm_frac": round(gbs / _peaks()["hbm_gbs"], 3)}


def run_variants(wl, inp, stream, flush):
    """The other measured configurations: on the chunk, h=4, the dense 64-head
    indexer in this library, MISA-dagger (k'=8192, all-head rerank to 2048) with
    bf16 and with FP8 keys (with the recall of each against the dense top-k), the
    unfused score + top-k sequence, the scoring with e4m3 queries and keys, one
    decode step on the full cache; and the
    DeepSeek-V3.2- and GLM-5-shaped whole-sequence prefills (32768 and 65536
    tokens)."""
    import torch

    from long_context_sparse_block_b200 import workloads as Wm
    from long_context_sparse_block_b200.indexer import IndexerShape, MisaIndexer

    def d16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()

    Q, K, w = d16(inp["Q"]), d16(inp["K"]), torch.from_numpy(inp["w"]).cuda()
    base = dict(n_q=wl.n_q, q_pos0=wl.q_pos0, n_k=wl.n_k, H=wl.H, d=wl.d, B=wl.B, k=wl.k)
    out = {}
    dense = MisaIndexer(IndexerShape(h=wl.H, dense=True, **base))
    out["dense_h64_ms"] = round(_time_ms(lambda: dense.run(Q, K, w), stream, flush), 4)
    ref = dense.run(Q, K, w).clone()
    for h in (8, 4):
        ix = MisaIndexer(IndexerShape(h=h, **base))
        out[f"misa_h{h}_ms"] = round(_time_ms(lambda: ix.run(Q, K, w), stream, flush), 4)
        out[f"misa_h{h}_recall_vs_dense"] = round(_recall(ix.run(Q, K, w), ref, wl.n_k), 4)
    dg = MisaIndexer(IndexerShape(h=wl.h, kp=8192, **base))
    out["dagger_ms"] = round(_time_ms(lambda: dg.run(Q, K, w), stream, flush), 4)
    out["dagger_recall_vs_dense"] = round(_recall(dg.run(Q, K, w), ref, wl.n_k), 4)
    del dense, ref, dg
    # FP8 keys (e4m3 + per-token scale): pooling and the rerank read the codes,
    # the fused scoring their bf16 decode (made once per chunk by the indexer)
    K8c, sc = Wm.e4m3_quantize_keys(Wm.bf16_values(inp["K"]).astype(np.float64))
    K8 = torch.from_numpy(K8c).cuda()
    ks = torch.from_numpy(sc).cuda()
    dense8 = MisaIndexer(IndexerShape(h=wl.H, dense=True, **base))
    ref8 = dense8.run(Q, K8, w, k_scale=ks).clone()
    del dense8
    dg8 = MisaIndexer(IndexerShape(h=wl.h, kp=8192, **base))
    out["dagger_fp8_ms"] = round(_time_ms(lambda: dg8.run(Q, K8, w, k_scale=ks), stream, flush), 4)
    fin8 = dg8.run(Q, K8, w, k_scale=ks)
    out["dagger_fp8_recall_vs_dense_fp8"] = round(_recall(fin8, ref8, wl.n_k), 4)
    dense_bf = MisaIndexer(IndexerShape(h=wl.H, dense=True, **base))
    out["dagger_fp8_recall_vs_dense_bf16"] = round(_recall(fin8, dense_bf.run(Q, K, w), wl.n_k), 4)
    del dense_bf, dg8, fin8, ref8, K8, ks     # (K8c, sc stay on the host)

    # end to end from pinned host buffers with three piece schedules (the main
    # e2e figure uses run_host's default, the ramp)
    from long_context_sparse_block_b200.indexer import ramp_pieces
    ixh = MisaIndexer(IndexerShape(h=wl.h, **base))
    Qh = torch.from_numpy(inp["Q"].view(np.int16)).pin_memory()
    Kh = torch.from_numpy(inp["K"].view(np.int16)).pin_memory()
    wh = torch.from_numpy(inp["w"]).pin_memory()
    idx_h = torch.empty((wl.n_q, wl.k), dtype=torch.int32).pin_memory()
    for label, pcs in (("p4", 4), ("p8", 8), ("ramp", ramp_pieces(wl.n_q))):
        out[f"e2e_{label}_ms"] = round(_time_ms(lambda: ixh.run_host(Qh, Kh, wh, out=idx_h, pieces=pcs),
                                                stream, flush), 4)
    # where the end-to-end time goes: events on the three streams of one run
    tl = []
    flush()
    ixh.run_host(Qh, Kh, wh, out=idx_h, timeline=tl)
    torch.cuda.synchronize()
    t0 = tl[0][1]
    out["e2e_ramp_timeline_ms"] = {label: round(t0.elapsed_time(ev), 3) for label, ev in tl[1:]}
    del ixh, Qh, Kh, wh, idx_h

    # the same chunk with its keys in a paged cache (pages of 64 keys in a
    # seeded random order in a larger pool, unused rows filled with +inf codes):
    # the indices must equal the contiguous ones
    from long_context_sparse_block_b200 import _lib as L
    ps = 64
    table, n_pages = Wm.page_table(wl.n_k, ps, seed=64)
    pages = torch.full((n_pages, ps, wl.d), 0x7F80, dtype=torch.int16, device="cuda")
    bt = torch.from_numpy(table).cuda()
    n_blocks = len(table)
    flat = torch.full((n_blocks * ps, wl.d), 0x7F80, dtype=torch.int16, device="cuda")
    flat[:wl.n_k] = K
    pages[bt.long()] = flat.view(n_blocks, ps, wl.d)
    del flat
    pk = L.PagedKeys(pages, bt, wl.n_k)
    ixp = MisaIndexer(IndexerShape(h=wl.h, **base))
    out["paged_chunk_ms"] = round(_time_ms(lambda: ixp.run(Q, pk, w), stream, flush), 4)
    sel_p = ixp.run(Q, pk, w).clone()
    sel_c = ixp.run(Q, K, w)
    out["paged_chunk_equal_contiguous"] = bool(torch.equal(sel_p, sel_c))
    out["paged_page_size"] = ps
    del ixp, pk, pages, bt, sel_p, sel_c

    # the unfused sequence on the chunk: every logit written (store mode), then
    # the standalone top-k reading them once (HBM-bound: 4 bytes per causal pair)
    from long_context_sparse_block_b200 import _lib
    ixu = MisaIndexer(IndexerShape(h=wl.h, **base))
    ixu.run(Q, K, w)   # routes the heads
    lg = ixu.logits
    pairs = wl.causal_pairs()
    t_s = _time_ms(lambda: _lib.misa_score_tokens(Q, w, ixu.heads, K, wl.q_pos0, logits=lg, h=wl.h),
                   stream, flush)
    t_k = _time_ms(lambda: _lib.misa_topk(lg, wl.q_pos0, wl.n_k, wl.k, idx=ixu.sel), stream, flush)
    out["unfused_score_ms"] = round(t_s, 4)
    out["unfused_score_tflops"] = round(2.0 * wl.h * wl.d * pairs / (t_s * 1e-3) / 1e12, 1)
    out["unfused_topk_ms"] = round(t_k, 4)
    out["unfused_topk_logit_gbs"] = round(4.0 * pairs / (t_k * 1e-3) / 1e9, 1)

    # the same scoring with e4m3 queries and keys (a scale per (query, head) row
    # and per key) multiplied as e4m3 on the tensor cores, and the top-2048 of
    # those logits against the bf16 selection
    Q8c, qs = Wm.e4m3_quantize_queries(Wm.bf16_values(inp["Q"]).astype(np.float64))
    Q8, qsc = torch.from_numpy(Q8c).cuda(), torch.from_numpy(qs).cuda()
    K8, ks = torch.from_numpy(K8c).cuda(), torch.from_numpy(sc).cuda()
    del Q8c
    sel_bf16 = ixu.sel.clone()
    t_8 = _time_ms(lambda: _lib.misa_score_tokens_fp8(Q8, qsc, w, ixu.heads, K8, ks, wl.q_pos0,
                                                      logits=lg, h=wl.h), stream, flush)
    out["fp8_qk_score_ms"] = round(t_8, 4)
    out["fp8_qk_score_tflops"] = round(2.0 * wl.h * wl.d * pairs / (t_8 * 1e-3) / 1e12, 1)
    _lib.misa_topk(lg, wl.q_pos0, wl.n_k, wl.k, idx=ixu.sel)
    out["fp8_qk_recall_vs_bf16"] = round(_recall(ixu.sel, sel_bf16, wl.n_k), 4)
    del Q8, qsc, K8, ks, sel_bf16

    # one decode step on the full cache: the newest query (position n_k - 1)
    # after its key was appended: re-pool the last block, route, score, select
    M = -(-wl.n_k // wl.B)
    kbar_hl = ixu.kbar_hl
    q1, w1 = Q[-1:].contiguous(), w[-1:].contiguous()
    heads1 = torch.empty((1, wl.h), dtype=torch.int32, device="cuda")
    lg1 = torch.empty((1, (wl.n_k + 3) // 4 * 4), dtype=torch.float32, device="cuda")[:, :wl.n_k]
    idx1 = torch.empty((1, wl.k), dtype=torch.int32, device="cuda")

    def decode_step():
        _lib.misa_pool_keys_range(K, wl.B, M - 1, M, kbar_hl=kbar_hl)
        _lib.misa_route_heads(q1, w1, kbar_hl, wl.n_k - 1, wl.n_k, wl.B, wl.h, heads=heads1)
        _lib.misa_score_tokens(q1, w1, heads1, K, wl.n_k - 1, logits=lg1, h=wl.h)
        _lib.misa_topk(lg1, wl.n_k - 1, wl.n_k, wl.k, idx=idx1)

    out["decode_step_ms"] = round(_time_ms(decode_step, stream, flush), 4)

    # batched decode: 64 sequences of 131072 keys each in one page pool, one
    # new query each (re-pool each sequence's last block, route, score, select)
    dec = DecodeBatch(wl, Q, K, w)
    t_db = _time_ms(dec.step, stream, flush)
    t_ds = _time_ms(dec.score_topk, stream, flush)
    out["decode_batch64_ms"] = round(t_db, 4)
    out["decode_batch64_score_topk_ms"] = round(t_ds, 4)
    out["decode_batch64_key_gbs"] = round(dec.key_bytes / (t_ds * 1e-3) / 1e9, 1)
    del dec
    # the same with the caches in e4m3 (a scale per key): half the bytes
    dec8 = DecodeBatch(wl, Q, torch.from_numpy(K8c).cuda(), w, k_scale=torch.from_numpy(sc).cuda())
    t_8 = _time_ms(dec8.score_topk, stream, flush)
    out["decode_batch64_fp8_ms"] = round(_time_ms(dec8.step, stream, flush), 4)
    out["decode_batch64_fp8_score_topk_ms"] = round(t_8, 4)
    out["decode_batch64_fp8_key_gbs"] = round(dec8.key_bytes / (t_8 * 1e-3) / 1e9, 1)
    del dec8
    del ixu, lg, Q, K, w

    # the prefill configurations (whole-sequence prefill, the fused path per
    # 8192-query sub-chunk; the first sub-chunk, whose prefix is shorter than
    # the 4096-key sample, takes the unfused sequence)
    for name in ("dsv32_32k", "glm5_64k"):
        cw = Wm.WORKLOADS[name]
        ci = Wm.generate(cw)
        Qc, Kc, wc = d16(ci["Q"]), d16(ci["K"]), torch.from_numpy(ci["w"]).cuda()
        ixc = MisaIndexer(IndexerShape(cw.n_q, cw.q_pos0, cw.n_k, cw.H, cw.d, cw.B, cw.h, cw.k))
        t = _time_ms(lambda: ixc.run(Qc, Kc, wc), stream, flush)
        _lib.misa_profile_start()
        ixc.run(Qc, Kc, wc)
        st = _lib.misa_profile_stop()
        cp = cw.causal_pairs()
        sel_ms = st["select_score"][0]
        # pairs of the sub-chunks that ran the select pass (prefix >= the sample)
        fused_pairs = sum(
            sum(cw.q_pos0 + t + 1 for t in (c0, c1 - 1)) * (c1 - c0) // 2
            for c0, c1 in ((c0, min(cw.n_q, c0 + ixc.sub)) for c0 in range(0, cw.n_q, ixc.sub))
            if cw.q_pos0 + c0 + 1 >= 4096)
        out[f"{name}_ms"] = round(t, 4)
        out[f"{name}_pairs_per_s"] = round(cp / (t * 1e-3), 1)
        out[f"{name}_select_tflops"] = (
            round(2.0 * cw.h * cw.d * fused_pairs / (sel_ms * 1e-3) / 1e12, 1) if sel_ms > 0 else None)
        del ixc, Qc, Kc, wc, ci
    return out


def run_reference(args, rank):
    """The oracle arm: W warm-up and K timed steps, each step the oracle over a
    fresh seeded sample of query rows (one single-threaded process per host
    core, about --ref-step-s seconds of wall time); a step's time is its wall
    time, and the value is each step's time per row scaled to the whole chunk,
    averaged over the timed steps."""
    if rank != 0:
        return None
    wl = W.WORKLOADS[args.workload]
    h = args.h or wl.h
    t_start = time.perf_counter()
    workers = _oracle_setup(wl, h, W.generate(wl))
    cal_t, _ = _oracle_worker([wl.n_q - 1])
    rows_per_step = min(wl.n_q, workers * max(1, int(args.ref_step_s / max(cal_t, 1e-3))))
    rng = np.random.default_rng(54321)
    walls, chunk_ms = [], []
    with mp.get_context("fork").Pool(workers) as pool:
        for i in range(args.warmup + args.steps):
            rows = np.sort(rng.choice(wl.n_q, size=rows_per_step, replace=False))
            wall, _, done = _oracle_step(pool, workers, rows)
            if i >= args.warmup:
                walls.append(wall)
                chunk_ms.append(wall * wl.n_q / done * 1e3)
    value = statistics.mean(chunk_ms)
    world = int(os.environ.get("WORLD_SIZE", 1))
    return {"metric": METRIC, "value": round(value, 1), "unit": "ms", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(statistics.mean(walls) * 1e3, 1),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "extrapolated": True,
            "config": {"workload": _workload_name(wl, h),
                       "sample_rows_per_step": rows_per_step,
                       "parallelism": f"{workers} single-threaded oracle processes on the host"},
            "cpu_baseline": {"value": round(value, 1), "unit": "ms", "cores": workers,
                             "kind": "oracle",
                             "sample": f"each step: {rows_per_step} seeded query rows of "
                                       f"{wl.n_q} (route + score + top-k each); the step's wall "
                                       f"time scaled by {wl.n_q}/{rows_per_step}"},
            "e2e": {"value": round(value, 1), "unit": "ms", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": round(time.perf_counter() - t_start, 1)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="chunk_128k")
    ap.add_argument("--h", type=int, default=0)
    ap.add_argument("--sub-chunk", type=int, default=8192)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-step-s", type=float, default=1.0,
                    help="oracle arm: wall seconds per step (each step a sample of rows)")
    ap.add_argument("--queries", type=int, default=0,
                    help="index only the first N queries of the chunk (profiling captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass (profiling)")
    ap.add_argument("--part", default="", choices=["", "decode", "topk"],
                    help="run one part alone for profiling captures (decode: the batched step)")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the h=4 / dense / MISA-dagger / FP8 measurements")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))

    if args.part == "topk":
        print(json.dumps(run_topk_part(args)), flush=True)
        return
    if args.part == "decode":
        print(json.dumps(run_decode_part(args)), flush=True)
        return

    if args.impl == "reference":
        out = run_reference(args, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    # the oracle's process pool is forked before any CUDA work (a fork after it would hang)
    wl = _workload(args)
    inp = W.generate(W.WORKLOADS[args.workload])  # each rank indexes its own chunk (same shape)
    if wl.n_q < inp["Q"].shape[0]:
        inp["Q"], inp["w"] = inp["Q"][:wl.n_q].copy(), inp["w"][:wl.n_q].copy()
    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(wl, args.h or wl.h, inp, budget_s=args.cpu_budget)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank, inp)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if out is not None:
        if cb is not None:
            out["cpu_baseline"] = cb
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
