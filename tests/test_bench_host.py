"""Host logic of the benchmark (no GPU): clock-record parsing, the set recall
of the variants, the workload cut for small captures and the peak source."""
import argparse
import os

import numpy as np
import torch

import bench


class _DoneProc:
    """Stands in for a finished nvidia-smi process."""
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler(lines):
    cs = bench.ClockSampler(0)
    cs.proc = _DoneProc()
    cs.lines = lines
    return cs


def test_clock_record_median_under_load_and_reasons():
    # fields: sm, max sm, power, active mask, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    idle = "345, 1965, 150.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    busy = "1965, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active"
    capped = "1800, 1965, 1000.0, 0x4, Not Active, Not Active, Not Active, Active"
    lines = [(0.0, idle), (1.0, busy), (1.1, capped), (1.2, busy), (5.0, idle)]
    rec = _sampler(lines).stop(t_begin=0.9, t_end=1.3)
    assert rec["sm_mhz"] == 1965.0          # median of the samples inside the region
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["samples"] == 3


def test_clock_record_flags_thermal_slowdown():
    hot = "1500, 1965, 1000.0, 0x40, Not Active, Active, Not Active, Not Active"
    rec = _sampler([(1.0, hot)]).stop(t_begin=0.5, t_end=1.5)
    assert rec["reasons"] == ["hw_thermal_slowdown"]


def test_clock_record_without_a_sample_in_the_region_takes_the_nearest():
    s = "1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    rec = _sampler([(10.0, s)]).stop(t_begin=9.0, t_end=9.5)
    assert rec["samples"] == 1 and rec["sm_mhz"] == 1965.0


def test_clock_record_without_nvidia_smi():
    cs = bench.ClockSampler(0)
    assert cs.stop()["reasons"] == ["nvidia-smi unavailable"]


def test_recall_of_token_sets_ignores_padding():
    ref = torch.tensor([[0, 3, 5, -1], [1, 2, 4, 6]], dtype=torch.int32)
    assert bench._recall(ref, ref, 8) == 1.0
    sel = torch.tensor([[0, 3, 7, -1], [-1, -1, -1, -1]], dtype=torch.int32)
    # row 0: 2 of 3 reference tokens found; row 1: none of 4
    assert abs(bench._recall(sel, ref, 8) - 2 / 7) < 1e-12
    # order inside a row does not matter
    assert bench._recall(torch.flip(ref, dims=[1]).contiguous(), ref, 8) == 1.0


def test_workload_cut_keeps_keys_and_positions():
    args = argparse.Namespace(workload="chunk_128k", queries=1024)
    wl = bench._workload(args)
    full = bench.W.WORKLOADS["chunk_128k"]
    assert (wl.n_q, wl.q_pos0, wl.n_k) == (1024, full.q_pos0, full.n_k)
    args.queries = 0
    assert bench._workload(args).n_q == full.n_q
    name = bench._workload_name(wl, wl.h)
    assert name.startswith("chunk_128k: 1024 queries at 122880..123903 x 131072 keys")


def test_peaks_source():
    p = bench._peaks()
    measured = os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json"))
    assert p["source"] == ("measured" if measured else "fallback")
    assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 500


def test_rank_inputs_permute_queries_only():
    inp = {"Q": np.arange(12).reshape(6, 2), "w": np.arange(6.0), "K": np.ones((4, 2))}
    assert bench.rank_inputs(inp, 0, 1) is inp
    r1 = bench.rank_inputs(inp, 1, 2)
    assert r1["K"] is inp["K"]
    order = r1["w"].astype(int)
    assert sorted(order.tolist()) == list(range(6))
    assert np.array_equal(r1["Q"], inp["Q"][order])
