"""Host-side pieces of bench.py that need no GPU: the clock sampler's time-window summary."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def test_clock_summary_keeps_only_the_window():
    import bench
    cs = bench.ClockSampler(0)
    cs.proc = object()   # pretend nvidia-smi started; rows are injected below
    cs.rows = [(0.5, 1965.0, 1965.0, set()),                   # idle, before the window
               (1.1, 1740.0, 1965.0, {"sw_power_cap"}),
               (1.2, 1750.0, 1965.0, {"sw_power_cap"}),
               (1.3, 1760.0, 1965.0, set()),
               (2.5, 1965.0, 1965.0, set())]                   # idle, after the window
    got = cs.summary(1.0, 2.0)
    assert got["samples"] == 3
    assert got["sm_mhz"] == 1750.0
    assert got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]
    empty = cs.summary(3.0, 4.0)
    assert empty["samples"] == 0 and empty["sm_mhz"] is None


def test_clock_summary_without_nvidia_smi():
    import bench
    cs = bench.ClockSampler(0)
    got = cs.summary(0.0, 1.0)
    assert got["reasons"] == ["nvidia-smi unavailable"] and got["samples"] == 0


def test_recorded_traffic_follows_the_sources():
    """The decode call's DRAM bytes are reported only while the kernel sources hash to the digest
    recorded with them (a changed kernel reports null, not a stale number)."""
    import bench
    rec = bench.MEASURED_TRAFFIC["b32_l4096"]
    assert bench.recorded_traffic("b32_l4096") in (None, rec["bytes"])
    assert bench.recorded_traffic("no_such_workload") is None
    saved = rec["sha256"]
    try:
        rec["sha256"] = "0" * 64
        assert bench.recorded_traffic("b32_l4096") is None
    finally:
        rec["sha256"] = saved


def test_job_throughput_is_whole_job():
    """value = the bytes every rank processed over the max-over-ranks time."""
    import bench
    assert abs(bench.job_throughput(1e9, 1, 1.0) - 1000.0) < 1e-9
    assert abs(bench.job_throughput(1e9, 4, 2.0) - 2000.0) < 1e-9


def test_step_work_counts_bytes_and_flops():
    """Per cached token per layer: 1152 bytes and 2*128*(576 + 512) flops; per sequence the absorb
    and un-absorb GEMMs (2 x 2*128*128*512 flops); the decode call's bytes add q_full in and out_lat
    out per sequence."""
    import bench
    lens = [3, 5]
    tokens, cache_bytes, flops, dec_bytes = bench.step_work(lens)
    assert tokens == 8 and cache_bytes == 8 * 1152
    assert flops == 8 * 2 * 128 * (576 + 512) + 2 * 2 * (2 * 128 * 128 * 512)
    assert dec_bytes == cache_bytes + 2 * 128 * (576 + 512) * 2


def test_balanced_plan_ranges_in_closed_form():
    """The identity the combine relies on: with the balanced plan's bounds (plan_bounds, the
    kernel's rule), tile j of sequence b sits in range ceil((y + 1) P / C) - 1 with y = W_b +
    SEG_COST + j its cost; range p began before b exactly when x_p = floor(p C / P) < W_b; and a
    range holding part of b is empty exactly when x_{p+1} = x_p.  Checked on random length mixes."""
    import random
    import bench
    rnd = random.Random(7)
    for _ in range(1500):
        P = rnd.randint(1, 80)
        tiles = [rnd.choice([0, 1, 2, 3, 5, 8, 13, 30, 64]) for _ in range(rnd.randint(1, 40))]
        if sum(tiles) == 0:
            continue
        C = sum(t + bench.SEG_COST for t in tiles if t > 0)
        bounds = bench.plan_bounds(tiles, P)
        x = [p * C // P for p in range(P + 1)]
        W = off = 0
        for t in tiles:
            if t == 0:
                continue
            for j in range(t):
                assert max(p for p in range(P) if bounds[p] <= off + j) == -(-(W + bench.SEG_COST + j + 1) * P // C) - 1
            for p in range(P):
                assert (bounds[p] < off) == (x[p] < W)
                if bounds[p] <= off + t - 1 and bounds[p + 1] > off:
                    assert (bounds[p] < bounds[p + 1]) == (x[p] < x[p + 1])
            W += bench.SEG_COST + t
            off += t


def test_partial_segments_follow_the_plan():
    """Range partials a decode call writes: per-sequence plan (r_b ranges of sequence b, partials
    only when r_b > 1) and the balanced plan (tiles end to end, a partial for every range that
    meets only part of a sequence), on hand-worked cases."""
    import bench
    assert bench.partial_segments([4096] * 32, 74) == 64             # 32 tiles each: 2 ranges per sequence
    assert bench.partial_segments([131072] * 4, 512) == 512          # 128 ranges of 8 tiles per sequence
    assert bench.partial_segments([1280, 1280], 4) == 4              # tiles 10, 10: 2 ranges each
    # balanced: tiles 2, 1, 3 on a cost line of 12 (2 per sequence start): ranges [0,1) [1,2) [2,3) [3,6)
    assert bench.plan_bounds([2, 1, 3], 4) == [0, 1, 2, 3, 6]
    assert bench.partial_segments([256, 128, 384], 4) == 2
    assert bench.partial_segments([128, 128], 2) == 0                # one range per sequence: no partials
    assert bench.partial_segments([0, 0], 4) == 0


def test_extra_workloads_spec():
    import bench
    assert bench.parse_extras("b32_l4096, b4_l131072@512") == [("b32_l4096", 0), ("b4_l131072", 512)]
    assert bench.parse_extras("") == []
