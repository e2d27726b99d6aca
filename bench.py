"""Benchmark of one MLA decode step (append -> absorb -> decode attention -> un-absorb).

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--splits P]
                [--extra-workloads A,B,...] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of synthetic input: append the batch's
new token (RoPE on k^R) into the latent cache, absorb W_UK into the queries, split-KV decode
attention over the cache, apply W_UV.  `value` is latent-cache HBM GB/s for the whole job
(bytes of cached rows the step must stream, summed over ranks, divided by the max-over-ranks
device time).  Inputs are resident in HBM before the timed region; the caches are rotated
between steps (several copies, together larger than the 126 MB L2) so no step reads a cache
the previous step left in L2.  N > 1 runs independent replicas (weak scaling): the decode of
disjoint batches needs no data exchange.

The headline workload is batch 128 with lengths uniform in [1024, 8192] over a 64-token paged
cache at permuted physical blocks (the B = 128, ~4K-context decode class).  The timed region is
K steps, bracketed by a barrier and a device synchronisation on both sides; when K steps last
less than MIN_TIMED_S, further K-step brackets follow back to back until the brackets together
last that long, so the clock samples come from timed work, and the reported time per step is
the total device time of all brackets over all their steps.  The other workloads are measured
the same way in the same run and reported under `by_workload`.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mla_inputs as mi  # noqa: E402

METRIC = "MLA decode step: latent-cache HBM GB/s, TFLOP/s, % roofline; tokens/s"
UNIT = "GB/s"
ROW_BYTES = 576 * 2
FLOP_PER_TOKEN = 2 * 128 * 576 + 2 * 128 * 512          # QK^T over [c|k_R] plus P.V over c
GEMM_FLOP_PER_SEQ = 2 * (2 * 128 * 128 * 512)           # absorb + un-absorb
L2_BYTES = 126 * 1024 * 1024
DEFAULT_WORKLOAD = "b128_u1024_8192_paged"
# measured after the headline in the same run (name, forced work ranges or 0 for the auto plan)
DEFAULT_EXTRAS = "b32_l4096,b4_l131072@512,l60_b256_log64_32768_paged"
MIN_TIMED_S = 1.0
NOMINAL_HBM_GBS, NOMINAL_BF16_TFLOPS = 8000.0, 2250.0   # B200 data-sheet figures (context)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def workload_shape(name):
    w = mi.WORKLOADS[name]
    lens = mi.workload_lengths(name)
    return w, lens


def step_work(lens):
    """Algorithmic bytes and flops of one step (per replica)."""
    tokens = int(np.sum(lens))
    B = len(lens)
    cache_bytes = tokens * ROW_BYTES
    flops = tokens * FLOP_PER_TOKEN + B * GEMM_FLOP_PER_SEQ
    # decode kernel's own algorithmic bytes: cache rows + q_full in + out_lat out
    decode_bytes = cache_bytes + B * 128 * 576 * 2 + B * 128 * 512 * 2
    return tokens, cache_bytes, flops, decode_bytes


class ClockSampler:
    """nvidia-smi clock/throttle sampling (every 50 ms) in a background reader that stamps each
    sample with the host's monotonic clock, so samples can be kept for a time window."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.rows = []   # (monotonic time, sm MHz, max MHz, active reasons)
        self.reader = None

    def start(self):
        import threading
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return

        def read():
            for line in self.proc.stdout:
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm, mx = float(f[1]), float(f[2])
                except ValueError:
                    continue
                act = {n for n, v in zip(self.NAMES, f[5:9]) if v.lower().startswith("active")}
                self.rows.append((time.monotonic(), sm, mx, act))

        self.reader = threading.Thread(target=read, daemon=True)
        self.reader.start()

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.reader is not None:
            self.reader.join(timeout=5)

    def summary(self, t0, t1):
        """Median SM clock, max clock and the union of active reasons of the samples in [t0, t1]."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = [r for r in self.rows if t0 <= r[0] <= t1]
        reasons = set()
        for r in rows:
            reasons |= r[3]
        return {"sm_mhz": statistics.median(r[1] for r in rows) if rows else None,
                "sm_max_mhz": max(r[2] for r in rows) if rows else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------------------------- oracle
def time_oracle(lens, budget_tokens=8192, seed=4242, form="explicit", index=0):
    """The fp64 oracle, as it stands, on one sequence of the workload: length lens[index]
    (truncated to `budget_tokens`), `form` = "explicit" (per-head K and V decompressed, textbook
    softmax) or "absorbed" (W_UK folded into the query, W_UV after attention).  Returns
    (tokens, seconds)."""
    import oracle
    L = int(min(int(lens[index % len(lens)]), budget_tokens))
    b = mi.decode_batch(seed, [L])
    w = mi.layer_weights(seed + 1)
    f = mi.bf16_to_f64
    args = (f(b.q_nope), f(b.q_pe), [f(x) for x in b.c], [f(x) for x in b.kr], f(w.w_uk), f(w.w_uv),
            1.0 / math.sqrt(192.0))
    t0 = time.perf_counter()
    oracle.decode_step(*args, q_pos=[L - 1], form=form)
    dt = time.perf_counter() - t0
    return L, dt


def time_oracle_sample(lens, min_seconds=12.0, max_seqs=64, form="explicit"):
    """Bounded CPU baseline: sequences of the workload in its own order (each truncated to 8192
    tokens, distinct seeds) through the oracle until about `min_seconds` of work.  Returns
    (tokens, seconds, sequences)."""
    tok, secs, n = 0, 0.0, 0
    while n < max_seqs and (n == 0 or secs < min_seconds):
        L, dt = time_oracle(lens, seed=4242 + n, form=form, index=n)
        tok, secs, n = tok + L, secs + dt, n + 1
    return tok, secs, n


def time_oracle_layers(lens, n_layers, n_seqs=8, n_sample_layers=2):
    """The whole-model workload's CPU sample: `n_sample_layers` layers x the first `n_seqs`
    sequences (full lengths) through the absorbed fp64 oracle, each layer with its own seeded
    weights and inputs, extrapolated to all layers and sequences of a step by cached tokens.
    Returns (sampled tokens, seconds, extrapolated seconds per step)."""
    tok, secs = 0, 0.0
    for layer in range(n_sample_layers):
        for i in range(n_seqs):
            L, dt = time_oracle(lens, budget_tokens=1 << 30, seed=8000 + 97 * layer + i, form="absorbed", index=i)
            tok, secs = tok + L, secs + dt
    step_tokens = int(np.sum(lens)) * n_layers
    return tok, secs, secs * step_tokens / max(tok, 1)


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        n = 1
    return max(n, 1), len(os.sched_getaffinity(0))


def run_reference(args, rank, world):
    if rank != 0:
        return
    w, lens = workload_shape(args.workload)
    for _ in range(args.warmup):
        time_oracle(lens, budget_tokens=256)
    tok, secs = 0, 0.0
    for i in range(args.steps):
        L, dt = time_oracle(lens, seed=4242 + i, index=i)
        tok += L
        secs += dt
    gbs = tok * ROW_BYTES / secs / 1e9
    threads, cores = cpu_threads()
    sample = (f"{args.steps} steps, each one sequence of the workload in its order ({tok} cached tokens in all, "
              f"each at most 8192; explicit fp64 form), GB/s of cached rows processed")
    line = {"impl": "reference", "metric": METRIC, "value": gbs, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": args.workload, "batch": len(lens),
                                            "seq_len": int(np.max(lens)), "paged": bool(w["paged"])},
            "cpu_baseline": {"value": gbs, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample,
                             "affinity_cores": cores},
            "e2e": {"value": gbs, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------- ours
def _new_token_inputs(batch, lens):
    last = np.asarray(lens, np.int32) - 1
    new_c = np.stack([batch.c[i][last[i]] for i in range(len(lens))])
    new_kr = np.stack([batch.kr[i][last[i]] for i in range(len(lens))])
    return last, new_c, new_kr


def _layer_from_host(name, device):
    """One layer whose inputs come from the seeded host generator (workloads that fit through numpy)."""
    from mla_latent_kv_20_b200 import harness as hz
    w, lens = workload_shape(name)
    seed = w["seed"]
    batch = mi.decode_batch(seed, lens)
    wts = mi.layer_weights(seed + 1)
    table, nblk = mi.block_permutation(seed + 2, lens) if w["paged"] else (None, 0)
    cache = hz.Cache(lens, w["paged"], table, nblk, device=device, fill_value=None)
    cache.fill(batch.c, batch.kr)
    last, new_c, new_kr = _new_token_inputs(batch, lens)
    host = dict(q_nope=batch.q_nope, q_pe=batch.q_pe, c_new=new_c, kr_new=new_kr)
    return dict(caches=[cache], w_uk=hz.bf16_tensor(wts.w_uk, device), w_uv=hz.bf16_tensor(wts.w_uv, device),
                host=host, dev={k: hz.bf16_tensor(v, device) for k, v in host.items()})


def _layer_on_device(name, layer, device, chunk_tokens=1 << 18):
    """One layer of a workload too large for host generation: every value is drawn on the device
    from a seeded torch generator (N(0,1) latents/keys/queries, N(0,1/512) weights), then the cache
    is filled through mla_cache_append."""
    import torch
    import mla_latent_kv_20_b200 as m
    from mla_latent_kv_20_b200 import harness as hz
    w, lens = workload_shape(name)
    seed = w["seed"] + 7919 * layer
    B = len(lens)
    g = torch.Generator(device=device)
    g.manual_seed(seed)

    def normal(shape, std=1.0):
        return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)

    table, nblk = mi.block_permutation(seed + 2, lens) if w["paged"] else (None, 0)
    cache = hz.Cache(lens, w["paged"], table, nblk, device=device, fill_value=None)
    seq_ids = torch.from_numpy(np.concatenate([np.full(L, i, np.int32) for i, L in enumerate(lens)])).to(device)
    pos = torch.from_numpy(np.concatenate([np.arange(L, dtype=np.int32) for L in lens])).to(device)
    for o in range(0, len(pos), chunk_tokens):
        n = min(chunk_tokens, len(pos) - o)
        m.cache_append(normal((n, 512)), normal((n, 64)), pos[o:o + n], cache.data, cache.desc,
                       seq_ids=seq_ids[o:o + n], block_table=cache.block_table)
    dev = dict(q_nope=normal((B, 128, 128)), q_pe=normal((B, 128, 64)), c_new=normal((B, 512)),
               kr_new=normal((B, 64)))
    return dict(caches=[cache], w_uk=normal((128, 128, 512), 1 / math.sqrt(512)),
                w_uv=normal((128, 512, 128), 1 / math.sqrt(512)), host=None, dev=dev)


def setup_replica(name, device, splits=0):
    import torch
    import mla_latent_kv_20_b200 as m
    w, lens = workload_shape(name)
    B = len(lens)
    n_layers = int(w.get("layers", 1))
    if n_layers == 1:
        layers = [_layer_from_host(name, device)]
        _, cache_bytes, _, _ = step_work(lens)
        n_copies = max(2, math.ceil(3 * L2_BYTES / max(cache_bytes, 1)))
        base = layers[0]["caches"][0]
        for _ in range(n_copies - 1):
            c = type(base).__new__(type(base))
            c.__dict__.update(base.__dict__)
            c.data = base.data.clone()
            layers[0]["caches"].append(c)
    else:
        layers = [_layer_on_device(name, l, device) for l in range(n_layers)]
    last = np.asarray(lens, np.int32) - 1
    base = layers[0]["caches"][0]
    # splits = 0: the auto work plan (ranges = resident CTA pairs); else that many forced ranges
    ws_bytes = m.decode_workspace_size(B, base.capacity(), splits)
    st = dict(B=B, lens=lens, w=w, layers=layers, splits=splits,
              n_splits=m.decode_num_splits(B, base.capacity(), splits),
              pos=torch.from_numpy(last).to(device), pos_host=last,
              seq_ids=torch.arange(B, dtype=torch.int32, device=device),
              q_full=torch.empty((B, 128, 576), dtype=torch.bfloat16, device=device),
              out_lat=torch.empty((B, 128, 512), dtype=torch.bfloat16, device=device),
              lse=torch.empty((B, 128), dtype=torch.float32, device=device),
              out=torch.empty((B, 128, 128), dtype=torch.bfloat16, device=device),
              workspace=torch.empty((max(ws_bytes, 16),), dtype=torch.uint8, device=device))
    return st


# DRAM bytes (read + write) of one mla_decode_attn call (decode kernel + combine kernel), from one
# ncu capture per workload, keyed by the SHA-256 of the sources that build those kernels and
# choose their launch shape.  A digest that no longer matches means the kernels changed since the
# counters were taken, and the traffic is reported as null.
TRAFFIC_SOURCES = ("csrc/decode_tc.cuh", "csrc/decode_common.cuh", "csrc/ptx.cuh", "csrc/append.cuh",
                   "csrc/decode_launch.cuh")
MEASURED_TRAFFIC = {   # workload[@ranges] -> {"bytes": int, "sha256": str, "profile": str}
    "b128_u1024_8192_paged": {
        "bytes": 692713728 + 27520512 + 36337664,
        "sha256": "8a3f5dfa12b42f6720b1337f7e46a5337e6e4a9823a12bd11a065ea0c4e23e0d",
        "profile": "profiles/decode_tc_b128_u1024_8192_paged.md (decode + combine, ncu cache flush per kernel)"},
    "b32_l4096": {
        "bytes": 155804416 + 3546368 + 16862976,
        "sha256": "8a3f5dfa12b42f6720b1337f7e46a5337e6e4a9823a12bd11a065ea0c4e23e0d",
        "profile": "profiles/decode_tc_b32_l4096.md (decode + combine, ncu cache flush per kernel)"},
}


def traffic_sources_digest():
    import hashlib
    h = hashlib.sha256()
    for rel in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, "mla_latent_kv_20_b200", rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload, splits=0):
    rec = MEASURED_TRAFFIC.get(workload if not splits else f"{workload}@{splits}")
    if rec is None or rec["sha256"] != traffic_sources_digest():
        return None
    return rec["bytes"]


LAUNCHES_PER_LAYER = 4   # append + absorb GEMM (with the q_pe rotation), decode ranges, combine, un-absorb GEMM


GRAPH_PHASES = ("append_absorb", "decode_attn", "unabsorb_v")


def layer_phase(st, i, li, k):
    """Phase k of GRAPH_PHASES for layer li of step i (cache copy i mod the copies)."""
    import mla_latent_kv_20_b200 as m
    layer = st["layers"][li]
    cache = layer["caches"][i % len(layer["caches"])]
    d = layer["dev"]
    if k == 0:
        # append the new tokens' rows and absorb their queries in one launch
        m.append_absorb(d["c_new"], d["kr_new"], st["pos"], cache.data, cache.desc, d["q_nope"], d["q_pe"],
                        layer["w_uk"], st["q_full"], seq_ids=st["seq_ids"], block_table=cache.block_table,
                        q_pos=st["pos"])
    elif k == 1:
        m.decode_attn(st["q_full"], cache.data, cache.seq_lens, cache.desc, st["workspace"], st["out_lat"],
                      lse=st["lse"], block_table=cache.block_table, num_splits=st["splits"])
    else:
        m.unabsorb_v(st["out_lat"], layer["w_uv"], st["out"])


def capture_step_graphs(st, n_rot, stream):
    """For each cache copy r: one graph of the whole step (every layer, every phase) and, per
    layer, one graph per phase of GRAPH_PHASES.  Kernel arguments (tensor maps included) are
    fixed at capture."""
    import torch
    steps, phases = [], []
    for r in range(n_rot):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for li in range(len(st["layers"])):
                for k in range(len(GRAPH_PHASES)):
                    layer_phase(st, r, li, k)
        steps.append(g)
        per_layer = []
        for li in range(len(st["layers"])):
            gs = []
            for k in range(len(GRAPH_PHASES)):
                gk = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gk, stream=stream):
                    layer_phase(st, r, li, k)
                gs.append(gk)
            per_layer.append(gs)
        phases.append(per_layer)
    return steps, phases


def measure_project_append(st, steps, warmup):
    """The next scope row built beside the step: mla_project_append (down-projection of the new
    tokens' hidden states + cache append) for the step's B new tokens.  Each call reads its 5.9 MB
    of weights from HBM (L2 flushed before every call, the way a multi-layer step meets them);
    timed per call with CUDA events.  Runs after the step's own measurements (it rewrites the new
    tokens' rows of cache copy 0)."""
    import torch
    import mla_latent_kv_20_b200 as m
    from mla_latent_kv_20_b200 import harness as hz
    B = st["B"]
    d = mi.down_projection(9001, B)
    h, wd, wk = hz.bf16_tensor(d.h), hz.bf16_tensor(d.w_dkv), hz.bf16_tensor(d.w_kr)
    cache = st["layers"][0]["caches"][0]
    # evict L2 by reading a buffer twice its size (a read leaves no dirty lines to write back
    # while the timed call runs)
    flush = torch.ones(64 << 20, dtype=torch.int32, device="cuda")

    def call():
        m.project_append(h, wd, wk, st["pos"], cache.data, cache.desc, seq_ids=st["seq_ids"],
                         block_table=cache.block_table)

    for _ in range(max(warmup, 1)):
        call()
    torch.cuda.synchronize()
    n = min(max(steps, 1), 200)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for e0, e1 in ev:
        flush.max()
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    ms = sorted(e0.elapsed_time(e1) for e0, e1 in ev)[n // 2]
    nbytes = 576 * mi.D_HIDDEN * 2 + B * mi.D_HIDDEN * 2 + B * 576 * 2
    hbm = load_peaks()[0]
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": "dp_split_kernel + dp_sum_kernel", "tokens": B, "us_per_call": ms * 1e3, "bound": "hbm",
            "algorithmic_bytes_per_launch": nbytes, "achieved": gbs, "peak": hbm, "unit": "GB/s",
            "frac": gbs / hbm, "l2": "evicted before each call by reading 256 MB (median of %d calls)" % n}


def measure_output_proj(st, steps, warmup):
    """The next scope row built after the step: mla_output_proj (W_O over the step's un-absorbed
    head outputs, y [B, 5120]).  The 168 MB weight (seeded on the device) is larger than L2, so
    every call streams it from HBM; timed per call with CUDA events (median)."""
    import torch
    import mla_latent_kv_20_b200 as m
    B = st["B"]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(9002)
    w_o = (torch.randn((mi.D_HIDDEN, mi.N_HEADS * mi.D_HEAD), device="cuda", generator=gen) *
           mi.DOWN_W_STD).to(torch.bfloat16)
    y = torch.empty((B, mi.D_HIDDEN), dtype=torch.bfloat16, device="cuda")

    def call():
        m.output_proj(st["out"], w_o, y)

    for _ in range(max(warmup, 1)):
        call()
    torch.cuda.synchronize()
    n = min(max(steps, 1), 200)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for e0, e1 in ev:
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    ms = sorted(e0.elapsed_time(e1) for e0, e1 in ev)[n // 2]
    nbytes = mi.D_HIDDEN * mi.N_HEADS * mi.D_HEAD * 2 + B * mi.N_HEADS * mi.D_HEAD * 2 + B * mi.D_HIDDEN * 2
    hbm = load_peaks()[0]
    gbs = nbytes / (ms * 1e-3) / 1e9
    del w_o
    return {"kernel": "out_proj_split_kernel + out_proj_sum_kernel", "sequences": B, "us_per_call": ms * 1e3, "bound": "hbm",
            "algorithmic_bytes_per_launch": nbytes, "achieved": gbs, "peak": hbm, "unit": "GB/s",
            "frac": gbs / hbm, "l2": "weight (168 MB) larger than L2 (median of %d back-to-back calls)" % n}


FP8_ROW_BYTES = 576 + 1   # E4M3 codes + the E8M0 scale byte of a token


def measure_fp8_decode(name, steps, warmup):
    """The FP8-cache row: the same workload's rows (the seeded host generator) appended as E4M3
    codes with power-of-two row scales (mla_cache_append_fp8), then mla_decode_attn_fp8 timed per
    call with CUDA events (median) over two rotated cache copies (larger than L2 together), with
    the workload's bf16 decode call timed the same way beside it.  Algorithmic bytes: 577 per
    cached token plus q_full in and out_lat out."""
    import torch
    import mla_latent_kv_20_b200 as m
    from mla_latent_kv_20_b200 import harness as hz
    w, lens = workload_shape(name)
    batch = mi.decode_batch(w["seed"], lens)
    table, nblk = mi.block_permutation(w["seed"] + 2, lens) if w["paged"] else (None, 0)
    caches = []
    for _ in range(2):
        c = hz.Fp8Cache(lens, w["paged"], table, nblk, fill_byte=None)
        c.fill(batch.c, batch.kr)
        caches.append(c)
    del batch
    B = len(lens)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(9004)
    qf = torch.randn((B, mi.N_HEADS, mi.D_ROW), device="cuda", generator=gen).to(torch.bfloat16)
    out_lat = torch.empty((B, mi.N_HEADS, mi.D_LATENT), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, mi.N_HEADS), dtype=torch.float32, device="cuda")
    ws = torch.empty((m.decode_workspace_size(B, caches[0].capacity(), 0),), dtype=torch.uint8, device="cuda")

    def call(i):
        c = caches[i % 2]
        m.decode_attn_fp8(qf, c.data, c.scales, c.seq_lens, c.desc, ws, out_lat, lse=lse, block_table=c.block_table)

    for i in range(max(warmup, 2)):
        call(i)
    torch.cuda.synchronize()
    n = min(max(steps, 2), 200)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i, (e0, e1) in enumerate(ev):
        e0.record()
        call(i)
        e1.record()
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    ms = sorted(e0.elapsed_time(e1) for e0, e1 in ev)[n // 2]
    tokens = int(np.sum(lens))
    nbytes = tokens * FP8_ROW_BYTES + B * mi.N_HEADS * (mi.D_ROW + mi.D_LATENT) * 2
    hbm, tc = load_peaks()[0], load_peaks()[1]
    gbs = nbytes / (ms * 1e-3) / 1e9
    tf = tokens * FLOP_PER_TOKEN / (ms * 1e-3) / 1e12
    del caches, qf, out_lat, lse, ws
    return {"kernel": "decode_tc_kernel<false, true> (FP8 codes expanded to bf16 in shared memory) + combine_kernel",
            "workload": name, "us_per_call": ms * 1e3, "bound": "hbm", "algorithmic_bytes_per_launch": nbytes,
            "bytes_per_token": FP8_ROW_BYTES, "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
            "tensor": {"achieved_tflops": tf, "peak": tc, "frac": tf / tc},
            "l2": "two cache copies rotated (%.0f MB each), median of %d calls" % (tokens * FP8_ROW_BYTES / 1e6, n)}


PREFILL_SEQS, PREFILL_PREFIX, PREFILL_CHUNK = 4, 3072, 1024


def measure_prefill(steps, warmup):
    """The chunked-prefill row (mla_prefill_attn, absorbed form): 4 sequences each append a chunk of
    1024 new tokens to a 3072-token prefix, and every new token attends causally to the 3073 ..
    4096 cached tokens up to itself (4096 query rows).  Synthetic N(0,1) cache rows and queries
    on the device; the 18.9 MB cache stays in L2 across the rows that share it, so the call is
    bound by the tensor cores: 278,528 flop per (query, cached token) pair.  Timed per call with
    CUDA events (median)."""
    import torch
    import mla_latent_kv_20_b200 as m
    from mla_latent_kv_20_b200 import harness as hz
    L = PREFILL_PREFIX + PREFILL_CHUNK
    gen = torch.Generator(device="cuda")
    gen.manual_seed(9003)
    cache = hz.Cache([L] * PREFILL_SEQS, False, fill_value=None)
    cache.data.copy_(torch.randn(cache.data.shape, device="cuda", generator=gen).to(torch.bfloat16))
    n = PREFILL_SEQS * PREFILL_CHUNK
    q_seq = torch.arange(PREFILL_SEQS, dtype=torch.int32, device="cuda").repeat_interleave(PREFILL_CHUNK)
    q_len = (torch.arange(PREFILL_CHUNK, dtype=torch.int32, device="cuda") + PREFILL_PREFIX + 1).repeat(PREFILL_SEQS)
    qf = torch.randn((n, mi.N_HEADS, mi.D_ROW), device="cuda", generator=gen).to(torch.bfloat16)
    out_lat = torch.empty((n, mi.N_HEADS, mi.D_LATENT), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((n, mi.N_HEADS), dtype=torch.float32, device="cuda")
    ws = torch.empty((m.decode_workspace_size(n, L, 0),), dtype=torch.uint8, device="cuda")

    def call():
        m.prefill_attn(qf, cache.data, q_seq, q_len, cache.desc, ws, out_lat, lse=lse)

    for _ in range(max(warmup, 1)):
        call()
    torch.cuda.synchronize()
    k = min(max(steps, 1), 10)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
    for e0, e1 in ev:
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    ms = sorted(e0.elapsed_time(e1) for e0, e1 in ev)[k // 2]
    pairs = int(q_len.sum().item())
    flops = pairs * 2 * mi.N_HEADS * (mi.D_ROW + mi.D_LATENT)
    _, tc_burst, tc_sustained, _ = load_peaks()
    peak = tc_sustained or tc_burst
    tf = flops / (ms * 1e-3) / 1e12
    del cache, qf, out_lat, lse, ws
    return {"kernel": "decode_tc_kernel<true> + combine_kernel", "sequences": PREFILL_SEQS,
            "new_tokens": n, "prefix": PREFILL_PREFIX, "ms_per_call": ms, "tokens_per_s": n / (ms * 1e-3),
            "bound": "tensor", "algorithmic_flops_per_launch": flops, "achieved": tf, "peak": peak,
            "peak_kind": "sustained bf16 (a call of several ms)", "unit": "TFLOP/s", "frac": tf / peak,
            "l2": "cache (18.9 MB) L2-resident, shared by the rows of a chunk (median of %d calls)" % k}


def run_step(st, i):
    """One decode step over every layer of the workload, through plain API calls."""
    for li in range(len(st["layers"])):
        for k in range(len(GRAPH_PHASES)):
            layer_phase(st, i, li, k)


class CudaRuntime:
    """The few CUDA runtime calls the end-to-end loop issues directly (async copies from and to
    pinned host memory, events without timing): the process's libcudart, loaded by torch."""
    H2D, D2H = 1, 2

    def __init__(self):
        import ctypes
        self.ct = ctypes
        lib = None
        for name in ("libcudart.so.12", "libcudart.so"):
            try:
                lib = ctypes.CDLL(name)
                break
            except OSError:
                continue
        if lib is None:
            import glob
            import torch
            cands = glob.glob(os.path.join(os.path.dirname(torch.__file__), "..", "nvidia", "cuda_runtime", "lib",
                                           "libcudart.so*"))
            lib = ctypes.CDLL(cands[0])
        P, SZ = ctypes.c_void_p, ctypes.c_size_t
        lib.cudaMemcpyAsync.argtypes = [P, P, SZ, ctypes.c_int, P]
        lib.cudaEventCreateWithFlags.argtypes = [ctypes.POINTER(P), ctypes.c_uint]
        lib.cudaEventRecord.argtypes = [P, P]
        lib.cudaStreamWaitEvent.argtypes = [P, P, ctypes.c_uint]
        lib.cudaEventDestroy.argtypes = [P]
        self.lib = lib

    def _ok(self, rc, what):
        if rc != 0:
            raise RuntimeError(f"{what} failed with CUDA error {rc}")

    def memcpy_async(self, dst, src, n, kind, stream):
        self._ok(self.lib.cudaMemcpyAsync(dst, src, n, kind, stream), "cudaMemcpyAsync")

    def events(self, n):
        out = []
        for _ in range(n):
            e = self.ct.c_void_p()
            self._ok(self.lib.cudaEventCreateWithFlags(self.ct.byref(e), 2), "cudaEventCreateWithFlags")  # no timing
            out.append(e)
        return out

    def record(self, ev, stream):
        self._ok(self.lib.cudaEventRecord(ev, stream), "cudaEventRecord")

    def wait(self, stream, ev):
        self._ok(self.lib.cudaStreamWaitEvent(stream, ev, 0), "cudaStreamWaitEvent")

    def destroy(self, evs):
        for e in evs:
            self.lib.cudaEventDestroy(e)


def reduce_max_over_ranks(values, world, device=None):
    """Element-wise max of per-rank timings across the process group (the slowest rank defines
    the job's time).  CPU tensors under gloo, CUDA tensors under nccl."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(bytes_per_rank, world, ms):
    """Whole-job GB/s: the units every rank processed divided by the max-over-ranks time."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


def hz_bits(t):
    from mla_latent_kv_20_b200 import harness as hz
    return hz.bf16_bits(t)


SEG_COST = 2   # tiles' worth of cost a segment start adds in the balanced plan (the decode plan's kSegCost)


def plan_bounds(tiles, P):
    """First global tile of each of the P ranges of the balanced plan, and T: the tiles of the
    batch laid end to end, a non-empty sequence costing SEG_COST + its tiles on a cost line that
    is cut into P pieces of equal cost; a cut inside a sequence's segment charge moves to the
    sequence's first tile."""
    T = sum(tiles)
    C = sum(t + SEG_COST for t in tiles if t > 0)
    bounds = []
    for p in range(P + 1):
        x = p * C // P
        W, off, b = 0, 0, T
        for t in tiles:
            if t == 0:
                continue
            if x < W + SEG_COST + t:
                b = off + max(0, x - W - SEG_COST)
                break
            W += SEG_COST + t
            off += t
        bounds.append(b)
    return bounds


def partial_segments(lens, P):
    """Range partials one decode call writes (and its combine reads back) under the work plan:
    with the per-sequence plan (every non-empty sequence has at least T/P of the T tiles) sequence
    b gets r_b = min(floor(P tiles_b / T), tiles_b) ranges and contributes r_b partials when r_b > 1;
    otherwise the balanced plan (plan_bounds) cuts the tiles laid end to end into P ranges, and
    every range that does not cover the whole of a sequence it meets writes a partial of that
    sequence.  Used only to report the partials' bytes."""
    tiles = [(int(L) + 127) // 128 for L in lens]
    T = sum(tiles)
    if T == 0:
        return 0
    nz = [t for t in tiles if t > 0]
    if min(nz) * P >= T:
        n = 0
        for t in nz:
            r = min(P * t // T, t)
            n += r if r > 1 else 0
        return n
    starts = plan_bounds(tiles, P)
    n, run = 0, 0
    for t in tiles:
        if t == 0:
            continue
        first = max(p for p in range(P) if starts[p] <= run)
        last = max(p for p in range(P) if starts[p] <= run + t - 1)
        if last > first:
            n += sum(1 for p in range(first, last + 1) if starts[p] < starts[p + 1])
        run += t
    return n


PARTIAL_BYTES = 128 * (512 + 2) * 4    # one range partial of one sequence: fp32 O rows, m and l of 128 heads


def measure_workload(name, splits, args, world, dev, barrier):
    """Set up one replica of a workload, time its step, its phases and its end-to-end loop.
    Returns the raw per-rank numbers and the facts of the workload (nothing reduced yet)."""
    import torch
    import mla_latent_kv_20_b200 as m
    st = setup_replica(name, dev, splits)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    for i in range(args.warmup):
        run_step(st, i)
    torch.cuda.synchronize()
    n_layers = len(st["layers"])
    # The timed step replays one CUDA graph of the step's launches (what a serving loop does).
    # A second loop replays one graph per phase, with events between them, to time the decode
    # call (and the other phases) on the device.
    n_rot = len(st["layers"][0]["caches"])
    cap_stream = torch.cuda.Stream()
    step_graphs, phase_graphs = capture_step_graphs(st, n_rot, cap_stream)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0

    def replay_phases(i, ev):
        for li in range(n_layers):
            for k, g in enumerate(phase_graphs[i % n_rot][li]):
                ev[li][k].record()
                g.replay()
            ev[li][len(GRAPH_PHASES)].record()

    for i in range(args.warmup):
        step_graphs[i % n_rot].replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    time.sleep(0.3)
    # K-step brackets, each between a barrier and a synchronisation on both sides, back to back
    # until they add up to MIN_TIMED_S of device time (every rank runs the same number: rank 0's
    # count is broadcast through the max-over-ranks reduction of a flag after each bracket).
    total_ms, brackets, host_ms = 0.0, 0, 0.0
    m0 = time.monotonic()
    while True:
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        t_start.record()
        h0 = time.perf_counter()
        for i in range(args.steps):
            step_graphs[(brackets * args.steps + i) % n_rot].replay()
        host_ms += (time.perf_counter() - h0) * 1e3
        t_end.record()
        torch.cuda.synchronize()
        barrier()
        total_ms += t_start.elapsed_time(t_end)
        brackets += 1
        more = 1.0 if (total_ms < args.min_timed_s * 1e3 and brackets < 100000) else 0.0
        if reduce_max_over_ranks([more], world, device=dev)[0] == 0.0:
            break
    m1 = time.monotonic()
    sampler.stop()
    ms = total_ms / (brackets * args.steps)
    clocks = sampler.summary(m0, m1)
    clocks["window"] = "timed region: %d bracket%s of %d steps (%.2f s)" % (
        brackets, "" if brackets == 1 else "s", args.steps, m1 - m0)
    # per-phase timing loop
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(len(GRAPH_PHASES) + 1)] for _ in range(n_layers)]
           for _ in range(args.steps)]
    for i in range(args.warmup):
        replay_phases(i, evs[i % args.steps])
    torch.cuda.synchronize()
    for i in range(args.steps):
        replay_phases(i, evs[i])
    torch.cuda.synchronize()
    phase_ms = {p: sum(lev[k].elapsed_time(lev[k + 1]) for step in evs for lev in step) / (args.steps * n_layers)
                for k, p in enumerate(GRAPH_PHASES)}
    dec_ms = phase_ms["decode_attn"]
    assert m.get_device_error() == 0
    del step_graphs, phase_graphs

    # End to end through the public API with host buffers, as a serving loop runs it: every step
    # copies its inputs (every layer's new-token rows and queries, and the positions: one packed
    # pinned buffer, one copy) from host memory, runs the step with plain API calls, and reads its
    # result back to pinned host memory.  The copies run on a second stream and overlap the
    # neighbouring steps' kernels: inputs and outputs are double-buffered, step i waits for its own
    # inputs, and its read-back waits for its own kernels.  Copies and the events that order them are
    # issued straight through the CUDA runtime (what a native serving loop calls).  The timed region
    # spans all K steps, from before the first input copy to the end of the last read-back.
    rt = CudaRuntime()
    copy_stream = torch.cuda.Stream()
    compute_stream = torch.cuda.current_stream()
    keys = [list(layer["dev"].keys()) for layer in st["layers"]]
    srcs = []
    for layer, ks in zip(st["layers"], keys):
        for k in ks:
            hsrc = layer["host"][k] if layer["host"] is not None else hz_bits(layer["dev"][k])
            srcs.append(np.ascontiguousarray(hsrc).view(np.uint8).reshape(-1))
    srcs.append(np.ascontiguousarray(st["pos_host"]).view(np.uint8).reshape(-1))
    offs, total = [], 0
    for a in srcs:
        offs.append(total)
        total += (a.size + 255) // 256 * 256          # every input 256-byte aligned in the packed buffer
    host_in = torch.empty(total, dtype=torch.uint8).pin_memory()
    hv = host_in.numpy()
    for a, o in zip(srcs, offs):
        hv[o:o + a.size] = a
    bufs = []   # two sets of (packed inputs, per-layer input views, pos view, out)
    for _ in range(2):
        flat = torch.empty(total, dtype=torch.uint8, device=dev)
        views, j = [], 0
        for layer, ks in zip(st["layers"], keys):
            d = {}
            for k in ks:
                t = layer["dev"][k]
                d[k] = flat[offs[j]:offs[j] + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                j += 1
            views.append(d)
        pos = flat[offs[j]:offs[j] + st["pos"].numel() * 4].view(torch.int32).view(st["pos"].shape)
        bufs.append((flat, views, pos, torch.empty_like(st["out"])))
    out_host = [torch.empty(st["out"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = total   # the packed buffer, padding included: what each step copies
    d2h = out_host[0].numel() * out_host[0].element_size()
    cs, ks_ = copy_stream.cuda_stream, compute_stream.cuda_stream
    in_ready, step_done, out_read = rt.events(2), rt.events(2), rt.events(2)

    def e2e_run(n):
        # copy stream: in(0), in(1), out(0), in(2), out(1), ...: the inputs of step i+1 are copied
        # while step i computes (their buffer's last reader, step i-1, is done: out(i-1) waited for it)
        def h2d_copy(i):
            rt.memcpy_async(bufs[i % 2][0].data_ptr(), host_in.data_ptr(), h2d, rt.H2D, cs)
            rt.record(in_ready[i % 2], cs)

        h2d_copy(0)
        for i in range(n):
            if i + 1 < n:
                h2d_copy(i + 1)
            _, views, pos, out = bufs[i % 2]
            for layer, d in zip(st["layers"], views):
                layer["dev"] = d
            st["pos"], st["out"] = pos, out
            rt.wait(ks_, in_ready[i % 2])
            if i >= 2:
                rt.wait(ks_, out_read[i % 2])      # step i-2's result has been read back
            run_step(st, i)
            rt.record(step_done[i % 2], ks_)
            rt.wait(cs, step_done[i % 2])
            rt.memcpy_async(out_host[i % 2].data_ptr(), out.data_ptr(), d2h, rt.D2H, cs)
            rt.record(out_read[i % 2], cs)

    saved = ([layer["dev"] for layer in st["layers"]], st["pos"], st["out"])
    e2e_run(args.warmup)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(copy_stream)
    e2e_run(args.steps)
    e1.record(copy_stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    for layer, d in zip(st["layers"], saved[0]):
        layer["dev"] = d
    st["pos"], st["out"] = saved[1], saved[2]
    rt.destroy(in_ready + step_done + out_read)
    assert m.get_device_error() == 0
    assert np.array_equal(hz_bits(out_host[(args.steps - 1) % 2]), hz_bits(st["out"]))   # the read-back is the result
    return dict(st=st, n_layers=n_layers, ms=ms, e2e_ms=e2e_ms, dec_ms=dec_ms, phase_ms=phase_ms, clocks=clocks,
                host_ms=host_ms / (brackets * args.steps), brackets=brackets, h2d=h2d, d2h=d2h)


def summarize(name, splits, r, world, peaks):
    """The reported numbers of one measured workload (times already reduced over ranks)."""
    st, n_layers = r["st"], r["n_layers"]
    hbm, tc, tc_sus, peak_kind = peaks
    tokens, cache_bytes, flops, dec_bytes = step_work(st["lens"])
    step_tokens, step_bytes, step_flops = tokens * n_layers, cache_bytes * n_layers, flops * n_layers
    ms, e2e_ms, dec_ms = r["ms"], r["e2e_ms"], r["dec_ms"]
    achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
    dec_flops = tokens * FLOP_PER_TOKEN
    roofline_s = max(step_bytes / (hbm * 1e9), step_flops / (tc * 1e12))
    n_part = partial_segments(st["lens"], st["n_splits"])
    cfg = {"workload": name, "batch": st["B"], "seq_len": int(np.max(st["lens"])), "layers": n_layers,
           "tokens_per_layer": tokens, "paged": bool(st["w"]["paged"]), "work_ranges": st["n_splits"],
           "work_ranges_forced": bool(splits),
           "l2": "inputs larger than L2: %d cache cop%s rotated, %.0f MB each" % (
               len(st["layers"][0]["caches"]) * n_layers,
               "y" if n_layers * len(st["layers"][0]["caches"]) == 1 else "ies", cache_bytes / 1e6),
           "parallelism": f"replicas x{world}"}
    return {
        "value": job_throughput(step_bytes, world, ms), "ms_per_step": ms, "config": cfg,
        "tflops": world * step_flops / (ms * 1e-3) / 1e12,
        "tokens_per_s": world * st["B"] / (ms * 1e-3),
        "decode_layer_ms": dec_ms, "phase_ms_per_layer": r["phase_ms"],
        "host_issue_ms_per_step": r["host_ms"],
        "roofline_step_frac": roofline_s / (ms * 1e-3),
        "roofline": {"kernel": "mla_decode_attn (split-KV decode + combine)", "bound": "hbm",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "peak_kind": peak_kind, "traffic": recorded_traffic(name, splits), "avg_launch_ms": dec_ms,
                     "algorithmic_bytes_per_launch": dec_bytes,
                     "tensor": {"achieved_tflops": dec_flops / (dec_ms * 1e-3) / 1e12, "peak": tc,
                                "frac": dec_flops / (dec_ms * 1e-3) / 1e12 / tc},
                     "nominal": {"hbm_peak": NOMINAL_HBM_GBS, "frac": achieved / NOMINAL_HBM_GBS,
                                 "bf16_peak_tflops": NOMINAL_BF16_TFLOPS},
                     "split_partials": {"segments": n_part, "bytes_written": n_part * PARTIAL_BYTES,
                                        "bytes_read_by_combine": n_part * PARTIAL_BYTES,
                                        "note": "not algorithmic bytes: reported beside them"}},
        "e2e": {"value": job_throughput(step_bytes, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"], "ms_per_step": e2e_ms},
        "clocks": r["clocks"], "timed_brackets": r["brackets"],
        "gpu_launches": LAUNCHES_PER_LAYER * n_layers * r["brackets"],   # per K steps: times K below
    }


def parse_extras(spec):
    out = []
    for item in (spec or "").split(","):
        item = item.strip()
        if not item:
            continue
        name, _, sp = item.partition("@")
        if name not in mi.WORKLOADS:
            raise SystemExit(f"unknown workload {name!r} in --extra-workloads")
        out.append((name, int(sp) if sp else 0))
    return out


def run_ours(args, rank, world, local_rank):
    import gc

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    import mla_latent_kv_20_b200 as m

    def barrier():
        if world > 1:
            dist.barrier()

    peaks = load_peaks()
    r = measure_workload(args.workload, args.splits, args, world, dev, barrier)
    r["ms"], r["e2e_ms"], r["dec_ms"] = reduce_max_over_ranks([r["ms"], r["e2e_ms"], r["dec_ms"]], world, device=dev)
    head = summarize(args.workload, args.splits, r, world, peaks)
    st = r["st"]
    next_rows = None if args.no_next_rows else {
        "project_append": measure_project_append(st, args.steps, args.warmup),
        "output_proj": measure_output_proj(st, args.steps, args.warmup),
        "prefill": measure_prefill(args.steps, args.warmup)}
    del r, st
    gc.collect()
    torch.cuda.empty_cache()
    if next_rows is not None:
        next_rows["fp8_decode"] = measure_fp8_decode(args.workload, args.steps, args.warmup)
        next_rows["fp8_decode"]["bf16_decode_us_same_workload"] = head["decode_layer_ms"] * 1e3
    gc.collect()
    torch.cuda.empty_cache()
    by_workload = {}
    for name, splits in parse_extras(args.extra_workloads):
        if name == args.workload and splits == args.splits:
            continue
        rx = measure_workload(name, splits, args, world, dev, barrier)
        rx["ms"], rx["e2e_ms"], rx["dec_ms"] = reduce_max_over_ranks([rx["ms"], rx["e2e_ms"], rx["dec_ms"]], world,
                                                                     device=dev)
        sx = summarize(name, splits, rx, world, peaks)
        sx["gpu_launches"] *= args.steps
        key = name if not splits else f"{name}@{splits}"
        if rank == 0 and not args.no_cpu_baseline and int(mi.WORKLOADS[name].get("layers", 1)) > 1:
            tok, dt, step_s = time_oracle_layers(rx["st"]["lens"], rx["n_layers"])
            threads, cores = cpu_threads()
            sx["cpu_baseline"] = {"value": tok * ROW_BYTES / dt / 1e9, "unit": UNIT, "cores": threads,
                                  "kind": "oracle", "form": "absorbed", "affinity_cores": cores,
                                  "extrapolated_s_per_step": step_s,
                                  "sample": f"2 layers x the first 8 sequences ({tok} cached tokens, full lengths) "
                                            f"through the absorbed fp64 oracle ({dt:.1f} s); GB/s of cached rows "
                                            f"processed, and the step time extrapolated by cached tokens to "
                                            f"{rx['n_layers']} layers x {len(rx['st']['lens'])} sequences"}
        by_workload[key] = sx
        del rx
        gc.collect()
        torch.cuda.empty_cache()
    assert m.get_device_error() == 0
    if rank != 0:
        return
    head["gpu_launches"] *= args.steps
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) latents/keys/queries, "
                                                     "N(0,1/512) weights)",
        "config": head["config"],
        "timed_step": "one CUDA graph replay per step (all launches of the step), K-step brackets back to back until "
                      "%.1f s; e2e uses plain API calls with one packed input copy and one read-back per step on a "
                      "second stream, double-buffered and overlapping the neighbouring steps' kernels; phase and "
                      "decode times from a second loop of per-phase graph replays with events" % args.min_timed_s,
    }
    for k in ("tflops", "tokens_per_s", "decode_layer_ms", "phase_ms_per_layer", "host_issue_ms_per_step",
              "roofline_step_frac", "roofline", "e2e", "gpu_launches", "clocks", "timed_brackets"):
        line[k] = head[k]
    line["next_rows"] = next_rows
    line["by_workload"] = by_workload
    if not args.no_cpu_baseline:
        lens = mi.workload_lengths(args.workload)
        tok, dt, nseq = time_oracle_sample(lens)
        tok_a, dt_a, nseq_a = time_oracle_sample(lens, min_seconds=4.0, form="absorbed")
        threads, cores = cpu_threads()
        line["cpu_baseline"] = {"value": tok * ROW_BYTES / dt / 1e9, "unit": UNIT, "cores": threads,
                                "kind": "oracle", "form": "explicit", "affinity_cores": cores,
                                "sample": f"the first {nseq} sequences of this workload ({tok} cached tokens, each "
                                          f"at most 8192), explicit fp64 form ({dt:.1f} s of CPU work), GB/s of "
                                          f"cached rows processed",
                                "absorbed": {"value": tok_a * ROW_BYTES / dt_a / 1e9, "unit": UNIT,
                                             "sample": f"the first {nseq_a} sequences ({tok_a} cached tokens), "
                                                       f"absorbed fp64 form ({dt_a:.1f} s)"}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(mi.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--splits", type=int, default=0, help="forced work ranges of the decode (0: the auto plan)")
    ap.add_argument("--extra-workloads", default=DEFAULT_EXTRAS,
                    help="comma-separated NAME or NAME@RANGES measured after the headline (empty: none)")
    ap.add_argument("--min-timed-s", type=float, default=MIN_TIMED_S)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true", help="skip the built next rows (profiling runs)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
