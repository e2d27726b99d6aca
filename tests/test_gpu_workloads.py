"""Parity at the full workload sizes, in the launch configuration bench.py times (the auto work
plan), or with 512 forced work ranges for the long-context workload (each of its 4 sequences of
131072 tokens is cut into 128 ranges of 8 tiles and merged from 128 partials), checked on sampled
sequences that the fp64 oracle computes one by one."""
import numpy as np
import pytest

import mla_inputs as mi
import oracle
from gpu_common import SCALE, assert_full_path, mean_rel

pytestmark = pytest.mark.gpu
f64 = mi.bf16_to_f64


def _run_workload(name, sample, explicit_first=True):
    import torch
    from mla_latent_kv_20_b200 import get_device_error
    from mla_latent_kv_20_b200 import harness as hz
    w = mi.WORKLOADS[name]
    lens = mi.workload_lengths(name)
    seed = w["seed"]
    batch = mi.decode_batch(seed, lens)
    wts = mi.layer_weights(seed + 1)
    table, nblk = mi.block_permutation(seed + 2, lens) if w["paged"] else (None, 0)
    cache = hz.Cache(lens, w["paged"], table, nblk, fill_value=None)
    cache.fill(batch.c, batch.kr)
    qpos = torch.from_numpy(np.asarray(lens, np.int32) - 1).cuda()
    out, out_lat, lse, _ = hz.decode_step(hz.bf16_tensor(batch.q_nope), hz.bf16_tensor(batch.q_pe),
                                          hz.bf16_tensor(wts.w_uk), hz.bf16_tensor(wts.w_uv), cache,
                                          q_pos=qpos, num_splits=int(w.get("test_ranges", 0)))
    torch.cuda.synchronize()
    assert get_device_error() == 0
    g_out = f64(hz.bf16_bits(out))
    g_lse = lse.cpu().numpy()
    for k, i in enumerate(sample):
        L = int(lens[i])
        form = "explicit" if (explicit_first and k == 0) else "absorbed"
        ref = oracle.decode_step(f64(batch.q_nope[i:i + 1]), f64(batch.q_pe[i:i + 1]), [f64(batch.c[i])],
                                 [f64(batch.kr[i])], f64(wts.w_uk), f64(wts.w_uv), SCALE, q_pos=[L - 1], form=form)
        assert_full_path(g_out[i], ref["out"][0])
        assert np.abs(g_lse[i] - ref["lse"][0]).max() <= 5e-3
        assert mean_rel(g_out[i], ref["out"][0]) <= 5e-3


def test_b1_l256():
    _run_workload("b1_l256", [0])


def test_b32_l4096():
    _run_workload("b32_l4096", [0, 17, 31])


def test_b128_paged_uniform_lengths():
    lens = mi.workload_lengths("b128_u1024_8192_paged")
    _run_workload("b128_u1024_8192_paged", [int(np.argmin(lens)), int(np.argmax(lens)), 64])


def test_b4_l131072_128_ranges_per_sequence():
    """The long-context workload split 128 ways per sequence (512 forced work ranges): the whole
    step against the oracle on two of the four sequences."""
    assert mi.WORKLOADS["b4_l131072"]["test_ranges"] == 512
    _run_workload("b4_l131072", [0, 2], explicit_first=False)


def test_b4_l131072_decode_kernel_128_partials():
    """The decode call alone on the same workload with 512 forced ranges, the query being the bf16
    rounding of the oracle's absorbed query: out_lat and lse of two sequences against the oracle's
    absorbed attention at the decode kernel's bound (each is merged from 128 range partials)."""
    import torch
    from mla_latent_kv_20_b200 import get_device_error
    from mla_latent_kv_20_b200 import harness as hz
    from gpu_common import assert_lse, assert_out_lat
    name = "b4_l131072"
    w = mi.WORKLOADS[name]
    lens = mi.workload_lengths(name)
    batch = mi.decode_batch(w["seed"], lens)
    wts = mi.layer_weights(w["seed"] + 1)
    cache = hz.Cache(lens, False, fill_value=None)
    cache.fill(batch.c, batch.kr)
    qa = oracle.absorb_q(f64(batch.q_nope), f64(wts.w_uk))
    qf_bits = mi.f64_to_bf16(oracle.q_full(qa, f64(batch.q_pe)))
    out_lat, lse = hz.decode(hz.bf16_tensor(qf_bits), cache, num_splits=512)
    torch.cuda.synchronize()
    assert get_device_error() == 0
    g_lat = f64(hz.bf16_bits(out_lat))
    g_lse = lse.cpu().numpy()
    for i in (1, 3):
        L = int(lens[i])
        rows = oracle.cache_rows(f64(batch.c[i]), f64(batch.kr[i]), np.arange(L))
        ref = oracle.attend_rows(f64(qf_bits[i]), rows, SCALE, mi.D_LATENT)
        assert_out_lat(g_lat[i], ref["out_lat"])
        assert_lse(g_lse[i], ref["lse"])


def test_l60_one_layer_full_size():
    """One layer of the 60-layer whole-model workload at its full per-layer size (batch 256,
    log-uniform lengths in [64, 32768], paged), sampled sequences against the oracle."""
    lens = mi.workload_lengths("l60_b256_log64_32768_paged")
    _run_workload("l60_b256_log64_32768_paged", [int(np.argmin(lens)), int(np.argmax(lens)), 100],
                  explicit_first=False)


def test_multi_layer_step_distinct_weights_and_caches():
    """A step over several layers, each with its own weights and paged cache, as the whole-model
    workload runs it: every layer's output matches the oracle for that layer."""
    import torch
    from mla_latent_kv_20_b200 import get_device_error
    from mla_latent_kv_20_b200 import harness as hz
    lens = mi.log_uniform_lengths(77, 8, 64, 3000)
    for layer in range(3):
        seed = 5000 + 7919 * layer
        b = mi.decode_batch(seed, lens)
        w = mi.layer_weights(seed + 1)
        table, nblk = mi.block_permutation(seed + 2, lens)
        cache = hz.Cache(lens, True, table, nblk, fill_value=float("nan"))
        cache.fill(b.c, b.kr)
        qpos = np.asarray(lens, np.int32) - 1
        out, _, lse, _ = hz.decode_step(hz.bf16_tensor(b.q_nope), hz.bf16_tensor(b.q_pe), hz.bf16_tensor(w.w_uk),
                                        hz.bf16_tensor(w.w_uv), cache, q_pos=torch.from_numpy(qpos).cuda())
        torch.cuda.synchronize()
        assert get_device_error() == 0
        ref = oracle.decode_step(f64(b.q_nope), f64(b.q_pe), [f64(x) for x in b.c], [f64(x) for x in b.kr],
                                 f64(w.w_uk), f64(w.w_uv), SCALE, q_pos=qpos, form="absorbed")
        assert_full_path(f64(hz.bf16_bits(out)), ref["out"])
        assert np.abs(lse.cpu().numpy() - ref["lse"]).max() <= 5e-3
