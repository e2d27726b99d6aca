"""GPU parity of the chunked prefill attention (mla_prefill_attn) against the fp64 oracle:
query row i attends causally to the first q_len[i] cached tokens of sequence q_seq[i]
(《DeepSeek-V2》深度解读报告 §4.2 prompt throughput; attention of §2.3/§2.4)."""
import numpy as np
import pytest

import mla_inputs as mi
import oracle
from gpu_common import SCALE, assert_lse, assert_out_lat_rows

pytestmark = pytest.mark.gpu

f64 = mi.bf16_to_f64


@pytest.fixture(scope="module")
def env():
    import torch
    assert torch.cuda.is_available()
    import mla_latent_kv_20_b200 as m
    from mla_latent_kv_20_b200 import harness as hz
    return m, hz, torch


def _chunks(lens, news, seed):
    """Rows of the new tokens: the last news[s] tokens of sequence s, in a seeded order."""
    q_seq = np.concatenate([np.full(n, s, np.int32) for s, n in enumerate(news)])
    q_len = np.concatenate([np.arange(L - n, L, dtype=np.int32) + 1 for L, n in zip(lens, news)])
    perm = np.random.default_rng(seed).permutation(len(q_seq))
    return q_seq[perm], q_len[perm]


def _prefill(env, cache, qf_bits, q_seq, q_len, splits=0):
    m, hz, torch = env
    n = len(q_seq)
    qf = hz.bf16_tensor(qf_bits)
    out_lat = torch.empty((n, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((n, 128), dtype=torch.float32, device="cuda")
    ws = torch.empty((max(m.decode_workspace_size(n, cache.capacity(), splits), 16),), dtype=torch.uint8, device="cuda")
    m.prefill_attn(qf, cache.data, torch.from_numpy(q_seq).cuda(), torch.from_numpy(q_len).cuda(), cache.desc, ws,
                   out_lat, lse=lse, block_table=cache.block_table, num_splits=splits)
    torch.cuda.synchronize()
    return f64(hz.bf16_bits(out_lat)), lse.cpu().numpy()


def _case(env, lens, news, seed, paged):
    m, hz, torch = env
    b = mi.decode_batch(seed, lens)
    w = mi.layer_weights(seed + 1)
    q_seq, q_len = _chunks(lens, news, seed + 2)
    qb = mi.decode_batch(seed + 3, [1] * len(q_seq))
    qf_bits = mi.f64_to_bf16(oracle.q_full(oracle.absorb_q(f64(qb.q_nope), f64(w.w_uk)), f64(qb.q_pe)))
    table, nblk = mi.block_permutation(seed + 4, lens) if paged else (None, 0)
    cache = hz.Cache(lens, paged, table, nblk, fill_value=float("nan") if paged else 0.0)
    cache.fill(b.c, b.kr)
    rows = [oracle.cache_rows(f64(b.c[s]), f64(b.kr[s]), np.arange(L)) for s, L in enumerate(lens)]
    return cache, qf_bits, q_seq, q_len, rows


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("splits", [0, 5])
def test_prefill_vs_oracle(env, paged, splits):
    m = env[0]
    lens, news = [300, 129, 520], [40, 1, 120]
    cache, qf_bits, q_seq, q_len, rows = _case(env, lens, news, 900, paged)
    g_lat, g_lse = _prefill(env, cache, qf_bits, q_seq, q_len, splits)
    assert m.get_device_error() == 0
    ref = oracle.prefill_rows(f64(qf_bits), rows, q_seq, q_len, SCALE, 512)
    for i in range(len(q_seq)):
        kv = rows[q_seq[i]][:q_len[i]]
        p = oracle.attend_rows(f64(qf_bits[i]), kv, SCALE, 512)["p"]
        assert_out_lat_rows(g_lat[i], ref["out_lat"][i], p @ np.abs(kv[:, :512]))
        assert_lse(g_lse[i], ref["lse"][i])


def test_prefill_many_rows_vs_oracle(env):
    """More than 512 query rows (the combine then gives each warp 8 heads of a row): 600 new tokens of
    two sequences, many rows split between work ranges."""
    m = env[0]
    lens, news = [640, 400], [360, 240]
    cache, qf_bits, q_seq, q_len, rows = _case(env, lens, news, 950, False)
    g_lat, g_lse = _prefill(env, cache, qf_bits, q_seq, q_len)
    assert m.get_device_error() == 0
    ref = oracle.prefill_rows(f64(qf_bits), rows, q_seq, q_len, SCALE, 512)
    for i in range(len(q_seq)):
        kv = rows[q_seq[i]][:q_len[i]]
        p = oracle.attend_rows(f64(qf_bits[i]), kv, SCALE, 512)["p"]
        assert_out_lat_rows(g_lat[i], ref["out_lat"][i], p @ np.abs(kv[:, :512]))
        assert_lse(g_lse[i], ref["lse"][i])


def test_prefill_paged_bit_identical_to_contiguous(env):
    lens, news = [200, 77], [64, 30]
    c1 = _case(env, lens, news, 910, False)
    c2 = _case(env, lens, news, 910, True)
    a = _prefill(env, *c1[:4])
    b = _prefill(env, *c2[:4])
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_prefill_row_equals_decode_of_its_prefix(env):
    """One query row of sequence 1 attending to its first L tokens gives the bits of a decode of a
    cache whose only sequence holds those L tokens (same lengths and ranges, so the same plan)."""
    m, hz, torch = env
    lens = [90, 333]
    b = mi.decode_batch(920, lens)
    cache = hz.Cache(lens, False)
    cache.fill(b.c, b.kr)
    L = 301
    alone = hz.Cache([L], False)
    alone.fill([b.c[1][:L]], [b.kr[1][:L]])
    qf_bits = mi.f64_to_bf16(np.random.default_rng(921).standard_normal((1, 128, 576)) * 0.1)
    g_lat, g_lse = _prefill(env, cache, qf_bits, np.array([1], np.int32), np.array([L], np.int32), splits=3)
    d_lat, d_lse = hz.decode(hz.bf16_tensor(qf_bits), alone, num_splits=3)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    assert np.array_equal(g_lat, f64(hz.bf16_bits(d_lat))) and np.array_equal(g_lse, d_lse.cpu().numpy())


def test_prefill_causal_rows_of_later_tokens_unread(env):
    """Overwriting the rows after a query's position (the rest of its own chunk) leaves its output
    bit-identical."""
    m, hz, torch = env
    lens, news = [260], [60]
    cache, qf_bits, q_seq, q_len, _ = _case(env, lens, news, 930, False)
    first = int(np.argmin(q_len))                        # the chunk's first token: position 200
    a = _prefill(env, cache, qf_bits, q_seq, q_len)
    cache.data.view(torch.int16)[int(q_len[first]):lens[0]].fill_(0x4000)   # bf16 2.0 in every later row
    b = _prefill(env, cache, qf_bits, q_seq, q_len)
    assert np.array_equal(a[0][first], b[0][first]) and np.array_equal(a[1][first], b[1][first])
    last = int(np.argmax(q_len))
    assert not np.array_equal(a[0][last], b[0][last])
    assert m.get_device_error() == 0


def test_prefill_sequence_outside_cache_is_reported(env):
    m, hz, torch = env
    lens = [64, 64]
    cache, qf_bits, _, _, _ = _case(env, lens, [1, 1], 940, False)
    q_seq, q_len = np.array([0, 7], np.int32), np.array([64, 64], np.int32)
    g_lat, g_lse = _prefill(env, cache, qf_bits, q_seq, q_len)
    assert m.get_device_error() & m.DEVERR_BLOCK_RANGE
    assert np.all(g_lat[1] == 0) and np.allclose(g_lse[1], np.log(64), atol=1e-5)   # zero rows: uniform weights
    assert np.all(np.isfinite(g_lat[0]))
