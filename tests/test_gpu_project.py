"""GPU parity of the fused down-projection + cache append (mla_project_append) against the fp64
oracle: rows [W_D^KV h | RoPE(W^KR h)] (《DeepSeek-V2》深度解读报告 §2.2, §2.4, §3.1; model
width 5120 from §3.3)."""
import numpy as np
import pytest

import mla_inputs as mi
import oracle
from gpu_common import assert_projection

pytestmark = pytest.mark.gpu

f64 = mi.bf16_to_f64


@pytest.fixture(scope="module")
def env():
    import torch
    assert torch.cuda.is_available()
    import mla_latent_kv_20_b200 as m
    from mla_latent_kv_20_b200 import harness as hz
    return m, hz, torch


def _run(env, n, seed, paged, lens=None):
    """n new tokens spread over the sequences of a cache; returns (rows written, oracle rows)."""
    m, hz, torch = env
    lens = lens or [300, 64, 129, 7, 1000]
    B = len(lens)
    rng = np.random.default_rng(seed)
    seq = rng.integers(0, B, n).astype(np.int32)
    pos = np.array([rng.integers(0, lens[s]) for s in seq], dtype=np.int32)
    # one token per (seq, pos) slot so every written row is checked
    _, first = np.unique(seq.astype(np.int64) * 100000 + pos, return_index=True)
    keep = np.sort(first)
    seq, pos = seq[keep], pos[keep]
    n = len(seq)
    d = mi.down_projection(seed, n)
    table, nblk = mi.block_permutation(seed + 1, lens) if paged else (None, 0)
    cache = hz.Cache(lens, paged, table, nblk)
    h = hz.bf16_tensor(d.h)
    wd = hz.bf16_tensor(d.w_dkv)
    wk = hz.bf16_tensor(d.w_kr)
    t_seq = torch.from_numpy(seq).cuda()
    t_pos = torch.from_numpy(pos).cuda()
    m.project_append(h, wd, wk, t_pos, cache.data, cache.desc, seq_ids=t_seq, block_table=cache.block_table)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    rows = hz.bf16_bits(cache.data)
    got = f64(rows[[cache.row_index(int(s), int(p)) for s, p in zip(seq, pos)]])
    ref = oracle.project_rows(f64(d.h), f64(d.w_dkv), f64(d.w_kr), pos)
    return got, ref


@pytest.mark.parametrize("n", [1, 31, 32, 33, 100])
@pytest.mark.parametrize("paged", [False, True])
def test_project_append_vs_oracle(env, n, paged):
    got, ref = _run(env, n, 500 + n, paged)
    assert_projection(got[:, :512], ref[:, :512])
    assert_projection(got[:, 512:], ref[:, 512:])


def test_project_append_full_batch(env):
    """256 new tokens (one per sequence of a 256-sequence batch), the largest decode batch of the
    workloads."""
    lens = [4096] * 256
    got, ref = _run(env, 256, 777, False, lens=lens)
    assert got.shape[0] > 200
    assert_projection(got, ref)


def test_project_append_paged_equals_contiguous(env):
    m, hz, torch = env
    got_c, _ = _run(env, 64, 901, False)
    got_p, _ = _run(env, 64, 901, True)
    assert np.array_equal(got_c, got_p)


def test_project_append_leaves_other_rows(env):
    m, hz, torch = env
    lens = [128, 128]
    cache = hz.Cache(lens, False, fill_value=0.0)
    d = mi.down_projection(31, 2)
    pos = torch.tensor([5, 127], dtype=torch.int32, device="cuda")
    m.project_append(hz.bf16_tensor(d.h), hz.bf16_tensor(d.w_dkv), hz.bf16_tensor(d.w_kr), pos, cache.data,
                     cache.desc)
    torch.cuda.synchronize()
    rows = hz.bf16_bits(cache.data)
    written = {cache.row_index(0, 5), cache.row_index(1, 127)}
    others = [r for r in range(rows.shape[0]) if r not in written]
    assert not rows[others].any()
    assert rows[sorted(written)].any(axis=1).all()


def test_project_append_out_of_range_is_reported_not_written(env):
    m, hz, torch = env
    lens = [64, 64]
    cache = hz.Cache(lens, False, max_seq_len=64)
    before = cache.data.clone()
    d = mi.down_projection(32, 2)
    pos = torch.tensor([64, -1], dtype=torch.int32, device="cuda")
    m.project_append(hz.bf16_tensor(d.h), hz.bf16_tensor(d.w_dkv), hz.bf16_tensor(d.w_kr), pos, cache.data,
                     cache.desc)
    torch.cuda.synchronize()
    assert m.get_device_error() & m.DEVERR_POS_RANGE
    assert torch.equal(before, cache.data)
    assert m.get_device_error() == 0
