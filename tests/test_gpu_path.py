"""GPU parity of every step of the decode path against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest

import mla_inputs as mi
import oracle
from gpu_common import (SCALE, assert_full_path, assert_lse, assert_out_lat, assert_projection,
                        f64_to_bf16_direct)

pytestmark = pytest.mark.gpu

f64 = mi.bf16_to_f64


@pytest.fixture(scope="module")
def env():
    import torch
    assert torch.cuda.is_available()
    import mla_latent_kv_20_b200 as m
    from mla_latent_kv_20_b200 import harness as hz
    return m, hz, torch


def _clear(m):
    assert m.get_device_error() == 0


# ----------------------------------------------------------------------------- append
@pytest.mark.parametrize("paged", [False, True])
def test_append_rows(env, paged):
    m, hz, torch = env
    lens = [1, 63, 64, 65, 200]
    b = mi.decode_batch(100, lens)
    table, nblk = mi.block_permutation(101, lens) if paged else (None, 0)
    cache = hz.Cache(lens, paged, table, nblk)
    cache.fill(b.c, b.kr)
    torch.cuda.synchronize()
    _clear(m)
    rows = hz.bf16_bits(cache.data)
    for i, L in enumerate(lens):
        idx = [cache.row_index(i, t) for t in range(L)]
        got = rows[idx]
        assert np.array_equal(got[:, :512], b.c[i])                       # latent copied bit-exactly
        ref = oracle.apply_rope(f64(b.kr[i]), np.arange(L))
        exp = f64_to_bf16_direct(ref)
        same = (got[:, 512:] == exp).mean()
        assert same >= 0.999, same                                       # one rounding of the fp64 rotation
        ulp = np.abs(got[:, 512:].astype(np.int32) - exp.astype(np.int32))
        assert ulp.max() <= 1


def test_append_paged_gather_matches_contiguous(env):
    m, hz, torch = env
    lens = [130, 64, 7]
    b = mi.decode_batch(110, lens)
    table, nblk = mi.block_permutation(111, lens)
    cp = hz.Cache(lens, True, table, nblk)
    cc = hz.Cache(lens, False)
    cp.fill(b.c, b.kr)
    cc.fill(b.c, b.kr)
    torch.cuda.synchronize()
    rp, rc = hz.bf16_bits(cp.data), hz.bf16_bits(cc.data)
    for i, L in enumerate(lens):
        a = rp[[cp.row_index(i, t) for t in range(L)]]
        c = rc[[cc.row_index(i, t) for t in range(L)]]
        assert np.array_equal(a, c)


def test_append_out_of_range_is_reported_not_written(env):
    m, hz, torch = env
    lens = [64, 64]
    cache = hz.Cache(lens, False, max_seq_len=64)
    before = cache.data.clone()
    c = hz.bf16_tensor(mi.f64_to_bf16(np.ones((2, 512))))
    kr = hz.bf16_tensor(mi.f64_to_bf16(np.ones((2, 64))))
    pos = torch.tensor([64, -1], dtype=torch.int32, device="cuda")
    m.cache_append(c, kr, pos, cache.data, cache.desc)
    torch.cuda.synchronize()
    assert m.get_device_error() & m.DEVERR_POS_RANGE
    assert torch.equal(before, cache.data)
    # paged: a block id outside the pool
    table = np.array([[0], [5]], dtype=np.int32)
    cp = hz.Cache(lens, True, table, 2)
    pos = torch.tensor([3, 3], dtype=torch.int32, device="cuda")
    m.cache_append(c, kr, pos, cp.data, cp.desc, block_table=cp.block_table)
    torch.cuda.synchronize()
    assert m.get_device_error() & m.DEVERR_BLOCK_RANGE
    _clear(m)


# ----------------------------------------------------------------------------- projections
@pytest.mark.parametrize("batch", [1, 5, 32, 100, 128, 300])   # 65..128 rows take two M tiles per CTA
def test_absorb_q(env, batch):
    m, hz, torch = env
    w = mi.layer_weights(200)
    b = mi.decode_batch(201, [1] * batch)
    q_full = torch.full((batch, 128, 576), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.absorb_q(hz.bf16_tensor(b.q_nope), hz.bf16_tensor(b.q_pe), hz.bf16_tensor(w.w_uk), q_full)
    torch.cuda.synchronize()
    _clear(m)
    g = hz.bf16_bits(q_full)
    ref = oracle.absorb_q(f64(b.q_nope), f64(w.w_uk))
    assert_projection(f64(g[..., :512]), ref)
    assert np.array_equal(g[..., 512:], b.q_pe)                           # copied when q_pos is NULL


def test_absorb_q_rotates_q_pe(env):
    m, hz, torch = env
    w = mi.layer_weights(210)
    b = mi.decode_batch(211, [1] * 6)
    qpos = np.array([0, 1, 63, 4095, 100000, 131071], dtype=np.int32)
    q_full = torch.empty((6, 128, 576), dtype=torch.bfloat16, device="cuda")
    m.absorb_q(hz.bf16_tensor(b.q_nope), hz.bf16_tensor(b.q_pe), hz.bf16_tensor(w.w_uk), q_full,
               q_pos=torch.from_numpy(qpos).cuda())
    torch.cuda.synchronize()
    g = hz.bf16_bits(q_full)[..., 512:]
    ref = f64_to_bf16_direct(oracle.apply_rope(f64(b.q_pe), qpos[:, None]))
    assert (g == ref).mean() >= 0.999
    assert np.abs(g.astype(np.int32) - ref.astype(np.int32)).max() <= 1


@pytest.mark.parametrize("batch", [1, 17, 256, 260])
def test_unabsorb_v(env, batch):
    m, hz, torch = env
    w = mi.layer_weights(300)
    rng = np.random.default_rng(301)
    lat = mi.f64_to_bf16(rng.standard_normal((batch, 128, 512)) * 0.05)
    out = torch.full((batch, 128, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.unabsorb_v(hz.bf16_tensor(lat), hz.bf16_tensor(w.w_uv), out)
    torch.cuda.synchronize()
    _clear(m)
    assert_projection(f64(hz.bf16_bits(out)), oracle.unabsorb_v(f64(lat), f64(w.w_uv)))


# ----------------------------------------------------------------------------- decode attention
def _decode_case(env, lens, seed, paged=False, splits=0):
    m, hz, torch = env
    b = mi.decode_batch(seed, lens)
    w = mi.layer_weights(seed + 1)
    qa = oracle.absorb_q(f64(b.q_nope), f64(w.w_uk))
    qf_bits = mi.f64_to_bf16(oracle.q_full(qa, f64(b.q_pe)))               # decode input from the oracle
    table, nblk = mi.block_permutation(seed + 2, lens) if paged else (None, 0)
    cache = hz.Cache(lens, paged, table, nblk, fill_value=float("nan") if paged else 0.0)
    cache.fill(b.c, b.kr)
    out_lat, lse = hz.decode(hz.bf16_tensor(qf_bits), cache, num_splits=splits)
    torch.cuda.synchronize()
    _clear(m)
    return b, qf_bits, f64(hz.bf16_bits(out_lat)), lse.cpu().numpy()


def _ref_rows(b, qf_bits, i):
    L = int(b.seq_lens[i])
    rows = oracle.cache_rows(f64(b.c[i]), f64(b.kr[i]), np.arange(L))
    return oracle.attend_rows(f64(qf_bits[i]), rows, SCALE, 512)


@pytest.mark.parametrize("lens", [[256], [1, 63, 64, 65, 127, 128, 129, 300]])
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_decode_vs_oracle(env, lens, splits):
    b, qf, g_lat, g_lse = _decode_case(env, lens, 400 + len(lens), splits=splits)
    for i in range(len(lens)):
        r = _ref_rows(b, qf, i)
        assert_out_lat(g_lat[i], r["out_lat"])
        assert_lse(g_lse[i], r["lse"])


def test_decode_rescales_on_growing_scores(env):
    """Scores that grow along the sequence: latent dim 0 of token t is 0.05 t and q_full's dim 0 runs
    from -40 to 40 over the heads, so the running maximum of the steepest heads rises by far more
    than the lazy-rescale threshold (2^8) on every tile and O is corrected on almost every tile,
    gentler heads are corrected every few tiles and falling heads never.  Partner warps of the
    softmax (the two token halves of a head) must take the same decision; checked contiguous with
    the automatic plan and paged with forced work ranges, against the oracle."""
    m, hz, torch = env
    lens = [1000, 700, 130, 64]
    b = mi.decode_batch(530, lens)
    for i, L in enumerate(lens):
        c = f64(b.c[i])
        c[:L, 0] = 0.05 * np.arange(L)
        b.c[i] = mi.f64_to_bf16(c)
    q = 0.5 * np.random.default_rng(531).standard_normal((len(lens), 128, 576))
    q[:, :, 0] = np.linspace(-40.0, 40.0, 128)
    qf_bits = mi.f64_to_bf16(q)
    for paged, splits in ((False, 0), (True, 3)):
        table, nblk = mi.block_permutation(532, lens) if paged else (None, 0)
        cache = hz.Cache(lens, paged, table, nblk, fill_value=float("nan") if paged else 0.0)
        cache.fill(b.c, b.kr)
        out_lat, lse = hz.decode(hz.bf16_tensor(qf_bits), cache, num_splits=splits)
        torch.cuda.synchronize()
        _clear(m)
        g_lat, g_lse = f64(hz.bf16_bits(out_lat)), lse.cpu().numpy()
        for i in range(len(lens)):
            r = _ref_rows(b, qf_bits, i)
            assert_out_lat(g_lat[i], r["out_lat"])
            assert_lse(g_lse[i], r["lse"])


def test_decode_paged_bit_identical_to_contiguous(env):
    lens = [1, 64, 65, 333, 1000]
    _, _, lat_c, lse_c = _decode_case(env, lens, 500, paged=False)
    _, _, lat_p, lse_p = _decode_case(env, lens, 500, paged=True)
    assert np.array_equal(lat_c, lat_p) and np.array_equal(lse_c, lse_p)


def test_decode_deterministic(env):
    lens = [700, 50]
    r1 = _decode_case(env, lens, 510, splits=4)
    r2 = _decode_case(env, lens, 510, splits=4)
    assert np.array_equal(r1[2], r2[2]) and np.array_equal(r1[3], r2[3])


def test_decode_empty_sequence(env):
    m, hz, torch = env
    lens = [0, 5]
    b = mi.decode_batch(520, lens)
    cache = hz.Cache(lens, False, max_seq_len=8)
    cache.fill(b.c, b.kr)
    qf = torch.randn((2, 128, 576), device="cuda").to(torch.bfloat16)
    out_lat, lse = hz.decode(qf, cache)
    torch.cuda.synchronize()
    _clear(m)
    assert torch.all(out_lat[0] == 0) and torch.all(torch.isneginf(lse[0]))
    assert torch.all(torch.isfinite(lse[1]))


def test_decode_seq_len_beyond_capacity_is_reported(env):
    m, hz, torch = env
    cache = hz.Cache([8, 8], False, max_seq_len=8)
    cache.seq_lens = torch.tensor([9, 8], dtype=torch.int32, device="cuda")
    qf = torch.zeros((2, 128, 576), dtype=torch.bfloat16, device="cuda")
    hz.decode(qf, cache)
    torch.cuda.synchronize()
    assert m.get_device_error() & m.DEVERR_SEQLEN_RANGE


# ----------------------------------------------------------------------------- whole step
@pytest.mark.parametrize("lens,paged", [([256], False), ([5, 64, 129, 1000], True)])
def test_full_step_vs_explicit_oracle(env, lens, paged):
    m, hz, torch = env
    seed = 600 + len(lens)
    b = mi.decode_batch(seed, lens)
    w = mi.layer_weights(seed + 1)
    table, nblk = mi.block_permutation(seed + 2, lens) if paged else (None, 0)
    cache = hz.Cache(lens, paged, table, nblk)
    cache.fill(b.c, b.kr)
    qpos = np.asarray(lens, np.int32) - 1
    out, out_lat, lse, _ = hz.decode_step(hz.bf16_tensor(b.q_nope), hz.bf16_tensor(b.q_pe), hz.bf16_tensor(w.w_uk),
                                          hz.bf16_tensor(w.w_uv), cache, q_pos=torch.from_numpy(qpos).cuda())
    torch.cuda.synchronize()
    _clear(m)
    ref = oracle.decode_step(f64(b.q_nope), f64(b.q_pe), [f64(x) for x in b.c], [f64(x) for x in b.kr],
                             f64(w.w_uk), f64(w.w_uv), SCALE, q_pos=qpos, form="explicit")
    assert_full_path(f64(hz.bf16_bits(out)), ref["out"])
    assert np.abs(lse.cpu().numpy() - ref["lse"]).max() <= 5e-3


# ----------------------------------------------------------------------------- fused append + absorb
@pytest.mark.parametrize("paged,n_tokens,batch", [(False, 4, 4), (True, 4, 4), (False, 7, 3), (True, 2, 33),
                                                   (True, 40, 128)])
def test_append_absorb_equals_separate_calls(env, paged, n_tokens, batch):
    """mla_append_absorb writes exactly the rows of mla_cache_append and the q_full of mla_absorb_q."""
    m, hz, torch = env
    lens = [5, 64, 65, 300]
    table, nblk = mi.block_permutation(301, lens) if paged else (None, 0)
    c1 = hz.Cache(lens, paged, table, nblk)
    c2 = hz.Cache(lens, paged, table, nblk)
    rng = np.random.default_rng(302 + n_tokens)
    seq = rng.integers(0, len(lens), n_tokens).astype(np.int32)
    pos = np.array([rng.integers(0, lens[s]) for s in seq], dtype=np.int32)
    _, keep = np.unique(seq.astype(np.int64) * 100000 + pos, return_index=True)
    seq, pos = seq[np.sort(keep)], pos[np.sort(keep)]
    b = mi.decode_batch(303, [1] * batch)
    w = mi.layer_weights(304)
    c_new = hz.bf16_tensor(mi.f64_to_bf16(rng.standard_normal((len(seq), 512))))
    kr_new = hz.bf16_tensor(mi.f64_to_bf16(rng.standard_normal((len(seq), 64))))
    t_seq, t_pos = torch.from_numpy(seq).cuda(), torch.from_numpy(pos).cuda()
    q_pos = torch.from_numpy(rng.integers(0, 131072, batch).astype(np.int32)).cuda()
    qn, qp, wuk = hz.bf16_tensor(b.q_nope), hz.bf16_tensor(b.q_pe), hz.bf16_tensor(w.w_uk)
    qf1 = torch.empty((batch, 128, 576), dtype=torch.bfloat16, device="cuda")
    qf2 = torch.empty_like(qf1)
    m.cache_append(c_new, kr_new, t_pos, c1.data, c1.desc, seq_ids=t_seq, block_table=c1.block_table)
    m.absorb_q(qn, qp, wuk, qf1, q_pos=q_pos)
    m.append_absorb(c_new, kr_new, t_pos, c2.data, c2.desc, qn, qp, wuk, qf2, seq_ids=t_seq,
                    block_table=c2.block_table, q_pos=q_pos)
    torch.cuda.synchronize()
    _clear(m)
    assert torch.equal(c1.data, c2.data)
    assert torch.equal(qf1, qf2)
