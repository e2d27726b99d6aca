"""FP8 (E4M3) latent cache on the GPU (《DeepSeek-V2》深度解读报告 §4.2 效率证据: FP8 serving with the
KV cache at about 6 bits per element; the format is this library's reading: 576 E4M3 codes per
token plus a power-of-two row scale kept as an E8M0 byte).

* mla_cache_append_fp8 writes, bit for bit, the codes and scales of the oracle's quantizer
  (oracle.fp8_cache_rows), contiguous and paged, and touches no other row.
* mla_decode_attn_fp8 matches the oracle's absorbed attention over the dequantized rows at the
  decode kernel's bound, for ragged tails, empty sequences and forced work ranges.
* Its result equals, bit for bit, mla_decode_attn over a bf16 cache holding the same dequantized
  values (exact in bf16), and paged equals contiguous.
"""
import numpy as np
import pytest

import mla_inputs as mi
import oracle
from gpu_common import SCALE, assert_lse, assert_out_lat

pytestmark = pytest.mark.gpu
f64 = mi.bf16_to_f64


def _e8m0(scales):
    """Scale values (powers of two) as E8M0 bytes 127 + log2(s)."""
    e = np.log2(np.asarray(scales, np.float64))
    assert np.array_equal(e, np.round(e))
    return (np.round(e) + 127).astype(np.uint8)


def _oracle_rows(batch, lens):
    """Per sequence: (codes, scale bytes, dequantized rows) from the oracle alone."""
    out = []
    for i, L in enumerate(lens):
        codes, s = oracle.fp8_cache_rows(f64(batch.c[i]), f64(batch.kr[i]), np.arange(L))
        out.append((codes, _e8m0(s), oracle.dequantize_rows(codes, s)))
    return out


def _fp8_cache(lens, paged, seed, batch):
    from mla_latent_kv_20_b200 import harness as hz
    table, nblk = mi.block_permutation(seed, lens) if paged else (None, 0)
    cache = hz.Fp8Cache(lens, paged, table, nblk, fill_byte=0x55)
    cache.fill(batch.c, batch.kr)
    return cache


def _rows_of(cache, i, L):
    return [cache.row_index(i, t) for t in range(L)]


@pytest.mark.parametrize("paged", [False, True])
def test_fp8_append_matches_oracle_quantizer(paged):
    import torch
    from mla_latent_kv_20_b200 import get_device_error
    lens = [1, 63, 64, 130, 300, 0, 77]
    b = mi.decode_batch(1201, lens)
    # crafted rows: a huge value among tiny ones (subnormal codes), exact E4M3 midpoints, a zero row
    b.c[4][5] = mi.f64_to_bf16(np.r_[3000.0, np.full(511, 0.01)])
    b.c[4][6] = mi.f64_to_bf16(np.r_[448.0, np.tile([1.0625, -1.1875, 3.25, 0.0078125], 127), [0.0] * 3])
    b.kr[4][6] = mi.f64_to_bf16(np.zeros(64))
    b.c[4][7] = mi.f64_to_bf16(np.zeros(512))
    b.kr[4][7] = mi.f64_to_bf16(np.zeros(64))
    cache = _fp8_cache(lens, paged, 1202, b)
    torch.cuda.synchronize()
    assert get_device_error() == 0
    codes = cache.data.cpu().numpy()
    scales = cache.scales.cpu().numpy()
    written = np.zeros(codes.shape[0], bool)
    for i, (c_ref, e_ref, _) in enumerate(_oracle_rows(b, lens)):
        rows = _rows_of(cache, i, lens[i])
        written[rows] = True
        assert np.array_equal(codes[rows], c_ref), (i, np.argwhere(codes[rows] != c_ref)[:4])
        assert np.array_equal(scales[rows], e_ref), i
    assert (codes[~written] == 0x55).all() and (scales[~written] == 0x55).all()   # no other row touched


def test_fp8_paged_rows_equal_contiguous_rows():
    import torch
    lens = [200, 64, 1, 129]
    b = mi.decode_batch(1211, lens)
    cc = _fp8_cache(lens, False, 0, b)
    cp = _fp8_cache(lens, True, 1212, b)
    torch.cuda.synchronize()
    for i, L in enumerate(lens):
        rc, rp = _rows_of(cc, i, L), _rows_of(cp, i, L)
        assert np.array_equal(cc.data[rc].cpu().numpy(), cp.data[rp].cpu().numpy())
        assert np.array_equal(cc.scales[rc].cpu().numpy(), cp.scales[rp].cpu().numpy())


def _query(seed, B):
    b = mi.decode_batch(seed, [0] * B)
    w = mi.layer_weights(seed + 1)
    qa = oracle.absorb_q(f64(b.q_nope), f64(w.w_uk))
    return mi.f64_to_bf16(oracle.q_full(qa, f64(b.q_pe)))


@pytest.mark.parametrize("paged,splits", [(False, 0), (True, 0), (False, 3), (True, 1)])
def test_fp8_decode_vs_oracle(paged, splits):
    import torch
    from mla_latent_kv_20_b200 import get_device_error
    from mla_latent_kv_20_b200 import harness as hz
    lens = [1, 63, 64, 65, 127, 128, 129, 0, 700]
    b = mi.decode_batch(1221, lens)
    cache = _fp8_cache(lens, paged, 1222, b)
    qf = _query(1223, len(lens))
    out_lat, lse = hz.decode_fp8(hz.bf16_tensor(qf), cache, num_splits=splits)
    torch.cuda.synchronize()
    assert get_device_error() == 0
    g_lat = f64(hz.bf16_bits(out_lat))
    g_lse = lse.cpu().numpy()
    for i, (_, _, rows) in enumerate(_oracle_rows(b, lens)):
        if lens[i] == 0:
            assert not g_lat[i].any() and np.isneginf(g_lse[i]).all()
            continue
        ref = oracle.attend_rows(f64(qf[i]), rows, SCALE, mi.D_LATENT)
        assert_out_lat(g_lat[i], ref["out_lat"])
        assert_lse(g_lse[i], ref["lse"])


def test_fp8_decode_equals_bf16_decode_of_the_decoded_rows():
    """The decoded values are exact in bf16, so the FP8 decode must give the bits of the bf16 decode
    over a cache holding them (same kernels, same plan); paged gives the bits of contiguous."""
    import torch
    from mla_latent_kv_20_b200 import harness as hz
    lens = [300, 1, 129, 64, 1000, 513]
    b = mi.decode_batch(1231, lens)
    qf = hz.bf16_tensor(_query(1232, len(lens)))
    fc = _fp8_cache(lens, False, 0, b)
    fp = _fp8_cache(lens, True, 1233, b)
    bc = hz.Cache(lens, False, max_seq_len=fc.desc.max_seq_len, fill_value=0.0)
    data = np.zeros((bc.data.shape[0], mi.D_ROW), np.uint16)
    for i, (_, _, rows) in enumerate(_oracle_rows(b, lens)):
        data[_rows_of(bc, i, lens[i])] = mi.f64_to_bf16(rows)
    bc.data.copy_(hz.bf16_tensor(data))
    for splits in (0, 4):
        ref_lat, ref_lse = hz.decode(qf, bc, num_splits=splits)
        for cache in (fc, fp):
            got_lat, got_lse = hz.decode_fp8(qf, cache, num_splits=splits)
            torch.cuda.synchronize()
            assert np.array_equal(hz.bf16_bits(got_lat), hz.bf16_bits(ref_lat)), (splits, cache.paged)
            assert np.array_equal(got_lse.cpu().numpy().view(np.uint32), ref_lse.cpu().numpy().view(np.uint32))


def test_fp8_decode_full_size_paged_workload():
    """The batch-128 paged workload (lengths uniform in [1024, 8192], 64-token pages at permuted
    blocks) as an FP8 cache, the launch the bench times (auto plan): sampled sequences against the
    oracle over their dequantized rows."""
    import torch
    from mla_latent_kv_20_b200 import get_device_error
    from mla_latent_kv_20_b200 import harness as hz
    name = "b128_u1024_8192_paged"
    w = mi.WORKLOADS[name]
    lens = mi.workload_lengths(name)
    b = mi.decode_batch(w["seed"], lens)
    cache = _fp8_cache(lens, True, w["seed"] + 2, b)
    qf = _query(w["seed"] + 3, len(lens))
    out_lat, lse = hz.decode_fp8(hz.bf16_tensor(qf), cache)
    torch.cuda.synchronize()
    assert get_device_error() == 0
    g_lat = f64(hz.bf16_bits(out_lat))
    g_lse = lse.cpu().numpy()
    for i in (int(np.argmin(lens)), int(np.argmax(lens)), 64):
        codes, s = oracle.fp8_cache_rows(f64(b.c[i]), f64(b.kr[i]), np.arange(lens[i]))
        ref = oracle.attend_rows(f64(qf[i]), oracle.dequantize_rows(codes, s), SCALE, mi.D_LATENT)
        assert_out_lat(g_lat[i], ref["out_lat"])
        assert_lse(g_lse[i], ref["lse"])
