"""The decode entry point that allocates nothing (mla_decode_attn_noalloc).

Some callers cannot obtain device memory while decoding: a plugin running inside a host engine
that owns every device allocation, or a fixed-budget deployment that forbids cudaMalloc after
start-up.  For them the library keeps the range partials in its own static 48 MiB device
buffer.  These tests call that entry point through the C ABI and check it against the
workspace-taking entry point, on two calls in a row with different inputs (the shared buffer
keeps the previous call's contents, which must not matter), and check that a problem whose
partials do not fit is refused before anything is launched.

The file name sorts last so that a run stopping at the first failure has run every other test.
"""
import ctypes

import numpy as np
import pytest

import mla_inputs as mi
import oracle
from gpu_common import assert_lse, assert_out_lat

pytestmark = pytest.mark.gpu

f64 = mi.bf16_to_f64


def _case(seed, lens, splits):
    import torch
    from mla_latent_kv_20_b200 import harness as hz
    b = mi.decode_batch(seed, lens)
    w = mi.layer_weights(seed + 1)
    qa = oracle.absorb_q(f64(b.q_nope), f64(w.w_uk))
    qf = hz.bf16_tensor(mi.f64_to_bf16(oracle.q_full(qa, f64(b.q_pe))))
    cache = hz.Cache(lens, False)
    cache.fill(b.c, b.kr)
    ref_lat, ref_lse = hz.decode(qf, cache, num_splits=splits)       # entry point with a caller workspace
    torch.cuda.synchronize()
    return qf, cache, ref_lat, ref_lse


def _call_noalloc(m, qf, cache, splits):
    import torch
    B = qf.shape[0]
    out_lat = torch.full((B, 128, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, 128), float("nan"), dtype=torch.float32, device="cuda")
    rc = m.lib.mla_decode_attn_noalloc(qf.data_ptr(), cache.data.data_ptr(), None, cache.seq_lens.data_ptr(),
                                       cache.desc, B, ctypes.c_float(1.0 / 192 ** 0.5), splits,
                                       out_lat.data_ptr(), lse.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert rc == 0, m.status_string(rc)
    torch.cuda.synchronize()
    return out_lat, lse


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import mla_latent_kv_20_b200 as m
    from mla_latent_kv_20_b200 import harness as hz
    cases = [(900, [700, 300, 1500, 129], 3), (910, [2000, 64, 1], 5)]
    for seed, lens, splits in cases:
        qf, cache, ref_lat, ref_lse = _case(seed, lens, splits)
        assert m.decode_workspace_size(len(lens), cache.capacity(), splits) <= m.NOALLOC_SCRATCH_BYTES
        got_lat, got_lse = _call_noalloc(m, qf, cache, splits)
        assert m.get_device_error() == 0
        assert_out_lat(f64(hz.bf16_bits(got_lat)), f64(hz.bf16_bits(ref_lat)))
        assert_lse(got_lse.cpu().numpy(), ref_lse.cpu().numpy())


def test_noalloc_refuses_partials_beyond_its_buffer():
    import mla_latent_kv_20_b200 as m
    d = m.contiguous_desc(4, 131072)
    assert m.decode_workspace_size(4, 131072, 1024) > m.NOALLOC_SCRATCH_BYTES
    fake = 0x10000   # never dereferenced: the size check comes first
    rc = m.lib.mla_decode_attn_noalloc(fake, fake, None, fake, d, 4, ctypes.c_float(0.07), 1024, fake, None, None)
    assert rc == 3   # MLA_ERR_WORKSPACE
    assert m.get_device_error() == 0
