"""The decode entry point that allocates nothing (mla_decode_attn_noalloc).

Some callers cannot obtain device memory while decoding: a plugin running inside a host engine
that owns every device allocation, or a fixed-budget deployment that forbids cudaMalloc after
start-up.  For them the library keeps the range partials in its own static device buffer.  This
test calls that entry point through the C ABI on two calls in a row with different inputs (the
shared buffer keeps the previous call's contents, which must not matter) and checks that each
result equals, bit for bit, the workspace-taking entry point's on the same inputs (both run the
same kernels with the same work plan), and that a call leaves the device's free memory unchanged.

The refusal of problems whose partials do not fit the buffer is host-side validation that
returns before any device call; it is checked without a GPU in test_abi_cpu.py.

The file name sorts last so that a run stopping at the first failure has run every other test.
"""
import ctypes

import numpy as np
import pytest

import mla_inputs as mi
import oracle

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


def _outputs(B):
    import torch
    out_lat = torch.full((B, 128, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, 128), float("nan"), dtype=torch.float32, device="cuda")
    return out_lat, lse


def _call_noalloc(m, qf, cache, splits, out_lat, lse):
    import torch
    rc = m.lib.mla_decode_attn_noalloc(qf.data_ptr(), cache.data.data_ptr(), None, cache.seq_lens.data_ptr(),
                                       cache.desc, qf.shape[0], ctypes.c_float(1.0 / 192 ** 0.5), splits,
                                       out_lat.data_ptr(), lse.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert rc == 0, m.status_string(rc)
    torch.cuda.synchronize()


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import torch
    import mla_latent_kv_20_b200 as m
    from mla_latent_kv_20_b200 import harness as hz
    cases = [(900, [700, 300, 1500, 129], 3), (910, [2000, 64, 1], 5)]
    for seed, lens, splits in cases:
        qf, cache, ref_lat, ref_lse = _case(seed, lens, splits)
        assert m.decode_workspace_size(len(lens), cache.capacity(), splits) <= m.NOALLOC_SCRATCH_BYTES
        out_lat, lse = _outputs(len(lens))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        _call_noalloc(m, qf, cache, splits, out_lat, lse)
        free_after = torch.cuda.mem_get_info()[0]
        assert free_after == free_before, (free_before, free_after)   # nothing allocated on the device
        assert m.get_device_error() == 0
        assert np.array_equal(hz.bf16_bits(out_lat), hz.bf16_bits(ref_lat))
        assert np.array_equal(lse.cpu().numpy().view(np.uint32), ref_lse.cpu().numpy().view(np.uint32))
