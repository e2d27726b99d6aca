"""Failure detection without a fault: a pipeline-style bounded wait on a barrier nothing arrives on
must give up within its limit, report MLA_DEVERR_WAIT_TIMEOUT with its site id, and leave the
context usable (the next calls run and match the oracle)."""
import numpy as np
import pytest

import mla_inputs as mi
import oracle
from gpu_common import assert_projection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    assert torch.cuda.is_available()
    import mla_latent_kv_20_b200 as m
    from mla_latent_kv_20_b200 import harness as hz
    return m, hz, torch


@pytest.mark.parametrize("limit_us", [500, 5000])
def test_bounded_wait_gives_up_and_context_survives(env, limit_us):
    m, hz, torch = env
    assert m.get_device_error() == 0
    res = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    m.selftest_wait_timeout(limit_us, res)
    code = m.get_device_error()
    r = res.cpu().numpy()
    assert r[0] == 0, "a wait on a barrier nothing arrives on completed"
    assert limit_us <= r[1] < limit_us + 100000, r[1]
    assert code & m.DEVERR_WAIT_TIMEOUT
    assert (code >> 8) & 0xFF == 0x7F
    # the context still works: an absorption after the timeout matches the oracle
    w = mi.layer_weights(880)
    b = mi.decode_batch(881, [1] * 3)
    q_full = torch.empty((3, 128, 576), dtype=torch.bfloat16, device="cuda")
    m.absorb_q(hz.bf16_tensor(b.q_nope), hz.bf16_tensor(b.q_pe), hz.bf16_tensor(w.w_uk), q_full)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    got = mi.bf16_to_f64(hz.bf16_bits(q_full))[..., :512]
    assert_projection(got, oracle.absorb_q(mi.bf16_to_f64(b.q_nope), mi.bf16_to_f64(w.w_uk)))
