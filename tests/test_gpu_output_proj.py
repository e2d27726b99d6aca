"""GPU parity of the output projection (mla_output_proj) against the fp64 oracle:
y[b] = W_O [concat_h out[b, h]] (《DeepSeek-V2》深度解读报告 §2.3; model width 5120 from §3.3)."""
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
    w_o = mi.output_weight(640)
    return m, hz, torch, w_o, hz.bf16_tensor(w_o)


def _heads_out(seed, batch):
    rng = np.random.Generator(np.random.PCG64(seed))
    return mi.f64_to_bf16(rng.standard_normal((batch, mi.N_HEADS, mi.D_HEAD)))


@pytest.mark.parametrize("batch", [1, 17, 32, 33, 100, 300])
def test_output_proj_vs_oracle(env, batch):
    m, hz, torch, w_o, w_o_dev = env
    out = _heads_out(700 + batch, batch)
    y = torch.empty((batch, mi.D_HIDDEN), dtype=torch.bfloat16, device="cuda")
    m.output_proj(hz.bf16_tensor(out), w_o_dev, y)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    got = f64(hz.bf16_bits(y))
    ref = oracle.output_proj(f64(out), f64(w_o))
    assert_projection(got, ref)


def test_output_proj_after_unabsorb(env):
    """The attention block's tail on the device (un-absorb then output projection) against the
    oracle's two steps on the same out_lat."""
    m, hz, torch, w_o, w_o_dev = env
    batch = 8
    w = mi.layer_weights(711)
    rng = np.random.Generator(np.random.PCG64(712))
    out_lat = mi.f64_to_bf16(rng.standard_normal((batch, mi.N_HEADS, mi.D_LATENT)) * 0.1)
    heads = torch.empty((batch, mi.N_HEADS, mi.D_HEAD), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((batch, mi.D_HIDDEN), dtype=torch.bfloat16, device="cuda")
    m.unabsorb_v(hz.bf16_tensor(out_lat), hz.bf16_tensor(w.w_uv), heads)
    m.output_proj(heads, w_o_dev, y)
    torch.cuda.synchronize()
    # reference from the device's own (bf16) head outputs, so only the projection is compared
    ref = oracle.output_proj(f64(hz.bf16_bits(heads)), f64(w_o))
    assert_projection(f64(hz.bf16_bits(y)), ref)
    # and the heads themselves against the oracle's un-absorb
    assert_projection(f64(hz.bf16_bits(heads)), oracle.unabsorb_v(f64(out_lat), f64(w.w_uv)))


def test_output_proj_deterministic(env):
    m, hz, torch, w_o, w_o_dev = env
    out = hz.bf16_tensor(_heads_out(720, 40))
    y1 = torch.empty((40, mi.D_HIDDEN), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty_like(y1)
    m.output_proj(out, w_o_dev, y1)
    m.output_proj(out, w_o_dev, y2)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
