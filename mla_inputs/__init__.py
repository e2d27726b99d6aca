"""Seeded synthetic inputs for MLA latent-KV decode, shared by the oracle and the CUDA path.

This module holds no attention arithmetic: it only draws numbers and rounds them to bf16.
Both sides (the fp64 oracle under ``oracle/`` and the CUDA library) consume the exact
same bf16 bit patterns produced here.

Value distributions follow the workload description of the decode step: latent rows c^KV,
raw decoupled-RoPE keys k^R, q_nope and q_pe ~ N(0, 1); W_UK and W_UV ~ N(0, 1/512)
(std 1/sqrt(512)).  Values are drawn in fp64 (numpy PCG64), rounded to fp32 and then to
bf16 with round-to-nearest-even.

bf16 tensors are carried as ``numpy.uint16`` bit patterns; ``bf16_to_f64`` widens them
exactly.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

N_HEADS = 128
D_HEAD = 128      # d_h: per-head width of q_nope and of the output
D_LATENT = 512    # d_c: width of the cached latent c^KV
D_ROPE = 64       # d_R: width of the shared decoupled-RoPE key k^R
D_ROW = D_LATENT + D_ROPE
D_HIDDEN = 5120   # d: model width ([DR] §3.3), input of the down-projections
DOWN_W_STD = 0.006   # initialisation std of the weights ([DR] §3.3)
PAGE = 64
W_STD = 1.0 / math.sqrt(512.0)


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (via fp32, both steps round-to-nearest-even); returns uint16 bits."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    nan = np.isnan(f)
    out = r.astype(np.uint16)
    if nan.any():
        out = np.where(nan, np.uint16(0x7FC0), out)
    return out


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_to_f32(b).astype(np.float64)


def _normal_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    return f64_to_bf16(rng.standard_normal(size=shape) * std)


@dataclasses.dataclass
class LayerWeights:
    w_uk: np.ndarray  # [H, d_h, d_c] bf16 bits: k^C_j = sum_k W_UK[h, j, k] c_k
    w_uv: np.ndarray  # [H, d_c, d_h] bf16 bits: v^C_j = sum_k W_UV[h, k, j] c_k


@dataclasses.dataclass
class DecodeBatch:
    """One decode step's inputs for a batch of sequences (one new query token per sequence)."""
    seq_lens: np.ndarray   # [B] int32, tokens attended (already including the new token)
    c: list                # per sequence: [L_b, d_c] bf16 bits (latent rows, positions 0..L_b-1)
    kr: list               # per sequence: [L_b, d_R] bf16 bits (k^R BEFORE RoPE)
    q_nope: np.ndarray     # [B, H, d_h] bf16 bits
    q_pe: np.ndarray       # [B, H, d_R] bf16 bits (taken as already rotated unless q_pos is used)


def layer_weights(seed: int, n_heads: int = N_HEADS, d_head: int = D_HEAD,
                  d_latent: int = D_LATENT) -> LayerWeights:
    rng = np.random.Generator(np.random.PCG64(seed))
    w_uk = _normal_bf16(rng, (n_heads, d_head, d_latent), W_STD)
    w_uv = _normal_bf16(rng, (n_heads, d_latent, d_head), W_STD)
    return LayerWeights(w_uk, w_uv)


@dataclasses.dataclass
class DownProjection:
    """Inputs of the fused down-projection + append: new tokens' hidden states and the weights
    that map them to the cached latent and RoPE key (recipe: hidden 5120 and the initialisation
    std 0.006 of [DR] §3.3; hidden states N(0, 1))."""
    h: np.ndarray        # [n, d] bf16 bits
    w_dkv: np.ndarray    # [d_c, d] bf16 bits: c^KV = W_D^KV h
    w_kr: np.ndarray     # [d_R, d] bf16 bits: k^R (before RoPE) = W^KR h


def down_projection(seed: int, n_tokens: int, d_hidden: int = D_HIDDEN, d_latent: int = D_LATENT,
                    d_rope: int = D_ROPE) -> DownProjection:
    rng = np.random.Generator(np.random.PCG64(seed))
    w_dkv = _normal_bf16(rng, (d_latent, d_hidden), DOWN_W_STD)
    w_kr = _normal_bf16(rng, (d_rope, d_hidden), DOWN_W_STD)
    h = _normal_bf16(rng, (n_tokens, d_hidden), 1.0)
    return DownProjection(h, w_dkv, w_kr)


def output_weight(seed: int, d_hidden: int = D_HIDDEN, n_heads: int = N_HEADS, d_head: int = D_HEAD) -> np.ndarray:
    """W_O [d, H * d_h] bf16 bits ~ N(0, 0.006^2) ([DR] §3.3 initialisation std)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return _normal_bf16(rng, (d_hidden, n_heads * d_head), DOWN_W_STD)


def decode_batch(seed: int, seq_lens, n_heads: int = N_HEADS, d_head: int = D_HEAD,
                 d_latent: int = D_LATENT, d_rope: int = D_ROPE) -> DecodeBatch:
    rng = np.random.Generator(np.random.PCG64(seed))
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    b = len(seq_lens)
    q_nope = _normal_bf16(rng, (b, n_heads, d_head))
    q_pe = _normal_bf16(rng, (b, n_heads, d_rope))
    c, kr = [], []
    for L in seq_lens:
        c.append(_normal_bf16(rng, (int(L), d_latent)))
        kr.append(_normal_bf16(rng, (int(L), d_rope)))
    return DecodeBatch(seq_lens, c, kr, q_nope, q_pe)


def uniform_lengths(seed: int, batch: int, lo: int, hi: int) -> np.ndarray:
    """Lengths drawn uniformly from the integers lo..hi inclusive."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(lo, hi + 1, size=batch).astype(np.int32)


def log_uniform_lengths(seed: int, batch: int, lo: int, hi: int) -> np.ndarray:
    """floor(exp(U[ln lo, ln hi])), clipped to [lo, hi]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    u = rng.uniform(math.log(lo), math.log(hi), size=batch)
    return np.clip(np.floor(np.exp(u)), lo, hi).astype(np.int32)


def block_permutation(seed: int, seq_lens, page: int = PAGE, max_blocks: int | None = None):
    """Paged layout: physical block ids are a seeded permutation of 0..sum(ceil(L_b/page))-1.

    Returns (block_table [B, max_blocks] int32 padded with -1, num_blocks).
    """
    seq_lens = np.asarray(seq_lens, dtype=np.int64)
    nblk = (seq_lens + page - 1) // page
    total = int(nblk.sum())
    if max_blocks is None:
        max_blocks = int(nblk.max()) if len(nblk) else 0
    rng = np.random.Generator(np.random.PCG64(seed))
    perm = rng.permutation(total).astype(np.int32)
    table = np.full((len(seq_lens), max(max_blocks, 1)), -1, dtype=np.int32)
    o = 0
    for i, n in enumerate(nblk):
        table[i, :n] = perm[o:o + n]
        o += n
    return table, total


# Workload presets: the five decode workloads (batch, length distribution, cache layout, seed).
WORKLOADS = {
    "b1_l256": dict(batch=1, lens="fixed", L=256, paged=False, seed=1001),
    "b32_l4096": dict(batch=32, lens="fixed", L=4096, paged=False, seed=1002),
    "b128_u1024_8192_paged": dict(batch=128, lens="uniform", lo=1024, hi=8192, paged=True, seed=1003),
    "b4_l131072": dict(batch=4, lens="fixed", L=131072, paged=False, seed=1004, test_ranges=512),
    "l60_b256_log64_32768_paged": dict(batch=256, lens="loguniform", lo=64, hi=32768, paged=True,
                                       seed=1005, layers=60),
}


def workload_lengths(name: str) -> np.ndarray:
    w = WORKLOADS[name]
    if w["lens"] == "fixed":
        return np.full(w["batch"], w["L"], dtype=np.int32)
    if w["lens"] == "uniform":
        return uniform_lengths(w["seed"] + 100, w["batch"], w["lo"], w["hi"])
    return log_uniform_lengths(w["seed"] + 100, w["batch"], w["lo"], w["hi"])
