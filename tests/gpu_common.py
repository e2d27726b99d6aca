"""Shared helpers of the GPU parity tests: tolerances and error metrics.

Tolerances (each derived from the arithmetic of the kernels it checks):
  * full path out[B,128,128] vs the explicit fp64 oracle: max-abs <= 2e-2 and mean-rel <= 5e-3,
    mean-rel = sum|g - r| / sum|r| over all elements;
  * kernel-level out_lat vs the fp64 oracle on the same bf16 q_full: elementwise
    |g - r| <= 2^-7 |r| + 2e-3 * max|r| (bf16 output rounding 2^-9 relative, bf16-rounded
    cached k^R moving scores by ~1e-3, fp32 accumulation) and mean-rel <= 3e-3;
  * out_lat of many rows at once (prefill): the bound above plus the worst case of P's rounding,
    2^-9 sum_t p_t |c_t| per element (P is rounded to bf16, relative error <= 2^-9 per weight,
    while the row sum uses the unrounded weights), with p from the oracle;
  * lse: |g - r| <= 2e-3 (natural log units);
  * projections (absorb / un-absorb): |g - r| <= 2^-8 |r| + 1e-4 * max|r| (exact bf16 products,
    fp32 accumulation over <= 512 terms, one bf16 rounding of the output).
"""
from __future__ import annotations

import math

import numpy as np

SCALE = 1.0 / math.sqrt(192.0)


def mean_rel(g, r) -> float:
    return float(np.abs(g - r).sum() / max(np.abs(r).sum(), 1e-300))


def assert_full_path(g, r):
    err = np.abs(g - r)
    assert err.max() <= 2e-2, f"max-abs {err.max():.3e}"
    assert mean_rel(g, r) <= 5e-3, f"mean-rel {mean_rel(g, r):.3e}"


def assert_out_lat(g, r):
    bound = 2.0 ** -7 * np.abs(r) + 2e-3 * np.abs(r).max()
    bad = np.abs(g - r) > bound
    assert not bad.any(), f"{bad.sum()} elements out of bound; worst excess {(np.abs(g - r) - bound).max():.3e}"
    assert mean_rel(g, r) <= 3e-3, f"mean-rel {mean_rel(g, r):.3e}"


def assert_out_lat_rows(g, r, pc):
    """g, r: out_lat of one query row [H, d_c]; pc[h, k] = sum_t p_{h,t} |c_{t,k}| from the oracle."""
    bound = 2.0 ** -7 * np.abs(r) + 2.0 ** -9 * pc + 2e-3 * np.abs(r).max()
    bad = np.abs(g - r) > bound
    assert not bad.any(), f"{bad.sum()} elements out of bound; worst excess {(np.abs(g - r) - bound).max():.3e}"
    assert mean_rel(g, r) <= 3e-3, f"mean-rel {mean_rel(g, r):.3e}"


def assert_lse(g, r):
    err = np.abs(g - r)
    assert err.max() <= 2e-3, f"lse max-abs {err.max():.3e}"


def assert_projection(g, r):
    bound = 2.0 ** -8 * np.abs(r) + 1e-4 * np.abs(r).max()
    bad = np.abs(g - r) > bound
    assert not bad.any(), f"{bad.sum()} elements out of bound; worst {np.abs(g - r)[bad].max():.3e}"


def f64_to_bf16_direct(x: np.ndarray) -> np.ndarray:
    """Round fp64 directly to the nearest bf16 (ties to even), returning uint16 bits.

    Used for the RoPE'd key: the kernel rounds its fp64 rotation once to bf16."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    flat, o = x.ravel(), out.ravel()
    f32 = flat.astype(np.float32)
    u = f32.view(np.uint32)
    for i in range(flat.size):
        # candidates: truncation of the fp32 neighbour and the next bf16 up/down
        hi = (int(u[i]) >> 16) & 0xFFFF
        cands = [(hi - 1) & 0xFFFF, hi, (hi + 1) & 0xFFFF]
        vals = [np.array([c << 16], dtype=np.uint32).view(np.float32)[0].astype(np.float64) for c in cands]
        d = [abs(v - flat[i]) for v in vals]
        best = min(d)
        ties = [c for c, dd in zip(cands, d) if dd == best]
        o[i] = ties[0] if len(ties) == 1 else [c for c in ties if c % 2 == 0][0]
    return out
