"""fp64 CPU oracle for DeepSeek-V2 Multi-head Latent Attention (MLA) decode.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module.  It shares no code with the CUDA library and
imports nothing from it.  Every function is plain numpy in float64, dimension-generic
(all sizes come from the argument shapes), with no blocking, fusion or reordering beyond
the definition it states.

Sources (page title, section):
  [DR] 《DeepSeek-V2》深度解读报告 (zako-mio.github.io llm-papers-knowledge-base)
       §2.1 KV Cache, §2.2 Low-Rank Key-Value Joint Compression, §2.3 Absorption,
       §2.4 Decoupled Rotary Position Embedding, §3.1 MLA 完整计算链路与参数核算.
  [XD] DeepSeek-V2论文解读：MoE架构如何实现训练成本降42.5%与KV缓存压93.3% (xdnf.cn),
       §2.1 MLA把KV缓存从瓶颈变成可压缩项.
  [DP] DeepSeek V2技术解析：MLA架构如何重塑大模型推理效率 (devpress.csdn.net), §1.

Readings where the pages are silent:
  * softmax scale 1/sqrt(d_h + d_R) = 1/sqrt(192) (the pages never state it);
  * RoPE on the decoupled branch uses the interleaved pairing (x[2i], x[2i+1]) rotated by
    pos * theta_i, theta_i = base^(-2i/d_R), base 10000 (the pages name RoPE but print no
    formula; this is the original RoPE definition);
  * W_UK is laid out [head, d_h, d_c] (k^C_j = sum_k W_UK[h,j,k] c_k) and W_UV is laid out
    [head, d_c, d_h] (v^C_j = sum_k W_UV[h,k,j] c_k);
  * the new token is appended before attention, so the query attends to itself;
  * W_O is laid out [d, H d_h] and applied after the un-absorb to the head-major concatenation of
    the heads' outputs (folding W_U^V into W_O ahead of time would need H x d_c x d weights, four
    times the bytes of the two-step form, so the two projections stay separate);
  * the down-projections are laid out [out, in] (W_D^KV [d_c, d], W^KR [d_R, d]) and k^R is the
    plain linear projection W^KR h_t (the pages draw the branch h_t -> k^R without naming its
    matrix), rotated by RoPE before it is cached.

  * FP8 latent cache ([DR] §4.2 效率证据 reports FP8 serving with the KV cache at about 6 bits per
    element, without a format): each cached row (the 576 values [c | RoPE(k^R)], taken before any
    bf16 rounding) is stored as 576 OCP E4M3 codes plus one scale per token, the power of two
    s = 2^k with k the smallest integer for which amax <= 448 * 2^k (amax the row's largest
    magnitude; s = 1 for an all-zero row); a value x is coded as the E4M3 value nearest (ties to
    even, saturating at +-448) to the fp32 rounding of x / s, and decodes to code_value * s, which
    a power-of-two scale keeps exact in bf16 and fp32.

Pins: every function here is checked by ``tests/test_oracle_pins.py`` against values that
do not come from this file (closed forms, library routines, brute-force scalar loops,
invariants).  No function is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

ROPE_BASE = 10000.0


# ----------------------------------------------------------------------------------------
# Cache-size arithmetic ([DR] §2.1 and §3.1; [XD] §2.1; [DP] §1)
# ----------------------------------------------------------------------------------------
def mha_cache_elems_per_token(n_heads: int, d_head: int, n_layers: int = 1) -> int:
    """Standard MHA caches one key and one value per head: 2 * n_h * d_h * l elements."""
    return 2 * n_heads * d_head * n_layers


def mla_cache_elems_per_token(d_latent: int, d_rope: int, n_layers: int = 1) -> int:
    """MLA caches the latent c^KV plus the shared decoupled key k^R: (d_c + d_R) * l."""
    return (d_latent + d_rope) * n_layers


# ----------------------------------------------------------------------------------------
# Decoupled RoPE ([DR] §2.4; position branch of the flow in §3.1)
# ----------------------------------------------------------------------------------------
def rope_inv_freq(d_rope: int, base: float = ROPE_BASE) -> np.ndarray:
    """theta_i = base^(-2i/d_R) for i = 0 .. d_R/2 - 1."""
    i = np.arange(d_rope // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d_rope)


def apply_rope(x: np.ndarray, pos, base: float = ROPE_BASE) -> np.ndarray:
    """Rotate each interleaved pair (x[2i], x[2i+1]) by the angle pos * theta_i.

    x: [..., d_R]; pos: scalar or array broadcastable to x.shape[:-1].
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    theta = rope_inv_freq(d, base)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta          # [..., d/2]
    cos, sin = np.cos(ang), np.sin(ang)
    xe, xo = x[..., 0::2], x[..., 1::2]
    y = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d,)), dtype=np.float64)
    y[..., 0::2] = xe * cos - xo * sin
    y[..., 1::2] = xe * sin + xo * cos
    return y


def cache_rows(c: np.ndarray, kr_raw: np.ndarray, pos, base: float = ROPE_BASE) -> np.ndarray:
    """The cached row of a token: [c^KV | RoPE(k^R, pos)], width d_c + d_R ([DR] §2.4)."""
    return np.concatenate([np.asarray(c, dtype=np.float64), apply_rope(kr_raw, pos, base)], axis=-1)


def project_rows(h: np.ndarray, w_dkv: np.ndarray, w_kr: np.ndarray, pos, base: float = ROPE_BASE) -> np.ndarray:
    """Cached rows straight from the hidden states ([DR] §2.2: c^KV = W_D^KV h; §3.1: k^R is the
    shared 64-wide projection of h on the RoPE branch; §2.4: RoPE applies to that branch only).

    h: [n, d]; w_dkv: [d_c, d] and w_kr: [d_R, d] (output index first, as a linear layer maps
    d inputs to d_c or d_R outputs); pos: [n].  Returns [n, d_c + d_R]: [W_D^KV h | RoPE(W^KR h)].
    """
    h = np.asarray(h, dtype=np.float64)
    c = h @ np.asarray(w_dkv, dtype=np.float64).T       # [n, d_c]
    kr_raw = h @ np.asarray(w_kr, dtype=np.float64).T   # [n, d_R]
    return cache_rows(c, kr_raw, pos, base)


# ----------------------------------------------------------------------------------------
# Explicit (non-absorbed) MLA: decompress per-head K and V ([DR] §2.2)
# ----------------------------------------------------------------------------------------
def decompress(c: np.ndarray, w_uk: np.ndarray, w_uv: np.ndarray):
    """k^C_t = W_UK c_t and v^C_t = W_UV c_t for every head.

    c: [L, d_c]; w_uk: [H, d_h, d_c]; w_uv: [H, d_c, d_h].  Returns kC, vC of shape [L, H, d_h].
    """
    c = np.asarray(c, dtype=np.float64)
    kC = np.einsum("hjk,lk->lhj", np.asarray(w_uk, np.float64), c, optimize=True)
    vC = np.einsum("hkj,lk->lhj", np.asarray(w_uv, np.float64), c, optimize=True)
    return kC, vC


def softmax_stats(s: np.ndarray):
    """Row-wise max-subtracted softmax along the last axis; returns (p, lse)."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    z = np.sum(e, axis=-1, keepdims=True)
    return e / z, (m + np.log(z))[..., 0]


def attend_explicit(q_nope, q_pe, c, kr_rot, w_uk, w_uv, scale):
    """Textbook MLA attention of one query token over L cached tokens, all heads.

    Per head h ([DR] §2.2 and §2.4: the score is the sum of the content and position channels):
      q_h = [q_nope_h ; q_pe_h] (d_h + d_R),  k_{t,h} = [k^C_{t,h} ; k^R_t],
      s_{h,t} = scale * q_h . k_{t,h},  p = softmax_t(s),  out_h = sum_t p_{h,t} v^C_{t,h}.
    Also returns out_lat_h = sum_t p_{h,t} c_t (the latent context the absorbed path produces)
    and lse_h = log sum_t exp(s_{h,t}).

    q_nope: [H, d_h]; q_pe: [H, d_R] (already rotated); c: [L, d_c]; kr_rot: [L, d_R].
    """
    q_nope = np.asarray(q_nope, np.float64)
    q_pe = np.asarray(q_pe, np.float64)
    c = np.asarray(c, np.float64)
    kr_rot = np.asarray(kr_rot, np.float64)
    kC, vC = decompress(c, w_uk, w_uv)                      # [L, H, d_h]
    H = q_nope.shape[0]
    L = c.shape[0]
    s = np.empty((H, L), dtype=np.float64)
    for h in range(H):
        q = np.concatenate([q_nope[h], q_pe[h]])            # [d_h + d_R]
        k = np.concatenate([kC[:, h, :], kr_rot], axis=1)   # [L, d_h + d_R]
        s[h] = scale * (k @ q)
    p, lse = softmax_stats(s)
    out = np.einsum("ht,thj->hj", p, vC, optimize=True)
    out_lat = p @ c
    return dict(out=out, out_lat=out_lat, lse=lse, p=p, s=s)


# ----------------------------------------------------------------------------------------
# Absorbed MLA ([DR] §2.3: q.(W_UK c) = (q W_UK).c; W_UV applied after attention)
# ----------------------------------------------------------------------------------------
def absorb_q(q_nope: np.ndarray, w_uk: np.ndarray) -> np.ndarray:
    """q_abs[..., h, k] = sum_j q_nope[..., h, j] W_UK[h, j, k]   ([..., H, d_h] -> [..., H, d_c])."""
    return np.einsum("...hj,hjk->...hk", np.asarray(q_nope, np.float64), np.asarray(w_uk, np.float64), optimize=True)


def unabsorb_v(out_lat: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """out[..., h, j] = sum_k out_lat[..., h, k] W_UV[h, k, j]   ([..., H, d_c] -> [..., H, d_h])."""
    return np.einsum("...hk,hkj->...hj", np.asarray(out_lat, np.float64), np.asarray(w_uv, np.float64), optimize=True)


def output_proj(out: np.ndarray, w_o: np.ndarray) -> np.ndarray:
    """The attention block's output projection after the un-absorb ([DR] §2.3: W_U^V belongs with
    the output projection W_O): y[b] = W_O [concat_h out[b, h]], heads concatenated head-major.

    out: [B, H, d_h]; w_o: [d, H * d_h] (output index first).  Returns [B, d].
    """
    out = np.asarray(out, dtype=np.float64)
    B = out.shape[0]
    return out.reshape(B, -1) @ np.asarray(w_o, dtype=np.float64).T


def q_full(q_abs: np.ndarray, q_pe: np.ndarray) -> np.ndarray:
    """The absorbed query row of a head: [q_abs (d_c) | q_pe (d_R)], matching the cached row layout."""
    return np.concatenate([np.asarray(q_abs, np.float64), np.asarray(q_pe, np.float64)], axis=-1)


def attend_rows(qf: np.ndarray, rows: np.ndarray, scale: float, d_latent: int):
    """Absorbed attention of one query over cached rows [c | k^R_rot].

    qf: [H, d_c + d_R] (absorbed query); rows: [L, d_c + d_R].
    s_{h,t} = scale * qf_h . row_t;  out_lat_h = sum_t softmax(s)_{h,t} row_t[:d_c].
    """
    qf = np.asarray(qf, np.float64)
    rows = np.asarray(rows, np.float64)
    s = scale * (qf @ rows.T)                               # [H, L]
    p, lse = softmax_stats(s)
    return dict(out_lat=p @ rows[:, :d_latent], lse=lse, p=p, s=s)


def attend_absorbed(q_nope, q_pe, c, kr_rot, w_uk, w_uv, scale):
    """Same result as ``attend_explicit`` through the absorbed form (separate code path)."""
    qa = absorb_q(q_nope, w_uk)
    rows = np.concatenate([np.asarray(c, np.float64), np.asarray(kr_rot, np.float64)], axis=1)
    r = attend_rows(q_full(qa, q_pe), rows, scale, c.shape[1])
    r["out"] = unabsorb_v(r["out_lat"], w_uv)
    r["q_abs"] = qa
    return r


# ----------------------------------------------------------------------------------------
# Split-KV partials and their merge (flash-decoding; not on the pages, a plain identity of
# the softmax: exp-weighted partial sums over disjoint token ranges merge exactly).
# ----------------------------------------------------------------------------------------
def partial_rows(qf, rows, scale, d_latent):
    """Unnormalised partial over a token range: (O = sum_t e^{s_t - m} c_t, m = max s, l = sum e^{s_t-m})."""
    s = scale * (np.asarray(qf, np.float64) @ np.asarray(rows, np.float64).T)
    m = np.max(s, axis=-1)
    e = np.exp(s - m[:, None])
    return e @ np.asarray(rows, np.float64)[:, :d_latent], m, e.sum(axis=-1)


def merge_partials(parts):
    """Merge [(O_s, m_s, l_s)] over disjoint ranges: out = sum w_s O_s / sum w_s l_s, w_s = e^{m_s - M}."""
    M = np.max(np.stack([p[1] for p in parts]), axis=0)
    num = sum(np.exp(p[1] - M)[:, None] * p[0] for p in parts)
    den = sum(np.exp(p[1] - M) * p[2] for p in parts)
    return num / den[:, None], M + np.log(den)


# ----------------------------------------------------------------------------------------
# Chunked prefill ([DR] §4.2 measures prompt throughput beside generation; the attention is
# that of §2.3/§2.4).  A chunk of new tokens is appended first; each new token then attends
# causally: to the tokens before it and to itself.
# ----------------------------------------------------------------------------------------
def prefill_rows(qf, seq_rows, q_seq, q_len, scale, d_latent):
    """Absorbed form, one query row at a time: row i attends to the first q_len[i] cached rows of
    sequence q_seq[i] (q_len = position + 1 is the causal mask).

    qf: [n, H, d_c + d_R]; seq_rows: list of [L_s, d_c + d_R], one per cache sequence.
    Returns out_lat [n, H, d_c] and lse [n, H]; a row with q_len 0 gives zeros and -inf.
    """
    qf = np.asarray(qf, np.float64)
    n, H = qf.shape[0], qf.shape[1]
    out_lat = np.zeros((n, H, d_latent))
    lse = np.full((n, H), -np.inf)
    for i in range(n):
        L = int(q_len[i])
        if L == 0:
            continue
        r = attend_rows(qf[i], np.asarray(seq_rows[int(q_seq[i])], np.float64)[:L], scale, d_latent)
        out_lat[i], lse[i] = r["out_lat"], r["lse"]
    return dict(out_lat=out_lat, lse=lse)


def prefill_explicit_masked(q_nope, q_pe, c, kr_rot, w_uk, w_uv, scale, q_pos):
    """Textbook causal attention of a chunk of queries of one sequence in the explicit form:
    per-head keys and values decompressed from the latents ([DR] §2.2), one score tensor
    s[h, i, t] = scale * [q_nope_ih ; q_pe_ih] . [k^C_th ; k^R_t] over all L cached tokens, the
    entries of tokens after the query's position (t > q_pos[i]) set to -inf, a softmax along t,
    then out = P v^C and out_lat = P c.

    q_nope: [n, H, d_h]; q_pe: [n, H, d_R] (rotated); c: [L, d_c]; kr_rot: [L, d_R]; q_pos: [n].
    """
    q_nope = np.asarray(q_nope, np.float64)
    q_pe = np.asarray(q_pe, np.float64)
    c = np.asarray(c, np.float64)
    kC, vC = decompress(c, w_uk, w_uv)                                   # [L, H, d_h]
    s = np.einsum("ihj,thj->hit", q_nope, kC, optimize=True)            # content channel
    s = s + np.einsum("ihr,tr->hit", q_pe, np.asarray(kr_rot, np.float64), optimize=True)
    s = scale * s
    L = c.shape[0]
    future = np.arange(L)[None, :] > np.asarray(q_pos)[:, None]          # [n, L]
    s = np.where(future[None, :, :], -np.inf, s)
    p, lse = softmax_stats(s)                                            # along t
    out = np.einsum("hit,thj->ihj", p, vC, optimize=True)
    out_lat = np.einsum("hit,tk->ihk", p, c, optimize=True)
    return dict(out=out, out_lat=out_lat, lse=lse.T)


# ----------------------------------------------------------------------------------------
# One whole decode step for a batch ([DR] §3.1 flow: append, absorb, attend, un-absorb)
# ----------------------------------------------------------------------------------------
def decode_step(q_nope, q_pe, cs, krs_raw, w_uk, w_uv, scale, base=ROPE_BASE,
                q_pos=None, form="explicit"):
    """Reference outputs for a batch.

    q_nope: [B, H, d_h]; q_pe: [B, H, d_R]; cs / krs_raw: per-sequence [L_b, d_c] / [L_b, d_R]
    (k^R before RoPE; token t sits at position t).  If q_pos is given, q_pe is rotated at
    q_pos[b]; otherwise q_pe is taken as already rotated.
    Returns dict of arrays out [B, H, d_h], out_lat [B, H, d_c], lse [B, H], q_abs [B, H, d_c].
    """
    B = len(cs)
    outs, lats, lses, qas = [], [], [], []
    for b in range(B):
        L = cs[b].shape[0]
        kr_rot = apply_rope(krs_raw[b], np.arange(L), base)
        qpe = q_pe[b] if q_pos is None else apply_rope(q_pe[b], q_pos[b], base)
        if form == "explicit":
            r = attend_explicit(q_nope[b], qpe, cs[b], kr_rot, w_uk, w_uv, scale)
            qa = absorb_q(q_nope[b], w_uk)
        else:
            r = attend_absorbed(q_nope[b], qpe, cs[b], kr_rot, w_uk, w_uv, scale)
            qa = r["q_abs"]
        outs.append(r["out"]); lats.append(r["out_lat"]); lses.append(r["lse"]); qas.append(qa)
    return dict(out=np.stack(outs), out_lat=np.stack(lats), lse=np.stack(lses), q_abs=np.stack(qas))


# ----------------------------------------------------------------------------------------
# FP8 (E4M3) latent cache ([DR] §4.2: FP8 serving, KV cache at about 6 bits per element).
# E4M3 (OCP 8-bit floating point, E4M3 variant): 1 sign bit, 4 exponent bits with bias 7,
# 3 mantissa bits; exponent field 0 holds the subnormals m * 2^-9; no infinities; the largest
# finite magnitude is 1.75 * 2^8 = 448 (exponent field 15, mantissa 6); field 15 with mantissa 7
# is NaN.
# ----------------------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 code (uint8) in float64, from the bit fields."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode_rne(v) -> np.ndarray:
    """The E4M3 code of each float32 value: round to the nearest representable magnitude, ties to
    the even mantissa, magnitudes at or beyond 448 saturate to 448; the sign is kept (also for
    zero).  NaN inputs are not handled."""
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    a = np.abs(v)
    sat = a >= E4M3_MAX
    # quantum of the binade: 2^(E - 3) for a in [2^E, 2^(E+1)), E >= -6; 2^-9 below 2^-6
    _, ex = np.frexp(np.where(a > 0, a, 1.0))          # a = f * 2^ex, f in [0.5, 1)
    E = np.maximum(ex - 1, -6)
    q = np.exp2(E - 3.0)
    n = np.rint(a / q)                                 # a / q is exact (q a power of two); rint is ties-to-even
    mag = np.where(sat, E4M3_MAX, n * q)
    # code of a representable magnitude: exponent field and mantissa from the value
    _, ex2 = np.frexp(np.where(mag > 0, mag, 1.0))
    E2 = ex2 - 1
    normal = mag >= 2.0 ** -6
    efield = np.where(normal, E2 + 7, 0)
    mfield = np.where(normal, np.rint((mag / np.exp2(E2) - 1.0) * 8.0), np.rint(mag / 2.0 ** -9))
    code = (efield.astype(np.int64) << 3) | mfield.astype(np.int64)
    code = np.where(mag == 0, 0, code)
    return (code | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def fp8_row_scale(amax):
    """The per-token scale: the power of two 2^k with k the smallest integer such that
    amax <= 448 * 2^k (1 for amax = 0).  Float32."""
    a = np.asarray(amax, dtype=np.float64)
    _, e = np.frexp(np.where(a > 0, a / E4M3_MAX, 1.0))      # a / 448 = f 2^e, f in [0.5, 1)
    k = e.astype(np.int64)                                   # 2^e >= a / 448 > 2^(e-1) up to the division's rounding
    k = np.where(a > E4M3_MAX * np.exp2(k), k + 1, k)        # settle k by exact comparisons with 448 * 2^k
    k = np.where(a <= E4M3_MAX * np.exp2(k - 1), k - 1, k)
    return np.where(a > 0, np.exp2(k), 1.0).astype(np.float32)


def quantize_rows(rows):
    """Per-token FP8 rows: rows [n, w] (values in any precision) -> (codes uint8 [n, w], scales fp32 [n]).

    s_t = fp8_row_scale(amax_t); code = E4M3 RNE of fp32(x / s_t) (x / s_t is exact: s_t is a power
    of two)."""
    r = np.asarray(rows, dtype=np.float64)
    s = fp8_row_scale(np.max(np.abs(r), axis=-1))
    v = (r / s.astype(np.float64)[..., None]).astype(np.float32)
    return e4m3_encode_rne(v), s


def dequantize_rows(codes, scales) -> np.ndarray:
    """code value * scale, in float64."""
    return e4m3_decode(codes) * np.asarray(scales, np.float64)[..., None]


def fp8_cache_rows(c, kr_raw, pos, base: float = ROPE_BASE):
    """The FP8 cached row of a token: the row [c^KV | RoPE(k^R, pos)] (fp64 rotation, no bf16 step)
    quantized per token."""
    return quantize_rows(cache_rows(c, kr_raw, pos, base))
