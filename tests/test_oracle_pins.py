"""Pins for the fp64 oracle: values that do not come from the oracle itself.

Each pin is a checker function taking the oracle callable(s) it pins, so that the mutation
tests at the bottom can plant a plausible mistake in a copy of the oracle (on the CPU) and
show that some pin fails.

Sources: 《DeepSeek-V2》深度解读报告 §2.1-§2.4 and §3.1; DeepSeek-V2论文解读 (xdnf.cn) §2.1;
DeepSeek V2技术解析 (devpress) §1.  The RoPE anchors follow the original RoPE definition
(theta_i = 10000^(-2i/d)), which the pages name but do not print.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

import mla_inputs as mi
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SCALE = 1.0 / math.sqrt(mi.D_HEAD + mi.D_ROPE)


# ------------------------------------------------------------------ brute-force helpers
def bf_matvec_uk(w_uk, c):
    """k^C[h][j] = sum_k W_UK[h][j][k] c[k], by scalar loops."""
    H, dh, dc = w_uk.shape
    return [[sum(float(w_uk[h, j, k]) * float(c[k]) for k in range(dc)) for j in range(dh)]
            for h in range(H)]


def bf_matvec_uv(w_uv, c):
    """v^C[h][j] = sum_k W_UV[h][k][j] c[k], by scalar loops."""
    H, dc, dh = w_uv.shape
    return [[sum(float(w_uv[h, k, j]) * float(c[k]) for k in range(dc)) for j in range(dh)]
            for h in range(H)]


def bf_attention(q_nope, q_pe, c, kr_rot, w_uk, w_uv, scale):
    """Scalar-loop MLA attention for tiny shapes (no numpy arithmetic)."""
    H, dh = q_nope.shape
    L = c.shape[0]
    kC = [bf_matvec_uk(w_uk, c[t]) for t in range(L)]
    vC = [bf_matvec_uv(w_uv, c[t]) for t in range(L)]
    out, out_lat, lse = [], [], []
    for h in range(H):
        s = []
        for t in range(L):
            acc = 0.0
            for j in range(dh):
                acc += float(q_nope[h, j]) * kC[t][h][j]
            for j in range(q_pe.shape[1]):
                acc += float(q_pe[h, j]) * float(kr_rot[t, j])
            s.append(acc * scale)
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        p = [x / z for x in e]
        out.append([sum(p[t] * vC[t][h][j] for t in range(L)) for j in range(dh)])
        out_lat.append([sum(p[t] * float(c[t, k]) for t in range(L)) for k in range(c.shape[1])])
        lse.append(m + math.log(z))
    return np.array(out), np.array(out_lat), np.array(lse)


def tiny_case(seed, L, H=2, dh=3, dc=4, dr=2):
    rng = np.random.default_rng(seed)
    return dict(q_nope=rng.standard_normal((H, dh)), q_pe=rng.standard_normal((H, dr)),
                c=rng.standard_normal((L, dc)), kr_rot=rng.standard_normal((L, dr)),
                w_uk=rng.standard_normal((H, dh, dc)) * 0.5, w_uv=rng.standard_normal((H, dc, dh)) * 0.5)


# ------------------------------------------------------------------ pin checkers
def check_rope_anchors(apply_rope):
    """Closed-form anchors: theta_0 = 1, theta_8 = 0.1, theta_16 = 0.01, theta_24 = 0.001 (d=64)."""
    for i, pos in ((0, 1), (8, 10), (16, 100), (24, 1000), (0, 7), (16, 300)):
        for odd in (0, 1):
            x = np.zeros(64)
            x[2 * i + odd] = 1.0
            y = apply_rope(x, pos)
            a = float(pos) * (10.0 ** (-4.0 * (2 * i) / 64.0))   # 10000^(-2i/64)
            z = np.exp(1j * a) * (1.0 if odd == 0 else 1j)          # (x_e + i x_o) e^{i a}
            expect = np.zeros(64)
            expect[2 * i], expect[2 * i + 1] = z.real, z.imag
            assert np.allclose(y, expect, rtol=0, atol=1e-12), (i, pos, odd)


def check_rope_invariants(apply_rope):
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 64))
    assert np.array_equal(apply_rope(x, 0), x)                           # identity at t = 0
    for pos in (1, 37, 4095, 131071):
        y = apply_rope(x, pos)
        assert np.allclose((y[:, 0::2] ** 2 + y[:, 1::2] ** 2), (x[:, 0::2] ** 2 + x[:, 1::2] ** 2),
                           rtol=1e-12, atol=1e-12)                         # each pair keeps its norm
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n in ((5, 2), (100, 97), (3000, 10)):
        lhs = apply_rope(q, m) @ apply_rope(k, n)
        rhs = apply_rope(q, m - n) @ k
        assert abs(lhs - rhs) < 1e-9 * (1 + abs(lhs))                     # depends only on m - n


def check_attention_bruteforce(attend):
    for seed, L in ((1, 1), (2, 2), (3, 5), (4, 4)):
        t = tiny_case(seed, L)
        out, lat, lse = bf_attention(t["q_nope"], t["q_pe"], t["c"], t["kr_rot"], t["w_uk"], t["w_uv"], 0.37)
        r = attend(t["q_nope"], t["q_pe"], t["c"], t["kr_rot"], t["w_uk"], t["w_uv"], 0.37)
        assert np.allclose(r["out"], out, rtol=1e-12, atol=1e-12)
        assert np.allclose(r["out_lat"], lat, rtol=1e-12, atol=1e-12)
        assert np.allclose(r["lse"], lse, rtol=1e-12, atol=1e-12)


def check_special_cases(attend):
    # L = 1: all weight on the single token, out = v^C of that token, out_lat = c, lse = s.
    t = tiny_case(11, 1)
    r = attend(t["q_nope"], t["q_pe"], t["c"], t["kr_rot"], t["w_uk"], t["w_uv"], 0.5)
    vC = np.array(bf_matvec_uv(t["w_uv"], t["c"][0]))
    assert np.allclose(r["out"], vC, rtol=0, atol=1e-13)
    assert np.allclose(r["out_lat"], np.broadcast_to(t["c"][0], r["out_lat"].shape), rtol=0, atol=1e-13)
    # zero query: uniform weights, out_lat = mean of the rows, lse = log L.
    t = tiny_case(12, 5)
    r = attend(np.zeros_like(t["q_nope"]), np.zeros_like(t["q_pe"]), t["c"], t["kr_rot"], t["w_uk"], t["w_uv"], 0.5)
    assert np.allclose(r["out_lat"], np.broadcast_to(t["c"].mean(axis=0), r["out_lat"].shape), atol=1e-13)
    assert np.allclose(r["lse"], math.log(5), atol=1e-13)
    # L = 2: the weight of token 0 is the logistic sigmoid of s_0 - s_1.
    t = tiny_case(13, 2)
    r = attend(t["q_nope"], t["q_pe"], t["c"], t["kr_rot"], t["w_uk"], t["w_uv"], 0.5)
    kC = [bf_matvec_uk(t["w_uk"], t["c"][i]) for i in range(2)]
    for h in range(2):
        s = [0.5 * (sum(t["q_nope"][h, j] * kC[i][h][j] for j in range(3)) +
                    sum(t["q_pe"][h, j] * t["kr_rot"][i, j] for j in range(2))) for i in range(2)]
        p0 = scipy.special.expit(s[0] - s[1])
        assert np.allclose(r["out_lat"][h], p0 * t["c"][0] + (1 - p0) * t["c"][1], atol=1e-13)


def check_absorb_unabsorb(absorb_q, unabsorb_v):
    rng = np.random.default_rng(21)
    w_uk = rng.standard_normal((2, 3, 4))
    w_uv = rng.standard_normal((2, 4, 3))
    qn = rng.standard_normal((2, 3))
    lat = rng.standard_normal((2, 4))
    qa = absorb_q(qn, w_uk)
    ov = unabsorb_v(lat, w_uv)
    for h in range(2):
        for k in range(4):
            assert abs(qa[h, k] - sum(qn[h, j] * w_uk[h, j, k] for j in range(3))) < 1e-13
        for j in range(3):
            assert abs(ov[h, j] - sum(lat[h, k] * w_uv[h, k, j] for k in range(4))) < 1e-13


# ------------------------------------------------------------------ the pins
def test_cache_size_against_pages():
    g = json.load(open(os.path.join(GOLDEN, "mla_sizes.json")))
    assert (mi.N_HEADS, mi.D_HEAD, mi.D_LATENT, mi.D_ROPE) == (g["n_heads"], g["d_head"], g["d_latent"], g["d_rope"])
    assert oracle.mla_cache_elems_per_token(mi.D_LATENT, mi.D_ROPE) == g["mla_elems_per_token_per_layer"] == mi.D_ROW
    assert oracle.mla_cache_elems_per_token(mi.D_LATENT, mi.D_ROPE, g["n_layers"]) == g["mla_elems_per_token_60_layers"]
    mha = oracle.mha_cache_elems_per_token(mi.N_HEADS, mi.D_HEAD)
    assert mha == 32768
    # the page's printed MHA product is an arithmetic slip (formula gives 1,966,080)
    assert oracle.mha_cache_elems_per_token(mi.N_HEADS, mi.D_HEAD, g["n_layers"]) == 1966080 != g["mha_figure_printed_on_page"]
    # GQA equivalence: 576 cached elements = 2.25 groups of (K, V) of width d_h
    assert oracle.mla_cache_elems_per_token(mi.D_LATENT, mi.D_ROPE) / (2 * mi.D_HEAD) == g["gqa_equivalent_groups"]
    assert mi.D_LATENT == 4 * mi.D_HEAD and mi.D_ROPE == mi.D_HEAD // 2


def test_rope_anchors():
    check_rope_anchors(oracle.apply_rope)


def test_rope_invariants():
    check_rope_invariants(oracle.apply_rope)


def test_rope_inv_freq_anchors():
    th = oracle.rope_inv_freq(64)
    assert th.shape == (32,)
    assert th[0] == 1.0 and abs(th[16] - 0.01) < 1e-16 and abs(th[8] - 0.1) < 1e-16


def test_softmax_against_scipy():
    rng = np.random.default_rng(3)
    for s in (rng.standard_normal((4, 9)) * 3, np.array([[1000.0, 999.0, -1000.0]]), np.zeros((2, 6))):
        p, lse = oracle.softmax_stats(s)
        assert np.allclose(p, scipy.special.softmax(s, axis=-1), rtol=1e-14, atol=1e-300)
        assert np.allclose(lse, scipy.special.logsumexp(s, axis=-1), rtol=1e-14)


@pytest.mark.parametrize("form", ["explicit", "absorbed"])
def test_bruteforce_tiny(form):
    check_attention_bruteforce(oracle.attend_explicit if form == "explicit" else oracle.attend_absorbed)


@pytest.mark.parametrize("form", ["explicit", "absorbed"])
def test_special_cases(form):
    check_special_cases(oracle.attend_explicit if form == "explicit" else oracle.attend_absorbed)


def test_absorb_unabsorb_bruteforce():
    check_absorb_unabsorb(oracle.absorb_q, oracle.unabsorb_v)


def test_absorbed_equals_explicit_full_dims():
    """Associativity ([DR] §2.3): the absorbed and explicit forms agree to 1e-10 in fp64."""
    w = mi.layer_weights(5)
    b = mi.decode_batch(6, [97])
    f = mi.bf16_to_f64
    L = 97
    kr = oracle.apply_rope(f(b.kr[0]), np.arange(L))
    args = (f(b.q_nope[0]), f(b.q_pe[0]), f(b.c[0]), kr, f(w.w_uk), f(w.w_uv), SCALE)
    e = oracle.attend_explicit(*args)
    a = oracle.attend_absorbed(*args)
    for k in ("out", "out_lat", "lse"):
        rel = np.abs(e[k] - a[k]).max() / np.abs(e[k]).max()
        assert rel <= 1e-10, (k, rel)


def test_token_permutation_invariance():
    t = tiny_case(31, 7, H=3, dh=4, dc=6, dr=2)
    r0 = oracle.attend_explicit(**{k: t[k] for k in ("q_nope", "q_pe", "c", "kr_rot", "w_uk", "w_uv")}, scale=0.4)
    perm = np.random.default_rng(1).permutation(7)
    r1 = oracle.attend_explicit(t["q_nope"], t["q_pe"], t["c"][perm], t["kr_rot"][perm], t["w_uk"], t["w_uv"], 0.4)
    for k in ("out", "out_lat", "lse"):
        assert np.allclose(r0[k], r1[k], rtol=1e-13, atol=1e-13)


def test_split_merge_identity():
    rng = np.random.default_rng(9)
    qf = rng.standard_normal((4, 10))
    rows = rng.standard_normal((37, 10))
    full = oracle.attend_rows(qf, rows, 0.8, 8)
    for cuts in ([0, 37], [0, 16, 37], [0, 1, 2, 30, 37], [0, 12, 24, 36, 37]):
        parts = [oracle.partial_rows(qf, rows[a:b], 0.8, 8) for a, b in zip(cuts[:-1], cuts[1:])]
        lat, lse = oracle.merge_partials(parts)
        assert np.allclose(lat, full["out_lat"], rtol=1e-13, atol=1e-13)
        assert np.allclose(lse, full["lse"], rtol=1e-13, atol=1e-13)


def test_score_scale_sanity():
    """With the workload distributions the scaled score has std ~1: q_abs.c has variance ~128,
    q_pe.k_R has variance 64, total 192, times 1/192."""
    w = mi.layer_weights(41)
    b = mi.decode_batch(42, [512])
    f = mi.bf16_to_f64
    qa = oracle.absorb_q(f(b.q_nope[0]), f(w.w_uk))
    rows = oracle.cache_rows(f(b.c[0]), f(b.kr[0]), np.arange(512))
    s = oracle.attend_rows(oracle.q_full(qa, f(b.q_pe[0])), rows, SCALE, mi.D_LATENT)["s"]
    assert 0.9 < s.std() < 1.1, s.std()


def test_decode_step_forms_agree():
    w = mi.layer_weights(51)
    b = mi.decode_batch(52, [1, 65, 130])
    f = mi.bf16_to_f64
    args = (f(b.q_nope), f(b.q_pe), [f(x) for x in b.c], [f(x) for x in b.kr], f(w.w_uk), f(w.w_uv), SCALE)
    e = oracle.decode_step(*args, form="explicit", q_pos=[0, 64, 129])
    a = oracle.decode_step(*args, form="absorbed", q_pos=[0, 64, 129])
    for k in ("out", "out_lat", "lse", "q_abs"):
        assert np.allclose(e[k], a[k], rtol=1e-10, atol=1e-12)


def test_bf16_rounding_ties_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 65504.0, 1e-40])
    b = mi.f64_to_bf16(x)
    # 1+2^-8 is halfway between 1 and 1+2^-7: ties go to the even mantissa (1.0);
    # 1+3*2^-8 is halfway between 1+2^-7 and 1+2^-6... ties to even -> 1+2^-6
    assert list(mi.bf16_to_f64(b)[:4]) == [1.0, 1.0, 1.0 + 2 ** -6, -2.5]


# ------------------------------------------------------------------ planted mistakes
def _fails(fn, *a):
    try:
        fn(*a)
    except AssertionError:
        return True
    return False


def test_pins_catch_planted_rope_mistakes():
    def sign_flip(x, pos, base=oracle.ROPE_BASE):
        return oracle.apply_rope(x, -np.asarray(pos), base)

    def half_split(x, pos, base=oracle.ROPE_BASE):
        x = np.asarray(x, np.float64)
        d = x.shape[-1]
        ang = np.asarray(pos, np.float64)[..., None] * oracle.rope_inv_freq(d, base)
        a, b = x[..., : d // 2], x[..., d // 2:]
        return np.concatenate([a * np.cos(ang) - b * np.sin(ang), a * np.sin(ang) + b * np.cos(ang)], -1)

    def wrong_exponent(x, pos, base=oracle.ROPE_BASE):
        x = np.asarray(x, np.float64)
        d = x.shape[-1]
        th = np.power(base, -np.arange(d // 2) / d)
        ang = np.asarray(pos, np.float64)[..., None] * th
        y = np.empty_like(x)
        y[..., 0::2] = x[..., 0::2] * np.cos(ang) - x[..., 1::2] * np.sin(ang)
        y[..., 1::2] = x[..., 0::2] * np.sin(ang) + x[..., 1::2] * np.cos(ang)
        return y

    for bad in (sign_flip, half_split, wrong_exponent):
        assert _fails(check_rope_anchors, bad) or _fails(check_rope_invariants, bad), bad.__name__


def test_pins_catch_planted_attention_mistakes():
    def drop_rope_channel(q_nope, q_pe, c, kr, w_uk, w_uv, scale):
        return oracle.attend_explicit(q_nope, np.zeros_like(q_pe), c, kr, w_uk, w_uv, scale)

    def reversed_uv_index(q_nope, q_pe, c, kr, w_uk, w_uv, scale):
        r = oracle.attend_explicit(q_nope, q_pe, c, kr, w_uk, w_uv, scale)
        r["out"] = np.einsum("hk,hkj->hj", r["out_lat"], np.asarray(w_uv)[:, ::-1, :])
        return r

    def no_max_shift_but_wrong_norm(q_nope, q_pe, c, kr, w_uk, w_uv, scale):
        r = oracle.attend_explicit(q_nope, q_pe, c, kr, w_uk, w_uv, scale)
        r["lse"] = r["lse"] - 1e-3
        return r

    for bad in (drop_rope_channel, reversed_uv_index, no_max_shift_but_wrong_norm):
        assert _fails(check_attention_bruteforce, bad), bad.__name__


def test_pins_catch_planted_absorb_mistakes():
    def uk_wrong_index(qn, w_uk):
        return np.einsum("hj,hjk->hk", qn, w_uk[::-1])          # heads swapped

    assert _fails(check_absorb_unabsorb, uk_wrong_index, oracle.unabsorb_v)


# ------------------------------------------------------------------ down-projection + append
def bf_project_rows(h, w_dkv, w_kr, pos, base=oracle.ROPE_BASE):
    """[W_D^KV h | RoPE(W^KR h)] by scalar loops: the rotation of each pair written out with
    math.cos / math.sin of pos * base^(-2i/d_R)."""
    n, d = h.shape
    dc, dr = w_dkv.shape[0], w_kr.shape[0]
    rows = []
    for t in range(n):
        c = [sum(float(w_dkv[j, k]) * float(h[t, k]) for k in range(d)) for j in range(dc)]
        kr = [sum(float(w_kr[j, k]) * float(h[t, k]) for k in range(d)) for j in range(dr)]
        rot = []
        for i in range(dr // 2):
            a = float(pos[t]) * float(base) ** (-2.0 * i / dr)
            x, y = kr[2 * i], kr[2 * i + 1]
            rot += [x * math.cos(a) - y * math.sin(a), x * math.sin(a) + y * math.cos(a)]
        rows.append(c + rot)
    return np.array(rows)


def check_project_rows(project_rows):
    rng = np.random.default_rng(11)
    h = rng.standard_normal((3, 7))
    w_dkv = rng.standard_normal((5, 7))
    w_kr = rng.standard_normal((4, 7))
    pos = np.array([0, 3, 1000])
    got = project_rows(h, w_dkv, w_kr, pos)
    assert got.shape == (3, 9)
    assert np.allclose(got, bf_project_rows(h, w_dkv, w_kr, pos), rtol=1e-12, atol=1e-12)
    # Selection weights reduce it to the plain append of (c, k^R) = parts of h.
    c = rng.standard_normal((2, 4))
    kr = rng.standard_normal((2, 2))
    hsel = np.concatenate([c, kr, rng.standard_normal((2, 3))], axis=1)       # d = 9
    sel_c = np.eye(4, 9)
    sel_k = np.eye(2, 9, k=4)
    p2 = np.array([5, 77])
    assert np.allclose(project_rows(hsel, sel_c, sel_k, p2), oracle.cache_rows(c, kr, p2), rtol=0, atol=1e-14)
    # Linear in h at fixed positions.
    h2 = rng.standard_normal((3, 7))
    lhs = project_rows(2.0 * h - 0.5 * h2, w_dkv, w_kr, pos)
    rhs = 2.0 * project_rows(h, w_dkv, w_kr, pos) - 0.5 * project_rows(h2, w_dkv, w_kr, pos)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def test_project_rows_pins():
    check_project_rows(oracle.project_rows)


def test_pins_catch_planted_projection_mistakes():
    def parts_swapped(h, w_dkv, w_kr, pos, base=oracle.ROPE_BASE):
        r = oracle.project_rows(h, w_dkv, w_kr, pos, base)
        dc = w_dkv.shape[0]
        return np.concatenate([r[:, dc:], r[:, :dc]], axis=1)

    def rope_on_latent(h, w_dkv, w_kr, pos, base=oracle.ROPE_BASE):
        r = oracle.project_rows(h, w_dkv, w_kr, pos, base)
        dc = w_dkv.shape[0] - w_dkv.shape[0] % 2
        r[:, :dc] = oracle.apply_rope(r[:, :dc], pos, base)
        return r

    def unrotated_key(h, w_dkv, w_kr, pos, base=oracle.ROPE_BASE):
        return oracle.project_rows(h, w_dkv, w_kr, np.zeros_like(np.asarray(pos)), base)

    for bad in (parts_swapped, rope_on_latent, unrotated_key):
        assert _fails(check_project_rows, bad), bad.__name__


# ------------------------------------------------------------------ output projection
def check_output_proj(output_proj):
    rng = np.random.default_rng(12)
    out = rng.standard_normal((3, 2, 3))          # B = 3, H = 2, d_h = 3
    w_o = rng.standard_normal((4, 6))             # d = 4, H d_h = 6
    got = output_proj(out, w_o)
    assert got.shape == (3, 4)
    # scalar loops over heads and head dims: y[b][i] = sum_h sum_j W_O[i][h*3 + j] out[b][h][j]
    bf = [[sum(float(w_o[i, h * 3 + j]) * float(out[b, h, j]) for h in range(2) for j in range(3))
           for i in range(4)] for b in range(3)]
    assert np.allclose(got, np.array(bf), rtol=1e-12, atol=1e-12)
    # one-hot weights pick single (head, dim) entries
    sel = np.zeros((4, 6))
    sel[0, 5] = sel[1, 0] = sel[2, 3] = sel[3, 1] = 1.0
    assert np.array_equal(output_proj(out, sel), np.stack([out[:, 1, 2], out[:, 0, 0], out[:, 1, 0], out[:, 0, 1]], 1))


def test_output_proj_pins():
    check_output_proj(oracle.output_proj)


def test_pins_catch_planted_output_proj_mistakes():
    def dim_major_concat(out, w_o):
        return np.asarray(out, np.float64).transpose(0, 2, 1).reshape(out.shape[0], -1) @ np.asarray(w_o).T

    def heads_reversed(out, w_o):
        return oracle.output_proj(np.asarray(out)[:, ::-1, :], w_o)

    for bad in (dim_major_concat, heads_reversed):
        assert _fails(check_output_proj, bad), bad.__name__


# ------------------------------------------------------------------ chunked prefill
def bf_prefill_row(qf, rows, L, scale, d_latent):
    """Scalar loops: one absorbed query row [H][d_c + d_R] over the first L rows."""
    H = len(qf)
    lat, lse = [], []
    for h in range(H):
        s = [scale * sum(float(qf[h][k]) * float(rows[t][k]) for k in range(len(qf[h]))) for t in range(L)]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        lat.append([sum(e[t] / z * float(rows[t][k]) for t in range(L)) for k in range(d_latent)])
        lse.append(m + math.log(z))
    return lat, lse


def prefill_case(seed, L=9, n=4, H=2, dh=3, dc=4, dr=2):
    """One sequence of L cached tokens whose last n are a new chunk (positions L-n .. L-1)."""
    t = tiny_case(seed, L, H, dh, dc, dr)
    rng = np.random.default_rng(seed + 100)
    t["q_nope"] = rng.standard_normal((n, H, dh))
    t["q_pe"] = rng.standard_normal((n, H, dr))
    t["q_pos"] = np.arange(L - n, L)
    return t


def check_prefill_bruteforce(prefill_rows):
    """Scalar-loop pin: every row attends to exactly the tokens at or before its position, in
    several sequences at once, and an empty row gives zeros and -inf."""
    t = prefill_case(31)
    rows = np.concatenate([t["c"], t["kr_rot"]], axis=1)
    other = np.random.default_rng(32).standard_normal((5, rows.shape[1]))
    qf = np.concatenate([oracle.absorb_q(t["q_nope"], t["w_uk"]), t["q_pe"]], axis=-1)
    qf = np.concatenate([qf, qf[:2]], axis=0)                       # two more rows, on sequence 1
    q_seq = np.array([0, 0, 0, 0, 1, 1])
    q_len = np.concatenate([t["q_pos"] + 1, [3, 0]])
    r = prefill_rows(qf, [rows, other], q_seq, q_len, 0.41, 4)
    for i in range(5):
        lat, lse = bf_prefill_row(qf[i], [rows, other][q_seq[i]], int(q_len[i]), 0.41, 4)
        assert np.allclose(r["out_lat"][i], lat, rtol=1e-12, atol=1e-12), i
        assert np.allclose(r["lse"][i], lse, rtol=1e-12, atol=1e-12), i
    assert np.array_equal(r["out_lat"][5], np.zeros_like(r["out_lat"][5])) and np.all(r["lse"][5] == -np.inf)


def check_prefill_causal(prefill_rows):
    """Rows of tokens after a query's position never reach it; its own row does."""
    t = prefill_case(33)
    rows = np.concatenate([t["c"], t["kr_rot"]], axis=1)
    qf = np.concatenate([oracle.absorb_q(t["q_nope"], t["w_uk"]), t["q_pe"]], axis=-1)
    q_seq, q_len = np.zeros(4, int), t["q_pos"] + 1
    base = prefill_rows(qf, [rows], q_seq, q_len, 0.41, 4)
    for i, p in enumerate(t["q_pos"]):
        later = rows.copy()
        later[p + 1:] = 1e3                                          # every token after position p
        r = prefill_rows(qf, [later], q_seq, q_len, 0.41, 4)
        assert np.array_equal(r["out_lat"][i], base["out_lat"][i]), i
        own = rows.copy()
        own[p] += 1.0                                                # the query's own token
        r = prefill_rows(qf, [own], q_seq, q_len, 0.41, 4)
        assert not np.allclose(r["out_lat"][i], base["out_lat"][i]), i


def check_prefill_against_masked_explicit(prefill_rows, prefill_explicit_masked):
    """The absorbed row-at-a-time form against the textbook masked-matrix form in the explicit
    (decompressed) basis, at the real head and latent widths."""
    rng = np.random.default_rng(35)
    H, dh, dc, dr, L, n = 4, mi.D_HEAD, mi.D_LATENT, mi.D_ROPE, 40, 7
    c = rng.standard_normal((L, dc))
    kr = rng.standard_normal((L, dr))
    w_uk = rng.standard_normal((H, dh, dc)) / math.sqrt(dc)
    w_uv = rng.standard_normal((H, dc, dh)) / math.sqrt(dc)
    qn, qp = rng.standard_normal((n, H, dh)), rng.standard_normal((n, H, dr))
    q_pos = np.array([33, 34, 35, 36, 37, 38, 39])
    ex = prefill_explicit_masked(qn, qp, c, kr, w_uk, w_uv, SCALE, q_pos)
    qf = np.concatenate([oracle.absorb_q(qn, w_uk), qp], axis=-1)
    r = prefill_rows(qf, [np.concatenate([c, kr], axis=1)], np.zeros(n, int), q_pos + 1, SCALE, dc)
    assert np.allclose(r["out_lat"], ex["out_lat"], rtol=1e-10, atol=1e-12)
    assert np.allclose(r["lse"], ex["lse"], rtol=1e-10, atol=1e-12)
    assert np.allclose(oracle.unabsorb_v(r["out_lat"], w_uv), ex["out"], rtol=1e-10, atol=1e-12)


def test_prefill_pins():
    check_prefill_bruteforce(oracle.prefill_rows)
    check_prefill_causal(oracle.prefill_rows)
    check_prefill_against_masked_explicit(oracle.prefill_rows, oracle.prefill_explicit_masked)


def test_pins_catch_planted_prefill_mistakes():
    def mask_off_by_one(qf, seq_rows, q_seq, q_len, scale, d_latent):          # the query misses itself
        return oracle.prefill_rows(qf, seq_rows, q_seq, np.maximum(np.asarray(q_len) - 1, 0), scale, d_latent)

    def sees_whole_sequence(qf, seq_rows, q_seq, q_len, scale, d_latent):      # no causal mask
        return oracle.prefill_rows(qf, seq_rows, q_seq, [len(seq_rows[s]) for s in q_seq], scale, d_latent)

    def first_sequence_only(qf, seq_rows, q_seq, q_len, scale, d_latent):      # map ignored
        return oracle.prefill_rows(qf, seq_rows, np.zeros_like(np.asarray(q_seq)), q_len, scale, d_latent)

    for bad in (mask_off_by_one, sees_whole_sequence, first_sequence_only):
        assert _fails(check_prefill_bruteforce, bad), bad.__name__

    def masked_inclusive(qn, qp, c, kr, w_uk, w_uv, scale, q_pos):             # masks the query's own token
        return oracle.prefill_explicit_masked(qn, qp, c, kr, w_uk, w_uv, scale, np.asarray(q_pos) - 1)

    assert _fails(check_prefill_against_masked_explicit, oracle.prefill_rows, masked_inclusive)


# ------------------------------------------------------------------ whole decode step: positions
# 《DeepSeek-V2》深度解读报告 §2.4 Decoupled RoPE: the shared key k^R of the token at position t is
# cached rotated by RoPE at t, and the query's position part q^R is rotated at the query's own
# position.  decode_step does that rotation itself (token t of sequence b sits at position t), so
# its positional glue is pinned here by scalar loops that rotate every pair with math.cos/sin.
def bf_rotate(x, pos, base=oracle.ROPE_BASE):
    """One interleaved RoPE rotation by scalar loops: pair (x[2i], x[2i+1]) turned by
    pos * base^(-2i/d)."""
    d = len(x)
    y = []
    for i in range(d // 2):
        a = float(pos) * float(base) ** (-2.0 * i / d)
        u, v = float(x[2 * i]), float(x[2 * i + 1])
        y += [u * math.cos(a) - v * math.sin(a), u * math.sin(a) + v * math.cos(a)]
    return np.array(y)


def bf_decode_step(q_nope, q_pe, cs, krs_raw, w_uk, w_uv, scale, q_pos=None):
    """Scalar-loop decode step: keys rotated at their token index, q^R at q_pos[b] (as given when
    q_pos is None), then the scalar-loop attention and the scalar-loop absorbed query."""
    out, lat, lse, qa = [], [], [], []
    for b in range(len(cs)):
        L = cs[b].shape[0]
        kr_rot = np.array([bf_rotate(krs_raw[b][t], t) for t in range(L)])
        qpe = np.array(q_pe[b]) if q_pos is None else np.array([bf_rotate(q_pe[b][h], q_pos[b])
                                                                 for h in range(q_pe.shape[1])])
        o, l_, s = bf_attention(q_nope[b], qpe, cs[b], kr_rot, w_uk, w_uv, scale)
        out.append(o); lat.append(l_); lse.append(s)
        H, dh, dc = w_uk.shape
        qa.append([[sum(float(q_nope[b, h, j]) * float(w_uk[h, j, k]) for j in range(dh)) for k in range(dc)]
                   for h in range(H)])
    return dict(out=np.array(out), out_lat=np.array(lat), lse=np.array(lse), q_abs=np.array(qa))


def check_decode_step_positions(decode_step):
    rng = np.random.default_rng(61)
    H, dh, dc, dr = 2, 3, 4, 4           # two RoPE pairs: theta_0 = 1 and theta_1 = 10000^(-1/2)
    lens = [3, 5]
    q_nope = rng.standard_normal((2, H, dh))
    q_pe = rng.standard_normal((2, H, dr))
    cs = [rng.standard_normal((L, dc)) for L in lens]
    krs = [rng.standard_normal((L, dr)) for L in lens]
    w_uk = rng.standard_normal((H, dh, dc)) * 0.5
    w_uv = rng.standard_normal((H, dc, dh)) * 0.5
    # the new token's own position (L - 1), an arbitrary one, and q^R taken as already rotated
    for q_pos in ([L - 1 for L in lens], [7, 1], None):
        ref = bf_decode_step(q_nope, q_pe, cs, krs, w_uk, w_uv, 0.45, q_pos)
        for form in ("explicit", "absorbed"):
            got = decode_step(q_nope, q_pe, cs, krs, w_uk, w_uv, 0.45, q_pos=q_pos, form=form)
            for k in ("out", "out_lat", "lse", "q_abs"):
                assert np.allclose(got[k], ref[k], rtol=1e-12, atol=1e-12), (q_pos, form, k)


def test_decode_step_positions_pin():
    check_decode_step_positions(oracle.decode_step)


def test_pins_catch_planted_decode_step_mistakes():
    # R(t) R(1) = R(t + 1): rotating every raw key by one position first plants "keys at t + 1".
    def keys_one_late(q_nope, q_pe, cs, krs, w_uk, w_uv, scale, base=oracle.ROPE_BASE, q_pos=None, form="explicit"):
        krs1 = [oracle.apply_rope(k, 1, base) for k in krs]
        return oracle.decode_step(q_nope, q_pe, cs, krs1, w_uk, w_uv, scale, base, q_pos, form)

    def keys_unrotated(q_nope, q_pe, cs, krs, w_uk, w_uv, scale, base=oracle.ROPE_BASE, q_pos=None, form="explicit"):
        # R(-t) R(t) = identity: undo the step's own rotation of token t
        krs0 = [oracle.apply_rope(k, -np.arange(len(k)), base) for k in krs]
        return oracle.decode_step(q_nope, q_pe, cs, krs0, w_uk, w_uv, scale, base, q_pos, form)

    def query_unrotated(q_nope, q_pe, cs, krs, w_uk, w_uv, scale, base=oracle.ROPE_BASE, q_pos=None, form="explicit"):
        return oracle.decode_step(q_nope, q_pe, cs, krs, w_uk, w_uv, scale, base, None, form)

    def query_at_length(q_nope, q_pe, cs, krs, w_uk, w_uv, scale, base=oracle.ROPE_BASE, q_pos=None, form="explicit"):
        qp = None if q_pos is None else [len(c) for c in cs]
        return oracle.decode_step(q_nope, q_pe, cs, krs, w_uk, w_uv, scale, base, qp, form)

    def query_negated_angle(q_nope, q_pe, cs, krs, w_uk, w_uv, scale, base=oracle.ROPE_BASE, q_pos=None, form="explicit"):
        qp = None if q_pos is None else [-p for p in q_pos]
        return oracle.decode_step(q_nope, q_pe, cs, krs, w_uk, w_uv, scale, base, qp, form)

    for bad in (keys_one_late, keys_unrotated, query_unrotated, query_at_length, query_negated_angle):
        assert _fails(check_decode_step_positions, bad), bad.__name__


# ------------------------------------------------------------------ FP8 (E4M3) latent cache
# 《DeepSeek-V2》深度解读报告 §4.2 效率证据: FP8 serving with the KV cache at about 6 bits per element.
# The format pinned here is OCP E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa bits,
# subnormals m * 2^-9, largest finite 448, S.1111.111 NaN, no infinities).
E4M3_ANCHORS = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x0F: 1.875 * 2.0 ** -6,
                0x38: 1.0, 0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x48: 4.0, 0x77: 240.0, 0x78: 256.0,
                0x7E: 448.0, 0x80: -0.0, 0xB8: -1.0, 0xFE: -448.0}


def check_e4m3_decode(e4m3_decode):
    codes = np.array(list(E4M3_ANCHORS), dtype=np.uint8)
    got = e4m3_decode(codes)
    for c, g in zip(codes, got):
        assert g == E4M3_ANCHORS[int(c)] and math.copysign(1, g) == math.copysign(1, E4M3_ANCHORS[int(c)]), hex(c)
    assert np.isnan(e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()
    assert not np.isnan(e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))).any()


def bf_e4m3_nearest(v):
    """Brute force: the non-negative finite code whose value (from the anchors' rule written out
    as scalar arithmetic) is nearest to |v|, ties to the even code, 448 for |v| >= 448; sign bit
    from v."""
    a = abs(float(v))
    best, bestd = None, None
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        val = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        d = abs(val - a)
        if best is None or d < bestd or (d == bestd and c % 2 == 0):
            best, bestd = c, d
    if a >= 448.0:
        best = 0x7E
    return best | (0x80 if math.copysign(1, float(v)) < 0 else 0)


def check_e4m3_encode(e4m3_encode_rne, e4m3_decode):
    # every finite code round-trips
    codes = np.arange(256, dtype=np.uint8)
    vals = e4m3_decode(codes)
    fin = ~np.isnan(vals)
    assert np.array_equal(e4m3_encode_rne(vals[fin].astype(np.float32)), codes[fin])
    # exact midpoints between neighbours, just above and below them, saturation, tiny values
    pos = np.sort(np.unique(np.abs(vals[fin])))
    mids = (pos[:-1] + pos[1:]) / 2
    rng = np.random.default_rng(71)
    probe = np.concatenate([mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
                            np.nextafter(mids.astype(np.float32), np.float32(1000)),
                            [448.0, 460.0, 479.99, 480.0, 1e6, 2.0 ** -10, 2.0 ** -11, 1e-30, 0.0],
                            rng.standard_normal(300) * 3, rng.standard_normal(100) * 200]).astype(np.float32)
    probe = np.concatenate([probe, -probe])
    got = e4m3_encode_rne(probe)
    want = np.array([bf_e4m3_nearest(x) for x in probe], dtype=np.uint8)
    assert np.array_equal(got, want), probe[got != want][:5]


def bf_pow2_scale(amax):
    """Brute force: the smallest power of two p (as 2^k, k an integer) with amax <= 448 p."""
    if amax == 0:
        return 1.0
    k = -200
    while amax > 448.0 * 2.0 ** k:
        k += 1
    return 2.0 ** k


def check_quantize_rows(quantize_rows, e4m3_decode):
    rng = np.random.default_rng(72)
    rows = rng.standard_normal((6, 576)) * np.array([1, 0.01, 100, 3, 1e-3, 1])[:, None]
    rows[5, 7] = 448.0 * 2.0 ** -2                                               # amax exactly 448 * 2^k
    codes, s = quantize_rows(rows)
    assert codes.dtype == np.uint8 and codes.shape == rows.shape and s.dtype == np.float32
    amax = np.abs(rows).max(axis=1)
    assert [float(x) for x in s] == [bf_pow2_scale(float(a)) for a in amax]      # power-of-two scale from the row max
    top = np.abs(rows).argmax(axis=1)
    assert all(0x76 <= (codes[i, top[i]] & 0x7F) <= 0x7E for i in range(6))     # the max codes into (224, 448]
    assert (codes[5, 7] & 0x7F) == 0x7E
    xh = e4m3_decode(codes) * s.astype(np.float64)[:, None]
    bound = 2.0 ** -4 * np.abs(rows) + 2.0 ** -10 * s.astype(np.float64)[:, None]   # half a step: normal / subnormal
    assert (np.abs(xh - rows) <= bound * (1 + 1e-12)).all()
    assert np.array_equal(np.sign(xh[xh != 0]), np.sign(rows[xh != 0]))
    # rows of representable values times a power of two come back exactly, scale included
    k = rng.integers(0, 0x7E, size=(3, 576)).astype(np.uint8)
    k[:, 5] = 0x7E
    vals = e4m3_decode(k) * (2.0 ** np.array([-3.0, 0.0, 5.0]))[:, None]
    c2, s2 = quantize_rows(vals)
    assert np.array_equal(c2, k) and np.array_equal(s2, np.float32([2.0 ** -3, 1.0, 2.0 ** 5]))
    # a code times its scale is exact in bf16 (8 significant bits): decoded values have <= 4
    dec = (e4m3_decode(codes) * s.astype(np.float64)[:, None]).astype(np.float32)
    assert np.array_equal(dec.view(np.uint32) & 0xFFFF, np.zeros_like(dec.view(np.uint32)))
    # sign symmetry and the all-zero row
    c3, s3 = quantize_rows(-rows)
    assert np.array_equal(c3, codes ^ 0x80) and np.array_equal(s3, s)
    c4, s4 = quantize_rows(np.zeros((1, 576)))
    assert not c4.any() and s4[0] == 1.0


def test_e4m3_and_fp8_quantizer_pins():
    check_e4m3_decode(oracle.e4m3_decode)
    check_e4m3_encode(oracle.e4m3_encode_rne, oracle.e4m3_decode)
    check_quantize_rows(oracle.quantize_rows, oracle.e4m3_decode)


def test_fp8_cache_rows_pin():
    """fp8_cache_rows quantizes the fp64 row [c | RoPE(k^R, pos)]: checked against the scalar-loop
    rotation and the brute-force nearest code, element by element."""
    rng = np.random.default_rng(73)
    c = rng.standard_normal((3, 8))
    kr = rng.standard_normal((3, 4)) * 3
    pos = [0, 5, 1000]
    codes, s = oracle.fp8_cache_rows(c, kr, pos)
    for t in range(3):
        row = list(c[t]) + list(bf_rotate(kr[t], pos[t]))
        st = bf_pow2_scale(max(abs(x) for x in row))
        assert s[t] == st
        want = [bf_e4m3_nearest(np.float32(x / float(st))) for x in row]
        assert list(codes[t]) == want


def test_pins_catch_planted_fp8_mistakes():
    def truncating(v):                       # rounds toward zero instead of to nearest
        v = np.asarray(v, np.float32)
        out = oracle.e4m3_encode_rne(v)
        dec = oracle.e4m3_decode(out)
        over = np.abs(dec) > np.abs(v.astype(np.float64))
        return np.where(over & ((out & 0x7F) > 0), out - 1, out).astype(np.uint8)

    def ties_away(v):                        # ties away from zero
        v = np.asarray(v, np.float32).astype(np.float64)
        a = np.abs(v)
        _, ex = np.frexp(np.where(a > 0, a, 1.0))
        q = np.exp2(np.maximum(ex - 1, -6) - 3.0)
        mag = np.minimum(np.floor(a / q + 0.5) * q, 448.0)
        return oracle.e4m3_encode_rne(np.copysign(mag, v).astype(np.float32))

    def no_saturation(v):                    # wraps past 448 into the NaN code
        out = oracle.e4m3_encode_rne(v)
        big = np.abs(np.asarray(v, np.float32)) >= 480
        return np.where(big, out | 0x7F, out).astype(np.uint8)

    for bad in (truncating, ties_away, no_saturation):
        assert _fails(check_e4m3_encode, bad, oracle.e4m3_decode), bad.__name__

    def bias_six(codes):                     # exponent bias 6 instead of 7
        return oracle.e4m3_decode(codes) * 2.0

    assert _fails(check_e4m3_decode, bias_six)

    def scale_from_240(rows):                # the E4M3-FNUZ maximum instead of 448
        r = np.asarray(rows, np.float64)
        s = np.exp2(np.ceil(np.log2(np.maximum(np.abs(r).max(axis=-1), 1e-300) / 240.0))).astype(np.float32)
        return oracle.e4m3_encode_rne((r / s.astype(np.float64)[..., None]).astype(np.float32)), s

    def scale_not_pow2(rows):                # amax / 448 itself
        r = np.asarray(rows, np.float64)
        s = (np.abs(r).max(axis=-1) / 448.0).astype(np.float32)
        s = np.where(s > 0, s, 1).astype(np.float32)
        return oracle.e4m3_encode_rne((r / s.astype(np.float64)[..., None]).astype(np.float32)), s

    for bad in (scale_from_240, scale_not_pow2):
        assert _fails(check_quantize_rows, bad, oracle.e4m3_decode), bad.__name__
