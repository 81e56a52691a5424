"""Pins of the fp64 oracle against what the VideoMLA paper and mathematics fix.

"VideoMLA: Low-Rank Latent KV Cache for Minute-Scale Autoregressive Video
Diffusion" (arXiv 2605.30351) prints no worked numerical example of the
attention path, so the oracle is pinned by (1) the cache-size numbers it prints,
(2) the exact equivalence of its App. E absorbed form with the §3.3 explicit
form, (3) a brute-force formulation with explicit block-diagonal rotation
matrices and scalar loops, (4) RoPE invariants (identity at the origin,
orthogonality, relative-position / shift invariance, the one-pair closed form),
(5) softmax and attention special cases with closed-form results, and (6)
ring-placement examples worked by hand.  Each pin is chosen so that a dropped
term, a wrong sign or index, or a transposed operand in the oracle fails at
least one of them; the mutation tests at the end plant such mistakes in a copy
of the oracle and check that the pins catch them.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import videomla_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cache_accounting.json")


# ---------------------------------------------------------------------------
# (1) printed numbers
# ---------------------------------------------------------------------------

def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_per_token_cache_counts_match_paper():
    g = _golden()["per_token"]
    lat = O.latent_scalars_per_token(g["d_c"], g["d_rope"])
    den = O.dense_scalars_per_token(g["n_heads"], g["d_head"])
    assert lat == g["latent_scalars"] == 224
    assert den == g["dense_scalars"] == 3072
    assert round(100.0 * (1.0 - lat / den), 1) == g["reduction_percent"]
    assert round(den / lat, 1) == g["reduction_factor"]


def test_dense_window_size_matches_paper():
    g = _golden()["dense_window"]
    den = O.dense_scalars_per_token(12, 128)
    scal = O.cache_scalars(g["layers"], g["frames"], g["tokens_per_frame"], den)
    assert round(scal / 1e9, 2) == g["scalars_billions"]
    assert round(O.cache_bytes(scal) / 1e9, 1) == g["gigabytes_bf16"]


def test_scd_comparison_matches_paper():
    g = _golden()["scd"]
    den = O.dense_scalars_per_token(12, 128)
    lat = O.latent_scalars_per_token(192, 32)
    full = O.cache_scalars(g["layers"], 21, 1560, den)
    scd = O.cache_scalars(g["scd_encoder_layers"], 21, 1560, den)
    vmla = O.cache_scalars(g["layers"], 21, 1560, lat)
    assert round(100.0 * (1.0 - scd / full), 1) == g["scd_dense_reduction_percent"]
    assert round(scd / vmla, 1) == g["videomla_vs_scd_factor"]


def test_table5a_memory_ratios_match_paper():
    g = _golden()["table5a_memory_ratio"]
    den = O.dense_scalars_per_token(12, 128)
    for d_c, printed in g["ratios"].items():
        assert round(den / O.latent_scalars_per_token(int(d_c), g["d_rope"]), 2) == printed


def test_geometry_and_rope_split_match_paper():
    g = _golden()
    geo = g["geometry"]
    assert geo["grid_h"] * geo["grid_w"] == geo["tokens_per_frame"]
    assert geo["tokens_per_frame"] * geo["frames_per_clip"] == geo["tokens_per_clip"]
    assert O.rope_pair_split(g["rope_split"]["d_rope"]) == tuple(g["rope_split"]["pairs_t_h_w"])
    # the sweep widths follow the same rule (reading) and always cover d_rope
    for d_rope in (8, 16, 32, 64, 96):
        t, h, w = O.rope_pair_split(d_rope)
        assert 2 * (t + h + w) == d_rope and h == w and t >= h


def test_composite_operator_rank_bounded_by_latent_width():
    # [VideoMLA] §5: M = [W_uk W_dkv ; W_uv W_dkv] has rank <= d_c by construction.
    rng = np.random.default_rng(0)
    d, H, d_c, d_nope, d_v = 64, 3, 10, 8, 8
    M = O.composite_kv_operator(rng.normal(size=(H * d_nope, d_c)),
                                rng.normal(size=(H * d_v, d_c)),
                                rng.normal(size=(d_c, d)))
    assert M.shape == (H * (d_nope + d_v), d)
    assert np.linalg.matrix_rank(M) == d_c


# ---------------------------------------------------------------------------
# RoPE invariants
# ---------------------------------------------------------------------------

def test_rope_frequencies_structure():
    omega, axis = O.rope_frequencies(32, 128)
    assert list(np.bincount(axis)) == [6, 5, 5]
    for a in range(3):
        w = omega[axis == a]
        assert w[0] == 1.0                                   # highest-frequency band first
        assert np.all(np.diff(w) < 0) and np.all(w > 0)
        r = w[1:] / w[:-1]                                   # one geometric ladder per axis
        assert np.allclose(r, r[0], rtol=0, atol=1e-15)
    # the t axis owns a wider band of the full head than h and w, so its ladder is finer
    assert omega[axis == 0][1] > omega[axis == 1][1] == omega[axis == 2][1]


def test_rope_identity_orthogonality_and_composition():
    rng = np.random.default_rng(1)
    v = rng.normal(size=(7, 32))
    omega, axis = O.rope_frequencies(32, 128)
    zero = O.rope_angles(np.zeros((7, 3), dtype=int), omega, axis)
    assert np.array_equal(O.rope_rotate(v, zero), v)
    pos = rng.integers(0, 60, size=(7, 3))
    th = O.rope_angles(pos, omega, axis)
    r = O.rope_rotate(v, th)
    assert np.allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(v, axis=-1), rtol=1e-14)
    pos2 = rng.integers(0, 60, size=(7, 3))
    th2 = O.rope_angles(pos2, omega, axis)
    assert np.allclose(O.rope_rotate(O.rope_rotate(v, th), th2),
                       O.rope_rotate(v, O.rope_angles(pos + pos2, omega, axis)), atol=1e-12)
    # rotating back by the negated angle restores the vector
    assert np.allclose(O.rope_rotate(r, -th), v, atol=1e-13)


def test_rope_single_pair_closed_form():
    # One complex pair: q . k after rotation = |q||k| cos(phi_k - phi_q + omega (n - m)).
    omega, axis = O.rope_frequencies(32, 128)
    for p in (0, 3, 7, 15):
        q = np.zeros(32); k = np.zeros(32)
        q[2 * p:2 * p + 2] = [1.3 * math.cos(0.4), 1.3 * math.sin(0.4)]
        k[2 * p:2 * p + 2] = [0.7 * math.cos(-1.1), 0.7 * math.sin(-1.1)]
        m = np.array([2, 5, 11]); n = np.array([9, 1, 40])
        s = O.rope_rotate(q, O.rope_angles(m, omega, axis)) @ O.rope_rotate(k, O.rope_angles(n, omega, axis))
        a = axis[p]
        expect = 1.3 * 0.7 * math.cos(-1.1 - 0.4 + omega[p] * (n[a] - m[a]))
        assert abs(s - expect) < 1e-13


def test_rope_scores_shift_invariant():
    # [VideoMLA] App. D.5 relies on RoPE being relative: shifting every query and
    # key position by the same (dt, dh, dw) leaves all scores unchanged.
    rng = np.random.default_rng(2)
    omega, axis = O.rope_frequencies(32, 128)
    q = rng.normal(size=(5, 32)); k = rng.normal(size=(9, 32))
    qp = rng.integers(0, 30, size=(5, 3)); kp = rng.integers(0, 30, size=(9, 3))
    def scores(dq):
        return (O.rope_rotate(q, O.rope_angles(qp + dq, omega, axis))
                @ O.rope_rotate(k, O.rope_angles(kp + dq, omega, axis)).T)
    s0 = scores(np.array([0, 0, 0]))
    for d in ([7, 0, 0], [0, 13, 0], [0, 0, 29], [40, 3, 11]):
        assert np.max(np.abs(scores(np.array(d)) - s0)) <= 1e-12 * np.max(np.abs(s0))


# ---------------------------------------------------------------------------
# ring placement and window decode, worked by hand
# ---------------------------------------------------------------------------

def test_window_keys_worked_example():
    # slots = 4, frames of T_f = 2 tokens (grid 1 x 2); oldest valid frame in
    # slot 2, three frames valid -> logical frames live in slots 2, 3, 0.
    rows, pos = O.window_keys(slots=4, oldest=2, n_valid=3, grid_h=1, grid_w=2)
    assert rows.tolist() == [4, 5, 6, 7, 0, 1]
    assert pos.tolist() == [[0, 0, 0], [0, 0, 1], [1, 0, 0], [1, 0, 1], [2, 0, 0], [2, 0, 1]]
    rows, pos = O.window_keys(slots=3, oldest=0, n_valid=1, grid_h=2, grid_w=2)
    assert rows.tolist() == [0, 1, 2, 3]
    assert pos.tolist() == [[0, 0, 0], [0, 0, 1], [0, 1, 0], [0, 1, 1]]


def test_window_queries_worked_example():
    q = O.window_queries(n_valid=3, n_query=2, grid_h=1, grid_w=2)
    assert q.tolist() == [[2, 0, 0], [2, 0, 1]]
    q = O.window_queries(n_valid=3, n_query=3, grid_h=1, grid_w=2)
    assert q.tolist() == [[1, 0, 1], [2, 0, 0], [2, 0, 1]]
    q = O.window_queries(n_valid=2, n_query=7, grid_h=2, grid_w=3)   # 2 x 3 grid, row-major
    assert q[-1].tolist() == [1, 1, 2] and q[0].tolist() == [0, 1, 2]


def test_cache_write_ring_placement_worked_example():
    # two frames of T_f = 2 starting at the last slot wrap to slot 0
    x = np.arange(4 * 3, dtype=np.float64).reshape(1, 4, 3) + 1.0
    W_dkv = np.eye(3)[:2]            # c = first two components of x
    W_kr = np.eye(3)[2:]             # k^R = last component of x
    cache = np.full((1, 3 * 2, 3), -7.0)
    O.cache_write(x, W_dkv, W_kr, None, 0.0, cache, slots=3, first_slot=2,
                  tokens_per_frame=2, normalize=False)
    assert cache[0, 4:6].tolist() == [[1, 2, 3], [4, 5, 6]]         # slot 2 <- frame 0
    assert cache[0, 0:2].tolist() == [[7, 8, 9], [10, 11, 12]]      # slot 0 <- frame 1
    assert np.all(cache[0, 2:4] == -7.0)                             # slot 1 untouched


def test_cache_write_rmsnorm_closed_forms():
    rng = np.random.default_rng(3)
    d, d_c, d_r = 24, 6, 4
    W_dkv = rng.normal(size=(d_c, d)); W_kr = rng.normal(size=(d_r, d))
    gamma = 1.0 + 0.1 * rng.normal(size=d_c)
    eps = 1e-6
    # one-hot token: the latent is the normalised column of W_dkv, times gamma
    x = np.zeros((1, 1, d)); x[0, 0, 5] = 1.0
    cache = np.zeros((1, 1, d_c + d_r))
    O.cache_write(x, W_dkv, W_kr, gamma, eps, cache, 1, 0, 1)
    col = W_dkv[:, 5]
    expect = gamma * col / math.sqrt(sum(v * v for v in col) / d_c + eps)
    assert np.allclose(cache[0, 0, :d_c], expect, rtol=1e-14)
    assert np.allclose(cache[0, 0, d_c:], W_kr[:, 5], rtol=1e-15)     # k^R: raw, unnormalised
    # unit gain: the latent has mean square ms / (ms + eps); scale invariant; k^R linear
    x = rng.normal(size=(1, 3, d))
    c1 = O.cache_write(x, W_dkv, W_kr, np.ones(d_c), eps, np.zeros((1, 3, d_c + d_r)), 3, 0, 1)
    c8 = O.cache_write(8 * x, W_dkv, W_kr, np.ones(d_c), eps, np.zeros((1, 3, d_c + d_r)), 3, 0, 1)
    raw = x[0] @ W_dkv.T
    ms = np.mean(raw ** 2, axis=-1)
    assert np.allclose(np.mean(c1[0, :, :d_c] ** 2, axis=-1), ms / (ms + eps), rtol=1e-13)
    assert np.allclose(c8[0, :, :d_c], c1[0, :, :d_c], rtol=1e-6)
    assert np.allclose(c8[0, :, d_c:], 8 * c1[0, :, d_c:], rtol=1e-13)


# ---------------------------------------------------------------------------
# attention: tiny problem helpers
# ---------------------------------------------------------------------------

TINY = dict(d=16, H=2, d_c=8, d_rope=8, d_nope=8, d_v=6, grid_h=2, grid_w=3, slots=3)


def _tiny_problem(seed=4, Nq=8, oldest=1, n_valid=3, rope_scale=1.0):
    rng = np.random.default_rng(seed)
    T = TINY
    T_f = T["grid_h"] * T["grid_w"]
    cache = rng.normal(size=(2, T["slots"] * T_f, T["d_c"] + T["d_rope"]))
    cache[..., T["d_c"]:] *= rope_scale
    return dict(
        q_nope=rng.normal(size=(2, Nq, T["H"], T["d_nope"])),
        q_rope=rng.normal(size=(2, Nq, T["H"], T["d_rope"])),
        W_uk=rng.normal(size=(T["H"] * T["d_nope"], T["d_c"])) / math.sqrt(T["d_c"]),
        W_uv=rng.normal(size=(T["H"] * T["d_v"], T["d_c"])) / math.sqrt(T["d_c"]),
        cache=cache, slots=T["slots"], oldest=oldest, n_valid=n_valid,
        grid_h=T["grid_h"], grid_w=T["grid_w"], d_c=T["d_c"])


def _brute_force(q_nope, q_rope, W_uk, W_uv, cache, slots, oldest, n_valid, grid_h, grid_w, d_c):
    """Independent formulation: scalar loops, explicit per-head K/V/Q, full
    d_rope x d_rope block-diagonal rotation matrices built entry by entry, and
    a two-pass softmax with math.exp."""
    B, Nq, H, d_nope = q_nope.shape
    d_rope = q_rope.shape[-1]
    d_v = W_uv.shape[0] // H
    T_f = grid_h * grid_w
    omega, axis = O.rope_frequencies(d_rope, d_nope + d_rope)

    def rot_matrix(t, h, w):
        R = [[0.0] * d_rope for _ in range(d_rope)]
        for p in range(d_rope // 2):
            ang = (t, h, w)[axis[p]] * omega[p]
            c, s = math.cos(ang), math.sin(ang)
            R[2 * p][2 * p] = c; R[2 * p][2 * p + 1] = -s
            R[2 * p + 1][2 * p] = s; R[2 * p + 1][2 * p + 1] = c
        return R

    def matvec(M, v):
        return [sum(M[r][c] * v[c] for c in range(len(v))) for r in range(len(M))]

    keys = []                                     # (row, t, h, w) in logical order
    for j in range(n_valid):
        slot = (oldest + j) % slots
        for p in range(T_f):
            keys.append((slot * T_f + p, j, p // grid_w, p % grid_w))
    total = n_valid * T_f
    out = np.zeros((B, Nq, H, d_v)); lse = np.zeros((B, Nq, H))
    for b in range(B):
        for h in range(H):
            Wk = [[W_uk[h * d_nope + r][c] for c in range(d_c)] for r in range(d_nope)]
            Wv = [[W_uv[h * d_v + r][c] for c in range(d_c)] for r in range(d_v)]
            K, V = [], []
            for (row, t, hh, ww) in keys:
                c = list(cache[b, row, :d_c])
                kr = matvec(rot_matrix(t, hh, ww), list(cache[b, row, d_c:]))
                K.append(matvec(Wk, c) + kr)
                V.append(matvec(Wv, c))
            for i in range(Nq):
                L = total - Nq + i
                t, p = L // T_f, L % T_f
                qr = matvec(rot_matrix(t, p // grid_w, p % grid_w), list(q_rope[b, i, h]))
                q = list(q_nope[b, i, h]) + qr
                s = [sum(a * k for a, k in zip(q, kk)) / math.sqrt(d_nope + d_rope) for kk in K]
                m = max(s)
                e = [math.exp(v - m) for v in s]
                l = sum(e)
                for dv in range(d_v):
                    out[b, i, h, dv] = sum(e[j] * V[j][dv] for j in range(len(K))) / l
                lse[b, i, h] = m + math.log(l)
    return out, lse


# ---------------------------------------------------------------------------
# (2)-(5) attention pins
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("oldest,n_valid,Nq", [(1, 3, 8), (2, 2, 6), (0, 1, 5), (2, 3, 18)])
def test_attention_matches_brute_force(oldest, n_valid, Nq):
    prob = _tiny_problem(Nq=Nq, oldest=oldest, n_valid=n_valid)
    ref_out, ref_lse = _brute_force(**prob)
    out, lse = O.attention_explicit(**prob)
    assert np.max(np.abs(out - ref_out)) < 1e-11
    assert np.max(np.abs(lse - ref_lse)) < 1e-11
    out2, lse2 = O.attention_absorbed(**prob)
    assert np.max(np.abs(out2 - ref_out)) < 1e-11
    assert np.max(np.abs(lse2 - ref_lse)) < 1e-11


def test_absorbed_equals_explicit_wan_shapes():
    # [VideoMLA] App. E: the absorbed form preserves the attention computation.
    rng = np.random.default_rng(5)
    H, d_c, d_rope, d_nope, d_v, gh, gw, slots = 12, 192, 32, 96, 128, 6, 8, 3
    T_f = gh * gw
    args = dict(
        q_nope=rng.normal(size=(1, 48, H, d_nope)), q_rope=rng.normal(size=(1, 48, H, d_rope)),
        W_uk=rng.normal(size=(H * d_nope, d_c)) / math.sqrt(d_c),
        W_uv=rng.normal(size=(H * d_v, d_c)) / math.sqrt(d_c),
        cache=rng.normal(size=(1, slots * T_f, d_c + d_rope)),
        slots=slots, oldest=0, n_valid=3, grid_h=gh, grid_w=gw, d_c=d_c)
    o1, l1 = O.attention_explicit(**args)
    o2, l2 = O.attention_absorbed(**args)
    assert np.linalg.norm(o1 - o2) <= 1e-12 * np.linalg.norm(o1)
    assert np.max(np.abs(l1 - l2)) <= 1e-12 * np.max(np.abs(l1))


def test_softmax_rows_sum_to_one():
    prob = _tiny_problem()
    _, _, P = O.attention_explicit(**prob, return_probs=True)
    assert np.all(P >= 0)
    assert np.max(np.abs(P.sum(axis=-1) - 1.0)) < 1e-14


def test_zero_query_gives_uniform_average():
    prob = _tiny_problem()
    prob["q_nope"][:] = 0.0
    prob["q_rope"][:] = 0.0
    out, lse = O.attention_absorbed(**prob)
    rows, _ = O.window_keys(prob["slots"], prob["oldest"], prob["n_valid"], 2, 3)
    mean_c = prob["cache"][:, rows, :prob["d_c"]].mean(axis=1)          # [B, d_c]
    H, d_v = TINY["H"], TINY["d_v"]
    for h in range(H):
        expect = mean_c @ prob["W_uv"][h * d_v:(h + 1) * d_v].T
        assert np.allclose(out[:, :, h], expect[:, None, :], atol=1e-13)
    assert np.allclose(lse, math.log(len(rows)), atol=1e-13)


def test_identical_keys_return_their_value():
    prob = _tiny_problem()
    prob["cache"][:] = prob["cache"][:, :1]                            # every row = row 0
    # identical content, but rotated rope keys differ by position: zero them out
    prob["cache"][..., prob["d_c"]:] = 0.0
    out, _ = O.attention_explicit(**prob)
    H, d_v = TINY["H"], TINY["d_v"]
    for h in range(H):
        v = prob["cache"][:, 0, :prob["d_c"]] @ prob["W_uv"][h * d_v:(h + 1) * d_v].T
        assert np.allclose(out[:, :, h], v[:, None, :], atol=1e-13)


def test_dominant_key_wins():
    prob = _tiny_problem(Nq=1)
    prob["q_nope"][:] = 0.0
    prob["q_rope"][:] = 0.0
    prob["q_rope"][..., 0] = 1.0                  # only the first t-pair, x component
    rows, pos = O.window_keys(prob["slots"], prob["oldest"], prob["n_valid"], 2, 3)
    target = rows[4]
    prob["cache"][..., prob["d_c"]:] = 0.0
    # the query sits at t = 2; choose the key's raw value so its rotated version
    # aligns with the rotated query: rotate by (t_q - t_k) * omega_0 = (2 - 0) * 1
    ang = 2.0 - pos[4][0]
    prob["cache"][:, target, prob["d_c"]] = 400.0 * math.cos(ang)
    prob["cache"][:, target, prob["d_c"] + 1] = 400.0 * math.sin(ang)
    out, _ = O.attention_absorbed(**prob)
    H, d_v = TINY["H"], TINY["d_v"]
    for h in range(H):
        v = prob["cache"][:, target, :prob["d_c"]] @ prob["W_uv"][h * d_v:(h + 1) * d_v].T
        assert np.allclose(out[:, 0, h], v, atol=1e-9)


# ---------------------------------------------------------------------------
# (6) the pins catch plausible mistakes (planted in the oracle, on the CPU)
# ---------------------------------------------------------------------------

def _mutant_disagrees(monkeypatch, name, fn):
    prob = _tiny_problem()
    ref_out, _ = _brute_force(**prob)
    with monkeypatch.context() as m:
        m.setattr(O, name, fn)
        out, _ = O.attention_absorbed(**prob)
    return np.max(np.abs(out - ref_out)) > 1e-6


def test_pins_catch_wrong_rotation_sign(monkeypatch):
    orig = O.rope_rotate
    assert _mutant_disagrees(monkeypatch, "rope_rotate", lambda v, th: orig(v, -th))


def test_pins_catch_dropped_rope_term(monkeypatch):
    assert _mutant_disagrees(monkeypatch, "rope_rotate", lambda v, th: 0.0 * v)


def test_pins_catch_wrong_query_frame(monkeypatch):
    orig = O.window_queries
    def shifted(n_valid, n_query, gh, gw, n_sink=0):
        q = orig(n_valid, n_query, gh, gw, n_sink).copy(); q[:, 0] -= 1; return q
    assert _mutant_disagrees(monkeypatch, "window_queries", shifted)


def test_pins_catch_swapped_grid_axes(monkeypatch):
    orig = O.token_grid_position
    assert _mutant_disagrees(monkeypatch, "token_grid_position",
                             lambda p, gw: orig(p, gw)[::-1])


def test_pins_catch_wrong_ring_order(monkeypatch):
    orig = O.window_keys
    def reversed_t(slots, oldest, n_valid, gh, gw, n_sink=0):
        rows, pos = orig(slots, oldest, n_valid, gh, gw, n_sink)
        pos = pos.copy(); pos[:, 0] = n_valid - 1 - pos[:, 0]
        return rows, pos
    assert _mutant_disagrees(monkeypatch, "window_keys", reversed_t)


# ---------------------------------------------------------------------------
# sink + FIFO window ([VideoMLA] App. D.4-D.5): one pinned sink frame before the
# ring, re-indexed to local t = 0 with the FIFO frames at t = 1 .. n_valid
# ---------------------------------------------------------------------------

def _sink_problem(seed=11, Nq=8, oldest=2, n_valid=3):
    prob = _tiny_problem(seed=seed, Nq=Nq, oldest=oldest, n_valid=n_valid)
    T = TINY
    T_f = T["grid_h"] * T["grid_w"]
    rng = np.random.default_rng(seed + 1)
    sink = rng.normal(size=(2, T_f, T["d_c"] + T["d_rope"]))
    prob["cache"] = np.concatenate([sink, prob["cache"]], axis=1)   # sink rows first
    return prob


def test_sink_window_equals_brute_force_on_relaid_window():
    """The sink window is the plain window whose logical frame 0 is the sink
    frame and frames 1.. the FIFO frames oldest first: re-lay the cache that
    way by hand and compare with the brute-force formulation."""
    prob = _sink_problem()
    T = TINY
    T_f = T["grid_h"] * T["grid_w"]
    slots, oldest, n_valid = prob["slots"], prob["oldest"], prob["n_valid"]
    frames = [prob["cache"][:, 0:T_f]]                               # the sink
    for j in range(n_valid):
        slot = (oldest + j) % slots
        frames.append(prob["cache"][:, T_f + slot * T_f:T_f + (slot + 1) * T_f])
    relaid = dict(prob, cache=np.concatenate(frames, axis=1), slots=n_valid + 1, oldest=0, n_valid=n_valid + 1)
    ref_out, ref_lse = _brute_force(**relaid)
    out, lse = O.attention_absorbed(**prob, n_sink=1)
    assert np.max(np.abs(out - ref_out)) < 1e-10
    assert np.max(np.abs(lse - ref_lse)) < 1e-10
    out_e, _ = O.attention_explicit(**prob, n_sink=1)
    assert np.max(np.abs(out_e - ref_out)) < 1e-10


def test_sink_window_positions():
    T_f = 6
    rows, pos = O.window_keys(slots=4, oldest=3, n_valid=2, grid_h=2, grid_w=3, n_sink=1)
    assert rows.tolist() == list(range(6)) + [6 + 3 * 6 + p for p in range(6)] + [6 + 0 * 6 + p for p in range(6)]
    assert pos[:T_f, 0].tolist() == [0] * T_f
    assert pos[T_f:2 * T_f, 0].tolist() == [1] * T_f and pos[2 * T_f:, 0].tolist() == [2] * T_f
    q = O.window_queries(n_valid=2, n_query=4, grid_h=2, grid_w=3, n_sink=1)
    assert q[:, 0].tolist() == [2] * 4 and q[:, 1].tolist() == [0, 1, 1, 1]


def test_sink_pin_catches_sink_after_fifo(monkeypatch):
    """Placing the sink after the FIFO frames (t = n_valid) must be caught."""
    prob = _sink_problem()
    base_out, _ = O.attention_absorbed(**prob, n_sink=1)
    orig = O.window_keys
    def sink_last(slots, oldest, n_valid, gh, gw, n_sink=0):
        rows, pos = orig(slots, oldest, n_valid, gh, gw, n_sink)
        pos = pos.copy()
        T_f = gh * gw
        pos[:n_sink * T_f, 0] = n_valid + n_sink          # sink moved to the end
        pos[n_sink * T_f:, 0] -= n_sink
        return rows, pos
    with monkeypatch.context() as m:
        m.setattr(O, "window_keys", sink_last)
        out, _ = O.attention_absorbed(**prob, n_sink=1)
    assert np.max(np.abs(out - base_out)) > 1e-6


# ---------------------------------------------------------------------------
# query path and output projection ([VideoMLA] Eq. 3-4, 6, App. D.2, Eq. 10-11)
# ---------------------------------------------------------------------------

def test_query_projection_brute_force_and_scale_invariance():
    rng = np.random.default_rng(31)
    H, d, d_q, d_nope, d_rope = 3, 10, 6, 4, 2
    x = rng.normal(size=(2, 5, d))
    W_dq = rng.normal(size=(d_q, d)); g = 1 + 0.1 * rng.normal(size=d_q)
    W_uq = rng.normal(size=(H * d_nope, d_q)); W_qr = rng.normal(size=(H * d_rope, d_q))
    eps = 1e-6
    qn, qr = O.query_projection(x, W_dq, g, eps, W_uq, W_qr, H)
    for b in range(2):
        for t in range(5):
            c = [sum(W_dq[i][k] * x[b, t, k] for k in range(d)) for i in range(d_q)]
            ms = sum(v * v for v in c) / d_q
            c = [g[i] * c[i] / math.sqrt(ms + eps) for i in range(d_q)]
            for h in range(H):
                for e in range(d_nope):
                    ref = sum(W_uq[h * d_nope + e][i] * c[i] for i in range(d_q))
                    assert abs(qn[b, t, h, e] - ref) < 1e-10
                for e in range(d_rope):
                    ref = sum(W_qr[h * d_rope + e][i] * c[i] for i in range(d_q))
                    assert abs(qr[b, t, h, e] - ref) < 1e-10
    # RMSNorm before the up-projections: scaling a token leaves its queries unchanged
    qn2, qr2 = O.query_projection(7.5 * x, W_dq, g, 0.0, W_uq, W_qr, H)
    qn0, qr0 = O.query_projection(x, W_dq, g, 0.0, W_uq, W_qr, H)
    assert np.max(np.abs(qn2 - qn0)) < 1e-10 and np.max(np.abs(qr2 - qr0)) < 1e-10


def test_output_projection_equals_absorbed_value_path():
    """Eq. 10-11: applying W_O,h to the head output W_uv,h (sum_j p_j c_j) equals
    applying B_h = W_O,h W_uv,h to the weighted latent sum; and a brute force."""
    rng = np.random.default_rng(32)
    H, d_v, d_c, d = 3, 4, 5, 7
    lat = rng.normal(size=(2, H, d_c))                  # sum_j p_j c_j per head
    W_uv = rng.normal(size=(H * d_v, d_c)); W_O = rng.normal(size=(d, H * d_v))
    o = np.stack([lat[:, h] @ W_uv[h * d_v:(h + 1) * d_v].T for h in range(H)], axis=1)   # [2, H, d_v]
    y = O.output_projection(o, W_O)
    y_abs = sum(lat[:, h] @ (W_O[:, h * d_v:(h + 1) * d_v] @ W_uv[h * d_v:(h + 1) * d_v]).T for h in range(H))
    assert np.max(np.abs(y - y_abs)) < 1e-10
    for n in range(2):
        for r in range(d):
            ref = sum(W_O[r][h * d_v + e] * o[n, h, e] for h in range(H) for e in range(d_v))
            assert abs(y[n, r] - ref) < 1e-10
