"""Pins of the CPU fp64 oracle against facts fixed outside the oracle itself.

Each test is chosen so that a plausible slip in the oracle (a wrong shift sign,
a dropped scale, a transposed operand, pooled cells on the wrong origin, a bad
log-sum-exp) fails at least one of them:

* a hand-worked example (tests/golden/hand_1x6.json) with closed-form values;
* shift 0 equals partitioned window attention written with numpy reshapes;
* one window covering the grid equals torch's CPU scaled_dot_product_attention;
* a dense-mask brute force on tiny grids, every shift;
* rolling the input by the shift commutes with the output, and shifts are
  periodic in the window size;
* closed forms (q = 0, constant v, pool factor 1, constant cells);
* the support of each output row is exactly its window (one-hot values and
  perturbations), and two blocks with shifts (0, w/2) reach neighbouring windows;
* large logits stay finite and pick the dominant key.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _P(shape, window, shift=(0, 0, 0), pool=(0, 0, 0), scale=None):
    import oracle
    B, T, Hg, Wg, H, d = shape
    return oracle.OracleParams(B, T, Hg, Wg, H, d, tuple(window), tuple(shift),
                               tuple(pool), scale)


def _expr(s):
    s = s.strip()
    if s == "0":
        return 0.0
    if s.startswith("ln "):
        return math.log(float(s[3:]))
    return float(eval(s, {"sqrt": math.sqrt}))


# --------------------------------------------------------------------------
# hand-worked example
# --------------------------------------------------------------------------

def test_hand_worked_example(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "hand_1x6.json")))
    grid = g["grid"]
    shape = (grid["B"], grid["T"], grid["Hg"], grid["Wg"], grid["H"], grid["d"])
    q = np.array(g["q"], dtype=np.float64).reshape(shape)
    k = np.array([_expr(s) for s in g["k_expr"]]).reshape(shape)
    v = np.array(g["v"], dtype=np.float64).reshape(shape)
    prm = _P(shape, g["window"], g["shift"], scale=g["scale"])
    out, lse = oracle_mod.window_attn(q, k, v, prm, want_lse=True)
    np.testing.assert_allclose(out.reshape(-1), g["out_no_pool"], rtol=0, atol=1e-13)
    want_lse = [_expr(s) for s in g["lse_no_pool_expr"]]
    np.testing.assert_allclose(lse.reshape(-1), want_lse, rtol=0, atol=1e-13)

    prm = _P(shape, g["window"], g["shift"], g["pool"], scale=g["scale"])
    out = oracle_mod.window_attn(q, k, v, prm).reshape(-1)
    a = _expr(g["out_pool_expr"]["window_123"])
    b = _expr(g["out_pool_expr"]["window_450"])
    np.testing.assert_allclose(out, [b, a, a, a, b, b], rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# special cases reducing to other routines
# --------------------------------------------------------------------------

def _partitioned_reference(q, k, v, window, scale):
    """Unshifted windows via reshape into [windows, m] blocks + dense softmax."""
    B, T, Hg, Wg, H, d = q.shape
    wt, wh, ww = window

    def blocks(x):
        r = x.reshape(B, T // wt, wt, Hg // wh, wh, Wg // ww, ww, H, d)
        r = r.transpose(0, 1, 3, 5, 7, 2, 4, 6, 8)  # b, it, iy, ix, h, lt, ly, lx, d
        return r.reshape(B, T // wt, Hg // wh, Wg // ww, H, wt * wh * ww, d)

    qb, kb, vb = blocks(q), blocks(k), blocks(v)
    z = scale * np.einsum("...ic,...jc->...ij", qb, kb)
    z = z - z.max(axis=-1, keepdims=True)
    a = np.exp(z)
    a = a / a.sum(axis=-1, keepdims=True)
    ob = np.einsum("...ij,...jc->...ic", a, vb)
    ob = ob.reshape(B, T // wt, Hg // wh, Wg // ww, H, wt, wh, ww, d)
    ob = ob.transpose(0, 1, 5, 2, 6, 3, 7, 4, 8)
    return ob.reshape(B, T, Hg, Wg, H, d)


@pytest.mark.parametrize("shape,window", [
    ((1, 1, 8, 8, 2, 16), (1, 4, 4)),
    ((2, 4, 6, 8, 1, 8), (2, 3, 4)),
    ((1, 1, 16, 16, 2, 64), (1, 8, 8)),
])
def test_shift_zero_is_partitioned_attention(oracle_mod, shape, window):
    r = _rng(11)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    sc = 1.0 / math.sqrt(shape[-1])
    got = oracle_mod.window_attn(q, k, v, _P(shape, window))
    want = _partitioned_reference(q, k, v, window, sc)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("shape", [(1, 1, 8, 8, 2, 16), (2, 3, 4, 5, 3, 8)])
def test_window_covering_grid_is_full_attention(oracle_mod, shape):
    r = _rng(12)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    B, T, Hg, Wg, H, d = shape
    N = T * Hg * Wg
    got, lse = oracle_mod.full_attn(q, k, v, _P(shape, (T, Hg, Wg)), want_lse=True)
    # a shifted window that covers the grid is the same set of keys
    got_s = oracle_mod.window_attn(q, k, v, _P(shape, (T, Hg, Wg), (1, 2, 3)))
    tq = torch.from_numpy(q).reshape(B, N, H, d).transpose(1, 2)
    tk = torch.from_numpy(k).reshape(B, N, H, d).transpose(1, 2)
    tv = torch.from_numpy(v).reshape(B, N, H, d).transpose(1, 2)
    want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    want = want.transpose(1, 2).reshape(shape).numpy()
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got_s, want, rtol=0, atol=1e-12)
    z = torch.einsum("bhic,bhjc->bhij", tq, tk) / math.sqrt(d)
    want_lse = torch.logsumexp(z, dim=-1).numpy()
    np.testing.assert_allclose(lse, want_lse, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# dense-mask brute force on tiny grids, every shift
# --------------------------------------------------------------------------

TINY = [
    ((1, 1, 4, 4, 2, 8), (1, 2, 2), (0, 0, 0)),
    ((1, 1, 8, 8, 1, 16), (1, 4, 4), (1, 2, 2)),
    ((1, 4, 6, 8, 1, 8), (2, 3, 4), (2, 3, 2)),
    ((2, 1, 6, 6, 2, 4), (1, 3, 2), (1, 3, 2)),
]


@pytest.mark.parametrize("shape,window,pool", TINY)
def test_oracle_matches_brute_force_all_shifts(oracle_mod, shape, window, pool):
    r = _rng(13)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    ranges = [range(-w, w + 1) for w in window]
    shifts = list(itertools.product(*ranges))
    if len(shifts) > 40:
        idx = _rng(5).choice(len(shifts), 40, replace=False)
        shifts = [shifts[i] for i in idx]
    for s in shifts:
        prm = _P(shape, window, s, pool)
        got, lse = oracle_mod.window_attn(q, k, v, prm, want_lse=True)
        want, want_lse = oracle_mod.brute_window_attn(q, k, v, window, s, pool,
                                                      want_lse=True)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12, err_msg=str(s))
        np.testing.assert_allclose(lse, want_lse, rtol=0, atol=1e-12, err_msg=str(s))


def test_brute_force_d64(oracle_mod):
    shape, window = (1, 1, 8, 8, 1, 64), (1, 4, 4)
    r = _rng(14)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    for s in [(0, 0, 0), (0, 1, 3), (0, 2, 2)]:
        got = oracle_mod.window_attn(q, k, v, _P(shape, window, s, (1, 2, 2)))
        want = oracle_mod.brute_window_attn(q, k, v, window, s, (1, 2, 2))
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_selected_queries_match_full_output(oracle_mod):
    shape, window, shift = (2, 2, 6, 8, 3, 8), (1, 3, 4), (1, 1, 2)
    r = _rng(15)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    prm = _P(shape, window, shift, (1, 2, 2))
    full, lse = oracle_mod.window_attn(q, k, v, prm, want_lse=True)
    N = 2 * 6 * 8
    sel = np.array([[b, n, h] for b in range(2) for n in (0, 5, 47, N - 1) for h in (0, 2)])
    part, plse = oracle_mod.window_attn(q, k, v, prm, want_lse=True, select=sel)
    B, T, Hg, Wg, H, d = shape
    flat = full.reshape(B, N, H, d)
    for i, (b, n, h) in enumerate(sel):
        np.testing.assert_array_equal(part[i], flat[b, n, h])
        assert plse[i] == lse[b, h, n]


# --------------------------------------------------------------------------
# roll commutation and periodicity
# --------------------------------------------------------------------------

@pytest.mark.parametrize("shape,window,shift", [
    ((1, 1, 8, 8, 2, 8), (1, 4, 4), (0, 2, 2)),
    ((1, 1, 12, 12, 1, 8), (1, 4, 6), (0, 1, 5)),
    ((1, 6, 6, 8, 1, 4), (3, 3, 4), (1, 2, 3)),
])
def test_roll_commutes_with_shift(oracle_mod, shape, window, shift):
    r = _rng(16)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    axes = (1, 2, 3)
    neg = tuple(-s for s in shift)
    got = oracle_mod.window_attn(q, k, v, _P(shape, window, shift))
    rq, rk, rv = (np.roll(x, neg, axis=axes) for x in (q, k, v))
    base = oracle_mod.window_attn(rq, rk, rv, _P(shape, window, (0, 0, 0)))
    want = np.roll(base, shift, axis=axes)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    per = tuple(s + w for s, w in zip(shift, window))
    got2 = oracle_mod.window_attn(q, k, v, _P(shape, window, per))
    np.testing.assert_allclose(got2, got, rtol=0, atol=0)


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

def test_zero_queries_give_window_mean(oracle_mod):
    shape, window, shift, pool = (1, 1, 8, 8, 2, 4), (1, 4, 4), (0, 1, 3), (1, 2, 4)
    r = _rng(17)
    k, v = r.standard_normal(shape), r.standard_normal(shape)
    q = np.zeros(shape)
    prm = _P(shape, window, shift, pool)
    out, lse = oracle_mod.window_attn(q, k, v, prm, want_lse=True)
    vp = v.reshape(1, 1, 4, 2, 2, 4, 2, 4).mean(axis=(3, 5))  # pooled cells of 2 x 4
    P = 4 * 2
    for y in range(8):
        for x in range(8):
            wy = ((y - 1) % 8) // 4
            wx = ((x - 3) % 8) // 4
            ys = [yy for yy in range(8) if ((yy - 1) % 8) // 4 == wy]
            xs = [xx for xx in range(8) if ((xx - 3) % 8) // 4 == wx]
            acc = sum(v[0, 0, yy, xx] for yy in ys for xx in xs) + vp.reshape(P, 2, 4).sum(0)
            np.testing.assert_allclose(out[0, 0, y, x], acc / (16 + P), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, math.log(16 + P), rtol=0, atol=1e-13)


def test_constant_values_give_constant_output(oracle_mod):
    shape = (1, 2, 6, 6, 2, 8)
    r = _rng(18)
    q, k = r.standard_normal(shape) * 3, r.standard_normal(shape) * 3
    c = r.standard_normal((2, 8))
    v = np.broadcast_to(c, shape).copy()
    out = oracle_mod.window_attn(q, k, v, _P(shape, (2, 3, 3), (1, 1, 2), (1, 2, 3)))
    np.testing.assert_allclose(out, np.broadcast_to(c, shape), rtol=0, atol=1e-13)


def test_pool_factor_one_and_constant_cells(oracle_mod):
    shape = (2, 2, 4, 6, 3, 8)
    r = _rng(19)
    x = r.standard_normal(shape)
    np.testing.assert_array_equal(oracle_mod.pool_kv(x, _P(shape, (1, 2, 2), pool=(1, 1, 1))), x)
    cells = r.standard_normal((2, 1, 2, 2, 3, 8))
    xc = np.repeat(np.repeat(np.repeat(cells, 2, axis=1), 2, axis=2), 3, axis=3)
    np.testing.assert_allclose(oracle_mod.pool_kv(xc, _P(shape, (1, 2, 2), pool=(2, 2, 3))),
                               cells, rtol=4e-16 * 12, atol=0)
    # a pooled token equal to a window key behaves like a duplicate of that key
    shape1 = (1, 1, 1, 4, 1, 1)
    q = np.ones(shape1)
    k = np.zeros(shape1)
    v = np.array([1.0, 2.0, 3.0, 4.0]).reshape(shape1)
    out = oracle_mod.window_attn(q, k, v, _P(shape1, (1, 1, 2), (0, 0, 0), (1, 1, 4)))
    # keys: own window (2 tokens) + one pooled token of mean 2.5, all logits 0
    want = np.array([(1 + 2 + 2.5) / 3, (1 + 2 + 2.5) / 3, (3 + 4 + 2.5) / 3, (3 + 4 + 2.5) / 3])
    np.testing.assert_allclose(out.reshape(-1), want, rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# support and receptive field
# --------------------------------------------------------------------------

def test_support_is_exactly_the_window(oracle_mod):
    T, Hg, Wg = 1, 6, 6
    N = T * Hg * Wg
    shape = (1, T, Hg, Wg, 1, N)
    window, shift = (1, 3, 3), (0, 1, 2)
    r = _rng(20)
    q, k = r.standard_normal(shape), r.standard_normal(shape)
    v = np.eye(N).reshape(shape)  # value of token j is the one-hot e_j
    out = oracle_mod.window_attn(q, k, v, _P(shape, window, shift)).reshape(N, N)
    iy = ((np.arange(Hg) - 1) % Hg) // 3
    ix = ((np.arange(Wg) - 2) % Wg) // 3
    wid = (iy[:, None] * 10 + ix[None, :]).reshape(N)
    for p in range(N):
        support = set(np.nonzero(out[p] > 0)[0].tolist())
        assert support == set(np.nonzero(wid == wid[p])[0].tolist())
        assert abs(out[p].sum() - 1.0) < 1e-13


def test_perturbation_reaches_only_window_then_neighbours(oracle_mod):
    shape = (1, 1, 8, 8, 1, 4)
    window = (1, 4, 4)
    r = _rng(21)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    src = (0, 0, 3, 3)  # (b, t, y, x) of the perturbed token

    def run(vv, s):
        return oracle_mod.window_attn(q, k, vv, _P(shape, window, s))

    def changed(f):
        v2 = v.copy()
        v2[src + (0,)] += 1.0
        a, b = f(v), f(v2)
        return np.abs(a - b).max(axis=(0, 1, 4, 5)) > 1e-12  # [Hg, Wg]

    one = changed(lambda vv: run(vv, (0, 0, 0)))
    want = np.zeros((8, 8), dtype=bool)
    want[0:4, 0:4] = True
    np.testing.assert_array_equal(one, want)
    # two blocks: unshifted then shifted by half a window; the output of the
    # first block is the value input of the second
    two = changed(lambda vv: run(run(vv, (0, 0, 0)), (0, 2, 2)))
    # the first block spreads to window [0,4)x[0,4); the second block's windows
    # (shift 2) that meet it are rows/cols {6,7,0,1} and {2,3,4,5}: all 64 tokens
    assert two.sum() > one.sum()
    assert two[5, 5] and two[7, 7] and not one[5, 5]


# --------------------------------------------------------------------------
# stability
# --------------------------------------------------------------------------

def test_large_logits_pick_dominant_key(oracle_mod):
    shape = (1, 1, 4, 4, 1, 2)
    q = np.zeros(shape)
    k = np.zeros(shape)
    v = np.arange(16 * 2, dtype=np.float64).reshape(shape)
    q[..., 0] = 1.0
    k[0, 0, 1, 1, 0, 0] = 1e4  # dominates its 2x2 window {0,1}x{0,1}
    out = oracle_mod.window_attn(q, k, v, _P(shape, (1, 2, 2), scale=1.0))
    assert np.isfinite(out).all()
    for y in range(2):
        for x in range(2):
            np.testing.assert_allclose(out[0, 0, y, x, 0], v[0, 0, 1, 1, 0], rtol=0, atol=1e-12)


def test_scaled_logits_match_brute_force(oracle_mod):
    shape = (1, 1, 8, 8, 2, 16)
    r = _rng(22)
    q = r.standard_normal(shape) * 30.0
    k, v = r.standard_normal(shape), r.standard_normal(shape)
    got = oracle_mod.window_attn(q, k, v, _P(shape, (1, 4, 4), (0, 2, 2)))
    want = oracle_mod.brute_window_attn(q, k, v, (1, 4, 4), (0, 2, 2))
    assert np.isfinite(got).all()
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# joint text + image attention (image queries: window + every text token;
# text queries: every token)
# --------------------------------------------------------------------------

JOINT = [
    ((1, 1, 4, 4, 2, 8), (1, 2, 2), (0, 1, 1), 3),
    ((2, 2, 4, 6, 1, 8), (1, 2, 3), (1, 1, 2), 5),
    ((1, 4, 6, 8, 1, 4), (2, 3, 4), (3, 2, 1), 1),
    ((1, 1, 4, 4, 1, 8), (1, 2, 2), (0, 0, 0), 0),
]


@pytest.mark.parametrize("shape,window,shift,L", JOINT)
def test_joint_matches_dense_mask_brute_force(oracle_mod, shape, window, shift, L):
    r = _rng(71)
    B, T, Hg, Wg, H, d = shape
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    qt, kt, vt = (r.standard_normal((B, L, H, d)) for _ in range(3))
    got = oracle_mod.joint_attn(q, k, v, qt, kt, vt, _P(shape, window, shift), want_lse=True)
    want = oracle_mod.brute_joint_attn(q, k, v, qt, kt, vt, window, shift, want_lse=True)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-12)


def test_joint_without_text_is_window_attention(oracle_mod):
    r = _rng(72)
    shape = (1, 2, 4, 6, 2, 8)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    empty = np.zeros((1, 0, 2, 8))
    out, out_t = oracle_mod.joint_attn(q, k, v, empty, empty, empty,
                                       _P(shape, (1, 2, 3), (1, 1, 1)))
    want = oracle_mod.window_attn(q, k, v, _P(shape, (1, 2, 3), (1, 1, 1)))
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-12)
    assert out_t.shape == (1, 0, 2, 8)


def test_joint_with_grid_window_is_full_attention_over_all_tokens(oracle_mod):
    """One window covering the grid: image and text queries both see every token,
    so both equal torch's SDPA over the concatenated sequence."""
    r = _rng(73)
    shape = (2, 1, 4, 4, 2, 8)
    B, T, Hg, Wg, H, d = shape
    N, L = T * Hg * Wg, 6
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    qt, kt, vt = (r.standard_normal((B, L, H, d)) for _ in range(3))
    out, out_t = oracle_mod.joint_attn(q, k, v, qt, kt, vt, _P(shape, (T, Hg, Wg), (0, 1, 2)))
    cat = lambda a, b: torch.from_numpy(np.concatenate([a.reshape(B, N, H, d), b], axis=1))
    tq, tk, tv = (cat(a, b).transpose(1, 2) for a, b in ((q, qt), (k, kt), (v, vt)))
    want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).transpose(1, 2).numpy()
    np.testing.assert_allclose(out, want[:, :N].reshape(shape), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out_t, want[:, N:], rtol=0, atol=1e-12)


def test_joint_zero_text_queries_average_every_value(oracle_mod):
    r = _rng(74)
    shape = (1, 1, 4, 4, 1, 8)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    kt, vt = (r.standard_normal((1, 3, 1, 8)) for _ in range(2))
    qt = np.zeros((1, 3, 1, 8))
    _, out_t, _, lse_t = oracle_mod.joint_attn(q, k, v, qt, kt, vt, _P(shape, (1, 2, 2)),
                                               want_lse=True)
    mean = (v.reshape(16, 8).sum(axis=0) + vt.reshape(3, 8).sum(axis=0)) / 19.0
    np.testing.assert_allclose(out_t[0, :, 0], np.tile(mean, (3, 1)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_t, np.log(19.0), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# grouped-query attention: K/V heads shared by groups of query heads
# --------------------------------------------------------------------------

@pytest.mark.parametrize("shape,window,shift,pool,Hkv", [
    ((1, 1, 4, 8, 4, 8), (1, 2, 4), (0, 1, 2), (0, 0, 0), 2),
    ((2, 2, 4, 4, 6, 4), (1, 2, 2), (1, 1, 1), (1, 2, 2), 3),
    ((1, 1, 4, 4, 4, 8), (1, 2, 2), (0, 1, 1), (1, 2, 2), 1),
])
def test_grouped_query_equals_repeated_kv_heads(oracle_mod, shape, window, shift, pool, Hkv):
    """Query head h reading K/V head h / (H / Hkv) is multi-head attention on K/V
    whose heads are each repeated H / Hkv times."""
    r = _rng(81)
    B, T, Hg, Wg, H, d = shape
    q = r.standard_normal(shape)
    k, v = (r.standard_normal((B, T, Hg, Wg, Hkv, d)) for _ in range(2))
    prm = _P(shape, window, shift, pool)
    prm.Hkv = Hkv
    got, lse = oracle_mod.window_attn(q, k, v, prm, want_lse=True)
    rep = lambda x: np.repeat(x, H // Hkv, axis=4)
    want, want_lse = oracle_mod.window_attn(q, rep(k), rep(v), _P(shape, window, shift, pool),
                                            want_lse=True)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, want_lse, rtol=0, atol=1e-12)


def test_grouped_query_joint_equals_repeated_kv_heads(oracle_mod):
    r = _rng(82)
    shape, Hkv, L = (1, 1, 4, 4, 4, 8), 2, 5
    B, T, Hg, Wg, H, d = shape
    q = r.standard_normal(shape)
    k, v = (r.standard_normal((B, T, Hg, Wg, Hkv, d)) for _ in range(2))
    qt = r.standard_normal((B, L, H, d))
    kt, vt = (r.standard_normal((B, L, Hkv, d)) for _ in range(2))
    prm = _P(shape, (1, 2, 2), (0, 1, 1))
    prm.Hkv = Hkv
    got = oracle_mod.joint_attn(q, k, v, qt, kt, vt, prm)
    rep = lambda x, ax: np.repeat(x, H // Hkv, axis=ax)
    want = oracle_mod.joint_attn(q, rep(k, 4), rep(v, 4), qt, rep(kt, 2), rep(vt, 2),
                                 _P(shape, (1, 2, 2), (0, 1, 1)))
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# backward: gradients of window attention
# --------------------------------------------------------------------------

def _dense_mask(T, Hg, Wg, window, shift):
    from oracle import window_ids
    it, iy, ix = (window_ids(G, w, s) for G, w, s in zip((T, Hg, Wg), window, shift))
    wid = np.stack(np.meshgrid(it, iy, ix, indexing="ij"), axis=-1).reshape(-1, 3)
    return np.all(wid[:, None, :] == wid[None, :, :], axis=-1)


@pytest.mark.parametrize("shape,window,shift,Hkv", [
    ((1, 1, 4, 6, 2, 8), (1, 2, 3), (0, 1, 2), 0),
    ((2, 4, 6, 4, 2, 4), (2, 3, 2), (1, 2, 1), 0),
    ((1, 1, 4, 4, 4, 8), (1, 2, 2), (0, 1, 1), 2),
])
def test_backward_matches_autograd_of_masked_attention(oracle_mod, shape, window, shift, Hkv):
    """The oracle's gradients equal torch autograd through masked SDPA (fp64),
    with the same-window mask, for plain and grouped-query heads."""
    r = _rng(91)
    B, T, Hg, Wg, H, d = shape
    hk = Hkv or H
    q, g = r.standard_normal(shape), r.standard_normal(shape)
    k, v = (r.standard_normal((B, T, Hg, Wg, hk, d)) for _ in range(2))
    prm = _P(shape, window, shift)
    prm.Hkv = Hkv
    dq, dk, dv = oracle_mod.window_attn_bwd(q, k, v, g, prm)
    N = T * Hg * Wg
    mask = torch.from_numpy(_dense_mask(T, Hg, Wg, window, shift))
    tq = torch.from_numpy(q).reshape(B, N, H, d).transpose(1, 2).requires_grad_()
    tk = torch.from_numpy(k).reshape(B, N, hk, d).transpose(1, 2).requires_grad_()
    tv = torch.from_numpy(v).reshape(B, N, hk, d).transpose(1, 2).requires_grad_()
    rep = lambda x: x.repeat_interleave(H // hk, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(tq, rep(tk), rep(tv), attn_mask=mask)
    o.backward(torch.from_numpy(g).reshape(B, N, H, d).transpose(1, 2))
    for got, t in ((dq, tq), (dk, tk), (dv, tv)):
        want = t.grad.transpose(1, 2).reshape(got.shape).numpy()
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("shape,window,shift,pool,Hkv", [
    ((1, 1, 4, 6, 2, 8), (1, 2, 3), (0, 1, 2), (1, 2, 3), 0),
    ((2, 2, 4, 4, 2, 4), (2, 2, 2), (1, 1, 1), (1, 2, 2), 0),
    ((1, 1, 4, 4, 4, 8), (1, 2, 2), (0, 1, 1), (1, 2, 2), 2),
])
def test_pooled_backward_matches_autograd(oracle_mod, shape, window, shift, pool, Hkv):
    """With pooled global memory: torch autograd (fp64) through the cell means
    (a reshape-mean), the keys and values [grid tokens, pooled tokens] and SDPA
    with the mask [same window | every pooled token]; the pooled tokens' gradient
    reaches k and v through the means."""
    r = _rng(93)
    B, T, Hg, Wg, H, d = shape
    hk = Hkv or H
    pt, ph, pw = pool
    q, g = r.standard_normal(shape), r.standard_normal(shape)
    k, v = (r.standard_normal((B, T, Hg, Wg, hk, d)) for _ in range(2))
    prm = _P(shape, window, shift, pool)
    prm.Hkv = Hkv
    dq, dk, dv = oracle_mod.window_attn_bwd(q, k, v, g, prm)
    N = T * Hg * Wg
    Pn = (T // pt) * (Hg // ph) * (Wg // pw)
    tq = torch.from_numpy(q).requires_grad_()
    tk = torch.from_numpy(k).requires_grad_()
    tv = torch.from_numpy(v).requires_grad_()
    cells = lambda x: x.reshape(B, T // pt, pt, Hg // ph, ph, Wg // pw, pw, hk, d).mean(
        dim=(2, 4, 6)).reshape(B, Pn, hk, d)
    keys = lambda x: torch.cat([x.reshape(B, N, hk, d), cells(x)], 1).transpose(1, 2)
    rep = lambda x: x.repeat_interleave(H // hk, dim=1)
    mask = torch.cat([torch.from_numpy(_dense_mask(T, Hg, Wg, window, shift)),
                      torch.ones(N, Pn, dtype=torch.bool)], 1)
    o = torch.nn.functional.scaled_dot_product_attention(
        tq.reshape(B, N, H, d).transpose(1, 2), rep(keys(tk)), rep(keys(tv)), attn_mask=mask)
    o.backward(torch.from_numpy(g).reshape(B, N, H, d).transpose(1, 2))
    for got, t in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, t.grad.numpy(), rtol=0, atol=1e-12)


def test_pooled_backward_matches_central_differences(oracle_mod):
    """d/dx of sum(dO * out) by central differences with pooled memory, at a few
    coordinates of q, k, v (k and v also move the pooled tokens)."""
    r = _rng(94)
    shape, window, shift, pool = (1, 1, 4, 4, 1, 4), (1, 2, 2), (0, 1, 1), (1, 2, 2)
    q, k, v, g = (r.standard_normal(shape) for _ in range(4))
    prm = _P(shape, window, shift, pool)
    dq, dk, dv = oracle_mod.window_attn_bwd(q, k, v, g, prm)
    f = lambda q_, k_, v_: float((oracle_mod.window_attn(q_, k_, v_, prm) * g).sum())
    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for idx in [(0, 0, 0, 0, 0, 1), (0, 0, 2, 3, 0, 2), (0, 0, 3, 0, 0, 3)]:
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += h
            up = f(*args)
            args[which][idx] -= 2 * h
            dn = f(*args)
            assert abs((up - dn) / (2 * h) - grad[idx]) < 1e-7


@pytest.mark.parametrize("shape,window,shift,L,Hkv", [
    ((1, 1, 4, 6, 2, 8), (1, 2, 3), (0, 1, 2), 3, 0),
    ((2, 2, 4, 4, 2, 4), (2, 2, 2), (1, 1, 1), 5, 0),
    ((1, 1, 4, 4, 4, 8), (1, 2, 2), (0, 1, 1), 2, 2),
    ((1, 1, 4, 4, 2, 4), (1, 2, 2), (0, 1, 1), 0, 0),
])
def test_joint_backward_matches_autograd(oracle_mod, shape, window, shift, L, Hkv):
    """Joint text + image gradients == torch autograd (fp64) through SDPA over the
    concatenated sequence [image, text] with the joint mask (image-image pairs
    windowed, every pair with a text token allowed)."""
    r = _rng(95)
    B, T, Hg, Wg, H, d = shape
    hk = Hkv or H
    N = T * Hg * Wg
    q, g = r.standard_normal(shape), r.standard_normal(shape)
    k, v = (r.standard_normal((B, T, Hg, Wg, hk, d)) for _ in range(2))
    qt, gt = r.standard_normal((B, L, H, d)), r.standard_normal((B, L, H, d))
    kt, vt = (r.standard_normal((B, L, hk, d)) for _ in range(2))
    prm = _P(shape, window, shift)
    prm.Hkv = Hkv
    got = oracle_mod.joint_attn_bwd(q, k, v, qt, kt, vt, g, gt, prm)
    ts = [torch.from_numpy(x).requires_grad_() for x in (q, k, v, qt, kt, vt)]
    cat = lambda a, b, h: torch.cat([a.reshape(B, N, h, d), b], 1).transpose(1, 2)
    rep = lambda x: x.repeat_interleave(H // hk, dim=1)
    mask = torch.ones(N + L, N + L, dtype=torch.bool)
    mask[:N, :N] = torch.from_numpy(_dense_mask(T, Hg, Wg, window, shift))
    o = torch.nn.functional.scaled_dot_product_attention(
        cat(ts[0], ts[3], H), rep(cat(ts[1], ts[4], hk)), rep(cat(ts[2], ts[5], hk)),
        attn_mask=mask)
    o.backward(cat(torch.from_numpy(g), torch.from_numpy(gt), H))
    for gg, t in zip(got, ts):
        np.testing.assert_allclose(gg, t.grad.numpy(), rtol=0, atol=1e-12)


def test_backward_matches_central_differences(oracle_mod):
    """d/dx of sum(dO * out) by central differences, at a few coordinates of q, k, v."""
    r = _rng(92)
    shape, window, shift = (1, 1, 4, 4, 1, 4), (1, 2, 2), (0, 1, 1)
    q, k, v, g = (r.standard_normal(shape) for _ in range(4))
    prm = _P(shape, window, shift)
    dq, dk, dv = oracle_mod.window_attn_bwd(q, k, v, g, prm)
    f = lambda q_, k_, v_: float((oracle_mod.window_attn(q_, k_, v_, prm) * g).sum())
    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for idx in [(0, 0, 0, 0, 0, 1), (0, 0, 2, 3, 0, 2), (0, 0, 3, 0, 0, 3)]:
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += h
            up = f(*args)
            args[which][idx] -= 2 * h
            dn = f(*args)
            assert abs((up - dn) / (2 * h) - grad[idx]) < 1e-7


# ---------------------------------------------------------------------------
# Grids the window does not divide (pad = True).  The pages are silent here; the
# reading pinned below: each axis padded at its far end to the next multiple of
# the window, the shift rolls the padded axis, padding is neither query nor key.
# ---------------------------------------------------------------------------
PADDED = [  # shape, window, pool
    ((1, 1, 5, 7, 2, 8), (1, 2, 3), (0, 0, 0)),
    ((1, 3, 5, 4, 1, 4), (2, 4, 3), (0, 0, 0)),
    ((2, 1, 3, 3, 1, 4), (1, 4, 4), (0, 0, 0)),   # window larger than the grid
    ((1, 1, 6, 10, 1, 8), (1, 4, 4), (1, 2, 5)),  # pooled cells divide the real grid
]


def _Ppad(shape, window, shift=(0, 0, 0), pool=(0, 0, 0), scale=None):
    prm = _P(shape, window, shift, pool, scale)
    prm.pad = True
    return prm


@pytest.mark.parametrize("shape,window,pool", PADDED)
def test_padded_matches_brute_force_all_shifts(oracle_mod, shape, window, pool):
    """Dense same-window mask from window ids on the padded axes, every shift."""
    r = _rng(301)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    shifts = list(itertools.product(*[range(-w, w + 1) for w in window]))
    if len(shifts) > 40:
        idx = _rng(302).choice(len(shifts), 40, replace=False)
        shifts = [shifts[i] for i in idx]
    for s in shifts:
        got, lse = oracle_mod.window_attn(q, k, v, _Ppad(shape, window, s, pool), want_lse=True)
        want, want_lse = oracle_mod.brute_window_attn(q, k, v, window, s, pool, want_lse=True,
                                                      pad=True)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12, err_msg=str(s))
        np.testing.assert_allclose(lse, want_lse, rtol=0, atol=1e-12, err_msg=str(s))


@pytest.mark.parametrize("shape,window", [(s, w) for s, w, _ in PADDED[:3]])
def test_padded_shift_zero_is_blockwise_attention(oracle_mod, shape, window):
    """Shift 0: the windows are the grid's blocks [j w, min((j + 1) w, G)) on each
    axis, the last one cut short; attention within each block by torch SDPA on
    the sliced tensors."""
    r = _rng(303)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    got = oracle_mod.window_attn(q, k, v, _Ppad(shape, window))
    B, T, Hg, Wg, H, d = shape
    want = np.zeros(shape)
    for t0 in range(0, T, window[0]):
        for y0 in range(0, Hg, window[1]):
            for x0 in range(0, Wg, window[2]):
                sl = (slice(None), slice(t0, t0 + window[0]), slice(y0, y0 + window[1]),
                      slice(x0, x0 + window[2]))
                blk = [torch.from_numpy(np.ascontiguousarray(a[sl])) for a in (q, k, v)]
                n = blk[0].shape[1] * blk[0].shape[2] * blk[0].shape[3]
                qb, kb, vb = (x.reshape(B, n, H, d).transpose(1, 2) for x in blk)
                o = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb)
                want[sl] = o.transpose(1, 2).reshape(blk[0].shape).numpy()
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_padded_equals_divisible_grid_with_masked_holes(oracle_mod):
    """Embed the grid in its padded (divisible) grid and run the unpadded oracle
    there: an extra feature puts every padding key's logit 1e4 below the rest,
    so its weight underflows to 0; real queries then match the padded call."""
    r = _rng(304)
    shape, window = (1, 3, 5, 7, 2, 8), (2, 2, 3)
    B, T, Hg, Wg, H, d = shape
    Tp, Hp, Wp = (-(-G // w) * w for G, w in zip((T, Hg, Wg), window))
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    sc = 1.0 / math.sqrt(d)
    qe, ke, ve = (np.zeros((B, Tp, Hp, Wp, H, d + 1)) for _ in range(3))
    qe[:, :T, :Hg, :Wg, :, :d] = q * sc
    qe[..., d] = 1.0
    ke[:, :T, :Hg, :Wg, :, :d] = k
    ke[..., d] = -1e4
    ke[:, :T, :Hg, :Wg, :, d] = 0.0
    ve[:, :T, :Hg, :Wg, :, :d] = v
    for s in [(0, 0, 0), (1, 1, 2), (1, 0, 1), (0, 1, 0)]:
        got, lse = oracle_mod.window_attn(q, k, v, _Ppad(shape, window, s), want_lse=True)
        emb, lse_e = oracle_mod.window_attn(qe, ke, ve, _P((B, Tp, Hp, Wp, H, d + 1), window, s,
                                                          scale=1.0), want_lse=True)
        np.testing.assert_allclose(got, emb[:, :T, :Hg, :Wg, :, :d], rtol=0, atol=1e-12)
        real = np.zeros((Tp, Hp, Wp), dtype=bool)
        real[:T, :Hg, :Wg] = True
        np.testing.assert_allclose(lse, lse_e[:, :, real.reshape(-1)], rtol=0, atol=1e-12)


def test_padded_flag_changes_nothing_when_the_window_divides(oracle_mod):
    r = _rng(305)
    shape, window = (1, 2, 8, 6, 2, 4), (2, 4, 3)
    q, k, v = (r.standard_normal(shape) for _ in range(3))
    for s in [(0, 0, 0), (1, 2, 1)]:
        a = oracle_mod.window_attn(q, k, v, _P(shape, window, s, (1, 2, 3)))
        b = oracle_mod.window_attn(q, k, v, _Ppad(shape, window, s, (1, 2, 3)))
        assert np.array_equal(a, b)


@pytest.mark.parametrize("shape,window,shift,pool,L", [
    ((1, 1, 5, 7, 2, 8), (1, 2, 3), (0, 1, 2), (0, 0, 0), 0),
    ((1, 3, 5, 4, 1, 4), (2, 4, 3), (1, 3, 1), (0, 0, 0), 0),
    ((1, 1, 6, 10, 2, 4), (1, 4, 4), (0, 1, 3), (1, 2, 5), 0),
    ((1, 1, 5, 7, 2, 4), (1, 2, 3), (0, 1, 2), (0, 0, 0), 3),
])
def test_padded_backward_matches_autograd(oracle_mod, shape, window, shift, pool, L):
    """Padded-grid gradients (window, pooled, joint) == torch autograd (fp64)
    through SDPA with the padded same-window mask (pooled cell means and text
    tokens appended as keys every query sees; text queries see every key)."""
    from oracle import window_ids
    r = _rng(306)
    B, T, Hg, Wg, H, d = shape
    N = T * Hg * Wg
    q, k, v, g = (r.standard_normal(shape) for _ in range(4))
    qt, kt, vt, gt = (r.standard_normal((B, L, H, d)) for _ in range(4))
    prm = _Ppad(shape, window, shift, pool)
    if L:
        got = oracle_mod.joint_attn_bwd(q, k, v, qt, kt, vt, g, gt, prm)
    else:
        got = oracle_mod.window_attn_bwd(q, k, v, g, prm)
    ids = [window_ids(G, w, s, pad=True) for G, w, s in zip((T, Hg, Wg), window, shift)]
    wid = np.stack(np.meshgrid(*ids, indexing="ij"), axis=-1).reshape(-1, 3)
    ts = [torch.from_numpy(x).requires_grad_() for x in (q, k, v, qt, kt, vt)]
    flat = lambda x: x.reshape(B, -1, H, d)
    keys, vals = [flat(ts[1])], [flat(ts[2])]
    if pool != (0, 0, 0):
        cell = lambda x: x.reshape(B, T // pool[0], pool[0], Hg // pool[1], pool[1],
                                   Wg // pool[2], pool[2], H, d).mean(dim=(2, 4, 6))
        keys.append(flat(cell(ts[1])))
        vals.append(flat(cell(ts[2])))
    keys.append(ts[4])
    vals.append(ts[5])
    qa = torch.cat([flat(ts[0]), ts[3]], 1).transpose(1, 2)
    ka = torch.cat(keys, 1).transpose(1, 2)
    va = torch.cat(vals, 1).transpose(1, 2)
    nk = ka.shape[2]
    mask = torch.ones(N + L, nk, dtype=torch.bool)
    mask[:N, :N] = torch.from_numpy(np.all(wid[:, None, :] == wid[None, :, :], axis=-1))
    o = torch.nn.functional.scaled_dot_product_attention(qa, ka, va, attn_mask=mask)
    o.backward(torch.cat([flat(torch.from_numpy(g)), torch.from_numpy(gt)], 1).transpose(1, 2))
    for gg, t in zip(got, ts):
        np.testing.assert_allclose(gg, t.grad.numpy(), rtol=0, atol=1e-12)


def test_e4m3_decoding_matches_the_format_definition():
    """The e4m3 inputs reach the oracle through torch's exact float8_e4m3fn ->
    float64 conversion; every one of the 256 codes decodes to the value the OCP
    e4m3 definition gives: sign bit, 4 exponent bits with bias 7, 3 mantissa
    bits, subnormals m * 2^-9 for exponent 0, no infinities, NaN only for
    S.1111.111 (so the largest finite magnitude is 448)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    got = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        if e == 15 and m == 7:
            assert math.isnan(got[c])
            continue
        mag = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        assert got[c] == (-mag if s else mag), c
    assert np.nanmax(np.abs(got)) == 448.0
