"""The oracle's pins must catch plausible mistakes.

Each case below plants one mistake in a copy of the C oracle (a textual edit of
oracle/basa_oracle.c compiled into a temporary library), routes the oracle
calls to that copy, and runs the pins of test_oracle.py: at least one pin must
fail.  The real oracle is never modified.
"""
import os
import subprocess

import pytest

import oracle
from oracle import build as obuild
from oracle.oracle import use_library

import test_oracle as pins

MUTANTS = {
    "shift sign on the column axis": ("floor_mod(x - p->sw, padded(p->Wg, p->ww, p->pad))",
                                      "floor_mod(x + p->sw, padded(p->Wg, p->ww, p->pad))"),
    "dropped softmax scale": ("z[j++] = p->scale * s;", "z[j++] = s;"),
    "pooled sum not divided": ("xp[o] = acc * inv;", "xp[o] = acc;"),
    "log-sum-exp without the max": ("*lse_out = mx + log(den);", "*lse_out = log(den);"),
    "window members without the shift": (
        "const int64_t xx = floor_mod(ix * p->ww + p->sw + lx, Wp);",
        "const int64_t xx = floor_mod(ix * p->ww + lx, Wp);"),
    "no max subtraction": ("z[i] = exp(z[i] - mx);", "z[i] = exp(z[i]);"),
    "rows and columns swapped for keys": (
        "const double* kv = k + kv_index(p, b, tok[3 * a], tok[3 * a + 1], tok[3 * a + 2], kv_head(p, h));",
        "const double* kv = k + kv_index(p, b, tok[3 * a], tok[3 * a + 2] % p->Hg, "
        "tok[3 * a + 1] % p->Wg, kv_head(p, h));"),
    "padded axis wrapped at the real grid size": (
        "const int64_t yy = floor_mod(iy * p->wh + p->sh + ly, Hp);",
        "const int64_t yy = floor_mod(iy * p->wh + p->sh + ly, p->Hg);"),
    "query window id on the real grid size": (
        "const int64_t iy = floor_mod(y - p->sh, padded(p->Hg, p->wh, p->pad)) / p->wh;",
        "const int64_t iy = floor_mod(y - p->sh, p->Hg) / p->wh;"),
    "pooled cells on the shifted origin": (
        "acc += x[kv_index(p, b, ct * p->pt + i, cy * p->ph + j,\n"
        "                                       cx * p->pw + l, h) + c];",
        "acc += x[kv_index(p, b, ct * p->pt + i, (cy * p->ph + j + 1) % p->Hg,\n"
        "                                       (cx * p->pw + l + 1) % p->Wg, h) + c];"),
    "softmax backward without the row term": (
        "dS[a * nk + c2] = P[a * nk + c2] * (dS[a * nk + c2] - Da);",
        "dS[a * nk + c2] = P[a * nk + c2] * dS[a * nk + c2];"),
    "pooled key gradient not divided by the cell size": (
        "dk[o + c] += inv * dkp[po + c];", "dk[o + c] += dkp[po + c];"),
    "joint backward: text query rows without the softmax scale": (
        "joint_row_bwd(qt + qo, dout_t + qo, kp, vp, dkp, dvp, N + L, d, p->scale, z, dpv,",
        "joint_row_bwd(qt + qo, dout_t + qo, kp, vp, dkp, dvp, N + L, d, 1.0, z, dpv,"),
    "K/V head by modulo instead of by group": (
        "static int64_t kv_head(const oracle_params* p, int64_t h) { return h / (p->H / kv_heads(p)); }",
        "static int64_t kv_head(const oracle_params* p, int64_t h) { return h % kv_heads(p); }"),
}


def _pins():
    yield pins.test_hand_worked_example, {}
    for shape, window in [((1, 1, 8, 8, 2, 16), (1, 4, 4)), ((2, 4, 6, 8, 1, 8), (2, 3, 4))]:
        yield pins.test_shift_zero_is_partitioned_attention, {"shape": shape, "window": window}
    yield pins.test_window_covering_grid_is_full_attention, {"shape": (2, 3, 4, 5, 3, 8)}
    for shape, window, pool in pins.TINY:
        yield pins.test_oracle_matches_brute_force_all_shifts, {"shape": shape, "window": window,
                                                                "pool": pool}
    yield pins.test_roll_commutes_with_shift, {"shape": (1, 1, 12, 12, 1, 8), "window": (1, 4, 6),
                                               "shift": (0, 1, 5)}
    yield pins.test_zero_queries_give_window_mean, {}
    yield pins.test_constant_values_give_constant_output, {}
    yield pins.test_pool_factor_one_and_constant_cells, {}
    yield pins.test_support_is_exactly_the_window, {}
    yield pins.test_large_logits_pick_dominant_key, {}
    yield pins.test_grouped_query_equals_repeated_kv_heads, {
        "shape": (1, 1, 4, 8, 4, 8), "window": (1, 2, 4), "shift": (0, 1, 2), "pool": (0, 0, 0),
        "Hkv": 2}
    yield pins.test_backward_matches_autograd_of_masked_attention, {
        "shape": (1, 1, 4, 6, 2, 8), "window": (1, 2, 3), "shift": (0, 1, 2), "Hkv": 0}
    yield pins.test_joint_backward_matches_autograd, {
        "shape": (1, 1, 4, 6, 2, 8), "window": (1, 2, 3), "shift": (0, 1, 2), "L": 3, "Hkv": 0}
    yield pins.test_pooled_backward_matches_autograd, {
        "shape": (1, 1, 4, 6, 2, 8), "window": (1, 2, 3), "shift": (0, 1, 2), "pool": (1, 2, 3),
        "Hkv": 0}
    for shape, window, shift, L in pins.JOINT:
        yield pins.test_joint_matches_dense_mask_brute_force, {"shape": shape, "window": window,
                                                              "shift": shift, "L": L}
    for shape, window, pool in pins.PADDED:
        yield pins.test_padded_matches_brute_force_all_shifts, {"shape": shape, "window": window,
                                                                "pool": pool}
    yield pins.test_padded_backward_matches_autograd, {
        "shape": (1, 1, 5, 7, 2, 8), "window": (1, 2, 3), "shift": (0, 1, 2), "pool": (0, 0, 0),
        "L": 0}


def _build_mutant(tmp_path, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    mutated = src.replace(old, new, 1)
    c = tmp_path / "mutant.c"
    c.write_text(mutated)
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", *obuild.FLAGS, "-o", str(so), str(c), "-lm"])
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, oracle_mod, name):
    old, new = MUTANTS[name]
    so = _build_mutant(tmp_path, old, new)
    failed = []
    with use_library(so):
        for fn, kw in _pins():
            try:
                fn(oracle_mod, **kw)
            except (AssertionError, ValueError, FloatingPointError):
                failed.append(fn.__name__)
    assert failed, f"no pin caught the mutant: {name}"
