"""Planted mistakes in the sketching-stage oracle must be caught by its pins.

Each case swaps one function of ``oracle.sketching_oracle`` for a copy with a
plausible slip (a transposed product, a dropped damping term, the wrong
factor, an unweighted mean, ties to the upper centroid, a lost cluster, no or
wrongly signed compensation) and runs the pins meant to catch it.  CPU only.
"""
import numpy as np
import pytest

import oracle
from oracle import sketching_oracle as so
from tests import test_oracle_sketch_pins as pins


def _gram_transposed(x):
    x64 = np.asarray(x, dtype=np.float64)
    return x64 @ x64.T


def _damped_no_dead_fix(h, damp):
    h = np.array(h, dtype=np.float64, copy=True)
    dg = np.diag(h).copy()
    np.fill_diagonal(h, dg + damp * float(np.mean(dg)))
    return h


def _damped_absolute(h, damp):
    h = np.array(h, dtype=np.float64, copy=True)
    dg = np.diag(h).copy()
    dg[dg == 0.0] = 1.0
    np.fill_diagonal(h, dg + damp)
    return h


def _factor_lower(h):
    u, hd = so._orig_inverse_factor(h)
    return u.T, hd


def _factor_of_h(h):
    low = np.linalg.cholesky(np.asarray(h, dtype=np.float64))
    return np.triu(low.T), np.diag(np.linalg.inv(h)).copy()


def _update_unweighted(vals_f32, weights, assign, cent_f32):
    return so._orig_lloyd_update(vals_f32, np.ones_like(weights), assign, cent_f32)


def _update_drops_empty(vals_f32, weights, assign, cent_f32):
    out = so._orig_lloyd_update(vals_f32, weights, assign, cent_f32)
    for c in range(out.shape[0]):
        if not np.any(assign == c):
            out[c] = 0.0
    return out


def _assign_ties_up(vals_f32, cent_f32):
    mid = so._midpoints(cent_f32)
    v = np.asarray(vals_f32, dtype=np.float32)
    return (v[:, None] >= mid[None, :]).sum(axis=1)


def _round_variant(sign=1.0, power=1, include_self=False, compensate=True):
    def run(theta, u, lut_f16, return_work=False):
        w = np.asarray(theta, dtype=np.float32).astype(np.float64).copy()
        n, d = w.shape
        gs = d // lut_f16.shape[1]
        rows = np.arange(n)
        idx = np.zeros((n, d), dtype=np.uint8)
        for j in range(d):
            cent = np.asarray(lut_f16[:, j // gs, :], dtype=np.float32)
            mid = so._midpoints(cent).astype(np.float64)
            c = (w[:, j][:, None] > mid).sum(axis=1)
            q = cent[rows, c].astype(np.float64)
            idx[:, j] = c
            if compensate:
                e = (w[:, j] - q) / u[j, j] ** power
                lo = j if include_self else j + 1
                w[:, lo:] -= sign * np.outer(e, u[j, lo:])
        return (idx, w) if return_work else idx
    run.__name__ = f"round_sign{sign}_pow{power}_self{include_self}_comp{compensate}"
    return run


CASES = [
    ("gram", _gram_transposed, lambda: pins.test_gram_is_a_sum_of_outer_products()),
    ("damped", _damped_no_dead_fix, lambda: pins.test_damping_closed_form_with_a_dead_column()),
    ("damped", _damped_absolute, lambda: pins.test_damping_closed_form_with_a_dead_column()),
    ("inverse_factor", _factor_lower, lambda: pins.test_inverse_factor_definition()),
    ("inverse_factor", _factor_of_h, lambda: pins.test_inverse_factor_definition()),
    ("inverse_factor", _factor_of_h, lambda: pins.test_factor_rows_are_the_trailing_block_inverses()),
    ("lloyd_update", _update_unweighted, lambda: pins.test_lloyd_one_centroid_is_the_weighted_mean()),
    ("lloyd_update", _update_unweighted, lambda: pins.test_lloyd_matches_scikit_learn_weighted_kmeans(8)),
    ("lloyd_update", _update_drops_empty, lambda: pins.test_lloyd_constant_group()),
    ("lloyd_assign", _assign_ties_up, lambda: pins.test_lloyd_constant_group()),
    ("sketch_round", _round_variant(compensate=False), lambda: pins.test_round_matches_least_squares_compensation_route()),
    ("sketch_round", _round_variant(sign=-1.0), lambda: pins.test_round_matches_least_squares_compensation_route()),
    ("sketch_round", _round_variant(power=2), lambda: pins.test_round_matches_least_squares_compensation_route()),
    ("sketch_round", _round_variant(include_self=True), lambda: pins.test_round_matches_least_squares_compensation_route()),
    ("sketch_round", _round_variant(compensate=False), lambda: pins.test_round_reduces_the_output_error_against_nearest_rounding()),
]


@pytest.mark.parametrize("name,mutant,check", CASES, ids=[f"{c[0]}-{c[1].__name__}" for c in CASES])
def test_planted_mistake_is_caught(monkeypatch, name, mutant, check):
    monkeypatch.setattr(so, "_orig_" + name, getattr(so, name), raising=False)
    monkeypatch.setattr(so, name, mutant)
    monkeypatch.setattr(oracle, name, mutant)
    with pytest.raises((AssertionError, ValueError, IndexError, np.linalg.LinAlgError)):
        check()
