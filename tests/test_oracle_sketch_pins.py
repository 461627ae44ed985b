"""Pins of the sketching-stage oracle (SpaLLM section 2.2; the "Sketch to
Adapt" OpenReview discussion, concern 1).

Every function is checked against something other than itself: brute force
(the Gram matrix as a sum of outer products), closed forms (damping, one
centroid, separated clusters, diagonal Hessians), library routines (a dense
inverse of trailing blocks; scikit-learn's weighted k-means from the same
start), the identity example of section 2.4, and an independent route for the
mapping that re-solves the least-squares compensation at every step from H
itself instead of using the factor U.
"""
import numpy as np
import pytest

import oracle
from compressive_fine_tuning_b200 import synth


def _spd(rng, d, s=None):
    x = synth.bf16_bits_to_f64(synth.make_calib(rng, s or 4 * d, d))
    return oracle.damped(oracle.gram(x), 0.01)


# ---------------------------------------------------------------------------
# Gram matrix, damping, inverse factor
# ---------------------------------------------------------------------------

def test_gram_is_a_sum_of_outer_products():
    rng = synth.rng_for(50000)
    x = synth.bf16_bits_to_f64(synth.make_calib(rng, 7, 5))
    want = np.zeros((5, 5))
    for t in range(7):
        for a in range(5):
            for b in range(5):
                want[a, b] += x[t, a] * x[t, b]
    np.testing.assert_allclose(oracle.gram(x), want, rtol=1e-14, atol=0)


def test_damping_closed_form_with_a_dead_column():
    h = np.array([[4.0, 1.0, 0.0], [1.0, 2.0, 0.0], [0.0, 0.0, 0.0]])
    got = oracle.damped(h, 0.1)
    lam = 0.1 * (4.0 + 2.0 + 1.0) / 3.0
    want = np.array([[4.0 + lam, 1.0, 0.0], [1.0, 2.0 + lam, 0.0], [0.0, 0.0, 1.0 + lam]])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)
    assert h[2, 2] == 0.0       # input untouched


def test_inverse_factor_definition():
    rng = synth.rng_for(50001)
    h = _spd(rng, 24)
    u, hd = oracle.inverse_factor(h)
    assert np.all(np.tril(u, -1) == 0.0) and np.all(np.diag(u) > 0)
    np.testing.assert_allclose((u.T @ u) @ h, np.eye(24), atol=1e-9)
    np.testing.assert_allclose(hd, np.diag(np.linalg.inv(h)), rtol=1e-10)


def test_factor_rows_are_the_trailing_block_inverses():
    """Row j of U times U_jj is the first row of inv(H[j:, j:]): the
    compensation for column j uses the inverse Hessian of the columns not yet
    mapped (Optimal Brain Surgeon over the remaining columns)."""
    rng = synth.rng_for(50002)
    h = _spd(rng, 16)
    u, _ = oracle.inverse_factor(h)
    for j in range(16):
        trail = np.linalg.inv(h[j:, j:])
        np.testing.assert_allclose(u[j, j] * u[j, j:], trail[0], rtol=1e-9, atol=1e-12)


# ---------------------------------------------------------------------------
# Weighted Lloyd's algorithm
# ---------------------------------------------------------------------------

def test_lloyd_one_centroid_is_the_weighted_mean():
    rng = synth.rng_for(50003)
    v = (rng.standard_normal(64) * 0.02).astype(np.float32)
    hd = synth.make_hinv_diag(rng, 64)
    cent, a, it = oracle.lloyd(v, hd, 1, 10)
    w = 1.0 / hd
    assert cent[0] == np.float32(np.sum(w * v.astype(np.float64)) / np.sum(w))
    assert np.all(a == 0) and it == 1


def test_lloyd_separated_clusters():
    """Values in four tight, far-apart clumps: Lloyd from the evenly spaced
    start ends with one centroid per clump at its weighted mean."""
    rng = synth.rng_for(50004)
    centers = np.array([-0.05, -0.01, 0.02, 0.06])
    lab = rng.integers(0, 4, size=200)
    lab[:4] = np.arange(4)
    v = (centers[lab] + rng.uniform(-1e-3, 1e-3, size=200)).astype(np.float32)
    hd = synth.make_hinv_diag(rng, 200)
    cent, a, _ = oracle.lloyd(v, hd, 4, 50)
    np.testing.assert_array_equal(a, lab)
    w = 1.0 / hd
    for c in range(4):
        m = lab == c
        assert cent[c] == np.float32(np.sum(w[m] * v[m].astype(np.float64)) / np.sum(w[m]))


@pytest.mark.parametrize("k", [4, 8])
def test_lloyd_matches_scikit_learn_weighted_kmeans(k):
    from sklearn.cluster import KMeans
    rng = synth.rng_for(50005 + k)
    v = (rng.standard_normal(512) * 0.02).astype(np.float32)
    hd = synth.make_hinv_diag(rng, 512)
    cent, a, it = oracle.lloyd(v, hd, k, 300)
    assert it < 300
    init = oracle.lloyd_init(v, k).astype(np.float64)[:, None]
    km = KMeans(n_clusters=k, init=init, n_init=1, max_iter=300, tol=0.0, algorithm="lloyd")
    km.fit(v.astype(np.float64)[:, None], sample_weight=1.0 / hd)
    ref = km.cluster_centers_[:, 0]
    np.testing.assert_allclose(cent.astype(np.float64), ref, rtol=2e-7, atol=1e-9)
    np.testing.assert_array_equal(a, km.labels_)


def test_lloyd_fixed_point_and_monotone_objective():
    rng = synth.rng_for(50006)
    v = (rng.standard_normal(1376) * 0.02).astype(np.float32)
    hd = synth.make_hinv_diag(rng, 1376)
    w = 1.0 / hd
    v64 = v.astype(np.float64)

    def objective(cent, a):
        return float(np.sum(w * (v64 - cent.astype(np.float64)[a]) ** 2))

    prev = np.inf
    for iters in range(1, 8):
        cent, a, _ = oracle.lloyd(v, hd, 16, iters)
        cur = objective(cent, a)
        assert cur <= prev * (1 + 1e-12)
        prev = cur
    cent, a, it = oracle.lloyd(v, hd, 16, 1000)
    assert it < 1000
    # converged: every value sits with its nearest centroid, every centroid is its members' mean
    dist = np.abs(v64[:, None] - cent.astype(np.float64)[None, :])
    assert np.all(dist[np.arange(v.size), a] <= dist.min(axis=1) * (1 + 1e-6) + 1e-12)
    for c in range(16):
        m = a == c
        if m.any():
            assert abs(cent[c] - np.sum(w[m] * v64[m]) / np.sum(w[m])) <= 1e-7 * abs(cent[c]) + 1e-12
    assert np.all(np.diff(cent) >= 0)


def test_lloyd_constant_group():
    v = np.full(96, 0.0125, dtype=np.float32)
    cent, a, _ = oracle.lloyd(v, np.ones(96), 4, 10)
    assert np.all(cent == np.float32(0.0125)) and np.all(a == 0)


# ---------------------------------------------------------------------------
# Column-by-column mapping with error compensation
# ---------------------------------------------------------------------------

def _nearest(vals, cent_f16):
    """Brute-force nearest fp16 centroid (ties to the lower index)."""
    c = cent_f16.astype(np.float64)
    dist = np.abs(vals[:, None] - c[None, :])
    return np.argmin(dist, axis=1)


def test_round_with_a_diagonal_factor_is_plain_nearest_rounding():
    rng = synth.rng_for(50007)
    n, d, gpr, bits = 6, 64, 2, 3
    theta = (rng.standard_normal((n, d)) * 0.02).astype(np.float32)
    lut = synth.make_lut(rng, 1, n, gpr, bits)[0]
    u = np.diag(rng.uniform(0.5, 1.5, size=d))
    idx = oracle.sketch_round(theta, u, lut)
    gs = d // gpr
    for i in range(n):
        for j in range(d):
            assert idx[i, j] == _nearest(theta[i, j:j + 1].astype(np.float64), lut[i, j // gs])[0]


def test_round_matches_least_squares_compensation_route():
    """At step j the columns not yet mapped take the values that minimise the
    output error given the columns already mapped:
    x_F = theta_F + inv(H_FF) H_{F,M} (theta_M - q_M).  Solved here directly
    from H at every step, without the factor U; the mapping must agree."""
    rng = synth.rng_for(50008)
    n, d, gpr, bits = 5, 12, 1, 2
    h = _spd(rng, d)
    u, _ = oracle.inverse_factor(h)
    theta = (rng.standard_normal((n, d)) * 0.02).astype(np.float32)
    lut = synth.make_lut(rng, 1, n, gpr, bits)[0]
    idx, work = oracle.sketch_round(theta, u, lut, return_work=True)
    t64 = theta.astype(np.float64)
    for i in range(n):
        cent = lut[i, 0].astype(np.float64)
        q = np.zeros(d)
        for j in range(d):
            m, f = slice(0, j), slice(j, d)
            x_f = t64[i, f] + np.linalg.solve(h[f, f], h[f, m] @ (t64[i, m] - q[m]))
            c = _nearest(x_f[:1], lut[i, 0])[0]
            assert idx[i, j] == c, (i, j)
            assert abs(work[i, j] - x_f[0]) <= 1e-12 + 1e-9 * abs(x_f[0])
            q[j] = cent[c]


def test_round_reduces_the_output_error_against_nearest_rounding():
    rng = synth.rng_for(50009)
    n, d, gpr, bits = 32, 96, 2, 2
    c = synth.sketch_case(50010, n, d, 4 * d)
    h = oracle.damped(oracle.gram(c.x), 0.01)
    u, _ = oracle.inverse_factor(h)
    lut = synth.make_lut(rng, 1, n, gpr, bits)[0]
    idx = oracle.sketch_round(c.theta, u, lut)
    gs = d // gpr
    near = np.stack([np.concatenate([_nearest(c.theta[i, g * gs:(g + 1) * gs].astype(np.float64), lut[i, g])
                                     for g in range(gpr)]) for i in range(n)])
    lo = oracle.proxy_loss(c.theta, oracle.dequant(idx, lut), h)
    hi = oracle.proxy_loss(c.theta, oracle.dequant(near.astype(np.uint8), lut), h)
    assert lo < 0.95 * hi


# ---------------------------------------------------------------------------
# The whole stage
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 4])
def test_identity_is_sketched_exactly(bits):
    """SpaLLM section 2.4: the identity matrix is represented exactly by two
    shared values, whatever the calibration data."""
    d = 64
    x = synth.bf16_bits_to_f64(synth.make_calib(synth.rng_for(50011), 256, d))
    theta = np.eye(d, dtype=np.float32)
    idx, lut = oracle.sketch_layer(theta, x, bits, 1)
    np.testing.assert_array_equal(oracle.dequant(idx, lut), np.eye(d))


def test_groups_with_few_distinct_values_are_sketched_exactly():
    rng = synth.rng_for(50012)
    n, d, gpr, bits = 8, 128, 4, 2
    vals = rng.choice(np.array([-0.03, -0.005, 0.01, 0.04], dtype=np.float16), size=(n, d)).astype(np.float32)
    x = synth.bf16_bits_to_f64(synth.make_calib(rng, 512, d))
    idx, lut = oracle.sketch_layer(vals, x, bits, gpr)
    np.testing.assert_array_equal(oracle.dequant(idx, lut), vals.astype(np.float64))
