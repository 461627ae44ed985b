"""Plain oracle of the sketching stage (test infrastructure only).

The stage turns a dense weight ``Theta`` [n, d] and calibration activations
``X`` [s, d] into the frozen index map and the first LUTs of the sketched
layer.  Pages: "SpaLLM: Unified Compressive Adaptation of LLMs with
Sketching", section 2.2 (row-wise parameter sketching, weighted Lloyd's
algorithm for learning sketched parameters, learning the sketching matrix,
groups per row) and the "Sketch to Adapt" OpenReview discussion (concern 1:
the mapping is fixed one column at a time, each step followed by an update
of the parameters not yet mapped; its Eq. 13 is cited there but not printed).

Steps, in the pages' order:

1. ``H = X^T X`` over the calibration tokens (the pages write ``X X^T`` with
   ``X`` in ``R^{s x d}``; the ``d x d`` product is the one whose quadratic
   form in ``theta`` is the squared partial output, so that is the reading).
2. Damping (the pages are silent; taken from the error-compensated rounding
   they cite, Frantar et al. 2022): a column with ``H_jj = 0`` gets
   ``H_jj = 1``, then ``damp * mean(diag H)`` is added to the diagonal.
3. ``U``: the upper Cholesky factor of ``H^-1`` (``H^-1 = U^T U``) and the
   diagonal of ``H^-1``.
4. Per (row, group), a weighted Lloyd's algorithm over the group's values
   with weights ``1 / [H^-1]_jj`` learns ``k = 2**bits`` centroids, which
   become the group's LUT (rounded to fp16).
5. Column by column, every value is mapped to its nearest fp16 centroid and
   the error is spread over the columns not yet mapped with the Optimal Brain
   Surgeon update ``-(theta_j - q_j) / U_jj * U_{j, j+1:}`` (the reading of
   Eq. 13).

Decisions that pick an integer (the cluster of a value, the centroid a value
rounds to) are made by comparisons against float32 midpoints of the sorted
centroids, ``(w_c + w_{c+1}) * 0.5`` in float32: a value goes to the number of
midpoints strictly below it, so a value on a midpoint goes to the lower
centroid.  Everything else is float64.

Readings the pages leave open (also listed with the design notes):
* Lloyd starts from ``k`` centroids evenly spaced over the group's range,
  ``min + (max - min) * (2c + 1) / (2k)`` in float64, stored as float32;
* a centroid is the float64 weighted mean of its members rounded to float32;
  an empty cluster keeps its centroid;
* Lloyd stops when an update leaves every assignment unchanged, or after
  ``max_iter`` updates.

Pins: every function is pinned in ``tests/test_oracle_sketch_pins.py``
(brute force, closed forms, library routines, the section 2.4 identity
example, an independent least-squares route for the rounding).
"""
from __future__ import annotations

import numpy as np


# ---------------------------------------------------------------------------
# Steps 1-3: the calibration Gram matrix and its inverse factor
# ---------------------------------------------------------------------------

def gram(x: np.ndarray) -> np.ndarray:
    """H = X^T X (float64) of calibration activations x [s, d]."""
    x64 = np.asarray(x, dtype=np.float64)
    return x64.T @ x64


def damped(h: np.ndarray, damp: float) -> np.ndarray:
    """Dead columns (H_jj == 0) get H_jj = 1; then damp * mean(diag H) joins
    the diagonal."""
    h = np.array(h, dtype=np.float64, copy=True)
    dg = np.diag(h).copy()
    dg[dg == 0.0] = 1.0
    lam = damp * float(np.mean(dg))
    np.fill_diagonal(h, dg + lam)
    return h


def inverse_factor(h: np.ndarray):
    """(U, diag(H^-1)) of a symmetric positive definite H: U is the upper
    Cholesky factor of H^-1, so H^-1 = U^T U."""
    hinv = np.linalg.inv(np.asarray(h, dtype=np.float64))
    hinv = 0.5 * (hinv + hinv.T)
    low = np.linalg.cholesky(hinv)     # H^-1 = L L^T
    return np.triu(low.T), np.diag(hinv).copy()


# ---------------------------------------------------------------------------
# Step 4: weighted Lloyd's algorithm per (row, group)
# ---------------------------------------------------------------------------

def _midpoints(cent_f32: np.ndarray) -> np.ndarray:
    c = np.asarray(cent_f32, dtype=np.float32)
    return (c[..., :-1] + c[..., 1:]) * np.float32(0.5)


def lloyd_init(vals_f32: np.ndarray, k: int) -> np.ndarray:
    """k centroids evenly spaced over [min, max] of the group (float32)."""
    mn = float(np.min(vals_f32))
    mx = float(np.max(vals_f32))
    return np.array([mn + (mx - mn) * (2 * c + 1) / (2 * k) for c in range(k)], dtype=np.float32)


def lloyd_assign(vals_f32: np.ndarray, cent_f32: np.ndarray) -> np.ndarray:
    """Cluster of every value: the number of float32 midpoints below it."""
    mid = _midpoints(cent_f32)
    v = np.asarray(vals_f32, dtype=np.float32)
    return (v[:, None] > mid[None, :]).sum(axis=1)


def lloyd_update(vals_f32: np.ndarray, weights: np.ndarray, assign: np.ndarray, cent_f32: np.ndarray) -> np.ndarray:
    """Each centroid becomes the weighted mean of its members (float64 sums,
    rounded to float32); an empty cluster keeps its centroid."""
    out = np.array(cent_f32, dtype=np.float32, copy=True)
    v64 = np.asarray(vals_f32, dtype=np.float32).astype(np.float64)
    for c in range(out.shape[0]):
        m = assign == c
        if np.any(m):
            out[c] = np.float32(np.sum(weights[m] * v64[m]) / np.sum(weights[m]))
    return out


def lloyd(vals_f32: np.ndarray, hinv_diag: np.ndarray, k: int, max_iter: int):
    """Weighted Lloyd's algorithm on one group's values.  Returns (centroids
    float32 [k], the assignment they induce, number of updates run)."""
    vals = np.asarray(vals_f32, dtype=np.float32)
    weights = 1.0 / np.asarray(hinv_diag, dtype=np.float64)
    cent = lloyd_init(vals, k)
    a = lloyd_assign(vals, cent)
    it = 0
    while it < max_iter:
        cent = lloyd_update(vals, weights, a, cent)
        it += 1
        a_new = lloyd_assign(vals, cent)
        changed = not np.array_equal(a_new, a)
        a = a_new
        if not changed:
            break
    return cent, a, it


def lloyd_luts(theta_f32: np.ndarray, hinv_diag: np.ndarray, bits: int, gpr: int, max_iter: int) -> np.ndarray:
    """fp16 LUTs [n, gpr, k]: Lloyd's centroids of every (row, group)."""
    theta = np.asarray(theta_f32, dtype=np.float32)
    n, d = theta.shape
    if gpr < 1 or d % gpr:
        raise ValueError("d must be a multiple of gpr")
    gs, k = d // gpr, 1 << bits
    out = np.zeros((n, gpr, k), dtype=np.float16)
    for i in range(n):
        for g in range(gpr):
            cols = slice(g * gs, (g + 1) * gs)
            cent, _, _ = lloyd(theta[i, cols], hinv_diag[cols], k, max_iter)
            out[i, g] = cent.astype(np.float16)
    return out


# ---------------------------------------------------------------------------
# Step 5: column-by-column mapping with error compensation
# ---------------------------------------------------------------------------

def sketch_round(theta: np.ndarray, u: np.ndarray, lut_f16: np.ndarray, return_work: bool = False):
    """idx [n, d] (uint8): column j of every row goes to the nearest fp16
    centroid of its group (float32 midpoints, ties to the lower centroid) of
    its current value; the columns after j then move by
    -(theta_j - q_j) / U_jj * U_{j, j+1:}.  The LUTs must be ascending."""
    w = np.asarray(theta, dtype=np.float32).astype(np.float64).copy()
    n, d = w.shape
    gpr = lut_f16.shape[1]
    gs = d // gpr
    rows = np.arange(n)
    idx = np.zeros((n, d), dtype=np.uint8)
    for j in range(d):
        cent = np.asarray(lut_f16[:, j // gs, :], dtype=np.float32)
        mid = _midpoints(cent).astype(np.float64)
        c = (w[:, j][:, None] > mid).sum(axis=1)
        q = cent[rows, c].astype(np.float64)
        idx[:, j] = c
        e = (w[:, j] - q) / u[j, j]
        w[:, j + 1:] -= np.outer(e, u[j, j + 1:])
    return (idx, w) if return_work else idx


def sketch_layer(theta: np.ndarray, x: np.ndarray, bits: int, gpr: int, damp: float = 0.01, max_iter: int = 100):
    """The whole stage: (idx uint8 [n, d], fp16 LUT [n, gpr, k])."""
    h = damped(gram(x), damp)
    u, hinv_diag = inverse_factor(h)
    lut = lloyd_luts(theta, hinv_diag, bits, gpr, max_iter)
    return sketch_round(theta, u, lut), lut


def proxy_loss(theta: np.ndarray, theta_hat: np.ndarray, h: np.ndarray) -> float:
    """sum over rows of (theta - theta_hat) H (theta - theta_hat)^T: the squared
    change of the layer output on the calibration tokens when H = X^T X."""
    e = np.asarray(theta, dtype=np.float64) - np.asarray(theta_hat, dtype=np.float64)
    return float(np.einsum("ij,jk,ik->", e, h, e))
