"""Plain float64 oracle of the sketched linear layer (test infrastructure only).

Notation (pages: "SpaLLM: Unified Compressive Adaptation of LLMs with
Sketching", section 2.2; "Sketch to Adapt" OpenReview discussion):

* ``Theta`` is an ``n x d`` weight (``n`` rows = output features, ``d``
  columns = input features).  Each row is split into ``gpr`` contiguous groups
  of ``gs = d / gpr`` columns ("groups per row", section 2.2).
* Each group keeps its own sketched parameter vector (LUT) ``w`` of
  ``k = 2**bits`` entries and a one-hot sketching matrix ``Pi`` (``gs x k``),
  so the group is approximated as ``Pi w`` (Eq. 1).  ``Pi`` is stored as the
  index map ``idx[i, j] in [0, k)``: the position of the one in row ``j`` of
  ``Pi``.
* Several LUT sets (tasks) may share one index map (section 2.3); token ``t``
  uses the set ``task[t]``.

The layer: ``Y = X Theta_hat^T`` (section 2.3, one compressed matmul per
layer), ``dX = dY Theta_hat`` (chain rule through the frozen map) and the LUT
gradient of the corrected Eq. 6, ``dL/dw = dL/dy (M X)^T``, which bins the
dense gradient ``dY^T X`` by (row, group, centroid).

The packed index format (4-bit two per byte, 2-bit four per byte, 3-bit as 32
indices per three little-endian uint32 words) is this library's own; the pages
leave index storage open.  Each packed row is zero-padded to a multiple of 16
bytes.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

ROW_ALIGN = 16


# ---------------------------------------------------------------------------
# Packed index format
# ---------------------------------------------------------------------------

def row_stride_bytes(d: int, bits: int) -> int:
    """Bytes per packed row: ceil(d * bits / 8) rounded up to 16."""
    raw = (d * bits + 7) // 8
    return (raw + ROW_ALIGN - 1) // ROW_ALIGN * ROW_ALIGN


def packed_bytes(n: int, d: int, bits: int) -> int:
    return n * row_stride_bytes(d, bits)


def _bit_positions(d: int, bits: int):
    """For index j and bit b of it: (byte, bit-in-byte) in the packed row.

    4-bit: index j is nibble (j & 1) of byte j >> 1 (low nibble first).
    2-bit: index j sits at bits 2*(j & 3) of byte j >> 2.
    3-bit: every 32 indices form a 96-bit little-endian stream stored as three
    uint32 words; index j of the chunk starts at stream bit 3*(j mod 32).
    In all three cases bit b of index j lands at stream bit bits*j + b of the
    row read as one little-endian bit stream, because the 3-bit words are
    little-endian and the chunks are 12 bytes long.
    """
    j = np.arange(d)[:, None]
    b = np.arange(bits)[None, :]
    p = j * bits + b
    return p // 8, p % 8


def pack(idx: np.ndarray, bits: int) -> np.ndarray:
    """uint8 [n, d] indices -> uint8 [n, row_stride_bytes] packed rows."""
    idx = np.asarray(idx, dtype=np.uint8)
    n, d = idx.shape
    if bits not in (2, 3, 4):
        raise ValueError("bits must be 2, 3 or 4")
    if bits == 3 and d % 32:
        raise ValueError("3-bit rows need d % 32 == 0")
    if np.any(idx >= (1 << bits)):
        raise ValueError("index out of range")
    out = np.zeros((n, row_stride_bytes(d, bits)), dtype=np.uint8)
    byte, bit = _bit_positions(d, bits)
    for b in range(bits):
        vals = ((idx >> b) & 1).astype(np.uint8) << bit[:, b].astype(np.uint8)
        # every (byte, bit) position receives exactly one bit, so OR == unbuffered add
        np.bitwise_or.at(out, (slice(None), byte[:, b]), vals)
    return out


def unpack(packed: np.ndarray, n: int, d: int, bits: int) -> np.ndarray:
    """uint8 [n, row_stride_bytes] packed rows -> uint8 [n, d] indices."""
    packed = np.asarray(packed, dtype=np.uint8).reshape(n, -1)
    if packed.shape[1] < row_stride_bytes(d, bits):
        raise ValueError("packed rows too short")
    byte, bit = _bit_positions(d, bits)
    idx = np.zeros((n, d), dtype=np.uint8)
    for b in range(bits):
        got = (packed[:, byte[:, b]] >> bit[:, b].astype(np.uint8)) & 1
        idx |= (got << b).astype(np.uint8)
    return idx


# ---------------------------------------------------------------------------
# Eq. 1 with groups per row: Theta_hat[i, j] = w[i, g(j)][idx[i, j]]
# ---------------------------------------------------------------------------

def _check_groups(d: int, gpr: int) -> int:
    if gpr < 1 or d % gpr:
        raise ValueError("d must be a multiple of gpr")
    return d // gpr


def dequant(idx: np.ndarray, lut: np.ndarray) -> np.ndarray:
    """Dense float64 Theta_hat [n, d] from idx [n, d] and one LUT set [n, gpr, k].

    Column j belongs to contiguous group j // gs (SpaLLM, section 2.2, groups
    per row) and takes the value its index selects in that group's table
    (Eq. 1).  fp16 -> float64 is exact.
    """
    n, d = idx.shape
    gpr = lut.shape[1]
    gs = _check_groups(d, gpr)
    lut64 = np.asarray(lut, dtype=np.float64)
    rows = np.arange(n)[:, None]
    groups = (np.arange(d) // gs)[None, :]
    return lut64[rows, groups, idx.astype(np.int64)]


def sketch_matrix(idx_group: np.ndarray, k: int) -> np.ndarray:
    """The one-hot sketching matrix Pi (gs x k) of one row group (Eq. 1)."""
    gs = idx_group.shape[0]
    pi = np.zeros((gs, k), dtype=np.float64)
    for j in range(gs):
        pi[j, int(idx_group[j])] = 1.0
    return pi


def dequant_via_sketch_matrix(idx: np.ndarray, lut: np.ndarray) -> np.ndarray:
    """Eq. 1 literally: each row group is Pi @ w.  Slow; for tiny inputs only."""
    n, d = idx.shape
    gpr, k = lut.shape[1], lut.shape[2]
    gs = _check_groups(d, gpr)
    out = np.zeros((n, d), dtype=np.float64)
    for i in range(n):
        for g in range(gpr):
            pi = sketch_matrix(idx[i, g * gs:(g + 1) * gs], k)
            out[i, g * gs:(g + 1) * gs] = pi @ np.asarray(lut[i, g], dtype=np.float64)
    return out


# ---------------------------------------------------------------------------
# The three products of the layer
# ---------------------------------------------------------------------------

def _task_groups(T: int, task: Optional[np.ndarray], ntask: int):
    if task is None:
        if ntask != 1:
            raise ValueError("several LUT sets need a task id per token")
        yield 0, np.arange(T)
        return
    task = np.asarray(task)
    if task.shape != (T,) or np.any(task < 0) or np.any(task >= ntask):
        raise ValueError("task ids out of range")
    for tau in range(ntask):
        rows = np.nonzero(task == tau)[0]
        if rows.size:
            yield tau, rows


def forward(x: np.ndarray, idx: np.ndarray, luts: np.ndarray,
            task: Optional[np.ndarray] = None) -> np.ndarray:
    """Y [T, n] = X Theta_hat^T, each token with its task's LUT set.

    luts: [ntask, n, gpr, k].  SpaLLM section 2.3: a single compressed matmul
    per layer; multiple LUT sets share one index map.
    """
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    n = idx.shape[0]
    y = np.zeros((T, n), dtype=np.float64)
    for tau, rows in _task_groups(T, task, luts.shape[0]):
        y[rows] = x[rows] @ dequant(idx, luts[tau]).T
    return y


def backward_input(dy: np.ndarray, idx: np.ndarray, luts: np.ndarray,
                   task: Optional[np.ndarray] = None) -> np.ndarray:
    """dX [T, d] = dY Theta_hat (chain rule through the frozen sketch)."""
    dy = np.asarray(dy, dtype=np.float64)
    T = dy.shape[0]
    d = idx.shape[1]
    dx = np.zeros((T, d), dtype=np.float64)
    for tau, rows in _task_groups(T, task, luts.shape[0]):
        dx[rows] = dy[rows] @ dequant(idx, luts[tau])
    return dx


def backward_lut(x: np.ndarray, dy: np.ndarray, idx: np.ndarray, gpr: int, k: int,
                 task: Optional[np.ndarray] = None, ntask: int = 1) -> np.ndarray:
    """dL/dw as float64 [ntask, n, gpr, k] (or [n, gpr, k] when ntask == 1 and no task ids).

    The loss is linear in w, so the gradient needs no LUT values: form the
    dense gradient G = dY^T X (n x d) of Theta_hat and add each G[i, j] into
    the bin (row i, group j // gs, centroid idx[i, j]).  This is the corrected
    Eq. 6 of the "Sketch to Adapt" discussion, summed over the virtual
    parameters that share a trainable one.
    """
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    n, d = idx.shape
    gs = _check_groups(d, gpr)
    T = x.shape[0]
    key = ((np.arange(n)[:, None] * gpr + (np.arange(d) // gs)[None, :]) * k
           + idx.astype(np.int64)).ravel()
    out = np.zeros((ntask, n, gpr, k), dtype=np.float64)
    for tau, rows in _task_groups(T, task, ntask):
        g = dy[rows].T @ x[rows]
        out[tau] = np.bincount(key, weights=g.ravel(), minlength=n * gpr * k).reshape(n, gpr, k)
    if task is None and ntask == 1:
        return out[0]
    return out


# ---------------------------------------------------------------------------
# Second route: the corrected Eq. 6 with the mapping matrix M (tiny sizes)
# ---------------------------------------------------------------------------

def _mapping_matrix(idx_group: np.ndarray, k: int) -> np.ndarray:
    """M (k x gs): column j is one-hot at idx[j] (the transpose of Pi)."""
    gs = idx_group.shape[0]
    m = np.zeros((k, gs), dtype=np.float64)
    m[idx_group.astype(np.int64), np.arange(gs)] = 1.0
    return m


def eq6_forward(x: np.ndarray, idx: np.ndarray, lut: np.ndarray) -> np.ndarray:
    """y_i = sum_g w_{i,g} (M_{i,g} X_g) with X as features x tokens (one LUT set)."""
    x = np.asarray(x, dtype=np.float64)
    n, d = idx.shape
    gpr, k = lut.shape[1], lut.shape[2]
    gs = _check_groups(d, gpr)
    xt = x.T  # d x T, columns are tokens
    y = np.zeros((n, x.shape[0]), dtype=np.float64)
    for i in range(n):
        for g in range(gpr):
            s = _mapping_matrix(idx[i, g * gs:(g + 1) * gs], k) @ xt[g * gs:(g + 1) * gs]
            y[i] += np.asarray(lut[i, g], dtype=np.float64) @ s
    return y.T


def eq6_backward_lut(x: np.ndarray, dy: np.ndarray, idx: np.ndarray, gpr: int, k: int) -> np.ndarray:
    """dL/dw_{i,g} = dL/dy_i (M_{i,g} X_g)^T, the corrected Eq. 6, per row and group."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    n, d = idx.shape
    gs = _check_groups(d, gpr)
    xt = x.T
    out = np.zeros((n, gpr, k), dtype=np.float64)
    for i in range(n):
        for g in range(gpr):
            s = _mapping_matrix(idx[i, g * gs:(g + 1) * gs], k) @ xt[g * gs:(g + 1) * gs]
            out[i, g] = dy[:, i] @ s.T
    return out


def bin_counts(idx: np.ndarray, gpr: int, k: int) -> np.ndarray:
    """cnt[i, g, c]: how many columns of group g in row i select centroid c."""
    n, d = idx.shape
    gs = _check_groups(d, gpr)
    key = ((np.arange(n)[:, None] * gpr + (np.arange(d) // gs)[None, :]) * k
           + idx.astype(np.int64)).ravel()
    return np.bincount(key, minlength=n * gpr * k).reshape(n, gpr, k)


# ---------------------------------------------------------------------------
# LUT update (the pages train the LUT values but name no optimizer)
# ---------------------------------------------------------------------------

def averaged_gradient(grad: np.ndarray, counts: Optional[np.ndarray]) -> np.ndarray:
    """The "averaging" variant of SpaLLM section 2.1: the gradient of a
    trainable LUT entry divided by the number of virtual parameters that share
    it (its static bin size; empty bins keep their zero gradient).  counts is
    [n, gpr, k] and applies to every LUT set."""
    grad = np.asarray(grad, dtype=np.float64)
    if counts is None:
        return grad
    return grad / np.maximum(np.asarray(counts, dtype=np.float64), 1.0)


def adamw_step(master: np.ndarray, m: np.ndarray, v: np.ndarray, grad: np.ndarray, step: int,
               lr: float, beta1: float, beta2: float, eps: float, weight_decay: float,
               counts: Optional[np.ndarray] = None):
    """One AdamW step (Adam with decoupled weight decay), written out:
    p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2;
    p <- p - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps).
    Returns the new (master, m, v) in float64."""
    g = averaged_gradient(grad, counts)
    p = np.asarray(master, dtype=np.float64) * (1.0 - lr * weight_decay)
    m = beta1 * np.asarray(m, dtype=np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, dtype=np.float64) + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** step)
    vhat = v / (1.0 - beta2 ** step)
    p = p - lr * mhat / (np.sqrt(vhat) + eps)
    return p, m, v


def sgd_step(master: np.ndarray, grad: np.ndarray, lr: float, counts: Optional[np.ndarray] = None) -> np.ndarray:
    """Plain gradient descent on the LUT values: p <- p - lr g."""
    return np.asarray(master, dtype=np.float64) - lr * averaged_gradient(grad, counts)


# ---------------------------------------------------------------------------
# Counting identities used by the pages
# ---------------------------------------------------------------------------

def trainable_params(shapes, layers: int, gpr: int, k: int) -> int:
    """n * gpr * k trainable LUT entries per matrix, summed over a model."""
    return layers * sum(n * gpr * k for n, _ in shapes)


def lora_params(shapes, layers: int, r: int) -> int:
    """A rank-r adapter on an n x d matrix trains r * (n + d) values."""
    return layers * sum(r * (n + d) for n, d in shapes)


def compression_factor(c: int, g: int, k: int) -> float:
    """A row of c values sketched into g groups of k entries ("Sketch to Adapt", reply W2)."""
    return c / (g * k)


def sketched_model_bytes(shapes, layers: int, bits: int, gpr: int, dense_params: int = 0) -> int:
    """Bytes of a sketched model: per matrix the packed indices (n * d * bits /
    8) and one fp16 LUT set (n * gpr * 2**bits * 2), summed over the layers,
    plus `dense_params` fp16 parameters kept unsketched (embeddings, head)."""
    k = 1 << bits
    per_layer = sum(n * d * bits // 8 + n * gpr * k * 2 for n, d in shapes)
    return layers * per_layer + 2 * dense_params
